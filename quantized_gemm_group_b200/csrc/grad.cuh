// grad.cuh -- input gradient of the weight-only linear, M <= 16 tokens:
//   dx[m, k] = sum_n dy[m, n] * s[n, g(k)] * (q[n, k] - z[n, g(k)])
// i.e. dx = dy . dequant(W) for y = x . dequant(W)^T.  Training in the
// quantized weight space needs it (GreenBitAI article: the Bitorch Engine
// paragraph on gradients of low-bit tensors, and the Q-SFT paragraph).
//
// Design (every weight byte is read once per 16-token pass; measured on B200
// the kernel is bound by instruction issue and latency, ~5.5 instructions per
// code, not by HBM):
//  * The contraction now runs over the output channels n, the rows of W.  A
//    CTA owns a slice of 128 input columns and streams its cluster rank's
//    share of the 128-row blocks, one block per ring stage.  In the
//    interleaved layout the codes of a block over 128 columns are one
//    contiguous range (8 KB at 4 bits, 4 KB at 2 bits), and so are its
//    scales and zeros over the slice's groups; the stage also holds the
//    block's 128 entries of each dy row.  One producer warp issues the bulk
//    copies; all of a stage's copies complete on one mbarrier.
//  * Up to 8 tokens, consumer warp j takes row tile j (16 rows) of each
//    block and all 128 columns; up to 16 tokens, two row tiles and 64
//    columns (so its partial sums fit in registers).  Each run of 16 columns
//    is one m16n8k8 tf32 mma.sync per half tile of 8 rows and per 8 tokens,
//    with A = the weights transposed (16 columns x 8 rows) and B = dy'
//    (8 rows x 8 tokens).
//  * The interleaved layout puts a row on lane / 4 and a column pair on
//    lane % 4 -- the register order of the forward product, whose
//    contraction runs over columns.  Here the contraction index must sit on
//    lane % 4, so lane (g, t) reads the two 16-byte slots 4t + g % 4 and
//    4t + g % 4 + 16 of the tile from shared memory: they hold rows t, t + 8
//    and t + 4, t + 12 at the columns 2 (g % 4) + 8 (g / 4) and the next one
//    of every run (even column in the lower half-word, odd in the upper).
//  * Operands: a code q at bit position p of a word becomes the fp32 value
//    2^23 + q 2^p with one AND/OR against the exponent of 2^23, and one
//    subtract of 2^23 + z 2^p leaves 2^p (q - z) exactly -- an exact tf32
//    value.  The second 8-row half of a tile sits BITS bits above the first,
//    a factor 2^BITS folded into the scale that multiplies its dy; the high
//    column pairs sit 2 BITS bits above the low ones, a factor taken off the
//    lane's sums at the end (both exact power-of-two scalings).
//    dy[m, n] s[n, g] is rounded once to tf32, the only rounding before the
//    fp32 accumulation.
//  * Warps' partial sums meet in shared memory (the idle ring) and are added
//    in warp order; CTAs of a cluster split the rows and meet in distributed
//    shared memory, added in rank order: deterministic, no global scratch.
//  * Every mbarrier wait is bounded; on expiry the kernel records
//    BQ_FLAG_TIMEOUT, stops issuing copies, waits (bounded) for the copies it
//    issued, and still joins the barriers.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "gemv.cuh"

namespace bq {
namespace cg = cooperative_groups;

constexpr int kGradSlice = 128;        // input columns per CTA
constexpr int kGradWarps = 8;          // consumer warps: the row tiles of a 128-row block
constexpr int kGradMaxStages = 8;
constexpr int kGradRedStride = 132;    // fp32 row stride of the cross-warp sums (conflict-free)
constexpr int kGradDyStride = 272;     // bytes per staged dy row (conflict-free token reads)

// Shared memory: ring of `stages` stages, each
//   codes [8192 B] | scales [gmax][rows] fp32 | zeros [gmax][rows] u8 | dy [M][272 B]
// (the ring is reused for the cross-warp sums once drained), then the cluster
// receive buffer, then the barriers and the abort flag.
struct GradSmem {
  int sb, s_off, z_off, dy_off, part_off, bar_off, total;
};

inline GradSmem grad_smem_layout(int M, int TOK, int gmax, int stages, int d) {
  GradSmem L;
  L.s_off = 8192;
  L.z_off = L.s_off + gmax * 128 * 4;
  L.dy_off = L.z_off + gmax * 128;
  L.sb = (L.dy_off + M * kGradDyStride + 127) / 128 * 128;
  int ring = stages * L.sb;
  const int red = kGradWarps * TOK * kGradRedStride * 4;
  if (ring < red) ring = red;
  L.part_off = (ring + 127) / 128 * 128;
  const int per = (M * kGradSlice + d - 1) / d;
  L.bar_off = L.part_off + (d * per * 4 + 127) / 128 * 128;
  L.total = L.bar_off + 2 * stages * 8 + 16;
  return L;
}

struct GradArgs {
  const uint16_t *dy;
  const uint8_t *packed;
  const float *scales;
  const uint8_t *zeros;
  const uint8_t *bit_map;  // width map (one entry per 128-row block), or null
  uint16_t *dx;
  int64_t N, K;
  int M;
  int stages;
  int prefetch_before_wait;  // weights may be streamed before the programmatic wait
  GradSmem L;
};

BQ_DEV int grad_block_rows(int64_t N, int64_t blk) {
  const int64_t r = N - blk * 128;
  return (int)(r < 128 ? r : 128);
}

BQ_DEV void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

BQ_DEV uint32_t to_tf32(float v) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(v));
  return r;
}

BQ_DEV uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

template <int XT> BQ_DEV float elem16_to_f32(uint32_t h);
template <> BQ_DEV float elem16_to_f32<1>(uint32_t h) { return __uint_as_float(h << 16); }
template <> BQ_DEV float elem16_to_f32<0>(uint32_t h) { return __half2float(__ushort_as_half((unsigned short)h)); }

// Producer warp: blocks [b0, b0 + nblk) of the CTA's column slice.  Under a
// width map (MIXED) each block has its own width (4 bits / group 128 or 2
// bits / group 64); its codes and metadata start after the blocks before it:
// a block of b bits holds 16 K b code bytes and 128 K / group metadata
// entries (running sums, from a warp reduction over the map up to b0).
template <int BITS, int G, bool MIXED>
BQ_DEV void grad_produce(const GradArgs &a, int64_t b0, int nblk, int64_t col0, uint32_t smem, uint32_t bars,
                         volatile int *abort, int lane) {
  const int S = a.stages;
  int64_t sb = 0, sg = 0;  // bits and group units (1 per 4-bit, 2 per 2-bit block) before block b0 + i
  if (MIXED) {
    for (int64_t jb = lane; jb < b0; jb += 32) {
      const int b = a.bit_map[jb];
      sb += b;
      sg += (b == 4) ? 1 : 2;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      sb += __shfl_xor_sync(0xffffffffu, sb, off);
      sg += __shfl_xor_sync(0xffffffffu, sg, off);
    }
  }
  auto stage_of = [&](int i) { return smem + (uint32_t)((i % S) * a.L.sb); };
  auto issue_weights = [&](int i) {  // lane 0, blocks in order: arm the stage, copy codes and metadata
    const int64_t blk = b0 + i;
    const int rows = grad_block_rows(a.N, blk);
    const int R = rows / 16;
    const uint32_t st = stage_of(i), full = bars + 8u * (i % S);
    const int bits = MIXED ? a.bit_map[blk] : BITS;
    if (MIXED && bits != 4 && bits != 2) {  // not a width: flag it, the stage carries dy only
      bq_flag(BQ_FLAG_BADMAP);
      mbar_arrive_expect_tx(full, (uint32_t)(a.M * rows * 2));
      sb += bits;
      sg += 2;
      return;
    }
    const int g = MIXED ? (bits == 4 ? 128 : 64) : G;
    const int T = (bits == 4) ? 64 : 128;
    const int TPS = kGradSlice / T;                                // column tiles in the slice
    const int GPS = (g <= kGradSlice) ? kGradSlice / g : 1;        // groups in the slice
    const uint32_t cb = (uint32_t)(TPS * R * 512);
    mbar_arrive_expect_tx(full, cb + (uint32_t)(GPS * rows * 5 + a.M * rows * 2));
    const int64_t code0 = MIXED ? 16 * a.K * sb : blk * 128 * a.K * BITS / 8;
    const int64_t meta0 = MIXED ? a.K * sg : 128 * (a.K / G) * blk;
    bulk_g2s(st, a.packed + code0 + (col0 / T) * R * 512, cb, full);
    const int64_t mi = meta0 + (col0 / g) * rows;
    bulk_g2s(st + a.L.s_off, a.scales + mi, (uint32_t)(GPS * rows * 4), full);
    bulk_g2s(st + a.L.z_off, a.zeros + mi, (uint32_t)(GPS * rows), full);
    sb += bits;
    sg += (bits == 4) ? 1 : 2;
  };
  auto issue_dy = [&](int i) {  // one dy row per lane
    const int64_t blk = b0 + i;
    const int rows = grad_block_rows(a.N, blk);
    const uint32_t st = stage_of(i), full = bars + 8u * (i % S);
    for (int m = lane; m < a.M; m += 32)
      bulk_g2s(st + a.L.dy_off + m * kGradDyStride, a.dy + m * a.N + blk * 128, (uint32_t)(rows * 2), full);
  };
  const int pre = nblk < S ? nblk : S;
  if (!a.prefetch_before_wait) pdl_wait();
  if (lane == 0)
    for (int i = 0; i < pre; ++i) issue_weights(i);
  __syncwarp();
  if (a.prefetch_before_wait) pdl_wait();
  for (int i = 0; i < pre; ++i) issue_dy(i);
  int issued = pre;
  for (int i = pre; i < nblk; ++i) {
    const uint32_t empty = bars + 8u * (S + i % S);
    const bool ok = __all_sync(0xffffffffu, (*abort == 0) && mbar_wait(empty, ((i / S) & 1) ^ 1));
    if (!ok) {
      if (lane == 0) {
        *abort = 1;
        bq_flag(BQ_FLAG_TIMEOUT);
      }
      break;
    }
    if (lane == 0) issue_weights(i);
    __syncwarp();
    issue_dy(i);
    issued = i + 1;
  }
  __syncwarp();
  if (*abort && lane == 0) {
    // let the copies already issued land before the ring is reused
    for (int i = (issued > S ? issued - S : 0); i < issued; ++i) mbar_wait(bars + 8u * (i % S), (i / S) & 1);
  }
}

// Consumer warp w.  CW = 1 (up to 8 tokens): row tile w of every block and
// all 8 runs of the slice.  CW = 2 (up to 16 tokens): row tiles 2 (w / 2) and
// 2 (w / 2) + 1 and runs 4 (w % 2) .. 4 (w % 2) + 3, so that a warp's partial
// sums (16 tokens x 64 columns) stay in registers.  acc[run][token block]
// [fragment] accumulates dx^T for the warp's runs: fragment q is column
// 16 run + 2 (g % 4) + 8 (g / 4) + q / 2 and token 8 nb + 2t + (q % 2), times
// 2^(2 ACC_BITS (g / 4)) (undone when the sums leave the registers).  A block
// of BITS < ACC_BITS (a width map's 2-bit blocks) has its codes at 2 BITS (g / 4)
// and makes up the difference on its A operand, whose rows g and g + 8 are the
// lane's columns (an exact power of two on an exact small integer).
// One staged block `st` of `rows` rows.
template <int XT, int BITS, int G, int NB, int CW, int ACC_BITS>
BQ_DEV void grad_consume_block(const GradArgs &a, int w, uint32_t st, int rows, int lane,
                               float (&acc)[8 / CW][NB][4]) {
  constexpr int T = (BITS == 4) ? 64 : 128;
  constexpr int RPT = T / 16;                                     // runs per column tile
  constexpr int RPG = ((G <= kGradSlice) ? G : kGradSlice) / 16;  // runs per group in the slice
  constexpr int RW = 8 / CW;                                      // runs per warp
  constexpr int GW = (RPG >= RW) ? 1 : RW / RPG;                  // groups per warp
  constexpr int RPGW = (RPG >= RW) ? RW : RPG;                    // runs per group per warp
  constexpr uint32_t QM = (1u << BITS) - 1;
  constexpr uint32_t kMagic = 0x4B000000u;                        // fp32 2^23
  const int g = lane >> 2, t = lane & 3;
  const int r_lo = (w % CW) * RW;                                 // the warp's first run
  const int rt0 = (w / CW) * CW;                                  // the warp's first row tile
  // lane group g takes the column pair (2 (g % 4) + 8 (g / 4), + 1) of every
  // run: both from the slots of column pair g % 4, whose slot index i =
  // h + 2 (g / 4) puts them at bit BITS h + hpos of the lower (even column)
  // and upper (odd column) half-word
  const uint32_t slot1 = 16u * (uint32_t)(4 * t + (g & 3));       // rows t, t + 8
  const uint32_t slot2 = slot1 + 16u * 16u;                       // rows t + 4, t + 12
  const uint32_t hpos = 2u * BITS * (uint32_t)(g >> 2);
  // 2^(2 (ACC_BITS - BITS) (g / 4)): the accumulators' convention for this lane's columns
  const float acc_fix = (ACC_BITS != BITS && (g >> 2)) ? (float)(1 << (2 * (ACC_BITS - BITS))) : 1.0f;
  const int R = rows / 16;
#pragma unroll
  for (int rti = 0; rti < CW; ++rti) {
    const int rt = rt0 + rti;
    if (rt >= R) break;
#pragma unroll
    for (int j = 0; j < GW; ++j) {
      const int gi = r_lo / RPG + j;  // group within the slice
      // the lane's rows in this tile: 16 rt + t + 4 aa + 8 h
      uint32_t bp[NB][2][2];
      float cz[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int aa = 0; aa < 2; ++aa) {
          const int nl = 16 * rt + t + 4 * aa + 8 * h;
          float s;
          uint32_t z;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(s) : "r"(st + a.L.s_off + (gi * rows + nl) * 4));
          asm volatile("ld.shared.u8 %0, [%1];" : "=r"(z) : "r"(st + a.L.z_off + gi * rows + nl));
          // the second half tile's codes sit BITS bits higher: scale its dy' down by 2^BITS
          const float sh = h ? s * (1.0f / (float)(1 << BITS)) : s;
          cz[h][aa] = __uint_as_float(kMagic | (z << (BITS * h + hpos)));  // 2^23 + z 2^(BITS h + hpos)
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const int m = g + 8 * nb;
            float dyv = 0.0f;
            if (m < a.M) {
              uint32_t hbits;
              asm volatile("ld.shared.u16 %0, [%1];" : "=r"(hbits) : "r"(st + a.L.dy_off + m * kGradDyStride + nl * 2));
              dyv = elem16_to_f32<XT>(hbits);
            }
            bp[nb][h][aa] = to_tf32(__fmul_rn(dyv, sh));
          }
        }
#pragma unroll
      for (int rr = 0; rr < RPGW; ++rr) {
        const int rl = j * RPGW + rr;  // run within the warp's range
        const int rs = r_lo + rl;      // run within the slice
        const int ct = rs / RPT;       // column tile
        const int wj = (BITS == 4) ? (rs % RPT) : (rs % RPT) / 2;
        const uint32_t tb = st + (uint32_t)((ct * R + rt) * 512 + wj * 4);
        uint32_t w1 = lds_u32(tb + slot1), w2 = lds_u32(tb + slot2);
        // 2 bits: the word's second run sits 8 bits higher (r_lo is even, so
        // the parity of rs is that of rl)
        if (BITS == 2 && (rl & 1)) {
          w1 >>= 8;
          w2 >>= 8;
        }
        const uint32_t w1o = w1 >> 16, w2o = w2 >> 16;  // odd columns
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t mask = QM << (BITS * h + hpos);
          uint32_t av[4];
          av[0] = __float_as_uint(__fsub_rn(__uint_as_float(and_or(w1, mask, kMagic)), cz[h][0]));
          av[1] = __float_as_uint(__fsub_rn(__uint_as_float(and_or(w1o, mask, kMagic)), cz[h][0]));
          av[2] = __float_as_uint(__fsub_rn(__uint_as_float(and_or(w2, mask, kMagic)), cz[h][1]));
          av[3] = __float_as_uint(__fsub_rn(__uint_as_float(and_or(w2o, mask, kMagic)), cz[h][1]));
          if (ACC_BITS != BITS) {
#pragma unroll
            for (int q = 0; q < 4; ++q) av[q] = __float_as_uint(__uint_as_float(av[q]) * acc_fix);
          }
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) mma_tf32(acc[rl][nb], av, bp[nb][h][0], bp[nb][h][1]);
        }
      }
    }
  }
}

// The consumer loop: blocks [b0, b0 + nblk); under a width map (MIXED) each
// block runs its own width's body, with the 4-bit accumulator convention.
template <int XT, int BITS, int G, int NB, int CW, bool MIXED>
BQ_DEV void grad_consume(const GradArgs &a, int w, int64_t b0, int nblk, uint32_t smem, uint32_t bars,
                         volatile int *abort, int lane, float (&acc)[8 / CW][NB][4]) {
  const int S = a.stages;
  for (int i = 0; i < nblk; ++i) {
    const uint32_t st = smem + (uint32_t)((i % S) * a.L.sb);
    const uint32_t full = bars + 8u * (i % S), empty = bars + 8u * (S + i % S);
    // the whole warp leaves together (mma.sync below needs every lane)
    if (!__all_sync(0xffffffffu, (*abort == 0) && mbar_wait(full, (i / S) & 1))) {
      if (lane == 0) {
        *abort = 1;
        bq_flag(BQ_FLAG_TIMEOUT);
      }
      break;
    }
    const int rows = grad_block_rows(a.N, b0 + i);
    if (!MIXED) {
      grad_consume_block<XT, BITS, G, NB, CW, BITS>(a, w, st, rows, lane, acc);
    } else {
      const int bits = a.bit_map[b0 + i];
      if (bits == 4) grad_consume_block<XT, 4, 128, NB, CW, 4>(a, w, st, rows, lane, acc);
      else if (bits == 2) grad_consume_block<XT, 2, 64, NB, CW, 4>(a, w, st, rows, lane, acc);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty);
  }
}

// Kernel.  grid = (K / 128, d); cluster = (1, d, 1); block = 9 warps (8
// consumers, warp 8 produces).  Cluster rank r streams the blocks
// [r nb / d, (r + 1) nb / d) of the nb = ceil(N / 128) row blocks.
template <int XT, int BITS, int G, int NB, bool MIXED = false>
__global__ void __launch_bounds__(32 * (kGradWarps + 1), 2) grad_input_kernel(const GradArgs a) {
  using MT = MmaT<XT>;
  constexpr int TOK = 8 * NB;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  cg::cluster_group cluster = cg::this_cluster();
  const int d = (int)cluster.dim_blocks().y;
  const int rank = (int)cluster.block_rank();
  const int64_t col0 = (int64_t)blockIdx.x * kGradSlice;
  const int64_t nbk = (a.N + 127) / 128;
  const int64_t b0 = nbk * rank / d, b1 = nbk * (rank + 1) / d;
  const int nblk = (int)(b1 - b0);
  const uint32_t smem = smem_u32(smem_raw);
  const uint32_t bars = smem + a.L.bar_off;
  volatile int *abort = reinterpret_cast<volatile int *>(smem_raw + a.L.bar_off + 2 * a.stages * 8);

  pdl_launch_dependents();
  // every CTA of the cluster must have started before any writes into
  // another's shared memory (the matching wait precedes those writes)
  if (d > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(bars + 8u * s, 1);
      mbar_init(bars + 8u * (a.stages + s), kGradWarps);
    }
    *abort = 0;
    mbar_fence_init();
  }
  __syncthreads();

  constexpr int CW = NB;  // column split of the consumer warps (see grad_consume)
  constexpr int RW = 8 / CW;
  float acc[RW][NB][4];
#pragma unroll
  for (int r = 0; r < RW; ++r)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[r][nb][q] = 0.0f;

  if (warp == kGradWarps) grad_produce<BITS, G, MIXED>(a, b0, nblk, col0, smem, bars, abort, lane);
  else grad_consume<XT, BITS, G, NB, CW, MIXED>(a, warp, b0, nblk, smem, bars, abort, lane, acc);
  __syncthreads();  // ring drained: reuse it for the cross-warp sums

  // red[warp row group][token][column]: warps w and w + 1 (CW = 2) cover the
  // two column halves of the same row tiles and share a row group
  constexpr int RG = kGradWarps / CW;
  float *red = reinterpret_cast<float *>(smem_raw);
  if (warp < kGradWarps) {
    const int g = lane >> 2, t = lane & 3;
    const int rgw = warp / CW, c0 = 16 * (warp % CW) * RW + 2 * (g & 3) + 8 * (g >> 2);
    const float unscale = (g >> 2) ? 1.0f / (float)(1 << (2 * BITS)) : 1.0f;  // exact
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int m = 8 * nb + 2 * t + (q & 1);
          const int col = c0 + 16 * r + (q >> 1);
          red[(rgw * TOK + m) * kGradRedStride + col] = acc[r][nb][q] * unscale;
        }
  }
  __syncthreads();
  const int E = a.M * kGradSlice;
  auto warp_sum = [&](int e) {
    const int m = e / kGradSlice, col = e % kGradSlice;
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < RG; ++w) v += red[(w * TOK + m) * kGradRedStride + col];
    return v;
  };
  if (d == 1) {
    pdl_wait();  // dx may be read by the previous kernel: write only after it completed
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      a.dx[(int64_t)(e / kGradSlice) * a.K + col0 + e % kGradSlice] = MT::out(warp_sum(e));
    return;
  }
  // element e belongs to rank e / per; each CTA stores its sum of e into the
  // owner's receive buffer recv[source rank][e - owner * per]; one cluster
  // barrier publishes them and each owner adds its slice in rank order
  const int per = (E + d - 1) / d;
  float *part = reinterpret_cast<float *>(smem_raw + a.L.part_off);
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int owner = e / per;
    cluster.map_shared_rank(part, owner)[rank * per + (e - owner * per)] = warp_sum(e);
  }
  cluster.sync();
  pdl_wait();
  const int e0 = rank * per, e1 = min(E, e0 + per);
  for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    float v = 0.0f;
    for (int q = 0; q < d; ++q) v += part[q * per + (e - e0)];
    a.dx[(int64_t)(e / kGradSlice) * a.K + col0 + e % kGradSlice] = MT::out(v);
  }
}

}  // namespace bq
