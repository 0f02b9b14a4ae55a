// gemv.cuh -- decode-path weight-only linear, M <= 16 tokens:
//   y[m, n] = sum_g s[n, g] * sum_{k in g} x[m, k] * (q[n, k] - z[n, g])
// ("A Survey of Low-bit Large Language Models", section 6.2: weight-only
// quantization dequantizes and runs a 16-bit matmul and gains by moving
// fewer bytes; "大模型量化实战" section 3.3: dequantize and multiply inside one
// kernel so no intermediate goes back to memory).
//
// Design (HBM-bound; every weight byte is read exactly once):
//  * A CTA owns one 128-row block (8 row tiles of 16; fewer in a last partial
//    block) and a K-slice of KC columns.  In the interleaved layout the codes
//    of a whole block for a run of column blocks are contiguous, and so are
//    its scales and its zeros for a run of groups.  One producer warp stages
//    the block's scales and zeros for the slice and the slice of x once (x
//    rows padded by 16 bytes so ldmatrix is conflict-free; padding tokens read
//    a 16-byte zero chunk), and streams the codes through a shared-memory ring
//    of 16 KB stages, one bulk asynchronous copy per stage (cp.async.bulk
//    completing on an mbarrier with a transaction count).  Bulk copies reach
//    full HBM bandwidth only when they are large (measured on B200: ~1.5-3
//    TB/s with 2 KB copies, 6.5-7 TB/s with 16-32 KB copies), hence this
//    layout.
//  * Consumer warp j reads its lane's 16-byte slot of row tile j in each
//    column block (conflict-free), builds exact (q - z) operands in registers
//    (one LOP3 against the 0x4300 bf16 magic exponent plus one bf16x2
//    subtract per register) and issues m16n8k16 mma.sync with x^T as the B
//    operand.  Each group accumulates in fp32 from zero; the group's fp32
//    scale is applied per row in an FMA into the running sum.
//  * CTAs splitting K form a thread-block cluster; each pushes its partial
//    sums into the owning rank's shared memory (distributed shared memory),
//    one cluster barrier publishes them, and each rank sums its slice in
//    fixed rank order: deterministic, no global scratch.  Without a split the
//    consumers write y directly.
//  * Programmatic dependent launch (opt-in): the kernel lets the next kernel
//    launch early and, when the caller guarantees that the weights are not
//    written by the preceding kernel, starts streaming weights before waiting
//    for it; x is always read after the wait.
//  * Every mbarrier wait is bounded; on expiry the kernel records
//    BQ_FLAG_TIMEOUT, stops issuing copies, waits (bounded) for the copies it
//    already issued, and still joins the cluster barriers.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"

namespace bq {
namespace cg = cooperative_groups;

template <int XT> struct MmaT;
template <> struct MmaT<1> {  // bf16
  static constexpr uint32_t kMagic = 0x43004300u;  // bf16x2 (128, 128)
  static constexpr uint32_t kOne2 = 0x3F803F80u;   // bf16x2 (1, 1)
  static BQ_DEV uint32_t zpair(uint32_t z) {     // bf16x2 (128 + z, 128 + z), exact
    uint32_t h = 0x4300u | z;
    return h | (h << 16);
  }
  static BQ_DEV uint32_t sub2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
  static BQ_DEV void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  static BQ_DEV uint16_t out(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }
};
template <> struct MmaT<0> {  // fp16
  static constexpr uint32_t kMagic = 0x64006400u;  // fp16x2 (1024, 1024)
  static constexpr uint32_t kOne2 = 0x3C003C00u;   // fp16x2 (1, 1)
  static BQ_DEV uint32_t zpair(uint32_t z) {
    uint32_t h = 0x6400u | z;
    return h | (h << 16);
  }
  static BQ_DEV uint32_t sub2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
  static BQ_DEV void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  static BQ_DEV uint16_t out(float v) { return __half_as_ushort(__float2half_rn(v)); }
};

BQ_DEV uint32_t and_or(uint32_t a, uint32_t mask, uint32_t magic) {  // (a & mask) | magic
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(magic));
  return r;
}

BQ_DEV void ldmatrix_x4(uint32_t (&r)[4], uint32_t smem_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr));
}

BQ_DEV uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

constexpr int kGemvMaxStages = 8;
constexpr int kGemvMaxConsumers = 8;

// Per-width stage geometry: a stage is SC columns of a full 128-row block,
// 16 KB of packed codes for either width (SC = 256 at 4 bits, 512 at 2 bits).
template <int BITS, int G> struct StageG {
  static constexpr int T = (BITS == 4) ? 64 : 128;   // tile width
  static constexpr int SC = (BITS == 4) ? 256 : 512;  // columns per stage
  static constexpr int TPS = SC / T;                  // column blocks per stage (4)
  static constexpr int GPS = SC / G;                  // groups per stage
  static constexpr int STEPS_PER_G = G / 16;
  static constexpr int W_BYTES = TPS * 8 * 512;       // packed codes of the block (16 KB)
  static_assert(SC % G == 0 && STEPS_PER_G % 2 == 0, "bad stage geometry");
};

// Shared-memory layout (bytes), all staged per CTA:
//   x     [M][KC + 8] 16-bit rows (only the real tokens), then a 16-byte
//         zero chunk that ldmatrix reads for padding tokens
//   meta  scales [KC/G][rows] fp32 (or binary16) then zeros [KC/G][rows] u8
//         of the block
//   ring  `stages` x 16 KB of packed codes
//   part  split-K receive buffer: S_k slices of ceil(TOK * rows / S_k) fp32
//   bars  full[stages], empty[stages], x/meta barrier, abort flag
struct GemvSmem {
  int zero_off, s_off, z_off, ring_off, part_off, bar_off, total;
};

inline GemvSmem gemv_smem_layout(int M, int TOK, int64_t KC, int groups, int stages) {
  GemvSmem L;
  L.zero_off = (int)(M * (KC + 8) * 2);
  L.s_off = (L.zero_off + 16 + 127) / 128 * 128;
  L.z_off = L.s_off + groups * 128 * 4;
  L.ring_off = (L.z_off + groups * 128 + 127) / 128 * 128;
  L.part_off = L.ring_off + stages * 16384;
  L.bar_off = L.part_off + (TOK * 128 + 8) * 4;
  L.total = L.bar_off + (2 * stages + 1) * 8 + 16;
  return L;
}

struct GemvArgs {
  const uint16_t *x;
  const uint8_t *packed;
  const void *scales;  // fp32, or binary16 when the kernel's S16 is set
  const uint8_t *zeros;
  const uint8_t *bit_map;
  uint16_t *y;
  int64_t K, N, KC;
  int M;
  int stages;
  int prefetch_before_wait;  // weights may be streamed before the programmatic wait
  GemvSmem L;
};

// Producer warp.  Streams the CTA's K-slice of its 128-row block through the
// ring, one 16 KB bulk copy per stage (contiguous in the interleaved layout),
// after lane 0 armed the stage's full barrier; stages the block's scales and
// zeros for the slice (two copies, contiguous in the interleaved metadata
// layout) and its x rows (one copy per token) once, on the x/meta barrier.
// `pk`, `sc`, `ze` point at the block's first byte (codes, scales of
// SB bytes each, zeros); `R` = row tiles.
template <int BITS, int G, int SB>
BQ_DEV void gemv_produce(const GemvArgs &a, const uint8_t *pk, const uint8_t *sc, const uint8_t *ze, int R,
                         int64_t kc0, uint32_t smem, uint32_t bars, volatile int *abort, int lane) {
  using SG = StageG<BITS, G>;
  const int n = (int)(a.KC / SG::SC);
  const int S = a.stages;
  const int rows = 16 * R;
  const uint32_t wb = (uint32_t)(SG::TPS * R * 512);
  const uint32_t xm_full = bars + 8u * (2 * S);
  const int groups = (int)(a.KC / G);
  auto issue = [&](int i, uint32_t full) {
    const uint32_t st = smem + (uint32_t)(a.L.ring_off + (i % S) * 16384);
    const int64_t ks = kc0 + (int64_t)i * SG::SC;
    bulk_g2s(st, pk + (ks / SG::T) * R * 512, wb, full);
  };
  auto stage_meta = [&]() {  // arms the x/meta barrier for metadata and x
    if (lane == 0) {
      mbar_arrive_expect_tx(xm_full, (uint32_t)(groups * rows * (SB + 1) + a.M * a.KC * 2));
      bulk_g2s(smem + a.L.s_off, sc + (kc0 / G) * rows * SB, (uint32_t)(groups * rows * SB), xm_full);
      bulk_g2s(smem + a.L.z_off, ze + (kc0 / G) * rows, (uint32_t)(groups * rows), xm_full);
    }
    __syncwarp();
  };
  auto stage_x = [&]() {
    for (int m = lane; m < a.M; m += 32)
      bulk_g2s(smem + (uint32_t)(m * (a.KC + 8) * 2), a.x + m * a.K + kc0, (uint32_t)(a.KC * 2), xm_full);
  };
  const int pre = n < S ? n : S;
  if (!a.prefetch_before_wait) pdl_wait();
  stage_meta();
  for (int i = 0; i < pre; ++i) {
    const uint32_t full = bars + 8u * i;
    if (lane == 0) {
      mbar_arrive_expect_tx(full, wb);
      issue(i, full);
    }
  }
  if (a.prefetch_before_wait) pdl_wait();
  stage_x();
  int issued = pre;
  int slot = pre % S, phase = (pre / S) & 1;
  for (int i = pre; i < n; ++i) {
    const uint32_t full = bars + 8u * slot, empty = bars + 8u * (S + slot);
    const bool ok = __all_sync(0xffffffffu, (*abort == 0) && mbar_wait(empty, phase ^ 1));
    if (!ok) {
      if (lane == 0) {
        *abort = 1;
        bq_flag(BQ_FLAG_TIMEOUT);
      }
      break;
    }
    if (lane == 0) {
      mbar_arrive_expect_tx(full, wb);
      issue(i, full);
    }
    issued = i + 1;
    if (++slot == S) {
      slot = 0;
      phase ^= 1;
    }
  }
  __syncwarp();
  if (*abort && lane == 0) {
    // let the copies already issued land before the CTA can exit
    mbar_wait(xm_full, 0);
    for (int i = (issued > S ? issued - S : 0); i < issued; ++i) mbar_wait(bars + 8u * (i % S), (i / S) & 1);
  }
}

// Consumer warp j: 16-row tile j of the CTA's block over the whole K-slice.
template <int XT, int BITS, int G, int NB, int SB>
BQ_DEV void gemv_consume(const GemvArgs &a, int j, int R, uint32_t smem, uint32_t bars, volatile int *abort,
                         int lane, float (&acc)[NB][4]) {
  using MT = MmaT<XT>;
  using SG = StageG<BITS, G>;
  constexpr uint32_t MASK = (BITS == 4) ? 0x000F000Fu : 0x00030003u;
  const int n = (int)(a.KC / SG::SC);
  const int S = a.stages;
  const int rows = 16 * R;
  const int r = lane >> 2;
  const int xstride = (int)(a.KC + 8) * 2;
  // ldmatrix row address of this lane for token block nb: token (lane & 7) +
  // 8 nb, column offset 8 (lane / 8) inside a pair of k16 steps; tokens >= M
  // read the zero chunk (and do not advance with k)
  uint32_t x_lane[NB];
  uint32_t x_step[NB];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int tok = (lane & 7) + 8 * nb;
    const bool real = tok < a.M;
    x_lane[nb] = real ? smem + (uint32_t)(tok * xstride + (lane >> 3) * 16) : smem + a.L.zero_off;
    x_step[nb] = real ? 1u : 0u;
  }
  // x and metadata staged; every wait is voted on, so the whole warp leaves
  // together (mma.sync below needs every lane)
  if (!__all_sync(0xffffffffu, (*abort == 0) && mbar_wait(bars + 8u * (2 * S), 0))) {
    if (lane == 0) {
      *abort = 1;
      bq_flag(BQ_FLAG_TIMEOUT);
    }
    return;
  }
  const uint32_t stile = smem + a.L.s_off + (j * 16 + r) * SB;
  const uint32_t ztile = smem + a.L.z_off + j * 16 + r;
  int slot = 0, phase = 0;
  for (int i = 0; i < n; ++i) {
    const uint32_t full = bars + 8u * slot, empty = bars + 8u * (S + slot);
    if (!__all_sync(0xffffffffu, (*abort == 0) && mbar_wait(full, phase))) {
      if (lane == 0) {
        *abort = 1;
        bq_flag(BQ_FLAG_TIMEOUT);
      }
      break;
    }
    const uint32_t wt = smem + (uint32_t)(a.L.ring_off + slot * 16384) + j * 512 + lane * 16;
    uint4 tiles[SG::TPS];
#pragma unroll
    for (int t = 0; t < SG::TPS; ++t) tiles[t] = lds_v4(wt + t * R * 512);
    // the stage's codes are in registers now: hand the slot back to the
    // producer before computing, so the ring keeps prefetching
    __syncwarp();
    if (lane == 0) mbar_arrive(empty);
    if (++slot == S) {
      slot = 0;
      phase ^= 1;
    }
#pragma unroll
    for (int gi = 0; gi < SG::GPS; ++gi) {
      const int g = i * SG::GPS + gi;  // group within the CTA's slice
      float s0, s1;
      uint32_t z0, z1;
      if (SB == 4) {
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(s0) : "r"(stile + g * rows * 4));
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(s1) : "r"(stile + (g * rows + 8) * 4));
      } else {  // binary16 scales, exact in fp32
        unsigned short h0, h1;
        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h0) : "r"(stile + g * rows * 2));
        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h1) : "r"(stile + (g * rows + 8) * 2));
        s0 = __half2float(__ushort_as_half(h0));
        s1 = __half2float(__ushort_as_half(h1));
      }
      asm volatile("ld.shared.u8 %0, [%1];" : "=r"(z0) : "r"(ztile + g * rows));
      asm volatile("ld.shared.u8 %0, [%1];" : "=r"(z1) : "r"(ztile + g * rows + 8));
      // bf16 with at most 8 tokens: the operands are the exact integers
      // 128 + q (magic exponent 0x4300), so y_group = s * (sum x (128 + q) -
      // (128 + z) sum x), the x sums of each token coming from one extra mma
      // against all-ones.  Otherwise (fp16: base 1024, larger cancellation;
      // 16 tokens: the extra mma would double the tensor work) exact (q - z)
      // operands from one 16-bit-pair subtract per register.
      constexpr bool kOnes = (XT == 1 && NB == 1);
      const uint32_t zz0 = MT::zpair(z0), zz1 = MT::zpair(z1);
      const float zf0 = kOnes ? (float)(128 + (int)z0) : 0.0f, zf1 = kOnes ? (float)(128 + (int)z1) : 0.0f;
      float c[2][NB][4], cx[NB][4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int q = 0; q < 4; ++q) c[h][nb][q] = 0.0f;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int q = 0; q < 4; ++q) cx[nb][q] = 0.0f;
#pragma unroll
      for (int sp = 0; sp < SG::STEPS_PER_G; sp += 2) {
        const int step0 = gi * SG::STEPS_PER_G + sp;               // k16 step within the stage
        const uint32_t kbytes = (uint32_t)((i * SG::SC + step0 * 16) * 2);  // column offset in x rows
        uint32_t bfr[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) ldmatrix_x4(bfr[nb], x_lane[nb] + x_step[nb] * kbytes);
#pragma unroll
        for (int ss = 0; ss < 2; ++ss) {
          const int step = step0 + ss;
          const int t = step / (SG::T / 16);
          const int run = step % (SG::T / 16);
          const uint32_t words[4] = {tiles[t].x, tiles[t].y, tiles[t].z, tiles[t].w};
          const uint32_t w = words[BITS == 4 ? run : run / 2];
          const int base = (BITS == 4) ? 0 : 4 * (run & 1);
          uint32_t av[4];
#pragma unroll
          for (int si = 0; si < 4; ++si) {
            av[si] = and_or(w >> (BITS * (base + si)), MASK, MT::kMagic);
            if (!kOnes) av[si] = MT::sub2(av[si], (si & 1) ? zz1 : zz0);
          }
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            MT::mma(c[ss][nb], av, bfr[nb][2 * ss], bfr[nb][2 * ss + 1]);
            if (kOnes) {
              const uint32_t ones[4] = {MT::kOne2, MT::kOne2, MT::kOne2, MT::kOne2};
              MT::mma(cx[nb], ones, bfr[nb][2 * ss], bfr[nb][2 * ss + 1]);
            }
          }
        }
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        acc[nb][0] = __fmaf_rn(s0, __fmaf_rn(-zf0, cx[nb][0], c[0][nb][0] + c[1][nb][0]), acc[nb][0]);
        acc[nb][1] = __fmaf_rn(s0, __fmaf_rn(-zf0, cx[nb][1], c[0][nb][1] + c[1][nb][1]), acc[nb][1]);
        acc[nb][2] = __fmaf_rn(s1, __fmaf_rn(-zf1, cx[nb][2], c[0][nb][2] + c[1][nb][2]), acc[nb][2]);
        acc[nb][3] = __fmaf_rn(s1, __fmaf_rn(-zf1, cx[nb][3], c[0][nb][3] + c[1][nb][3]), acc[nb][3]);
      }
    }
  }
}

// Kernel.  grid = (ceil(N / 128), S_k); cluster = (1, S_k, 1); block = 9
// warps (8 consumers, one per 16-row tile of the block; warp 8 produces).
// bit_map == nullptr: uniform BITS / G.  Otherwise one width per 128-row
// block and the CTA runs (4, 128) or (2, 64).
template <int XT, int BITS, int G, int NB, bool MIXED, bool S16 = false>
__global__ void __launch_bounds__(32 * (kGemvMaxConsumers + 1), 2)
gemv_kernel(const GemvArgs a) {
  constexpr int SB = S16 ? 2 : 4;  // bytes per scale
  using MT = MmaT<XT>;
  constexpr int TOK = 8 * NB;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NC = kGemvMaxConsumers;
  cg::cluster_group cluster = cg::this_cluster();
  const int SK = (int)cluster.dim_blocks().y;
  const int rank = (int)cluster.block_rank();
  const int64_t kc0 = (int64_t)blockIdx.y * a.KC;
  const int64_t blk = blockIdx.x;
  const int64_t row0 = blk * 128;
  const int R = (int)((a.N - row0) / 16 < 8 ? (a.N - row0) / 16 : 8);  // row tiles in the block
  const int ROWS = 16 * R;
  const uint32_t smem = smem_u32(smem_raw);
  const uint32_t bars = smem + a.L.bar_off;
  volatile int *abort = reinterpret_cast<volatile int *>(smem_raw + a.L.bar_off + (2 * a.stages + 1) * 8);
  float *part = reinterpret_cast<float *>(smem_raw + a.L.part_off);

  pdl_launch_dependents();
  // every CTA of the cluster must have started before any writes into
  // another's shared memory (the matching wait precedes those writes)
  if (SK > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  // the zero chunk read by padding tokens
  if (threadIdx.x == 0) *reinterpret_cast<uint4 *>(smem_raw + a.L.zero_off) = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(bars + 8u * s, 1);
      mbar_init(bars + 8u * (a.stages + s), R);
    }
    mbar_init(bars + 8u * (2 * a.stages), 1);
    *abort = 0;
    mbar_fence_init();
  }
  __syncthreads();

  // width of this block and where its codes / metadata start
  int bits = BITS;
  const uint8_t *pk;
  const uint8_t *sc;
  const uint8_t *ze;
  if (!MIXED) {
    pk = a.packed + blk * 128 * a.K * BITS / 8;
    sc = reinterpret_cast<const uint8_t *>(a.scales) + blk * 128 * (a.K / G) * SB;
    ze = a.zeros + blk * 128 * (a.K / G);
  } else {
    int64_t sb = 0, sg = 0;
    for (int64_t jb = lane; jb < blk; jb += 32) {
      const int b = a.bit_map[jb];
      sb += b;
      sg += (b == 4) ? 1 : 2;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      sb += __shfl_xor_sync(0xffffffffu, sb, off);
      sg += __shfl_xor_sync(0xffffffffu, sg, off);
    }
    pk = a.packed + sb * 16 * a.K;
    sc = reinterpret_cast<const uint8_t *>(a.scales) + sg * a.K * SB;
    ze = a.zeros + sg * a.K;
    bits = a.bit_map[blk];
    if (bits != 4 && bits != 2) {
      if (threadIdx.x == 0) bq_flag(BQ_FLAG_BADMAP);
      bits = 0;
    }
  }

  float acc[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[nb][q] = 0.0f;

  if (warp == NC) {
    if (bits != 0) {
      if (!MIXED) gemv_produce<BITS, G, SB>(a, pk, sc, ze, R, kc0, smem, bars, abort, lane);
      else if (bits == 4) gemv_produce<4, 128, SB>(a, pk, sc, ze, R, kc0, smem, bars, abort, lane);
      else gemv_produce<2, 64, SB>(a, pk, sc, ze, R, kc0, smem, bars, abort, lane);
    }
  } else if (bits != 0 && warp < R) {
    if (!MIXED) gemv_consume<XT, BITS, G, NB, SB>(a, warp, R, smem, bars, abort, lane, acc);
    else if (bits == 4) gemv_consume<XT, 4, 128, NB, SB>(a, warp, R, smem, bars, abort, lane, acc);
    else gemv_consume<XT, 2, 64, NB, SB>(a, warp, R, smem, bars, abort, lane, acc);
  }

  if (SK == 1) {
    // no split: every consumer writes its own rows and tokens
    pdl_wait();  // y may be read by the previous kernel: write only after it completed
    if (warp < R) {
      const int r = lane >> 2, c = lane & 3;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = warp * 16 + r + 8 * (q >> 1);
          const int tok = nb * 8 + 2 * c + (q & 1);
          if (tok < a.M) a.y[(int64_t)tok * a.N + row0 + row] = MT::out(acc[nb][q]);
        }
    }
    return;
  }
  // split-K: element e = tok * ROWS + row belongs to rank e / per; every CTA
  // stores its partial of e straight into the owner's receive buffer
  // recv[source rank][e - owner * per] (distributed shared memory), one
  // cluster barrier publishes all of them, and each owner sums its slice in
  // rank order.  No remote access follows the barrier.
  const int E = TOK * ROWS;
  const int per = (E + SK - 1) / SK;
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (warp < R) {
    const int r = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = warp * 16 + r + 8 * (q >> 1);
        const int tok = nb * 8 + 2 * c + (q & 1);
        const int e = tok * ROWS + row;
        const int owner = e / per;
        cluster.map_shared_rank(part, owner)[rank * per + (e - owner * per)] = acc[nb][q];
      }
  }
  cluster.sync();
  pdl_wait();  // y may be read by the previous kernel: write only after it completed
  const int e0 = rank * per, e1 = min(E, e0 + per);
  for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int tok = e / ROWS, row = e % ROWS;
    if (tok >= a.M) continue;
    float sum = 0.0f;
    for (int q = 0; q < SK; ++q) sum += part[q * per + (e - e0)];
    a.y[(int64_t)tok * a.N + row0 + row] = MT::out(sum);
  }
}

}  // namespace bq
