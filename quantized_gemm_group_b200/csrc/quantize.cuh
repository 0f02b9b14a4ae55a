// quantize.cuh -- group-wise asymmetric MinMax quantizer with bit packing.
//
// Method: GreenBitAI article ("只需单卡 RTX 3090 ..."), classic Group-wise MinMax,
// INT4 / group 128 and INT2 / group 64; arithmetic per
// "大模型量化实战：从原理到4-bit部署的完整指南" section 2.2 and "低比特量化",
// section "Zero Point".  See group_params() / code_pair() in common.cuh.
//
// HBM-bound: 2 bytes read per weight, b/8 + 5/g bytes written.  Two kernels:
//   * canonical layout: a thread owns 8 consecutive weights (one 16-byte
//     load), a group spans g/8 adjacent lanes and is reduced with shuffles;
//     the thread writes its 8 codes as one 32-bit (4-bit) or 16-bit (2-bit)
//     word; scales / zeros row-major [rows, cols/g].
//   * interleaved layout: a warp owns a unit of 16 rows x U columns
//     (U = max(tile width, g)); lane L takes exactly the weights whose codes
//     form its own 16-byte slot of each 512-byte tile, so no permutation pass
//     is needed; groups are reduced over the 4 lanes sharing a row; tiles and
//     scales / zeros go to their 128-row-block-major places (il_tile_offset,
//     il_meta_index).  A producer warp stages the weights by TMA
//     (quantize_tma_kernel); mixed maps load them per lane (load_unit).
// The per-element arithmetic runs on packed f32x2 operations (two elements
// per instruction); the clamp to 2^b - 1 is only evaluated in groups whose
// largest element needs it.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace bq {

// ---------------------------------------------------------------------------
// canonical layout
// ---------------------------------------------------------------------------

// Quantize 8 consecutive weights held as 4 packed 16-bit pairs; the group
// spans LANES = G/8 adjacent lanes.  Returns the 8 codes packed LSB-first.
template <int WT, int BITS, int G, int SCHEME = 0>
BQ_DEV uint32_t quant8_canonical(uint4 v, bool active, float *s_out, uint8_t *z_out, bool *bad) {
  using E = Elem<WT>;
  constexpr int LANES = G / 8;
  constexpr int QMAX = (1 << BITS) - 1;
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t mn2 = E::min2(E::min2(w[0], w[1]), E::min2(w[2], w[3]));
  uint32_t mx2 = E::max2(E::max2(w[0], w[1]), E::max2(w[2], w[3]));
  float mn = fmin_nan(E::lo(mn2), E::hi(mn2));
  float mx = fmax_nan(E::lo(mx2), E::hi(mx2));
  if (!active) { mn = 0.0f; mx = 0.0f; }
#pragma unroll
  for (int off = 1; off < LANES; off <<= 1) {
    mn = fmin_nan(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  GroupParams p = group_params<QMAX, SCHEME>(mn, mx);
  *s_out = p.s;
  *z_out = (uint8_t)p.z;
  *bad = p.bad;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint2 q = code_pair<QMAX, WT == 0, true>(E::pair(w[i]), p);
    packed |= (q.x | (q.y << BITS)) << (BITS * 2 * i);
  }
  return packed;
}

// W viewed flat: element e of the matrix = W[e], groups of G start at
// multiples of G, codes packed flat.
template <int WT, int BITS, int G, int UNROLL, int SCHEME = 0>
__global__ void __launch_bounds__(256)
quantize_canonical_kernel(const uint16_t *__restrict__ W, int64_t elems,
                          uint8_t *__restrict__ packed, void *__restrict__ scales,
                          uint8_t *__restrict__ zeros) {
  constexpr int LANES = G / 8;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t chunks = (elems + 255) / 256;  // 256 weights per warp step
  bool bad_any = false;
  for (int64_t c0 = warp * UNROLL; c0 < chunks; c0 += nwarps * UNROLL) {
    uint4 v[UNROLL];
    bool act[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      int64_t e = (c0 + u) * 256 + lane * 8;
      act[u] = (c0 + u < chunks) && (e < elems);
      v[u] = act[u] ? ld_stream_v4(W + e) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      int64_t e = (c0 + u) * 256 + lane * 8;
      float s;
      uint8_t z;
      bool bad;
      uint32_t pk = quant8_canonical<WT, BITS, G, SCHEME>(v[u], act[u], &s, &z, &bad);
      if (!act[u]) continue;
      bad_any |= bad;
      if (BITS == 4) {
        reinterpret_cast<uint32_t *>(packed)[e / 8] = pk;
      } else {
        reinterpret_cast<uint16_t *>(packed)[e / 8] = (uint16_t)pk;
      }
      if ((lane % LANES) == 0) {
        store_scale<SCHEME>(scales, e / G, s);
        zeros[e / G] = z;
      }
    }
  }
  if (bad_any) bq_flag(BQ_FLAG_NONFINITE);
}

// ---------------------------------------------------------------------------
// interleaved (tiled) layout
// ---------------------------------------------------------------------------

template <int BITS> struct TileGeom {
  static constexpr int T = (BITS == 4) ? 64 : 128;  // tile width in columns
};

// Bit offset, inside the lane's word, of the even column of slot
// (h: 0 row r / 1 row r+8, hp: 0 columns 2c,2c+1 / 1 columns 2c+8,2c+9) of
// 16-column run `run` of the tile; the odd column sits 16 bits higher.
template <int BITS>
BQ_DEV constexpr int tile_bit(int run, int h, int hp) {
  return BITS == 4 ? 4 * (h + 2 * hp) : 2 * (4 * (run & 1) + h + 2 * hp);
}
template <int BITS>
BQ_DEV constexpr int tile_word(int run) { return BITS == 4 ? run : run / 2; }

template <int BITS, int G> struct UnitGeom {
  static constexpr int T = TileGeom<BITS>::T;
  static constexpr int U = (G > T) ? G : T;     // unit width
  static constexpr int RUNS = U / 16;
  static constexpr int RUNS_PER_G = G / 16;
  static constexpr int NG = U / G;              // groups per row in the unit
  static constexpr int TILES = U / T;
  static constexpr int RUNS_PER_TILE = T / 16;
};

// Unit weights of one lane: [h][run][hp] 16-bit pairs.
template <int BITS, int G> struct UnitRegs {
  uint32_t x[2][UnitGeom<BITS, G>::RUNS][2];
};

template <int BITS, int G>
BQ_DEV void load_unit(UnitRegs<BITS, G> &u, const uint16_t *__restrict__ W, int64_t K, int64_t row0,
                      int64_t col0, int lane) {
  const int r = lane >> 2, c = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint16_t *rowp = W + (row0 + r + 8 * h) * K + col0 + 2 * c;
#pragma unroll
    for (int j = 0; j < UnitGeom<BITS, G>::RUNS; ++j) {
      u.x[h][j][0] = ld_nc_u32(rowp + 16 * j);
      u.x[h][j][1] = ld_nc_u32(rowp + 16 * j + 8);
    }
  }
}

// Codes of one (row half, group) of the unit added into the lane's tile
// words (every code owns its own bit field, so adding is ORing).  A group
// that needs no clamp adds each rounded quotient's raw bit pattern times
// 2^(bit position) -- one integer multiply-add per code, off the ALU pipe --
// and then, once per word, (z - kRoundMagicBits) times the sum of its
// positions' 2^(bit position): modulo 2^32 the magic cancels and every field
// receives round(x / s) + z.  A clamp group packs clamped codes directly.
template <int WT, int BITS, int G, bool CLAMP>
BQ_DEV void codes_of_group(const UnitRegs<BITS, G> &u, int h, int gi, const GroupParams &p,
                           uint32_t (&word)[UnitGeom<BITS, G>::TILES][4]) {
  using UG = UnitGeom<BITS, G>;
  using E = Elem<WT>;
  constexpr int QMAX = (1 << BITS) - 1;
#pragma unroll
  for (int jj = 0; jj < UG::RUNS_PER_G; ++jj) {
    const int j = gi * UG::RUNS_PER_G + jj;
    const int t = j / UG::RUNS_PER_TILE, jt = j % UG::RUNS_PER_TILE;
    uint32_t &w = word[t][tile_word<BITS>(jt)];
    if (CLAMP) {
#pragma unroll
      for (int hp = 0; hp < 2; ++hp) {
        const uint2 q = code_pair<QMAX, WT == 0, true>(E::pair(u.x[h][j][hp]), p);
        w += __byte_perm(q.x, q.y, 0x5410) << tile_bit<BITS>(jt, h, hp);
      }
    } else {
      uint32_t posmask = 0;
#pragma unroll
      for (int hp = 0; hp < 2; ++hp) {
        const int bp = tile_bit<BITS>(jt, h, hp);
        const float2 m = rounded_quotients<WT == 0>(E::pair(u.x[h][j][hp]), p);
        w += __float_as_uint(m.x) * (1u << bp);
        w += __float_as_uint(m.y) * (1u << (bp + 16));
        posmask += (1u << bp) + (1u << (bp + 16));
      }
      w += (uint32_t)p.zc * posmask;
    }
  }
}

// Quantize one loaded unit: rows row0..row0+15, columns col0..col0+U-1 of an
// N x K matrix; `packed`, `scales`, `zeros` are that matrix's own.
// The four lanes of a quad share one row (r = lane / 4) and hold C = 2 x NG
// (row half, group) combinations of it.  Their min / max are reduced across
// the quad by a reduce-scatter (exchange with lane ^ 2, then lane ^ 1, each
// step keeping half of the list while it is longer than one), so each lane
// ends up with max(1, C / 4) whole combinations, computes their parameters,
// stores their scale and zero, and the codes of every combination take the
// parameters from the lane that computed them by shuffle.
template <int WT, int BITS, int G, int SCHEME = 0>
BQ_DEV bool quantize_unit(const UnitRegs<BITS, G> &u, int64_t N, int64_t K, int64_t row0, int64_t col0,
                          uint8_t *__restrict__ packed, void *__restrict__ scales,
                          uint8_t *__restrict__ zeros, int lane) {
  using UG = UnitGeom<BITS, G>;
  using E = Elem<WT>;
  constexpr int QMAX = (1 << BITS) - 1;
  constexpr int NG = UG::NG;
  constexpr int C = 2 * NG;                  // combinations (h, gi), k = h * NG + gi
  constexpr int HALF = C / 2;
  constexpr int LF = (C >= 4) ? C / 4 : 1;   // combinations finished per lane
  const int r = lane >> 2, c = lane & 3;

  // this lane's partial min / max of every combination
  float vmn[C], vmx[C];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      uint32_t mn2 = u.x[h][gi * UG::RUNS_PER_G][0], mx2 = mn2;
#pragma unroll
      for (int j = gi * UG::RUNS_PER_G; j < (gi + 1) * UG::RUNS_PER_G; ++j) {
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) {
          mn2 = E::min2(mn2, u.x[h][j][hp]);
          mx2 = E::max2(mx2, u.x[h][j][hp]);
        }
      }
      vmn[h * NG + gi] = fmin_nan(E::lo(mn2), E::hi(mn2));
      vmx[h * NG + gi] = fmax_nan(E::lo(mx2), E::hi(mx2));
    }
  }
  // step 1: with lane ^ 2, keep the upper half of the list if lane bit 1 is set
  const bool up2 = (c & 2) != 0;
  float amn[HALF], amx[HALF];
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float kmn = up2 ? vmn[HALF + i] : vmn[i], smn = up2 ? vmn[i] : vmn[HALF + i];
    const float kmx = up2 ? vmx[HALF + i] : vmx[i], smx = up2 ? vmx[i] : vmx[HALF + i];
    amn[i] = fmin_nan(kmn, __shfl_xor_sync(0xffffffffu, smn, 2));
    amx[i] = fmax_nan(kmx, __shfl_xor_sync(0xffffffffu, smx, 2));
  }
  // step 2: with lane ^ 1, halve again (or, with one left, reduce it)
  float fmn[LF], fmx[LF];
  const bool up1 = (c & 1) != 0;
#pragma unroll
  for (int i = 0; i < LF; ++i) {
    if (HALF >= 2) {
      const float kmn = up1 ? amn[LF + i] : amn[i], smn = up1 ? amn[i] : amn[LF + i];
      const float kmx = up1 ? amx[LF + i] : amx[i], smx = up1 ? amx[i] : amx[LF + i];
      fmn[i] = fmin_nan(kmn, __shfl_xor_sync(0xffffffffu, smn, 1));
      fmx[i] = fmax_nan(kmx, __shfl_xor_sync(0xffffffffu, smx, 1));
    } else {
      fmn[i] = fmin_nan(amn[0], __shfl_xor_sync(0xffffffffu, amn[0], 1));
      fmx[i] = fmax_nan(amx[0], __shfl_xor_sync(0xffffffffu, amx[0], 1));
    }
  }
  // combinations held: base + i, base from the two lane bits
  const int base = (up2 ? HALF : 0) + ((HALF >= 2 && up1) ? LF : 0);
  bool bad_any = false;
  GroupParams own[LF];
  const int64_t GK = K / G;
#pragma unroll
  for (int i = 0; i < LF; ++i) {
    own[i] = group_params<QMAX, SCHEME>(fmn[i], fmx[i]);
    bad_any |= own[i].bad;
    if (HALF >= 2 || !up1) {  // with C = 2, lanes c and c ^ 1 hold the same combination
      const int k = base + i, h = k / NG, gi = k % NG;
      const int64_t idx = il_meta_index(row0 + r + 8 * h, col0 / G + gi, N, GK);
      store_scale<SCHEME>(scales, idx, own[i].s);
      zeros[idx] = (uint8_t)own[i].z;
    }
  }

  uint32_t word[UG::TILES][4];
#pragma unroll
  for (int t = 0; t < UG::TILES; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) word[t][i] = 0u;
#pragma unroll
  for (int k = 0; k < C; ++k) {
    // the lane of this quad that finished combination k, and its slot there
    const int src_c = (k >= HALF ? 2 : 0) + ((HALF >= 2 && (k % HALF) >= LF) ? 1 : 0);
    const int slot = (HALF >= 2) ? (k % HALF) % LF : 0;
    const int src = (lane & ~3) | src_c;
    const GroupParams &o = own[slot];
    GroupParams p;
    p.r = __shfl_sync(0xffffffffu, o.r, src);
    p.sd = __shfl_sync(0xffffffffu, o.sd, src);
    p.zc = __shfl_sync(0xffffffffu, o.zc, src);
    const int fl = __shfl_sync(0xffffffffu, (o.fast ? 1 : 0) | (o.clamp ? 2 : 0), src);
    p.fast = (fl & 1) != 0;
    p.clamp = (fl & 2) != 0;
    const int h = k / NG, gi = k % NG;
    if (p.clamp) codes_of_group<WT, BITS, G, true>(u, h, gi, p, word);
    else codes_of_group<WT, BITS, G, false>(u, h, gi, p, word);
  }
#pragma unroll
  for (int t = 0; t < UG::TILES; ++t) {
    const int64_t off = il_tile_offset(row0 / 16, col0 / UG::T + t, N, K, BITS);
    st_v4(packed + off + lane * 16, make_uint4(word[t][0], word[t][1], word[t][2], word[t][3]));
  }
  return bad_any;
}

// ---------------------------------------------------------------------------
// interleaved layout, weights staged by TMA
// ---------------------------------------------------------------------------
// Per unit the arithmetic and stores of quantize_unit, with the weights
// brought into shared memory by TMA rather than loaded into registers:
// a super-unit is 64 rows x U columns (four 16-row units), loaded as U / 64
// boxes of 64 columns x 64 rows with the 128-byte swizzle (16-byte chunk c
// of row r stored at chunk c ^ (r % 8)), which makes each lane's 4-byte
// reads conflict-free.  A producer warp keeps a ring of super-units in
// flight; consumer warps 0-3 take the even ring slots and warps 4-7 the odd
// ones, warp w quantizing row tile w % 4.  CTAs stride over the super-units.
constexpr int kQtConsumers = 8;
constexpr int kQtThreads = 32 * (kQtConsumers + 1);
// CTAs per SM: three where the unit fits 72 registers without spilling
// (groups 32 to 128; measured on B200: 2-10% faster than two), else two.
template <int G> constexpr int qt_ctas_per_sm() { return (G >= 32 && G <= 128) ? 3 : 2; }

template <int BITS, int G>
BQ_DEV void load_unit_smem(UnitRegs<BITS, G> &u, uint32_t su, int t, int lane) {
  const int r = lane >> 2, c = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = 16 * t + r + 8 * h;  // row % 8 == r
#pragma unroll
    for (int j = 0; j < UnitGeom<BITS, G>::RUNS; ++j) {
#pragma unroll
      for (int hp = 0; hp < 2; ++hp) {
        const int col = 16 * j + 8 * hp + 2 * c;
        const uint32_t addr = su + (uint32_t)((col / 64) * 8192 + row * 128 + ((((col % 64) / 8) ^ r) << 4) +
                                              (col % 8) * 2);
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(u.x[h][j][hp]) : "r"(addr));
      }
    }
  }
}

template <int WT, int BITS, int G, int SCHEME = 0>
__global__ void __launch_bounds__(kQtThreads, qt_ctas_per_sm<G>())
quantize_tma_kernel(const __grid_constant__ CUtensorMap wmap, int64_t N, int64_t K, int stages,
                    uint8_t *__restrict__ packed, void *__restrict__ scales, uint8_t *__restrict__ zeros) {
  using UG = UnitGeom<BITS, G>;
  constexpr uint32_t SU_BYTES = (uint32_t)(UG::U / 64) * 8192u;
  extern __shared__ __align__(1024) unsigned char qt_raw[];
  const uint32_t raw = smem_u32(qt_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // the launch adds 1024 bytes of slack
  const uint32_t bars = sbase + (uint32_t)stages * SU_BYTES;
  volatile int *abort = reinterpret_cast<volatile int *>(qt_raw + (sbase - raw) + stages * SU_BYTES + 16 * stages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ku = K / UG::U;
  const int64_t nsu = ((N + 63) / 64) * ku;
  // super-units of this CTA: blockIdx.x, + gridDim.x, ...
  const int n = (int)((nsu - blockIdx.x + gridDim.x - 1) / gridDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(bars + 8u * s, 1);
      mbar_init(bars + 8u * (stages + s), kQtConsumers / 2);
    }
    *abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == kQtConsumers) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int slot = i % stages;
        if (i >= stages && !mbar_wait(bars + 8u * (stages + slot), ((i / stages) & 1) ^ 1)) {
          *abort = 1;
          bq_flag(BQ_FLAG_TIMEOUT);
          break;
        }
        const int64_t su = blockIdx.x + (int64_t)i * gridDim.x;
        const int64_t rb = su / ku;
        const int col0 = (int)((su - rb * ku) * UG::U), row0 = (int)(rb * 64);
        const uint32_t full = bars + 8u * slot;
        mbar_arrive_expect_tx(full, SU_BYTES);
#pragma unroll
        for (int b = 0; b < UG::U / 64; ++b)
          tma_load_2d(sbase + (uint32_t)slot * SU_BYTES + b * 8192u, &wmap, col0 + 64 * b, row0, full);
        issued = i + 1;
      }
      if (*abort) {  // the loads already issued land before the CTA exits
        for (int i = (issued > stages ? issued - stages : 0); i < issued; ++i)
          mbar_wait(bars + 8u * (i % stages), (i / stages) & 1, 1u << 20);
      }
    }
    return;
  }
  const int par = warp / 4, t = warp % 4;
  bool bad = false;
  for (int i = par; i < n; i += 2) {
    const int slot = i % stages;
    // the whole warp leaves together (the group reductions shuffle across lanes)
    if (!__all_sync(0xffffffffu, (*abort == 0) && mbar_wait(bars + 8u * slot, (i / stages) & 1))) {
      if (lane == 0) {
        *abort = 1;
        bq_flag(BQ_FLAG_TIMEOUT);
      }
      break;
    }
    const int64_t su = blockIdx.x + (int64_t)i * gridDim.x;
    const int64_t rb = su / ku;
    const int64_t col0 = (su - rb * ku) * UG::U, row0 = rb * 64 + 16 * t;
    if (row0 < N) {
      UnitRegs<BITS, G> u;
      load_unit_smem<BITS, G>(u, sbase + (uint32_t)slot * SU_BYTES, t, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8u * (stages + slot));
      bad |= quantize_unit<WT, BITS, G, SCHEME>(u, N, K, row0, col0, packed, scales, zeros, lane);
    } else {
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8u * (stages + slot));
    }
  }
  if (bad) bq_flag(BQ_FLAG_NONFINITE);
}

// ---------------------------------------------------------------------------
// mixed precision: per 128-row block width from a device bit map
// ---------------------------------------------------------------------------

// Offsets of 128-row block `blk` of a mixed matrix with K columns: packed
// byte offset and group offset, summed over the blocks before it.
BQ_DEV void mixed_block_offsets(const uint8_t *__restrict__ bit_map, int64_t blk, int64_t K,
                                int lane, int64_t *code_off, int64_t *group_off) {
  int64_t sb = 0, sg = 0;
  for (int64_t j = lane; j < blk; j += 32) {
    int b = bit_map[j];
    sb += b;
    sg += (b == 4) ? 1 : 2;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sb += __shfl_xor_sync(0xffffffffu, sb, off);
    sg += __shfl_xor_sync(0xffffffffu, sg, off);
  }
  *code_off = sb * 16 * K;  // 128 rows * K cols * b / 8 bytes
  *group_off = sg * K;      // 128 rows * K / g groups, g = 128 (b=4) or 64 (b=2)
}

template <int WT>
__global__ void __launch_bounds__(256)
quantize_mixed_tiled_kernel(const uint16_t *__restrict__ W, int64_t N, int64_t K,
                            const uint8_t *__restrict__ bit_map, uint8_t *__restrict__ packed,
                            float *__restrict__ scales, uint8_t *__restrict__ zeros) {
  // Both production widths use 16 x 128 units: max(64, 128) and max(128, 64).
  constexpr int U = 128;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t ku = K / U;
  const int64_t units = (N / 16) * ku;
  bool bad = false, badmap = false;
  for (int64_t u = warp; u < units; u += nwarps) {
    const int64_t rb = u / ku, kb = u - rb * ku;
    const int64_t blk = rb / 8;
    const int bits = bit_map[blk];
    int64_t co, go;
    mixed_block_offsets(bit_map, blk, K, lane, &co, &go);
    const int64_t row_in_blk = (rb % 8) * 16;
    const uint16_t *Wb = W + blk * 128 * K;
    if (bits == 4) {
      UnitRegs<4, 128> ur;
      load_unit(ur, Wb, K, row_in_blk, kb * U, lane);
      bad |= quantize_unit<WT, 4, 128>(ur, 128, K, row_in_blk, kb * U, packed + co, scales + go, zeros + go, lane);
    } else if (bits == 2) {
      UnitRegs<2, 64> ur;
      load_unit(ur, Wb, K, row_in_blk, kb * U, lane);
      bad |= quantize_unit<WT, 2, 64>(ur, 128, K, row_in_blk, kb * U, packed + co, scales + go, zeros + go, lane);
    } else {
      badmap = true;
    }
  }
  if (bad) bq_flag(BQ_FLAG_NONFINITE);
  if (badmap) bq_flag(BQ_FLAG_BADMAP);
}

// Canonical mixed: a warp quantizes 256 consecutive weights of one row; the
// block's codes are flat within its own 128 x K region.
template <int WT>
__global__ void __launch_bounds__(256)
quantize_mixed_canonical_kernel(const uint16_t *__restrict__ W, int64_t N, int64_t K,
                                const uint8_t *__restrict__ bit_map, uint8_t *__restrict__ packed,
                                float *__restrict__ scales, uint8_t *__restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t per_row = K / 256;
  const int64_t chunks = N * per_row;
  bool bad_any = false, badmap = false;
  for (int64_t ch = warp; ch < chunks; ch += nwarps) {
    const int64_t row = ch / per_row, kc = ch - row * per_row;
    const int64_t blk = row / 128;
    const int bits = bit_map[blk];
    int64_t co, go;
    mixed_block_offsets(bit_map, blk, K, lane, &co, &go);
    const int64_t e_in_blk = (row % 128) * K + kc * 256 + lane * 8;  // flat index inside block
    uint4 v = ld_stream_v4(W + blk * 128 * K + e_in_blk);
    float s;
    uint8_t z;
    bool bad;
    if (bits == 4) {
      uint32_t pk = quant8_canonical<WT, 4, 128>(v, true, &s, &z, &bad);
      reinterpret_cast<uint32_t *>(packed + co)[e_in_blk / 8] = pk;
      if ((lane % 16) == 0) { scales[go + e_in_blk / 128] = s; zeros[go + e_in_blk / 128] = z; }
      bad_any |= bad;
    } else if (bits == 2) {
      uint32_t pk = quant8_canonical<WT, 2, 64>(v, true, &s, &z, &bad);
      reinterpret_cast<uint16_t *>(packed + co)[e_in_blk / 8] = (uint16_t)pk;
      if ((lane % 8) == 0) { scales[go + e_in_blk / 64] = s; zeros[go + e_in_blk / 64] = z; }
      bad_any |= bad;
    } else {
      badmap = true;
    }
  }
  if (bad_any) bq_flag(BQ_FLAG_NONFINITE);
  if (badmap) bq_flag(BQ_FLAG_BADMAP);
}

}  // namespace bq
