// dequant.cuh -- W_hat = (q - z) * s ("低比特量化", section "Zero Point"),
// computed in fp32 and rounded once to the output type.  A test / inspection
// utility: the linear kernels never materialize W_hat.
#pragma once
#include "common.cuh"

namespace bq {

template <int OT> struct OutT;
template <> struct OutT<0> { using T = __half; static BQ_DEV T cvt(float v) { return __float2half_rn(v); } };
template <> struct OutT<1> { using T = __nv_bfloat16; static BQ_DEV T cvt(float v) { return __float2bfloat16_rn(v); } };
template <> struct OutT<2> { using T = float; static BQ_DEV T cvt(float v) { return v; } };

BQ_DEV float deq(uint32_t q, uint8_t z, float s) { return __fmul_rn((float)((int)q - (int)z), s); }

// canonical: element e of the (block) matrix is flat; one thread per 8 codes.
template <int OT, int BITS>
BQ_DEV void dequant8_canonical(const uint8_t *__restrict__ packed, const float *__restrict__ scales,
                               const uint8_t *__restrict__ zeros, int group, int64_t e,
                               typename OutT<OT>::T *__restrict__ out) {
  uint32_t w = (BITS == 4) ? reinterpret_cast<const uint32_t *>(packed)[e / 8]
                           : reinterpret_cast<const uint16_t *>(packed)[e / 8];
  const float s = scales[e / group];
  const uint8_t z = zeros[e / group];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t q = (w >> (BITS * i)) & ((1u << BITS) - 1);
    out[e + i] = OutT<OT>::cvt(deq(q, z, s));
  }
}

template <int OT, int BITS>
__global__ void dequant_canonical_kernel(const uint8_t *__restrict__ packed, const float *__restrict__ scales,
                                         const uint8_t *__restrict__ zeros, int group, int64_t elems,
                                         typename OutT<OT>::T *__restrict__ out) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t * 8 < elems;
       t += (int64_t)gridDim.x * blockDim.x)
    dequant8_canonical<OT, BITS>(packed, scales, zeros, group, t * 8, out);
}

// interleaved: one warp per 512-byte tile (logical row tile rt, column block
// kt); lane L owns rows r, r+8 and column pairs (2c, 2c+1), (2c+8, 2c+9) of
// every 16-column run.
template <int OT, int BITS>
BQ_DEV void dequant_tile(const uint8_t *__restrict__ packed, const float *__restrict__ scales,
                         const uint8_t *__restrict__ zeros, int group, int64_t N, int64_t K, int64_t tile,
                         int lane, typename OutT<OT>::T *__restrict__ out) {
  constexpr int T = (BITS == 4) ? 64 : 128;
  const int64_t kt_per_row = K / T;
  const int64_t rt = tile / kt_per_row, kt = tile % kt_per_row;
  const int64_t row0 = rt * 16, col0 = kt * T;
  const int r = lane >> 2, c = lane & 3;
  const uint4 v = *reinterpret_cast<const uint4 *>(packed + il_tile_offset(rt, kt, N, K, BITS) + lane * 16);
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
  const int64_t GK = K / group;
#pragma unroll
  for (int run = 0; run < T / 16; ++run) {
    const uint32_t w = words[BITS == 4 ? run : run / 2];
#pragma unroll
    for (int slot = 0; slot < 4; ++slot) {
      const int h = slot & 1, hp = slot >> 1;
      const int64_t row = row0 + r + 8 * h;
      const int64_t col = col0 + 16 * run + 2 * c + 8 * hp;
      int f_even, f_odd;
      if (BITS == 4) { f_even = slot; f_odd = slot + 4; }
      else { f_even = 4 * (run & 1) + slot; f_odd = f_even + 8; }
      const uint32_t mask = (1u << BITS) - 1;
      const uint32_t q0 = (w >> (BITS * f_even)) & mask, q1 = (w >> (BITS * f_odd)) & mask;
      const int64_t mi = il_meta_index(row, col / group, N, GK);
      const float s = scales[mi];
      const uint8_t z = zeros[mi];
      out[row * K + col] = OutT<OT>::cvt(deq(q0, z, s));
      out[row * K + col + 1] = OutT<OT>::cvt(deq(q1, z, s));
    }
  }
}

template <int OT, int BITS>
__global__ void dequant_tiled_kernel(const uint8_t *__restrict__ packed, const float *__restrict__ scales,
                                     const uint8_t *__restrict__ zeros, int group, int64_t N, int64_t K,
                                     typename OutT<OT>::T *__restrict__ out) {
  constexpr int T = (BITS == 4) ? 64 : 128;
  const int lane = threadIdx.x & 31;
  const int64_t tiles = (N / 16) * (K / T);
  for (int64_t t = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; t < tiles;
       t += ((int64_t)gridDim.x * blockDim.x) >> 5)
    dequant_tile<OT, BITS>(packed, scales, zeros, group, N, K, t, lane, out);
}

// mixed: one warp per 512-byte tile of either width; a 128-row block holds
// 8 * K / T tiles of its width.
template <int OT, bool TILED>
__global__ void dequant_mixed_kernel(const uint8_t *__restrict__ packed, const float *__restrict__ scales,
                                     const uint8_t *__restrict__ zeros, const uint8_t *__restrict__ bit_map,
                                     int64_t N, int64_t K, typename OutT<OT>::T *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t nblk = N / 128;
  for (int64_t blk = warp; blk < nblk; blk += nwarps) {
    int64_t sb = 0, sg = 0;
    for (int64_t j = 0; j < blk; ++j) { sb += bit_map[j]; sg += (bit_map[j] == 4) ? 1 : 2; }
    const uint8_t *pk = packed + sb * 16 * K;
    const float *sc = scales + sg * K;
    const uint8_t *ze = zeros + sg * K;
    typename OutT<OT>::T *o = out + blk * 128 * K;
    const int bits = bit_map[blk];
    if (bits != 4 && bits != 2) { if (lane == 0) bq_flag(BQ_FLAG_BADMAP); continue; }
    if (TILED) {
      const int64_t tiles = 8 * K / (bits == 4 ? 64 : 128);
      for (int64_t t = 0; t < tiles; ++t) {
        if (bits == 4) dequant_tile<OT, 4>(pk, sc, ze, 128, 128, K, t, lane, o);
        else dequant_tile<OT, 2>(pk, sc, ze, 64, 128, K, t, lane, o);
      }
    } else {
      for (int64_t e = lane * 8; e < 128 * K; e += 256) {
        if (bits == 4) dequant8_canonical<OT, 4>(pk, sc, ze, 128, e, o);
        else dequant8_canonical<OT, 2>(pk, sc, ze, 64, e, o);
      }
    }
  }
}

}  // namespace bq
