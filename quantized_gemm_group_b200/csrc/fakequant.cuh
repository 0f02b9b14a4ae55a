// fakequant.cuh -- fake quantization (the forward of quantization-aware
// training): W_hat = (q - z) * s with q, s, z those of the group-wise MinMax
// quantizer, in one pass and without storing codes, scales or zeros
// ("大模型量化实战：从原理到4-bit部署的完整指南", section 5.2: a FakeQuantize
// module simulates round(x/s) + z in the forward pass; "A Survey of Low-bit
// Large Language Models", section 8.1).  HBM-bound: 2 bytes read and 2 (or 4)
// written per weight.  The codes come from the same per-group arithmetic as
// the canonical quantizer (quant8_canonical) and each W_hat element from the
// same fp32 product as the dequantizer (deq), rounded once to the output
// type, so the result equals bq_dequantize(bq_quantize(W)) bit for bit.
#pragma once
#include "common.cuh"
#include "dequant.cuh"
#include "quantize.cuh"

namespace bq {

template <int WT, int OT, int BITS, int G, int UNROLL>
__global__ void __launch_bounds__(256)
fake_quant_kernel(const uint16_t *__restrict__ W, int64_t elems, typename OutT<OT>::T *__restrict__ out) {
  using T = typename OutT<OT>::T;
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
      const int64_t e = (c0 + u) * 256 + lane * 8;
      act[u] = (c0 + u < chunks) && (e < elems);
      v[u] = act[u] ? ld_stream_v4(W + e) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t e = (c0 + u) * 256 + lane * 8;
      float s;
      uint8_t z;
      bool bad;
      const uint32_t pk = quant8_canonical<WT, BITS, G>(v[u], act[u], &s, &z, &bad);
      if (!act[u]) continue;
      bad_any |= bad;
      T o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = OutT<OT>::cvt(deq((pk >> (BITS * i)) & ((1u << BITS) - 1), z, s));
      // 8 consecutive outputs: one 16-byte store (two for fp32)
      const uint4 *src = reinterpret_cast<const uint4 *>(o);
      uint4 *dst = reinterpret_cast<uint4 *>(out + e);
#pragma unroll
      for (int k = 0; k < (int)(8 * sizeof(T) / 16); ++k) dst[k] = src[k];
    }
  }
  if (bad_any) bq_flag(BQ_FLAG_NONFINITE);
}

}  // namespace bq
