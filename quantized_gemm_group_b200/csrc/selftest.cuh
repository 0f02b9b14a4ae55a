// selftest.cuh -- exhaustive check of the quantizer's refined division.
//
// The quantizer computes round(x / s) from a correctly rounded quotient
// obtained by refinement (div_refined, common.cuh) instead of the IEEE
// division.  Scaling x and s by powers of two scales every step exactly as
// long as nothing over- or underflows, so comparing against __fdiv_rn for
// every fp32 divisor of one binade and every fp16 numerator covers every
// (significand, relative exponent) pair the quantizer meets with fp16 or bf16
// weights (bf16 significands are a subset of fp16 ones).
#pragma once
#include "common.cuh"

namespace bq {

template <int REFINE>
BQ_DEV float div_refine_n(float x, float s, float r) {
  float q = __fmul_rn(x, r);
#pragma unroll
  for (int i = 0; i < REFINE; ++i) {
    const float e = __fmaf_rn(-s, q, x);
    q = __fmaf_rn(e, r, q);
  }
  return q;
}

// One thread per divisor bit pattern; every fp16 numerator with |x| < 64.
template <int REFINE>
__global__ void check_division_kernel(uint32_t s_begin, uint32_t s_end, unsigned long long *result) {
  unsigned long long bad = 0, checked = 0;
  for (uint64_t sb = s_begin + (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; sb < s_end;
       sb += (uint64_t)gridDim.x * blockDim.x) {
    const float s = __uint_as_float((uint32_t)sb);
    const float r = __frcp_rn(s);
    for (uint32_t hb = 0; hb < 0x5400u; ++hb) {  // |x| < 64, both signs
#pragma unroll
      for (int sign = 0; sign < 2; ++sign) {
        const float x = __half2float(__ushort_as_half((unsigned short)(hb | (sign << 15))));
        const float ref = __fdiv_rn(x, s);
        const float got = div_refine_n<REFINE>(x, s, r);
        // identical bits, except that a zero quotient may come back as +0 for
        // x = -0 (both round to the same code)
        if (__float_as_uint(ref) != __float_as_uint(got) && !(ref == 0.0f && got == 0.0f)) {
          if (bad == 0 && atomicCAS(result + 2, 0ull, (unsigned long long)sb) == 0ull)
            result[3] = hb | (sign << 15);
          ++bad;
        }
      }
    }
    checked += 2 * 0x5400u;
  }
  atomicAdd(result + 0, bad);
  atomicAdd(result + 1, checked);
}

// The quantizer's division by the constant number of levels (div_const):
// every fp32 bit pattern in [x_begin, x_end) against the IEEE division by D.
template <int D>
__global__ void check_const_division_kernel(uint32_t x_begin, uint32_t x_end, unsigned long long *result) {
  unsigned long long bad = 0, checked = 0;
  for (uint64_t xb = x_begin + (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; xb < x_end;
       xb += (uint64_t)gridDim.x * blockDim.x) {
    const float x = __uint_as_float((uint32_t)xb);
    const float ref = __fdiv_rn(x, (float)D);
    const float got = div_const<D>(x);
    // identical bits (NaN inputs: any NaN)
    if (__float_as_uint(ref) != __float_as_uint(got) && !(ref != ref && got != got)) {
      if (bad == 0 && atomicCAS(result + 2, 0ull, (unsigned long long)xb) == 0ull) result[3] = D;
      ++bad;
    }
    ++checked;
  }
  atomicAdd(result + 0, bad);
  atomicAdd(result + 1, checked);
}

}  // namespace bq

namespace bq {

// One thread waits, through the bounded wait every kernel of the library
// uses, on the first phase of an mbarrier that nothing ever arrives on.
// After `limit` polls the wait gives up, the kernel records BQ_FLAG_TIMEOUT
// and returns normally: the failure path of a bounded wait, exercised
// without a hang or a fault.
__global__ void bounded_wait_kernel(uint32_t limit) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(b, 0, limit)) bq_flag(BQ_FLAG_TIMEOUT);
}

}  // namespace bq
