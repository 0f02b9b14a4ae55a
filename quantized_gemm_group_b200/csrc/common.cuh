// common.cuh -- device helpers shared by the bq kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#define BQ_DEV __device__ __forceinline__

// Device status word: bit flags, read and cleared by bq_device_status().
enum : unsigned {
  BQ_FLAG_NONFINITE = 1u,
  BQ_FLAG_BADMAP = 2u,
  BQ_FLAG_TIMEOUT = 4u,
};
__device__ unsigned int g_bq_status;

BQ_DEV void bq_flag(unsigned f) { atomicOr(&g_bq_status, f); }

// ---------------------------------------------------------------------------
// memory access
// ---------------------------------------------------------------------------

// Streaming 16-byte load through the non-coherent path, not kept in L1.
BQ_DEV uint4 ld_stream_v4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// 4-byte read-only load kept in L1 (neighbouring lanes re-use the sector).
BQ_DEV uint32_t ld_nc_u32(const void *p) {
  uint32_t r;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

BQ_DEV void st_v4(void *p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// ---------------------------------------------------------------------------
// 16-bit element types
// ---------------------------------------------------------------------------

template <int WT> struct Elem;
template <> struct Elem<0> {  // fp16
  using T = __half;
  using T2 = __half2;
  static BQ_DEV float lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xffff))); }
  static BQ_DEV float hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }
  static BQ_DEV uint32_t min2(uint32_t a, uint32_t b) {
    __half2 r = __hmin2_nan(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
  }
  static BQ_DEV uint32_t max2(uint32_t a, uint32_t b) {
    __half2 r = __hmax2_nan(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
  }
  static BQ_DEV uint16_t from_float(float v) { return __half_as_ushort(__float2half_rn(v)); }
};
template <> struct Elem<1> {  // bf16
  using T = __nv_bfloat16;
  using T2 = __nv_bfloat162;
  static BQ_DEV float lo(uint32_t w) { return __uint_as_float(w << 16); }
  static BQ_DEV float hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
  static BQ_DEV uint32_t min2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmin2_nan(*reinterpret_cast<__nv_bfloat162 *>(&a),
                                   *reinterpret_cast<__nv_bfloat162 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
  }
  static BQ_DEV uint32_t max2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmax2_nan(*reinterpret_cast<__nv_bfloat162 *>(&a),
                                   *reinterpret_cast<__nv_bfloat162 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
  }
  static BQ_DEV uint16_t from_float(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }
};

// NaN-propagating fp32 min / max.
BQ_DEV float fmin_nan(float a, float b) {
  float r;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
BQ_DEV float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// ---------------------------------------------------------------------------
// Correctly rounded x / s for the quantizer's hot loop.
//
// Division by refinement (P. Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990;
// restated as Markstein's theorem in Muller et al., "Handbook of
// Floating-Point Arithmetic"): with r = RN(1/s) and a quotient estimate q
// within one ulp of x/s, the fused residual e = x - s*q is exact and
// RN(q + e*r) is the correctly rounded quotient.  The first refinement of
// q0 = RN(x*r) (error below 1.5 ulp) gives a faithful q1; the second
// refinement then returns RN(x/s).  Valid while no step over- or underflows:
// callers use it only for 2^-60 <= s <= 2^60, where every quotient whose
// rounding matters (|x/s| >= 1/4) keeps its residuals normal.  Checked
// exhaustively against the IEEE division (__fdiv_rn) by the GPU tests.
// ---------------------------------------------------------------------------
BQ_DEV float div_refined(float x, float s, float r) {
  float q0 = __fmul_rn(x, r);
  float e0 = __fmaf_rn(-s, q0, x);
  float q1 = __fmaf_rn(e0, r, q0);
  float e1 = __fmaf_rn(-s, q1, x);
  return __fmaf_rn(e1, r, q1);
}

// Round half to even to an integer for |t| < 2^22: adding 1.5 * 2^23 leaves
// a unit in the last place of 1, so the fp32 add rounds t to an integer
// (ties to even) and the low mantissa bits hold 2^22 + round(t).
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23
constexpr int kRoundMagicBits = 0x4B400000;  // its bit pattern
BQ_DEV int round_even_small(float t) {
  return __float_as_int(__fadd_rn(t, kRoundMagic)) - kRoundMagicBits;
}

// Per-group quantization parameters, computed exactly as the reading of the
// method prescribes (range widened to contain 0, fp32 IEEE steps).
struct GroupParams {
  float s;       // stored scale (0 for an all-zero group)
  float sd;      // divisor used for the codes (1 for an all-zero group: 0/1 = 0)
  float r;       // RN(1/sd)
  int zc;        // z - kRoundMagicBits: added to the rounded bits of x/sd
  int z;         // zero point
  bool fast;     // 2^-60 <= sd <= 2^60: the refined division applies
  bool bad;      // non-finite input or overflowing scale
};

BQ_DEV GroupParams group_params(float mn, float mx, int qmax) {
  GroupParams p;
  p.bad = !(fabsf(mn) <= 3.402823466e38f) || !(fabsf(mx) <= 3.402823466e38f);
  float lo = fminf(mn, 0.0f);
  float hi = fmaxf(mx, 0.0f);
  float s = __fdiv_rn(__fsub_rn(hi, lo), (float)qmax);
  p.bad |= !(s <= 3.402823466e38f);
  if (p.bad || s == 0.0f) {
    // all-zero group: s = 0, z = 0 and every x is +-0, so x / 1 rounds to 0
    // and every code is 0.  A bad group gets the same (unspecified) treatment.
    p.s = 0.0f;
    p.sd = 1.0f;
    p.r = 1.0f;
    p.z = 0;
    p.zc = -kRoundMagicBits;
    p.fast = true;
    return p;
  }
  p.s = s;
  p.sd = s;
  p.z = __float2int_rn(__fdiv_rn(-lo, s));
  p.zc = p.z - kRoundMagicBits;
  p.fast = (s >= 8.67361738e-19f) && (s <= 1.15292150e18f);  // 2^-60 .. 2^60
  p.r = __frcp_rn(s);
  return p;
}

// Code of one element: min(round(x/s) + z, qmax).  round(x/s) + z >= 0 holds
// for every x of the group (x >= lo gives round(x/s) >= round(lo/s) = -z), so
// the unsigned min is the clamp; it also keeps a flagged bad group's garbage
// inside its own field.  ALWAYS_FAST: fp16 inputs, whose scales always lie in
// [2^-28, 2^16].
template <int QMAX, bool ALWAYS_FAST>
BQ_DEV uint32_t code_of(float x, const GroupParams &p) {
  float t = (ALWAYS_FAST || p.fast) ? div_refined(x, p.sd, p.r) : __fdiv_rn(x, p.sd);
  int q = __float_as_int(__fadd_rn(t, kRoundMagic)) + p.zc;
  return min((uint32_t)q, (uint32_t)QMAX);
}
