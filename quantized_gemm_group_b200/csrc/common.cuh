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
  static BQ_DEV float2 pair(uint32_t w) { return __half22float2(*reinterpret_cast<__half2 *>(&w)); }
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
  static BQ_DEV float2 pair(uint32_t w) { return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)); }
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

// RN(x / D) for the small constant divisors 2^b - 1 and 2^(b-1) - 1: the
// refined quotient above with r = RN(1/D) (a constant), where its residuals
// stay normal (2^-100 <= |x| <= 2^120); the IEEE division elsewhere.
template <int D>
BQ_DEV float div_const(float x) {
  static_assert(D == 1 || D == 3 || D == 7 || D == 15, "no reciprocal constant for this divisor");
  if (D == 1) return x;
  // RN(1/15), RN(1/3), RN(1/7) in fp32 (0x3d888889, 0x3eaaaaab, 0x3e124925)
  constexpr float kInv = (D == 15) ? 0x1.111112p-4f : (D == 3) ? 0x1.555556p-2f : 0x1.24924ap-3f;
  const float ax = fabsf(x);
  if (ax >= 0x1p-100f && ax <= 0x1p120f) return div_refined(x, (float)D, kInv);
  return __fdiv_rn(x, (float)D);
}

// RN(x / s) given r = RN(1/s): the refined quotient when s lies in
// [2^-60, 2^60] (`fast`), where every quotient whose rounding to an integer
// matters keeps its residuals normal; the IEEE division otherwise.
BQ_DEV float div_group(float x, float s, float r, bool fast) {
  return fast ? div_refined(x, s, r) : __fdiv_rn(x, s);
}

// Per-group quantization parameters, computed exactly as the reading of the
// method prescribes (range widened to contain 0, correctly rounded fp32
// steps: every quotient below equals the IEEE division's).
struct GroupParams {
  float s;       // stored scale (0 for an all-zero group)
  float sd;      // divisor used for the codes (1 for an all-zero group: 0/1 = 0)
  float r;       // RN(1/sd)
  int zc;        // z - kRoundMagicBits: added to the rounded bits of x/sd
  int z;         // zero point
  bool fast;     // 2^-60 <= sd <= 2^60: the refined division applies
  bool clamp;    // some code of the group would reach 2^b (or the group is bad)
  bool bad;      // non-finite input or overflowing scale
};

// Symmetric abs-max scheme ("大模型量化实战", section 2.3): s = max|x| /
// (2^(b-1) - 1), zero point 0, codes stored offset by 2^(b-1) (z = 2^(b-1)),
// so the same code rounding, storage and dequantization apply.  An all-zero
// group stores s = 0 and every code equal to z.
template <int QMAX>
BQ_DEV GroupParams group_params_sym(float mn, float mx) {
  constexpr int ZC = (QMAX + 1) / 2;
  GroupParams p;
  p.bad = !(fabsf(mn) <= 3.402823466e38f) || !(fabsf(mx) <= 3.402823466e38f);
  const float amax = fmaxf(fabsf(mn), fabsf(mx));
  const float s = div_const<ZC - 1>(amax);
  p.bad |= !(s <= 3.402823466e38f);
  p.z = ZC;
  p.zc = ZC - kRoundMagicBits;
  if (p.bad || s == 0.0f) {
    p.s = 0.0f;
    p.sd = 1.0f;
    p.r = 1.0f;
    p.fast = true;
    p.clamp = true;
    return p;
  }
  p.s = s;
  p.sd = s;
  p.fast = (s >= 8.67361738e-19f) && (s <= 1.15292150e18f);  // 2^-60 .. 2^60
  p.r = __frcp_rn(s);
  p.clamp = __float2int_rn(div_group(amax, s, p.r, p.fast)) + ZC > QMAX;
  return p;
}

// SCHEME 0: asymmetric MinMax (below); 1: symmetric abs-max; 2: asymmetric
// MinMax with the scale stored as binary16: s rounded to the nearest binary16
// (ties to even; a positive s below the binary16 range takes 2^-24, one
// above it marks the group non-finite), and z and the codes computed from
// that stored value.
template <int QMAX, int SCHEME = 0>
BQ_DEV GroupParams group_params(float mn, float mx) {
  if (SCHEME == 1) return group_params_sym<QMAX>(mn, mx);
  GroupParams p;
  p.bad = !(fabsf(mn) <= 3.402823466e38f) || !(fabsf(mx) <= 3.402823466e38f);
  float lo = fminf(mn, 0.0f);
  float hi = fmaxf(mx, 0.0f);
  float s = div_const<QMAX>(__fsub_rn(hi, lo));
  if (SCHEME == 2 && s > 0.0f && s <= 3.402823466e38f) {
    s = __half2float(__float2half_rn(s));
    if (s == 0.0f) s = 0x1p-24f;
  }
  p.bad |= !(s <= 3.402823466e38f);
  if (p.bad || s == 0.0f) {
    // all-zero group: s = 0, z = 0 and every x is +-0, so x / 1 rounds to 0
    // and every code is 0.  A bad group gets the same (unspecified) codes.
    p.s = 0.0f;
    p.sd = 1.0f;
    p.r = 1.0f;
    p.z = 0;
    p.zc = -kRoundMagicBits;
    p.fast = true;
    p.clamp = true;
    return p;
  }
  p.s = s;
  p.sd = s;
  p.fast = (s >= 8.67361738e-19f) && (s <= 1.15292150e18f);  // 2^-60 .. 2^60
  p.r = __frcp_rn(s);
  p.z = __float2int_rn(div_group(-lo, s, p.r, p.fast));
  p.zc = p.z - kRoundMagicBits;
  // Codes are monotone in x, so only the largest element can overflow:
  // round(hi / s) + z > 2^b - 1 decides whether this group needs the clamp.
  p.clamp = __float2int_rn(div_group(hi, s, p.r, p.fast)) + p.z > QMAX;
  return p;
}

// x / s rounded to an integer (ties to even) for two elements, still carrying
// the 1.5 * 2^23 magic: the low bits of each result's bit pattern minus
// kRoundMagicBits are round(x / s).  ALWAYS_FAST as in code_pair.
template <bool ALWAYS_FAST>
BQ_DEV float2 rounded_quotients(float2 v, const GroupParams &p) {
  float2 t;
  if (ALWAYS_FAST || p.fast) {
    const float2 r2 = make_float2(p.r, p.r), ns2 = make_float2(-p.sd, -p.sd);
    float2 q0 = __fmul2_rn(v, r2);
    float2 e0 = __ffma2_rn(ns2, q0, v);
    float2 q1 = __ffma2_rn(e0, r2, q0);
    float2 e1 = __ffma2_rn(ns2, q1, v);
    t = __ffma2_rn(e1, r2, q1);
  } else {
    t = make_float2(__fdiv_rn(v.x, p.sd), __fdiv_rn(v.y, p.sd));
  }
  return __fadd2_rn(t, make_float2(kRoundMagic, kRoundMagic));
}

// Store a group scale: fp32, or (SCHEME 2) the binary16 value it already is.
template <int SCHEME>
BQ_DEV void store_scale(void *scales, int64_t i, float s) {
  if (SCHEME == 2) reinterpret_cast<uint16_t *>(scales)[i] = __half_as_ushort(__float2half_rn(s));
  else reinterpret_cast<float *>(scales)[i] = s;
}

// Codes of two elements of one group.
// code = min(round(x/s) + z, 2^b - 1); round(x/s) + z >= 0 always holds
// (x >= lo gives round(x/s) >= round(lo/s) = -z), and round(x/s) + z can
// exceed 2^b - 1 only in groups flagged `clamp`.  The unsigned min also keeps
// a bad group's garbage inside its own field.  ALWAYS_FAST: fp16 inputs,
// whose scales always lie in [2^-28, 2^16].
template <int QMAX, bool ALWAYS_FAST, bool CLAMP>
BQ_DEV uint2 code_pair(float2 v, const GroupParams &p) {
  const float2 m = rounded_quotients<ALWAYS_FAST>(v, p);
  uint32_t a = (uint32_t)(__float_as_int(m.x) + p.zc);
  uint32_t b = (uint32_t)(__float_as_int(m.y) + p.zc);
  if (CLAMP) {
    a = min(a, (uint32_t)QMAX);
    b = min(b, (uint32_t)QMAX);
  }
  return make_uint2(a, b);
}

// ---------------------------------------------------------------------------
// interleaved layout addressing (see include/bq.h)
// ---------------------------------------------------------------------------

// 16-row tiles of a 128-row block (8, or fewer in the last partial block).
BQ_DEV int64_t il_block_tiles(int64_t rt, int64_t N) {
  const int64_t b = rt / 8;
  const int64_t left = N / 16 - 8 * b;
  return left < 8 ? left : 8;
}
// Byte offset of tile (global row tile rt, column block kt) of an N x K
// matrix whose column blocks are T wide and hold BITS-bit codes.
BQ_DEV int64_t il_tile_offset(int64_t rt, int64_t kt, int64_t N, int64_t K, int bits) {
  const int64_t b = rt / 8;
  return b * 128 * K * bits / 8 + (kt * il_block_tiles(rt, N) + rt % 8) * 512;
}
// Metadata index of group g of row n (G groups per row).
BQ_DEV int64_t il_meta_index(int64_t n, int64_t g, int64_t N, int64_t G) {
  const int64_t b = n / 128;
  return 128 * G * b + g * (16 * il_block_tiles(n / 16, N)) + n % 128;
}

// ---------------------------------------------------------------------------
// mbarrier / bulk-copy (TMA) helpers
// ---------------------------------------------------------------------------

BQ_DEV uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

BQ_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
BQ_DEV void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
BQ_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
BQ_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
BQ_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of the phase with the given parity.
BQ_DEV bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// One 2D tensor-map (TMA) tile load into this CTA's shared memory,
// completing on `bar`; coordinates (c0 innermost, c1) in elements.
BQ_DEV void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Bounded wait on the phase with the given parity: false after `limit` polls.
constexpr uint32_t kWaitLimit = 1u << 22;
BQ_DEV bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t limit = kWaitLimit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
// One bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
BQ_DEV void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start
// launching / wait until the previous one has completed and its memory is
// visible.  Both are no-ops when the launch did not opt in.
BQ_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
BQ_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
