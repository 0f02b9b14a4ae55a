// bq_api.cu -- C ABI of the quantizer / weight-only linear library (see
// include/bq.h for the contract of every entry point).  Host-side argument
// validation, launch geometry and dispatch onto the sm_100a kernels.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/bq.h"
#include "common.cuh"
#include "dequant.cuh"
#include "fakequant.cuh"
#include "grad.cuh"
#include "gemm.cuh"
#include "gemv.cuh"
#include "quantize.cuh"
#include "selftest.cuh"

using namespace bq;

namespace {

constexpr int kThreads = 256;

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int kMaxDevices = 64;

// cudaFuncAttributeMaxDynamicSharedMemorySize is a per-device setting of a
// kernel: it is set on each device the first time the kernel needs more than
// the default there (one record per kernel -- the template argument is the
// kernel itself, not its type, which instantiations share -- and device; two
// threads racing only set it twice).
template <auto Kern>
bool ensure_smem(int bytes) {
  static std::atomic<int> set_to[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < kMaxDevices && set_to[dev].load(std::memory_order_acquire) >= bytes) return true;
  if (cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  if (dev >= 0 && dev < kMaxDevices) {
    int cur = set_to[dev].load(std::memory_order_relaxed);
    while (cur < bytes && !set_to[dev].compare_exchange_weak(cur, bytes, std::memory_order_acq_rel)) {
    }
  }
  return true;
}

bq_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

int64_t grid_for(int64_t warps_of_work) {
  int64_t blocks = (warps_of_work + (kThreads / 32) - 1) / (kThreads / 32);
  int64_t cap = (int64_t)sm_count() * 8;  // 8 x 256 threads = 2048 per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return blocks;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (no
// link-time dependency on libcuda).
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A [rows, cols] 16-bit row-major matrix as a 2D tensor map with boxes of
// box_cols x box_rows elements, 128-byte swizzle (box_cols * 2 <= 128), rows
// and columns past the edges read as zero.
bool make_map_2d(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, bool bf16, int box_cols,
                 int box_rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                   const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool valid_bits(int bits) { return bits == 2 || bits == 4; }
int tile_width(int bits) { return bits == 4 ? 64 : 128; }

// ---------------------------------------------------------------------------
// quantize dispatch
// ---------------------------------------------------------------------------

template <int WT, int BITS, int SCHEME>
bq_status quantize_canonical(const uint16_t *W, int64_t elems, int group, uint8_t *packed, void *scales,
                             uint8_t *zeros, cudaStream_t st) {
  const int64_t grid = grid_for((elems + 255) / 256);
#define BQ_QC(G)                                                                              \
  case G:                                                                                     \
    quantize_canonical_kernel<WT, BITS, G, 4, SCHEME><<<grid, kThreads, 0, st>>>(W, elems, packed, scales, zeros); \
    break;
  if constexpr (SCHEME == 2) {  // binary16 scales: the linear layer's groups, INT4 g128 and INT2 g64
    switch (group) {
      BQ_QC(64) BQ_QC(128)
      default: return BQ_ERR_UNSUPPORTED;
    }
  } else {
    switch (group) {
      BQ_QC(8) BQ_QC(16) BQ_QC(32) BQ_QC(64) BQ_QC(128) BQ_QC(256)
      default: return BQ_ERR_UNSUPPORTED;
    }
  }
#undef BQ_QC
  return launch_status();
}

// Interleaved layout: the TMA-staged kernel, two CTAs per SM, each with a ring
// of super-units (64 rows x U columns) in about 110 KB of shared memory.
template <int WT, int BITS, int G, int SCHEME>
bq_status quantize_tma(const uint16_t *W, int64_t N, int64_t K, uint8_t *packed, void *scales, uint8_t *zeros,
                       cudaStream_t st) {
  constexpr int U = UnitGeom<BITS, G>::U;
  constexpr int SU = (U / 64) * 8192;
  constexpr int kBudget = (227 * 1024) / qt_ctas_per_sm<G>() - 1024;  // shared memory per CTA
  auto kern = quantize_tma_kernel<WT, BITS, G, SCHEME>;
  if (!ensure_smem<quantize_tma_kernel<WT, BITS, G, SCHEME>>(kBudget)) return BQ_ERR_CUDA;
  int stages = (kBudget - 1024 - 16) / (SU + 16);
  if (stages > 8) stages = 8;
  if (stages < 2) return BQ_ERR_UNSUPPORTED;
  const int smem = stages * SU + 16 * stages + 16 + 1024;
  CUtensorMap map;
  if (!make_map_2d(&map, W, N, K, WT == 1, 64, 64)) return BQ_ERR_CUDA;
  const int64_t nsu = ((N + 63) / 64) * (K / U);
  int64_t grid = qt_ctas_per_sm<G>() * (int64_t)sm_count();
  if (grid > nsu) grid = nsu;
  kern<<<(unsigned)grid, kQtThreads, smem, st>>>(map, N, K, stages, packed, scales, zeros);
  return launch_status();
}

template <int WT, int BITS, int SCHEME>
bq_status quantize_tiled(const uint16_t *W, int64_t N, int64_t K, int group, uint8_t *packed, void *scales,
                         uint8_t *zeros, cudaStream_t st) {
  if constexpr (SCHEME == 2) {  // binary16 scales: the linear layer's groups, INT4 g128 and INT2 g64
    if (group == 64) return quantize_tma<WT, BITS, 64, SCHEME>(W, N, K, packed, scales, zeros, st);
    if (group == 128) return quantize_tma<WT, BITS, 128, SCHEME>(W, N, K, packed, scales, zeros, st);
    return BQ_ERR_UNSUPPORTED;
  } else switch (group) {
    case 16: return quantize_tma<WT, BITS, 16, SCHEME>(W, N, K, packed, scales, zeros, st);
    case 32: return quantize_tma<WT, BITS, 32, SCHEME>(W, N, K, packed, scales, zeros, st);
    case 64: return quantize_tma<WT, BITS, 64, SCHEME>(W, N, K, packed, scales, zeros, st);
    case 128: return quantize_tma<WT, BITS, 128, SCHEME>(W, N, K, packed, scales, zeros, st);
    case 256: return quantize_tma<WT, BITS, 256, SCHEME>(W, N, K, packed, scales, zeros, st);
    default: return BQ_ERR_UNSUPPORTED;
  }
}

template <int WT, int OT, int BITS>
bq_status fake_quant_dispatch(const uint16_t *W, int64_t elems, int group, void *out, cudaStream_t st) {
  using T = typename OutT<OT>::T;
  const int64_t grid = grid_for((elems + 255) / 256);
  T *o = reinterpret_cast<T *>(out);
#define BQ_FQ(G_)                                                                           \
  case G_:                                                                                  \
    fake_quant_kernel<WT, OT, BITS, G_, 2><<<grid, kThreads, 0, st>>>(W, elems, o);          \
    break;
  switch (group) {
    BQ_FQ(8) BQ_FQ(16) BQ_FQ(32) BQ_FQ(64) BQ_FQ(128) BQ_FQ(256)
    default: return BQ_ERR_UNSUPPORTED;
  }
#undef BQ_FQ
  return launch_status();
}

template <int WT, int OT>
bq_status fake_quant_bits(const uint16_t *W, int64_t elems, int bits, int group, void *out, cudaStream_t st) {
  return bits == 4 ? fake_quant_dispatch<WT, OT, 4>(W, elems, group, out, st)
                   : fake_quant_dispatch<WT, OT, 2>(W, elems, group, out, st);
}

bool canonical_group_ok(int g) { return g == 8 || g == 16 || g == 32 || g == 64 || g == 128 || g == 256; }
bool tiled_group_ok(int g) { return g == 16 || g == 32 || g == 64 || g == 128 || g == 256; }

// ---------------------------------------------------------------------------
// dequant dispatch
// ---------------------------------------------------------------------------

template <int OT>
bq_status dequant_uniform(const uint8_t *packed, const float *scales, const uint8_t *zeros, int bits, int group,
                          int64_t N, int64_t K, bq_layout layout, void *out, cudaStream_t st) {
  using T = typename OutT<OT>::T;
  T *o = reinterpret_cast<T *>(out);
  if (layout == BQ_LAYOUT_CANONICAL) {
    const int64_t elems = N * K;
    const int64_t grid = grid_for((elems / 8 + 31) / 32);
    if (bits == 4) dequant_canonical_kernel<OT, 4><<<grid, kThreads, 0, st>>>(packed, scales, zeros, group, elems, o);
    else dequant_canonical_kernel<OT, 2><<<grid, kThreads, 0, st>>>(packed, scales, zeros, group, elems, o);
  } else {
    const int64_t tiles = (N / 16) * (K / tile_width(bits));
    const int64_t grid = grid_for(tiles);
    if (bits == 4) dequant_tiled_kernel<OT, 4><<<grid, kThreads, 0, st>>>(packed, scales, zeros, group, N, K, o);
    else dequant_tiled_kernel<OT, 2><<<grid, kThreads, 0, st>>>(packed, scales, zeros, group, N, K, o);
  }
  return launch_status();
}

template <int OT>
bq_status dequant_mixed(const uint8_t *packed, const float *scales, const uint8_t *zeros, const uint8_t *bit_map,
                        int64_t N, int64_t K, bq_layout layout, void *out, cudaStream_t st) {
  using T = typename OutT<OT>::T;
  const int64_t grid = grid_for(N / 128);
  if (layout == BQ_LAYOUT_CANONICAL)
    dequant_mixed_kernel<OT, false><<<grid, kThreads, 0, st>>>(packed, scales, zeros, bit_map, N, K, reinterpret_cast<T *>(out));
  else
    dequant_mixed_kernel<OT, true><<<grid, kThreads, 0, st>>>(packed, scales, zeros, bit_map, N, K, reinterpret_cast<T *>(out));
  return launch_status();
}

// ---------------------------------------------------------------------------
// GEMV (M <= 16) geometry and dispatch
// ---------------------------------------------------------------------------

// 0: plain launches; 1: programmatic dependent launch (the kernel waits for
// the previous one before reading anything); 2: as 1, and weights may be
// streamed before that wait (the caller guarantees the preceding kernel does
// not write them).  -1: not read from the environment yet.
std::atomic<int> g_overlap_mode{-1};

int overlap_mode() {
  int m = g_overlap_mode.load(std::memory_order_relaxed);
  if (m < 0) {
    const char *e = getenv("BQ_OVERLAP");
    const int v = (e && (e[0] == '1' || e[0] == '2')) ? e[0] - '0' : 0;
    g_overlap_mode.compare_exchange_strong(m, v);
    m = g_overlap_mode.load(std::memory_order_relaxed);
  }
  return m;
}

struct GemvGeom {
  int NB, SK, stages;
  int64_t KC;
};

constexpr int kTwoCtaSmem = 112 * 1024;   // per-CTA budget that keeps two CTAs per SM
constexpr int kMaxSmem = 227 * 1024;

int deepest_ring(int M, int tok, int64_t kc, int groups, int budget) {
  for (int cand = kGemvMaxStages; cand >= 2; --cand)
    if (gemv_smem_layout(M, tok, kc, groups, cand).total <= budget) return cand;
  return 0;
}

// Split-K S_k (CTAs per cluster, dividing K / SC, at most 8) and ring depth.
// Preferred: the smallest split that gives every SM a CTA while two CTAs
// still fit per SM.  Otherwise the largest split that fits two CTAs per SM
// (more CTAs, more bytes in flight); otherwise the largest that fits at all.
// G_max: the smallest group size the kernel may meet (most metadata).
GemvGeom gemv_geometry(int M, int64_t N, int64_t K, int SC, int G_min) {
  // Split-K S_k: the smallest divisor of the stage count (at most 8) that
  // gives at least 4/5 of the SMs a CTA.  When that is more CTAs than SMs,
  // two CTAs share an SM (112 KB of shared memory each); otherwise one CTA
  // per SM with the deepest ring that fits.  (Measured on B200 over the
  // Llama-3-8B decode shapes, INT4 and INT2, M = 1 and 16: within ~10% of
  // the best split in every case.)
  GemvGeom g;
  g.NB = (M <= 8) ? 1 : 2;
  const int tok = 8 * g.NB;
  const int64_t rc = (N + 127) / 128;
  const int64_t nst = K / SC;
  const int64_t sms = sm_count();
  g.SK = 0;
  for (int d = 1; d <= 8; ++d) {
    if (nst % d) continue;
    const int64_t kc = K / d;
    const int groups = (int)(kc / G_min);
    const int st2 = deepest_ring(M, tok, kc, groups, kTwoCtaSmem);
    const int st1 = deepest_ring(M, tok, kc, groups, kMaxSmem);
    if (!st1) continue;
    g.SK = d;
    g.stages = (rc * d > sms && st2) ? st2 : st1;
    if (5 * rc * d >= 4 * sms) break;
  }
  if (g.SK == 0) {
    g.SK = 8;
    g.stages = 2;
  }
  g.KC = K / g.SK;
  return g;
}

template <int XT, int BITS, int G, int NB, bool MIXED, bool S16>
bq_status launch_gemv_t(const GemvGeom &g, GemvArgs a, int G_min, cudaStream_t st) {
  auto kern = gemv_kernel<XT, BITS, G, NB, MIXED, S16>;
  if (!ensure_smem<gemv_kernel<XT, BITS, G, NB, MIXED, S16>>(kMaxSmem)) return BQ_ERR_CUDA;
  a.stages = g.stages;
  a.KC = g.KC;
  a.L = gemv_smem_layout(a.M, 8 * NB, g.KC, (int)(g.KC / G_min), g.stages);
  if (a.L.total > kMaxSmem) return BQ_ERR_SHAPE;
  const int mode = overlap_mode();
  a.prefetch_before_wait = (mode == 2) ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((a.N + 127) / 128), (unsigned)g.SK, 1);
  cfg.blockDim = dim3(32 * (kGemvMaxConsumers + 1), 1, 1);
  cfg.dynamicSmemBytes = (size_t)a.L.total;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = 1;
  attrs[na].val.clusterDim.y = (unsigned)g.SK;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  if (mode >= 1) {
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  return BQ_OK;
}

// Stage width: 256 columns at 4 bits, 512 at 2 bits; a mixed matrix uses
// 512-column splits so that both widths tile every CTA's slice.
template <int XT, int BITS, int G, bool MIXED, bool S16 = false>
bq_status launch_gemv_dispatch(const GemvArgs &a, cudaStream_t st) {
  const int split_unit = MIXED ? 512 : StageG<BITS, G>::SC;
  if (a.K % split_unit) return BQ_ERR_SHAPE;
  const int G_min = MIXED ? 64 : G;
  GemvGeom g = gemv_geometry(a.M, a.N, a.K, split_unit, G_min);
  if (g.NB == 1) return launch_gemv_t<XT, BITS, G, 1, MIXED, S16>(g, a, G_min, st);
  return launch_gemv_t<XT, BITS, G, 2, MIXED, S16>(g, a, G_min, st);
}

// s16: binary16 scales (uniform INT4 g128 or INT2 g64 only).
template <int XT>
bq_status gemv_dispatch(const uint16_t *x, int M, int64_t K, const uint8_t *packed, const void *scales, bool s16,
                        const uint8_t *zeros, const uint8_t *bit_map, int bits, int group, int64_t N, uint16_t *y,
                        cudaStream_t st) {
  GemvArgs a = {};
  a.x = x;
  a.packed = packed;
  a.scales = scales;
  a.zeros = zeros;
  a.bit_map = bit_map;
  a.y = y;
  a.K = K;
  a.N = N;
  a.M = M;
  if (s16) {
    if (bit_map) return BQ_ERR_UNSUPPORTED;
    if (bits == 4 && group == 128) return launch_gemv_dispatch<XT, 4, 128, false, true>(a, st);
    if (bits == 2 && group == 64) return launch_gemv_dispatch<XT, 2, 64, false, true>(a, st);
    return BQ_ERR_UNSUPPORTED;
  }
  if (bit_map) return launch_gemv_dispatch<XT, 4, 128, true>(a, st);
#define BQ_GV(B, G_) \
  if (bits == B && group == G_) return launch_gemv_dispatch<XT, B, G_, false>(a, st);
  BQ_GV(4, 128) BQ_GV(2, 64) BQ_GV(4, 32) BQ_GV(4, 64) BQ_GV(4, 256) BQ_GV(2, 32) BQ_GV(2, 128) BQ_GV(2, 256)
#undef BQ_GV
  return BQ_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// input gradient (M <= 16 per pass) geometry and dispatch
// ---------------------------------------------------------------------------

struct GradGeom {
  int NB, d, stages;
};

// Cluster size d (CTAs splitting the rows of one 128-column slice, at most 8
// and at most one per 128-row block): enough CTAs for two per SM; the ring
// as deep as two CTAs per SM allow.
GradGeom grad_geometry(int M, int64_t N, int64_t K, int gmax) {
  GradGeom g;
  g.NB = (M <= 8) ? 1 : 2;
  const int64_t slices = K / kGradSlice, nbk = (N + 127) / 128;
  int64_t d = (2 * sm_count()) / (slices > 0 ? slices : 1);
  if (d > 8) d = 8;
  if (d > nbk) d = nbk;
  if (d < 1) d = 1;
  g.d = (int)d;
  g.stages = 2;
  for (int s = kGradMaxStages; s >= 2; --s)
    if (grad_smem_layout(M, 8 * g.NB, gmax, s, g.d).total <= kTwoCtaSmem) {
      g.stages = s;
      break;
    }
  return g;
}

template <int XT, int BITS, int G, int NB, bool MIXED = false>
bq_status launch_grad_t(const GradGeom &g, GradArgs a, cudaStream_t st) {
  auto kern = grad_input_kernel<XT, BITS, G, NB, MIXED>;
  if (!ensure_smem<grad_input_kernel<XT, BITS, G, NB, MIXED>>(kMaxSmem)) return BQ_ERR_CUDA;
  // metadata groups per 128-column slice: a width map's 2-bit blocks have two
  constexpr int gmax = MIXED ? 2 : ((G <= kGradSlice) ? kGradSlice / G : 1);
  a.stages = g.stages;
  a.L = grad_smem_layout(a.M, 8 * NB, gmax, g.stages, g.d);
  if (a.L.total > kMaxSmem) return BQ_ERR_SHAPE;
  const int mode = overlap_mode();
  a.prefetch_before_wait = (mode == 2) ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.K / kGradSlice), (unsigned)g.d, 1);
  cfg.blockDim = dim3(32 * (kGradWarps + 1), 1, 1);
  cfg.dynamicSmemBytes = (size_t)a.L.total;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = 1;
  attrs[na].val.clusterDim.y = (unsigned)g.d;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  if (mode >= 1) {
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  return BQ_OK;
}

template <int XT>
bq_status grad_dispatch(const uint16_t *dy, int M, int64_t N, const uint8_t *packed, const float *scales,
                        const uint8_t *zeros, const uint8_t *bit_map, int bits, int group, int64_t K, uint16_t *dx,
                        cudaStream_t st) {
  GradArgs a = {};
  a.dy = dy;
  a.packed = packed;
  a.scales = scales;
  a.zeros = zeros;
  a.bit_map = bit_map;
  a.dx = dx;
  a.N = N;
  a.K = K;
  a.M = M;
  if (bit_map) {  // width map: the 4-bit kernel with per-block widths
    const GradGeom g = grad_geometry(M, N, K, 2);
    return g.NB == 1 ? launch_grad_t<XT, 4, 128, 1, true>(g, a, st) : launch_grad_t<XT, 4, 128, 2, true>(g, a, st);
  }
#define BQ_GD(B, G_)                                                                  \
  if (bits == B && group == G_) {                                                     \
    const GradGeom g = grad_geometry(M, N, K, (G_ <= kGradSlice) ? kGradSlice / G_ : 1); \
    return g.NB == 1 ? launch_grad_t<XT, B, G_, 1>(g, a, st) : launch_grad_t<XT, B, G_, 2>(g, a, st); \
  }
  BQ_GD(4, 128) BQ_GD(2, 64) BQ_GD(4, 32) BQ_GD(4, 64) BQ_GD(4, 256) BQ_GD(2, 32) BQ_GD(2, 128) BQ_GD(2, 256)
#undef BQ_GD
  return BQ_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// prefill GEMM (tcgen05)
// ---------------------------------------------------------------------------

// Token count from which bq_linear takes the tensor-core GEMM instead of
// passes of the decode kernel over 16-token blocks.
constexpr int64_t kGemmMinTokens = 64;

// x [M, K] 16-bit row-major as a 2D tensor map: boxes of 64 columns (128 B,
// one swizzle atom) x 256 rows, 128-byte swizzle, rows past M read as zero.
bool make_x_map(CUtensorMap *map, const uint16_t *x, int64_t M, int64_t K, int xt) {
  return make_map_2d(map, x, M, K, xt == 1, 64, kGemmTokTile);
}

template <int XT, int BITS, int G, bool MIXED = false, bool S16 = false>
bq_status launch_gemm_t(const uint16_t *x, int64_t M, int64_t K, const GemmArgs &a, int SK, cudaStream_t st) {
  auto kern = gemm_kernel<XT, BITS, G, MIXED, S16>;
  // the warpgroups' setmaxnreg shares must fit in the registers the block is
  // launched with, or the raising warpgroups would wait forever (a property
  // of the compiled kernel, checked once per process)
  static std::atomic<int> regs_ok{0};  // 0 unknown, 1 ok, -1 too few
  if (regs_ok.load(std::memory_order_acquire) == 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return BQ_ERR_CUDA;
    regs_ok.store((int64_t)fa.numRegs * kGemmThreads >= (int64_t)kGemmRegsNeeded ? 1 : -1, std::memory_order_release);
  }
  if (regs_ok.load(std::memory_order_acquire) < 0) return BQ_ERR_UNSUPPORTED;
  if (!ensure_smem<gemm_kernel<XT, BITS, G, MIXED, S16>>(GemmSmem::total)) return BQ_ERR_CUDA;
  CUtensorMap map;
  if (!make_x_map(&map, x, M, K, XT)) return BQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  const unsigned tiles_x = (unsigned)(a.N / kGemmRowTile), tiles_y = (unsigned)((M + kGemmTokTile - 1) / kGemmTokTile);
  if (SK > 1 && cudaMemsetAsync(a.ws_ctr, 0, (size_t)tiles_x * tiles_y * sizeof(unsigned), st) != cudaSuccess)
    return BQ_ERR_CUDA;
  cfg.gridDim = dim3(tiles_x, tiles_y, (unsigned)SK);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)GemmSmem::total;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  int na = 0;
  if (overlap_mode() >= 1) {
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, map, a);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  return BQ_OK;
}

// N a multiple of 128 (whole blocks), groups a multiple of 64 columns (a
// width map's groups 128 and 64 are), at least kGemmMinTokens tokens.
bool gemm_eligible(int64_t M, int64_t N, const uint8_t *bit_map, int group) {
  return M >= kGemmMinTokens && N % kGemmRowTile == 0 && (bit_map || group % kGemmChunk == 0) &&
         M <= 65535LL * kGemmTokTile;
}

// Split-K plan of the tensor-core kernel: when the output tiles (128 rows x
// 256 tokens) fill fewer than half of the SMs, SK CTAs share each tile, each
// a K range of whole code stages (256 columns at 4 bits, 512 at 2 bits or
// under a width map), so that tiles x SK fills one wave (SK <= 8).  The
// partial tiles and per-tile counters live in the caller's workspace.
struct GemmSplit {
  int SK, unit;
  int64_t tiles;
  size_t part_bytes, bytes;
};

GemmSplit gemm_split_plan(int64_t M, int64_t N, int64_t K, int bits, bool mixed) {
  GemmSplit p;
  p.unit = (mixed || bits == 2) ? 512 : 256;
  p.tiles = (N / kGemmRowTile) * ((M + kGemmTokTile - 1) / kGemmTokTile);
  const int64_t sms = sm_count();
  int64_t sk = (p.tiles > 0) ? sms / p.tiles : 1;
  if (sk > 8) sk = 8;
  if (sk > K / p.unit) sk = K / p.unit;
  if (2 * p.tiles > sms || sk < 2 || K % p.unit) sk = 1;
  p.SK = (int)sk;
  p.part_bytes = (size_t)p.tiles * sk * kGemmTokTile * kGemmRowTile * sizeof(float);
  p.bytes = (p.SK > 1) ? p.part_bytes + (size_t)p.tiles * sizeof(unsigned) : 0;
  return p;
}

template <int XT>
bq_status gemm_dispatch(const uint16_t *x, int64_t M, int64_t K, const uint8_t *packed, const void *scales, bool s16,
                        const uint8_t *zeros, const uint8_t *bit_map, int bits, int group, int64_t N, uint16_t *y,
                        void *workspace, size_t workspace_bytes, cudaStream_t st) {
  GemmArgs a = {};
  a.packed = packed;
  a.scales = scales;
  a.zeros = zeros;
  a.bit_map = bit_map;
  a.y = y;
  a.M = M;
  a.K = K;
  a.N = N;
  const GemmSplit sp = gemm_split_plan(M, N, K, bits, bit_map != nullptr);
  int SK = 1;
  if (sp.SK > 1 && workspace && workspace_bytes >= sp.bytes) {
    SK = sp.SK;
    a.ws_part = reinterpret_cast<float *>(workspace);
    a.ws_ctr = reinterpret_cast<unsigned *>(reinterpret_cast<char *>(workspace) + sp.part_bytes);
    a.split_unit = sp.unit;
  }
  if (s16) {
    if (bit_map) return BQ_ERR_UNSUPPORTED;
    if (bits == 4 && group == 128) return launch_gemm_t<XT, 4, 128, false, true>(x, M, K, a, SK, st);
    if (bits == 2 && group == 64) return launch_gemm_t<XT, 2, 64, false, true>(x, M, K, a, SK, st);
    return BQ_ERR_UNSUPPORTED;
  }
  if (bit_map) return launch_gemm_t<XT, 4, 128, true>(x, M, K, a, SK, st);
#define BQ_GM(B, G_) \
  if (bits == B && group == G_) return launch_gemm_t<XT, B, G_>(x, M, K, a, SK, st);
  BQ_GM(4, 128) BQ_GM(2, 64) BQ_GM(4, 64) BQ_GM(4, 256) BQ_GM(2, 128) BQ_GM(2, 256)
#undef BQ_GM
  return BQ_ERR_UNSUPPORTED;
}

bool linear_group_ok(int bits, int g) {
  (void)bits;
  return g == 32 || g == 64 || g == 128 || g == 256;
}

// bq_quantize / bq_quantize_symmetric / bq_quantize_f16s: the same
// validation and layouts, SCHEME 0 asymmetric MinMax, 1 symmetric abs-max,
// 2 asymmetric MinMax with binary16 scales.
template <int SCHEME>
bq_status quantize_any(const void *W, bq_dtype wtype, int64_t rows, int64_t cols, int bits, int group,
                       bq_layout layout, void *packed, void *scales, uint8_t *zeros, void *stream) {
  if (rows < 0 || cols < 0) return BQ_ERR_SHAPE;
  if (!valid_bits(bits) || (wtype != BQ_F16 && wtype != BQ_BF16)) return BQ_ERR_UNSUPPORTED;
  if (layout != BQ_LAYOUT_CANONICAL && layout != BQ_LAYOUT_INTERLEAVED) return BQ_ERR_UNSUPPORTED;
  if (layout == BQ_LAYOUT_CANONICAL ? !canonical_group_ok(group) : !tiled_group_ok(group)) return BQ_ERR_UNSUPPORTED;
  if (cols % group) return BQ_ERR_SHAPE;
  if (layout == BQ_LAYOUT_CANONICAL) {
    if ((cols * bits) % 32) return BQ_ERR_SHAPE;
  } else {
    const int64_t U = group > tile_width(bits) ? group : tile_width(bits);
    if (rows % 16 || cols % U) return BQ_ERR_SHAPE;
  }
  if (rows == 0 || cols == 0) return BQ_OK;
  if (!W || !packed || !scales || !zeros) return BQ_ERR_NULL;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(scales, SCHEME == 2 ? 2 : 4)) return BQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t *w = reinterpret_cast<const uint16_t *>(W);
  uint8_t *pk = reinterpret_cast<uint8_t *>(packed);
  if (layout == BQ_LAYOUT_CANONICAL) {
    const int64_t elems = rows * cols;
    if (wtype == BQ_F16) return bits == 4 ? quantize_canonical<0, 4, SCHEME>(w, elems, group, pk, scales, zeros, st)
                                          : quantize_canonical<0, 2, SCHEME>(w, elems, group, pk, scales, zeros, st);
    return bits == 4 ? quantize_canonical<1, 4, SCHEME>(w, elems, group, pk, scales, zeros, st)
                     : quantize_canonical<1, 2, SCHEME>(w, elems, group, pk, scales, zeros, st);
  }
  if (wtype == BQ_F16) return bits == 4 ? quantize_tiled<0, 4, SCHEME>(w, rows, cols, group, pk, scales, zeros, st)
                                        : quantize_tiled<0, 2, SCHEME>(w, rows, cols, group, pk, scales, zeros, st);
  return bits == 4 ? quantize_tiled<1, 4, SCHEME>(w, rows, cols, group, pk, scales, zeros, st)
                   : quantize_tiled<1, 2, SCHEME>(w, rows, cols, group, pk, scales, zeros, st);
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================

extern "C" {

const char *bq_version(void) { return "bq 0.1 (sm_100a)"; }

const char *bq_status_string(bq_status s) {
  switch (s) {
    case BQ_OK: return "BQ_OK";
    case BQ_ERR_NULL: return "BQ_ERR_NULL: a required pointer is NULL";
    case BQ_ERR_SHAPE: return "BQ_ERR_SHAPE: sizes inconsistent or not tile multiples";
    case BQ_ERR_ALIGN: return "BQ_ERR_ALIGN: pointer not aligned as required";
    case BQ_ERR_UNSUPPORTED: return "BQ_ERR_UNSUPPORTED: bits/group/layout/dtype not supported";
    case BQ_ERR_WORKSPACE: return "BQ_ERR_WORKSPACE";
    case BQ_ERR_NONFINITE: return "BQ_ERR_NONFINITE: non-finite weight or overflowing scale";
    case BQ_ERR_TIMEOUT: return "BQ_ERR_TIMEOUT: a bounded wait in a kernel gave up";
    case BQ_ERR_CUDA: return "BQ_ERR_CUDA: CUDA runtime error";
  }
  return "unknown bq_status";
}

size_t bq_packed_bytes(int64_t rows, int64_t cols, int bits) {
  if (rows < 0 || cols < 0 || !valid_bits(bits)) return 0;
  return (size_t)(rows * cols * bits / 8);
}

size_t bq_group_count(int64_t rows, int64_t cols, int group) {
  if (rows < 0 || cols < 0 || group <= 0 || cols % group) return 0;
  return (size_t)(rows * (cols / group));
}

bq_status bq_mixed_offsets(const uint8_t *bit_map, int64_t rows, int64_t cols, int64_t *code_off,
                           int64_t *group_off) {
  if (!bit_map || !code_off || !group_off) return BQ_ERR_NULL;
  if (rows < 0 || cols < 0 || rows % 128) return BQ_ERR_SHAPE;
  const int64_t nb = rows / 128;
  code_off[0] = 0;
  group_off[0] = 0;
  for (int64_t i = 0; i < nb; ++i) {
    const int b = bit_map[i];
    if (!valid_bits(b)) return BQ_ERR_UNSUPPORTED;
    const int g = (b == 4) ? 128 : 64;
    if (cols % g) return BQ_ERR_SHAPE;
    code_off[i + 1] = code_off[i] + 128 * cols * b / 8;
    group_off[i + 1] = group_off[i] + 128 * (cols / g);
  }
  return BQ_OK;
}

bq_status bq_quantize(const void *W, bq_dtype wtype, int64_t rows, int64_t cols, int bits, int group,
                      bq_layout layout, void *packed, float *scales, uint8_t *zeros, void *stream) {
  return quantize_any<0>(W, wtype, rows, cols, bits, group, layout, packed, scales, zeros, stream);
}

bq_status bq_quantize_symmetric(const void *W, bq_dtype wtype, int64_t rows, int64_t cols, int bits, int group,
                                bq_layout layout, void *packed, float *scales, uint8_t *zeros, void *stream) {
  return quantize_any<1>(W, wtype, rows, cols, bits, group, layout, packed, scales, zeros, stream);
}

bq_status bq_quantize_f16s(const void *W, bq_dtype wtype, int64_t rows, int64_t cols, int bits, int group,
                           bq_layout layout, void *packed, uint16_t *scales, uint8_t *zeros, void *stream) {
  if (!((bits == 4 && group == 128) || (bits == 2 && group == 64))) return BQ_ERR_UNSUPPORTED;
  return quantize_any<2>(W, wtype, rows, cols, bits, group, layout, packed, scales, zeros, stream);
}

bq_status bq_quantize_mixed(const void *W, bq_dtype wtype, int64_t rows, int64_t cols, const uint8_t *bit_map,
                            bq_layout layout, void *packed, float *scales, uint8_t *zeros, void *stream) {
  if (rows < 0 || cols < 0) return BQ_ERR_SHAPE;
  if (wtype != BQ_F16 && wtype != BQ_BF16) return BQ_ERR_UNSUPPORTED;
  if (layout != BQ_LAYOUT_CANONICAL && layout != BQ_LAYOUT_INTERLEAVED) return BQ_ERR_UNSUPPORTED;
  if (rows % 128) return BQ_ERR_SHAPE;
  if (cols % (layout == BQ_LAYOUT_CANONICAL ? 256 : 128)) return BQ_ERR_SHAPE;
  if (rows == 0 || cols == 0) return BQ_OK;
  if (!W || !bit_map || !packed || !scales || !zeros) return BQ_ERR_NULL;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(scales, 4)) return BQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t *w = reinterpret_cast<const uint16_t *>(W);
  uint8_t *pk = reinterpret_cast<uint8_t *>(packed);
  if (layout == BQ_LAYOUT_INTERLEAVED) {
    const int64_t grid = grid_for((rows / 16) * (cols / 128));
    if (wtype == BQ_F16) quantize_mixed_tiled_kernel<0><<<grid, kThreads, 0, st>>>(w, rows, cols, bit_map, pk, scales, zeros);
    else quantize_mixed_tiled_kernel<1><<<grid, kThreads, 0, st>>>(w, rows, cols, bit_map, pk, scales, zeros);
  } else {
    const int64_t grid = grid_for(rows * (cols / 256));
    if (wtype == BQ_F16) quantize_mixed_canonical_kernel<0><<<grid, kThreads, 0, st>>>(w, rows, cols, bit_map, pk, scales, zeros);
    else quantize_mixed_canonical_kernel<1><<<grid, kThreads, 0, st>>>(w, rows, cols, bit_map, pk, scales, zeros);
  }
  return launch_status();
}

bq_status bq_dequantize(const void *packed, const float *scales, const uint8_t *zeros, const uint8_t *bit_map,
                        int bits, int group, int64_t rows, int64_t cols, bq_layout layout, void *W_out,
                        bq_dtype otype, void *stream) {
  if (rows < 0 || cols < 0) return BQ_ERR_SHAPE;
  if (otype != BQ_F16 && otype != BQ_BF16 && otype != BQ_F32) return BQ_ERR_UNSUPPORTED;
  if (layout != BQ_LAYOUT_CANONICAL && layout != BQ_LAYOUT_INTERLEAVED) return BQ_ERR_UNSUPPORTED;
  if (bit_map) {
    if (rows % 128 || cols % 128) return BQ_ERR_SHAPE;
  } else {
    if (!valid_bits(bits)) return BQ_ERR_UNSUPPORTED;
    if (group <= 0 || group % 8 || cols % group) return BQ_ERR_SHAPE;
    if (layout == BQ_LAYOUT_CANONICAL) {
      if ((cols * bits) % 32) return BQ_ERR_SHAPE;
    } else {
      if (group % 16 || rows % 16 || cols % tile_width(bits)) return BQ_ERR_SHAPE;
    }
  }
  if (rows == 0 || cols == 0) return BQ_OK;
  if (!packed || !scales || !zeros || !W_out) return BQ_ERR_NULL;
  if (!aligned(packed, 16) || !aligned(W_out, 16) || !aligned(scales, 4)) return BQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint8_t *pk = reinterpret_cast<const uint8_t *>(packed);
  if (bit_map) {
    if (otype == BQ_F16) return dequant_mixed<0>(pk, scales, zeros, bit_map, rows, cols, layout, W_out, st);
    if (otype == BQ_BF16) return dequant_mixed<1>(pk, scales, zeros, bit_map, rows, cols, layout, W_out, st);
    return dequant_mixed<2>(pk, scales, zeros, bit_map, rows, cols, layout, W_out, st);
  }
  if (otype == BQ_F16) return dequant_uniform<0>(pk, scales, zeros, bits, group, rows, cols, layout, W_out, st);
  if (otype == BQ_BF16) return dequant_uniform<1>(pk, scales, zeros, bits, group, rows, cols, layout, W_out, st);
  return dequant_uniform<2>(pk, scales, zeros, bits, group, rows, cols, layout, W_out, st);
}

bq_status bq_fake_quantize(const void *W, bq_dtype wtype, int64_t rows, int64_t cols, int bits, int group,
                           void *W_out, bq_dtype otype, void *stream) {
  if (rows < 0 || cols < 0) return BQ_ERR_SHAPE;
  if (wtype != BQ_F16 && wtype != BQ_BF16) return BQ_ERR_UNSUPPORTED;
  if (otype != BQ_F16 && otype != BQ_BF16 && otype != BQ_F32) return BQ_ERR_UNSUPPORTED;
  if (!valid_bits(bits) || !canonical_group_ok(group)) return BQ_ERR_UNSUPPORTED;
  if (cols % group) return BQ_ERR_SHAPE;
  if (rows == 0 || cols == 0) return BQ_OK;
  if (!W || !W_out) return BQ_ERR_NULL;
  if (!aligned(W, 16) || !aligned(W_out, 16)) return BQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t *w = reinterpret_cast<const uint16_t *>(W);
  const int64_t elems = rows * cols;
  if (wtype == BQ_F16) {
    if (otype == BQ_F16) return fake_quant_bits<0, 0>(w, elems, bits, group, W_out, st);
    if (otype == BQ_BF16) return fake_quant_bits<0, 1>(w, elems, bits, group, W_out, st);
    return fake_quant_bits<0, 2>(w, elems, bits, group, W_out, st);
  }
  if (otype == BQ_F16) return fake_quant_bits<1, 0>(w, elems, bits, group, W_out, st);
  if (otype == BQ_BF16) return fake_quant_bits<1, 1>(w, elems, bits, group, W_out, st);
  return fake_quant_bits<1, 2>(w, elems, bits, group, W_out, st);
}

}  // extern "C"

namespace {

// bq_linear, bq_linear_f16s and bq_linear_ws: s16 selects binary16 scales;
// a workspace lets the tensor-core kernel split K (see gemm_split_plan).
bq_status linear_any(const void *x, bq_dtype xtype, int64_t M, int64_t K, const void *packed, const void *scales,
                     bool s16, const uint8_t *zeros, const uint8_t *bit_map, int bits, int group, int64_t N,
                     bq_layout layout, void *y, void *stream, void *workspace = nullptr, size_t workspace_bytes = 0) {
  if (M < 0 || K < 0 || N < 0) return BQ_ERR_SHAPE;
  if (s16 && (bit_map || !((bits == 4 && group == 128) || (bits == 2 && group == 64)))) return BQ_ERR_UNSUPPORTED;
  if (xtype != BQ_F16 && xtype != BQ_BF16) return BQ_ERR_UNSUPPORTED;
  if (layout != BQ_LAYOUT_INTERLEAVED) return BQ_ERR_UNSUPPORTED;
  if (bit_map) {
    if (N % 128 || K % 512) return BQ_ERR_SHAPE;
  } else {
    if (!valid_bits(bits) || !linear_group_ok(bits, group)) return BQ_ERR_UNSUPPORTED;
    if (N % 16 || K % (bits == 4 ? 256 : 512)) return BQ_ERR_SHAPE;
  }
  if (M == 0 || N == 0) return BQ_OK;
  if (!y) return BQ_ERR_NULL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) {  // an empty sum: x is not read
    return cudaMemsetAsync(y, 0, (size_t)(M * N * 2), st) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
  }
  if (!x) return BQ_ERR_NULL;
  if (!packed || !scales || !zeros) return BQ_ERR_NULL;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(packed, 16) || !aligned(scales, 16) || !aligned(zeros, 16))
    return BQ_ERR_ALIGN;
  const uint16_t *xx = reinterpret_cast<const uint16_t *>(x);
  uint16_t *yy = reinterpret_cast<uint16_t *>(y);
  const uint8_t *pk = reinterpret_cast<const uint8_t *>(packed);
  if (gemm_eligible(M, N, bit_map, group))
    return (xtype == BQ_BF16)
               ? gemm_dispatch<1>(xx, M, K, pk, scales, s16, zeros, bit_map, bits, group, N, yy, workspace,
                                  workspace_bytes, st)
               : gemm_dispatch<0>(xx, M, K, pk, scales, s16, zeros, bit_map, bits, group, N, yy, workspace,
                                  workspace_bytes, st);
  // Otherwise token blocks of at most 16 go through the decode kernel.
  for (int64_t m0 = 0; m0 < M; m0 += 16) {
    const int mb = (int)((M - m0) < 16 ? (M - m0) : 16);
    bq_status s = (xtype == BQ_BF16)
                      ? gemv_dispatch<1>(xx + m0 * K, mb, K, pk, scales, s16, zeros, bit_map, bits, group, N,
                                         yy + m0 * N, st)
                      : gemv_dispatch<0>(xx + m0 * K, mb, K, pk, scales, s16, zeros, bit_map, bits, group, N,
                                         yy + m0 * N, st);
    if (s != BQ_OK) return s;
  }
  return BQ_OK;
}

}  // namespace

extern "C" {

bq_status bq_linear(const void *x, bq_dtype xtype, int64_t M, int64_t K, const void *packed, const float *scales,
                    const uint8_t *zeros, const uint8_t *bit_map, int bits, int group, int64_t N,
                    bq_layout layout, void *y, void *stream) {
  return linear_any(x, xtype, M, K, packed, scales, false, zeros, bit_map, bits, group, N, layout, y, stream);
}

bq_status bq_linear_f16s(const void *x, bq_dtype xtype, int64_t M, int64_t K, const void *packed,
                         const uint16_t *scales, const uint8_t *zeros, int bits, int group, int64_t N,
                         bq_layout layout, void *y, void *stream) {
  return linear_any(x, xtype, M, K, packed, scales, true, zeros, nullptr, bits, group, N, layout, y, stream);
}

size_t bq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int mixed) {
  if (M < kGemmMinTokens || N <= 0 || K <= 0 || N % kGemmRowTile) return 0;
  return gemm_split_plan(M, N, K, bits, mixed != 0).bytes;
}

bq_status bq_linear_ws(const void *x, bq_dtype xtype, int64_t M, int64_t K, const void *packed, const float *scales,
                       const uint8_t *zeros, const uint8_t *bit_map, int bits, int group, int64_t N,
                       bq_layout layout, void *y, void *workspace, size_t workspace_bytes, void *stream) {
  if (workspace && !aligned(workspace, 256)) return BQ_ERR_ALIGN;
  return linear_any(x, xtype, M, K, packed, scales, false, zeros, bit_map, bits, group, N, layout, y, stream,
                    workspace, workspace_bytes);
}

bq_status bq_linear_grad_input(const void *dy, bq_dtype dtype, int64_t M, int64_t N, const void *packed,
                               const float *scales, const uint8_t *zeros, const uint8_t *bit_map, int bits,
                               int group, int64_t K, bq_layout layout, void *dx, void *stream) {
  if (M < 0 || K < 0 || N < 0) return BQ_ERR_SHAPE;
  if (dtype != BQ_F16 && dtype != BQ_BF16) return BQ_ERR_UNSUPPORTED;
  if (layout != BQ_LAYOUT_INTERLEAVED) return BQ_ERR_UNSUPPORTED;
  if (bit_map) {
    if (N % 128 || K % kGradSlice) return BQ_ERR_SHAPE;
  } else {
    if (!valid_bits(bits) || !linear_group_ok(bits, group)) return BQ_ERR_UNSUPPORTED;
    if (N % 16 || K % kGradSlice || K % group) return BQ_ERR_SHAPE;
  }
  if (M == 0 || K == 0) return BQ_OK;
  if (!dx) return BQ_ERR_NULL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (N == 0) {  // an empty sum: dy and W are not read
    return cudaMemsetAsync(dx, 0, (size_t)(M * K * 2), st) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
  }
  if (!dy || !packed || !scales || !zeros) return BQ_ERR_NULL;
  if (!aligned(dy, 16) || !aligned(dx, 16) || !aligned(packed, 16) || !aligned(scales, 16) || !aligned(zeros, 16))
    return BQ_ERR_ALIGN;
  const uint16_t *g = reinterpret_cast<const uint16_t *>(dy);
  uint16_t *out = reinterpret_cast<uint16_t *>(dx);
  const uint8_t *pk = reinterpret_cast<const uint8_t *>(packed);
  for (int64_t m0 = 0; m0 < M; m0 += 16) {
    const int mb = (int)((M - m0) < 16 ? (M - m0) : 16);
    bq_status s = (dtype == BQ_BF16)
                      ? grad_dispatch<1>(g + m0 * N, mb, N, pk, scales, zeros, bit_map, bits, group, K, out + m0 * K, st)
                      : grad_dispatch<0>(g + m0 * N, mb, N, pk, scales, zeros, bit_map, bits, group, K, out + m0 * K,
                                         st);
    if (s != BQ_OK) return s;
  }
  return BQ_OK;
}

bq_status bq_check_division(uint32_t s_bits_begin, uint32_t s_bits_end, int refinements,
                            unsigned long long *result, void *stream) {
  if (!result) return BQ_ERR_NULL;
  if (s_bits_end <= s_bits_begin) return BQ_ERR_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t grid = sm_count() * 8;
  if (refinements == 1) check_division_kernel<1><<<grid, kThreads, 0, st>>>(s_bits_begin, s_bits_end, result);
  else if (refinements == 2) check_division_kernel<2><<<grid, kThreads, 0, st>>>(s_bits_begin, s_bits_end, result);
  else return BQ_ERR_UNSUPPORTED;
  return launch_status();
}

bq_status bq_check_const_division(int divisor, uint32_t x_bits_begin, uint32_t x_bits_end,
                                  unsigned long long *result, void *stream) {
  if (!result) return BQ_ERR_NULL;
  if (x_bits_end <= x_bits_begin) return BQ_ERR_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t grid = sm_count() * 8;
  if (divisor == 15) check_const_division_kernel<15><<<grid, kThreads, 0, st>>>(x_bits_begin, x_bits_end, result);
  else if (divisor == 7) check_const_division_kernel<7><<<grid, kThreads, 0, st>>>(x_bits_begin, x_bits_end, result);
  else if (divisor == 3) check_const_division_kernel<3><<<grid, kThreads, 0, st>>>(x_bits_begin, x_bits_end, result);
  else return BQ_ERR_UNSUPPORTED;
  return launch_status();
}

bq_status bq_selftest_bounded_wait(uint32_t limit, void *stream) {
  if (limit < 1 || limit > (1u << 20)) return BQ_ERR_UNSUPPORTED;
  bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit);
  return launch_status();
}

bq_status bq_set_option(int option, int value) {
  if (option == BQ_OPT_LINEAR_OVERLAP) {
    if (value < 0 || value > 2) return BQ_ERR_UNSUPPORTED;
    g_overlap_mode.store(value);
    return BQ_OK;
  }
  return BQ_ERR_UNSUPPORTED;
}

int bq_get_option(int option) {
  if (option == BQ_OPT_LINEAR_OVERLAP) return overlap_mode();
  return -1;
}

bq_status bq_device_status(void *stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return BQ_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_bq_status, sizeof(v)) != cudaSuccess) return BQ_ERR_CUDA;
  if (v) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_bq_status, &zero, sizeof(zero)) != cudaSuccess) return BQ_ERR_CUDA;
  }
  if (v & BQ_FLAG_NONFINITE) return BQ_ERR_NONFINITE;
  if (v & BQ_FLAG_BADMAP) return BQ_ERR_UNSUPPORTED;
  if (v & BQ_FLAG_TIMEOUT) return BQ_ERR_TIMEOUT;
  return BQ_OK;
}

}  // extern "C"
