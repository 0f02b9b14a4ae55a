// gemv.cuh -- decode-path weight-only linear, M <= 16 tokens:
//   y[m, n] = sum_g s[n, g] * sum_{k in g} x[m, k] * (q[n, k] - z[n, g])
// ("A Survey of Low-bit Large Language Models", section 6.2: weight-only
// quantization dequantizes and runs a 16-bit matmul, and gains by moving
// fewer bytes; "大模型量化实战" section 3.3: dequantize and multiply inside one
// kernel so no intermediate goes back to memory).
//
// Design (HBM-bound; the weights are read exactly once):
//  * Codes use the interleaved layout: lane L's 16-byte slot of a 512-byte
//    tile is, word by word, the A operand of a 16x8x16 bf16 mma.sync for
//    rows (L/4, L/4+8) of the 16-row tile.  One LOP3 per register builds
//    (128 + q) pairs as bf16x2 (magic exponent 0x4300), one HSUB2 removes
//    (128 + z): the operand is the exact integer q - z.
//  * x^T is the B operand (8 tokens per mma; two mmas for M > 8).  A CTA
//    stages its K-slice of x once in shared memory (rows padded by 16 bytes
//    so ldmatrix is conflict-free) and reads fragments with ldmatrix.x4.
//  * Each group's products accumulate in fp32 from zero; the group's fp32
//    scale is then applied per row in an FMA into the running sum.
//  * A CTA covers 16*R rows and a K-slice; its warps split that slice
//    further; warp partials meet in shared memory.  CTAs that split K form a
//    thread-block cluster and the partials are reduced through distributed
//    shared memory in fixed rank order: deterministic, no global scratch.
//  * Tile loads for the next super-unit are issued before the current one is
//    computed (register double buffering).
#pragma once
#include <cooperative_groups.h>
#include <type_traits>

#include "common.cuh"

namespace bq {
namespace cg = cooperative_groups;

template <int XT> struct MmaT;
template <> struct MmaT<1> {  // bf16
  static constexpr uint32_t kMagic = 0x43004300u;  // bf16x2 (128, 128)
  static BQ_DEV uint32_t zpair(uint32_t z) {     // bf16x2 (128 + z, 128 + z), exact
    uint32_t h = 0x4300u | z;
    return h | (h << 16);
  }
  static BQ_DEV uint32_t sub2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&a), *reinterpret_cast<__nv_bfloat162 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
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
  static BQ_DEV uint32_t zpair(uint32_t z) {
    uint32_t h = 0x6400u | z;
    return h | (h << 16);
  }
  static BQ_DEV uint32_t sub2(uint32_t a, uint32_t b) {
    __half2 r = __hsub2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
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

// Shared-memory layout (dynamic), CTA = NWR x NWK warps covering
// ROWS = 16 * R * NWR rows and KC = NWK * KW columns:
//   xs   [8*NB][KC + 8] activations (16-bit), rows padded by 16 bytes
//   red  [NWK][8*NB][ROWS] fp32 partials of the K-slices (token-major)
//   part [8*NB][ROWS] fp32 CTA partial (token-major), read by the cluster
inline size_t gemv_smem_bytes(int NB, int R, int NWR, int NWK, int64_t KC) {
  const size_t tok = 8 * NB, rows = 16 * R * NWR;
  return tok * (KC + 8) * 2 + (size_t)NWK * tok * rows * 4 + tok * rows * 4;
}

// Body of one warp over its K range for the CTA's R row tiles.  `pk`, `sc`,
// `ze` address the matrix (or the mixed block) the rows belong to; `row0` is
// the first row relative to them and `kw0` the warp's first column.
template <int XT, int BITS, int G, int NB, int R>
BQ_DEV void gemv_warp(const uint8_t *__restrict__ pk, const float *__restrict__ sc,
                      const uint8_t *__restrict__ ze, int64_t K, int64_t row0, int64_t kw0, int64_t KW,
                      int64_t kc0, uint32_t xs_base, int xs_stride_bytes, int lane, float (&acc)[R][NB][4]) {
  using MT = MmaT<XT>;
  constexpr int T = (BITS == 4) ? 64 : 128;       // tile width
  constexpr int SU = (G > T) ? G : T;              // super-unit width
  constexpr int TILES = SU / T;
  constexpr int STEPS_PER_G = G / 16;
  constexpr int GROUPS = SU / G;
  constexpr uint32_t MASK = (BITS == 4) ? 0x000F000Fu : 0x00030003u;
  const int r = lane >> 2;
  const int64_t GK = K / G;
  const int64_t KT = K / T;

  // ldmatrix row address of this lane: token lane%8 (+8 for the second
  // block), column offset 8*(lane/8) inside a pair of k16 steps.
  const uint32_t xs_lane = xs_base + (uint32_t)((lane & 7) * xs_stride_bytes + (lane >> 3) * 16);

  const int nsu = (int)(KW / SU);
  uint4 buf[2][R][TILES];
  uint32_t zb[2][R][GROUPS][2];
  float sb[2][R][GROUPS][2];

  auto load_su = [&](int i, auto slot_c) {
    constexpr int slot = decltype(slot_c)::value;
    const int64_t col = kw0 + (int64_t)i * SU;
#pragma unroll
    for (int rb = 0; rb < R; ++rb) {
      const int64_t rt = row0 / 16 + rb;
#pragma unroll
      for (int t = 0; t < TILES; ++t)
        buf[slot][rb][t] = ld_stream_v4(pk + (rt * KT + col / T + t) * 512 + lane * 16);
#pragma unroll
      for (int gi = 0; gi < GROUPS; ++gi)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t idx = (row0 + rb * 16 + r + 8 * h) * GK + col / G + gi;
          sb[slot][rb][gi][h] = __ldg(sc + idx);
          zb[slot][rb][gi][h] = __ldg(ze + idx);
        }
    }
  };

  auto compute_su = [&](int i, auto slot_c) {
    constexpr int slot = decltype(slot_c)::value;
    const int64_t col_in_cta = kw0 - kc0 + (int64_t)i * SU;
#pragma unroll
    for (int gi = 0; gi < GROUPS; ++gi) {
      float c[R][NB][4];
      uint32_t zz[R][2];
#pragma unroll
      for (int rb = 0; rb < R; ++rb) {
        zz[rb][0] = MT::zpair(zb[slot][rb][gi][0]);
        zz[rb][1] = MT::zpair(zb[slot][rb][gi][1]);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int j = 0; j < 4; ++j) c[rb][nb][j] = 0.0f;
      }
#pragma unroll
      for (int sp = 0; sp < STEPS_PER_G; sp += 2) {  // pairs of k16 steps
        const int step0 = gi * STEPS_PER_G + sp;
        uint32_t bfr[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
          ldmatrix_x4(bfr[nb], xs_lane + (uint32_t)(nb * 8 * xs_stride_bytes) +
                                   (uint32_t)((col_in_cta + step0 * 16) * 2));
#pragma unroll
        for (int ss = 0; ss < 2; ++ss) {
          const int step = step0 + ss;
          const int t = step / (T / 16);    // tile within the super-unit
          const int run = step % (T / 16);  // 16-column run within the tile
#pragma unroll
          for (int rb = 0; rb < R; ++rb) {
            const uint4 v = buf[slot][rb][t];
            const uint32_t words[4] = {v.x, v.y, v.z, v.w};
            const uint32_t w = words[BITS == 4 ? run : run / 2];
            const int base = (BITS == 4) ? 0 : 4 * (run & 1);
            uint32_t a[4];
#pragma unroll
            for (int si = 0; si < 4; ++si) {
              const uint32_t p = and_or(w >> (BITS * (base + si)), MASK, MT::kMagic);
              a[si] = MT::sub2(p, zz[rb][si & 1]);
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) MT::mma(c[rb][nb], a, bfr[nb][2 * ss], bfr[nb][2 * ss + 1]);
          }
        }
      }
#pragma unroll
      for (int rb = 0; rb < R; ++rb) {
        const float s0 = sb[slot][rb][gi][0], s1 = sb[slot][rb][gi][1];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          acc[rb][nb][0] = __fmaf_rn(s0, c[rb][nb][0], acc[rb][nb][0]);
          acc[rb][nb][1] = __fmaf_rn(s0, c[rb][nb][1], acc[rb][nb][1]);
          acc[rb][nb][2] = __fmaf_rn(s1, c[rb][nb][2], acc[rb][nb][2]);
          acc[rb][nb][3] = __fmaf_rn(s1, c[rb][nb][3], acc[rb][nb][3]);
        }
      }
    }
  };

  using S0 = std::integral_constant<int, 0>;
  using S1 = std::integral_constant<int, 1>;
  if (nsu > 0) load_su(0, S0{});
  for (int i = 0; i < nsu; i += 2) {
    if (i + 1 < nsu) load_su(i + 1, S1{});
    compute_su(i, S0{});
    if (i + 1 < nsu) {
      if (i + 2 < nsu) load_su(i + 2, S0{});
      compute_su(i + 1, S1{});
    }
  }
}

// Kernel.  grid = (N / ROWS, S); cluster = (1, S, 1); block = NWR * NWK
// warps.  Warp w covers rows 16 R (w % NWR) .. of the CTA and the K-slice
// w / NWR.  bit_map == nullptr: uniform BITS / G.  Otherwise one width per
// 128-row block (ROWS divides 128) and the CTA runs (4, 128) or (2, 64).
template <int XT, int BITS, int G, int NB, int R, bool MIXED>
__global__ void __launch_bounds__(256)
gemv_kernel(const uint16_t *__restrict__ x, int M, int64_t K, const uint8_t *__restrict__ packed,
            const float *__restrict__ scales, const uint8_t *__restrict__ zeros,
            const uint8_t *__restrict__ bit_map, int64_t N, uint16_t *__restrict__ y, int64_t KC, int64_t KW,
            int NWR) {
  using MT = MmaT<XT>;
  extern __shared__ __align__(16) unsigned char smem[];
  const int NW = blockDim.x >> 5;
  const int NWK = NW / NWR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wr = warp % NWR, wk = warp / NWR;
  cg::cluster_group cluster = cg::this_cluster();
  const int S = (int)cluster.dim_blocks().y;
  const int rank = (int)cluster.block_rank();
  constexpr int TOK = 8 * NB;
  const int ROWS = 16 * R * NWR;
  const int64_t kc0 = (int64_t)blockIdx.y * KC;
  const int64_t row0 = (int64_t)blockIdx.x * ROWS;

  uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
  const int xs_stride = (int)(KC + 8);  // elements
  float *red = reinterpret_cast<float *>(smem + (size_t)TOK * xs_stride * 2);
  float *part = red + (size_t)NWK * TOK * ROWS;

  // Wait for the previous kernel in the stream before touching x or y
  // (programmatic dependent launch; a no-op otherwise).
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // stage x[:, kc0 : kc0 + KC] (token rows >= M are zero)
  const int64_t chunks_per_row = KC / 8;
  for (int64_t i = threadIdx.x; i < TOK * chunks_per_row; i += blockDim.x) {
    const int m = (int)(i / chunks_per_row);
    const int64_t ch = i - m * chunks_per_row;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (m < M) v = *reinterpret_cast<const uint4 *>(x + (int64_t)m * K + kc0 + ch * 8);
    *reinterpret_cast<uint4 *>(xs + (int64_t)m * xs_stride + ch * 8) = v;
  }
  __syncthreads();

  float acc[R][NB][4];
#pragma unroll
  for (int rb = 0; rb < R; ++rb)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[rb][nb][j] = 0.0f;

  const uint32_t xs_base = (uint32_t)__cvta_generic_to_shared(xs);
  const int64_t kw0 = kc0 + (int64_t)wk * KW;
  const int64_t wrow0 = row0 + (int64_t)wr * 16 * R;
  if (!MIXED) {
    gemv_warp<XT, BITS, G, NB, R>(packed, scales, zeros, K, wrow0, kw0, KW, kc0, xs_base, xs_stride * 2, lane, acc);
  } else {
    const int64_t blk = row0 / 128;
    int64_t sb = 0, sg = 0;
    for (int64_t j = lane; j < blk; j += 32) {
      const int b = bit_map[j];
      sb += b;
      sg += (b == 4) ? 1 : 2;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      sb += __shfl_xor_sync(0xffffffffu, sb, off);
      sg += __shfl_xor_sync(0xffffffffu, sg, off);
    }
    const uint8_t *pk = packed + sb * 16 * K;
    const float *sc = scales + sg * K;
    const uint8_t *ze = zeros + sg * K;
    const int bits = bit_map[blk];
    const int64_t rr0 = wrow0 - blk * 128;
    if (bits == 4) {
      gemv_warp<XT, 4, 128, NB, R>(pk, sc, ze, K, rr0, kw0, KW, kc0, xs_base, xs_stride * 2, lane, acc);
    } else if (bits == 2) {
      gemv_warp<XT, 2, 64, NB, R>(pk, sc, ze, K, rr0, kw0, KW, kc0, xs_base, xs_stride * 2, lane, acc);
    } else if (lane == 0) {
      bq_flag(BQ_FLAG_BADMAP);
    }
  }

  // warp partials -> shared (token-major), one slice per K-slice wk
  {
    const int r = lane >> 2, c = lane & 3;
    float *w = red + (size_t)wk * TOK * ROWS;
#pragma unroll
    for (int rb = 0; rb < R; ++rb)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = wr * 16 * R + rb * 16 + r + 8 * (j >> 1);
          const int tok = nb * 8 + 2 * c + (j & 1);
          w[tok * ROWS + row] = acc[rb][nb][j];
        }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < TOK * ROWS; e += blockDim.x) {
    float s = 0.0f;
    for (int q = 0; q < NWK; ++q) s += red[(size_t)q * TOK * ROWS + e];
    part[e] = s;
  }
  // every CTA of the cluster has its partial in shared memory
  cluster.sync();
  // rank q reduces a slice of the elements over all ranks, in rank order
  const int E = TOK * ROWS;
  const int per = (E + S - 1) / S;
  const int e0 = rank * per, e1 = min(E, e0 + per);
  for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    float s = 0.0f;
    for (int q = 0; q < S; ++q) s += cluster.map_shared_rank(part, q)[e];
    const int tok = e / ROWS, row = e % ROWS;
    if (tok < M) y[(int64_t)tok * N + row0 + row] = MT::out(s);
  }
  // keep every CTA's shared memory alive until all remote reads are done
  cluster.sync();
}

}  // namespace bq
