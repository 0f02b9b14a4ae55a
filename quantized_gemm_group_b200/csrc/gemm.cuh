// gemm.cuh -- prefill / training-forward weight-only linear for large M:
//   y[m, n] = sum_g s[n, g] * sum_{k in g} x[m, k] * (q[n, k] - z[n, g])
// on the 5th-generation tensor cores (tcgen05.mma, accumulators in tensor
// memory).  Same contraction as the decode kernel ("A Survey of Low-bit Large
// Language Models", section 6.2 weight-only: dequantize, then a 16-bit
// matmul); here it is a real dense contraction with M >= 2048 tokens.
//
// Tile: one 128-row block of the interleaved weight layout (MMA M = 128, the
// A operand) x 256 tokens (MMA N = 256, the B operand), the whole K range in
// chunks of 64 columns (one 128-byte swizzle atom of bf16).
// Warp roles (24 warps, 6 warpgroups):
//   warp 0      producer: x chunks by TMA (2D tensor map, 128-byte swizzle,
//               rows past M zero-filled) and the block's packed codes and
//               zeros by bulk copies (16 KB stages, contiguous in the layout)
//   warps 1-2   lane 0 issues tcgen05.mma and commits: warp 1 for the even
//               groups (TMEM buffer 0), warp 2 for the odd ones; warp 1 also
//               allocates the tensor memory
//   warp 3      idle (completes the first warpgroup)
//   warps 4-7   dequantize: exact (q - z) bf16 pairs (LOP3 + 0x4300 magic +
//               bf16x2 subtract) stored into the 128B-swizzled K-major A
//               layout, then a proxy fence and a progress word
//   warps 8-23  epilogue (4 per TMEM lane quadrant, 64 token columns each):
//               per quantization group, tcgen05.ld the group's fp32 partial
//               (one TMEM lane = one weight row, so the group's scale is one
//               scalar per thread), FMA into register accumulators, release
//               the buffer; at the end write y (transposed, bf16)
// Each group accumulates from zero in one of two TMEM buffers (2 x 256 fp32
// columns = all 512); the exact integer operand keeps bf16 exact, and the
// fp32 scale is applied outside the tensor core.
// Synchronisation.  Measured on B200: an mbarrier wait (try_wait, test_wait,
// relaxed or acquire) executed by the thread that has tcgen05.mma
// instructions outstanding stalls it for ~500 cycles behind them, while a
// plain shared-memory load does not.  So the MMA thread never waits on an
// mbarrier: the dequant warps wait for the x bytes of a stage (TMA mbarrier),
// write the A tile, and publish "chunk c is ready" in a per-warp progress
// word; the epilogue warps count their releases of each TMEM buffer in a
// per-buffer counter (a buffer's next use waits for all 16 releases of its
// previous one, so the counts are exact);
// the MMA thread polls those words with plain loads, then orders its MMAs
// after them with tcgen05.fence::after_thread_sync.  It releases stages and
// announces finished groups with tcgen05.commit onto mbarriers, which the
// other roles wait on.
// Every mbarrier wait is bounded; on expiry the kernel records
// BQ_FLAG_TIMEOUT, stops, waits (bounded) for the asynchronous work it
// issued, frees its tensor memory and returns.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace bq {

constexpr int kGemmTokTile = 256;      // MMA N
constexpr int kGemmRowTile = 128;      // MMA M (one interleaved-layout block)
constexpr int kGemmChunk = 64;         // K columns per chunk (128 B of bf16)
constexpr int kGemmXStages = 3;        // x chunk ring (32 KB each)
constexpr int kGemmAStages = 5;        // dequantized A tile ring (16 KB each)
constexpr int kGemmWStages = 2;        // packed-code ring (16 KB + zeros)
constexpr int kGemmEpiWarps = 16;
constexpr int kGemmWarpProd = 0, kGemmWarpMma = 1, kGemmWarpDeq0 = 4, kGemmWarpEpi0 = 8;
constexpr int kGemmThreads = (kGemmWarpEpi0 + kGemmEpiWarps) * 32;  // 768
// Register split (setmaxnreg, per warpgroup of 4 warps): producer / MMA
// warpgroup, dequant warpgroup, four epilogue warpgroups.  Their sum must
// not exceed what the block was launched with (threads x registers per
// thread at launch); the host checks the launch count before the first
// launch.
constexpr int kGemmRegsCtl = 56, kGemmRegsDeq = 72, kGemmRegsEpi = 88;
constexpr int kGemmRegsNeeded = 128 * kGemmRegsCtl + 128 * kGemmRegsDeq + 512 * kGemmRegsEpi;

template <int BITS, int G> struct GemmG {
  static constexpr int T = (BITS == 4) ? 64 : 128;    // tile width of the layout
  static constexpr int SC = (BITS == 4) ? 256 : 512;   // columns per 16 KB code stage
  static constexpr int CPS = SC / kGemmChunk;          // chunks per code stage
  static constexpr int GPS = SC / G;                   // groups per code stage
  static constexpr int CPG = G / kGemmChunk;           // chunks per group (>= 1)
  static_assert(G % kGemmChunk == 0, "group must be a multiple of 64 columns");
};

// Shared-memory layout (offsets from a 1024-byte aligned base).
struct GemmSmem {
  static constexpr int X_BYTES = kGemmTokTile * 128;   // 32 KB
  static constexpr int A_BYTES = kGemmRowTile * 128;   // 16 KB
  static constexpr int W_BYTES = 16384;
  static constexpr int Z_BYTES = 8 * 128;              // zeros of up to 8 groups x 128 rows
  static constexpr int x_off = 0;
  static constexpr int a_off = x_off + kGemmXStages * X_BYTES;
  static constexpr int w_off = a_off + kGemmAStages * A_BYTES;
  static constexpr int z_off = w_off + kGemmWStages * W_BYTES;
  static constexpr int bar_off = z_off + kGemmWStages * Z_BYTES;
  // barriers (GemmBars), then the TMEM address and the abort flag
  static constexpr int nbar = 2 * kGemmXStages + kGemmAStages + 2 * kGemmWStages + 4;
  static constexpr int prog_off = (bar_off + nbar * 8 + 15) & ~15;  // 4 dequant progress words (16 B)
  static constexpr int xprog_off = prog_off + 16;                    // x chunks landed
  static constexpr int epi_off = xprog_off + 4;                      // releases of TMEM buffer 0, 1
  static constexpr int tmem_off = epi_off + 8 + 4;
  static constexpr int abort_off = tmem_off + 8;
  static constexpr int last_off = abort_off + 4;       // split-K: this CTA arrived last
  static constexpr int total = abort_off + 8 + 1024;   // + alignment slack
};

struct GemmArgs {
  const uint8_t *packed;
  const void *scales;  // fp32, or binary16 when the kernel's S16 is set
  const uint8_t *zeros;
  const uint8_t *bit_map;
  uint16_t *y;
  int64_t M, K, N;
  // split-K (gridDim.z CTAs per output tile, each a K range of whole
  // `split_unit`-column units): fp32 partial tiles [tile][rank][token][row]
  // and one arrival counter per tile (zero before the launch); unused when
  // gridDim.z == 1.  Inside the roles K is the CTA's range and k0x its first
  // column in x.
  float *ws_part;
  unsigned *ws_ctr;
  int split_unit;
  int64_t k0x;
};

// Shared-memory addresses of the mbarriers.
struct GemmBars {
  uint32_t full, empty;      // [kGemmXStages]: x TMA bytes / one MMA commit
  uint32_t a_empty;          // [kGemmAStages]: one MMA commit
  uint32_t w_full, w_empty;  // [kGemmWStages]: code bytes / 4 dequant warps
  uint32_t d_full;           // [2]: one MMA commit per group
  uint32_t done;             // [2]: MMA drain of each issuer on the abort path
  BQ_DEV explicit GemmBars(uint32_t base) {
    full = base;
    empty = full + 8u * kGemmXStages;
    a_empty = empty + 8u * kGemmXStages;
    w_full = a_empty + 8u * kGemmAStages;
    w_empty = w_full + 8u * kGemmWStages;
    d_full = w_empty + 8u * kGemmWStages;
    done = d_full + 16u;
  }
};

BQ_DEV uint4 lds_volatile_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.volatile.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
BQ_DEV uint32_t lds_volatile(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
BQ_DEV void sts_release(uint32_t addr, uint32_t v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
BQ_DEV void red_release_add(uint32_t addr, uint32_t v) {
  asm volatile("red.release.cta.shared::cta.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 / TMA primitives
// ---------------------------------------------------------------------------

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row groups of
// 128-byte rows are 1024 bytes apart (stride byte offset); the leading byte
// offset is unused for this layout; version 1; layout type 2 (128B swizzle).
BQ_DEV uint64_t umma_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                  // leading byte offset (16 B, unused)
  d |= (uint64_t)(1024u >> 4) << 32;        // stride byte offset
  d |= (uint64_t)1u << 46;                  // descriptor version
  d |= (uint64_t)2u << 61;                  // 128-byte swizzle
  return d;
}

// Instruction descriptor for kind::f16: fp32 accumulate (bits 4-5 = 1), A and
// B both bf16 (bits 7-9, 10-12 = 1; XT == 1) or both fp16 (0; XT == 0), both
// K-major, N >> 3 at bit 17, M >> 4 at bit 24.
template <int XT>
constexpr uint32_t gemm_idesc() {
  return (1u << 4) | ((uint32_t)XT << 7) | ((uint32_t)XT << 10) | ((uint32_t)(kGemmTokTile >> 3) << 17) |
         ((uint32_t)(kGemmRowTile >> 4) << 24);
}

template <int XT>
BQ_DEV void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(gemm_idesc<XT>()), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
BQ_DEV void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
BQ_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
BQ_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
BQ_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16 consecutive fp32 columns of this thread's TMEM lane.
BQ_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

template <uint32_t N> BQ_DEV void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <uint32_t N> BQ_DEV void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }


// Byte offset of bf16 element (row, k) of a 128-byte-swizzled K-major tile
// (rows of 64 elements; the 16-byte chunk index is XORed with row % 8).
BQ_DEV uint32_t sw128_offset(int row, int k) {
  const int chunk = (k >> 3) ^ (row & 7);
  return (uint32_t)(row * 128 + chunk * 16 + (k & 7) * 2);
}

// ---------------------------------------------------------------------------
// roles
// ---------------------------------------------------------------------------

// Producer (one thread): every 64-column x chunk of the token tile by TMA,
// and the block's 16 KB code stages plus the zeros of their groups by bulk
// copies.  It polls both rings without blocking and issues whichever has a
// free slot; a long stretch without progress counts as a timeout.
template <int BITS, int G>
BQ_DEV void gemm_produce(const GemmArgs &a, const CUtensorMap *xmap, const uint8_t *pk, const uint8_t *ze, int tok0,
                         uint32_t sbase, const GemmBars &B, volatile int *abort) {
  using GG = GemmG<BITS, G>;
  const int nchunks = (int)(a.K / kGemmChunk);
  const int nstages = (int)(a.K / GG::SC);
  constexpr uint32_t zb = (uint32_t)(GG::GPS * 128);
  const uint32_t xprog = sbase + GemmSmem::xprog_off;
  int ci = 0, si = 0, xi = 0;  // x chunks issued, code stages issued, x chunks published
  uint32_t idle = 0;
  while (xi < nchunks || si < nstages) {
    if (*abort) break;
    bool progress = false;
    if (si < nstages) {
      const int ws = si % kGemmWStages;
      if (si < kGemmWStages || mbar_test_wait(B.w_empty + 8u * ws, ((si / kGemmWStages) & 1) ^ 1)) {
        const uint32_t full = B.w_full + 8u * ws;
        mbar_arrive_expect_tx(full, 16384u + zb);
        bulk_g2s(sbase + GemmSmem::w_off + ws * GemmSmem::W_BYTES, pk + (int64_t)si * 16384, 16384u, full);
        bulk_g2s(sbase + GemmSmem::z_off + ws * GemmSmem::Z_BYTES, ze + (int64_t)si * GG::GPS * 128, zb, full);
        ++si;
        progress = true;
      }
    }
    if (ci < nchunks) {
      const int st = ci % kGemmXStages;
      if (ci < kGemmXStages || mbar_test_wait(B.empty + 8u * st, ((ci / kGemmXStages) & 1) ^ 1)) {
        const uint32_t full = B.full + 8u * st;
        mbar_arrive_expect_tx(full, (uint32_t)GemmSmem::X_BYTES);
        tma_load_2d(sbase + GemmSmem::x_off + st * GemmSmem::X_BYTES, xmap, (int)(a.k0x + ci * kGemmChunk), tok0,
                    full);
        ++ci;
        progress = true;
      }
    }
    // publish the x chunks that have landed, in order
    if (xi < ci && mbar_test_wait(B.full + 8u * (xi % kGemmXStages), (xi / kGemmXStages) & 1)) {
      ++xi;
      sts_release(xprog, (uint32_t)xi);
      progress = true;
    }
    if (progress) {
      idle = 0;
    } else if (++idle > (kWaitLimit << 2)) {
      *abort = 1;
      bq_flag(BQ_FLAG_TIMEOUT);
      break;
    }
  }
  // the last fill of every slot has landed before the CTA may exit (only
  // waits on the abort path: otherwise the consumers took them all)
  for (int j = 1; j <= kGemmXStages && j <= ci; ++j) {
    const int c = ci - j;
    mbar_wait(B.full + 8u * (c % kGemmXStages), (c / kGemmXStages) & 1, 1u << 20);
  }
  for (int j = 1; j <= kGemmWStages && j <= si; ++j) {
    const int c = si - j;
    mbar_wait(B.w_full + 8u * (c % kGemmWStages), (c / kGemmWStages) & 1, 1u << 20);
  }
}

// Dequantize warp d (0..3): row tiles 2d, 2d+1 of every chunk.  The operand
// is (q - z) as an exact 16-bit float of x's type: bf16 128 + q (0x4300 | q)
// minus 128 + z, or fp16 1024 + q (0x6400 | q) minus 1024 + z.
template <int XT, int BITS, int G>
BQ_DEV void gemm_dequant(const GemmArgs &a, int d, int lane, uint32_t sbase, const GemmBars &B,
                         volatile int *abort) {
  const uint32_t prog = sbase + GemmSmem::prog_off + 4u * d;
  using GG = GemmG<BITS, G>;
  constexpr uint32_t MASK = (BITS == 4) ? 0x000F000Fu : 0x00030003u;
  constexpr uint32_t MAGIC = XT ? 0x4300u : 0x6400u;
  const int nchunks = (int)(a.K / kGemmChunk);
  const int r = lane >> 2, c = lane & 3;
  // byte offset, inside an A tile, of (row r of tile 2d, column 2c); the
  // 16-byte chunk j of a 128-byte swizzled row sits at (j ^ r) * 16
  const uint32_t rbase = (uint32_t)((2 * d * 16 + r) * 128 + 4 * c);
  const uint32_t rx = (uint32_t)(r << 4);
  int st = 0, ph = 0, ws = 0, wph = 0;
  for (int ci = 0; ci < nchunks; ++ci) {
    const int cin = ci % GG::CPS;  // chunk inside the code stage
    // every wait is voted on, so the whole warp leaves together
    if (!__all_sync(0xffffffffu, (*abort == 0) && (cin != 0 || mbar_wait(B.w_full + 8u * ws, wph)) &&
                                     (ci < kGemmAStages || mbar_wait(B.a_empty + 8u * st, ph ^ 1)))) {
      if (lane == 0) {
        *abort = 1;
        bq_flag(BQ_FLAG_TIMEOUT);
      }
      break;
    }
    const uint32_t wst = sbase + GemmSmem::w_off + ws * GemmSmem::W_BYTES;
    const uint32_t zst = sbase + GemmSmem::z_off + ws * GemmSmem::Z_BYTES;
    const uint32_t ast = sbase + GemmSmem::a_off + st * GemmSmem::A_BYTES;
    // column block and word range of this 64-column chunk
    const int kt = (BITS == 4) ? cin : cin / 2;
    const int run0 = (BITS == 4) ? 0 : 4 * (cin & 1);
    const int gin = (cin * kGemmChunk) / G;  // group inside the code stage
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      const int t = 2 * d + tt;
      uint4 v;
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                   : "r"(wst + (kt * 8 + t) * 512 + lane * 16));
      const uint32_t words[4] = {v.x, v.y, v.z, v.w};
      uint32_t z0, z1;
      asm volatile("ld.shared.u8 %0, [%1];" : "=r"(z0) : "r"(zst + gin * 128 + t * 16 + r));
      asm volatile("ld.shared.u8 %0, [%1];" : "=r"(z1) : "r"(zst + gin * 128 + t * 16 + r + 8));
      const uint32_t zz0 = (MAGIC | z0) * 0x10001u, zz1 = (MAGIC | z1) * 0x10001u;
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {  // 16-column runs of the chunk
        const int run = run0 + rr;
        const uint32_t w = words[BITS == 4 ? run : run / 2];
        const int base = (BITS == 4) ? 0 : 4 * (run & 1);
#pragma unroll
        for (int si = 0; si < 4; ++si) {
          // slot si: row r (+8 if si odd), columns 2c, 2c+1 (+8 if si >= 2)
          const uint32_t p = ((w >> (BITS * (base + si))) & MASK) | (MAGIC * 0x10001u);
          uint32_t val;
          if (XT)
            asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(val) : "r"(p), "r"((si & 1) ? zz1 : zz0));
          else
            asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(val) : "r"(p), "r"((si & 1) ? zz1 : zz0));
          const uint32_t addr = ast + rbase + (((uint32_t)(2 * rr + (si >> 1)) << 4) ^ rx) +
                                (uint32_t)(tt * 16 * 128 + (si & 1) * 8 * 128);
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(val) : "memory");
        }
      }
    }
    fence_proxy_async_smem();  // generic-proxy stores -> tensor-core reads
    __syncwarp();
    if (lane == 0) sts_release(prog, (uint32_t)(ci + 1));
    if (cin == GG::CPS - 1) {
      if (lane == 0) mbar_arrive(B.w_empty + 8u * ws);
      if (++ws == kGemmWStages) { ws = 0; wph ^= 1; }
    }
    if (++st == kGemmAStages) { st = 0; ph ^= 1; }
  }
}

// MMA issuers: two threads (lane 0 of warps 1 and 2); issuer `which` owns
// the groups g with g % 2 == which, i.e. TMEM buffer `which`.  Measured on
// B200: any shared-memory load (or mbarrier wait) by a thread with
// tcgen05.mma outstanding returns only after those MMAs have completed, so a
// single issuer leaves the tensor core idle for ~600 cycles at every
// readiness check; with two issuers on independent accumulators, one
// issuer's MMAs run while the other waits.  Before chunk c the issuer polls
// (plain shared loads) until every dequant warp and the x producer have
// published c as ready and, when c starts a group g >= 2, until the epilogue
// has released group g - 2's buffer.
template <int XT, int BITS, int G>
BQ_DEV void gemm_mma(const GemmArgs &a, int which, uint32_t tmem, uint32_t sbase, const GemmBars &B,
                     volatile int *abort) {
  using GG = GemmG<BITS, G>;
  const int ngroups = (int)(a.K / G);
  const uint32_t prog = sbase + GemmSmem::prog_off, xprog = sbase + GemmSmem::xprog_off;
  const uint32_t epi = sbase + GemmSmem::epi_off;
  const uint32_t d_tmem = tmem + (uint32_t)(which * kGemmTokTile);
  constexpr uint32_t kSpinLimit = kWaitLimit << 4;
  for (int g = which; g < ngroups; g += 2) {
    for (int cig = 0; cig < GG::CPG; ++cig) {
      const int ci = g * GG::CPG + cig;
      const int xs = ci % kGemmXStages, as = ci % kGemmAStages;
      // readiness of chunk ci
      bool ok = true;
      for (uint32_t spin = 0;; ++spin) {
        const uint4 p = lds_volatile_v4(prog);
        const uint32_t need = (uint32_t)ci;
        bool ready = p.x > need && p.y > need && p.z > need && p.w > need && lds_volatile(xprog) > need;
        // buffer `which` was last used by group g - 2: all its releases counted
        if (ready && cig == 0 && g >= 2) ready = lds_volatile(epi + 4u * which) >= (uint32_t)(kGemmEpiWarps * (g >> 1));
        if (ready) break;
        if (spin > kSpinLimit || *abort) { ok = false; break; }
      }
      if (!ok) {
        if (!*abort) bq_flag(BQ_FLAG_TIMEOUT);
        *abort = 1;
        return;
      }
      tc_fence_after();
      const uint32_t abase = sbase + GemmSmem::a_off + as * GemmSmem::A_BYTES;
      const uint32_t xbase = sbase + GemmSmem::x_off + xs * GemmSmem::X_BYTES;
#pragma unroll
      for (int kk = 0; kk < kGemmChunk / 16; ++kk)
        umma_f16<XT>(d_tmem, umma_desc_sw128(abase + kk * 32), umma_desc_sw128(xbase + kk * 32),
                     (cig > 0 || kk > 0) ? 1u : 0u);
      umma_commit(B.empty + 8u * xs);
      umma_commit(B.a_empty + 8u * as);
      if (cig == GG::CPG - 1) umma_commit(B.d_full + 8u * which);
    }
  }
}

// Epilogue warp e (0..15, warps 8-23): TMEM lanes 32 (warp % 4) .. +31 (weight rows),
// token columns 64 (e / 4) .. +63.
// One group scale from the block-major metadata: fp32, or binary16 (exact
// in fp32).
template <bool S16>
BQ_DEV float load_scale(const void *sc, int64_t i) {
  if (S16) return __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short *>(sc) + i)));
  return __ldg(reinterpret_cast<const float *>(sc) + i);
}

template <int XT, int BITS, int G, bool S16>
BQ_DEV void gemm_epilogue(const GemmArgs &a, const void *sc, int e, int warp, int lane, uint32_t tmem,
                          uint32_t sbase, const GemmBars &B, volatile int *abort, int64_t row0, int tok0) {
  const int ngroups = (int)(a.K / G);
  const uint32_t d_full = B.d_full;
  const uint32_t epi = sbase + GemmSmem::epi_off;
  const int quad = warp & 3;
  const int rloc = quad * 32 + lane;          // row inside the block = TMEM lane
  const int col0 = (e >> 2) * 64;             // token columns of this warp
  float acc[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) acc[i] = 0.0f;
  const uint32_t lane_addr = ((uint32_t)(quad * 32) << 16);
  float s_next = load_scale<S16>(sc, rloc);   // scale of group 0 (block-major metadata)
  bool ok = true;
  for (int g = 0; g < ngroups; ++g) {
    const int buf = g & 1;
    const float s = s_next;
    if (g + 1 < ngroups) s_next = load_scale<S16>(sc, (int64_t)(g + 1) * 128 + rloc);
    // tcgen05.ld below is warp-collective: the whole warp leaves together
    if (!__all_sync(0xffffffffu, mbar_wait(d_full + 8u * buf, (g >> 1) & 1))) {
      *abort = 1;
      bq_flag(BQ_FLAG_TIMEOUT);
      ok = false;
      break;
    }
    tc_fence_after();
    const float2 s2 = make_float2(s, s);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float v[16];
      tmem_ld16(tmem + lane_addr + (uint32_t)(buf * kGemmTokTile + col0 + cc * 16), v);
#pragma unroll
      for (int i = 0; i < 16; i += 2) {  // packed fp32x2 FMA: two columns per instruction
        const float2 r = __ffma2_rn(s2, make_float2(v[i], v[i + 1]), make_float2(acc[cc * 16 + i], acc[cc * 16 + i + 1]));
        acc[cc * 16 + i] = r.x;
        acc[cc * 16 + i + 1] = r.y;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) red_release_add(epi + 4u * buf, 1u);  // buffer g & 1 is free again
  }
  const int SK = (int)gridDim.z;
  // y is [M][N], token-major; this thread owns row (row0 + rloc)
  const int64_t n = row0 + rloc;
  if (SK == 1) {
    if (!ok || *abort) return;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const int64_t tok = tok0 + col0 + i;
      if (tok < a.M)
        a.y[tok * a.N + n] = XT ? __bfloat16_as_ushort(__float2bfloat16_rn(acc[i])) : __half_as_ushort(__float2half_rn(acc[i]));
    }
    return;
  }
  // Split-K: store this CTA's partial tile (token-major, so a warp's 32 rows
  // of one token are one 128-byte line), fence, and count the arrival; the
  // CTA that arrives last sums the partials in rank order and writes y.  No
  // CTA waits for another.  Every epilogue warp reaches both barriers, also
  // after a timeout (which then skips the arrival, so no CTA writes y).
  const int64_t tile = blockIdx.x + (int64_t)blockIdx.y * gridDim.x;
  const int rank = (int)blockIdx.z;
  const bool good = ok && !*abort;
  (void)rank;
  float *mine = a.ws_part + (tile * SK + rank) * (int64_t)(kGemmTokTile * kGemmRowTile);
  if (good) {
#pragma unroll
    for (int i = 0; i < 64; ++i) mine[(col0 + i) * kGemmRowTile + rloc] = acc[i];
  }
  __threadfence();
  asm volatile("bar.sync 1, %0;" ::"n"(kGemmEpiWarps * 32) : "memory");
  const uint32_t lastw = sbase + GemmSmem::last_off;
  if (e == 0 && lane == 0) {
    uint32_t is_last = 0;
    if (!*abort) is_last = (atomicAdd(a.ws_ctr + tile, 1u) == (unsigned)(SK - 1)) ? 1u : 0u;
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(lastw), "r"(is_last) : "memory");
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kGemmEpiWarps * 32) : "memory");
  uint32_t is_last;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(is_last) : "r"(lastw) : "memory");
  if (!is_last) return;
  __threadfence();
  // every rank's partial (this CTA's own included) from the workspace, in
  // rank order; the 64 loads of one rank are independent of each other
  const float *parts = a.ws_part + tile * SK * (int64_t)(kGemmTokTile * kGemmRowTile) + col0 * kGemmRowTile + rloc;
#pragma unroll
  for (int i = 0; i < 64; ++i) acc[i] = __ldcg(parts + i * kGemmRowTile);
  for (int q = 1; q < SK; ++q) {
    const float *pq = parts + (int64_t)q * (kGemmTokTile * kGemmRowTile);
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] += __ldcg(pq + i * kGemmRowTile);
  }
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const int64_t tok = tok0 + col0 + i;
    if (tok < a.M)
      a.y[tok * a.N + n] = XT ? __bfloat16_as_ushort(__float2bfloat16_rn(acc[i])) : __half_as_ushort(__float2half_rn(acc[i]));
  }
  if (e == 0 && lane == 0) a.ws_ctr[tile] = 0u;  // ready for the next call
}

// The roles of one CTA for a block of width BITS, group G.
template <int XT, int BITS, int G, bool S16>
BQ_DEV void gemm_roles(const GemmArgs &a, const CUtensorMap *xmap, const uint8_t *pk, const void *sc,
                       const uint8_t *ze, int warp, int lane, uint32_t tmem, uint32_t sbase, const GemmBars &B,
                       volatile int *abort, int64_t row0, int tok0) {
  if (warp < kGemmWarpDeq0) {
    setmaxnreg_dec<kGemmRegsCtl>();
    if (warp == kGemmWarpProd && lane == 0) gemm_produce<BITS, G>(a, xmap, pk, ze, tok0, sbase, B, abort);
    if ((warp == kGemmWarpMma || warp == kGemmWarpMma + 1) && lane == 0)
      gemm_mma<XT, BITS, G>(a, warp - kGemmWarpMma, tmem, sbase, B, abort);
  } else if (warp < kGemmWarpEpi0) {
    setmaxnreg_dec<kGemmRegsDeq>();
    gemm_dequant<XT, BITS, G>(a, warp - kGemmWarpDeq0, lane, sbase, B, abort);
  } else {
    setmaxnreg_inc<kGemmRegsEpi>();
    gemm_epilogue<XT, BITS, G, S16>(a, sc, warp - kGemmWarpEpi0, warp, lane, tmem, sbase, B, abort, row0, tok0);
  }
}

// grid = (N / 128 weight blocks, ceil(M / 256) token tiles); 768 threads;
// one CTA per SM (shared memory), all 512 TMEM columns.  MIXED: a width map
// (Layer-mix / Channel-mix) gives each 128-row block 4 bits (group 128) or 2
// bits (group 64); the CTA's block has one width, so it runs that width's
// roles, its codes and metadata found by running sums over the map (a block
// of b bits holds 16 K b code bytes and 128 K / group metadata entries).
template <int XT, int BITS, int G, bool MIXED, bool S16 = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap xmap, const GemmArgs a) {
  constexpr int SB = S16 ? 2 : 4;  // bytes per scale
  extern __shared__ __align__(1024) unsigned char gsm_raw[];
  // 1024-byte aligned base for the swizzled tiles
  const uint32_t raw = smem_u32(gsm_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char *smem = gsm_raw + (sbase - raw);
  volatile int *abort = reinterpret_cast<volatile int *>(smem + GemmSmem::abort_off);
  volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + GemmSmem::tmem_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t blk = blockIdx.x;
  const int64_t row0 = blk * kGemmRowTile;
  const int tok0 = blockIdx.y * kGemmTokTile;

  // width of this block and where its codes / metadata start
  int bits = BITS;
  const uint8_t *pk;
  const uint8_t *sc;
  const uint8_t *ze;
  if (!MIXED) {
    pk = a.packed + blk * kGemmRowTile * a.K * BITS / 8;
    sc = reinterpret_cast<const uint8_t *>(a.scales) + blk * kGemmRowTile * (a.K / G) * SB;
    ze = a.zeros + blk * kGemmRowTile * (a.K / G);
  } else {
    // every warp sums the map over the blocks before this one (shuffles)
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
    bits = a.bit_map[blk];
    pk = a.packed + sb * 16 * a.K;
    sc = reinterpret_cast<const uint8_t *>(a.scales) + sg * a.K * SB;
    ze = a.zeros + sg * a.K;
    if (bits != 4 && bits != 2) {  // the whole CTA leaves before allocating anything
      if (threadIdx.x == 0) bq_flag(BQ_FLAG_BADMAP);
      return;
    }
  }

  const GemmBars B(sbase + GemmSmem::bar_off);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmXStages; ++i) {
      mbar_init(B.full + 8u * i, 1);   // the x producer's expect_tx arrival (+ the TMA bytes)
      mbar_init(B.empty + 8u * i, 1);  // one MMA commit
    }
    for (int i = 0; i < kGemmAStages; ++i) mbar_init(B.a_empty + 8u * i, 1);  // one MMA commit
    for (int i = 0; i < kGemmWStages; ++i) {
      mbar_init(B.w_full + 8u * i, 1);
      mbar_init(B.w_empty + 8u * i, 4);   // 4 dequant warps
    }
    for (int i = 0; i < 2; ++i) mbar_init(B.d_full + 8u * i, 1);  // one MMA commit per group
    mbar_init(B.done, 1);
    mbar_init(B.done + 8u, 1);
    volatile uint32_t *words = reinterpret_cast<volatile uint32_t *>(smem + GemmSmem::prog_off);
    for (int i = 0; i < 7; ++i) words[i] = 0u;  // dequant progress, x landed, released buffers
    *abort = 0;
    mbar_fence_init();
  }
  if (warp == kGemmWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     sbase + GemmSmem::tmem_off)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // split-K: this CTA's K range, whole units of split_unit columns, and its
  // block's codes / scales / zeros from the range's first column
  GemmArgs al = a;
  if (gridDim.z > 1) {
    const int64_t SK = gridDim.z, nu = a.K / a.split_unit;
    const int64_t k0 = (blockIdx.z * nu / SK) * a.split_unit, k1 = ((blockIdx.z + 1) * nu / SK) * a.split_unit;
    const int bb = MIXED ? bits : BITS;
    const int gsz = (!MIXED || bits == BITS) ? G : 64;
    pk += k0 * 16 * bb;  // 128 rows x k0 columns x bb / 8 bytes
    sc += (k0 / gsz) * kGemmRowTile * SB;
    ze += (k0 / gsz) * kGemmRowTile;
    al.K = k1 - k0;
    al.k0x = k0;
  }
  pdl_wait();
  if (!MIXED || bits == BITS) gemm_roles<XT, BITS, G, S16>(al, &xmap, pk, sc, ze, warp, lane, tmem, sbase, B, abort, row0, tok0);
  else gemm_roles<XT, 2, 64, S16>(al, &xmap, pk, sc, ze, warp, lane, tmem, sbase, B, abort, row0, tok0);

  // everything issued by this CTA has finished before the tensor memory goes
  tc_fence_before();
  __syncthreads();
  if ((warp == kGemmWarpMma || warp == kGemmWarpMma + 1) && *abort && lane == 0) {
    // wait (bounded) for this issuer's MMAs still in flight: commit to the
    // barrier kept for this, then wait for its first phase
    const uint32_t done = B.done + 8u * (warp - kGemmWarpMma);
    umma_commit(done);
    mbar_wait(done, 0, 1u << 20);
  }
  __syncthreads();
  if (warp == kGemmWarpMma) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

}  // namespace bq
