// Device primitives for the sm_100a kernels: mbarriers with bounded waits,
// TMA tile loads (each CTA loads its own tiles), tcgen05 MMA / TMEM helpers, UMMA
// descriptors, and the tile-window geometry shared by every kernel.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vattn_internal.h"

namespace vattn {

// ---------------------------------------------------------------------------
// error word (first writer wins): the library's device status word, whose
// address reaches every kernel through DevCtl
// ---------------------------------------------------------------------------
__device__ __forceinline__ void report_error(int* word, int code) {
  if (word) atomicCAS(word, 0, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// Debug build (-DVATTN_DEBUG=1): bounds checks on the rows, tiles and TMA
// coordinates the kernels compute.  A failed check records
// VATTN_ERR_DEVICE_BOUNDS in the status word (first writer wins) and the
// caller skips the access and stops; in the default build every check is the
// constant `true` and compiles away.
// ---------------------------------------------------------------------------
#ifndef VATTN_DEBUG
#define VATTN_DEBUG 0
#endif
constexpr bool kDebugChecks = VATTN_DEBUG != 0;

__device__ __forceinline__ bool dcheck(bool ok, int* err_word) {
  if constexpr (kDebugChecks) {
    if (!ok) report_error(err_word, VATTN_ERR_DEVICE_BOUNDS);
    return ok;
  } else {
    (void)err_word;
    return true;
  }
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false when the
// CTA's abort flag is raised or the time limit runs out; in the latter case
// the caller's CTA is marked aborted and the device error word is set.
struct WaitCtx {
  volatile int* abort_flag;  // CTA-shared
  uint64_t timeout_ns;
  int* err_word;
};

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*w.abort_flag) return false;
      if (globaltimer_ns() - t0 > w.timeout_ns) {
        *w.abort_flag = 1;
        report_error(w.err_word, VATTN_ERR_DEVICE_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait that ignores the abort flag: used on the teardown path to let
// copies and MMAs already in flight finish before shared memory and TMEM are
// released.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0 && globaltimer_ns() - t0 > w.timeout_ns) {
      report_error(w.err_word, VATTN_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// TMA (tiled, 3D and 5D; every load fills only the issuing CTA's shared memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// Box coordinates (c0 innermost = head_dim element, c1 = row, c2 = batch*head).
// c0 is always a multiple of 64 elements (128 bytes) here.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// 5-D box (raster [bh][T][H][W][d] maps); coordinates innermost first.
__device__ __forceinline__ void tma_load_5d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], "
      "[%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 / TMEM
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 columns of 32-bit: thread i of the warp gets lane (base+i), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// ---------------------------------------------------------------------------
// UMMA descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor, SWIZZLE_128B, sm_100 version bits.
// start/lbo/sbo in bytes.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t start, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((start >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // layout: SWIZZLE_128B
  return d;
}
// Instruction descriptor, kind::f16, bf16 x bf16 -> f32.
// a_mn / b_mn: operand is MN-major (1) or K-major (0).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                       // D format f32
         | (1u << 7)                     // A bf16
         | (1u << 10)                    // B bf16
         | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// numeric helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Packed fp32x2 arithmetic (sm_100): two lanes per instruction.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Three-input maximum (sm_100 PTX).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA/ALU pipes instead of the MUFU unit, for x <= 64.
// Range reduction in the style of Cody and Waite: n = round-to-nearest(x) via
// the 1.5*2^23 shifter, f = x - n in [-1/2, 1/2]; 2^f by a degree-3
// polynomial whose coefficients were fitted for this library (minimax
// relative error on [-1/2, 1/2] by Lawson's iteratively reweighted least
// squares; max relative error 7.5e-5, far below the 2^-9 of the bf16 P it
// feeds); n is then added to the polynomial's exponent field.  x is clamped
// below at -125, so the smallest result is about 2^-125 instead of 0.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float j = x + 12582912.0f;
  const float n = j - 12582912.0f;
  const float f = x - n;
  float p = fmaf(0.05517166f, f, 0.24261113f);
  p = fmaf(p, f, 0.69326097f);
  p = fmaf(p, f, 0.99992806f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(j) << 23));
}

// Pack two floats to bf16x2 (round to nearest even): lo goes to the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Two floats to e4m3 (round to nearest even, saturating): lo in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));  // first operand -> upper byte
  return r;
}
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// tile-window geometry ("Fast Video Generation with Sliding Tile Attention",
// abstract: each query tile attends to a 3D window of key tiles)
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int win_start(int a, int w, int n) {
  int s = a - w / 2;
  int hi = n - w > 0 ? n - w : 0;
  s = s < 0 ? 0 : s;
  return s > hi ? hi : s;
}
__host__ __device__ __forceinline__ int win_extent(int w, int n) { return w < n ? w : n; }

// The query tiles whose window contains key tile k along one dim form a
// contiguous range [lo, hi] because the window start is non-decreasing in a.
__host__ __device__ __forceinline__ void inverse_range(int k, int w, int n, int* lo, int* hi) {
  const int e = win_extent(w, n);
  int l = n, h = -1;
  int a0 = k - w - 1 < 0 ? 0 : k - w - 1;
  int a1 = k + w + 1 > n - 1 ? n - 1 : k + w + 1;
  for (int a = a0; a <= a1; ++a) {
    const int s = win_start(a, w, n);
    if (s <= k && k < s + e) {
      l = a < l ? a : l;
      h = a > h ? a : h;
    }
  }
  *lo = l;
  *hi = h;
}

// Window of tile a along one dim for any window mode (see WIN_* in
// vattn_internal.h); ext may vary from tile to tile for the partition modes.
__host__ __device__ __forceinline__ void tile_range(int a, int w, int n, int mode, int* start, int* ext) {
  if (mode == WIN_SLIDING) {
    *start = win_start(a, w, n);
    *ext = win_extent(w, n);
    return;
  }
  const int size = mode == WIN_SHIFTED ? w + 1 : w;
  const int off = mode == WIN_SHIFTED ? (w + 1) / 2 : 0;
  const int b = (a + off) / size;
  int lo = b * size - off, hi = (b + 1) * size - off;
  lo = lo < 0 ? 0 : lo;
  hi = hi > n ? n : hi;
  *start = lo;
  *ext = hi - lo;
}

// Query tiles whose window holds key tile k along one dim, for any mode: the
// partition modes are symmetric (the block itself).
__host__ __device__ __forceinline__ void tile_inverse(int k, int w, int n, int mode, int* lo, int* hi) {
  if (mode == WIN_SLIDING) {
    inverse_range(k, w, n, lo, hi);
    return;
  }
  int s, e;
  tile_range(k, w, n, mode, &s, &e);
  *lo = s;
  *hi = s + e - 1;
}

// A box of tiles streamed as runs: for every (t, h) tile row of the box, the
// w-range of tiles is contiguous in tile-major memory.
struct TileBox {
  int t0, h0, w0;   // first tile coordinate
  int et, eh, ew;   // extent in tiles
};

// ---------------------------------------------------------------------------
// 128-row query blocks over the tile-major rows of the sliding tile.  A tile
// volume that is an odd multiple of 64 rows (192 at 1080p and 4K) would leave
// one half-empty block per tile; instead w-adjacent tiles of a tile row
// (w = 2i, 2i+1) share their blocks: k = s / 128 whole blocks of each and one
// block straddling the two (the first tile's last 64 rows, the second's first
// 64).  An odd last tile of the row takes k + 1 blocks of its own.  The
// straddling block attends to the union of the two windows, which along w
// start at most one tile apart (sliding windows); the rows of each tile mask
// the key tile outside their own window.
// ---------------------------------------------------------------------------
constexpr int PAIR_MAX_UNITS = 64;  // tiles per tile row that a unit table can describe

struct PairPlan {
  int k;    // whole 128-row blocks per tile (pairing only)
  int nw;   // tiles per tile row (Nw); 1 unpaired (each tile a row of its own)
  int np;   // pairs per tile row (Nw / 2); 0 unpaired
  int bpr;  // query blocks per tile row
  // Unit table (partition windows): units > 0 replaces the uniform pairs
  // (2i, 2i+1) by `units` units per tile row, each one tile or a pair of
  // adjacent tiles whose windows coincide (pairs never cross a partition).
  int units;
  uint8_t unit_tile[PAIR_MAX_UNITS];            // first tile (w) of the unit
  uint8_t unit_pair[PAIR_MAX_UNITS];            // 1: the unit is tiles w, w + 1
  uint16_t unit_block[PAIR_MAX_UNITS + 1];      // first query block of the unit in its row
};

// Windows of w-adjacent tiles aw, aw + 1 coincide along w (then along t and h
// too: a pair shares its tile row).
inline bool windows_coincide(const DevGeom& g, int key_nw, int aw) {
  int s0, e0, s1, e1;
  tile_range(aw, g.ww, key_nw, g.wmode, &s0, &e0);
  tile_range(aw + 1, g.ww, key_nw, g.wmode, &s1, &e1);
  return s0 == s1 && e0 == e1;
}

// key_nw: tiles of the key grid along w (the query grid's, or the coarse grid
// of the hierarchical branch).
//  - Sliding windows: uniform pairs (2i, 2i+1); a straddling block streams
//    the union of the two windows (one tile wider when they start a tile
//    apart), whose first key tile must lie in both windows, so the windows
//    need at least two tiles along w.
//  - Partition windows (cross-window attention): a pair needs its two tiles
//    in the same block, so that their windows coincide (no mask, no union).
//    When every uniform pair does (e.g. shifted blocks of 4 whose cuts fall
//    on even tiles), the uniform plan; otherwise a unit table built left to
//    right (e.g. blocks of 3: tiles 0-1 paired, 2 alone, 3-4 paired, ...).
inline PairPlan make_pair_plan(const DevGeom& g, int key_nw, bool allow) {
  PairPlan pp;
  pp.k = 0;
  pp.nw = 1;
  pp.np = 0;
  pp.bpr = (g.s + 127) / 128;
  pp.units = 0;
  if (!allow || g.s % 128 != 64 || g.Nw < 2) return pp;
  const int k = g.s / 128;
  bool uniform = false;
  if (g.wmode == WIN_SLIDING) {
    uniform = win_extent(g.ww, key_nw) >= 2;
  } else if (key_nw == g.Nw) {
    uniform = true;
    for (int aw = 0; aw + 1 < g.Nw; aw += 2) uniform = uniform && windows_coincide(g, key_nw, aw);
    if (!uniform && g.Nw <= PAIR_MAX_UNITS) {
      int u = 0, blocks = 0, pairs = 0;
      for (int aw = 0; aw < g.Nw; ++u) {
        const bool pair = aw + 1 < g.Nw && windows_coincide(g, key_nw, aw);
        pp.unit_tile[u] = (uint8_t)aw;
        pp.unit_pair[u] = pair ? 1 : 0;
        pp.unit_block[u] = (uint16_t)blocks;
        blocks += pair ? 2 * k + 1 : k + 1;
        pairs += pair ? 1 : 0;
        aw += pair ? 2 : 1;
      }
      pp.unit_block[u] = (uint16_t)blocks;
      if (pairs > 0) {
        pp.k = k;
        pp.nw = g.Nw;
        pp.units = u;
        pp.bpr = blocks;
      }
      return pp;
    }
  }
  if (uniform) {
    pp.k = k;
    pp.nw = g.Nw;
    pp.np = g.Nw / 2;
    pp.bpr = pp.np * (2 * pp.k + 1) + (g.Nw % 2) * (pp.k + 1);
  }
  return pp;
}
// The plan pairs tiles (uniform pairs or a unit table): launch the PAIR
// kernel instance with pair_plan_blocks query blocks.
inline bool pair_plan_active(const PairPlan& pp) { return pp.np > 0 || pp.units > 0; }
inline long long pair_plan_blocks(const DevGeom& g, const PairPlan& pp) {
  return (long long)(g.n_tiles / pp.nw) * pp.bpr;
}

struct QueryBlock {
  int tile;      // tile whose window the key stream starts from
  int row0;      // first row (tile-major)
  int valid;     // rows of the block that exist
  int sub;       // block within its tile (unpaired)
  int straddle;  // rows [0, 64) in tile `tile`, [64, 128) in tile `tile` + 1
};

__host__ __device__ __forceinline__ QueryBlock paired_query_block(const DevGeom& g, const PairPlan& pp, int qblk) {
  QueryBlock b;
  const int r = qblk / pp.bpr, i = qblk - r * pp.bpr;
  int a, sb;
  bool in_pair;
  if (pp.units > 0) {  // unit table: the unit holding block i of the row
    int u = 0;
    while (u + 1 < pp.units && pp.unit_block[u + 1] <= i) ++u;
    a = r * pp.nw + pp.unit_tile[u];
    sb = i - pp.unit_block[u];
    in_pair = pp.unit_pair[u] != 0;
  } else {
    // tile row r (unpaired: tile r), block i of it; pair pi (np: the row's
    // odd last tile), block sb of the pair
    const int span = 2 * pp.k + 1;
    const int pi = i / span < pp.np ? i / span : pp.np;
    a = r * pp.nw + 2 * pi;
    sb = i - pi * span;
    in_pair = pi < pp.np;
  }
  b.row0 = a * g.s + sb * 128;
  const int left = (in_pair ? 2 * g.s : g.s) - sb * 128;
  b.valid = left < 128 ? left : 128;
  b.tile = a + (in_pair && sb > pp.k ? 1 : 0);
  b.straddle = in_pair && sb == pp.k;
  b.sub = sb;
  return b;
}

// Straddling block of tiles a, a + 1: how far (0 or 1 tiles) the second
// tile's window along w starts after the first's.
__device__ __forceinline__ int straddle_shift(const DevGeom& g, int key_nw, int cfw, int a) {
  const int aw = a % g.Nw;
  int s0, e0, s1, e1;
  tile_range(aw / cfw, g.ww, key_nw, g.wmode, &s0, &e0);
  tile_range((aw + 1) / cfw, g.ww, key_nw, g.wmode, &s1, &e1);
  return s1 - s0;
}

// A straddling block over windows one tile apart streams each run of ew + 1
// key tiles from its second tile (w0 + 1, in both windows) to w0 + ew and then
// w0: run offset o -> offset in the unrotated run (tiles of s rows).
__device__ __forceinline__ int rotated_offset(int o, int s, int ew) {
  const int ti = o / s;
  return (ti < ew ? ti + 1 : 0) * s + (o - ti * s);
}

// Run offsets [x0, x0 + s) that the rows of the first tile (second = false:
// the tile w0 + ew) or of the second tile (second = true: the tile w0) do not
// see, in the rotated order.
__device__ __forceinline__ int straddle_excluded_start(int s, int ew, bool second) {
  return (second ? ew : ew - 1) * s;
}

}  // namespace vattn
