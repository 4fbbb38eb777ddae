// Definitions of the forward kernel (attn_fwd.cu): launch parameters, the key
// stream of a query block, the 5-D raster TMA load, the e4m3 tensor-core
// instructions and the debug-build bounds checks.
#pragma once

#include "common.cuh"

namespace vattn {
namespace fwd {

constexpr int BM = 128;  // query rows per block
constexpr int BN = 128;  // keys per block

struct Params {
  DevGeom g;
  int mode;
  int G;             // rows per TMA sub-box of a key block (divides the tile volume)
  int q_blocks_per_tile;
  PairPlan pair;     // STA query blocks (see PairPlan; used by the PAIR instance)
  int Nk;            // key rows per batch*head in the K/V tensors
  float scale_log2;  // scale * log2(e)
  __nv_bfloat16* o;
  float* lse;
  const __nv_bfloat16* o_local;
  const float* gvec;
  __nv_bfloat16* blend_out;
  // key-side tile grid and coarse factor (STA): the sliding tile has the query
  // grid and factor 1; the hierarchical branch the coarse grid and h_pool
  int kNt, kNh, kNw, cft, cfh, cfw;
  const __nv_bfloat16* merge_o;  // hierarchical: fine-key O and LSE to merge with (NULL = none)
  const float* merge_lse;
  const int* qk_amax;            // e4m3 Q*K^T: absmax bits of Q and K per batch*head
  const int* v_amax;             // e4m3 P*V: absmax bits of V per batch*head
  // raster (STA only): Q, K, V, O and LSE in raster token order.  The tensor
  // maps are 5-D (d, W, H, T, batch*head); a load is a box of whole t-slices
  // of one tile, which lands in shared memory in the tile-major row order.
  int raster;
  DevCtl ctl;
};

// D[tmem] (+)= A[smem] * B[smem], e4m3 x e4m3 -> f32, K = 32 per instruction
__device__ __forceinline__ void mma_ss_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Instruction descriptor, kind::f8f6f4: A, B e4m3 (format 0), K-major; D f32.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// The same with B MN-major (the P*V product: V rows are keys, d contiguous).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32_bmn(int M, int N) { return idesc_e4m3_f32(M, N) | (1u << 16); }
// D[tmem] (+)= A[tmem] * B[smem], e4m3 x e4m3 -> f32, K = 32 per instruction
// (A packs four e4m3 values per 32-bit TMEM column)
__device__ __forceinline__ void mma_ts_e4m3(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Key stream of one CTA: `runs` runs of `run_len` contiguous rows.
struct Stream {
  int runs, run_len, eh, t0, h0, w0;
  int ew;   // window tiles along w (sliding tile)
  // straddling query block whose two tiles' windows start one tile apart: each
  // run holds the union, ew + 1 tiles, streamed from the second (w0 + 1, in
  // both windows) to w0 + ew and then w0 (only in the first tile's window)
  int rot;
  __device__ __forceinline__ int length() const { return runs * run_len; }
};

__device__ __forceinline__ Stream make_stream(const Params& p, int q_tile) {
  Stream s;
  if (p.mode == FWD_STA) {
    const DevGeom& g = p.g;
    const int at = q_tile / (g.Nh * g.Nw), ah = (q_tile / g.Nw) % g.Nh, aw = q_tile % g.Nw;
    int et, ew;
    tile_range(at / p.cft, g.wt, p.kNt, g.wmode, &s.t0, &et);
    tile_range(ah / p.cfh, g.wh, p.kNh, g.wmode, &s.h0, &s.eh);
    tile_range(aw / p.cfw, g.ww, p.kNw, g.wmode, &s.w0, &ew);
    s.runs = et * s.eh;
    s.run_len = ew * g.s;
    s.ew = ew;
  } else {
    s.runs = 1;
    s.run_len = p.Nk;
    s.eh = 1;
    s.t0 = s.h0 = s.w0 = 0;
    s.ew = 1;
  }
  s.rot = 0;
  return s;
}

// Query block -> its rows (QueryBlock) and the key stream it attends to:
// sliding tile, the window of the block's tile or, for a straddling block, the
// union of the windows of tiles a and a + 1; global, every pooled key.
template <bool PAIR>
__device__ __forceinline__ QueryBlock query_block(const Params& p, int qblk) {
  QueryBlock b;
  const DevGeom& g = p.g;
  if (PAIR && p.mode == FWD_STA) return paired_query_block(g, p.pair, qblk);
  b.straddle = 0;
  if (p.mode == FWD_STA) {
    b.tile = qblk / p.q_blocks_per_tile;
    b.sub = qblk - b.tile * p.q_blocks_per_tile;
    b.row0 = b.tile * g.s + b.sub * BM;
    b.valid = min(BM, g.s - b.sub * BM);
  } else {
    b.tile = 0;
    b.row0 = qblk * BM;
    b.valid = min(BM, g.N - b.row0);
    b.sub = 0;
  }
  return b;
}

template <bool PAIR>
__device__ __forceinline__ Stream make_block_stream(const Params& p, const QueryBlock& b) {
  Stream s = make_stream(p, b.tile);
  if (PAIR && b.straddle && straddle_shift(p.g, p.kNw, p.cfw, b.tile) != 0) {
    s.rot = 1;
    s.run_len += p.g.s;
  }
  return s;
}

// Key row (within the batch*head slice) of stream position v < length().
__device__ __forceinline__ int stream_row(const Params& p, const Stream& s, int v) {
  if (p.mode != FWD_STA) return v;
  const int r = v / s.run_len, o = v - r * s.run_len;
  const int kt = s.t0 + r / s.eh, kh = s.h0 + r % s.eh;
  // a branch, not a select: evaluated for every sub-box, the rotation's
  // division cost the bf16 paired forward 20% (XU pipe, shared with exp2)
  if (s.rot) return ((kt * p.kNh + kh) * p.kNw + s.w0) * p.g.s + rotated_offset(o, p.g.s, s.ew);
  return ((kt * p.kNh + kh) * p.kNw + s.w0) * p.g.s + o;
}

// Walks the key stream one sub-box of G rows at a time with no integer
// division in the loop (the e4m3 kernel's loaders; tile-major rows).  Integer
// division runs on the XU pipe that also computes the softmax's exponentials:
// the e4m3 kernel is bound by that pipe and instruction issue, and dropping
// the loaders' per-sub-box divisions made it 4-8% faster, while the bf16
// kernel, held by the power cap, measured 1-2% slower with the cursor and
// keeps the direct address computation (stream_row, stream_box).
// Sliding tile: run (kt, kh), tile ti of the run, row lo of the tile; global:
// the flat position v.  Past the end of the stream `left` reaches 0.
struct KeyCursor {
  int kt, kh, ti, lo;
  int left;  // sub-boxes left in the stream
  int v;     // flat position (global)
};

__device__ __forceinline__ KeyCursor key_cursor(const Params& p, const Stream& s, int L_total) {
  KeyCursor c;
  c.kt = s.t0;
  c.kh = s.h0;
  c.ti = c.lo = 0;
  c.left = (L_total + p.G - 1) / p.G;
  c.v = 0;
  return c;
}

// Key row (within the batch*head slice) of the cursor's sub-box; past the end,
// row Nk (zero fill).
__device__ __forceinline__ int cursor_row(const Params& p, const Stream& s, const KeyCursor& c) {
  if (c.left <= 0) return p.Nk;
  if (p.mode != FWD_STA) return c.v;
  const int wt = s.rot ? (c.ti < s.ew ? c.ti + 1 : 0) : c.ti;
  return ((c.kt * p.kNh + c.kh) * p.kNw + s.w0 + wt) * p.g.s + c.lo;
}

// Next sub-box.  G divides the tile volume, so a sub-box never crosses a tile.
__device__ __forceinline__ void cursor_next(const Params& p, const Stream& s, KeyCursor& c, int tiles_per_run) {
  --c.left;
  c.v += p.G;
  c.lo += p.G;
  if (c.lo >= p.g.s) {
    c.lo = 0;
    if (++c.ti == tiles_per_run) {
      c.ti = 0;
      if (++c.kh == s.h0 + s.eh) {
        c.kh = s.h0;
        ++c.kt;
      }
    }
  }
}

// Raster box of key stream position v (a multiple of the sub-box rows): the
// x, y, t of its first token; past the end, t = T (a zero-filled box).
__device__ __forceinline__ void stream_box(const Params& p, const Stream& s, int v, int L_total, int* x, int* y,
                                           int* t) {
  const DevGeom& g = p.g;
  if (v >= L_total) {
    *x = 0;
    *y = 0;
    *t = g.T;
    return;
  }
  const int r = v / s.run_len, o = v - r * s.run_len;
  const int kt = s.t0 + r / s.eh, kh = s.h0 + r % s.eh;
  const int tile_in_run = o / g.s, lo = o - tile_in_run * g.s;
  *x = (s.w0 + tile_in_run) * g.tw;
  *y = kh * g.th;
  *t = kt * g.tt + lo / (g.th * g.tw);
}

// Debug build: a key sub-box of G rows at stream position v is either wholly
// inside the key rows (v < L_total) or the zero-filled box past the end.
__device__ __forceinline__ bool key_box_ok(const Params& p, const Stream& s, int v, int L_total) {
  if (p.raster) {
    const DevGeom& g = p.g;
    int x, y, t;
    stream_box(p, s, v, L_total, &x, &y, &t);
    if (v >= L_total) return x == 0 && y == 0 && t == g.T;
    const int nt = p.G / (g.th * g.tw);
    return x >= 0 && x + g.tw <= g.W && y >= 0 && y + g.th <= g.H && t >= 0 && t + nt <= g.T;
  }
  if (v >= L_total) return true;  // row Nk: zero fill
  const int row = stream_row(p, s, v);
  // sliding tile: sub-boxes never straddle a tile; global: only the last may run past the end
  return row >= 0 && (p.mode == FWD_STA ? row + p.G <= p.Nk : row < p.Nk);
}

// Debug build: every sub-box of key block j.
__device__ __forceinline__ bool key_block_ok(const Params& p, const Stream& s, int j, int L_total) {
  bool ok = true;
  for (int u = 0; u < BN / p.G; ++u) ok = ok && key_box_ok(p, s, j * BN + u * p.G, L_total);
  return ok;
}

// Debug build: the query block's rows start inside the slice, and an output
// row lies in its batch*head slice.
__device__ __forceinline__ bool query_block_ok(const Params& p, int q_row0, int q_valid) {
  return q_row0 >= 0 && q_valid > 0 && q_row0 + q_valid <= p.g.N;
}
__device__ __forceinline__ bool out_row_ok(const Params& p, int bh, size_t grow) {
  return grow >= (size_t)bh * p.g.N && grow < (size_t)(bh + 1) * p.g.N;
}

}  // namespace fwd
}  // namespace vattn
