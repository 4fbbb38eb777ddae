// Definitions of the backward kernels (attn_bwd.cu): row streams over boxes
// of tiles, the pooling index maps, the bulk copy of L / D rows and the
// launch parameters of the dK / dV and dQ kernels.
#pragma once

#include "common.cuh"

namespace vattn {
namespace bwd {

constexpr float LOG2E = 1.4426950408889634f;

// A row stream over a box of tiles (see TileBox) or a flat range.
struct RowStream {
  int runs, run_len, eh, t0, h0, w0;
  int ew;    // window tiles along w (window_stream)
  int rot;   // straddling query block over windows one tile apart (see rotated_offset)
  bool tiled;
  __device__ __forceinline__ int length() const { return runs * run_len; }
  __device__ __forceinline__ int row(const DevGeom& g, int v) const {
    if (!tiled) return v;
    const int r = v / run_len, o = v - r * run_len;
    const int kt = t0 + r / eh, kh = h0 + r % eh;
    // a branch, not a select, so that the rotation's division is not
    // evaluated for every sub-box (XU pipe, shared with exp2)
    if (rot) return ((kt * g.Nh + kh) * g.Nw + w0) * g.s + rotated_offset(o, g.s, ew);
    return ((kt * g.Nh + kh) * g.Nw + w0) * g.s + o;
  }
};

__device__ __forceinline__ RowStream flat_stream(int n) {
  RowStream s;
  s.runs = 1;
  s.run_len = n;
  s.eh = 1;
  s.t0 = s.h0 = s.w0 = 0;
  s.ew = 1;
  s.rot = 0;
  s.tiled = false;
  return s;
}

// Debug build: the rows [v, v + G) of stream position v lie inside the
// stream's tensor (n rows per batch*head): a tiled stream's sub-box never
// straddles a tile, a flat stream's only past its end; past the end of the
// stream the zero-filled row n is loaded.
__device__ __forceinline__ bool stream_box_ok(const RowStream& st, const DevGeom& g, int v, int G, int len, int n) {
  if (v >= len) return true;
  const int row = st.row(g, v);
  return row >= 0 && (st.tiled ? row + G <= n : row < n);
}

// Key tiles kept by query tile q (its window).  The keys are the tiles of gk:
// the query grid itself for the sliding tile (cf = 1); the coarse grid of the
// hierarchical branch, whose window is centred on q's tile index / cf.  Rows
// of the stream are rows of gk (RowStream::row(gk, v)).
__device__ __forceinline__ RowStream window_stream(const DevGeom& g, const DevGeom& gk, int cft, int cfh, int cfw,
                                                   int q) {
  const int at = q / (g.Nh * g.Nw), ah = (q / g.Nw) % g.Nh, aw = q % g.Nw;
  RowStream s;
  int et, ew;
  tile_range(at / cft, g.wt, gk.Nt, g.wmode, &s.t0, &et);
  tile_range(ah / cfh, g.wh, gk.Nh, g.wmode, &s.h0, &s.eh);
  tile_range(aw / cfw, g.ww, gk.Nw, g.wmode, &s.w0, &ew);
  s.runs = et * s.eh;
  s.run_len = ew * g.s;
  s.ew = ew;
  s.rot = 0;
  s.tiled = true;
  return s;
}

// Query tiles whose window holds key tile k of gk (the inverse window): per
// dim a contiguous range of gk tiles, i.e. of query tiles [lo*cf, (hi+1)*cf),
// so again a box of tiles; rows are rows of the query grid g.
__device__ __forceinline__ RowStream inverse_stream(const DevGeom& g, const DevGeom& gk, int cft, int cfh, int cfw,
                                                    int k) {
  const int kt = k / (gk.Nh * gk.Nw), kh = (k / gk.Nw) % gk.Nh, kw = k % gk.Nw;
  int lt, ht, lh, hh, lw, hw;
  tile_inverse(kt, g.wt, gk.Nt, g.wmode, &lt, &ht);
  tile_inverse(kh, g.wh, gk.Nh, g.wmode, &lh, &hh);
  tile_inverse(kw, g.ww, gk.Nw, g.wmode, &lw, &hw);
  RowStream s;
  s.t0 = lt * cft;
  s.h0 = lh * cfh;
  s.w0 = lw * cfw;
  s.eh = (hh - lh + 1) * cfh;
  s.runs = (ht - lt + 1) * cft * s.eh;
  s.run_len = (hw - lw + 1) * cfw * g.s;
  s.ew = (hw - lw + 1) * cfw;
  s.rot = 0;
  s.tiled = true;
  return s;
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Index, in gk's tile-major order, of the pool block holding tile-major token
// `tok` of g (the medium-pooled grid cut into tiles: hierarchical branch).
__device__ __forceinline__ int coarse_of_tiled(const DevGeom& g, const DevGeom& gk, int tok) {
  const int tile = tok / g.s, l = tok - tile * g.s;
  const int at = tile / (g.Nh * g.Nw), ah = (tile / g.Nw) % g.Nh, aw = tile % g.Nw;
  const int lt = l / (g.th * g.tw), lh = (l / g.tw) % g.th, lw = l % g.tw;
  const int t = (at * g.tt + lt) / g.pt, y = (ah * g.th + lh) / g.ph, x = (aw * g.tw + lw) / g.pw;
  const int ct = t / gk.tt, ch = y / gk.th, cw = x / gk.tw;
  return ((ct * gk.Nh + ch) * gk.Nw + cw) * gk.s + ((t - ct * gk.tt) * gk.th + (y - ch * gk.th)) * gk.tw +
         (x - cw * gk.tw);
}

// pooled-raster index of the pool block holding tile-major token `tok`
__device__ __forceinline__ int pooled_of_tiled(const DevGeom& g, int tok) {
  const int tile = tok / g.s, l = tok - tile * g.s;
  const int at = tile / (g.Nh * g.Nw), ah = (tile / g.Nw) % g.Nh, aw = tile % g.Nw;
  const int lt = l / (g.th * g.tw), lh = (l / g.tw) % g.th, lw = l % g.tw;
  const int t = at * g.tt + lt, y = ah * g.th + lh, x = aw * g.tw + lw;
  return ((t / g.pt) * g.PH + y / g.ph) * g.PW + x / g.pw;
}

// Two launches make dQ: GLOBAL (dense 128-row query blocks against all pooled
// keys, fp32 result to a workspace) and LOCAL (query blocks inside one query
// tile against its kept window; adds the GLOBAL part and writes bf16 dQ).
// HIER: the coarse window of medium-pooled keys (hierarchical branch), fp32
// partial dQ out (acc_out) for the fine pass to add.
enum { DQ_LOCAL = 0, DQ_GLOBAL = 1, DQ_HIER = 2 };

struct DqParams {
  DevGeom g;
  DevGeom gk;        // key tile grid (= g but for DQ_HIER: the coarse grid)
  int cft, cfh, cfw; // coarse factor (1 but for DQ_HIER)
  int mode;          // DQ_LOCAL / DQ_GLOBAL / DQ_HIER
  int G0;            // key sub-box rows of the local stream
  int q_blocks_per_tile;
  PairPlan pair;     // LOCAL / HIER query blocks (see PairPlan; used by the PAIR instance)
  float c2;
  float scale;
  const float* nlse2;    // log2(gamma) - LSE*log2(e) of this branch
  const float* ndelta;   // -rowsum(dO*O)
  const float* acc_in;   // LOCAL: fp32 global-branch dQ to add (NULL = none)
  int acc_pooled;        // acc_in holds pooled rows: add acc_in[pool(tok)] / block size
  float* acc_out;        // GLOBAL: fp32 output
  __nv_bfloat16* dq;     // LOCAL: bf16 output
  DevCtl ctl;
};

// HIER: keys are the coarse tiles of the medium-pooled grid (hierarchical
// branch): the inverse coarse window of fine query tiles, fp32 dK_h / dV_h out.
enum { DKDV_LOCAL = 0, DKDV_GLOBAL = 1, DKDV_HIER = 2 };

struct DkdvParams {
  DevGeom g;
  DevGeom gk;        // key tile grid (= g but for DKDV_HIER: the coarse grid)
  int cft, cfh, cfw; // coarse factor (1 but for DKDV_HIER)
  int hier_add;      // LOCAL: dkp_in / dvp_in are rows of gadd in tile-major order
  DevGeom gadd;      // the coarse grid of those rows (hier_add only)
  int mode;          // DKDV_LOCAL / DKDV_GLOBAL / DKDV_HIER
  int Gq;            // query sub-box rows (divides the tile volume, <= 64)
  int kv_blocks_per_tile;
  PairPlan pair;     // LOCAL key blocks (see PairPlan; used by the PAIR instance)
  int Nk;            // key rows per batch*head (N or Np)
  float c2;          // scale * log2(e)
  float scale;
  const float* nlse2;    // log2(gamma) - LSE*log2(e) per query row
  const float* ndelta;   // -rowsum(dO*O)
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dkp_out;
  float* dvp_out;
  const float* dkp_in;   // pool-backward addend for LOCAL (NULL = none), already scaled
  const float* dvp_in;
  DevCtl ctl;
};

}  // namespace bwd
}  // namespace vattn
