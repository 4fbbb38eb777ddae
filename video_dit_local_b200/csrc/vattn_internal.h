// Internal declarations shared by the host entry points and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/vattn.h"

namespace vattn {

// Flattened, validated geometry handed to every kernel by value.
struct DevGeom {
  int B, heads, d;          // batch, heads, head_dim
  int N, Np;                // tokens, pooled tokens
  int T, H, W;
  int tt, th, tw;           // tile
  int wt, wh, ww;           // window (tiles)
  int pt, ph, pw;           // pool
  int Nt, Nh, Nw;           // tiles per dim
  int s;                    // tile volume
  int n_tiles, kept;        // tiles, kept tiles per query tile
  int PT, PH, PW;           // pooled grid
  int wmode;                // key-tile window: WIN_SLIDING, WIN_PARTITION, WIN_SHIFTED
};

// Key-tile window of a query tile along one dim:
//   WIN_SLIDING   the sliding tile window (clamped into the grid);
//   WIN_PARTITION the block of `window` consecutive tiles holding the tile;
//   WIN_SHIFTED   the block of `window + 1` tiles with cuts moved by
//                 floor((window + 1) / 2) (cross-window attention).
enum { WIN_SLIDING = 0, WIN_PARTITION = 1, WIN_SHIFTED = 2 };

// Runtime knobs shared by the attention kernels.
struct DevCtl {
  unsigned long long timeout_ns;
  int* err_word;            // device status word (first writer wins)
  int debug_flags;          // VATTN_DEBUG_* bits (vattn.h)
};

DevCtl current_ctl();

// Records `msg` as this thread's last error and returns `code`.
int record_error(int code, const char* msg);

// Device address of the library's __device__ variable `symbol` in the calling
// thread's current CUDA context (the primary context of the current device
// is created when none is current).  Cached per context: the first lookup in
// a context calls cudaGetSymbolAddress, so make it before any stream capture.
cudaError_t context_symbol_address(const void* symbol, void** out);

// -- reorder / pooling (reorder.cu) --
cudaError_t launch_permute(const DevGeom& g, const void* src, void* dst, int64_t row_bytes, bool to_tiled,
                           cudaStream_t st);
cudaError_t launch_kept_tiles(const DevGeom& g, int32_t* out, cudaStream_t st);
cudaError_t launch_pool_kv(const DevGeom& g, const void* k, const void* v, void* kp, void* vp, cudaStream_t st);
// Pooling with the pooled rows written in the tile-major order of `gc`, the
// pooled grid cut into tiles (the coarse tiles of the hierarchical branch).
cudaError_t launch_pool_kv_tiled(const DevGeom& g, const DevGeom& gc, const void* k, const void* v, void* kp,
                                 void* vp, cudaStream_t st);
// One bf16 tensor [bh][rows_per_bh][d] to e4m3 bytes with one scale per
// batch*head: amax[bh * amax_stride] receives the absmax as float bits; the
// dequantised value is byte * absmax / 448.
cudaError_t launch_quant_e4m3(const void* x, long long rows_per_bh, long long bh, int d, void* x8, int* amax,
                              int amax_stride, cudaStream_t st);
cudaError_t launch_pool_qkv(const DevGeom& g, const void* q, const void* k, const void* v, void* qp, void* kp,
                            void* vp, cudaStream_t st);
cudaError_t launch_upsample_blend(const DevGeom& g, const void* o_p, const void* o_l, const float* gvec, void* out,
                                  cudaStream_t st);
// Learned symmetric branch: depthwise strided compression of Q, K, V
// (weights [heads][p_t*p_h*p_w][d] fp32), and upsampling into the bf16 raster
// field u followed by the 3x3x3 depthwise restoration (w3 [heads][27][d]) and
// the blend with o_l.
cudaError_t launch_compress_qkv(const DevGeom& g, const void* q, const void* k, const void* v, const float* wq,
                                const float* wk, const float* wv, void* qp, void* kp, void* vp, cudaStream_t st);
cudaError_t launch_upsample_conv3_blend(const DevGeom& g, const void* o_p, void* u, const float* w3,
                                        const void* o_l, const float* gvec, void* out, cudaStream_t st);
cudaError_t launch_upsample_transpose(const DevGeom& g, const void* dout, const float* gvec, void* dop,
                                      cudaStream_t st);

// -- attention forward (attn_fwd.cu) --
enum FwdMode { FWD_STA = 0, FWD_GLOBAL = 1 };
struct FwdArgs {
  const void* q;
  const void* k;        // STA: K (tile-major, N rows); GLOBAL: K_p (Np rows)
  const void* v;
  void* o;              // bf16 out (may be NULL when blend_out is set and o_branch is not wanted)
  float* lse;           // may be NULL
  float scale;
  // blend epilogue (GLOBAL only): out = g*o_local + (1-g)*this_branch
  const void* o_local;  // NULL = no blend
  const float* g;
  void* blend_out;
  // STA only, hierarchical branch: keys are the tiles of `kgeom` (the coarse
  // grid) and a query tile's window is centred on its tile index divided by
  // cf; the result is merged with (merge_o, merge_lse) as one softmax over
  // both key sets.  kgeom NULL = plain sliding tile.
  const DevGeom* kgeom;
  int cf[3];
  const void* merge_o;
  const float* merge_lse;
  // STA only: q and k hold e4m3 bytes (Q*K^T on the f8f6f4 tensor path);
  // qk_amax[2 bh] / [2 bh + 1] are the absmax float bits of Q / K (scale
  // absmax / 448).  d = 128 only.
  const int* qk_amax;
  // with qk_amax: v holds e4m3 bytes too (P*V on the f8f6f4 tensor path, P
  // rounded to e4m3); v_amax[bh] is V's absmax float bits (scale absmax / 448)
  const int* v_amax;
  // STA only: q, k, v, o and lse in raster token order (5-D tensor maps; the
  // tile's t-slice, th*tw rows, must divide 128 and the key sub-box)
  bool raster;
};
cudaError_t launch_attn_fwd(const DevGeom& g, FwdMode mode, const FwdArgs& a, cudaStream_t st);
cudaError_t launch_exp2_poly(const float* x, float* y, long long n, cudaStream_t st);

// -- attention backward (attn_bwd.cu) --
struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* kp;         // pooled K/V (dual only)
  const void* vp;
  const void* dout;
  const void* o_l;        // local-branch output (or the STA output)
  const float* lse_l;
  const void* o_g;        // global-branch output (dual only)
  const float* lse_g;
  const float* g;         // blend factor per head, NULL = STA only (g = 1)
  float scale;
  void* dq;
  void* dk;
  void* dv;
  float* dg;              // optional
  // workspace pieces
  float* ndelta_l;        // [B,h,N] -rowsum(dO*O_l)
  float* ndelta_g;        // [B,h,N] -rowsum(dO*O_g)
  float* nlse2_l;         // [B,h,N] log2(gamma_l) - LSE_l*log2(e)
  float* nlse2_g;         // [B,h,N] log2(gamma_g) - LSE_g*log2(e)
  float* dkp;             // [B,h,Np,d] fp32
  float* dvp;
  float* dq_acc;          // [B,h,N,d] fp32 global-branch part of dQ (dual only)
  bool dq_acc_pooled;     // dq_acc holds pooled rows [B,h,Np,d]: add dq_acc[pool(tok)] / block size
};
cudaError_t launch_bwd_preprocess(const DevGeom& g, const BwdArgs& a, bool dual, cudaStream_t st);
// One branch: -D = -rowsum(dout*o), -L = log2(gamma) - lse*log2(e) with gamma = gvec[h]
// (gvec NULL: gamma = 1).
cudaError_t launch_preprocess_branch(const DevGeom& g, const void* dout, const void* o, const float* lse,
                                     const float* gvec, float* ndelta, float* nlse2, cudaStream_t st);
cudaError_t launch_bwd_dq(const DevGeom& g, const BwdArgs& a, bool dual, cudaStream_t st);
cudaError_t launch_bwd_dq_global(const DevGeom& g, const BwdArgs& a, cudaStream_t st);
cudaError_t launch_bwd_dkdv_local(const DevGeom& g, const BwdArgs& a, bool dual, cudaStream_t st);
cudaError_t launch_bwd_dkdv_global(const DevGeom& g, const BwdArgs& a, cudaStream_t st);
// Hierarchical branch (g.pool = h_pool, gc = the coarse grid).  coarse_keys:
// dK/dV of the medium-pooled keys a.kp / a.vp into fp32 a.dkp / a.dvp; else the
// fine keys' dK/dV (bf16 a.dk / a.dv) plus a.dkp / a.dvp through the pooling.
// Both use the joint softmax's a.nlse2_l / a.ndelta_l.
cudaError_t launch_bwd_dkdv_hier(const DevGeom& g, const DevGeom& gc, const BwdArgs& a, bool coarse_keys,
                                 cudaStream_t st);
// dQ of the coarse keys into fp32 a.dq_acc (launch_bwd_dq(dual = true) adds it).
cudaError_t launch_bwd_dq_hier(const DevGeom& g, const DevGeom& gc, const BwdArgs& a, cudaStream_t st);

// TMA descriptor for a [rows_per_bh x bh] stack of rows of `d` bf16 elements,
// box = 64 elements x box_rows rows x 1, 128-byte swizzle.  Returns false and
// fills *err on failure.
bool make_tmap_rows(CUtensorMap* map, const void* base, int d, long long rows_per_bh, long long bh, int box_rows,
                    const char** err);
// 5-D map over a raster [bh][T][H][W][d] bf16 tensor: box = 64 elements x
// tile-w x tile-h x box_t t-slices x 1, 128-byte swizzle.
bool make_tmap_raster(CUtensorMap* map, const void* base, int d, const DevGeom& g, long long bh, int box_t,
                      const char** err);
// 5-D map over a raster [bh][T][H][W][d] bf16 tensor with an unswizzled box of
// box_c channels x box_x x box_y x box_t voxels x 1 (zeros outside the grid).
bool make_tmap_conv_box(CUtensorMap* map, const void* base, int d, const DevGeom& g, long long bh, int box_c,
                        int box_x, int box_y, int box_t, const char** err);
bool make_tmap_rows_u8(CUtensorMap* map, const void* base, int d, long long rows_per_bh, long long bh, int box_rows,
                       const char** err);

}  // namespace vattn
