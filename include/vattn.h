/*
 * vattn — dual-branch 3D video attention on B200 (sm_100a).
 *
 * Full 3D attention over a video latent token grid T x H x W is split into
 *   - a local branch: sliding-tile attention.  Every query tile attends only
 *     to the key tiles inside a 3D window of tiles around it
 *     ("Fast Video Generation with Sliding Tile Attention", abstract);
 *   - a global branch: every full-resolution query attends to average-pooled
 *     keys and values ("UltraGen: High-Resolution Video Generation with
 *     Hierarchical Attention" §4.2, spatially compressed global attention;
 *     "AtlasVid ..." abstract, asymmetric global-local attention);
 * and the two outputs are blended per head, O = g*O_local + (1-g)*O_global
 * ("UltraGen ..." §4.1, time-aware fusion factor, taken here as a given g).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates device memory on these calls; scratch space is passed in
 *    as `workspace` (size from vattn_workspace_size).
 *  - Q/K/V/O/dQ/dK/dV are [batch, heads, N, head_dim] bfloat16, head_dim
 *    contiguous, N = T*H*W.  Attention calls take TILE-MAJOR token order
 *    (see vattn_tile_permute); permute/unpermute take/produce RASTER order,
 *    raster token n = (t*H + y)*W + x.
 *  - LSE is [batch, heads, N] float32 in the same token order as O: the
 *    natural log of the softmax denominator, scale included.
 *  - K_p/V_p are [batch, heads, N_p, head_dim] bfloat16 in pooled-raster
 *    order, N_p = (T/p_t)(H/p_h)(W/p_w).
 *  - g is float32 [heads], shared across the batch, values in [0, 1].
 *  - Every pointer must be 16-byte aligned (VATTN_ERR_ALIGN otherwise).
 *  - T, H, W must be divisible by the tile and by the pool sizes
 *    (VATTN_ERR_SHAPE); head_dim must be 64 or 128 and the tile volume a
 *    multiple of 16 (VATTN_ERR_UNSUPPORTED).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Argument errors are returned synchronously and nothing is
 *    launched.  A device-side wait that exceeds its time limit makes the
 *    kernel record VATTN_ERR_DEVICE_TIMEOUT and return early; read it with
 *    vattn_get_status.
 *  - On any non-OK return, vattn_last_error() gives a message (thread-local).
 */
#ifndef VATTN_H
#define VATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Geometry of one call.  All triples are in (t, h, w) order.
 * tile   : tokens per tile along each dim; tile volume s = t_t*t_h*t_w.
 * window : tiles kept along each dim around the query tile.  Window start
 *          along a dim with n tiles is clamp(a - window/2, 0, max(n - window, 0))
 *          and its extent min(window, n), so every query tile keeps
 *          prod(min(window, n)) tiles.
 * pool   : K/V pooling block for the global branch (ignored by STA-only calls). */
typedef struct {
  int64_t batch, heads, head_dim;
  int32_t T, H, W;
  int32_t tile[3];
  int32_t window[3];
  int32_t pool[3];
} vattn_geom;

typedef enum {
  VATTN_OK = 0,
  VATTN_ERR_INVALID_ARG = -1,
  VATTN_ERR_SHAPE = -2,
  VATTN_ERR_UNSUPPORTED = -3,
  VATTN_ERR_ALIGN = -4,
  VATTN_ERR_CUDA = -5,
  VATTN_ERR_DEVICE_TIMEOUT = -6,
  VATTN_ERR_WORKSPACE = -7,
  VATTN_ERR_DEVICE_BOUNDS = -8   /* debug build only: a kernel computed an out-of-range row, tile or
                                    coordinate, skipped the access and stopped (vattn_get_status) */
} vattn_status;

/* Operation ids for vattn_workspace_size. */
enum {
  VATTN_OP_DUAL_FWD = 1,
  VATTN_OP_STA_BWD = 2,
  VATTN_OP_DUAL_BWD = 3,
  VATTN_OP_DUAL_SYM_FWD = 4,
  VATTN_OP_DUAL_SYM_BWD = 5,
  VATTN_OP_STA_FWD_HOST = 6, /* per chunk of batch*head slices: pass heads = the chunk size in geom */
  VATTN_OP_HIER_FWD = 7,     /* geom->pool = the medium pool factor h_pool */
  VATTN_OP_HIER_BWD = 8,
  VATTN_OP_STA_FWD_FP8 = 9,
  VATTN_OP_DUAL_FWD_FP8 = 10,
  VATTN_OP_DUAL_SYM_LEARNED_FWD = 11
};

/* Raster -> tile-major row gather.  Tile-major position of raster token
 * (t, y, x) is tile_id*s + local_id with
 *   tile_id  = ((t/t_t)*N_h + y/t_h)*N_w + x/t_w,
 *   local_id = ((t%t_t)*t_h + y%t_h)*t_w + x%t_w
 * ("AtlasVid ..." abstract, reordered spatiotemporal windows; "Fast Video
 * Generation with Sliding Tile Attention" abstract, tile-by-tile operation).
 * src/dst: batch*heads*N rows of row_bytes bytes each (row_bytes a positive
 * multiple of 4: 2*head_dim for Q/K/V/O, 4 for LSE).  src and dst must not
 * overlap. */
int vattn_tile_permute(const vattn_geom* geom, const void* src_raster, void* dst_tiled,
                       int64_t row_bytes, void* stream);

/* Inverse of vattn_tile_permute (tile-major -> raster). */
int vattn_tile_unpermute(const vattn_geom* geom, const void* src_tiled, void* dst_raster,
                         int64_t row_bytes, void* stream);

/* Kept-tile list ("Fast Video Generation with Sliding Tile Attention",
 * abstract: each query tile attends to the key tiles of a 3D window around
 * it).  out: device int32 [n_tiles][kept], n_tiles = prod(grid/tile),
 * kept = prod(min(window, tiles per dim)); row = query tile id (tile-major),
 * entries = key tile ids ordered t outermost, w fastest. */
int vattn_kept_tiles(const vattn_geom* geom, int32_t* out, void* stream);

/* Sliding-tile attention forward (local branch).  For query i in tile a:
 * S_ij = scale*q_i.k_j over the tokens j of a's kept tiles;
 * LSE_i = ln sum_j exp(S_ij); O_i = sum_j exp(S_ij - LSE_i) v_j.
 * q, k, v, o: tile-major bf16 [B,h,N,d]; lse: float32 [B,h,N] tile-major. */
int vattn_sta_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale,
                  void* o, float* lse, void* stream);

/* Cross-window local attention forward ("UltraGen ..." §4.3: window
 * partitions alternating between adjacent layers, K x K windows and shifted
 * (K+1) x (K+1) partitions).  Along every dim the tile grid is cut into
 * consecutive blocks: shifted = 0 uses blocks of window[d] tiles starting at
 * tile 0; shifted = 1 uses blocks of window[d] + 1 tiles whose cuts are moved
 * by floor((window[d] + 1) / 2); blocks at the grid edge are truncated.  Each
 * query tile attends to all tiles of its block.  Arguments and layouts as in
 * vattn_sta_fwd. */
int vattn_xwin_fwd(const vattn_geom* geom, int shifted, const void* q, const void* k, const void* v,
                   float scale, void* o, float* lse, void* stream);

/* Backward of vattn_xwin_fwd (same contract as vattn_sta_bwd; workspace size
 * vattn_workspace_size(VATTN_OP_STA_BWD)). */
int vattn_xwin_bwd(const vattn_geom* geom, int shifted, const void* q, const void* k, const void* v,
                   const void* o, const float* lse, const void* dout, float scale, void* dq, void* dk,
                   void* dv, void* workspace, size_t ws_bytes, void* stream);

/* Hierarchical local attention ("UltraGen: High-Resolution Video Generation
 * with Hierarchical Attention" §4.3, hierarchical local attention: an
 * intermediate-scale attention over coarse windows).  Each query attends, in
 * ONE softmax, to
 *   - its sliding-tile keys (as vattn_sta_fwd), and
 *   - the keys and values average-pooled by h_pool = geom->pool, restricted to
 *     a window of geom->window coarse tiles: the pooled grid is cut into tiles
 *     of the same shape, a coarse tile spans h_pool fine tiles per dim, and
 *     the window (clamped as the sliding tile's) is centred on the coarse tile
 *     holding the query tile.
 * Needs tiles-per-dim divisible by h_pool.  Tile-major q, k, v [B,h,N,d] bf16;
 * o tile-major; lse [B,h,N] fp32 tile-major (the joint softmax's natural-log
 * denominator) or NULL.  workspace >= vattn_workspace_size(VATTN_OP_HIER_FWD):
 * medium-pooled K/V in coarse tile-major order, then O and LSE of the fine
 * keys alone.  Errors are returned before any launch. */
int vattn_hier_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale, void* o,
                   float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Backward of vattn_hier_fwd: dq, dk, dv (bf16, tile-major) from q, k, v, the
 * forward's o and lse (required) and dout.  The medium-pooled keys' gradients
 * flow back to every token of their pool block divided by its size.
 * workspace >= vattn_workspace_size(VATTN_OP_HIER_BWD): pooled K/V, the row
 * terms D and L, fp32 dK/dV of the pooled keys and the fp32 coarse part of dQ.
 * Deterministic (no atomics). */
int vattn_hier_bwd(const vattn_geom* geom, const void* q, const void* k, const void* v, const void* o,
                   const float* lse, const void* dout, float scale, void* dq, void* dk, void* dv, void* workspace,
                   size_t ws_bytes, void* stream);

/* Sliding-tile forward on RASTER-order tensors: the raster <-> tile-major
 * reorder (vattn_tile_permute / unpermute) fused into the attention kernel.
 * q, k, v [B,h,N,d] bf16 raster; o bf16 raster; lse fp32 [B,h,N] raster or
 * NULL.  The kernel's loads are boxes of whole t-slices of a tile (5-D tensor
 * maps), so a tile's t-slice of th*tw tokens must divide 128 and the key
 * sub-box (the largest power of two <= 128 dividing the tile volume); else
 * VATTN_ERR_UNSUPPORTED.  The result equals vattn_tile_permute +
 * vattn_sta_fwd + vattn_tile_unpermute bit for bit. */
int vattn_sta_fwd_raster(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale, void* o,
                         float* lse, void* stream);

/* Sliding-tile forward in FP8 (e4m3) on the f8f6f4 tensor path, for
 * inference: both products, Q*K^T and P*V, take e4m3 operands, in the spirit
 * of the 8-bit attention the pages cite ("SageAttention"), which the pages do
 * not define further.
 *  - Q, K and V are quantised per batch*head: scale s = absmax / 448 (the
 *    largest finite e4m3), byte = round-to-nearest-even e4m3 of
 *    x * (448 / absmax) with saturation; S = bytes(Q) bytes(K)^T * s_Q * s_K *
 *    scale in fp32.
 *  - P is rounded to e4m3 in the units 2^(S*log2(e) - m + 6), where the
 *    running row maximum m is moved whenever a row's maximum grows by more
 *    than a factor 4, so the largest P is at most 2^8 and probabilities down
 *    to about 2^-15 of the row maximum keep a normal e4m3 value; the row sum
 *    is accumulated in fp32 from the unrounded P; O = P_e4m3 bytes(V) * s_V /
 *    row sum.
 * Same arguments and layouts as vattn_sta_fwd; d = 128 only.
 * workspace >= vattn_workspace_size(VATTN_OP_STA_FWD_FP8), in this order
 * (each part starting on a 256-byte boundary): e4m3 Q, K, V [B,h,N,d]; the
 * absmax bits as int32 [B*h][2] (Q, K); the absmax bits of V, int32 [B*h].
 * They hold this call's values afterwards. */
int vattn_sta_fwd_fp8(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale, void* o,
                      float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Dual forward (inference) with both branches in FP8 (e4m3), as
 * vattn_sta_fwd_fp8: O = g*O_local + (1-g)*O_global with K_p, V_p the bf16
 * average pools of K, V (as vattn_pool_kv), and Q, K, V, K_p, V_p quantised
 * with one absmax scale per batch*head each.  Tile-major q, k, v, o; g fp32
 * [heads].  workspace >= vattn_workspace_size(VATTN_OP_DUAL_FWD_FP8), in this
 * order (each part starting on a 256-byte boundary): e4m3 Q, K, V [B,h,N,d];
 * e4m3 K_p, V_p [B,h,N_p,d]; absmax bits int32 [B*h][2] of (Q, K) and of
 * (Q, K_p); absmax bits int32 [B*h] of V and of V_p; bf16 O_local [B,h,N,d];
 * bf16 K_p, V_p [B,h,N_p,d].  d = 128 only. */
int vattn_dual_fwd_fp8(const vattn_geom* geom, const void* q, const void* k, const void* v, const float* g, float scale,
                       void* o, void* workspace, size_t ws_bytes, void* stream);

/* Sliding-tile forward on HOST buffers in raster order, pipelined.  The
 * batch*head range is cut into chunks of `chunk_slices` slices; for every
 * chunk the host->device copy of Q, K, V, the attention (the raster kernel
 * of vattn_sta_fwd_raster when the tile allows it, else permute +
 * vattn_sta_fwd + unpermute), and the device->host copy of O (and LSE) run on three library
 * streams, so that copies in both directions overlap the compute of the
 * neighbouring chunks (two staging slots, reused in turn).
 *  q, k, v : host bf16 [B,h,N,d] raster; o: host bf16 raster; lse: host fp32
 *            [B,h,N] raster or NULL.  Pinned host memory gives full overlap.
 *  workspace: device memory, >= 2 * vattn_workspace_size(VATTN_OP_STA_FWD_HOST)
 *            computed on a geometry whose heads = chunk_slices and batch = 1.
 *  The work is ordered after earlier work on `stream`, and `stream` is made
 *  to wait for all of it: synchronise `stream` before reading o / lse.
 *  Calls from several host threads on one device are serialised.  When a
 *  CUDA call fails after part of the pipeline was enqueued, the library
 *  streams are synchronised before the error returns (o / lse undefined). */
int vattn_sta_fwd_host(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale,
                       void* o, float* lse, int64_t chunk_slices, void* workspace, size_t ws_bytes,
                       void* stream);

/* Average pooling of K and V over p_t x p_h x p_w token blocks ("UltraGen ..."
 * §4.2: latents downsampled before global attention).  Inputs tile-major
 * [B,h,N,d]; outputs pooled-raster [B,h,N_p,d].  fp32 sum, exact divide by
 * the block size, one round-to-nearest-even to bf16. */
int vattn_pool_kv(const vattn_geom* geom, const void* k_tiled, const void* v_tiled, void* kp,
                  void* vp, void* stream);

/* Global branch forward: every query (tile-major, full resolution) attends to
 * all N_p pooled keys, no mask ("UltraGen ..." §4.1-4.2).  o, lse as in
 * vattn_sta_fwd. */
int vattn_global_fwd(const vattn_geom* geom, const void* q, const void* kp, const void* vp,
                     float scale, void* o, float* lse, void* stream);

/* Dual-branch forward: pool, local branch, global branch, and the per-head
 * blend O = g*O_l + (1-g)*O_g ("UltraGen ..." §4.1).  q/k/v/o tile-major.
 * o_l/lse_l/o_g/lse_g/kp/vp: optional outputs that the backward needs; pass
 * all six NULL for inference, or all six non-NULL.  When they are NULL the
 * intermediates live in `workspace` (ws_bytes >= vattn_workspace_size
 * (VATTN_OP_DUAL_FWD)); otherwise workspace may be NULL. */
int vattn_dual_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v,
                   const float* g, float scale, void* o, void* o_l, float* lse_l, void* o_g,
                   float* lse_g, void* kp, void* vp, void* workspace, size_t ws_bytes, void* stream);

/* Scratch held by the library for vattn_dual_fwd_noalloc (bytes). */
#define VATTN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* Dual-branch inference forward that allocates nothing.  The pages have no
 * counterpart: this entry point exists for callers that cannot call
 * cudaMalloc (a plug-in inside a host framework whose memory pool has already
 * reserved the device and offers no allocation hook; a latency-critical path
 * that forbids allocation after start-up).  It computes what vattn_dual_fwd
 * computes with all six saved outputs NULL, but takes the workspace from a
 * static device array of VATTN_NOALLOC_SCRATCH_BYTES that every GPU which
 * loads the library holds until the process exits.
 *  - Geometries whose dual-forward workspace (vattn_workspace_size
 *    (VATTN_OP_DUAL_FWD)) exceeds VATTN_NOALLOC_SCRATCH_BYTES are rejected
 *    with VATTN_ERR_WORKSPACE before anything is launched.
 *  - The scratch has one device address per CUDA context.  The first call
 *    in each context (the current device's primary context, or whichever
 *    context the caller made current) resolves it with cudaGetSymbolAddress
 *    and caches it under the context's unique id; make that first call before
 *    any stream capture.
 *  - All calls on a device share the one scratch array and it keeps the last
 *    call's contents (nothing in it has to start at zero).  Calls whose work
 *    overlaps on the GPU (other streams, other host threads) race on it:
 *    serialise them.
 * Arguments, layouts and errors are otherwise those of vattn_dual_fwd. */
int vattn_dual_fwd_noalloc(const vattn_geom* geom, const void* q, const void* k, const void* v,
                           const float* g, float scale, void* o, void* stream);

/* Dual-branch forward with the symmetric compressed global branch
 * ("UltraGen ..." §4.2: the latent is downsampled before global attention
 * and brought back to full resolution afterwards).  Q, K and V are all
 * average-pooled; the pooled queries attend to all pooled keys; the pooled
 * result O_p is upsampled to the full grid by separable linear interpolation
 * along t, y and x with half-pixel centres (source coordinate (i + 1/2)/p -
 * 1/2, clamped at the edges); O = g*O_l + (1-g)*upsample(O_p).
 * Saved outputs for the backward (all seven NULL for inference, then the
 * intermediates live in `workspace` of vattn_workspace_size
 * (VATTN_OP_DUAL_SYM_FWD)): o_l [B,h,N,d] bf16, lse_l [B,h,N] fp32 (both
 * tile-major), qp, kp, vp, o_p [B,h,N_p,d] bf16 and lse_p [B,h,N_p] fp32 (all
 * pooled-raster). */
int vattn_dual_sym_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v,
                       const float* g, float scale, void* o, void* o_l, float* lse_l, void* qp, void* kp,
                       void* vp, void* o_p, float* lse_p, void* workspace, size_t ws_bytes, void* stream);

/* Dual-branch forward with the learned compressed global branch
 * ("UltraGen ..." §4.2: depthwise convolution of stride k for the
 * compression; bilinear upsampling and a 3D convolution for the restoration,
 * processing space and time jointly).  Inference only; the weights are
 * inputs (random ones stand in for trained values).
 *  - compression: Q, K, V each by a depthwise convolution whose stride equals
 *    its p_t x p_h x p_w kernel (geom->pool), no bias:
 *    x_p[t',y',x',c] = sum_taps w[h][tap][c] * x[t'p_t+dt, y'p_h+dy, x'p_w+dx, c];
 *    wq, wk, wv: fp32 [heads][p_t*p_h*p_w][d], taps in (dt, dy, dx) raster
 *    order (uniform taps 1/(p_t p_h p_w) give vattn_dual_sym_fwd's pooling);
 *  - the pooled queries attend to all pooled keys (scale);
 *  - restoration: the upsampling of vattn_dual_sym_fwd, then a 3x3x3
 *    depthwise convolution with zero padding, no bias:
 *    O_g[t,y,x,c] = sum w3[h][tap][c] * U[t+a, y+b, x+e, c], taps (a, b, e)
 *    over {-1, 0, 1}^3 in raster order; w3: fp32 [heads][27][d] (the
 *    identity tap 13 alone gives vattn_dual_sym_fwd's output);
 *  - O = g*O_l + (1-g)*O_g.
 * q, k, v, o: bf16 [B,h,N,d] tile-major; d a multiple of 8; weight pointers
 * 16-byte aligned.  workspace >= vattn_workspace_size
 * (VATTN_OP_DUAL_SYM_LEARNED_FWD), in this order (each 256-byte aligned):
 * O_l [B,h,N,d] bf16, Q_p, K_p, V_p, O_p [B,h,N_p,d] bf16 (pooled raster),
 * U [B,h,N,d] bf16 (raster: the upsampled pooled output, rounded to bf16). */
int vattn_dual_sym_learned_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v,
                               const float* g, const float* wq, const float* wk, const float* wv,
                               const float* w3, float scale, void* o, void* workspace, size_t ws_bytes,
                               void* stream);

/* Backward of vattn_dual_sym_fwd from its saved outputs: dq, dk, dv (bf16,
 * tile-major) through the pooling of all three inputs and the upsampling.
 * workspace >= vattn_workspace_size(VATTN_OP_DUAL_SYM_BWD). */
int vattn_dual_sym_bwd(const vattn_geom* geom, const void* q, const void* k, const void* v,
                       const float* g, const void* o_l, const float* lse_l, const void* qp, const void* kp,
                       const void* vp, const void* o_p, const float* lse_p, const void* dout, float scale,
                       void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, void* stream);

/* Sliding-tile attention backward.  Given q, k, v, the forward's o and lse
 * and the upstream gradient dout (all tile-major), writes dq, dk, dv (bf16,
 * tile-major).  dV = P^T dO, dP = dO V^T, dS = P*(dP - rowsum(dO*O)),
 * dQ = scale dS K, dK = scale dS^T Q over the kept pairs only.
 * workspace >= vattn_workspace_size(VATTN_OP_STA_BWD). */
int vattn_sta_bwd(const vattn_geom* geom, const void* q, const void* k, const void* v,
                  const void* o, const float* lse, const void* dout, float scale, void* dq,
                  void* dk, void* dv, void* workspace, size_t ws_bytes, void* stream);

/* Dual-branch backward: the gradients of O = g*O_l + (1-g)*O_g w.r.t. q, k,
 * v, including the path through the pooling (dK = dK_l + pool^T(dK_p), same
 * for V), from the forward's saved o_l, lse_l, o_g, lse_g, kp, vp.
 * dg (float32 [heads], optional, NULL = skip): sum over batch and tokens of
 * dO . (O_l - O_g).  workspace >= vattn_workspace_size(VATTN_OP_DUAL_BWD). */
int vattn_dual_bwd(const vattn_geom* geom, const void* q, const void* k, const void* v,
                   const float* g, const void* o_l, const float* lse_l, const void* o_g,
                   const float* lse_g, const void* kp, const void* vp, const void* dout,
                   float scale, void* dq, void* dk, void* dv, float* dg, void* workspace,
                   size_t ws_bytes, void* stream);

/* Scratch bytes that `op` needs for `geom` (0 if none). */
int vattn_workspace_size(int op, const vattn_geom* geom, size_t* bytes);

/* Synchronises `stream`, reads and clears the library's device error word and
 * the CUDA error state.  Returns VATTN_OK, VATTN_ERR_DEVICE_TIMEOUT or
 * VATTN_ERR_CUDA. */
int vattn_get_status(void* stream);

/* Message for the last non-OK return on this thread ("" if none). */
const char* vattn_last_error(void);

/* Releases what the library keeps between calls: the three streams and eight
 * events of vattn_sta_fwd_host's pipeline, on every device where a call
 * created them, after waiting for the work queued on them.  A later
 * vattn_sta_fwd_host creates them again.  Nothing else is held: tensor-map
 * descriptors are built per call and passed to the kernels by value, and the
 * scratch of vattn_dual_fwd_noalloc is a static device array that lives as
 * long as the loaded library.  Safe from any thread at any time (it waits for
 * a vattn_sta_fwd_host call in progress); the current device is left as it
 * was.  Returns VATTN_OK, or VATTN_ERR_CUDA if a synchronisation or a destroy
 * failed (the handles are released all the same). */
int vattn_shutdown(void);

/* Flags of vattn_debug_set. */
#define VATTN_DEBUG_SKIP_ARRIVAL 1  /* the attention kernels' load warp skips its first arrival */

/* Test hook.  flags: VATTN_DEBUG_SKIP_ARRIVAL makes the consumer's bounded
 * wait run out (no fault, no hang).  timeout_ns: the device wait limit
 * (<= 0 restores the default, 2 s).  Affects calls made after it on any
 * thread. */
int vattn_debug_set(int flags, int64_t timeout_ns);


/* Test hook: y[i] = the library's polynomial 2^x[i] (the one the attention
 * forward can run on the FMA pipe for one chunk of its exponentials; off in
 * the default build), for checking against CUDA's exp2f.  x, y: device
 * float32 [n]. */
int vattn_debug_exp2(const float* x, float* y, int64_t n, void* stream);

/* Test hook (host only, no device work): the 128-row query blocks of the
 * sliding-tile forward for `geom` with window mode `window_mode` (0 sliding,
 * 1 partition, 2 shifted partition), as the bf16 tile-major launch lays them
 * out, including the pairing of w-adjacent tiles of an odd multiple of 64
 * rows.  out: host int32 [capacity][4] = first row (tile-major), rows that
 * exist, straddle flag (rows [0, 64) in `tile`, [64, 128) in `tile` + 1),
 * tile whose window the key stream starts from.  *n_blocks receives the
 * block count (entries past capacity are not written). */
int vattn_debug_query_blocks(const vattn_geom* geom, int window_mode, int32_t* out, int64_t capacity,
                             int64_t* n_blocks);

/* Library version string. */
const char* vattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VATTN_H */
