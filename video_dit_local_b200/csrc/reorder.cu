// HBM-bound kernels: raster <-> tile-major row gather, the kept-tile list, and
// K/V average pooling.  All of them are grid-stride loops over 16-byte
// vectors with 32-bit index math done by multiply-high division.
#include <algorithm>

#include "common.cuh"

namespace vattn {

// Unsigned 32-bit division by a runtime constant via a precomputed
// multiplier (Granlund & Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994): q = (umulhi(n, m) + n) >> s  for n < 2^31.
struct FastDiv {
  uint32_t d, m, s;
  FastDiv() = default;
  explicit FastDiv(uint32_t div) : d(div) {
    s = 0;
    while ((1u << s) < div) ++s;  // s = ceil(log2(div))
    const uint64_t one = 1;
    m = static_cast<uint32_t>(((one << 32) * ((one << s) - div)) / div + 1);
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const { return (__umulhi(n, m) + n) >> s; }
};

struct ReorderParams {
  FastDiv s, nhnw, nw, thtw, tw;      // tile-major -> raster
  FastDiv W, H, tt, th, tww;          // raster -> tile-major
  uint32_t T, Hh, Ww, ttt, tth, ttw, Nh, Nw, vol;
};

// tile-major position m -> raster token
__device__ __forceinline__ uint32_t tiled_to_raster(const ReorderParams& p, uint32_t m) {
  const uint32_t tile = p.s.div(m);
  const uint32_t l = m - tile * p.vol;
  const uint32_t at = p.nhnw.div(tile);
  const uint32_t rem = tile - at * p.Nh * p.Nw;
  const uint32_t ah = p.nw.div(rem);
  const uint32_t aw = rem - ah * p.Nw;
  const uint32_t lt = p.thtw.div(l);
  const uint32_t rl = l - lt * p.tth * p.ttw;
  const uint32_t lh = p.tw.div(rl);
  const uint32_t lw = rl - lh * p.ttw;
  return ((at * p.ttt + lt) * p.Hh + ah * p.tth + lh) * p.Ww + aw * p.ttw + lw;
}

// raster token (t, y, x) -> tile-major position
__device__ __forceinline__ uint32_t coords_to_tiled(const ReorderParams& p, uint32_t t, uint32_t y, uint32_t x) {
  const uint32_t at = p.tt.div(t), ah = p.th.div(y), aw = p.tww.div(x);
  const uint32_t lt = t - at * p.ttt, lh = y - ah * p.tth, lw = x - aw * p.ttw;
  return ((at * p.Nh + ah) * p.Nw + aw) * p.vol + (lt * p.tth + lh) * p.ttw + lw;
}

__device__ __forceinline__ uint32_t raster_to_tiled(const ReorderParams& p, uint32_t n) {
  const uint32_t r = p.W.div(n);
  const uint32_t x = n - r * p.Ww;
  const uint32_t t = p.H.div(r);
  const uint32_t y = r - t * p.Hh;
  return coords_to_tiled(p, t, y, x);
}

static ReorderParams make_params(const DevGeom& g) {
  ReorderParams p;
  p.s = FastDiv(g.s);
  p.nhnw = FastDiv(g.Nh * g.Nw);
  p.nw = FastDiv(g.Nw);
  p.thtw = FastDiv(g.th * g.tw);
  p.tw = FastDiv(g.tw);
  p.W = FastDiv(g.W);
  p.H = FastDiv(g.H);
  p.tt = FastDiv(g.tt);
  p.th = FastDiv(g.th);
  p.tww = FastDiv(g.tw);
  p.T = g.T;
  p.Hh = g.H;
  p.Ww = g.W;
  p.ttt = g.tt;
  p.tth = g.th;
  p.ttw = g.tw;
  p.Nh = g.Nh;
  p.Nw = g.Nw;
  p.vol = g.s;
  return p;
}

// Every destination row is written once.  A row is `units` words of UNIT
// bytes (uint4 when the row is a multiple of 16 bytes, else uint32).  Indices
// are 32-bit: the host splits the batch*head range so that every launch
// covers fewer than 2^31 words.  TO_TILED: dst is tile-major, src raster.
template <bool TO_TILED, typename U>
__global__ void __launch_bounds__(256) permute_kernel(ReorderParams p, FastDiv per_row, FastDiv n_rows,
                                                       const U* __restrict__ src, U* __restrict__ dst,
                                                       uint32_t total, int* err) {
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint32_t row = per_row.div(i);
    const uint32_t c = i - row * per_row.d;
    const uint32_t bh = n_rows.div(row);
    const uint32_t r = row - bh * n_rows.d;
    const uint32_t sr = TO_TILED ? tiled_to_raster(p, r) : raster_to_tiled(p, r);
    if (!dcheck(sr < n_rows.d, err)) continue;
    const U v = __ldg(src + ((size_t)bh * n_rows.d + sr) * per_row.d + c);
    __stcs(dst + i, v);
  }
}

static int grid_for(long long work, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (work + threads - 1) / threads;
  long long cap = (long long)sms * 8;  // 8 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  return (int)(blocks < 1 ? 1 : blocks);
}

template <typename U>
static cudaError_t permute_typed(const DevGeom& g, const void* src, void* dst, uint32_t units, bool to_tiled,
                                 cudaStream_t st) {
  const ReorderParams p = make_params(g);
  int* err = current_ctl().err_word;
  const long long per_bh = (long long)g.N * units;
  const long long bh_total = (long long)g.B * g.heads;
  long long chunk = ((1ll << 31) - 1) / per_bh;
  if (chunk < 1) return cudaErrorInvalidValue;
  for (long long b0 = 0; b0 < bh_total; b0 += chunk) {
    const long long nb = bh_total - b0 < chunk ? bh_total - b0 : chunk;
    const uint32_t total = (uint32_t)(nb * per_bh);
    const U* s = (const U*)src + b0 * per_bh;
    U* d = (U*)dst + b0 * per_bh;
    const int grid = grid_for(total, 256);
    if (to_tiled)
      permute_kernel<true, U><<<grid, 256, 0, st>>>(p, FastDiv(units), FastDiv(g.N), s, d, total, err);
    else
      permute_kernel<false, U><<<grid, 256, 0, st>>>(p, FastDiv(units), FastDiv(g.N), s, d, total, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_permute(const DevGeom& g, const void* src, void* dst, int64_t row_bytes, bool to_tiled,
                           cudaStream_t st) {
  if ((long long)g.B * g.heads * g.N == 0) return cudaSuccess;
  if (row_bytes % 16 == 0) return permute_typed<uint4>(g, src, dst, (uint32_t)(row_bytes / 16), to_tiled, st);
  return permute_typed<uint32_t>(g, src, dst, (uint32_t)(row_bytes / 4), to_tiled, st);
}

// ---------------------------------------------------------------------------
// kept-tile list
// ---------------------------------------------------------------------------
__global__ void kept_tiles_kernel(DevGeom g, int32_t* __restrict__ out) {
  const int total = g.n_tiles * g.kept;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int qt = i / g.kept, j = i - qt * g.kept;
    const int at = qt / (g.Nh * g.Nw), ah = (qt / g.Nw) % g.Nh, aw = qt % g.Nw;
    const int et = win_extent(g.wt, g.Nt), eh = win_extent(g.wh, g.Nh), ew = win_extent(g.ww, g.Nw);
    (void)et;
    const int jt = j / (eh * ew), jh = (j / ew) % eh, jw = j % ew;
    const int kt = win_start(at, g.wt, g.Nt) + jt;
    const int kh = win_start(ah, g.wh, g.Nh) + jh;
    const int kw = win_start(aw, g.ww, g.Nw) + jw;
    out[i] = (kt * g.Nh + kh) * g.Nw + kw;
  }
}

cudaError_t launch_kept_tiles(const DevGeom& g, int32_t* out, cudaStream_t st) {
  const int total = g.n_tiles * g.kept;
  kept_tiles_kernel<<<grid_for(total, 256), 256, 0, st>>>(g, out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K/V average pooling: tile-major input -> pooled-raster output
// ("UltraGen ..." §4.2, spatially compressed global attention)
// ---------------------------------------------------------------------------
struct PoolParams {
  ReorderParams rp;
  ReorderParams rpo;   // output order when out_tiled: tile-major over the pooled grid
  FastDiv PW, PH;      // pooled grid divisions
  uint32_t pt, ph, pw, PWv, PHv, N, Np, vpr;
  float inv_cnt;
  int out_tiled;
};

// Up to three tensors pooled in one launch (K and V; or Q, K and V).
struct PoolTensors {
  const uint4* src[3];
  uint4* dst[3];
  int count;
};

// One thread produces one 16-byte vector (8 bf16) of one pooled row: the fp32
// sum of the block's tokens in (t, y, x) order, divided by the block size
// (one correctly rounded fp32 division), one round-to-nearest-even to bf16.
// PWC > 0 is the pool width known at compile time: the PWC loads of one
// (t, y) row of the block are issued together before they are summed (in the
// same x order), so more loads are in flight per thread.
template <int PWC>
__global__ void __launch_bounds__(256) pool_kv_kernel(PoolParams p, FastDiv per_row, FastDiv n_prow,
                                                       FastDiv rows_per_tensor, PoolTensors ts, int* err) {
  const uint32_t total = (uint32_t)ts.count * rows_per_tensor.d * p.vpr;
  const uint32_t stride = gridDim.x * blockDim.x;
  const float cnt = (float)(p.pt * p.ph * p.pw);
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint32_t row2 = per_row.div(i);
    const uint32_t c = i - row2 * p.vpr;
    const uint32_t which = rows_per_tensor.div(row2);
    const uint32_t row = row2 - which * rows_per_tensor.d;
    const uint32_t bh = n_prow.div(row);
    const uint32_t u = row - bh * p.Np;
    const uint32_t r = p.PW.div(u);
    const uint32_t ux = u - r * p.PWv;
    const uint32_t ut = p.PH.div(r);
    const uint32_t uy = r - ut * p.PHv;
    const uint4* src = ts.src[which] + (size_t)bh * p.N * p.vpr + c;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (uint32_t a = 0; a < p.pt; ++a)
      for (uint32_t b = 0; b < p.ph; ++b) {
        if constexpr (PWC > 0) {
          uint4 w[PWC];
#pragma unroll
          for (int x = 0; x < PWC; ++x) {
            const uint32_t m = coords_to_tiled(p.rp, ut * p.pt + a, uy * p.ph + b, ux * PWC + x);
            w[x] = dcheck(m < p.N, err) ? __ldg(src + (size_t)m * p.vpr) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int x = 0; x < PWC; ++x) {
            const uint32_t ww[4] = {w[x].x, w[x].y, w[x].z, w[x].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc[2 * e] += bf16lo(ww[e]);
              acc[2 * e + 1] += bf16hi(ww[e]);
            }
          }
        } else {
          for (uint32_t x = 0; x < p.pw; ++x) {
            const uint32_t m = coords_to_tiled(p.rp, ut * p.pt + a, uy * p.ph + b, ux * p.pw + x);
            if (!dcheck(m < p.N, err)) continue;
            const uint4 w = __ldg(src + (size_t)m * p.vpr);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc[2 * e] += bf16lo(ww[e]);
              acc[2 * e + 1] += bf16hi(ww[e]);
            }
          }
        }
      }
    uint4 o;
    o.x = pack_bf16(acc[0] / cnt, acc[1] / cnt);
    o.y = pack_bf16(acc[2] / cnt, acc[3] / cnt);
    o.z = pack_bf16(acc[4] / cnt, acc[5] / cnt);
    o.w = pack_bf16(acc[6] / cnt, acc[7] / cnt);
    const uint32_t uo = p.out_tiled ? coords_to_tiled(p.rpo, ut, uy, ux) : u;
    if (!dcheck(uo < p.Np, err)) continue;
    ts.dst[which][((size_t)bh * p.Np + uo) * p.vpr + c] = o;
  }
}

static PoolParams make_pool_params(const DevGeom& g) {
  PoolParams p;
  p.rp = make_params(g);
  p.PW = FastDiv(g.PW);
  p.PH = FastDiv(g.PH);
  p.pt = g.pt;
  p.ph = g.ph;
  p.pw = g.pw;
  p.PWv = g.PW;
  p.PHv = g.PH;
  p.N = g.N;
  p.Np = g.Np;
  p.vpr = g.d / 8;
  p.inv_cnt = 1.0f / (float)(g.pt * g.ph * g.pw);
  p.rpo = p.rp;
  p.out_tiled = 0;
  return p;
}

static cudaError_t pool_tensors(const DevGeom& g, int count, const void* const* src, void* const* dst,
                                cudaStream_t st, const DevGeom* gout = nullptr) {
  PoolParams p = make_pool_params(g);
  if (gout) {
    p.rpo = make_params(*gout);
    p.out_tiled = 1;
  }
  const long long per_bh = (long long)g.Np * p.vpr;
  const long long bh_total = (long long)g.B * g.heads;
  if (per_bh * bh_total == 0) return cudaSuccess;
  const long long chunk = ((1ll << 31) - 1) / (per_bh * count);  // every launch below 2^31 vectors
  if (chunk < 1) return cudaErrorInvalidValue;
  for (long long b0 = 0; b0 < bh_total; b0 += chunk) {
    const long long nb = bh_total - b0 < chunk ? bh_total - b0 : chunk;
    const uint32_t rows = (uint32_t)(nb * g.Np);
    const size_t in_off = (size_t)b0 * g.N * p.vpr, out_off = (size_t)b0 * g.Np * p.vpr;
    PoolTensors ts;
    ts.count = count;
    for (int i = 0; i < 3; ++i) {
      const int j = i < count ? i : 0;
      ts.src[i] = (const uint4*)src[j] + in_off;
      ts.dst[i] = (uint4*)dst[j] + out_off;
    }
    const int grid = grid_for((long long)count * rows * p.vpr, 256);
    int* err = current_ctl().err_word;
    if (g.pw == 4)
      pool_kv_kernel<4><<<grid, 256, 0, st>>>(p, FastDiv(p.vpr), FastDiv(g.Np), FastDiv(rows), ts, err);
    else if (g.pw == 8)
      pool_kv_kernel<8><<<grid, 256, 0, st>>>(p, FastDiv(p.vpr), FastDiv(g.Np), FastDiv(rows), ts, err);
    else if (g.pw == 2)
      pool_kv_kernel<2><<<grid, 256, 0, st>>>(p, FastDiv(p.vpr), FastDiv(g.Np), FastDiv(rows), ts, err);
    else
      pool_kv_kernel<0><<<grid, 256, 0, st>>>(p, FastDiv(p.vpr), FastDiv(g.Np), FastDiv(rows), ts, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_pool_kv(const DevGeom& g, const void* k, const void* v, void* kp, void* vp, cudaStream_t st) {
  const void* src[2] = {k, v};
  void* dst[2] = {kp, vp};
  return pool_tensors(g, 2, src, dst, st);
}

cudaError_t launch_pool_kv_tiled(const DevGeom& g, const DevGeom& gc, const void* k, const void* v, void* kp,
                                 void* vp, cudaStream_t st) {
  const void* src[2] = {k, v};
  void* dst[2] = {kp, vp};
  return pool_tensors(g, 2, src, dst, st, &gc);
}

cudaError_t launch_pool_qkv(const DevGeom& g, const void* q, const void* k, const void* v, void* qp, void* kp,
                            void* vp, cudaStream_t st) {
  const void* src[3] = {q, k, v};
  void* dst[3] = {qp, kp, vp};
  return pool_tensors(g, 3, src, dst, st);
}

// ---------------------------------------------------------------------------
// FP8 (e4m3) quantisation of Q and K for the FP8 Q*K^T forward: one scale per
// batch*head and tensor, s = absmax / 448 (448 = largest finite e4m3), so
// x8 = RNE_e4m3(x * (448 / absmax)) with saturation.  e4m3 is a floating
// format: one scale per head only has to keep values in range.
// ---------------------------------------------------------------------------
// absmax of one [bh][vec_per_bh] tensor per batch*head into amax[bh * stride]
__global__ void __launch_bounds__(256) absmax_kernel(const uint4* x, int* amax, int stride, uint32_t vec_per_bh) {
  const uint32_t bh = blockIdx.y;
  const uint4* src = x + (size_t)bh * vec_per_bh;
  float m = 0.f;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < vec_per_bh; i += gridDim.x * blockDim.x) {
    const uint4 w = __ldg(src + i);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf16lo(ww[e])), fabsf(bf16hi(ww[e]))));
  }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // non-negative floats order like their bit patterns
  if ((threadIdx.x & 31) == 0) atomicMax(&amax[(size_t)bh * stride], __float_as_int(m));
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));  // first operand -> upper byte
  return r;
}

__global__ void __launch_bounds__(256) quant_kernel(const uint4* x, const int* amax, int stride, uint2* x8,
                                                    uint32_t vec_per_bh) {
  const uint32_t bh = blockIdx.y;
  const float a = __int_as_float(amax[(size_t)bh * stride]);
  const float inv = a > 0.f ? 448.f / a : 1.f;
  const uint4* src = x + (size_t)bh * vec_per_bh;
  uint2* dst = x8 + (size_t)bh * vec_per_bh;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < vec_per_bh; i += gridDim.x * blockDim.x) {
    const uint4 w = __ldg(src + i);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    uint32_t b[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) b[e] = e4m3x2(bf16lo(ww[e]) * inv, bf16hi(ww[e]) * inv);
    dst[i] = make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
  }
}

cudaError_t launch_quant_e4m3(const void* x, long long rows_per_bh, long long bh, int d, void* x8, int* amax,
                              int amax_stride, cudaStream_t st) {
  const long long vec = rows_per_bh * d / 8;
  if (bh == 0 || vec == 0) return cudaSuccess;
  if (vec >= (1ll << 31)) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemset2DAsync(amax, sizeof(int) * amax_stride, 0, sizeof(int), bh, st);
  if (e != cudaSuccess) return e;
  const int blocks = (int)std::min<long long>((vec + 255) / 256, 128);
  absmax_kernel<<<dim3(blocks, (unsigned)bh), 256, 0, st>>>((const uint4*)x, amax, amax_stride, (uint32_t)vec);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  quant_kernel<<<dim3(blocks, (unsigned)bh), 256, 0, st>>>((const uint4*)x, amax, amax_stride, (uint2*)x8,
                                                           (uint32_t)vec);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Upsampling of the symmetric global branch ("UltraGen ..." §4.2: the
// compressed latent is brought back to the full grid): separable linear
// interpolation along t, y, x with half-pixel centres, source coordinate
// (i + 1/2)/p - 1/2 clamped to the pooled grid.
// ---------------------------------------------------------------------------
struct Interp {
  int i0, i1;
  float f;  // weight of i1; i0 gets 1 - f
};

__device__ __forceinline__ Interp interp_of(int i, int p, int n_in) {
  float src = ((float)i + 0.5f) / (float)p - 0.5f;
  src = fminf(fmaxf(src, 0.f), (float)(n_in - 1));
  Interp r;
  r.i0 = (int)floorf(src);
  r.i1 = min(r.i0 + 1, n_in - 1);
  r.f = src - (float)r.i0;
  return r;
}

struct UpParams {
  ReorderParams rp;
  int N, Np, PT, PH, PW, pt, ph, pw, vpr, heads;
  int bh_offset;  // batch*head index of the launch's first slice (for g)
};

// O[tok] = g*O_l[tok] + (1 - g)*upsample(O_p)[tok], tile-major out; one thread
// per 16-byte vector of an output row.
__global__ void __launch_bounds__(256) upsample_blend_kernel(UpParams p, FastDiv per_row, FastDiv n_rows,
                                                              const uint4* __restrict__ op, const uint4* __restrict__ ol,
                                                              const float* __restrict__ gvec, uint4* __restrict__ out,
                                                              uint32_t total) {
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint32_t row = per_row.div(i);
    const uint32_t c = i - row * p.vpr;
    const uint32_t bh = n_rows.div(row);
    const uint32_t m = row - bh * p.N;
    const uint32_t n = tiled_to_raster(p.rp, m);
    const uint32_t ty = p.rp.W.div(n);
    const uint32_t x = n - ty * p.rp.Ww;
    const uint32_t t = p.rp.H.div(ty);
    const uint32_t y = ty - t * p.rp.Hh;
    const Interp it = interp_of(t, p.pt, p.PT), iy = interp_of(y, p.ph, p.PH), ix = interp_of(x, p.pw, p.PW);
    const uint4* base = op + (size_t)bh * p.Np * p.vpr + c;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const float w = (a ? it.f : 1.f - it.f) * (b ? iy.f : 1.f - iy.f) * (cc ? ix.f : 1.f - ix.f);
          if (w == 0.f) continue;
          const int u = ((a ? it.i1 : it.i0) * p.PH + (b ? iy.i1 : iy.i0)) * p.PW + (cc ? ix.i1 : ix.i0);
          const uint4 v = __ldg(base + (size_t)u * p.vpr);
          const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] += w * bf16lo(vv[e]);
            acc[2 * e + 1] += w * bf16hi(vv[e]);
          }
        }
    const float gh = gvec[(bh + p.bh_offset) % p.heads];
    const uint4 l = __ldg(ol + (size_t)row * p.vpr + c);
    const uint32_t lv[4] = {l.x, l.y, l.z, l.w};
    uint32_t r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      r[e] = pack_bf16(gh * bf16lo(lv[e]) + (1.f - gh) * acc[2 * e], gh * bf16hi(lv[e]) + (1.f - gh) * acc[2 * e + 1]);
    out[(size_t)row * p.vpr + c] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

// dO_p[u] = (1 - g) * sum over full-grid tokens of w(token, u) * dO[token]:
// the adjoint of the upsampling, gathered per pooled row (bf16 out, fp32 sums).
// Along a dim the tokens whose stencil reaches pooled index j lie in
// [j*p - p, j*p + 2p) (clamped); their weights are recomputed here.
__global__ void __launch_bounds__(256) upsample_transpose_kernel(UpParams p, FastDiv per_row, FastDiv n_rows,
                                                                  const uint4* __restrict__ dout,
                                                                  const float* __restrict__ gvec,
                                                                  uint4* __restrict__ dop, uint32_t total) {
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint32_t row = per_row.div(i);
    const uint32_t c = i - row * p.vpr;
    const uint32_t bh = n_rows.div(row);
    const int u = (int)(row - bh * p.Np);
    const int ux = u % p.PW, uy = (u / p.PW) % p.PH, ut = u / (p.PW * p.PH);
    const uint4* base = dout + (size_t)bh * p.N * p.vpr + c;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    const int t0 = max(ut * p.pt - p.pt, 0), t1 = min(ut * p.pt + 2 * p.pt, p.rp.T);
    const int y0 = max(uy * p.ph - p.ph, 0), y1 = min(uy * p.ph + 2 * p.ph, p.rp.Hh);
    const int x0 = max(ux * p.pw - p.pw, 0), x1 = min(ux * p.pw + 2 * p.pw, p.rp.Ww);
    for (int t = t0; t < t1; ++t) {
      const Interp it = interp_of(t, p.pt, p.PT);
      const float wt = (it.i0 == ut ? 1.f - it.f : 0.f) + (it.i1 == ut ? it.f : 0.f);
      if (wt == 0.f) continue;
      for (int y = y0; y < y1; ++y) {
        const Interp iy = interp_of(y, p.ph, p.PH);
        const float wy = (iy.i0 == uy ? 1.f - iy.f : 0.f) + (iy.i1 == uy ? iy.f : 0.f);
        if (wy == 0.f) continue;
        for (int x = x0; x < x1; ++x) {
          const Interp ix = interp_of(x, p.pw, p.PW);
          const float wx = (ix.i0 == ux ? 1.f - ix.f : 0.f) + (ix.i1 == ux ? ix.f : 0.f);
          if (wx == 0.f) continue;
          const float w = wt * wy * wx;
          const uint32_t m = coords_to_tiled(p.rp, t, y, x);
          const uint4 v = __ldg(base + (size_t)m * p.vpr);
          const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] += w * bf16lo(vv[e]);
            acc[2 * e + 1] += w * bf16hi(vv[e]);
          }
        }
      }
    }
    const float gg = 1.f - gvec[(bh + p.bh_offset) % p.heads];
    dop[(size_t)row * p.vpr + c] = make_uint4(pack_bf16(gg * acc[0], gg * acc[1]), pack_bf16(gg * acc[2], gg * acc[3]),
                                              pack_bf16(gg * acc[4], gg * acc[5]), pack_bf16(gg * acc[6], gg * acc[7]));
  }
}

static UpParams make_up_params(const DevGeom& g) {
  UpParams p;
  p.rp = make_params(g);
  p.N = g.N;
  p.Np = g.Np;
  p.PT = g.PT;
  p.PH = g.PH;
  p.PW = g.PW;
  p.pt = g.pt;
  p.ph = g.ph;
  p.pw = g.pw;
  p.vpr = g.d / 8;
  p.heads = g.heads;
  p.bh_offset = 0;
  return p;
}

cudaError_t launch_upsample_blend(const DevGeom& g, const void* o_p, const void* o_l, const float* gvec, void* out,
                                  cudaStream_t st) {
  const UpParams p = make_up_params(g);
  const long long per_bh = (long long)g.N * p.vpr, bh_total = (long long)g.B * g.heads;
  if (per_bh * bh_total == 0) return cudaSuccess;
  const long long chunk = ((1ll << 31) - 1) / per_bh;
  if (chunk < 1) return cudaErrorInvalidValue;
  for (long long b0 = 0; b0 < bh_total; b0 += chunk) {
    const long long nb = bh_total - b0 < chunk ? bh_total - b0 : chunk;
    const uint32_t total = (uint32_t)(nb * per_bh);
    const size_t full = (size_t)b0 * g.N * p.vpr, pooled = (size_t)b0 * g.Np * p.vpr;
    UpParams q = p;
    q.bh_offset = (int)b0;
    upsample_blend_kernel<<<grid_for(total, 256), 256, 0, st>>>(q, FastDiv(p.vpr), FastDiv(g.N),
                                                              (const uint4*)o_p + pooled, (const uint4*)o_l + full,
                                                              gvec, (uint4*)out + full, total);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Learned variant of the symmetric global branch ("UltraGen ..." §4.2):
// compression by a depthwise convolution whose stride equals its
// p_t x p_h x p_w kernel, restoration by the upsampling above followed by a
// 3 x 3 x 3 depthwise convolution (zero padding).  Weights are fp32, taps-major
// ([heads][taps][d]) so that one thread's 8 (or 4) channels of one tap are
// contiguous.  All HBM-bound except the restoring convolution, whose 27 taps
// read the fp32 upsampled field U mostly from L1 / L2.
// ---------------------------------------------------------------------------

struct CompressWeights {
  const float* w[3];
};

// One thread: one 16-byte vector (8 channels) of one pooled row of one
// tensor; fp32 sum over the taps in (dt, dy, dx) order, one RNE to bf16.
__global__ void __launch_bounds__(256) compress_kernel(PoolParams p, FastDiv per_row, FastDiv n_prow,
                                                        FastDiv rows_per_tensor, PoolTensors ts, CompressWeights cw,
                                                        int heads, int bh0, int* err) {
  const uint32_t total = (uint32_t)ts.count * rows_per_tensor.d * p.vpr;
  const uint32_t stride = gridDim.x * blockDim.x;
  const int taps = (int)(p.pt * p.ph * p.pw), d = (int)p.vpr * 8;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint32_t row2 = per_row.div(i);
    const uint32_t c = i - row2 * p.vpr;
    const uint32_t which = rows_per_tensor.div(row2);
    const uint32_t row = row2 - which * rows_per_tensor.d;
    const uint32_t bh = n_prow.div(row);
    const uint32_t u = row - bh * p.Np;
    const uint32_t r = p.PW.div(u);
    const uint32_t ux = u - r * p.PWv;
    const uint32_t ut = p.PH.div(r);
    const uint32_t uy = r - ut * p.PHv;
    const uint4* src = ts.src[which] + (size_t)bh * p.N * p.vpr + c;
    const float* wt = cw.w[which] + (size_t)((bh0 + (int)bh) % heads) * taps * d + c * 8;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    int tap = 0;
    for (uint32_t a = 0; a < p.pt; ++a)
      for (uint32_t b = 0; b < p.ph; ++b)
        for (uint32_t x = 0; x < p.pw; ++x, ++tap) {
          const uint32_t m = coords_to_tiled(p.rp, ut * p.pt + a, uy * p.ph + b, ux * p.pw + x);
          if (!dcheck(m < p.N, err)) continue;
          const uint4 v = __ldg(src + (size_t)m * p.vpr);
          const float4 w0 = __ldg(reinterpret_cast<const float4*>(wt + (size_t)tap * d));
          const float4 w1 = __ldg(reinterpret_cast<const float4*>(wt + (size_t)tap * d) + 1);
          const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] = fmaf(wv[2 * e], bf16lo(vv[e]), acc[2 * e]);
            acc[2 * e + 1] = fmaf(wv[2 * e + 1], bf16hi(vv[e]), acc[2 * e + 1]);
          }
        }
    uint4 o;
    o.x = pack_bf16(acc[0], acc[1]);
    o.y = pack_bf16(acc[2], acc[3]);
    o.z = pack_bf16(acc[4], acc[5]);
    o.w = pack_bf16(acc[6], acc[7]);
    if (!dcheck(u < p.Np, err)) continue;
    ts.dst[which][((size_t)bh * p.Np + u) * p.vpr + c] = o;
  }
}

cudaError_t launch_compress_qkv(const DevGeom& g, const void* q, const void* k, const void* v, const float* wq,
                                const float* wk, const float* wv, void* qp, void* kp, void* vp, cudaStream_t st) {
  PoolParams p = make_pool_params(g);
  const int count = 3;
  const long long per_bh = (long long)g.Np * p.vpr;
  const long long bh_total = (long long)g.B * g.heads;
  if (per_bh * bh_total == 0) return cudaSuccess;
  if (g.d % 8 != 0) return cudaErrorInvalidValue;
  const long long chunk = ((1ll << 31) - 1) / (per_bh * count);  // every launch below 2^31 vectors
  if (chunk < 1) return cudaErrorInvalidValue;
  const void* src[3] = {q, k, v};
  void* dst[3] = {qp, kp, vp};
  CompressWeights cw;
  cw.w[0] = wq;
  cw.w[1] = wk;
  cw.w[2] = wv;
  for (long long b0 = 0; b0 < bh_total; b0 += chunk) {
    const long long nb = bh_total - b0 < chunk ? bh_total - b0 : chunk;
    const uint32_t rows = (uint32_t)(nb * g.Np);
    const size_t in_off = (size_t)b0 * g.N * p.vpr, out_off = (size_t)b0 * g.Np * p.vpr;
    PoolTensors ts;
    ts.count = count;
    for (int i = 0; i < 3; ++i) {
      ts.src[i] = (const uint4*)src[i] + in_off;
      ts.dst[i] = (uint4*)dst[i] + out_off;
    }
    const int grid = grid_for((long long)count * rows * p.vpr, 256);
    compress_kernel<<<grid, 256, 0, st>>>(p, FastDiv(p.vpr), FastDiv(g.Np), FastDiv(rows), ts, cw, g.heads,
                                          (int)b0, current_ctl().err_word);
  }
  return cudaGetLastError();
}

// U = upsample(O_p) rounded to bf16, raster rows; one thread per 8 channels
// of a row (bf16 halves the restoring convolution's staging traffic; O_p is
// bf16 already).
__global__ void __launch_bounds__(256) upsample_raster_kernel(UpParams p, FastDiv per_row, FastDiv n_rows,
                                                               const uint4* __restrict__ op, uint4* __restrict__ u,
                                                               uint32_t total) {
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint32_t row = per_row.div(i);
    const uint32_t c = i - row * p.vpr;
    const uint32_t bh = n_rows.div(row);
    const uint32_t n = row - bh * p.N;  // raster token
    const uint32_t ty = p.rp.W.div(n);
    const uint32_t x = n - ty * p.rp.Ww;
    const uint32_t t = p.rp.H.div(ty);
    const uint32_t y = ty - t * p.rp.Hh;
    const Interp it = interp_of(t, p.pt, p.PT), iy = interp_of(y, p.ph, p.PH), ix = interp_of(x, p.pw, p.PW);
    const uint4* base = op + (size_t)bh * p.Np * p.vpr + c;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const float w = (a ? it.f : 1.f - it.f) * (b ? iy.f : 1.f - iy.f) * (cc ? ix.f : 1.f - ix.f);
          if (w == 0.f) continue;
          const int src = ((a ? it.i1 : it.i0) * p.PH + (b ? iy.i1 : iy.i0)) * p.PW + (cc ? ix.i1 : ix.i0);
          const uint4 v = __ldg(base + (size_t)src * p.vpr);
          const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] += w * bf16lo(vv[e]);
            acc[2 * e + 1] += w * bf16hi(vv[e]);
          }
        }
    u[(size_t)row * p.vpr + c] = make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]),
                                            pack_bf16(acc[4], acc[5]), pack_bf16(acc[6], acc[7]));
  }
}

// O[tok] = g*O_l[tok] + (1 - g)*conv3(U)[tok], tile-major out.  conv3: sum
// over the 27 taps (a, b, e) of w3[h][tap][c] * U[t + a, y + b, x + e][c],
// zero outside the grid.  One CTA: one (batch*head, t), CONV_Y rows of
// CONV_X voxels, CONV_C channels.  The bf16 U box it reads (3 x (CONV_Y + 2) x
// (CONV_X + 2) voxels x CONV_C channels) arrives in shared memory by one
// 5-D tensor-map copy (zero-filled outside the grid), so each U value is read
// from L2 about 4.8 times (the halo) instead of 27 and no thread spends
// instructions on staging.  Each thread computes CONV_Y outputs (one x, four
// channels) down a column: per (t offset a, x offset e) it holds the three
// y-taps' weights and reads each of the CONV_Y + 2 box rows once, unpacked
// once and applied to every output row it feeds (sum order a, e, b).
constexpr int CONV_X = 32, CONV_Y = 4, CONV_C = 32, CONV_THREADS = 256;
constexpr int CONV_MIN_CTAS = 4;  // 64 registers: four CTAs per SM
constexpr int CONV_BX = CONV_X + 2, CONV_BY = CONV_Y + 2;
constexpr int CONV_BOX = 3 * CONV_BY * CONV_BX * CONV_C * 2;
constexpr int CONV_SMEM = CONV_BOX + 16 + 128;  // box, barrier and abort flag, alignment slack

__global__ void __launch_bounds__(CONV_THREADS, CONV_MIN_CTAS)
    conv3_blend_kernel(const __grid_constant__ CUtensorMap tm_u, UpParams p, const float* __restrict__ w3,
                       const uint2* __restrict__ ol, const float* __restrict__ gvec, uint2* __restrict__ out,
                       int tiles_x, int tiles_y, int chunks_c, DevCtl ctl) {
  extern __shared__ __align__(128) uint8_t conv_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(conv_raw) + 127) & ~uintptr_t(127));
  const uint2* box = reinterpret_cast<const uint2*>(sm);  // [3][CONV_BY][CONV_BX][CONV_C / 4]: 4 bf16 channels each
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + CONV_BOX);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CONV_BOX + 8);
  const int H = (int)p.rp.Hh, W = (int)p.rp.Ww;
  const int d = (int)p.vpr * 8;
  const uint32_t bh = blockIdx.y;
  int rest = blockIdx.x;
  const int cchunk = rest % chunks_c;
  rest /= chunks_c;
  const int xt = rest % tiles_x;
  rest /= tiles_x;
  const int yt = rest % tiles_y;
  const int t = rest / tiles_y;
  const int x0 = xt * CONV_X, y0 = yt * CONV_Y, c0 = cchunk * CONV_C;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // voxel (a, b, e) of the box holds U[t - 1 + a, y0 - 1 + b, x0 - 1 + e]; the
  // innermost coordinate c0 is a multiple of 32 channels (64 bytes)
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, CONV_BOX);
    tma_load_5d(sm, &tm_u, bar, c0, x0 - 1, y0 - 1, t - 1, (int)bh);
  }
  WaitCtx wc;
  wc.abort_flag = abort_flag;
  wc.timeout_ns = ctl.timeout_ns;
  wc.err_word = ctl.err_word;
  const bool landed = __syncthreads_and(mbar_wait(bar, 0, wc));
  if (!landed) {  // let the copy in flight finish before the CTA releases its shared memory
    if (threadIdx.x == 0) mbar_wait_drain(bar, 0, wc);
    return;
  }
  const int q = threadIdx.x % (CONV_C / 4);   // channel quad
  const int xl = threadIdx.x / (CONV_C / 4);  // 0 .. CONV_X - 1
  const int x = x0 + xl;
  const float* wb = w3 + (size_t)((int)(bh + p.bh_offset) % p.heads) * 27 * d + c0 + q * 4;
  float4 acc[CONV_Y];
#pragma unroll
  for (int r = 0; r < CONV_Y; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int e = 0; e < 3; ++e) {
      float4 wv[3];
#pragma unroll
      for (int b = 0; b < 3; ++b) wv[b] = __ldg(reinterpret_cast<const float4*>(wb + (size_t)((a * 3 + b) * 3 + e) * d));
#pragma unroll
      for (int j = 0; j < CONV_BY; ++j) {
        const uint2 uv = box[((a * CONV_BY + j) * CONV_BX + xl + e) * (CONV_C / 4) + q];
        const float u0 = bf16lo(uv.x), u1 = bf16hi(uv.x), u2 = bf16lo(uv.y), u3 = bf16hi(uv.y);
#pragma unroll
        for (int b = 0; b < 3; ++b) {
          const int r = j - b;
          if (r < 0 || r >= CONV_Y) continue;
          acc[r].x = fmaf(wv[b].x, u0, acc[r].x);
          acc[r].y = fmaf(wv[b].y, u1, acc[r].y);
          acc[r].z = fmaf(wv[b].z, u2, acc[r].z);
          acc[r].w = fmaf(wv[b].w, u3, acc[r].w);
        }
      }
    }
  if (x >= W) return;
  const float gh = gvec[(bh + p.bh_offset) % p.heads];
  const uint32_t v2 = p.vpr * 2;  // 8-byte (4-channel) vectors per row
#pragma unroll
  for (int r = 0; r < CONV_Y; ++r) {
    const int y = y0 + r;
    if (y >= H) break;
    const size_t row = (size_t)bh * p.N + coords_to_tiled(p.rp, (uint32_t)t, (uint32_t)y, (uint32_t)x);
    const size_t idx = row * v2 + (c0 >> 2) + q;
    const uint2 l = __ldg(ol + idx);
    out[idx] = make_uint2(pack_bf16(gh * bf16lo(l.x) + (1.f - gh) * acc[r].x, gh * bf16hi(l.x) + (1.f - gh) * acc[r].y),
                          pack_bf16(gh * bf16lo(l.y) + (1.f - gh) * acc[r].z, gh * bf16hi(l.y) + (1.f - gh) * acc[r].w));
  }
}

cudaError_t launch_upsample_conv3_blend(const DevGeom& g, const void* o_p, void* u, const float* w3,
                                        const void* o_l, const float* gvec, void* out, cudaStream_t st) {
  const UpParams p = make_up_params(g);
  const long long bh_total = (long long)g.B * g.heads;
  const long long per_bh8 = (long long)g.N * p.vpr;
  if (per_bh8 * bh_total == 0) return cudaSuccess;
  if (g.d % CONV_C != 0) return cudaErrorInvalidValue;
  const int tiles_x = (g.W + CONV_X - 1) / CONV_X, tiles_y = (g.H + CONV_Y - 1) / CONV_Y, chunks_c = g.d / CONV_C;
  const long long ctas = (long long)g.T * tiles_y * tiles_x * chunks_c;
  if (ctas >= (1ll << 31)) return cudaErrorInvalidValue;
  const long long chunk = ((1ll << 31) - 1) / per_bh8;
  if (chunk < 1) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(conv3_blend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CONV_SMEM);
  if (e != cudaSuccess) return e;
  const DevCtl ctl = current_ctl();
  for (long long b0 = 0; b0 < bh_total; b0 += chunk) {
    const long long nb = bh_total - b0 < chunk ? bh_total - b0 : chunk;
    if (nb > 65535) return cudaErrorInvalidValue;  // grid.y; batch*heads < 65536 is checked up front
    UpParams q = p;
    q.bh_offset = (int)b0;
    const size_t pooled = (size_t)b0 * g.Np * p.vpr, full8 = (size_t)b0 * g.N * p.vpr;
    const uint32_t total8 = (uint32_t)(nb * per_bh8);
    upsample_raster_kernel<<<grid_for(total8, 256), 256, 0, st>>>(q, FastDiv(p.vpr), FastDiv(g.N),
                                                                 (const uint4*)o_p + pooled, (uint4*)u + full8,
                                                                 total8);
    CUtensorMap tm;
    const char* err = nullptr;
    if (!make_tmap_conv_box(&tm, (const uint4*)u + full8, g.d, g, nb, CONV_C, CONV_BX, CONV_BY, 3, &err))
      return cudaErrorInvalidValue;
    conv3_blend_kernel<<<dim3((unsigned)ctas, (unsigned)nb), CONV_THREADS, CONV_SMEM, st>>>(
        tm, q, w3, (const uint2*)o_l + 2 * full8, gvec, (uint2*)out + 2 * full8, tiles_x, tiles_y, chunks_c, ctl);
  }
  return cudaGetLastError();
}

cudaError_t launch_upsample_transpose(const DevGeom& g, const void* dout, const float* gvec, void* dop,
                                      cudaStream_t st) {
  const UpParams p = make_up_params(g);
  const long long per_bh = (long long)g.Np * p.vpr, bh_total = (long long)g.B * g.heads;
  if (per_bh * bh_total == 0) return cudaSuccess;
  if (per_bh * bh_total >= (1ll << 31)) return cudaErrorInvalidValue;
  const uint32_t total = (uint32_t)(per_bh * bh_total);
  upsample_transpose_kernel<<<grid_for(total, 256), 256, 0, st>>>(p, FastDiv(p.vpr), FastDiv(g.Np),
                                                                 (const uint4*)dout, gvec, (uint4*)dop, total);
  return cudaGetLastError();
}

}  // namespace vattn
