// C-ABI entry points: argument validation, workspace carving, TMA descriptor
// encoding and kernel launches on the caller's stream.  No device memory is
// allocated here.
#include <atomic>
#include <cstdarg>
#include <mutex>
#include <cstdio>
#include <cstring>
#include <string>

#include "common.cuh"

namespace vattn {

__device__ int g_error_word = 0;

static thread_local std::string t_last_error;
static std::atomic<int> s_debug_flags{0};  // VATTN_DEBUG_* bits
static std::atomic<long long> s_timeout_ns{2000000000ll};

// ---------------------------------------------------------------------------
// Device addresses of the library's __device__ variables, per CUDA context.
// A variable has one address per context that loaded the module, so a cache
// keyed on the device index would hand out a dangling address once the
// caller makes another context current (a framework's own context, or the
// primary context recreated after cudaDeviceReset).  The key is the context's
// unique id (cuCtxGetId, never reused within the process), fetched through
// the driver entry points like the tensor-map encoder.
// ---------------------------------------------------------------------------
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

static bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

cudaError_t context_symbol_address(const void* symbol, void** out) {
  struct Entry {
    unsigned long long ctx;
    const void* symbol;
    void* addr;
  };
  constexpr int kEntries = 64;
  static Entry table[kEntries] = {};
  static int used = 0, next = 0;
  static std::mutex mu;
  unsigned long long id = 0;
  if (current_context_id(&id)) {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < used; ++i)
      if (table[i].ctx == id && table[i].symbol == symbol) {
        *out = table[i].addr;
        return cudaSuccess;
      }
  }
  // Miss (or no context yet): resolve, which also creates the primary
  // context when none is current, then record under the now-current id.
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, symbol);
  if (e != cudaSuccess) return e;
  if (p == nullptr) return cudaErrorInvalidSymbol;
  if (current_context_id(&id)) {
    std::lock_guard<std::mutex> lk(mu);
    int slot;
    if (used < kEntries) {
      slot = used++;
    } else {  // full: overwrite round robin (an evicted entry is resolved again)
      slot = next;
      next = (next + 1) % kEntries;
    }
    table[slot] = Entry{id, symbol, p};
  }
  *out = p;
  return cudaSuccess;
}

// Address of the current context's status word.
static int* error_word_ptr() {
  void* p = nullptr;
  if (context_symbol_address(reinterpret_cast<const void*>(&g_error_word), &p) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

DevCtl current_ctl() {
  DevCtl c;
  c.timeout_ns = (unsigned long long)s_timeout_ns.load();
  c.err_word = error_word_ptr();
  c.debug_flags = s_debug_flags.load();
  return c;
}

static int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
static int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

int record_error(int code, const char* msg) {
  t_last_error = msg ? msg : "";
  return code;
}

static int ok() {
  t_last_error.clear();
  return VATTN_OK;
}

static int cuda_fail(cudaError_t e, const char* what) {
  return fail(VATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point (no link-time
// dependency on libcuda)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_tmap_rows(CUtensorMap* map, const void* base, int d, long long rows_per_bh, long long bh, int box_rows,
                    const char** err) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    *err = "cuTensorMapEncodeTiled unavailable";
    return false;
  }
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows_per_bh, (cuuint64_t)bh};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows_per_bh * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed";
    return false;
  }
  return true;
}

bool make_tmap_raster(CUtensorMap* map, const void* base, int d, const DevGeom& g, long long bh, int box_t,
                      const char** err) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    *err = "cuTensorMapEncodeTiled unavailable";
    return false;
  }
  const cuuint64_t row = (cuuint64_t)d * 2;
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T, (cuuint64_t)bh};
  cuuint64_t strides[4] = {row, row * g.W, row * g.W * g.H, row * g.W * g.H * g.T};
  cuuint32_t box[5] = {64, (cuuint32_t)g.tw, (cuuint32_t)g.th, (cuuint32_t)box_t, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed";
    return false;
  }
  return true;
}

// Raster [bh][T][H][W][d] bf16 as a 5-D map with an unswizzled box of
// box_c channels x box_x x box_y x box_t voxels of one slice: the box lands in
// shared memory densely, channels fastest, and reads zeros outside the grid.
bool make_tmap_conv_box(CUtensorMap* map, const void* base, int d, const DevGeom& g, long long bh, int box_c,
                        int box_x, int box_y, int box_t, const char** err) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    *err = "cuTensorMapEncodeTiled unavailable";
    return false;
  }
  const cuuint64_t row = (cuuint64_t)d * 2;
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T, (cuuint64_t)bh};
  cuuint64_t strides[4] = {row, row * g.W, row * g.W * g.H, row * g.W * g.H * g.T};
  cuuint32_t box[5] = {(cuuint32_t)box_c, (cuuint32_t)box_x, (cuuint32_t)box_y, (cuuint32_t)box_t, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed";
    return false;
  }
  return true;
}

// The same for rows of `d` bytes (e4m3): box = 128 bytes x box_rows x 1.
bool make_tmap_rows_u8(CUtensorMap* map, const void* base, int d, long long rows_per_bh, long long bh, int box_rows,
                       const char** err) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    *err = "cuTensorMapEncodeTiled unavailable";
    return false;
  }
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows_per_bh, (cuuint64_t)bh};
  cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)rows_per_bh * d};
  cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed";
    return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// validation
// ---------------------------------------------------------------------------
enum Need { NEED_TILE = 1, NEED_POOL = 2, NEED_ATTN = 4 };

static int build_geom(const vattn_geom* in, int need, DevGeom* g) {
  if (!in) return fail(VATTN_ERR_INVALID_ARG, "geom is NULL");
  if (in->batch < 0 || in->heads < 0) return fail(VATTN_ERR_INVALID_ARG, "batch/heads must be >= 0");
  if (in->T <= 0 || in->H <= 0 || in->W <= 0) return fail(VATTN_ERR_INVALID_ARG, "T, H, W must be > 0");
  for (int i = 0; i < 3; ++i) {
    if (in->tile[i] <= 0 || in->window[i] <= 0) return fail(VATTN_ERR_INVALID_ARG, "tile/window must be > 0");
    if ((need & NEED_POOL) && in->pool[i] <= 0) return fail(VATTN_ERR_INVALID_ARG, "pool must be > 0");
  }
  if (in->T % in->tile[0] || in->H % in->tile[1] || in->W % in->tile[2])
    return fail(VATTN_ERR_SHAPE, "grid %dx%dx%d not divisible by tile %dx%dx%d", in->T, in->H, in->W, in->tile[0],
                in->tile[1], in->tile[2]);
  if ((need & NEED_POOL) && (in->T % in->pool[0] || in->H % in->pool[1] || in->W % in->pool[2]))
    return fail(VATTN_ERR_SHAPE, "grid %dx%dx%d not divisible by pool %dx%dx%d", in->T, in->H, in->W, in->pool[0],
                in->pool[1], in->pool[2]);
  const long long N = (long long)in->T * in->H * in->W;
  if (N >= (1ll << 31)) return fail(VATTN_ERR_UNSUPPORTED, "N = T*H*W must be < 2^31");
  if ((need & NEED_ATTN) && in->head_dim != 64 && in->head_dim != 128)
    return fail(VATTN_ERR_UNSUPPORTED, "head_dim %lld not supported (64 or 128)", (long long)in->head_dim);
  if (in->head_dim <= 0 || in->head_dim > 4096) return fail(VATTN_ERR_INVALID_ARG, "head_dim out of range");
  if (in->batch >= 65536 || in->heads >= 65536 || in->batch * in->heads >= 65536)
    return fail(VATTN_ERR_UNSUPPORTED, "batch*heads must be < 65536");
  g->B = (int)in->batch;
  g->heads = (int)in->heads;
  g->d = (int)in->head_dim;
  g->N = (int)N;
  g->T = in->T;
  g->H = in->H;
  g->W = in->W;
  g->tt = in->tile[0];
  g->th = in->tile[1];
  g->tw = in->tile[2];
  g->wt = in->window[0];
  g->wh = in->window[1];
  g->ww = in->window[2];
  g->pt = (need & NEED_POOL) ? in->pool[0] : 1;
  g->ph = (need & NEED_POOL) ? in->pool[1] : 1;
  g->pw = (need & NEED_POOL) ? in->pool[2] : 1;
  g->Nt = g->T / g->tt;
  g->Nh = g->H / g->th;
  g->Nw = g->W / g->tw;
  g->s = g->tt * g->th * g->tw;
  g->n_tiles = g->Nt * g->Nh * g->Nw;
  g->kept = win_extent(g->wt, g->Nt) * win_extent(g->wh, g->Nh) * win_extent(g->ww, g->Nw);
  g->wmode = WIN_SLIDING;
  g->PT = g->T / g->pt;
  g->PH = g->H / g->ph;
  g->PW = g->W / g->pw;
  g->Np = g->PT * g->PH * g->PW;
  if ((need & NEED_ATTN) && g->s % 16 != 0)
    return fail(VATTN_ERR_UNSUPPORTED, "tile volume %d must be a multiple of 16", g->s);
  return VATTN_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE_PTR(p)                                                                  \
  do {                                                                                  \
    if (!(p)) return fail(VATTN_ERR_INVALID_ARG, "%s is NULL", #p);                     \
    if (!aligned16(p)) return fail(VATTN_ERR_ALIGN, "%s is not 16-byte aligned", #p);   \
  } while (0)

#define CHECK_LAUNCH(expr, what)                 \
  do {                                           \
    cudaError_t e_ = (expr);                     \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

static inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static bool empty_geom(const DevGeom& g) { return (long long)g.B * g.heads == 0; }

struct DualFwdWs {
  size_t o_l, kp, vp, total;
};
static DualFwdWs dual_fwd_ws(const DevGeom& g) {
  DualFwdWs w;
  const size_t bh = (size_t)g.B * g.heads;
  w.o_l = 0;
  w.kp = align256(bh * g.N * g.d * 2);
  w.vp = w.kp + align256(bh * g.Np * g.d * 2);
  w.total = w.vp + align256(bh * g.Np * g.d * 2);
  return w;
}
// Backward workspace: per-row D and prescaled LSE for each branch, the pooled
// branch's fp32 dK_p/dV_p, and the fp32 global-branch part of dQ.
struct BwdWs {
  size_t ndelta_l, nlse2_l, ndelta_g, nlse2_g, dkp, dvp, dq_acc, total;
};
static BwdWs bwd_ws(const DevGeom& g, bool dual) {
  BwdWs w;
  const size_t bh = (size_t)g.B * g.heads;
  const size_t row = align256(bh * g.N * 4);
  w.ndelta_l = 0;
  w.nlse2_l = row;
  if (!dual) {
    w.ndelta_g = w.nlse2_g = w.dkp = w.dvp = w.dq_acc = w.total = 2 * row;
    return w;
  }
  w.ndelta_g = 2 * row;
  w.nlse2_g = 3 * row;
  w.dkp = 4 * row;
  w.dvp = w.dkp + align256(bh * g.Np * g.d * 4);
  w.dq_acc = w.dvp + align256(bh * g.Np * g.d * 4);
  w.total = w.dq_acc + align256(bh * g.N * g.d * 4);
  return w;
}

struct SymFwdWs {
  size_t o_l, qp, kp, vp, o_p, total;
};
static SymFwdWs sym_fwd_ws(const DevGeom& g) {
  SymFwdWs w;
  const size_t bh = (size_t)g.B * g.heads;
  const size_t pooled = align256(bh * g.Np * g.d * 2);
  w.o_l = 0;
  w.qp = align256(bh * g.N * g.d * 2);
  w.kp = w.qp + pooled;
  w.vp = w.kp + pooled;
  w.o_p = w.vp + pooled;
  w.total = w.o_p + pooled;
  return w;
}
struct SymLearnedWs {
  size_t o_l, qp, kp, vp, o_p, u, total;
};
static SymLearnedWs sym_learned_ws(const DevGeom& g) {
  SymLearnedWs w;
  const SymFwdWs f = sym_fwd_ws(g);
  const size_t bh = (size_t)g.B * g.heads;
  w.o_l = f.o_l;
  w.qp = f.qp;
  w.kp = f.kp;
  w.vp = f.vp;
  w.o_p = f.o_p;
  w.u = f.total;
  w.total = w.u + align256(bh * g.N * g.d * 2);
  return w;
}
struct SymBwdWs {
  size_t dop, ndelta_l, nlse2_l, ndelta_p, nlse2_p, dkp, dvp, dqp, total;
};
static SymBwdWs sym_bwd_ws(const DevGeom& g) {
  SymBwdWs w;
  const size_t bh = (size_t)g.B * g.heads;
  const size_t row = align256(bh * g.N * 4), prow = align256(bh * g.Np * 4), pf = align256(bh * g.Np * g.d * 4);
  w.dop = 0;
  w.ndelta_l = align256(bh * g.Np * g.d * 2);
  w.nlse2_l = w.ndelta_l + row;
  w.ndelta_p = w.nlse2_l + row;
  w.nlse2_p = w.ndelta_p + prow;
  w.dkp = w.nlse2_p + prow;
  w.dvp = w.dkp + pf;
  w.dqp = w.dvp + pf;
  w.total = w.dqp + pf;
  return w;
}

// FP8 forward: e4m3 Q, K bytes and the per-batch*head absmax words.
struct Fp8FwdWs {
  size_t q8, k8, v8, amax, vamax, total;
};
static Fp8FwdWs fp8_fwd_ws(const DevGeom& g) {
  Fp8FwdWs w;
  const size_t bh = (size_t)g.B * g.heads;
  const size_t t = align256(bh * g.N * g.d);
  w.q8 = 0;
  w.k8 = t;
  w.v8 = 2 * t;
  w.amax = 3 * t;
  w.vamax = w.amax + align256(bh * 2 * 4);
  w.total = w.vamax + align256(bh * 4);
  return w;
}

// FP8 dual forward, in the order the header documents.
struct DualFp8Ws {
  size_t q8, k8, v8, kp8, vp8, amax_l, amax_g, vamax_l, vamax_g, o_l, kp, vp, total;
};
static DualFp8Ws dual_fp8_ws(const DevGeom& g) {
  DualFp8Ws w;
  const size_t bh = (size_t)g.B * g.heads;
  const size_t t8 = align256(bh * g.N * g.d), p8 = align256(bh * g.Np * g.d), am = align256(bh * 2 * 4),
               av = align256(bh * 4);
  w.q8 = 0;
  w.k8 = t8;
  w.v8 = 2 * t8;
  w.kp8 = 3 * t8;
  w.vp8 = w.kp8 + p8;
  w.amax_l = w.vp8 + p8;
  w.amax_g = w.amax_l + am;
  w.vamax_l = w.amax_g + am;
  w.vamax_g = w.vamax_l + av;
  w.o_l = w.vamax_g + av;
  w.kp = w.o_l + align256(bh * g.N * g.d * 2);
  w.vp = w.kp + align256(bh * g.Np * g.d * 2);
  w.total = w.vp + align256(bh * g.Np * g.d * 2);
  return w;
}

// Hierarchical forward: medium-pooled K, V (coarse tile-major), then the
// fine-key O and LSE that the coarse pass merges with.
struct HierFwdWs {
  size_t kh, vh, o_f, lse_f, total;
};
static HierFwdWs hier_fwd_ws(const DevGeom& g) {
  HierFwdWs w;
  const size_t bh = (size_t)g.B * g.heads;
  const size_t kv = align256(bh * g.Np * g.d * 2);
  w.kh = 0;
  w.vh = kv;
  w.o_f = 2 * kv;
  w.lse_f = w.o_f + align256(bh * g.N * g.d * 2);
  w.total = w.lse_f + align256(bh * g.N * 4);
  return w;
}

// Hierarchical backward: pooled K, V (bf16, coarse tile-major), -D and -L
// rows, fp32 dK/dV of the pooled keys, fp32 coarse part of dQ.
struct HierBwdWs {
  size_t kh, vh, ndelta, nlse2, dkh, dvh, dq_acc, total;
};
static HierBwdWs hier_bwd_ws(const DevGeom& g) {
  HierBwdWs w;
  const size_t bh = (size_t)g.B * g.heads;
  const size_t kv = align256(bh * g.Np * g.d * 2), row = align256(bh * g.N * 4), kvf = align256(bh * g.Np * g.d * 4);
  w.kh = 0;
  w.vh = kv;
  w.ndelta = 2 * kv;
  w.nlse2 = w.ndelta + row;
  w.dkh = w.nlse2 + row;
  w.dvh = w.dkh + kvf;
  w.dq_acc = w.dvh + kvf;
  w.total = w.dq_acc + align256(bh * g.N * g.d * 4);
  return w;
}

// Device staging of one chunk of the host-buffer forward: raster Q, K, V,
// tile-major Q, K, V, O, LSE, and raster O, LSE.
struct HostChunkWs {
  size_t qr, kr, vr, qt, kt, vt, ot, lt, orr, lr, total;
};
static HostChunkWs host_chunk_ws(const DevGeom& g) {
  HostChunkWs w;
  const size_t bh = (size_t)g.B * g.heads;
  const size_t t = align256(bh * g.N * g.d * 2), l = align256(bh * g.N * 4);
  w.qr = 0;
  w.kr = t;
  w.vr = 2 * t;
  w.qt = 3 * t;
  w.kt = 4 * t;
  w.vt = 5 * t;
  w.ot = 6 * t;
  w.orr = 7 * t;
  w.lt = 8 * t;
  w.lr = 8 * t + l;
  w.total = 8 * t + 2 * l;
  return w;
}

// Library streams and events of the host-buffer pipeline, one set per device.
struct HostPipe {
  cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
  cudaEvent_t last = nullptr;  // the previous call's end on these streams
  std::mutex mu;
  bool ready = false;
};
static HostPipe* host_pipe(int dev) {
  static HostPipe pipes[64];
  if (dev < 0 || dev >= 64) return nullptr;
  return &pipes[dev];
}
// Destroys whatever streams and events `p` holds (the caller has waited for
// their work) and returns the first error met.
static cudaError_t host_pipe_release(HostPipe& p) {
  cudaError_t first = cudaSuccess;
  auto keep = [&first](cudaError_t e) {
    if (first == cudaSuccess) first = e;
  };
  for (cudaStream_t* s : {&p.in, &p.comp, &p.out}) {
    if (*s) keep(cudaStreamDestroy(*s));
    *s = nullptr;
  }
  cudaEvent_t* evs[] = {&p.start, &p.last, &p.in_done[0], &p.in_done[1], &p.comp_done[0], &p.comp_done[1],
                        &p.out_done[0], &p.out_done[1]};
  for (cudaEvent_t* ev : evs) {
    if (*ev) keep(cudaEventDestroy(*ev));
    *ev = nullptr;
  }
  p.ready = false;
  return first;
}

static cudaError_t host_pipe_init(HostPipe& p) {
  if (p.ready) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  auto ok_so_far = [&e](cudaError_t r) { return (e = r) == cudaSuccess; };
  bool made = ok_so_far(cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking)) &&
              ok_so_far(cudaStreamCreateWithFlags(&p.comp, cudaStreamNonBlocking)) &&
              ok_so_far(cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking)) &&
              ok_so_far(cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming)) &&
              ok_so_far(cudaEventCreateWithFlags(&p.last, cudaEventDisableTiming));
  for (int i = 0; made && i < 2; ++i)
    made = ok_so_far(cudaEventCreateWithFlags(&p.in_done[i], cudaEventDisableTiming)) &&
           ok_so_far(cudaEventCreateWithFlags(&p.comp_done[i], cudaEventDisableTiming)) &&
           ok_so_far(cudaEventCreateWithFlags(&p.out_done[i], cudaEventDisableTiming));
  if (!made) {  // nothing was used yet: drop what was created
    host_pipe_release(p);
    return e;
  }
  p.ready = true;
  return cudaSuccess;
}

// The pooled grid seen as a token sequence of its own (queries = pooled rows).
static DevGeom pooled_as_tokens(const DevGeom& g) {
  DevGeom p = g;
  p.N = g.Np;
  return p;
}

}  // namespace vattn

using namespace vattn;

extern "C" {

const char* vattn_version(void) { return "vattn 0.1.0 (sm_100a)"; }

const char* vattn_last_error(void) { return t_last_error.c_str(); }

int vattn_debug_set(int flags, int64_t timeout_ns) {
  s_debug_flags.store(flags);
  s_timeout_ns.store(timeout_ns > 0 ? (long long)timeout_ns : 2000000000ll);
  return ok();
}

int vattn_debug_exp2(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0) return fail(VATTN_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return ok();
  REQUIRE_PTR(x);
  REQUIRE_PTR(y);
  CHECK_LAUNCH(launch_exp2_poly(x, y, n, (cudaStream_t)stream), "debug_exp2 launch");
  return ok();
}

int vattn_debug_query_blocks(const vattn_geom* geom, int window_mode, int32_t* out, int64_t capacity,
                             int64_t* n_blocks) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_ATTN, &g);
  if (r) return r;
  if (window_mode < WIN_SLIDING || window_mode > WIN_SHIFTED) return fail(VATTN_ERR_INVALID_ARG, "bad window mode");
  REQUIRE_PTR(n_blocks);
  if (capacity > 0) REQUIRE_PTR(out);
  g.wmode = window_mode;
  const PairPlan pp = make_pair_plan(g, g.Nw, true);
  const int qbpt = (g.s + 127) / 128;
  const long long n = pair_plan_active(pp) ? pair_plan_blocks(g, pp) : (long long)g.n_tiles * qbpt;
  *n_blocks = n;
  for (long long b = 0; b < n && b < capacity; ++b) {
    QueryBlock qb;
    if (pair_plan_active(pp)) {
      qb = paired_query_block(g, pp, (int)b);
    } else {
      qb.tile = (int)(b / qbpt);
      qb.sub = (int)(b - (long long)qb.tile * qbpt);
      qb.row0 = qb.tile * g.s + qb.sub * 128;
      qb.valid = g.s - qb.sub * 128 < 128 ? g.s - qb.sub * 128 : 128;
      qb.straddle = 0;
    }
    out[4 * b] = qb.row0;
    out[4 * b + 1] = qb.valid;
    out[4 * b + 2] = qb.straddle;
    out[4 * b + 3] = qb.tile;
  }
  return ok();
}

int vattn_get_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pending CUDA error");
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (word != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    return fail(word, "device reported status %d (a bounded wait ran out)", word);
  }
  return ok();
}

int vattn_shutdown(void) {
  int prev = -1;
  int code = VATTN_OK;
  std::string msg;
  for (int dev = 0; dev < 64; ++dev) {
    HostPipe& p = *host_pipe(dev);
    std::lock_guard<std::mutex> lk(p.mu);
    if (!p.ready) continue;
    if (prev < 0 && cudaGetDevice(&prev) != cudaSuccess) prev = 0;
    cudaError_t e = cudaSetDevice(dev);
    if (e == cudaSuccess) {
      // wait for the pipeline's copies and kernels before the handles go
      for (cudaStream_t s : {p.in, p.comp, p.out}) {
        const cudaError_t r = cudaStreamSynchronize(s);
        if (e == cudaSuccess) e = r;
      }
      const cudaError_t r = host_pipe_release(p);
      if (e == cudaSuccess) e = r;
    }
    if (e != cudaSuccess && code == VATTN_OK) {
      code = VATTN_ERR_CUDA;
      msg = std::string("shutdown of the host pipeline on device ") + std::to_string(dev) + ": " +
            cudaGetErrorString(e);
    }
  }
  if (prev >= 0) cudaSetDevice(prev);
  if (code != VATTN_OK) return record_error(code, msg.c_str());
  return ok();
}

int vattn_workspace_size(int op, const vattn_geom* geom, size_t* bytes) {
  if (!bytes) return fail(VATTN_ERR_INVALID_ARG, "bytes is NULL");
  DevGeom g;
  int need = NEED_TILE | NEED_ATTN | (op == VATTN_OP_STA_BWD ? 0 : NEED_POOL);
  int r = build_geom(geom, need, &g);
  if (r) return r;
  switch (op) {
    case VATTN_OP_DUAL_FWD: *bytes = dual_fwd_ws(g).total; break;
    case VATTN_OP_STA_BWD: *bytes = bwd_ws(g, false).total; break;
    case VATTN_OP_DUAL_BWD: *bytes = bwd_ws(g, true).total; break;
    case VATTN_OP_DUAL_SYM_FWD: *bytes = sym_fwd_ws(g).total; break;
    case VATTN_OP_DUAL_SYM_BWD: *bytes = sym_bwd_ws(g).total; break;
    case VATTN_OP_DUAL_SYM_LEARNED_FWD: *bytes = sym_learned_ws(g).total; break;
    case VATTN_OP_STA_FWD_HOST: *bytes = host_chunk_ws(g).total; break;
    case VATTN_OP_HIER_FWD: *bytes = hier_fwd_ws(g).total; break;
    case VATTN_OP_HIER_BWD: *bytes = hier_bwd_ws(g).total; break;
    case VATTN_OP_STA_FWD_FP8: *bytes = fp8_fwd_ws(g).total; break;
    case VATTN_OP_DUAL_FWD_FP8: *bytes = dual_fp8_ws(g).total; break;
    default: return fail(VATTN_ERR_INVALID_ARG, "unknown op %d", op);
  }
  return ok();
}

int vattn_tile_permute(const vattn_geom* geom, const void* src, void* dst, int64_t row_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE, &g);
  if (r) return r;
  if (row_bytes <= 0 || row_bytes % 4) return fail(VATTN_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 4");
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(src);
  REQUIRE_PTR(dst);
  if (src == dst) return fail(VATTN_ERR_INVALID_ARG, "src and dst must not overlap");
  CHECK_LAUNCH(launch_permute(g, src, dst, row_bytes, true, (cudaStream_t)stream), "tile_permute launch");
  return ok();
}

int vattn_tile_unpermute(const vattn_geom* geom, const void* src, void* dst, int64_t row_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE, &g);
  if (r) return r;
  if (row_bytes <= 0 || row_bytes % 4) return fail(VATTN_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 4");
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(src);
  REQUIRE_PTR(dst);
  if (src == dst) return fail(VATTN_ERR_INVALID_ARG, "src and dst must not overlap");
  CHECK_LAUNCH(launch_permute(g, src, dst, row_bytes, false, (cudaStream_t)stream), "tile_unpermute launch");
  return ok();
}

int vattn_kept_tiles(const vattn_geom* geom, int32_t* out, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE, &g);
  if (r) return r;
  REQUIRE_PTR(out);
  CHECK_LAUNCH(launch_kept_tiles(g, out, (cudaStream_t)stream), "kept_tiles launch");
  return ok();
}

int vattn_sta_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale, void* o,
                  float* lse, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_ATTN, &g);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(o);
  if (lse && !aligned16(lse)) return fail(VATTN_ERR_ALIGN, "lse is not 16-byte aligned");
  FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.scale = scale;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, a, (cudaStream_t)stream), "sta_fwd launch");
  return ok();
}

int vattn_xwin_fwd(const vattn_geom* geom, int shifted, const void* q, const void* k, const void* v, float scale,
                   void* o, float* lse, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_ATTN, &g);
  if (r) return r;
  if (shifted != 0 && shifted != 1) return fail(VATTN_ERR_INVALID_ARG, "shifted must be 0 or 1");
  g.wmode = shifted ? WIN_SHIFTED : WIN_PARTITION;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(o);
  if (lse && !aligned16(lse)) return fail(VATTN_ERR_ALIGN, "lse is not 16-byte aligned");
  FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.scale = scale;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, a, (cudaStream_t)stream), "xwin_fwd launch");
  return ok();
}

}  // extern "C"

// Enqueues the chunk pipeline of vattn_sta_fwd_host on the library streams.
static int sta_fwd_host_enqueue(HostPipe& p, const DevGeom& g, const DevGeom& gc, const HostChunkWs& w, const void* q,
                                const void* k, const void* v, float scale, void* o, float* lse, long long chunk_slices,
                                void* workspace, cudaStream_t caller) {
  const long long total = (long long)g.B * g.heads;
  CHECK_LAUNCH(cudaEventRecord(p.start, caller), "event record");
  // the library streams also wait for the previous call's end (its caller may
  // have used another stream): its staging slots are reused below.  Waiting
  // on a never-recorded event is a no-op.
  CHECK_LAUNCH(cudaStreamWaitEvent(p.in, p.last, 0), "stream wait");
  CHECK_LAUNCH(cudaStreamWaitEvent(p.comp, p.last, 0), "stream wait");
  CHECK_LAUNCH(cudaStreamWaitEvent(p.in, p.start, 0), "stream wait");
  CHECK_LAUNCH(cudaStreamWaitEvent(p.comp, p.start, 0), "stream wait");
  CHECK_LAUNCH(cudaStreamWaitEvent(p.out, p.start, 0), "stream wait");
  const size_t row = (size_t)g.N * g.d * 2, lrow = (size_t)g.N * 4;
  const int nchunks = (int)((total + chunk_slices - 1) / chunk_slices);
  // the tile reorder fused into the kernel when the t-slice allows it
  int G = 1;
  while (G < 128 && g.s % (G * 2) == 0) G *= 2;
  const bool raster = 128 % (g.th * g.tw) == 0 && G % (g.th * g.tw) == 0;
  for (int c = 0; c < nchunks; ++c) {
    const int slot = c & 1;
    const long long s0 = (long long)c * chunk_slices;
    const long long ns = total - s0 < chunk_slices ? total - s0 : chunk_slices;
    DevGeom gk = gc;
    gk.heads = (int)ns;
    uint8_t* ws = (uint8_t*)workspace + slot * w.total;
    // the slot's inputs are free once the compute two chunks back is done; its
    // outputs once that chunk's copy-out is done
    if (c >= 2) {
      CHECK_LAUNCH(cudaStreamWaitEvent(p.in, p.comp_done[slot], 0), "stream wait");
      CHECK_LAUNCH(cudaStreamWaitEvent(p.comp, p.out_done[slot], 0), "stream wait");
    }
    const size_t bytes = (size_t)ns * row;
    CHECK_LAUNCH(cudaMemcpyAsync(ws + w.qr, (const uint8_t*)q + s0 * row, bytes, cudaMemcpyHostToDevice, p.in), "H2D q");
    CHECK_LAUNCH(cudaMemcpyAsync(ws + w.kr, (const uint8_t*)k + s0 * row, bytes, cudaMemcpyHostToDevice, p.in), "H2D k");
    CHECK_LAUNCH(cudaMemcpyAsync(ws + w.vr, (const uint8_t*)v + s0 * row, bytes, cudaMemcpyHostToDevice, p.in), "H2D v");
    CHECK_LAUNCH(cudaEventRecord(p.in_done[slot], p.in), "event record");
    CHECK_LAUNCH(cudaStreamWaitEvent(p.comp, p.in_done[slot], 0), "stream wait");
    if (raster) {
      FwdArgs a{};
      a.q = ws + w.qr;
      a.k = ws + w.kr;
      a.v = ws + w.vr;
      a.o = ws + w.orr;
      a.lse = lse ? (float*)(ws + w.lr) : nullptr;
      a.scale = scale;
      a.raster = true;
      CHECK_LAUNCH(launch_attn_fwd(gk, FWD_STA, a, p.comp), "sta_fwd (raster)");
    } else {
      CHECK_LAUNCH(launch_permute(gk, ws + w.qr, ws + w.qt, g.d * 2, true, p.comp), "permute q");
      CHECK_LAUNCH(launch_permute(gk, ws + w.kr, ws + w.kt, g.d * 2, true, p.comp), "permute k");
      CHECK_LAUNCH(launch_permute(gk, ws + w.vr, ws + w.vt, g.d * 2, true, p.comp), "permute v");
      FwdArgs a{};
      a.q = ws + w.qt;
      a.k = ws + w.kt;
      a.v = ws + w.vt;
      a.o = ws + w.ot;
      a.lse = lse ? (float*)(ws + w.lt) : nullptr;
      a.scale = scale;
      CHECK_LAUNCH(launch_attn_fwd(gk, FWD_STA, a, p.comp), "sta_fwd");
      CHECK_LAUNCH(launch_permute(gk, ws + w.ot, ws + w.orr, g.d * 2, false, p.comp), "unpermute o");
      if (lse) CHECK_LAUNCH(launch_permute(gk, ws + w.lt, ws + w.lr, 4, false, p.comp), "unpermute lse");
    }
    CHECK_LAUNCH(cudaEventRecord(p.comp_done[slot], p.comp), "event record");
    CHECK_LAUNCH(cudaStreamWaitEvent(p.out, p.comp_done[slot], 0), "stream wait");
    CHECK_LAUNCH(cudaMemcpyAsync((uint8_t*)o + s0 * row, ws + w.orr, bytes, cudaMemcpyDeviceToHost, p.out), "D2H o");
    if (lse)
      CHECK_LAUNCH(cudaMemcpyAsync((uint8_t*)lse + s0 * lrow, ws + w.lr, (size_t)ns * lrow, cudaMemcpyDeviceToHost, p.out),
                   "D2H lse");
    CHECK_LAUNCH(cudaEventRecord(p.out_done[slot], p.out), "event record");
  }
  // the caller's stream waits for every copy-out (and therefore for everything)
  for (int slot = 0; slot < 2 && slot < nchunks; ++slot)
    CHECK_LAUNCH(cudaStreamWaitEvent(caller, p.out_done[slot], 0), "stream wait");
  CHECK_LAUNCH(cudaEventRecord(p.last, p.out), "event record");
  return ok();
}

extern "C" int vattn_sta_fwd_host(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale,
                                  void* o, float* lse, int64_t chunk_slices, void* workspace, size_t ws_bytes,
                                  void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_ATTN, &g);
  if (r) return r;
  if (empty_geom(g)) return ok();
  if (!q || !k || !v || !o) return fail(VATTN_ERR_INVALID_ARG, "q, k, v and o must be non-NULL host pointers");
  const long long total = (long long)g.B * g.heads;
  if (chunk_slices <= 0 || chunk_slices > total) return fail(VATTN_ERR_INVALID_ARG, "chunk_slices out of range");
  DevGeom gc = g;  // one chunk: batch 1, heads = chunk_slices (the attention path has no per-head state here)
  gc.B = 1;
  gc.heads = (int)chunk_slices;
  const HostChunkWs w = host_chunk_ws(gc);
  if (!workspace || ws_bytes < 2 * w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", 2 * w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  int dev = 0;
  CHECK_LAUNCH(cudaGetDevice(&dev), "cudaGetDevice");
  HostPipe* pp = host_pipe(dev);
  if (!pp) return fail(VATTN_ERR_UNSUPPORTED, "device index out of range");
  std::lock_guard<std::mutex> lk(pp->mu);
  CHECK_LAUNCH(host_pipe_init(*pp), "pipeline stream/event creation");
  r = sta_fwd_host_enqueue(*pp, g, gc, w, q, k, v, scale, o, lse, chunk_slices, workspace, (cudaStream_t)stream);
  if (r != VATTN_OK) {
    // part of the pipeline may be in flight, and `last` does not cover it:
    // let it finish, so that no later call reuses a staging slot under it
    const std::string msg = t_last_error;
    cudaStreamSynchronize(pp->in);
    cudaStreamSynchronize(pp->comp);
    cudaStreamSynchronize(pp->out);
    record_error(r, msg.c_str());
  }
  return r;
}

extern "C" {

// Fine geometry (pool = h_pool) and the coarse grid: the medium-pooled grid
// cut into tiles of the same shape.
static int build_hier(const vattn_geom* geom, DevGeom* g, DevGeom* gc) {
  int r = build_geom(geom, NEED_TILE | NEED_POOL | NEED_ATTN, g);
  if (r) return r;
  if (g->Nt % g->pt || g->Nh % g->ph || g->Nw % g->pw)
    return fail(VATTN_ERR_SHAPE, "tiles per dim %dx%dx%d not divisible by the hierarchical pool %dx%dx%d", g->Nt, g->Nh,
                g->Nw, g->pt, g->ph, g->pw);
  vattn_geom c = *geom;
  c.T = geom->T / geom->pool[0];
  c.H = geom->H / geom->pool[1];
  c.W = geom->W / geom->pool[2];
  c.pool[0] = c.pool[1] = c.pool[2] = 1;
  return build_geom(&c, NEED_TILE | NEED_ATTN, gc);
}

int vattn_hier_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale, void* o,
                   float* lse, void* workspace, size_t ws_bytes, void* stream) {
  DevGeom g, gc;
  int r = build_hier(geom, &g, &gc);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(o);
  if (lse && !aligned16(lse)) return fail(VATTN_ERR_ALIGN, "lse is not 16-byte aligned");
  const HierFwdWs w = hier_fwd_ws(g);
  if (!workspace || ws_bytes < w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  uint8_t* ws = (uint8_t*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  CHECK_LAUNCH(launch_pool_kv_tiled(g, gc, k, v, ws + w.kh, ws + w.vh, st), "hier_fwd pool launch");
  FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = ws + w.o_f;
  a.lse = (float*)(ws + w.lse_f);
  a.scale = scale;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, a, st), "hier_fwd fine launch");
  FwdArgs b{};
  b.q = q;
  b.k = ws + w.kh;
  b.v = ws + w.vh;
  b.o = o;
  b.lse = lse;
  b.scale = scale;
  b.kgeom = &gc;
  b.cf[0] = g.pt;
  b.cf[1] = g.ph;
  b.cf[2] = g.pw;
  b.merge_o = ws + w.o_f;
  b.merge_lse = (const float*)(ws + w.lse_f);
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, b, st), "hier_fwd coarse launch");
  return ok();
}

int vattn_hier_bwd(const vattn_geom* geom, const void* q, const void* k, const void* v, const void* o,
                   const float* lse, const void* dout, float scale, void* dq, void* dk, void* dv, void* workspace,
                   size_t ws_bytes, void* stream) {
  DevGeom g, gc;
  int r = build_hier(geom, &g, &gc);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(o);
  REQUIRE_PTR(lse);
  REQUIRE_PTR(dout);
  REQUIRE_PTR(dq);
  REQUIRE_PTR(dk);
  REQUIRE_PTR(dv);
  const HierBwdWs w = hier_bwd_ws(g);
  if (!workspace || ws_bytes < w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  uint8_t* ws = (uint8_t*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  CHECK_LAUNCH(launch_pool_kv_tiled(g, gc, k, v, ws + w.kh, ws + w.vh, st), "hier_bwd pool launch");
  float* ndelta = (float*)(ws + w.ndelta);
  float* nlse2 = (float*)(ws + w.nlse2);
  CHECK_LAUNCH(launch_preprocess_branch(g, dout, o, lse, nullptr, ndelta, nlse2, st), "hier_bwd preprocess launch");
  BwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.kp = ws + w.kh;
  a.vp = ws + w.vh;
  a.dout = dout;
  a.scale = scale;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.ndelta_l = a.ndelta_g = ndelta;  // one softmax over both key sets
  a.nlse2_l = a.nlse2_g = nlse2;
  a.dkp = (float*)(ws + w.dkh);
  a.dvp = (float*)(ws + w.dvh);
  a.dq_acc = (float*)(ws + w.dq_acc);
  a.dq_acc_pooled = false;
  CHECK_LAUNCH(launch_bwd_dkdv_hier(g, gc, a, true, st), "hier_bwd coarse dK/dV launch");
  CHECK_LAUNCH(launch_bwd_dkdv_hier(g, gc, a, false, st), "hier_bwd fine dK/dV launch");
  CHECK_LAUNCH(launch_bwd_dq_hier(g, gc, a, st), "hier_bwd coarse dQ launch");
  CHECK_LAUNCH(launch_bwd_dq(g, a, true, st), "hier_bwd fine dQ launch");
  return ok();
}

int vattn_sta_fwd_raster(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale, void* o,
                         float* lse, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_ATTN, &g);
  if (r) return r;
  const int slice = g.th * g.tw;
  int G = 1;
  while (G < 128 && g.s % (G * 2) == 0) G *= 2;
  if (128 % slice || G % slice)
    return fail(VATTN_ERR_UNSUPPORTED, "tile t-slice of %d tokens must divide 128 and the key sub-box of %d rows", slice,
                G);
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(o);
  if (lse && !aligned16(lse)) return fail(VATTN_ERR_ALIGN, "lse is not 16-byte aligned");
  FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.scale = scale;
  a.raster = true;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, a, (cudaStream_t)stream), "sta_fwd_raster launch");
  return ok();
}

int vattn_dual_fwd_fp8(const vattn_geom* geom, const void* q, const void* k, const void* v, const float* gvec, float scale,
                       void* o, void* workspace, size_t ws_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_POOL | NEED_ATTN, &g);
  if (r) return r;
  if (g.d != 128) return fail(VATTN_ERR_UNSUPPORTED, "the FP8 forward supports head_dim 128 only");
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(gvec);
  REQUIRE_PTR(o);
  const DualFp8Ws w = dual_fp8_ws(g);
  if (!workspace || ws_bytes < w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  uint8_t* ws = (uint8_t*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  const long long bh = (long long)g.B * g.heads;
  int* amax_l = (int*)(ws + w.amax_l);
  int* amax_g = (int*)(ws + w.amax_g);
  int* vamax_l = (int*)(ws + w.vamax_l);
  int* vamax_g = (int*)(ws + w.vamax_g);
  CHECK_LAUNCH(launch_pool_kv(g, k, v, ws + w.kp, ws + w.vp, st), "dual_fwd_fp8 pool launch");
  CHECK_LAUNCH(launch_quant_e4m3(q, g.N, bh, g.d, ws + w.q8, amax_l, 2, st), "dual_fwd_fp8 quantise Q launch");
  CHECK_LAUNCH(launch_quant_e4m3(k, g.N, bh, g.d, ws + w.k8, amax_l + 1, 2, st), "dual_fwd_fp8 quantise K launch");
  CHECK_LAUNCH(launch_quant_e4m3(v, g.N, bh, g.d, ws + w.v8, vamax_l, 1, st), "dual_fwd_fp8 quantise V launch");
  CHECK_LAUNCH(launch_quant_e4m3(ws + w.kp, g.Np, bh, g.d, ws + w.kp8, amax_g + 1, 2, st),
               "dual_fwd_fp8 quantise K_p launch");
  CHECK_LAUNCH(launch_quant_e4m3(ws + w.vp, g.Np, bh, g.d, ws + w.vp8, vamax_g, 1, st),
               "dual_fwd_fp8 quantise V_p launch");
  // the global pass's Q scale: the same absmax as the local pass's
  CHECK_LAUNCH(cudaMemcpy2DAsync(amax_g, 2 * sizeof(int), amax_l, 2 * sizeof(int), sizeof(int), bh,
                                 cudaMemcpyDeviceToDevice, st),
               "dual_fwd_fp8 scale copy");
  FwdArgs a{};
  a.q = ws + w.q8;
  a.k = ws + w.k8;
  a.v = ws + w.v8;
  a.o = ws + w.o_l;
  a.scale = scale;
  a.qk_amax = amax_l;
  a.v_amax = vamax_l;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, a, st), "dual_fwd_fp8 local launch");
  FwdArgs b{};
  b.q = ws + w.q8;
  b.k = ws + w.kp8;
  b.v = ws + w.vp8;
  b.scale = scale;
  b.o_local = ws + w.o_l;
  b.g = gvec;
  b.blend_out = o;
  b.qk_amax = amax_g;
  b.v_amax = vamax_g;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_GLOBAL, b, st), "dual_fwd_fp8 global launch");
  return ok();
}

int vattn_sta_fwd_fp8(const vattn_geom* geom, const void* q, const void* k, const void* v, float scale, void* o,
                      float* lse, void* workspace, size_t ws_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_ATTN, &g);
  if (r) return r;
  if (g.d != 128) return fail(VATTN_ERR_UNSUPPORTED, "the FP8 forward supports head_dim 128 only");
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(o);
  if (lse && !aligned16(lse)) return fail(VATTN_ERR_ALIGN, "lse is not 16-byte aligned");
  const Fp8FwdWs w = fp8_fwd_ws(g);
  if (!workspace || ws_bytes < w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  uint8_t* ws = (uint8_t*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  int* amax = (int*)(ws + w.amax);
  const long long bh = (long long)g.B * g.heads;
  CHECK_LAUNCH(launch_quant_e4m3(q, g.N, bh, g.d, ws + w.q8, amax, 2, st), "sta_fwd_fp8 quantise Q launch");
  CHECK_LAUNCH(launch_quant_e4m3(k, g.N, bh, g.d, ws + w.k8, amax + 1, 2, st), "sta_fwd_fp8 quantise K launch");
  int* vamax = (int*)(ws + w.vamax);
  CHECK_LAUNCH(launch_quant_e4m3(v, g.N, bh, g.d, ws + w.v8, vamax, 1, st), "sta_fwd_fp8 quantise V launch");
  FwdArgs a{};
  a.q = ws + w.q8;
  a.k = ws + w.k8;
  a.v = ws + w.v8;
  a.o = o;
  a.lse = lse;
  a.scale = scale;
  a.qk_amax = amax;
  a.v_amax = vamax;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, a, st), "sta_fwd_fp8 launch");
  return ok();
}

int vattn_pool_kv(const vattn_geom* geom, const void* k, const void* v, void* kp, void* vp, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_POOL, &g);
  if (r) return r;
  if (g.d % 8) return fail(VATTN_ERR_UNSUPPORTED, "head_dim must be a multiple of 8");
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(kp);
  REQUIRE_PTR(vp);
  CHECK_LAUNCH(launch_pool_kv(g, k, v, kp, vp, (cudaStream_t)stream), "pool_kv launch");
  return ok();
}

int vattn_global_fwd(const vattn_geom* geom, const void* q, const void* kp, const void* vp, float scale, void* o,
                     float* lse, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_POOL | NEED_ATTN, &g);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(kp);
  REQUIRE_PTR(vp);
  REQUIRE_PTR(o);
  if (lse && !aligned16(lse)) return fail(VATTN_ERR_ALIGN, "lse is not 16-byte aligned");
  FwdArgs a{};
  a.q = q;
  a.k = kp;
  a.v = vp;
  a.o = o;
  a.lse = lse;
  a.scale = scale;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_GLOBAL, a, (cudaStream_t)stream), "global_fwd launch");
  return ok();
}

int vattn_dual_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v, const float* gvec,
                   float scale, void* o, void* o_l, float* lse_l, void* o_g, float* lse_g, void* kp, void* vp,
                   void* workspace, size_t ws_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_POOL | NEED_ATTN, &g);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(gvec);
  REQUIRE_PTR(o);
  const int n_saved = (o_l != nullptr) + (lse_l != nullptr) + (o_g != nullptr) + (lse_g != nullptr) +
                      (kp != nullptr) + (vp != nullptr);
  if (n_saved != 0 && n_saved != 6)
    return fail(VATTN_ERR_INVALID_ARG, "o_l, lse_l, o_g, lse_g, kp, vp must be all NULL or all non-NULL");
  cudaStream_t st = (cudaStream_t)stream;
  if (n_saved == 0) {
    const DualFwdWs w = dual_fwd_ws(g);
    if (!workspace || ws_bytes < w.total)
      return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
    if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
    uint8_t* ws = (uint8_t*)workspace;
    o_l = ws + w.o_l;
    kp = ws + w.kp;
    vp = ws + w.vp;
  } else {
    REQUIRE_PTR(o_l);
    REQUIRE_PTR(lse_l);
    REQUIRE_PTR(o_g);
    REQUIRE_PTR(lse_g);
    REQUIRE_PTR(kp);
    REQUIRE_PTR(vp);
  }
  CHECK_LAUNCH(launch_pool_kv(g, k, v, kp, vp, st), "dual_fwd pool launch");
  FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o_l;
  a.lse = lse_l;
  a.scale = scale;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, a, st), "dual_fwd local launch");
  FwdArgs b{};
  b.q = q;
  b.k = kp;
  b.v = vp;
  b.o = o_g;  // NULL at inference: only the blended output is written
  b.lse = lse_g;
  b.scale = scale;
  b.o_local = o_l;
  b.g = gvec;
  b.blend_out = o;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_GLOBAL, b, st), "dual_fwd global launch");
  return ok();
}

int vattn_dual_sym_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v, const float* gvec,
                       float scale, void* o, void* o_l, float* lse_l, void* qp, void* kp, void* vp, void* o_p,
                       float* lse_p, void* workspace, size_t ws_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_POOL | NEED_ATTN, &g);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(gvec);
  REQUIRE_PTR(o);
  const int n_saved = (o_l != nullptr) + (lse_l != nullptr) + (qp != nullptr) + (kp != nullptr) + (vp != nullptr) +
                      (o_p != nullptr) + (lse_p != nullptr);
  if (n_saved != 0 && n_saved != 7)
    return fail(VATTN_ERR_INVALID_ARG, "o_l, lse_l, qp, kp, vp, o_p, lse_p must be all NULL or all non-NULL");
  if (n_saved == 0) {
    const SymFwdWs w = sym_fwd_ws(g);
    if (!workspace || ws_bytes < w.total)
      return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
    if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
    uint8_t* ws = (uint8_t*)workspace;
    o_l = ws + w.o_l;
    qp = ws + w.qp;
    kp = ws + w.kp;
    vp = ws + w.vp;
    o_p = ws + w.o_p;
  } else {
    REQUIRE_PTR(o_l);
    REQUIRE_PTR(lse_l);
    REQUIRE_PTR(qp);
    REQUIRE_PTR(kp);
    REQUIRE_PTR(vp);
    REQUIRE_PTR(o_p);
    REQUIRE_PTR(lse_p);
  }
  cudaStream_t st = (cudaStream_t)stream;
  CHECK_LAUNCH(launch_pool_qkv(g, q, k, v, qp, kp, vp, st), "dual_sym_fwd pool launch");
  FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o_l;
  a.lse = lse_l;
  a.scale = scale;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, a, st), "dual_sym_fwd local launch");
  FwdArgs b{};
  b.q = qp;
  b.k = kp;
  b.v = vp;
  b.o = o_p;
  b.lse = lse_p;
  b.scale = scale;
  CHECK_LAUNCH(launch_attn_fwd(pooled_as_tokens(g), FWD_GLOBAL, b, st), "dual_sym_fwd pooled attention launch");
  CHECK_LAUNCH(launch_upsample_blend(g, o_p, o_l, gvec, o, st), "dual_sym_fwd upsample launch");
  return ok();
}

int vattn_dual_sym_learned_fwd(const vattn_geom* geom, const void* q, const void* k, const void* v,
                               const float* gvec, const float* wq, const float* wk, const float* wv,
                               const float* w3, float scale, void* o, void* workspace, size_t ws_bytes,
                               void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_POOL | NEED_ATTN, &g);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(gvec);
  REQUIRE_PTR(wq);
  REQUIRE_PTR(wk);
  REQUIRE_PTR(wv);
  REQUIRE_PTR(w3);
  REQUIRE_PTR(o);
  if (g.d % 8 != 0) return fail(VATTN_ERR_SHAPE, "head_dim %d is not a multiple of 8", g.d);
  if (!aligned16(wq) || !aligned16(wk) || !aligned16(wv) || !aligned16(w3))
    return fail(VATTN_ERR_ALIGN, "weights are not 16-byte aligned");
  const SymLearnedWs w = sym_learned_ws(g);
  if (!workspace || ws_bytes < w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  uint8_t* ws = (uint8_t*)workspace;
  void* o_l = ws + w.o_l;
  void* qp = ws + w.qp;
  void* kp = ws + w.kp;
  void* vp = ws + w.vp;
  void* o_p = ws + w.o_p;
  void* u = ws + w.u;
  cudaStream_t st = (cudaStream_t)stream;
  CHECK_LAUNCH(launch_compress_qkv(g, q, k, v, wq, wk, wv, qp, kp, vp, st), "dual_sym_learned_fwd compress launch");
  FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o_l;
  a.scale = scale;
  CHECK_LAUNCH(launch_attn_fwd(g, FWD_STA, a, st), "dual_sym_learned_fwd local launch");
  FwdArgs b{};
  b.q = qp;
  b.k = kp;
  b.v = vp;
  b.o = o_p;
  b.scale = scale;
  CHECK_LAUNCH(launch_attn_fwd(pooled_as_tokens(g), FWD_GLOBAL, b, st), "dual_sym_learned_fwd pooled attention launch");
  CHECK_LAUNCH(launch_upsample_conv3_blend(g, o_p, u, w3, o_l, gvec, o, st), "dual_sym_learned_fwd restore launch");
  return ok();
}

int vattn_dual_sym_bwd(const vattn_geom* geom, const void* q, const void* k, const void* v, const float* gvec,
                       const void* o_l, const float* lse_l, const void* qp, const void* kp, const void* vp,
                       const void* o_p, const float* lse_p, const void* dout, float scale, void* dq, void* dk,
                       void* dv, void* workspace, size_t ws_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_POOL | NEED_ATTN, &g);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(gvec);
  REQUIRE_PTR(o_l);
  REQUIRE_PTR(lse_l);
  REQUIRE_PTR(qp);
  REQUIRE_PTR(kp);
  REQUIRE_PTR(vp);
  REQUIRE_PTR(o_p);
  REQUIRE_PTR(lse_p);
  REQUIRE_PTR(dout);
  REQUIRE_PTR(dq);
  REQUIRE_PTR(dk);
  REQUIRE_PTR(dv);
  const SymBwdWs w = sym_bwd_ws(g);
  if (!workspace || ws_bytes < w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  uint8_t* ws = (uint8_t*)workspace;
  void* dop = ws + w.dop;
  cudaStream_t st = (cudaStream_t)stream;
  const DevGeom gp = pooled_as_tokens(g);
  // pooled branch: dO_p = (1-g) * upsample^T(dO), then the pooled attention backward
  CHECK_LAUNCH(launch_upsample_transpose(g, dout, gvec, dop, st), "dual_sym_bwd upsample^T launch");
  CHECK_LAUNCH(launch_preprocess_branch(gp, dop, o_p, lse_p, nullptr, (float*)(ws + w.ndelta_p),
                                        (float*)(ws + w.nlse2_p), st),
               "dual_sym_bwd pooled preprocess launch");
  BwdArgs b{};
  b.q = qp;
  b.kp = kp;
  b.vp = vp;
  b.dout = dop;
  b.scale = scale;
  b.ndelta_g = (float*)(ws + w.ndelta_p);
  b.nlse2_g = (float*)(ws + w.nlse2_p);
  b.dkp = (float*)(ws + w.dkp);
  b.dvp = (float*)(ws + w.dvp);
  b.dq_acc = (float*)(ws + w.dqp);
  CHECK_LAUNCH(launch_bwd_dkdv_global(gp, b, st), "dual_sym_bwd pooled dk/dv launch");
  CHECK_LAUNCH(launch_bwd_dq_global(gp, b, st), "dual_sym_bwd pooled dq launch");
  // local branch (gamma = g), with the pooled gradients added through pool^T
  CHECK_LAUNCH(launch_preprocess_branch(g, dout, o_l, lse_l, gvec, (float*)(ws + w.ndelta_l),
                                        (float*)(ws + w.nlse2_l), st),
               "dual_sym_bwd local preprocess launch");
  BwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.scale = scale;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.ndelta_l = (float*)(ws + w.ndelta_l);
  a.nlse2_l = (float*)(ws + w.nlse2_l);
  a.dkp = (float*)(ws + w.dkp);
  a.dvp = (float*)(ws + w.dvp);
  a.dq_acc = (float*)(ws + w.dqp);
  a.dq_acc_pooled = true;
  CHECK_LAUNCH(launch_bwd_dkdv_local(g, a, true, st), "dual_sym_bwd local dk/dv launch");
  CHECK_LAUNCH(launch_bwd_dq(g, a, true, st), "dual_sym_bwd local dq launch");
  return ok();
}

int vattn_sta_bwd(const vattn_geom* geom, const void* q, const void* k, const void* v, const void* o,
                  const float* lse, const void* dout, float scale, void* dq, void* dk, void* dv, void* workspace,
                  size_t ws_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_ATTN, &g);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(o);
  REQUIRE_PTR(lse);
  REQUIRE_PTR(dout);
  REQUIRE_PTR(dq);
  REQUIRE_PTR(dk);
  REQUIRE_PTR(dv);
  const BwdWs w = bwd_ws(g, false);
  if (!workspace || ws_bytes < w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  BwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.o_l = o;
  a.lse_l = lse;
  a.scale = scale;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.ndelta_l = (float*)((uint8_t*)workspace + w.ndelta_l);
  a.nlse2_l = (float*)((uint8_t*)workspace + w.nlse2_l);
  cudaStream_t st = (cudaStream_t)stream;
  CHECK_LAUNCH(launch_bwd_preprocess(g, a, false, st), "sta_bwd preprocess launch");
  CHECK_LAUNCH(launch_bwd_dkdv_local(g, a, false, st), "sta_bwd dk/dv launch");
  CHECK_LAUNCH(launch_bwd_dq(g, a, false, st), "sta_bwd dq launch");
  return ok();
}

int vattn_xwin_bwd(const vattn_geom* geom, int shifted, const void* q, const void* k, const void* v, const void* o,
                   const float* lse, const void* dout, float scale, void* dq, void* dk, void* dv, void* workspace,
                   size_t ws_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_ATTN, &g);
  if (r) return r;
  if (shifted != 0 && shifted != 1) return fail(VATTN_ERR_INVALID_ARG, "shifted must be 0 or 1");
  g.wmode = shifted ? WIN_SHIFTED : WIN_PARTITION;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(o);
  REQUIRE_PTR(lse);
  REQUIRE_PTR(dout);
  REQUIRE_PTR(dq);
  REQUIRE_PTR(dk);
  REQUIRE_PTR(dv);
  const BwdWs w = bwd_ws(g, false);
  if (!workspace || ws_bytes < w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  BwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.o_l = o;
  a.lse_l = lse;
  a.scale = scale;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.ndelta_l = (float*)((uint8_t*)workspace + w.ndelta_l);
  a.nlse2_l = (float*)((uint8_t*)workspace + w.nlse2_l);
  cudaStream_t st = (cudaStream_t)stream;
  CHECK_LAUNCH(launch_bwd_preprocess(g, a, false, st), "xwin_bwd preprocess launch");
  CHECK_LAUNCH(launch_bwd_dkdv_local(g, a, false, st), "xwin_bwd dk/dv launch");
  CHECK_LAUNCH(launch_bwd_dq(g, a, false, st), "xwin_bwd dq launch");
  return ok();
}

int vattn_dual_bwd(const vattn_geom* geom, const void* q, const void* k, const void* v, const float* gvec,
                   const void* o_l, const float* lse_l, const void* o_g, const float* lse_g, const void* kp,
                   const void* vp, const void* dout, float scale, void* dq, void* dk, void* dv, float* dg,
                   void* workspace, size_t ws_bytes, void* stream) {
  DevGeom g;
  int r = build_geom(geom, NEED_TILE | NEED_POOL | NEED_ATTN, &g);
  if (r) return r;
  if (empty_geom(g)) return ok();
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(gvec);
  REQUIRE_PTR(o_l);
  REQUIRE_PTR(lse_l);
  REQUIRE_PTR(o_g);
  REQUIRE_PTR(lse_g);
  REQUIRE_PTR(kp);
  REQUIRE_PTR(vp);
  REQUIRE_PTR(dout);
  REQUIRE_PTR(dq);
  REQUIRE_PTR(dk);
  REQUIRE_PTR(dv);
  if (dg && !aligned16(dg)) return fail(VATTN_ERR_ALIGN, "dg is not 16-byte aligned");
  const BwdWs w = bwd_ws(g, true);
  if (!workspace || ws_bytes < w.total)
    return fail(VATTN_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(VATTN_ERR_ALIGN, "workspace is not 16-byte aligned");
  BwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.kp = kp;
  a.vp = vp;
  a.dout = dout;
  a.o_l = o_l;
  a.lse_l = lse_l;
  a.o_g = o_g;
  a.lse_g = lse_g;
  a.g = gvec;
  a.scale = scale;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dg = dg;
  uint8_t* ws = (uint8_t*)workspace;
  a.ndelta_l = (float*)(ws + w.ndelta_l);
  a.ndelta_g = (float*)(ws + w.ndelta_g);
  a.nlse2_l = (float*)(ws + w.nlse2_l);
  a.nlse2_g = (float*)(ws + w.nlse2_g);
  a.dkp = (float*)(ws + w.dkp);
  a.dvp = (float*)(ws + w.dvp);
  a.dq_acc = (float*)(ws + w.dq_acc);
  cudaStream_t st = (cudaStream_t)stream;
  CHECK_LAUNCH(launch_bwd_preprocess(g, a, true, st), "dual_bwd preprocess launch");
  CHECK_LAUNCH(launch_bwd_dkdv_global(g, a, st), "dual_bwd global dk/dv launch");
  CHECK_LAUNCH(launch_bwd_dkdv_local(g, a, true, st), "dual_bwd local dk/dv launch");
  CHECK_LAUNCH(launch_bwd_dq_global(g, a, st), "dual_bwd global dq launch");
  CHECK_LAUNCH(launch_bwd_dq(g, a, true, st), "dual_bwd dq launch");
  return ok();
}

}  // extern "C"
