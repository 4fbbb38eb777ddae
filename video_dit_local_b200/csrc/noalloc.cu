// Dual-branch inference forward for callers that cannot allocate device
// memory.
//
// Who needs it: a caller running inside a host framework that has already
// reserved the device's memory through its own pool and gives plug-ins no
// allocation hook (a cudaMalloc from the plug-in fails or fragments that
// pool), and a caller on a latency-critical path that forbids allocation
// after start-up (cudaMalloc/cudaFree may synchronise the device).  Such a
// caller cannot provide the workspace that vattn_dual_fwd needs for its
// intermediates (the local-branch output and the pooled K/V).
//
// What it does: the same computation as vattn_dual_fwd without saved outputs,
// with the workspace taken from a file-scope device array that the library
// holds on every GPU that loads it, until the process exits.  It allocates
// nothing itself.
#include <cstdio>

#include "common.cuh"

namespace vattn {

// Largest workspace this entry point can serve (a single-head 1080p-shaped
// call needs about 52 MB).
constexpr size_t kNoAllocScratchBytes = VATTN_NOALLOC_SCRATCH_BYTES;

// The scratch itself.  In host code `g_noalloc_scratch` names a host-side
// stand-in, not device memory: only the address returned by
// cudaGetSymbolAddress may be handed to kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Set-up, once per CUDA context (the current device's primary context unless
// the caller made another one current): resolve the scratch array's device
// address with cudaGetSymbolAddress.  Later calls in the same context reuse
// the cached address, so the first call in a context must come before any
// stream capture.
int scratch_address(void** out) {
  const cudaError_t e = context_symbol_address(reinterpret_cast<const void*>(&g_noalloc_scratch), out);
  if (e != cudaSuccess) {
    char msg[192];
    snprintf(msg, sizeof(msg), "vattn_dual_fwd_noalloc: cudaGetSymbolAddress of the scratch failed: %s",
             cudaGetErrorString(e));
    return record_error(VATTN_ERR_CUDA, msg);
  }
  return VATTN_OK;
}
}  // namespace

}  // namespace vattn

extern "C" int vattn_dual_fwd_noalloc(const vattn_geom* geom, const void* q, const void* k, const void* v,
                                      const float* g, float scale, void* o, void* stream) {
  using namespace vattn;
  size_t need = 0;
  int r = vattn_workspace_size(VATTN_OP_DUAL_FWD, geom, &need);
  if (r != VATTN_OK) return r;
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "vattn_dual_fwd_noalloc: this geometry needs %zu bytes of scratch but the library's static scratch "
             "holds %zu; call vattn_dual_fwd with a caller-owned workspace instead",
             need, kNoAllocScratchBytes);
    return record_error(VATTN_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  r = scratch_address(&scratch);
  if (r != VATTN_OK) return r;
  // The intermediates (local-branch output, pooled K/V) are fully written
  // before they are read, so the scratch needs no clearing between calls.
  return vattn_dual_fwd(geom, q, k, v, g, scale, o, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, scratch,
                        kNoAllocScratchBytes, stream);
}
