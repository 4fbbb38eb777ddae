// Attention backward (placeholder until the tcgen05 backward kernels land).
#include "common.cuh"

namespace vattn {

cudaError_t launch_bwd_preprocess(const DevGeom&, const BwdArgs&, bool, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_bwd_dq(const DevGeom&, const BwdArgs&, bool, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_bwd_dkdv_local(const DevGeom&, const BwdArgs&, bool, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_bwd_dkdv_global(const DevGeom&, const BwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace vattn
