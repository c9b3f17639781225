// Temporary: tensor-core prefill kernels not yet built.
#include "launch.h"
namespace hils {
size_t score_tc_workspace(const Shape&) { return 0; }
cudaError_t launch_score_topk_tc(const Shape&, const void*, const void*, const float*, int32_t*, float*, cudaStream_t,
                                 const DevCtx&) { return cudaErrorNotSupported; }
cudaError_t launch_qcal_tc(const Shape&, const void*, const void*, const void*, const void*, int, int, void*,
                           cudaStream_t, const DevCtx&) { return cudaErrorNotSupported; }
}  // namespace hils
