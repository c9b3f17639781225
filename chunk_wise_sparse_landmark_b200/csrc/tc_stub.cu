// Temporary: tensor-core prefill kernels not yet built.
#include "launch.h"
namespace hils {
cudaError_t launch_qcal_tc(const Shape&, const void*, const void*, const void*, const void*, int, int, void*,
                           cudaStream_t, const DevCtx&) { return cudaErrorNotSupported; }
}  // namespace hils
