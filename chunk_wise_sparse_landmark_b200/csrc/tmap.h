// Host helper: TMA tensor maps (cuTensorMapEncodeTiled through the runtime's
// driver entry point, so the library needs no link against libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hils {

// Tiled map over a bf16 tensor of `rank` dims (dims[0] innermost, element
// counts), byte strides of dims 1..rank-1, box sizes per dim, and swizzle.
// Returns cudaSuccess or an error (never throws).
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle);

// Multiprocessor count of the current device (queried once per device).
int device_sm_count();

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (device, kernel);
// later calls for the same pair return immediately.
cudaError_t ensure_dynamic_smem(const void* func, int bytes);

}  // namespace hils
