// vca_host.h -- host-side helpers shared by the vca entry points: error
// strings, tensor-map encoding through the driver entry point, the wait limit.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "../../include/vca.h"

namespace vca {

void set_error(const char* fmt, ...);
int fail(int code, const char* fmt, ...);
uint64_t wait_limit_ns();

// Returns VCA_OK or VCA_ERR_CUDA after a kernel launch.
int check_launch(const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// cuTensorMapEncodeTiled through cudaGetDriverEntryPoint (no link to libcuda).
int encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle);

}  // namespace vca
