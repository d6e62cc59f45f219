// Host-side helpers shared by the entry points of liblsa: argument checks,
// per-device launch facts and the driver's tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lsa.h"

namespace lsa {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Number of SMs of the current device (cached per device), or -1 without a device.
int device_sm_count();

// Records the last CUDA error as LSA_ERR_CUDA (clearing it), or returns LSA_OK.
int launch_status();

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library does not link libcuda directly, so it loads on machines
// without a driver).  Returns nullptr when the driver is unavailable.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

}  // namespace lsa

unsigned* lsa_device_status_ptr();
