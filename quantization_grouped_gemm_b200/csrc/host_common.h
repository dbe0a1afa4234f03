// Host-side helpers of the fp8qgg C ABI: argument checks, device properties
// and TMA tensor-map encoding through the driver entry point (the library
// does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>

#include "../../include/fp8qgg.h"

namespace fp8qgg {

inline bool aligned(const void *p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

struct DeviceInfo {
  int device;
  int sm_count;
  int cc_major;
  int cc_minor;
};

// Properties of the current device (cached per device ordinal).
bool device_info(DeviceInfo *out);

// cudaFuncSetAttribute(kernel, MaxDynamicSharedMemorySize, bytes) on the
// current device, once per (device, kernel): later calls with no larger size
// skip the runtime call.
bool set_max_dynamic_smem(const void *kernel, int bytes);

// Largest finite magnitude of the encoding.
inline float format_max(int fmt) { return fmt == FP8QGG_E4M3FNUZ ? 240.0f : 448.0f; }

// The scaling maximum: scale_max when > 0, else the format's largest finite.
inline float effective_scale_max(int fmt, float scale_max) {
  return scale_max > 0.0f ? scale_max : format_max(fmt);
}

// Pre-clamp magnitudes above this value are counted as saturated: one fp32
// ulp above the encoding's largest finite value.
inline float saturation_threshold(int fmt) {
  return std::nextafter(format_max(fmt), INFINITY);
}

// cuTensorMapEncodeTiled through cudaGetDriverEntryPoint.  Returns false if
// the entry point is missing or the driver rejects the description.
bool encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t rank,
                       void *base, const uint64_t *dims, const uint64_t *strides_bytes,
                       const uint32_t *box, CUtensorMapSwizzle swizzle);

}  // namespace fp8qgg
