// Host-side helpers and the small entry points of the fp8qgg C ABI.
#include <mutex>

#include "host_common.h"

namespace fp8qgg {

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_valid[kMaxDevices];
std::mutex g_dev_mutex;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}
}  // namespace

bool device_info(DeviceInfo *out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (!g_dev_valid[dev]) {
    DeviceInfo d{};
    d.device = dev;
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    if (cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) !=
        cudaSuccess)
      return false;
    if (cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) !=
        cudaSuccess)
      return false;
    g_dev[dev] = d;
    g_dev_valid[dev] = true;
  }
  *out = g_dev[dev];
  return true;
}

namespace {
struct SmemAttr {
  int device;
  const void *kernel;
  int bytes;
};
constexpr int kMaxSmemAttrs = 256;
SmemAttr g_smem_attr[kMaxSmemAttrs];
int g_smem_attr_n = 0;
std::mutex g_smem_mutex;
}  // namespace

bool set_max_dynamic_smem(const void *kernel, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(g_smem_mutex);
  for (int i = 0; i < g_smem_attr_n; ++i)
    if (g_smem_attr[i].device == dev && g_smem_attr[i].kernel == kernel &&
        g_smem_attr[i].bytes >= bytes)
      return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  for (int i = 0; i < g_smem_attr_n; ++i)
    if (g_smem_attr[i].device == dev && g_smem_attr[i].kernel == kernel) {
      g_smem_attr[i].bytes = bytes;
      return true;
    }
  if (g_smem_attr_n < kMaxSmemAttrs) g_smem_attr[g_smem_attr_n++] = SmemAttr{dev, kernel, bytes};
  return true;
}

bool encode_tensor_map(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t rank, void *base,
                       const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                       CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[5];
  cuuint64_t s[4];
  cuuint32_t b[5];
  cuuint32_t e[5];
  for (uint32_t i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) s[i] = strides_bytes[i];
  }
  const CUresult r =
      fn(map, dtype, rank, base, d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fp8qgg

extern "C" int fp8_native_format(void) { return FP8QGG_E4M3FN; }

extern "C" const char *fp8qgg_error_string(int code) {
  switch (code) {
    case FP8QGG_OK: return "ok";
    case FP8QGG_ERR_NULL: return "a required pointer is NULL";
    case FP8QGG_ERR_SHAPE: return "bad size, leading dimension or group count";
    case FP8QGG_ERR_ALIGN: return "base pointer or leading dimension misaligned";
    case FP8QGG_ERR_UNSUPPORTED: return "bad flag or unsupported combination";
    case FP8QGG_ERR_CUDA: return "a CUDA runtime or driver call failed";
    default: return "unknown error";
  }
}
