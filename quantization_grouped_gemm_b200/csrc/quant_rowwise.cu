// Rowwise FP8 quantisation: absmax per row -> scale -> clamp -> RNE e4m3 cast,
// in one pass over HBM ("FP8 su GPU AMD: ..." (ai-radar.it): one scale per
// activation row, introduction; the amax/scale/clamp/cast chain, section
// "Il guadagno vero è nel movimento dei dati").
//
// Design (B200): a row is owned by a team of G warps (G = 1, 2, 4 or 8) and is
// held entirely in registers between the absmax and the cast, so each input
// byte crosses HBM once and nothing intermediate is materialised.  Loads are
// 16-byte vectors, consecutive lanes on consecutive vectors (each warp
// instruction covers 512 contiguous bytes).  The absmax runs on the bf16 bit
// patterns with per-halfword unsigned max, then a warp shuffle tree, then
// shared memory across the team.  The grid is persistent (resident blocks x
// SM count) and walks rows with a grid stride.
#include <algorithm>
#include <mutex>

#include "device_common.cuh"
#include "host_common.h"

namespace fp8qgg {

constexpr int kRowThreads = 256;  // 8 warps per block

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int VPL, int G, int FMT, bool FAST>
__global__ void __launch_bounds__(kRowThreads)
    quant_rowwise_kernel(const uint4 *__restrict__ x, int64_t rows, int nvec, int64_t ld_x_vec,
                         uint8_t *__restrict__ q, int64_t ld_q, float *__restrict__ scales,
                         float smax, float sat_thr, unsigned long long *sat_count) {
  constexpr int kTeams = (kRowThreads / 32) / G;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int team = warp / G;
  const int wt = warp % G;
  __shared__ uint32_t red[kRowThreads / 32];
  uint32_t sat = 0;

  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kTeams + team; row < rows;
       row += static_cast<int64_t>(gridDim.x) * kTeams) {
    const uint4 *xr = x + row * ld_x_vec;
    uint4 v[VPL];
    uint32_t am = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int idx = (i * G + wt) * 32 + lane;
      if (idx < nvec) {
        v[i] = __ldcs(xr + idx);
      } else {
        v[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      am = absmax_acc(am, v[i].x);
      am = absmax_acc(am, v[i].y);
      am = absmax_acc(am, v[i].z);
      am = absmax_acc(am, v[i].w);
    }
    am = absmax_bits(am);
    uint32_t m = max(am & 0xFFFFu, am >> 16);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    if constexpr (G > 1) {
      if (lane == 0) red[warp] = m;
      named_bar_sync(1 + team, 32 * G);
      m = 0;
#pragma unroll
      for (int j = 0; j < G; ++j) m = max(m, red[team * G + j]);
      named_bar_sync(1 + team, 32 * G);
    }
    const float s = scale_from_amax(bf16_bits_to_float(m), smax);
    if (wt == 0 && lane == 0) scales[row] = s;

    uint8_t *qr = q + row * ld_q;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int idx = (i * G + wt) * 32 + lane;
      if (idx < nvec) {
        uint2 o;
        if constexpr (FAST) {
          const uint64_t s2 = pack_f32x2(s, s);
          o.x = quant_pair_fast<FMT>(v[i].x, s2) | (quant_pair_fast<FMT>(v[i].y, s2) << 16);
          o.y = quant_pair_fast<FMT>(v[i].z, s2) | (quant_pair_fast<FMT>(v[i].w, s2) << 16);
        } else {
          o.x = quant_pair<FMT>(v[i].x, s, smax, sat_thr, sat) |
                (quant_pair<FMT>(v[i].y, s, smax, sat_thr, sat) << 16);
          o.y = quant_pair<FMT>(v[i].z, s, smax, sat_thr, sat) |
                (quant_pair<FMT>(v[i].w, s, smax, sat_thr, sat) << 16);
        }
        *reinterpret_cast<uint2 *>(qr + static_cast<int64_t>(idx) * 8) = o;
      }
    }
  }
  if (!FAST && sat_count) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(0xFFFFFFFFu, sat, off);
    if (lane == 0 && sat) atomicAdd(sat_count, static_cast<unsigned long long>(sat));
  }
}

namespace {

using RowKernel = void (*)(const uint4 *, int64_t, int, int64_t, uint8_t *, int64_t, float *,
                           float, float, unsigned long long *);

constexpr int kVplChoices[] = {1, 2, 4, 6, 8, 12, 16};
constexpr int kNumVpl = sizeof(kVplChoices) / sizeof(kVplChoices[0]);
constexpr int kGChoices[] = {1, 2, 4, 8};
constexpr int kNumG = 4;

template <int FMT, bool FAST, int GI, int VI>
RowKernel row_kernel_at() {
  return quant_rowwise_kernel<kVplChoices[VI], kGChoices[GI], FMT, FAST>;
}

template <int FMT, bool FAST, int GI, int... VIs>
void fill_row(RowKernel *t, std::integer_sequence<int, VIs...>) {
  ((t[GI * kNumVpl + VIs] = row_kernel_at<FMT, FAST, GI, VIs>()), ...);
}

template <int FMT, bool FAST>
void fill_table(RowKernel *t) {
  fill_row<FMT, FAST, 0>(t, std::make_integer_sequence<int, kNumVpl>{});
  fill_row<FMT, FAST, 1>(t, std::make_integer_sequence<int, kNumVpl>{});
  fill_row<FMT, FAST, 2>(t, std::make_integer_sequence<int, kNumVpl>{});
  fill_row<FMT, FAST, 3>(t, std::make_integer_sequence<int, kNumVpl>{});
}

// [format][fast]: the fast kernels skip the clamp and the saturation count
struct RowTable {
  RowKernel k[2][2][kNumG * kNumVpl];
  RowTable() {
    fill_table<FP8QGG_E4M3FN, false>(k[0][0]);
    fill_table<FP8QGG_E4M3FN, true>(k[0][1]);
    fill_table<FP8QGG_E4M3FNUZ, false>(k[1][0]);
    fill_table<FP8QGG_E4M3FNUZ, true>(k[1][1]);
  }
};

const RowTable &row_table() {
  static RowTable t;
  return t;
}

}  // namespace

// Picks the team size and vectors per lane for a row of nvec 16-byte vectors.
// Returns false when the row is longer than the largest team can hold.
bool rowwise_plan(int64_t nvec, int *gi_out, int *vi_out) {
  for (int gi = 0; gi < kNumG; ++gi) {
    const int64_t per_lane = (nvec + 32 * kGChoices[gi] - 1) / (32 * kGChoices[gi]);
    for (int vi = 0; vi < kNumVpl; ++vi) {
      if (per_lane <= kVplChoices[vi]) {
        *gi_out = gi;
        *vi_out = vi;
        return true;
      }
    }
  }
  return false;
}

}  // namespace fp8qgg

using namespace fp8qgg;

extern "C" int fp8_quant_rowwise(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                                 uint8_t *q, int64_t ld_q, float *scales, int fmt,
                                 float scale_max, uint64_t *sat_count, void *stream) {
  if (rows < 0 || cols < 1 || cols > 32768) return FP8QGG_ERR_SHAPE;
  if (ld_x < cols || ld_q < cols) return FP8QGG_ERR_SHAPE;
  if (fmt != FP8QGG_E4M3FN && fmt != FP8QGG_E4M3FNUZ) return FP8QGG_ERR_UNSUPPORTED;
  if (!(scale_max >= 0.0f) || scale_max > 3.0e38f) return FP8QGG_ERR_UNSUPPORTED;
  if (rows == 0) return FP8QGG_OK;
  if (!x || !q || !scales) return FP8QGG_ERR_NULL;
  if (cols % 8 || ld_x % 8 || ld_q % 8) return FP8QGG_ERR_ALIGN;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scales, 4)) return FP8QGG_ERR_ALIGN;
  if (sat_count && !aligned(sat_count, 8)) return FP8QGG_ERR_ALIGN;

  int gi = 0, vi = 0;
  if (!rowwise_plan(cols / 8, &gi, &vi)) return FP8QGG_ERR_SHAPE;
  const float smax = effective_scale_max(fmt, scale_max);
  const float sat_thr = saturation_threshold(fmt);
  const bool fast = sat_count == nullptr && smax >= format_max(fmt);
  RowKernel kern = row_table().k[fmt][fast ? 1 : 0][gi * kNumVpl + vi];

  DeviceInfo dev;
  if (!device_info(&dev)) return FP8QGG_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRowThreads, 0) !=
      cudaSuccess)
    return FP8QGG_ERR_CUDA;
  per_sm = std::max(per_sm, 1);
  const int teams = (kRowThreads / 32) / kGChoices[gi];
  const int64_t want = (rows + teams - 1) / teams;
  const int grid = static_cast<int>(std::min<int64_t>(want, int64_t(per_sm) * dev.sm_count));

  kern<<<grid, kRowThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4 *>(x), rows, static_cast<int>(cols / 8), ld_x / 8, q, ld_q, scales,
      smax, sat_thr, reinterpret_cast<unsigned long long *>(sat_count));
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}

namespace fp8qgg {

// Elementwise encode of fp32 values (no scaling): 8 values per thread step.
template <int FMT>
__global__ void __launch_bounds__(256) cast_f32_kernel(const float *__restrict__ y, int64_t n,
                                                       uint8_t *__restrict__ q) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t groups = n / 8;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += stride) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __ldcs(y + 8 * g + i);
    uint2 o;
    o.x = cvt_x2<FMT>(v[0], v[1]) | (cvt_x2<FMT>(v[2], v[3]) << 16);
    o.y = cvt_x2<FMT>(v[4], v[5]) | (cvt_x2<FMT>(v[6], v[7]) << 16);
    uint8_t *dst = q + 8 * g;
    if ((reinterpret_cast<uintptr_t>(dst) & 7) == 0) {
      *reinterpret_cast<uint2 *>(dst) = o;
    } else {
      for (int i = 0; i < 8; ++i) dst[i] = static_cast<uint8_t>(((i < 4 ? o.x : o.y) >> (8 * (i & 3))) & 0xFF);
    }
  }
  if (blockIdx.x == 0 && threadIdx.x < n - groups * 8) {
    const int64_t i = groups * 8 + threadIdx.x;
    q[i] = static_cast<uint8_t>(cvt_x2<FMT>(y[i], 0.0f) & 0xFF);
  }
}

}  // namespace fp8qgg

extern "C" int fp8_cast_f32(const float *y, int64_t n, uint8_t *q, int fmt, void *stream) {
  if (n < 0) return FP8QGG_ERR_SHAPE;
  if (fmt != FP8QGG_E4M3FN && fmt != FP8QGG_E4M3FNUZ) return FP8QGG_ERR_UNSUPPORTED;
  if (n == 0) return FP8QGG_OK;
  if (!y || !q) return FP8QGG_ERR_NULL;
  if (!aligned(y, 4)) return FP8QGG_ERR_ALIGN;
  DeviceInfo dev;
  if (!device_info(&dev)) return FP8QGG_ERR_CUDA;
  const int64_t groups = std::max<int64_t>(1, n / 8);
  const int grid = static_cast<int>(std::min<int64_t>((groups + 255) / 256, int64_t(dev.sm_count) * 8));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (fmt == FP8QGG_E4M3FN)
    cast_f32_kernel<FP8QGG_E4M3FN><<<grid, 256, 0, s>>>(y, n, q);
  else
    cast_f32_kernel<FP8QGG_E4M3FNUZ><<<grid, 256, 0, s>>>(y, n, q);
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}
