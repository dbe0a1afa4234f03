// Jagged column-wise FP8 quantisation: for every expert group (rows given by
// the int32 offsets tensor) and every column, absmax -> scale -> clamp -> RNE
// e4m3 cast, in one pass over HBM, with an optional fused transpose.
//
// Sources: "FP8 su GPU AMD: ..." (ai-radar.it) — introduction (one scale per
// column of each expert's weights, an offsets tensor routing tokens), section
// "Il guadagno vero è nel movimento dei dati" (the chain; the backward's
// .t().contiguous().t() copy removed and scale-and-cast fused; the output tile
// of the column-scales kernel transposed on chip so that stores coalesce;
// relaxed atomics for commutative reductions).  "AMD Boosts PyTorch FP8
// Training on Instinct GPUs", third paragraph (same facts).
//
// B200 design.  Work is split into items (group e, 64-column tile, chunk of
// at most 512 rows).  A persistent grid (cooperative launch, so every block
// is resident) walks the items in order with a grid stride.  Per item:
//   1. TMA copies the chunk (bf16, 128 B per row) into shared memory; it is
//      the only HBM read of those bytes.
//   2. Column absmax from shared memory (per-halfword unsigned max on the
//      bf16 magnitude bits, then across warps).
//   3. A group taller than one chunk combines its chunks' partial absmax
//      with relaxed atomicMax in a caller-provided workspace and an arrival
//      counter.  The chunks of one (group, tile) unit are consecutive items,
//      so when there are no more chunks than resident blocks all of them are
//      in flight together and the bounded wait always completes.
//   4. Scale, clamp and cast from shared memory.  SAME layout stores 8-byte
//      runs per row.  TRANSPOSED layout casts into a shared-memory staging
//      tile laid out [column][token], then writes each output row (one
//      column of x) as 16-byte runs along the tokens: consecutive threads,
//      consecutive addresses.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "device_common.cuh"
#include "host_common.h"

namespace fp8qgg {

constexpr int kColThreads = 256;
constexpr int kCW = 64;            // columns per tile: 128 bytes of bf16 per row
constexpr int kBoxRows = 128;      // rows per TMA box (16 KB)
constexpr int kChunkRows = 512;    // rows held on chip per item
constexpr int kMaxGroups = 1024;
constexpr int kStgPitch = 144;     // bytes per staging row: 128 tokens + 16 pad
constexpr int kStgRows = 128;      // tokens per staging block

struct ColSmem {
  uint32_t tile[kChunkRows * kCW / 2];   // [row][32 words], each word = 2 bf16 columns
  uint8_t stg[kCW * kStgPitch];          // [column][token] codes, TRANSPOSED only
  uint32_t red[kColThreads / 32][32];
  uint32_t amax_bits[kCW];
  float scale[kCW];
  int32_t end[kMaxGroups];
  int32_t item_prefix[kMaxGroups + 1];
  uint64_t bar;
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Clamped group ends and the cumulative item count per group, computed by
// warp 0 with shuffle scans.  end_e = min(R, max(0, max_{j<=e} offsets[j]))
// is the closed form of "start_e = end_{e-1}, end_e = clamp(offsets[e],
// start_e, R)".  Each group, empty or not, contributes max(1, chunks) items
// per column tile, so that every (group, tile) writes its scales.
__device__ void build_item_table(ColSmem &sm, const int32_t *offsets, int num_groups,
                                 int64_t rows_total, int n_ct, int32_t *status) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  int32_t carry_end = 0;
  int32_t carry_items = 0;
  bool bad = false;
  const int32_t R = static_cast<int32_t>(rows_total);
  for (int base = 0; base < num_groups; base += 32) {
    const int e = base + lane;
    const int32_t raw = e < num_groups ? __ldg(offsets + e) : INT32_MIN;
    int32_t run = max(raw, 0);
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t o = __shfl_up_sync(0xFFFFFFFFu, run, d);
      if (lane >= d) run = max(run, o);
    }
    const int32_t endv = min(R, max(carry_end, run));
    int32_t prev = __shfl_up_sync(0xFFFFFFFFu, endv, 1);
    if (lane == 0) prev = carry_end;
    if (e < num_groups) {
      if (raw < prev || raw > R) bad = true;
    }
    const int32_t h = endv - prev;
    int32_t items = e < num_groups ? max(1, (h + kChunkRows - 1) / kChunkRows) * n_ct : 0;
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t o = __shfl_up_sync(0xFFFFFFFFu, items, d);
      if (lane >= d) items += o;
    }
    if (e < num_groups) {
      sm.end[e] = endv;
      sm.item_prefix[e + 1] = carry_items + items;
    }
    carry_end = __shfl_sync(0xFFFFFFFFu, endv, 31);
    carry_items += __shfl_sync(0xFFFFFFFFu, items, 31);
  }
  if (lane == 0) sm.item_prefix[0] = 0;
  bad = __any_sync(0xFFFFFFFFu, bad);
  if (bad && lane == 0 && blockIdx.x == 0) status_or(status, FP8QGG_STATUS_BAD_OFFSETS);
}

// Scale and encode two bf16 values that sit in one 32-bit word but belong to
// two different columns (two different scales).
template <int FMT>
__device__ __forceinline__ uint32_t quant_pair2(uint32_t packed, float s0, float s1, float smax,
                                                float sat_thr, uint32_t &sat) {
  const float x0 = __uint_as_float(packed << 16);
  const float x1 = __uint_as_float(packed & 0xFFFF0000u);
  float y0 = __fmul_rn(x0, s0);
  float y1 = __fmul_rn(x1, s1);
  sat += (fabsf(y0) > sat_thr) + (fabsf(y1) > sat_thr);
  y0 = fminf(fmaxf(y0, -smax), smax);
  y1 = fminf(fmaxf(y1, -smax), smax);
  return cvt_x2<FMT>(y0, y1);
}

template <int FMT, int LAYOUT, bool FAST>
__global__ void __launch_bounds__(kColThreads, 2)
    quant_colwise_jagged_kernel(const __grid_constant__ CUtensorMap xmap, int64_t rows_total,
                                int cols, const int32_t *__restrict__ offsets, int num_groups,
                                uint8_t *__restrict__ q, int64_t ld_q,
                                float *__restrict__ scales, float smax, float sat_thr,
                                unsigned long long *sat_count, int32_t *status,
                                uint32_t *__restrict__ ws_amax, uint32_t *__restrict__ ws_cnt) {
  extern __shared__ uint8_t smem_raw[];
  ColSmem &sm = *reinterpret_cast<ColSmem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_ct = (cols + kCW - 1) / kCW;

  if (tid == 0) {
    prefetch_tensormap(&xmap);
    mbar_init(&sm.bar, 1);
    fence_mbarrier_init();
  }
  build_item_table(sm, offsets, num_groups, rows_total, n_ct, status);
  __syncthreads();

  const int32_t total_items = sm.item_prefix[num_groups];
  uint32_t phase = 0;
  uint32_t sat = 0;

  for (int32_t t = blockIdx.x; t < total_items; t += gridDim.x) {
    // ---- decode the item: group e (binary search), column tile ct, chunk p
    int lo = 0, hi = num_groups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.item_prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int32_t gstart = e ? sm.end[e - 1] : 0;
    const int32_t gend = sm.end[e];
    const int32_t nchunks = (sm.item_prefix[e + 1] - sm.item_prefix[e]) / n_ct;
    const int32_t local = t - sm.item_prefix[e];
    const int ct = local / nchunks;
    const int p = local % nchunks;
    const int c0 = ct * kCW;
    const int32_t r0 = gstart + p * kChunkRows;
    const int32_t r1 = min(gend, r0 + kChunkRows);
    const int nrows = max(0, r1 - r0);

    // ---- 1. chunk -> shared memory (TMA; rows past r1 are loaded but ignored)
    if (nrows > 0) {
      const int nbox = (nrows + kBoxRows - 1) / kBoxRows;
      if (tid == 0) {
        mbar_arrive_expect_tx(&sm.bar, nbox * kBoxRows * kCW * 2);
        for (int b = 0; b < nbox; ++b)
          tma_load_2d(&sm.tile[b * kBoxRows * kCW / 2], &xmap, &sm.bar, c0, r0 + b * kBoxRows);
      }
      volatile int never = 0;
      const bool landed = mbar_wait(&sm.bar, phase, &never);
      phase ^= 1;
      // a copy that never lands stops this block: every later wait would be
      // out of phase
      if (__syncthreads_or(!landed)) {
        if (tid == 0) status_or(status, FP8QGG_STATUS_TIMEOUT);
        break;
      }
    }

    // ---- 2. column absmax over the chunk's valid rows
    uint32_t am = 0;
    for (int rr = warp; rr < nrows; rr += kColThreads / 32)
      am = abs_max_bf16x2(am, sm.tile[rr * 32 + lane]);
    sm.red[warp][lane] = am;
    __syncthreads();
    if (warp == 0) {
      uint32_t m = 0;
#pragma unroll
      for (int w = 0; w < kColThreads / 32; ++w) m = __vmaxu2(m, sm.red[w][lane]);
      sm.amax_bits[2 * lane] = (m & 0xFFFFu) << 16;
      sm.amax_bits[2 * lane + 1] = m & 0xFFFF0000u;
    }
    __syncthreads();

    // ---- 3. combine partial absmax across the unit's chunks
    if (nchunks > 1) {
      if (nchunks > static_cast<int32_t>(gridDim.x)) {
        if (tid == 0 && p == 0) status_or(status, FP8QGG_STATUS_GROUP_TOO_TALL);
      } else {
        const int64_t unit = static_cast<int64_t>(e) * n_ct + ct;
        if (tid < kCW && c0 + tid < cols)
          atomicMax(&ws_amax[static_cast<int64_t>(e) * cols + c0 + tid], sm.amax_bits[tid]);
        __syncthreads();
        if (tid == 0) {
          __threadfence();
          atomicAdd(&ws_cnt[unit], 1u);
          if (ld_acquire_u32(&ws_cnt[unit]) < static_cast<uint32_t>(nchunks)) {
            const uint64_t t0 = global_timer_ns();
            while (ld_acquire_u32(&ws_cnt[unit]) < static_cast<uint32_t>(nchunks)) {
              if (global_timer_ns() - t0 > kWaitLimitNs) {
                status_or(status, FP8QGG_STATUS_TIMEOUT);
                break;
              }
              __nanosleep(64);
            }
          }
        }
        __syncthreads();
        if (tid < kCW && c0 + tid < cols)
          sm.amax_bits[tid] = ld_relaxed_u32(&ws_amax[static_cast<int64_t>(e) * cols + c0 + tid]);
      }
    }
    if (tid < kCW) {
      const float s = scale_from_amax(__uint_as_float(sm.amax_bits[tid]), smax);
      sm.scale[tid] = s;
      if (p == 0 && c0 + tid < cols) scales[static_cast<int64_t>(e) * cols + c0 + tid] = s;
    }
    __syncthreads();

    // ---- 4. scale, clamp, cast, store
    if constexpr (LAYOUT == FP8QGG_LAYOUT_SAME) {
      for (int idx = tid; idx < nrows * 8; idx += kColThreads) {
        const int rr = idx >> 3;
        const int j = idx & 7;
        if (c0 + 8 * j >= cols) continue;
        const uint4 v = *reinterpret_cast<const uint4 *>(&sm.tile[rr * 32 + 4 * j]);
        const float *s = &sm.scale[8 * j];
        uint2 o;
        if constexpr (FAST) {
          o.x = quant_pair_fast<FMT>(v.x, pack_f32x2(s[0], s[1])) |
                (quant_pair_fast<FMT>(v.y, pack_f32x2(s[2], s[3])) << 16);
          o.y = quant_pair_fast<FMT>(v.z, pack_f32x2(s[4], s[5])) |
                (quant_pair_fast<FMT>(v.w, pack_f32x2(s[6], s[7])) << 16);
        } else {
          o.x = quant_pair2<FMT>(v.x, s[0], s[1], smax, sat_thr, sat) |
                (quant_pair2<FMT>(v.y, s[2], s[3], smax, sat_thr, sat) << 16);
          o.y = quant_pair2<FMT>(v.z, s[4], s[5], smax, sat_thr, sat) |
                (quant_pair2<FMT>(v.w, s[6], s[7], smax, sat_thr, sat) << 16);
        }
        *reinterpret_cast<uint2 *>(q + static_cast<int64_t>(r0 + rr) * ld_q + c0 + 8 * j) = o;
      }
    } else {
      const float s0 = sm.scale[2 * lane];
      const float s1 = sm.scale[2 * lane + 1];
      const uint64_t s01 = pack_f32x2(s0, s1);
      for (int32_t A = r0 & ~15; A < r1; A += kStgRows) {
        // cast: warp w covers tokens [A + 16w, A + 16w + 16) of column pair `lane`
        const int32_t gb = A + 16 * warp;
        if (gb < r1 && gb + 16 > r0) {
          uint32_t lo4[4] = {0u, 0u, 0u, 0u};
          uint32_t hi4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int32_t g = gb + i;
            const uint32_t wv = (g >= r0 && g < r1) ? sm.tile[(g - r0) * 32 + lane] : 0u;
            uint32_t c2;
            if constexpr (FAST)
              c2 = quant_pair_fast<FMT>(wv, s01);
            else
              c2 = quant_pair2<FMT>(wv, s0, s1, smax, sat_thr, sat);
            lo4[i >> 2] |= (c2 & 0xFFu) << (8 * (i & 3));
            hi4[i >> 2] |= (c2 >> 8) << (8 * (i & 3));
          }
          *reinterpret_cast<uint4 *>(&sm.stg[(2 * lane) * kStgPitch + 16 * warp]) =
              make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
          *reinterpret_cast<uint4 *>(&sm.stg[(2 * lane + 1) * kStgPitch + 16 * warp]) =
              make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
        }
        __syncthreads();
        // store: thread -> column tid/4, two 16-token segments
        const int c = tid >> 2;
        if (c0 + c < cols) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int seg = (tid & 3) * 2 + h;
            const int32_t g = A + 16 * seg;
            if (g >= r1 || g + 16 <= r0) continue;
            uint8_t *dst = q + static_cast<int64_t>(c0 + c) * ld_q + g;
            const uint8_t *src = &sm.stg[c * kStgPitch + 16 * seg];
            if (g >= r0 && g + 16 <= r1) {
              *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(src);
            } else {
              for (int b = 0; b < 16; ++b)
                if (g + b >= r0 && g + b < r1) dst[b] = src[b];
            }
          }
        }
        __syncthreads();
      }
    }
    __syncthreads();
  }

  if (!FAST && sat_count) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(0xFFFFFFFFu, sat, off);
    if (lane == 0 && sat) atomicAdd(sat_count, static_cast<unsigned long long>(sat));
  }
}

namespace {

using ColKernel = void (*)(const CUtensorMap, int64_t, int, const int32_t *, int, uint8_t *,
                           int64_t, float *, float, float, unsigned long long *, int32_t *,
                           uint32_t *, uint32_t *);

template <int FMT, bool FAST>
ColKernel col_kernel_fmt(int layout) {
  return layout == FP8QGG_LAYOUT_SAME
             ? quant_colwise_jagged_kernel<FMT, FP8QGG_LAYOUT_SAME, FAST>
             : quant_colwise_jagged_kernel<FMT, FP8QGG_LAYOUT_TRANSPOSED, FAST>;
}

// The fast kernels skip the clamp and the saturation count (see quant_pair_fast).
ColKernel col_kernel(int fmt, int layout, bool fast) {
  if (fmt == FP8QGG_E4M3FN)
    return fast ? col_kernel_fmt<FP8QGG_E4M3FN, true>(layout)
                : col_kernel_fmt<FP8QGG_E4M3FN, false>(layout);
  return fast ? col_kernel_fmt<FP8QGG_E4M3FNUZ, true>(layout)
              : col_kernel_fmt<FP8QGG_E4M3FNUZ, false>(layout);
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

size_t colwise_amax_bytes(int64_t cols, int32_t num_groups) {
  return round_up(static_cast<size_t>(num_groups) * static_cast<size_t>(cols) * 4, 256);
}

size_t colwise_count_bytes(int64_t cols, int32_t num_groups) {
  const int64_t n_ct = (cols + kCW - 1) / kCW;
  return round_up(static_cast<size_t>(num_groups) * static_cast<size_t>(n_ct) * 4, 256);
}

// Validates the arguments of a jagged column-wise call; returns FP8QGG_OK or
// the error code.
int colwise_check(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                  const int32_t *offsets, int32_t num_groups, uint8_t *q, int64_t ld_q,
                  int layout, float *scales, int fmt, float scale_max, uint64_t *sat_count,
                  int32_t *dev_status) {
  if (rows_total < 0 || rows_total > INT32_MAX - kChunkRows) return FP8QGG_ERR_SHAPE;
  if (cols < 1 || cols > INT32_MAX / 2 || ld_x < cols) return FP8QGG_ERR_SHAPE;
  if (num_groups < 1 || num_groups > kMaxGroups) return FP8QGG_ERR_SHAPE;
  if (fmt != FP8QGG_E4M3FN && fmt != FP8QGG_E4M3FNUZ) return FP8QGG_ERR_UNSUPPORTED;
  if (layout != FP8QGG_LAYOUT_SAME && layout != FP8QGG_LAYOUT_TRANSPOSED)
    return FP8QGG_ERR_UNSUPPORTED;
  if (!(scale_max >= 0.0f) || scale_max > 3.0e38f) return FP8QGG_ERR_UNSUPPORTED;
  if (layout == FP8QGG_LAYOUT_SAME && ld_q < cols) return FP8QGG_ERR_SHAPE;
  if (layout == FP8QGG_LAYOUT_TRANSPOSED && ld_q < rows_total) return FP8QGG_ERR_SHAPE;
  if (!offsets || !scales) return FP8QGG_ERR_NULL;
  if (rows_total > 0 && (!x || !q)) return FP8QGG_ERR_NULL;
  if (cols % 8 || ld_x % 8) return FP8QGG_ERR_ALIGN;
  if (layout == FP8QGG_LAYOUT_SAME && ld_q % 8) return FP8QGG_ERR_ALIGN;
  if (layout == FP8QGG_LAYOUT_TRANSPOSED && ld_q % 16) return FP8QGG_ERR_ALIGN;
  if ((x && !aligned(x, 16)) || (q && !aligned(q, 16)) || !aligned(scales, 4) ||
      !aligned(offsets, 4))
    return FP8QGG_ERR_ALIGN;
  if (sat_count && !aligned(sat_count, 8)) return FP8QGG_ERR_ALIGN;
  if (dev_status && !aligned(dev_status, 4)) return FP8QGG_ERR_ALIGN;
  const int64_t n_ct = (cols + kCW - 1) / kCW;
  const int64_t max_items = (rows_total / kChunkRows + num_groups + 1) * n_ct;
  if (max_items > INT32_MAX) return FP8QGG_ERR_SHAPE;
  return FP8QGG_OK;
}

// Enqueues the kernel.  ws_amax / ws_cnt must already be zero on `stream`.
int colwise_launch(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                   const int32_t *offsets, int32_t num_groups, uint8_t *q, int64_t ld_q,
                   int layout, float *scales, int fmt, float scale_max, uint64_t *sat_count,
                   int32_t *dev_status, uint32_t *ws_amax, uint32_t *ws_cnt,
                   cudaStream_t stream) {
  // With no rows no copy is ever issued, so the map may stay empty.
  CUtensorMap xmap;
  memset(&xmap, 0, sizeof xmap);
  if (rows_total > 0) {
    const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows_total)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ld_x) * 2};
    const uint32_t box[2] = {kCW, kBoxRows};
    if (!encode_tensor_map(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x),
                           dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return FP8QGG_ERR_CUDA;
  }

  DeviceInfo dev;
  if (!device_info(&dev)) return FP8QGG_ERR_CUDA;
  const float smax_eff = effective_scale_max(fmt, scale_max);
  ColKernel kern =
      col_kernel(fmt, layout, sat_count == nullptr && smax_eff >= format_max(fmt));
  const int smem = static_cast<int>(sizeof(ColSmem)) + 1024;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FP8QGG_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kColThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return FP8QGG_ERR_CUDA;
  const int64_t n_ct = (cols + kCW - 1) / kCW;
  const int64_t max_items = (rows_total / kChunkRows + num_groups + 1) * n_ct;
  const int grid = static_cast<int>(std::min<int64_t>(max_items, int64_t(per_sm) * dev.sm_count));

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kColThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float smax = effective_scale_max(fmt, scale_max);
  const float sat_thr = saturation_threshold(fmt);
  const cudaError_t err = cudaLaunchKernelEx(
      &cfg, kern, xmap, rows_total, static_cast<int>(cols), offsets, static_cast<int>(num_groups),
      q, ld_q, scales, smax, sat_thr, reinterpret_cast<unsigned long long *>(sat_count),
      dev_status, ws_amax, ws_cnt);
  return err == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}

}  // namespace fp8qgg

using namespace fp8qgg;

extern "C" size_t fp8_quant_colwise_jagged_workspace_size(int64_t rows_total, int64_t cols,
                                                          int32_t num_groups) {
  (void)rows_total;
  if (cols < 1 || num_groups < 1) return 256;
  return colwise_amax_bytes(cols, num_groups) + colwise_count_bytes(cols, num_groups);
}

extern "C" int fp8_quant_colwise_jagged(const void *x, int64_t rows_total, int64_t cols,
                                        int64_t ld_x, const int32_t *offsets, int32_t num_groups,
                                        uint8_t *q, int64_t ld_q, int layout, float *scales,
                                        int fmt, float scale_max, uint64_t *sat_count,
                                        int32_t *dev_status, void *workspace,
                                        size_t workspace_bytes, void *stream) {
  int rc = colwise_check(x, rows_total, cols, ld_x, offsets, num_groups, q, ld_q, layout, scales,
                         fmt, scale_max, sat_count, dev_status);
  if (rc != FP8QGG_OK) return rc;
  if (!workspace) return FP8QGG_ERR_NULL;
  if (!aligned(workspace, 16)) return FP8QGG_ERR_ALIGN;
  const size_t need = fp8_quant_colwise_jagged_workspace_size(rows_total, cols, num_groups);
  if (workspace_bytes < need) return FP8QGG_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, need, s) != cudaSuccess) return FP8QGG_ERR_CUDA;
  uint32_t *ws_amax = static_cast<uint32_t *>(workspace);
  uint32_t *ws_cnt = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) +
                                                  colwise_amax_bytes(cols, num_groups));
  return colwise_launch(x, rows_total, cols, ld_x, offsets, num_groups, q, ld_q, layout, scales,
                        fmt, scale_max, sat_count, dev_status, ws_amax, ws_cnt, s);
}

// ---------------------------------------------------------------------------
// Entry point for callers that must not allocate device memory.
//
// Some callers cannot hand this library a workspace: runtimes that plan their
// whole device-memory budget up front and forbid cudaMalloc afterwards (an
// allocation can synchronise the device and fragments the plan), or plugin
// interfaces that pass tensors but no scratch buffer.  For them the scratch
// lives in a fixed array in this library's device image instead.  Each GPU that
// loads the library holds this array (kNoAllocScratchBytes) until the process
// exits.  All calls share it, so calls on one device that could overlap in time
// on the GPU race with each other; order them on one stream (or with events).

namespace fp8qgg {

constexpr size_t kNoAllocScratchBytes = FP8QGG_NOALLOC_SCRATCH_BYTES;
static_assert(kNoAllocScratchBytes % 256 == 0, "scratch must keep 256-byte granules");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxScratchDevices = 64;
void *g_scratch_addr[kMaxScratchDevices];
std::mutex g_scratch_mutex;
}  // namespace

// Device address of the fixed scratch array on the current device.  In host
// code `g_noalloc_scratch` only names a host-side stand-in, so the address is
// looked up once per device (with that device current) and cached.
static bool noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices) return false;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return false;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return true;
}

}  // namespace fp8qgg

extern "C" int fp8_quant_colwise_jagged_noalloc(const void *x, int64_t rows_total, int64_t cols,
                                                int64_t ld_x, const int32_t *offsets,
                                                int32_t num_groups, uint8_t *q, int64_t ld_q,
                                                int layout, float *scales, int fmt,
                                                float scale_max, uint64_t *sat_count,
                                                int32_t *dev_status, void *stream) {
  int rc = colwise_check(x, rows_total, cols, ld_x, offsets, num_groups, q, ld_q, layout, scales,
                         fmt, scale_max, sat_count, dev_status);
  if (rc != FP8QGG_OK) return rc;
  const size_t need = fp8_quant_colwise_jagged_workspace_size(rows_total, cols, num_groups);
  if (need > kNoAllocScratchBytes) return FP8QGG_ERR_SHAPE;
  void *scratch = nullptr;
  if (!noalloc_scratch(&scratch)) return FP8QGG_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the previous call's partial maxima and counters must not leak into this one
  if (cudaMemsetAsync(scratch, 0, need, s) != cudaSuccess) return FP8QGG_ERR_CUDA;
  uint32_t *ws_amax = static_cast<uint32_t *>(scratch);
  uint32_t *ws_cnt = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(scratch) +
                                                  colwise_amax_bytes(cols, num_groups));
  return colwise_launch(x, rows_total, cols, ld_x, offsets, num_groups, q, ld_q, layout, scales,
                        fmt, scale_max, sat_count, dev_status, ws_amax, ws_cnt, s);
}
