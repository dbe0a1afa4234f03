// MXFP8 quantisation: one E8M0 scale per block of 32 consecutive elements
// along the contraction axis, e4m3fn elements.
//
// The pages name MXFP8 quantisation and grouped GEMM kernels as the next
// step ("AMD Primus adds FP8/MXFP8 kernels ...", section "What Primus adds for
// MoE training on MI355X"; "AMD Boosts PyTorch FP8 Training on Instinct
// GPUs", last paragraph; "FP8 su GPU AMD ...", section "Cosa significa per chi
// gestisce cluster locali") without defining the format; it is taken from the
// OCP Microscaling (MX) v1.0 definition: a block's scale is 2^E with
// E = floor(log2(amax)) - 8 (8: the exponent of e4m3fn's largest binade),
// clamped to [-127, 127] and stored as the byte E + 127; an element's code is
// the round-to-nearest-even e4m3fn encoding of x / 2^E, saturating at 448.
// Readings for the cases the definition leaves open: the absmax skips NaN,
// an all-zero block takes E = -127, an infinite absmax E = 127.
//
// The scale of a block depends on its 32 elements only, so each kernel reads
// its input once and needs no cross-block reduction:
// Scales are stored packed for the grouped GEMM: one 32-bit word per (row,
// group of four blocks = 128 elements of the contraction axis), byte j the
// scale of block 4g + j, and the words of one group g contiguous over the
// rows (word g * ld_sw + r).  The GEMM then reads, per 128-deep stage, one
// contiguous run of words for the rows of its tile.
//  - rowwise: a lane owns 8 consecutive columns (one 16-byte load), four
//    lanes one block; the block absmax is two shuffles away, and four
//    shuffles gather a group's four scale bytes into one word;
//  - column-wise along each expert group's tokens, written transposed in the
//    padded layout (group e from token P_e = sum_{j<e} round_up(size_j, 128),
//    zero codes up to P_e + round_up(size_e, 128)): a thread block takes a
//    tile of 128 tokens x 256 columns, eight warps of 16 tokens; the two warps
//    of a 32-token block meet in shared memory for its column absmax; the
//    codes go through a 128-byte-swizzled shared-memory tile to one bulk
//    tensor store (whole 128-byte lines, padding zeros included); a tile is
//    one 128-token group, so its 256 scale words are contiguous (one 1 KB
//    store).
#include <algorithm>
#include <cstring>

#include "device_common.cuh"
#include "host_common.h"
#include "quant_tile.cuh"

namespace fp8qgg {

// E of a block from its absmax as bf16 magnitude bits (never NaN: the absmax
// skips NaN).  A normal bf16 with exponent field f lies in [2^(f-127),
// 2^(f-126)), so floor(log2) = f - 127 and E = f - 135; zero and subnormal
// magnitudes (f = 0) are below 2^-126 and clamp to -127; f = 255 is infinity.
__device__ __forceinline__ int mx_exponent(uint32_t amax_bits) {
  const int f = static_cast<int>((amax_bits >> 7) & 0xFFu);
  if (f == 255) return 127;
  return max(f - 135, -127);
}

// 2^-E as an fp32 multiplier (exact: E = 127 gives the subnormal 2^-127).
// x * 2^-E is then exact wherever it can reach a nonzero code.
__device__ __forceinline__ float mx_multiplier(int e) {
  return e >= 127 ? __uint_as_float(0x00400000u)
                  : __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

// Eight bf16 values (one 16-byte vector) with one multiplier -> 8 codes.
__device__ __forceinline__ uint2 mx_encode8(const uint4 &v, float f) {
  uint32_t sat = 0;
  const uint32_t c0 = enc_pair<FP8QGG_E4M3FN, true>(lo_f(v.x), hi_f(v.x), f, f, 0.f, 0.f, sat);
  const uint32_t c1 = enc_pair<FP8QGG_E4M3FN, true>(lo_f(v.y), hi_f(v.y), f, f, 0.f, 0.f, sat);
  const uint32_t c2 = enc_pair<FP8QGG_E4M3FN, true>(lo_f(v.z), hi_f(v.z), f, f, 0.f, 0.f, sat);
  const uint32_t c3 = enc_pair<FP8QGG_E4M3FN, true>(lo_f(v.w), hi_f(v.w), f, f, 0.f, 0.f, sat);
  return make_uint2(c0 | (c1 << 16), c2 | (c3 << 16));
}

// Absmax magnitude bits of the 8 bf16 values of a vector.
__device__ __forceinline__ uint32_t absmax8(const uint4 &v) {
  const uint32_t a2 = absmax_bits(
      absmax_acc(absmax_acc(absmax_acc(absmax_acc(0u, v.x), v.y), v.z), v.w));
  return max(a2 & 0xFFFFu, a2 >> 16);
}

// ------------------------------------------------------------------ rowwise
constexpr int kMxRowThreads = 256;

__device__ __forceinline__ int64_t id_of(int64_t base, int u, int64_t nwarps) {
  return base + u * nwarps;
}
constexpr int kMxRowUnroll = 4;  // 256-column segments in flight per warp

struct MxRowParams {
  const uint4 *x;
  int64_t ld_x16;  // row pitch in 16-byte vectors
  int64_t rows;
  int64_t segs;    // 256-column segments per row
  int cols;
  int ngroups;     // 128-column groups (scale words per row)
  uint8_t *q;
  int64_t ld_q;
  uint32_t *sw;    // scale words [ngroups, ld_sw]
  int64_t ld_sw;
};

__global__ void __launch_bounds__(kMxRowThreads) mx_rowwise_kernel(const MxRowParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t units = p.rows * p.segs;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kMxRowThreads / 32);
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kMxRowThreads + threadIdx.x) >> 5;
  for (int64_t base = warp0; base < units; base += nwarps * kMxRowUnroll) {
    uint4 v[kMxRowUnroll];
    int64_t row[kMxRowUnroll];
    int col[kMxRowUnroll];
    bool ok[kMxRowUnroll];
#pragma unroll
    for (int u = 0; u < kMxRowUnroll; ++u) {
      const int64_t id = id_of(base, u, nwarps);
      row[u] = id / p.segs;
      col[u] = static_cast<int>(id - row[u] * p.segs) * 256 + 8 * lane;
      ok[u] = id < units && col[u] < p.cols;
      v[u] = ok[u] ? __ldcs(p.x + row[u] * p.ld_x16 + col[u] / 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kMxRowUnroll; ++u) {
      uint32_t m = absmax8(v[u]);
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      const int e = mx_exponent(m);
      const uint2 c = mx_encode8(v[u], mx_multiplier(e));
      // the word of 128-column group (lane >> 4): the bytes of lanes l0, l0 + 4,
      // l0 + 8, l0 + 12 (columns past the row's end give byte 0)
      const uint32_t byte = static_cast<uint32_t>(e + 127);
      const int l0 = lane & 16;
      const uint32_t word = __shfl_sync(0xFFFFFFFFu, byte, l0) |
                            (__shfl_sync(0xFFFFFFFFu, byte, l0 + 4) << 8) |
                            (__shfl_sync(0xFFFFFFFFu, byte, l0 + 8) << 16) |
                            (__shfl_sync(0xFFFFFFFFu, byte, l0 + 12) << 24);
      if (ok[u]) __stcs(reinterpret_cast<uint2 *>(p.q + row[u] * p.ld_q + col[u]), c);
      const int64_t g = (id_of(base, u, nwarps) - row[u] * p.segs) * 2 + (lane >> 4);
      if ((lane & 15) == 0 && id_of(base, u, nwarps) < units && g < p.ngroups)
        p.sw[g * p.ld_sw + row[u]] = word;
    }
  }
}

// ------------------------------------------------------- column-wise, padded
constexpr int kMxColWarps = 8;
constexpr int kMxColThreads = 32 * kMxColWarps;
constexpr int kMxColWidth = 256;  // columns per tile
constexpr int kMxMaxGroups = 1024;
constexpr uint32_t kMxTileBytes = kMxColWidth * kTileTokens;
static_assert(kMxColWarps * kTileRowsPerWarp == kTileTokens, "eight warps of 16 tokens");

struct MxColSmem {
  uint8_t tile[2][kMxTileBytes];           // transposed code tiles (1024-byte aligned)
  uint32_t red[kMxColWarps][kMxColWidth / 2];  // per-warp column absmax (bf16 pairs)
  uint32_t sbytes[kMxColWidth];            // per column: the tile's scale word
  int32_t start[kMxMaxGroups];
  int32_t end[kMxMaxGroups];
  int32_t pstart[kMxMaxGroups];
  int32_t tpre[kMxMaxGroups + 1];          // tiles of the groups before group e
};

struct MxColParams {
  const uint4 *x;
  int64_t ld_x16;
  int64_t rows_total;
  int cols;
  int np;  // 256-column panels
  const int32_t *offsets;
  int num_groups;
  uint32_t *sw;    // scale words [tokens / 128, ld_sw]
  int64_t ld_sw;
  int32_t *status;
};

__global__ void __launch_bounds__(kMxColThreads, 2)
    mx_colwise_kernel(const __grid_constant__ CUtensorMap qmap, const MxColParams p) {
  extern __shared__ uint8_t smem_raw[];
  MxColSmem &sm = *align_smem_1024<MxColSmem>(smem_raw);
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int G = p.num_groups;
  if (tid == 0) prefetch_tensormap(&qmap);
  // clamped group bounds, padded starts and tile prefix (one warp)
  if (tid < 32) {
    const int32_t R = static_cast<int32_t>(p.rows_total);
    int32_t carry_end = 0, carry_pad = 0, carry_t = 0;
    bool bad = false;
    for (int base = 0; base < G; base += 32) {
      const int e = base + lane;
      const int32_t raw = e < G ? __ldg(p.offsets + e) : INT32_MIN;
      int32_t run = max(raw, 0);
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t o = __shfl_up_sync(0xFFFFFFFFu, run, d);
        if (lane >= d) run = max(run, o);
      }
      const int32_t endv = min(R, max(carry_end, run));
      int32_t prev = __shfl_up_sync(0xFFFFFFFFu, endv, 1);
      if (lane == 0) prev = carry_end;
      if (e < G && (raw < prev || raw > R)) bad = true;
      const int32_t nb = e < G ? (endv - prev + kTileTokens - 1) / kTileTokens : 0;
      int32_t ps = nb * kTileTokens, nt = nb * p.np;
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t o1 = __shfl_up_sync(0xFFFFFFFFu, ps, d);
        const int32_t o2 = __shfl_up_sync(0xFFFFFFFFu, nt, d);
        if (lane >= d) {
          ps += o1;
          nt += o2;
        }
      }
      if (e < G) {
        sm.start[e] = prev;
        sm.end[e] = endv;
        sm.pstart[e] = carry_pad + ps - nb * kTileTokens;
        sm.tpre[e] = carry_t + nt - nb * p.np;
      }
      carry_end = __shfl_sync(0xFFFFFFFFu, endv, 31);
      carry_pad += __shfl_sync(0xFFFFFFFFu, ps, 31);
      carry_t += __shfl_sync(0xFFFFFFFFu, nt, 31);
    }
    if (lane == 0) sm.tpre[G] = carry_t;
    bad = __any_sync(0xFFFFFFFFu, bad);
    if (bad && lane == 0 && blockIdx.x == 0) status_or(p.status, FP8QGG_STATUS_BAD_OFFSETS);
  }
  __syncthreads();
  const int32_t total = sm.tpre[G];
  uint8_t *sb8 = reinterpret_cast<uint8_t *>(sm.sbytes);
  int it = 0;
  for (int32_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
    // tile t -> group e (last group whose prefix is <= t), panel, block
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.tpre[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int32_t nb = (sm.end[e] - sm.start[e] + kTileTokens - 1) / kTileTokens;
    const int32_t local = t - sm.tpre[e];
    const int q = local / nb;
    const int32_t b = local - q * nb;
    const int c0 = q * kMxColWidth;
    const int col = c0 + 8 * lane;
    const bool c_ok = col < p.cols;
    const int32_t r0 = sm.start[e] + b * kTileTokens + kTileRowsPerWarp * w;
    const int32_t r1 = sm.end[e];
    uint4 v[kTileRowsPerWarp];
    const uint4 *src = p.x + static_cast<int64_t>(r0) * p.ld_x16 + col / 8;
#pragma unroll
    for (int k = 0; k < kTileRowsPerWarp; ++k)
      v[k] = (c_ok && r0 + k < r1) ? __ldcs(src + k * p.ld_x16) : make_uint4(0u, 0u, 0u, 0u);
    // the warp's 16-row column absmax, as bf16 magnitude pairs
    uint32_t acc[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < kTileRowsPerWarp; ++k) {
      acc[0] = absmax_acc(acc[0], v[k].x);
      acc[1] = absmax_acc(acc[1], v[k].y);
      acc[2] = absmax_acc(acc[2], v[k].z);
      acc[3] = absmax_acc(acc[3], v[k].w);
    }
    *reinterpret_cast<uint4 *>(&sm.red[w][4 * lane]) =
        make_uint4(absmax_bits(acc[0]), absmax_bits(acc[1]), absmax_bits(acc[2]),
                   absmax_bits(acc[3]));
    uint8_t *tile = sm.tile[it & 1];
    // the store issued from this tile buffer two tiles ago has read it
    if (tid == 0) bulk_wait_read<1>();
    __syncthreads();
    // the 32-token block of warps 2k, 2k+1: its column absmax and scale
    const uint4 mine = *reinterpret_cast<const uint4 *>(&sm.red[w][4 * lane]);
    const uint4 other = *reinterpret_cast<const uint4 *>(&sm.red[w ^ 1][4 * lane]);
    // per-half max of magnitude bits (non-NaN bf16 magnitudes order like
    // unsigned 16-bit integers)
    const uint32_t m2[4] = {__vmaxu2(mine.x, other.x), __vmaxu2(mine.y, other.y),
                            __vmaxu2(mine.z, other.z), __vmaxu2(mine.w, other.w)};
    float s[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t pair = m2[j >> 1];
      const uint32_t m = (j & 1) ? (pair >> 16) : (pair & 0xFFFFu);
      const int ex = mx_exponent(m);
      s[j] = mx_multiplier(ex);
      if (!(w & 1)) sb8[4 * (8 * lane + j) + (w >> 1)] = static_cast<uint8_t>(ex + 127);
    }
    uint32_t sat = 0;
    tile_col_codes<FP8QGG_E4M3FN, true>(v, s, tile, w, lane, 0.f, 0.f, sat);
    fence_proxy_async_smem();
    __syncthreads();
    const int32_t tok = sm.pstart[e] + b * kTileTokens;
    if (tid == 0) {
      tma_store_2d(&qmap, tile, tok, c0);
      bulk_commit();
    }
    if (c0 + tid < p.cols) p.sw[static_cast<int64_t>(tok / kTileTokens) * p.ld_sw + c0 + tid] = sm.sbytes[tid];
  }
  if (tid == 0) bulk_wait_all();  // the tiles stay valid until their stores have read them
}

}  // namespace fp8qgg

using namespace fp8qgg;

extern "C" int fp8_mx_quant_rowwise(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                                    uint8_t *q, int64_t ld_q, uint32_t *scales, int64_t ld_sw,
                                    void *stream) {
  if (rows < 0 || cols < 1 || cols % 32 || cols > INT32_MAX / 2) return FP8QGG_ERR_SHAPE;
  if (ld_x < cols || ld_q < cols || ld_sw < rows) return FP8QGG_ERR_SHAPE;
  if (rows == 0) return FP8QGG_OK;
  if (!x || !q || !scales) return FP8QGG_ERR_NULL;
  if (!aligned(x, 16) || ld_x % 8 || !aligned(q, 8) || ld_q % 8) return FP8QGG_ERR_ALIGN;
  if (!aligned(scales, 4)) return FP8QGG_ERR_ALIGN;
  DeviceInfo dev;
  if (!device_info(&dev)) return FP8QGG_ERR_CUDA;
  MxRowParams prm;
  prm.x = static_cast<const uint4 *>(x);
  prm.ld_x16 = ld_x / 8;
  prm.rows = rows;
  prm.segs = (cols + 255) / 256;
  prm.cols = static_cast<int>(cols);
  prm.ngroups = static_cast<int>((cols + 127) / 128);
  prm.q = q;
  prm.ld_q = ld_q;
  prm.sw = scales;
  prm.ld_sw = ld_sw;
  const int64_t warps = (rows * prm.segs + kMxRowUnroll - 1) / kMxRowUnroll;
  const int64_t want = (warps + kMxRowThreads / 32 - 1) / (kMxRowThreads / 32);
  const int grid = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(want, int64_t(dev.sm_count) * 8)));
  mx_rowwise_kernel<<<grid, kMxRowThreads, 0, static_cast<cudaStream_t>(stream)>>>(prm);
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}

extern "C" int fp8_mx_quant_colwise_padded(const void *x, int64_t rows_total, int64_t cols,
                                           int64_t ld_x, const int32_t *offsets,
                                           int32_t num_groups, uint8_t *q, int64_t ld_q,
                                           uint32_t *scales, int64_t ld_sw, int32_t *dev_status,
                                           void *stream) {
  if (rows_total < 0 || cols < 1 || cols > INT32_MAX / 2 || ld_x < cols) return FP8QGG_ERR_SHAPE;
  if (num_groups < 1 || num_groups > kMxMaxGroups) return FP8QGG_ERR_SHAPE;
  const int64_t tokens = rows_total + int64_t(kTileTokens) * num_groups;
  if (tokens > INT32_MAX / 2 || ld_q < tokens || ld_sw < cols) return FP8QGG_ERR_SHAPE;
  if (!offsets || !scales) return FP8QGG_ERR_NULL;
  if (rows_total > 0 && (!x || !q)) return FP8QGG_ERR_NULL;
  if (cols % 8 || ld_x % 8 || ld_q % 16) return FP8QGG_ERR_ALIGN;
  if ((x && !aligned(x, 16)) || (q && !aligned(q, 16)) || !aligned(scales, 4) ||
      !aligned(offsets, 4))
    return FP8QGG_ERR_ALIGN;
  if (dev_status && !aligned(dev_status, 4)) return FP8QGG_ERR_ALIGN;
  if (rows_total == 0) return FP8QGG_OK;  // every group is empty: nothing is written
  const int np = static_cast<int>((cols + kMxColWidth - 1) / kMxColWidth);
  const int64_t tiles = (rows_total / kTileTokens + num_groups) * int64_t(np);
  if (tiles > INT32_MAX / 2) return FP8QGG_ERR_SHAPE;
  CUtensorMap qmap;
  memset(&qmap, 0, sizeof qmap);
  {
    // codes [cols][ld_q tokens]; boxes of 128 tokens x 256 columns (fewer
    // columns when the tensor has fewer), 128-byte swizzle
    const uint64_t dims[2] = {static_cast<uint64_t>(ld_q), static_cast<uint64_t>(cols)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ld_q)};
    const uint32_t box[2] = {static_cast<uint32_t>(kTileTokens),
                             static_cast<uint32_t>(std::min<int64_t>(kMxColWidth, cols))};
    if (!encode_tensor_map(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return FP8QGG_ERR_CUDA;
  }
  DeviceInfo dev;
  if (!device_info(&dev)) return FP8QGG_ERR_CUDA;
  const int smem = static_cast<int>(sizeof(MxColSmem)) + 1024;
  if (!set_max_dynamic_smem(reinterpret_cast<const void *>(mx_colwise_kernel), smem))
    return FP8QGG_ERR_CUDA;
  MxColParams prm;
  prm.x = static_cast<const uint4 *>(x);
  prm.ld_x16 = ld_x / 8;
  prm.rows_total = rows_total;
  prm.cols = static_cast<int>(cols);
  prm.np = np;
  prm.offsets = offsets;
  prm.num_groups = num_groups;
  prm.sw = scales;
  prm.ld_sw = ld_sw;
  prm.status = dev_status;
  const int grid = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(tiles, int64_t(dev.sm_count) * 2)));
  mx_colwise_kernel<<<grid, kMxColThreads, smem, static_cast<cudaStream_t>(stream)>>>(qmap, prm);
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}
