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
//  - rowwise: a warp takes 32 rows x one 128-column group; a lane owns 8
//    consecutive columns of a row (one 16-byte load), four lanes one block;
//    the block absmax is two shuffles away, the block bytes go to a per-warp
//    table in shared memory, and the group's 32 row words leave as one
//    128-byte store;
//  - column-wise along each expert group's tokens, written transposed in the
//    padded layout (group e from token P_e = sum_{j<e} round_up(size_j, 128),
//    zero codes up to P_e + round_up(size_e, 128)): tiles of 128 tokens x 256
//    columns stream in by TMA through a two-stage shared-memory ring; eight
//    consumer warps of 16 tokens reduce and encode a tile; the two warps
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
// A warp takes 32 rows x one 128-column group: sixteen lanes per row (8
// columns each, one 16-byte load), two rows per load instruction, sixteen
// loads in flight per lane.  A block's four lanes meet by two shuffles; the
// block bytes of the 32 rows go to a per-warp table, so that the group's
// scale words end up one per lane and leave as one 128-byte store.
constexpr int kMxRowThreads = 256;
constexpr int kMxRowsPerWarp = 32;

struct MxRowParams {
  const uint4 *x;
  int64_t ld_x16;  // row pitch in 16-byte vectors
  int64_t rows;
  int cols;
  int ngroups;     // 128-column groups (scale words per row)
  int64_t units;   // ceil(rows / 32) * ngroups
  uint8_t *q;
  int64_t ld_q;
  uint32_t *sw;    // scale words [ngroups, ld_sw]
  int64_t ld_sw;
};

__global__ void __launch_bounds__(kMxRowThreads, 2) mx_rowwise_kernel(const MxRowParams p) {
  // per warp: the scale bytes [32 rows][4 blocks] of its unit; row j's word
  // is then one 4-byte read
  __shared__ uint32_t rowsb[kMxRowThreads / 32][kMxRowsPerWarp];
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;          // which of the two rows of a load
  const int c16 = lane & 15;           // 8-column slot within the group
  uint8_t *rb = reinterpret_cast<uint8_t *>(rowsb[threadIdx.x >> 5]);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kMxRowThreads / 32);
  for (int64_t u = (static_cast<int64_t>(blockIdx.x) * kMxRowThreads + threadIdx.x) >> 5;
       u < p.units; u += nwarps) {
    const int64_t rb_i = u / p.ngroups;  // once per 32 x 128 unit
    const int g = static_cast<int>(u - rb_i * p.ngroups);
    const int64_t r0 = rb_i * kMxRowsPerWarp;
    const int col = 128 * g + 8 * c16;
    const bool c_ok = col < p.cols;
    uint4 v[kMxRowsPerWarp / 2];
#pragma unroll
    for (int i = 0; i < kMxRowsPerWarp / 2; ++i) {
      const int64_t r = r0 + 2 * i + half;
      v[i] = (c_ok && r < p.rows) ? __ldcs(p.x + r * p.ld_x16 + col / 8)
                                  : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kMxRowsPerWarp / 2; ++i) {
      uint32_t m = absmax8(v[i]);
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      const int e = mx_exponent(m);
      const uint2 c = mx_encode8(v[i], mx_multiplier(e));
      const int64_t r = r0 + 2 * i + half;
      if (c_ok && r < p.rows) __stcs(reinterpret_cast<uint2 *>(p.q + r * p.ld_q + col), c);
      // the block's byte (columns past the row's end give byte 0)
      if ((c16 & 3) == 0) rb[4 * (2 * i + half) + (c16 >> 2)] = static_cast<uint8_t>(e + 127);
    }
    __syncwarp();
    if (r0 + lane < p.rows)
      p.sw[static_cast<int64_t>(g) * p.ld_sw + r0 + lane] = rowsb[threadIdx.x >> 5][lane];
    __syncwarp();  // the table is rewritten by the warp's next unit
  }
}

// ------------------------------------------------------- column-wise, padded
// One persistent thread block per SM: a producer warp copies the input tiles
// (128 rows x 256 columns of bf16, 64 KB) with TMA into a two-stage ring in
// shared memory, so that the next tile streams in while eight consumer warps
// (16 rows each) reduce, encode and store the current one.
constexpr int kMxColWarps = 8;                       // consumers
constexpr int kMxColThreads = 32 * kMxColWarps + 32;  // + the producer warp
constexpr int kMxColConsumers = 32 * kMxColWarps;
constexpr int kMxColWidth = 256;  // columns per tile
constexpr int kMxMaxGroups = 1024;
constexpr int kMxColStages = 2;
constexpr uint32_t kMxTileBytes = kMxColWidth * kTileTokens;
constexpr uint32_t kMxInBytes = kTileTokens * kMxColWidth * 2;
static_assert(kMxColWarps * kTileRowsPerWarp == kTileTokens, "eight warps of 16 tokens");

struct MxColSmem {
  uint8_t in[kMxColStages][kMxInBytes];    // input tiles, row-major (1024-byte aligned)
  uint8_t tile[2][kMxTileBytes];           // transposed code tiles
  uint32_t red[kMxColWarps][kMxColWidth / 2];  // per-warp column absmax (bf16 pairs)
  uint32_t sbytes[kMxColWidth];            // per column: the tile's scale word
  uint32_t rowsb[kMxColWarps][2 * kTileRowsPerWarp];  // dual form: row scale bytes of a warp
  int32_t start[kMxMaxGroups];
  int32_t end[kMxMaxGroups];
  int32_t pstart[kMxMaxGroups];
  int32_t tpre[kMxMaxGroups + 1];          // tiles of the groups before group e
  uint64_t full[kMxColStages];
  uint64_t empty[kMxColStages];
  int abort;
};

struct MxColParams {
  int64_t rows_total;
  int cols;
  int box_cols;  // columns of an input tile (min(256, cols))
  int np;        // 256-column panels
  const int32_t *offsets;
  int num_groups;
  uint32_t *sw;  // scale words [tokens / 128, ld_sw]
  int64_t ld_sw;
  int32_t *status;
  // dual form: rowwise codes [rows_total, ld_qr] and scale words [cols / 128, ld_swr]
  uint8_t *q_row;
  int64_t ld_qr;
  uint32_t *swr;
  int64_t ld_swr;
};

struct MxColTile {
  int e, q;
  int32_t b;
};

__device__ __forceinline__ MxColTile mx_col_tile(const MxColSmem &sm, int G, int32_t t) {
  // tile t -> group e (last group whose prefix is <= t), panel, block
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sm.tpre[mid] <= t) lo = mid; else hi = mid - 1;
  }
  MxColTile r;
  r.e = lo;
  const int32_t nb = (sm.end[lo] - sm.start[lo] + kTileTokens - 1) / kTileTokens;
  const int32_t local = t - sm.tpre[lo];
  r.q = local / nb;
  r.b = local - r.q * nb;
  return r;
}

// Named barrier over the consumer warps that also ANDs a flag across them.
__device__ __forceinline__ bool consumers_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kMxColConsumers)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kMxColConsumers) : "memory");
}

// One thread block of nine warps per SM: a sub-partition holds three of them,
// which caps a thread at 168 registers.
template <bool DUAL>
__global__ void __launch_bounds__(kMxColThreads, 1)
    mx_colwise_kernel(const __grid_constant__ CUtensorMap xmap,
                      const __grid_constant__ CUtensorMap qmap, const MxColParams p) {
  extern __shared__ uint8_t smem_raw[];
  MxColSmem &sm = *align_smem_1024<MxColSmem>(smem_raw);
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int G = p.num_groups;
  if (tid == 0) {
    prefetch_tensormap(&xmap);
    prefetch_tensormap(&qmap);
    for (int s = 0; s < kMxColStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kMxColWarps);
    }
    sm.abort = 0;
    fence_mbarrier_init();
  }
  // clamped group bounds, padded starts and tile prefix (one warp)
  if (w == kMxColWarps) {
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
  volatile int *abort = &sm.abort;
  const uint32_t in_bytes = static_cast<uint32_t>(kTileTokens * p.box_cols * 2);

  if (w == kMxColWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t armed = 0, last_par[kMxColStages] = {0, 0};
      int i = 0;
      bool ok = true;
      for (int32_t t = blockIdx.x; t < total; t += gridDim.x, ++i) {
        const int st = i % kMxColStages;
        const uint32_t ph = (i / kMxColStages) & 1;
        if (!mbar_wait(&sm.empty[st], ph ^ 1, abort)) {
          ok = false;
          break;
        }
        const MxColTile tl = mx_col_tile(sm, G, t);
        mbar_arrive_expect_tx(&sm.full[st], in_bytes);
        tma_load_2d(sm.in[st], &xmap, &sm.full[st], tl.q * kMxColWidth,
                    sm.start[tl.e] + tl.b * kTileTokens);
        armed |= 1u << st;
        last_par[st] = ph;
      }
      if (!ok) {
        *abort = 1;
        status_or(p.status, FP8QGG_STATUS_TIMEOUT);
      }
      // copies in flight land before the block can exit
      volatile int never = 0;
      for (int s = 0; s < kMxColStages; ++s)
        if (armed & (1u << s)) (void)mbar_wait(&sm.full[s], last_par[s], &never);
    }
  } else {
    // ------------------------------------------------------------ consumers
    uint8_t *sb8 = reinterpret_cast<uint8_t *>(sm.sbytes);
    const int row_bytes = p.box_cols * 2;
    int i = 0;
    for (int32_t t = blockIdx.x; t < total; t += gridDim.x, ++i) {
      const int st = i % kMxColStages;
      const uint32_t ph = (i / kMxColStages) & 1;
      const MxColTile tl = mx_col_tile(sm, G, t);
      const int c0 = tl.q * kMxColWidth;
      const bool c_ok = c0 + 8 * lane < p.cols;
      const int32_t rw0 = sm.start[tl.e] + tl.b * kTileTokens + kTileRowsPerWarp * w;
      const int32_t r1 = sm.end[tl.e];
      const bool got = mbar_wait(&sm.full[st], ph, abort);
      uint4 v[kTileRowsPerWarp];
      const uint8_t *src = sm.in[st] + (kTileRowsPerWarp * w) * row_bytes + 16 * lane;
#pragma unroll
      for (int k = 0; k < kTileRowsPerWarp; ++k)
        v[k] = (got && c_ok && rw0 + k < r1) ? *reinterpret_cast<const uint4 *>(src + k * row_bytes)
                                             : make_uint4(0u, 0u, 0u, 0u);
      if constexpr (!DUAL) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[st]);  // the stage may be refilled
      }
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
      uint8_t *tile = sm.tile[i & 1];
      // the store issued from this code tile two tiles ago has read it
      if (tid == 0) bulk_wait_read<1>();
      if (!consumers_and(got)) {
        if (tid == 0) {
          *abort = 1;
          status_or(p.status, FP8QGG_STATUS_TIMEOUT);
        }
        break;
      }
      // the 32-token block of warps 2k, 2k+1: per-half max of the magnitude
      // bits (non-NaN bf16 magnitudes order like unsigned 16-bit integers)
      const uint4 mine = *reinterpret_cast<const uint4 *>(&sm.red[w][4 * lane]);
      const uint4 other = *reinterpret_cast<const uint4 *>(&sm.red[w ^ 1][4 * lane]);
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
      if constexpr (DUAL) {
        // the rowwise MX quantisation of the same rows, re-read from the
        // stage (the column-wise registers are free now): a 32-column block is
        // four lanes; the row's scale word of a 128-column group (lanes
        // 16h .. 16h + 15) is gathered by four shuffles, and lane 16h + j
        // keeps the word of row rw0 + j for one coalesced store
        // block scale bytes [16 rows][8 blocks] of the warp; a lane's row word
        // is then one 4-byte read
        uint8_t *rb = reinterpret_cast<uint8_t *>(&sm.rowsb[w][0]);
#pragma unroll
        for (int k = 0; k < kTileRowsPerWarp; ++k) {
          const uint4 vk = (c_ok && rw0 + k < r1)
                               ? *reinterpret_cast<const uint4 *>(src + k * row_bytes)
                               : make_uint4(0u, 0u, 0u, 0u);
          uint32_t m = absmax8(vk);
          m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
          m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
          const int ex = mx_exponent(m);
          const uint2 c = mx_encode8(vk, mx_multiplier(ex));
          if (c_ok && rw0 + k < r1)
            __stcs(reinterpret_cast<uint2 *>(p.q_row + static_cast<int64_t>(rw0 + k) * p.ld_qr +
                                             c0 + 8 * lane),
                   c);
          if ((lane & 3) == 0) rb[8 * k + (lane >> 2)] = static_cast<uint8_t>(ex + 127);
        }
        __syncwarp();
        // lane 16h + j: row rw0 + j, blocks 4h .. 4h + 3 (the 128-column group 2q + h)
        const uint32_t myword = sm.rowsb[w][2 * (lane & 15) + (lane >> 4)];
        const int g = 2 * tl.q + (lane >> 4);
        if (rw0 + (lane & 15) < r1 && 128 * g < p.cols)
          p.swr[static_cast<int64_t>(g) * p.ld_swr + rw0 + (lane & 15)] = myword;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[st]);  // the stage may be refilled
      }
      consumers_sync();
      const int32_t tok = sm.pstart[tl.e] + tl.b * kTileTokens;
      if (tid == 0) {
        tma_store_2d(&qmap, tile, tok, c0);
        bulk_commit();
      }
      if (c0 + tid < p.cols)
        p.sw[static_cast<int64_t>(tok / kTileTokens) * p.ld_sw + c0 + tid] = sm.sbytes[tid];
      // sbytes and red are rewritten only after the next tile's first barrier
    }
    if (tid == 0) bulk_wait_all();  // the code tiles stay valid until their stores have read them
  }
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
  prm.cols = static_cast<int>(cols);
  prm.ngroups = static_cast<int>((cols + 127) / 128);
  prm.units = (rows + kMxRowsPerWarp - 1) / kMxRowsPerWarp * prm.ngroups;
  prm.q = q;
  prm.ld_q = ld_q;
  prm.sw = scales;
  prm.ld_sw = ld_sw;
  const int64_t want = (prm.units + kMxRowThreads / 32 - 1) / (kMxRowThreads / 32);
  const int grid = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(want, int64_t(dev.sm_count) * 4)));
  mx_rowwise_kernel<<<grid, kMxRowThreads, 0, static_cast<cudaStream_t>(stream)>>>(prm);
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}

namespace fp8qgg {

// Checks and launch shared by the column-wise MX call and its dual form
// (q_row non-null).
int mx_colwise_launch(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                      const int32_t *offsets, int32_t num_groups, uint8_t *q, int64_t ld_q,
                      uint32_t *scales, int64_t ld_sw, uint8_t *q_row, int64_t ld_qr,
                      uint32_t *scales_row, int64_t ld_swr, int32_t *dev_status, void *stream) {
  const bool dual = q_row != nullptr;
  if (rows_total < 0 || cols < 1 || cols > INT32_MAX / 2 || ld_x < cols) return FP8QGG_ERR_SHAPE;
  if (num_groups < 1 || num_groups > kMxMaxGroups) return FP8QGG_ERR_SHAPE;
  const int64_t tokens = rows_total + int64_t(kTileTokens) * num_groups;
  if (tokens > INT32_MAX / 2 || ld_q < tokens || ld_sw < cols) return FP8QGG_ERR_SHAPE;
  if (dual && (cols % 32 || ld_qr < cols || ld_swr < rows_total)) return FP8QGG_ERR_SHAPE;
  if (!offsets || !scales || (dual && !scales_row)) return FP8QGG_ERR_NULL;
  if (rows_total > 0 && (!x || !q)) return FP8QGG_ERR_NULL;
  if (cols % 8 || ld_x % 8 || ld_q % 16) return FP8QGG_ERR_ALIGN;
  if ((x && !aligned(x, 16)) || (q && !aligned(q, 16)) || !aligned(scales, 4) ||
      !aligned(offsets, 4))
    return FP8QGG_ERR_ALIGN;
  if (dual && (!aligned(q_row, 8) || ld_qr % 8 || !aligned(scales_row, 4))) return FP8QGG_ERR_ALIGN;
  if (dev_status && !aligned(dev_status, 4)) return FP8QGG_ERR_ALIGN;
  if (rows_total == 0) return FP8QGG_OK;  // every group is empty: nothing is written
  const int np = static_cast<int>((cols + kMxColWidth - 1) / kMxColWidth);
  const int64_t tiles = (rows_total / kTileTokens + num_groups) * int64_t(np);
  if (tiles > INT32_MAX / 2) return FP8QGG_ERR_SHAPE;
  const int box_cols = static_cast<int>(std::min<int64_t>(kMxColWidth, cols));
  CUtensorMap xmap, qmap;
  memset(&xmap, 0, sizeof xmap);
  memset(&qmap, 0, sizeof qmap);
  {
    // input [rows_total][ld_x] bf16; boxes of 128 rows x 256 columns, no swizzle
    const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows_total)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ld_x) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(box_cols), static_cast<uint32_t>(kTileTokens)};
    if (!encode_tensor_map(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims,
                           strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return FP8QGG_ERR_CUDA;
  }
  {
    // codes [cols][ld_q tokens]; boxes of 128 tokens x 256 columns (fewer
    // columns when the tensor has fewer), 128-byte swizzle
    const uint64_t dims[2] = {static_cast<uint64_t>(ld_q), static_cast<uint64_t>(cols)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ld_q)};
    const uint32_t box[2] = {static_cast<uint32_t>(kTileTokens), static_cast<uint32_t>(box_cols)};
    if (!encode_tensor_map(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return FP8QGG_ERR_CUDA;
  }
  DeviceInfo dev;
  if (!device_info(&dev)) return FP8QGG_ERR_CUDA;
  auto kern = dual ? mx_colwise_kernel<true> : mx_colwise_kernel<false>;
  const int smem = static_cast<int>(sizeof(MxColSmem)) + 1024;
  if (!set_max_dynamic_smem(reinterpret_cast<const void *>(kern), smem)) return FP8QGG_ERR_CUDA;
  MxColParams prm;
  prm.rows_total = rows_total;
  prm.cols = static_cast<int>(cols);
  prm.box_cols = box_cols;
  prm.np = np;
  prm.offsets = offsets;
  prm.num_groups = num_groups;
  prm.sw = scales;
  prm.ld_sw = ld_sw;
  prm.status = dev_status;
  prm.q_row = q_row;
  prm.ld_qr = ld_qr;
  prm.swr = scales_row;
  prm.ld_swr = ld_swr;
  const int grid =
      static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, int64_t(dev.sm_count))));
  kern<<<grid, kMxColThreads, smem, static_cast<cudaStream_t>(stream)>>>(xmap, qmap, prm);
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}

}  // namespace fp8qgg

extern "C" int fp8_mx_quant_colwise_padded(const void *x, int64_t rows_total, int64_t cols,
                                           int64_t ld_x, const int32_t *offsets,
                                           int32_t num_groups, uint8_t *q, int64_t ld_q,
                                           uint32_t *scales, int64_t ld_sw, int32_t *dev_status,
                                           void *stream) {
  return mx_colwise_launch(x, rows_total, cols, ld_x, offsets, num_groups, q, ld_q, scales, ld_sw,
                           nullptr, 0, nullptr, 0, dev_status, stream);
}

extern "C" int fp8_mx_quant_dual_padded(const void *x, int64_t rows_total, int64_t cols,
                                        int64_t ld_x, const int32_t *offsets, int32_t num_groups,
                                        uint8_t *q_row, int64_t ld_qr, uint32_t *scales_row,
                                        int64_t ld_swr, uint8_t *q_col, int64_t ld_qc,
                                        uint32_t *scales_col, int64_t ld_swc, int32_t *dev_status,
                                        void *stream) {
  if (!q_row) return FP8QGG_ERR_NULL;
  return mx_colwise_launch(x, rows_total, cols, ld_x, offsets, num_groups, q_col, ld_qc,
                           scales_col, ld_swc, q_row, ld_qr, scales_row, ld_swr, dev_status,
                           stream);
}
