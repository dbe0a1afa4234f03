// Jagged column-wise FP8 quantisation: for every expert group (rows given by
// the int32 offsets tensor) and every column, absmax -> scale -> clamp -> RNE
// e4m3 cast, in the same layout or with a fused transpose (tokens at their
// original positions).  The padded transposed layout and the dual-output form
// run on the panel kernel (quant_panels.cu); this file also holds the entry
// points, the argument checks and the no-allocation variant for all layouts.
//
// Sources: "FP8 su GPU AMD: ..." (ai-radar.it) — introduction (one scale per
// column of each expert's weights, an offsets tensor routing tokens), section
// "Il guadagno vero è nel movimento dei dati" (the chain; the backward's
// .t().contiguous().t() copy removed and scale-and-cast fused; the output tile
// of the column-scales kernel transposed on chip so that stores coalesce).
// "AMD Boosts PyTorch FP8 Training on Instinct GPUs", third paragraph.
//
// B200 design.  A unit is one (group, 64-column tile): 128-byte row segments.
// Two blocks per SM; in each, one producer warp streams rows with TMA into a
// ring of six 112-row slots (14 KB) and each of seven consumer warps owns 16
// rows of every slot and works on them alone (absmax, cast, store straight
// from registers), meeting the other warps only once per task to combine the
// column absmax.
//
// Work is a list of tasks taken from an atomic counter:
//  - a unit whose rows fit in four slots (448 rows) is one "whole" task:
//    every lane keeps its part of the rows in registers between the absmax and
//    the cast (one HBM read) and frees each slot at once, so the ring keeps
//    streaming;
//  - a taller unit is cut into chunks of equal height (at most four slots),
//    and every chunk gives two tasks: an "amax" task (column absmax of the
//    chunk, merged into the unit's absmax in global memory with atomic max,
//    then counted in the unit's arrival counter by one warp) and a "cast"
//    task (the producer waits for the unit's count and copies the unit's
//    absmax into the task's first slot; the consumers derive the scales,
//    read the chunk again and cast it).  A cast task is placed in the list
//    after every amax task of its unit and about 1.5 grid-widths of tasks
//    later, so the chunk it reads again is still in L2 and the wait is
//    short.  Chunks of one tall group are spread over many SMs, so a skewed
//    routing (one expert with many tokens) keeps every SM busy.
// Tall units come first, largest group first, then whole units largest first.
// A task only ever waits for tasks that were handed out before it, each held
// by a running block, so the blocks need not be co-resident.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "device_common.cuh"
#include "host_common.h"
#include "quant_panels.h"

namespace fp8qgg {

// Build-time shape of the kernel.  The defaults are the best of the variants
// measured on B200 (the others were slower or spilled registers).
#ifndef FP8QGG_COLWISE_CONSUMER_WARPS
#define FP8QGG_COLWISE_CONSUMER_WARPS 7   // consumer warps per block (+ the producer)
#endif
#ifndef FP8QGG_COLWISE_BLOCKS_PER_SM
#define FP8QGG_COLWISE_BLOCKS_PER_SM 2
#endif
#ifndef FP8QGG_COLWISE_SUB_ROWS
#define FP8QGG_COLWISE_SUB_ROWS 16        // rows of a slot owned by one consumer warp
#endif
#ifndef FP8QGG_COLWISE_SLOTS
#define FP8QGG_COLWISE_SLOTS 6            // ring depth
#endif
#ifndef FP8QGG_COLWISE_CHUNK_BOXES
#define FP8QGG_COLWISE_CHUNK_BOXES 4      // slots of a whole unit / of a chunk
#endif
#ifndef FP8QGG_COLWISE_LAG_HALF_GRIDS
#define FP8QGG_COLWISE_LAG_HALF_GRIDS 3   // cast task lag, in half grid-widths of tasks
#endif

constexpr int kCW = 64;                 // columns per unit: 128 bytes of bf16 per row
constexpr int kWords = kCW / 2;         // 32-bit words (column pairs) per row
constexpr int kSubRows = FP8QGG_COLWISE_SUB_ROWS;
constexpr int kLaneRows = kSubRows / 4; // rows of a lane's block
constexpr int kConsumerWarps = FP8QGG_COLWISE_CONSUMER_WARPS;
constexpr int kBlocksPerSM = FP8QGG_COLWISE_BLOCKS_PER_SM;
constexpr int kBoxRows = kSubRows * kConsumerWarps;  // rows per ring slot (112: 14 KB)
constexpr int kSlots = FP8QGG_COLWISE_SLOTS;
constexpr int kChunkBoxes = FP8QGG_COLWISE_CHUNK_BOXES;
constexpr int kChunkRows = kChunkBoxes * kBoxRows;   // rows of a whole unit / of a chunk
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kColThreads = kConsumers + 32;         // + one producer warp
constexpr int kMaxGroups = 1024;
constexpr uint32_t kSubBytes = kSubRows * kCW * 2;
constexpr uint32_t kBoxBytes = kBoxRows * kCW * 2;
constexpr int kUnitAmaxWords = kCW;     // global absmax of a tall unit: one word per column
constexpr int kRedBufs = kSlots + 1;
static_assert(kChunkBoxes < kSlots, "a task leaves a ring slot free (its first slot may wait for the producer while the others are issued)");
static_assert(kChunkRows % 16 == 0 && kBoxRows % 16 == 0, "boxes and chunks keep 16-row alignment");
static_assert(kLaneRows == 4 || kLaneRows == 8, "a lane's block is 4 or 8 rows");

enum : int8_t { kTaskWhole = 0, kTaskAmax = 1, kTaskCast = 2, kTaskEnd = 3 };
enum : int8_t { kFirstBox = 1, kLastBox = 2, kWriteScales = 4 };

struct SlotMeta {
  int32_t y;       // first row of the slot
  int32_t v0, v1;  // rows [v0, v1) of the slot belong to the task
  int32_t c0;      // first column of the unit
  int32_t e;       // group
  int32_t tu;      // tall unit (amax and cast tasks)
  int32_t target;  // chunk arrivals that complete the tall unit's absmax
  int8_t kind;
  int8_t flags;
  int16_t nbox;    // slots of the task
};
static_assert(sizeof(SlotMeta) == 32, "slot metadata is two 16-byte words");


struct ColSmem {
  uint32_t ring[kSlots][kBoxRows * kWords];  // [row][32 words]; word = 2 bf16 columns
  // per-warp column absmax of a whole or amax task, one buffer per task that
  // can be in flight: a warp runs at most kSlots slots (so kSlots tasks)
  // ahead of another, which may still be reading its buffer
  alignas(16) uint32_t red[kRedBufs][kConsumerWarps][kWords];
  alignas(16) SlotMeta meta[kSlots];
  alignas(16) uint32_t samax[kSlots][kUnitAmaxWords];  // cast tasks: the unit's absmax words
  int32_t end[kMaxGroups];
  int32_t order[kMaxGroups];                 // groups by row span, largest first
  int32_t prefix[kMaxGroups];                // tall groups: first amax task of the group
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  uint64_t red_bar[kRedBufs];
  int32_t n_tall, na, lag, total;
  int abort;
};
static_assert(offsetof(ColSmem, red) % 16 == 0 && offsetof(ColSmem, ring) % 1024 == 0,
              "16-byte shared-memory accesses and TMA destinations stay aligned");

// Clamped group ends (warp 0): end_e = min(R, max(0, max_{j<=e} offsets[j]))
// is the closed form of "start_e = end_{e-1}, end_e = clamp(offsets[e],
// start_e, R)".
__device__ void build_group_ends(ColSmem &sm, const int32_t *offsets, int num_groups,
                                 int64_t rows_total, int32_t *status) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  int32_t carry_end = 0;
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
    if (e < num_groups && (raw < prev || raw > R)) bad = true;
    if (e < num_groups) sm.end[e] = endv;
    carry_end = __shfl_sync(0xFFFFFFFFu, endv, 31);
  }
  bad = __any_sync(0xFFFFFFFFu, bad);
  if (bad && lane == 0 && blockIdx.x == 0) status_or(status, FP8QGG_STATUS_BAD_OFFSETS);
}

__device__ __forceinline__ int32_t group_start(const ColSmem &sm, int e) {
  return e ? sm.end[e - 1] : 0;
}

// Rows a group's units cover: from their first row (the group's first row
// rounded down with bmask, to 16 rows) to the group's end (0 for an empty
// group).
__device__ __forceinline__ int32_t group_span(const ColSmem &sm, int e, int32_t bmask) {
  const int32_t s = group_start(sm, e);
  const int32_t g = sm.end[e];
  return g > s ? g - (s & bmask) : 0;
}

// Units start on the 16-aligned row at or below a group's first row.
constexpr int32_t kBaseMask = ~15;

struct Task {
  int16_t kind;
  int32_t e, ct, k, C, tu;
  int32_t gstart, r0, r1;  // group's first row; the task's rows [r0, r1)
};

// Task t of the list.  Tall units' amax tasks form stream A, their cast tasks
// stream B (same order); the list opens with L = min(lag, |A|) tasks of A,
// then alternates A, B, and ends with the rest of B, so cast task j follows
// amax task j + L.  Whole units follow.
__device__ Task decode_task(const ColSmem &sm, int32_t t, int n_ct, int32_t bmask) {
  Task r;
  const int32_t NA = sm.na;
  if (t < 2 * NA) {
    const int32_t L = min(sm.lag, NA);
    bool is_amax;
    int32_t j;
    if (t < L) {
      is_amax = true;
      j = t;
    } else if (t < L + 2 * (NA - L)) {
      const int32_t o = t - L;
      is_amax = !(o & 1);
      j = is_amax ? L + (o >> 1) : (o >> 1);
    } else {
      is_amax = false;
      j = (NA - L) + (t - L - 2 * (NA - L));
    }
    int lo = 0, hi = sm.n_tall - 1;  // the tall group holding task j
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.prefix[mid] <= j) lo = mid; else hi = mid - 1;
    }
    r.e = sm.order[lo];
    r.gstart = group_start(sm, r.e);
    const int32_t gend = sm.end[r.e];
    const int32_t a = r.gstart & bmask;
    r.C = (gend - a + kChunkRows - 1) / kChunkRows;
    // chunks of equal height (a multiple of 16, at most kChunkRows)
    const int32_t ch = ((gend - a + r.C - 1) / r.C + 15) & ~15;
    const int32_t rr = j - sm.prefix[lo];
    r.ct = rr / r.C;
    r.k = rr - r.ct * r.C;
    r.tu = lo * n_ct + r.ct;
    r.r0 = a + r.k * ch;
    r.r1 = min(gend, r.r0 + ch);
    r.kind = is_amax ? kTaskAmax : kTaskCast;
  } else {
    const int32_t s = t - 2 * NA;
    const int i = sm.n_tall + s / n_ct;
    r.ct = s - (s / n_ct) * n_ct;
    r.e = sm.order[i];
    r.gstart = group_start(sm, r.e);
    const int32_t gend = sm.end[r.e];
    r.r0 = r.gstart & bmask;
    r.r1 = gend > r.gstart ? gend : r.r0;
    r.k = 0;
    r.C = 1;
    r.tu = -1;
    r.kind = kTaskWhole;
  }
  return r;
}

// Every consumer lane owns a kLaneRows x 8 block of its warp's part of a
// slot: rows kLaneRows * rq + k (rq = lane / 8) and columns 8c8 .. 8c8 + 7
// (c8 = lane % 8), one 16-byte shared-memory load per row.
struct Block {
  uint4 d[kLaneRows];  // row k: columns 8c8 .. 8c8 + 7 as four bf16 pairs
};

// Loads the lane's block of rows [r0, r1) (other rows read as zero).
__device__ __forceinline__ void load_block(Block &b, const uint32_t *sub, int32_t ys, int32_t r0,
                                           int32_t r1, int lane) {
  const int rq = lane >> 3, c8 = lane & 7;
  const uint4 *src = reinterpret_cast<const uint4 *>(sub + kLaneRows * rq * kWords + 4 * c8);
  if (r0 == ys && r1 == ys + kSubRows) {  // the warp's rows all belong to the task
#pragma unroll
    for (int k = 0; k < kLaneRows; ++k) b.d[k] = src[k * (kWords / 4)];
  } else {
#pragma unroll
    for (int k = 0; k < kLaneRows; ++k) {
      const int32_t row = ys + kLaneRows * rq + k;
      b.d[k] = (row >= r0 && row < r1) ? src[k * (kWords / 4)] : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

__device__ __forceinline__ void amax_block(uint4 &am, const Block &b) {
#pragma unroll
  for (int k = 0; k < kLaneRows; ++k) {
    am.x = absmax_acc(am.x, b.d[k].x);
    am.y = absmax_acc(am.y, b.d[k].y);
    am.z = absmax_acc(am.z, b.d[k].z);
    am.w = absmax_acc(am.w, b.d[k].w);
  }
}

// Magnitude bit patterns of a running absmax (comparable as unsigned halves).
__device__ __forceinline__ uint4 finish_amax(uint4 am) {
  return make_uint4(absmax_bits(am.x), absmax_bits(am.y), absmax_bits(am.z), absmax_bits(am.w));
}

// The lane's 8 column scales: s[j] for column 8c8 + j.  The paired
// multiplies take them as (s[2p], s[2p + 1]) (SAME: adjacent columns, which
// are adjacent registers) or (s[j], s[j]) (TRANSPOSED: one column, two rows).
template <int LAYOUT>
struct ColScales {
  float s[8];
};

// The four lanes that share columns 8c8 .. 8c8 + 7 (rq = 0..3) divide for two
// of them each (columns 8c8 + 2rq, 8c8 + 2rq + 1) and swap the results, so
// each IEEE division runs once per warp and column.  Called by all 32 lanes.
template <int LAYOUT>
__device__ __forceinline__ void scales_from_bits(ColScales<LAYOUT> &sc, const uint32_t (&a)[8],
                                                 float smax, int lane) {
  const int rq = lane >> 3;
  const uint32_t b0 = rq == 0 ? a[0] : rq == 1 ? a[2] : rq == 2 ? a[4] : a[6];
  const uint32_t b1 = rq == 0 ? a[1] : rq == 1 ? a[3] : rq == 2 ? a[5] : a[7];
  const float s0 = scale_from_amax(bf16_bits_to_float(b0), smax);
  const float s1 = scale_from_amax(bf16_bits_to_float(b1), smax);
#pragma unroll
  for (int pq = 0; pq < 4; ++pq) {
    const int src = (lane & 7) | (pq << 3);
    sc.s[2 * pq] = __shfl_sync(0xFFFFFFFFu, s0, src);
    sc.s[2 * pq + 1] = __shfl_sync(0xFFFFFFFFu, s1, src);
  }
}

template <int LAYOUT>
__device__ __forceinline__ void write_scales(const ColScales<LAYOUT> &sc, float *scales, int e,
                                             int c0, int cols, int lane) {
  const int c = c0 + 8 * lane;
  if (lane < 8 && c < cols) {
    float4 *dst = reinterpret_cast<float4 *>(scales + static_cast<int64_t>(e) * cols + c);
    if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
      dst[0] = make_float4(sc.s[0], sc.s[1], sc.s[2], sc.s[3]);
      dst[1] = make_float4(sc.s[4], sc.s[5], sc.s[6], sc.s[7]);
    } else {
      float *d = scales + static_cast<int64_t>(e) * cols + c;
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = sc.s[i];
    }
  }
}

// Scale, clamp and encode two values (each with its own scale); the first
// goes to the low byte.  FAST: one packed multiply, no clamp, no count (see
// quant_pair_fast).
template <int FMT, bool FAST>
__device__ __forceinline__ uint32_t enc2(float x0, float x1, uint64_t s01, float s0, float s1,
                                         float smax, float sat_thr, uint32_t &sat) {
  if constexpr (FAST) {
    uint64_t xx, yy;
    asm("mov.b64 %0, {%1, %2};" : "=l"(xx) : "f"(x0), "f"(x1));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(yy) : "l"(xx), "l"(s01));
    float y0, y1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(yy));
    return cvt_x2<FMT>(y0, y1);
  } else {
    float y0 = __fmul_rn(x0, s0);
    float y1 = __fmul_rn(x1, s1);
    sat += (fabsf(y0) > sat_thr) + (fabsf(y1) > sat_thr);
    y0 = clamp_keep_nan(y0, smax);
    y1 = clamp_keep_nan(y1, smax);
    return cvt_x2<FMT>(y0, y1);
  }
}

__device__ __forceinline__ uint32_t word_at(const uint4 &v, int p) {
  return p == 0 ? v.x : p == 1 ? v.y : p == 2 ? v.z : v.w;
}

// Casts the lane's block (rows [r0, r1) of the warp part starting at row ys)
// and stores the codes; rows outside [r0, r1) belong to other groups and are
// never written.  SAME: one 8-byte store per row (columns 8c8 .. 8c8 + 7).
// TRANSPOSED: adjacent rows of one column are encoded together, and one store
// per column holds the lane's kLaneRows tokens; the four lanes with the same
// c8 write 4 * kLaneRows consecutive tokens of that column.
template <int FMT, int LAYOUT, bool FAST>
__device__ __forceinline__ void cast_block(const Block &b, int32_t ys, int32_t r0, int32_t r1,
                                           int c0, int cols, uint8_t *__restrict__ q,
                                           int64_t ld_q, const ColScales<LAYOUT> &sc, float smax,
                                           float sat_thr, uint32_t &sat, int lane) {
  const int rq = lane >> 3, c8 = lane & 7;
  const int32_t rb = ys + kLaneRows * rq;  // the block's first row
  if (r0 >= r1 || rb >= r1 || rb + kLaneRows <= r0 || c0 + 8 * c8 >= cols) return;
  if constexpr (LAYOUT == FP8QGG_LAYOUT_SAME) {
#pragma unroll
    for (int k = 0; k < kLaneRows; ++k) {
      const int32_t row = rb + k;
      if (row < r0 || row >= r1) continue;
      uint32_t c[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const uint32_t w = word_at(b.d[k], p);
        c[p] = enc2<FMT, FAST>(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u),
                               pack_f32x2(sc.s[2 * p], sc.s[2 * p + 1]), sc.s[2 * p],
                               sc.s[2 * p + 1], smax, sat_thr, sat);
      }
      *reinterpret_cast<uint2 *>(q + static_cast<int64_t>(row) * ld_q + c0 + 8 * c8) =
          make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
    }
  } else {
    const bool full = rb >= r0 && rb + kLaneRows <= r1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int p = j >> 1;
      uint32_t c[kLaneRows / 2];
#pragma unroll
      for (int m = 0; m < kLaneRows / 2; ++m) {
        const uint32_t w0 = word_at(b.d[2 * m], p);
        const uint32_t w1 = word_at(b.d[2 * m + 1], p);
        const float x0 = __uint_as_float((j & 1) ? (w0 & 0xFFFF0000u) : (w0 << 16));
        const float x1 = __uint_as_float((j & 1) ? (w1 & 0xFFFF0000u) : (w1 << 16));
        c[m] = enc2<FMT, FAST>(x0, x1, pack_f32x2(sc.s[j], sc.s[j]), sc.s[j], sc.s[j], smax,
                               sat_thr, sat);
      }
      uint32_t tok[kLaneRows / 4];  // the lane's tokens of column 8c8 + j
#pragma unroll
      for (int i = 0; i < kLaneRows / 4; ++i) tok[i] = c[2 * i] | (c[2 * i + 1] << 16);
      uint8_t *dst = q + static_cast<int64_t>(c0 + 8 * c8 + j) * ld_q + rb;
      if (full) {
        if constexpr (kLaneRows == 8)
          *reinterpret_cast<uint2 *>(dst) = make_uint2(tok[0], tok[kLaneRows / 4 - 1]);
        else
          *reinterpret_cast<uint32_t *>(dst) = tok[0];
      } else {
#pragma unroll
        for (int k = 0; k < kLaneRows; ++k)
          if (rb + k >= r0 && rb + k < r1)
            dst[k] = static_cast<uint8_t>(tok[k >> 2] >> (8 * (k & 3)));
      }
    }
  }
}

__device__ __forceinline__ void split_bits(uint32_t (&a)[8], const uint4 &m) {
  a[0] = m.x & 0xFFFFu; a[1] = m.x >> 16; a[2] = m.y & 0xFFFFu; a[3] = m.y >> 16;
  a[4] = m.z & 0xFFFFu; a[5] = m.z >> 16; a[6] = m.w & 0xFFFFu; a[7] = m.w >> 16;
}

template <int FMT, int LAYOUT, bool FAST>
__global__ void __launch_bounds__(kColThreads, kBlocksPerSM)
    quant_colwise_jagged_kernel(const __grid_constant__ CUtensorMap xmap_box,
                                const __grid_constant__ CUtensorMap xmap_sub, int64_t rows_total,
                                int cols, const int32_t *__restrict__ offsets, int num_groups,
                                uint8_t *__restrict__ q, int64_t ld_q,
                                float *__restrict__ scales, float smax, float sat_thr,
                                unsigned long long *sat_count, int32_t *status,
                                uint32_t *__restrict__ work_counter, uint32_t *__restrict__ arrive,
                                uint32_t *__restrict__ unit_amax, int32_t units_cap,
                                UnitWait uw) {
  extern __shared__ uint8_t smem_raw[];
  ColSmem &sm = *align_smem_1024<ColSmem>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_ct = (cols + kCW - 1) / kCW;

  if (tid == kConsumers) {
    prefetch_tensormap(&xmap_box);
    prefetch_tensormap(&xmap_sub);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.full[s], 2);  // the copy's bytes + two producer arrivals
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    for (int b = 0; b < kRedBufs; ++b) mbar_init(&sm.red_bar[b], kConsumerWarps);
    sm.abort = 0;
    fence_mbarrier_init();
  }
  build_group_ends(sm, offsets, num_groups, rows_total, status);
  __syncthreads();
  // groups ranked by row span, largest first (ties by index)
  for (int e = tid; e < num_groups; e += kColThreads) {
    const int32_t se = group_span(sm, e, kBaseMask);
    int rank = 0;
    for (int f = 0; f < num_groups; ++f) {
      const int32_t sf = group_span(sm, f, kBaseMask);
      rank += (sf > se) || (sf == se && f < e);
    }
    sm.order[rank] = e;
  }
  __syncthreads();
  // tall groups (span above one chunk) are a prefix of the order; prefix sums
  // of their amax-task counts (n_ct units x chunks each)
  if (warp == 0) {
    int32_t carry = 0;
    int n_tall = 0;
    for (int base = 0; base < num_groups; base += 32) {
      const int i = base + lane;
      int32_t c = 0;
      if (i < num_groups) {
        const int32_t sp = group_span(sm, sm.order[i], kBaseMask);
        if (sp > kChunkRows) c = n_ct * ((sp + kChunkRows - 1) / kChunkRows);
      }
      int32_t incl = c;
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += o;
      }
      if (i < num_groups) sm.prefix[i] = carry + incl - c;
      n_tall += __popc(__ballot_sync(0xFFFFFFFFu, c > 0));
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) {
      sm.n_tall = n_tall;
      sm.na = carry;
      const int32_t c_max =
          n_tall ? (group_span(sm, sm.order[0], kBaseMask) + kChunkRows - 1) / kChunkRows : 0;
      sm.lag = max(FP8QGG_COLWISE_LAG_HALF_GRIDS * static_cast<int32_t>(gridDim.x) / 2, c_max);
      sm.total = 2 * carry + (num_groups - n_tall) * n_ct;
    }
  }
  __syncthreads();
  if (sm.n_tall * n_ct > units_cap) {  // cannot happen for clamped ends; guards the workspace
    if (tid == 0 && blockIdx.x == 0) status_or(status, FP8QGG_STATUS_BAD_OFFSETS);
    return;
  }

  volatile int *abort = &sm.abort;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t slot = 0, phase = 0;
      uint32_t armed = 0;  // slots whose latest phase carries a copy
      uint32_t armed_par[kSlots];
      int pending = -1;  // cast task slot still owed its second arrival
      bool ok = true;
      // A cast task's first slot also carries the unit's absmax: the producer
      // waits (bounded) until every chunk of the unit has been counted, then
      // copies the 64 absmax words into the slot before its second arrival.
      auto fetch_unit_amax = [&](const SlotMeta &m, uint32_t *dst) -> bool {
        const uint32_t *cnt = arrive + m.tu;
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
        const uint32_t target = static_cast<uint32_t>(m.target) + uw.extra_arrivals;
        if (v < target) {
          const uint64_t t0 = global_timer_ns();
          while (true) {
            __nanosleep(256);
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
            if (v >= target) break;
            if (*abort || global_timer_ns() - t0 > uw.limit_ns) return false;
          }
        }
        const uint4 *src =
            reinterpret_cast<const uint4 *>(unit_amax + static_cast<int64_t>(m.tu) * kUnitAmaxWords);
        uint4 words[kUnitAmaxWords / 4];
#pragma unroll
        for (int i = 0; i < kUnitAmaxWords / 4; ++i) words[i] = __ldcg(src + i);
#pragma unroll
        for (int i = 0; i < kUnitAmaxWords / 4; ++i) reinterpret_cast<uint4 *>(dst)[i] = words[i];
        return true;
      };
      auto push = [&](const SlotMeta &m, int j0, int j1, bool load) -> bool {
        if (!mbar_wait(&sm.empty[slot], phase ^ 1, abort)) return false;
        sm.meta[slot] = m;
        if (load) {
          if (j0 == 0 && j1 == kConsumerWarps - 1) {
            mbar_arrive_expect_tx(&sm.full[slot], kBoxBytes);
            tma_load_2d(sm.ring[slot], &xmap_box, &sm.full[slot], m.c0, m.y);
          } else {
            mbar_arrive_expect_tx(&sm.full[slot], (j1 - j0 + 1) * kSubBytes);
            for (int j = j0; j <= j1; ++j)
              tma_load_2d(sm.ring[slot] + j * kSubRows * kWords, &xmap_sub, &sm.full[slot], m.c0,
                          m.y + j * kSubRows);
          }
          armed |= 1u << slot;
          armed_par[slot] = phase;
        } else {
          mbar_arrive(&sm.full[slot]);
          armed &= ~(1u << slot);
        }
        // A cast task's first slot waits for its second arrival until the
        // unit's absmax is in the slot; the task's other slots are issued
        // first, so the fetch overlaps their copies.  (They never need the
        // first slot back: a task has fewer slots than the ring.)
        if (m.kind == kTaskCast && (m.flags & kFirstBox))
          pending = static_cast<int>(slot);
        else
          mbar_arrive(&sm.full[slot]);
        if (++slot == kSlots) { slot = 0; phase ^= 1; }
        return true;
      };
      // the deferred second arrival comes even after a failed fetch, so that
      // the phase still ends when the copy lands
      auto finish_pending = [&](const SlotMeta &m) -> bool {
        if (pending < 0) return true;
        const bool fetched = fetch_unit_amax(m, sm.samax[pending]);
        mbar_arrive(&sm.full[pending]);
        pending = -1;
        return fetched;
      };
      const int32_t total = sm.total;
      // task indices are taken two ahead, hiding the counter's round trip
      int32_t t = static_cast<int32_t>(atomicAdd(work_counter, 1u));
      int32_t next = static_cast<int32_t>(atomicAdd(work_counter, 1u));
      while (ok && t < total) {
        const int32_t next2 = static_cast<int32_t>(atomicAdd(work_counter, 1u));
        const Task tk = decode_task(sm, t, n_ct, kBaseMask);
        SlotMeta m;
        m.c0 = tk.ct * kCW;
        m.e = tk.e;
        m.tu = tk.tu;
        m.target = tk.C;
        m.kind = tk.kind;
        if (tk.r1 <= tk.r0) {  // empty group: scales only
          m.y = tk.r0;
          m.v0 = m.v1 = tk.r0;
          m.flags = kFirstBox | kLastBox;
          m.nbox = 1;
          ok = push(m, 0, 0, false);
        } else {
          const int nb = (tk.r1 - tk.r0 + kBoxRows - 1) / kBoxRows;
          m.nbox = static_cast<int16_t>(nb);
          for (int b = 0; ok && b < nb; ++b) {
            m.y = tk.r0 + b * kBoxRows;
            m.v0 = max(tk.gstart, m.y);
            m.v1 = min(tk.r1, m.y + kBoxRows);
            m.flags = (b == 0 ? kFirstBox : 0) | (b == nb - 1 ? kLastBox : 0) |
                      (tk.kind == kTaskCast && tk.k == 0 ? kWriteScales : 0);
            ok = push(m, (m.v0 - m.y) / kSubRows, (m.v1 - 1 - m.y) / kSubRows, true);
          }
          if (ok) ok = finish_pending(m);
        }
        t = next;
        next = next2;
      }
      if (ok) {
        SlotMeta m{};
        m.kind = kTaskEnd;
        ok = push(m, 0, 0, false);
      }
      if (!ok) {
        *abort = 1;
        status_or(status, FP8QGG_STATUS_TIMEOUT);
        if (pending >= 0) mbar_arrive(&sm.full[pending]);
        // copies already issued land before the block may exit
        volatile int never = 0;
        for (int s2 = 0; s2 < kSlots; ++s2)
          if (armed & (1u << s2)) (void)mbar_wait(&sm.full[s2], armed_par[s2], &never);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int w = warp;
    const int c8 = lane & 7;
    uint32_t slot = 0, phase = 0;
    uint32_t sat = 0;
    int rbuf = 0;
    uint32_t rpar = 0;  // bit b: parity of the next phase of red_bar[b]
    static_assert(kRedBufs <= 32, "parity bits fit one word");
    ColScales<LAYOUT> sc;
    uint4 chunk_am = make_uint4(0u, 0u, 0u, 0u);  // amax tasks: absmax over the chunk so far
    uint32_t pub_turn = 0;  // the warp that publishes the next amax task
    bool failed = false;
    auto advance = [&]() {
      if (++slot == kSlots) { slot = 0; phase ^= 1; }
    };
    auto release = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
    };
    while (!failed) {
      // every wait is decided for the whole warp, so that its lanes never part
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.full[slot], phase, abort))) { failed = true; break; }
      SlotMeta m = sm.meta[slot];
      if (m.kind == kTaskEnd) break;
      if (m.kind == kTaskWhole) {
        // up to kChunkBoxes slots; the lane keeps its blocks in registers and
        // frees each slot at once, so the ring keeps streaming
        Block blk[kChunkBoxes];
        int32_t ysb[kChunkBoxes], r0b[kChunkBoxes], r1b[kChunkBoxes];
        uint4 am = make_uint4(0u, 0u, 0u, 0u);
        const int nb = m.nbox;
#pragma unroll
        for (int b = 0; b < kChunkBoxes; ++b) {
          ysb[b] = 0;
          r0b[b] = r1b[b] = 0;
          if (b < nb && !failed) {
            if (b > 0) {
              advance();
              if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.full[slot], phase, abort))) {
                failed = true;
                continue;
              }
              m = sm.meta[slot];
            }
            ysb[b] = m.y + w * kSubRows;
            r0b[b] = max(m.v0, ysb[b]);
            r1b[b] = min(m.v1, ysb[b] + kSubRows);
            load_block(blk[b], sm.ring[slot] + w * kSubRows * kWords, ysb[b], r0b[b], r1b[b],
                       lane);
            release();
            amax_block(am, blk[b]);
          }
        }
        if (failed) break;
        // the warp's column absmax (rows meet by shuffles), then the warps'
        // meet in shared memory
        am = finish_amax(am);
#pragma unroll
        for (int d = 8; d < 32; d <<= 1) {
          am.x = __vmaxu2(am.x, __shfl_xor_sync(0xFFFFFFFFu, am.x, d));
          am.y = __vmaxu2(am.y, __shfl_xor_sync(0xFFFFFFFFu, am.y, d));
          am.z = __vmaxu2(am.z, __shfl_xor_sync(0xFFFFFFFFu, am.z, d));
          am.w = __vmaxu2(am.w, __shfl_xor_sync(0xFFFFFFFFu, am.w, d));
        }
        if (lane < 8) *reinterpret_cast<uint4 *>(&sm.red[rbuf][w][4 * c8]) = am;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.red_bar[rbuf]);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.red_bar[rbuf], (rpar >> rbuf) & 1u, abort))) {
          failed = true;
          break;
        }
        rpar ^= 1u << rbuf;
        uint4 mm = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int wp = 0; wp < kConsumerWarps; ++wp) {
          const uint4 v = *reinterpret_cast<const uint4 *>(&sm.red[rbuf][wp][4 * c8]);
          mm.x = __vmaxu2(mm.x, v.x);
          mm.y = __vmaxu2(mm.y, v.y);
          mm.z = __vmaxu2(mm.z, v.z);
          mm.w = __vmaxu2(mm.w, v.w);
        }
        if (++rbuf == kRedBufs) rbuf = 0;
        uint32_t a[8];
        split_bits(a, mm);
        scales_from_bits<LAYOUT>(sc, a, smax, lane);
        if (w == 0) write_scales<LAYOUT>(sc, scales, m.e, m.c0, cols, lane);
        uint8_t *const qe = q;
#pragma unroll
        for (int b = 0; b < kChunkBoxes; ++b)
          if (b < nb)
            cast_block<FMT, LAYOUT, FAST>(blk[b], ysb[b], r0b[b], r1b[b], m.c0, cols, qe, ld_q, sc,
                                          smax, sat_thr, sat, lane);
      } else {
        const int32_t ys = m.y + w * kSubRows;
        const int32_t r0 = max(m.v0, ys);
        const int32_t r1 = min(m.v1, ys + kSubRows);
        if (m.kind == kTaskCast && (m.flags & kFirstBox)) {
          // the unit's absmax words came with the slot (read before it is freed)
          const uint4 x0 = *reinterpret_cast<const uint4 *>(&sm.samax[slot][8 * c8]);
          const uint4 x1 = *reinterpret_cast<const uint4 *>(&sm.samax[slot][8 * c8 + 4]);
          const uint32_t a[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          scales_from_bits<LAYOUT>(sc, a, smax, lane);
        }
        Block blk;
        load_block(blk, sm.ring[slot] + w * kSubRows * kWords, ys, r0, r1, lane);
        release();
        if (m.kind == kTaskCast) {
          if ((m.flags & kFirstBox) && (m.flags & kWriteScales) && w == 0)
            write_scales<LAYOUT>(sc, scales, m.e, m.c0, cols, lane);
          cast_block<FMT, LAYOUT, FAST>(blk, ys, r0, r1, m.c0, cols,
                                        q, ld_q, sc, smax,
                                        sat_thr, sat, lane);
        } else {
          uint4 &am = chunk_am;
          amax_block(am, blk);
          if (m.flags & kLastBox) {
            am = finish_amax(am);
#pragma unroll
            for (int d = 8; d < 32; d <<= 1) {
              am.x = __vmaxu2(am.x, __shfl_xor_sync(0xFFFFFFFFu, am.x, d));
              am.y = __vmaxu2(am.y, __shfl_xor_sync(0xFFFFFFFFu, am.y, d));
              am.z = __vmaxu2(am.z, __shfl_xor_sync(0xFFFFFFFFu, am.z, d));
              am.w = __vmaxu2(am.w, __shfl_xor_sync(0xFFFFFFFFu, am.w, d));
            }
            // the warps' partials meet in shared memory; one warp (turn by
            // turn) merges the chunk's absmax into the unit's words in global
            // memory and counts the chunk, the others go on at once
            if (lane < 8) *reinterpret_cast<uint4 *>(&sm.red[rbuf][w][4 * c8]) = am;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.red_bar[rbuf]);
            if (w == static_cast<int>(pub_turn)) {
              if (!__all_sync(0xFFFFFFFFu,
                              mbar_wait(&sm.red_bar[rbuf], (rpar >> rbuf) & 1u, abort))) {
                failed = true;
                break;
              }
              uint32_t mm = 0;
#pragma unroll
              for (int wp = 0; wp < kConsumerWarps; ++wp) mm = __vmaxu2(mm, sm.red[rbuf][wp][lane]);
              uint32_t *ua = unit_amax + static_cast<int64_t>(m.tu) * kUnitAmaxWords + 2 * lane;
              atomicMax(ua, mm & 0xFFFFu);
              atomicMax(ua + 1, mm >> 16);
              __threadfence();  // every lane's merges are visible before the count
              __syncwarp();
              if (lane == 0) atomicAdd(arrive + m.tu, 1u);
            }
            rpar ^= 1u << rbuf;
            if (++rbuf == kRedBufs) rbuf = 0;
            if (++pub_turn == kConsumerWarps) pub_turn = 0;
            am = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      advance();
    }
    if (failed) {
      *abort = 1;
      if (lane == 0) status_or(status, FP8QGG_STATUS_TIMEOUT);
    }
    if (!FAST && sat_count) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(0xFFFFFFFFu, sat, off);
      if (lane == 0 && sat) atomicAdd(sat_count, static_cast<unsigned long long>(sat));
    }
  }
}

namespace {

using ColKernel = void (*)(const CUtensorMap, const CUtensorMap, int64_t, int, const int32_t *,
                           int, uint8_t *, int64_t, float *, float, float, unsigned long long *,
                           int32_t *, uint32_t *, uint32_t *, uint32_t *, int32_t, UnitWait);

std::mutex g_unit_wait_mutex;
UnitWait g_unit_wait{0u, kWaitLimitNs};

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

// Scratch layout: [0, 256) the work counter; then one arrival counter per
// tall unit (rounded up to 256 bytes); then 64 absmax words per tall unit.
// A tall group has at least kChunkRows - 14 rows, so at most
// rows_total / (kChunkRows - 16) groups are tall.
struct ColScratch {
  int64_t units_cap;
  size_t arrive_off, amax_off, bytes;
};

ColScratch colwise_scratch(int64_t rows_total, int64_t cols, int32_t num_groups) {
  ColScratch s;
  const int64_t n_ct = (std::max<int64_t>(cols, 1) + kCW - 1) / kCW;
  const int64_t tall = std::min<int64_t>(std::max<int32_t>(num_groups, 0),
                                         std::max<int64_t>(rows_total, 0) / (kChunkRows - 16));
  s.units_cap = tall * n_ct;
  s.arrive_off = 256;
  s.amax_off = s.arrive_off + (static_cast<size_t>(s.units_cap) * 4 + 255) / 256 * 256;
  s.bytes = s.amax_off + static_cast<size_t>(s.units_cap) * kUnitAmaxWords * 4;
  return s;
}

}  // namespace

UnitWait current_unit_wait() {
  std::lock_guard<std::mutex> lock(g_unit_wait_mutex);
  return g_unit_wait;
}

// Validates the arguments of a jagged column-wise call; returns FP8QGG_OK or
// the error code.
int colwise_check(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                  const int32_t *offsets, int32_t num_groups, uint8_t *q, int64_t ld_q,
                  int layout, float *scales, int fmt, float scale_max, uint64_t *sat_count,
                  int32_t *dev_status) {
  if (rows_total < 0 || rows_total > INT32_MAX - 4 * kChunkRows) return FP8QGG_ERR_SHAPE;
  if (cols < 1 || cols > INT32_MAX / 2 || ld_x < cols) return FP8QGG_ERR_SHAPE;
  if (num_groups < 1 || num_groups > kMaxGroups) return FP8QGG_ERR_SHAPE;
  if (fmt != FP8QGG_E4M3FN && fmt != FP8QGG_E4M3FNUZ) return FP8QGG_ERR_UNSUPPORTED;
  if (layout != FP8QGG_LAYOUT_SAME && layout != FP8QGG_LAYOUT_TRANSPOSED &&
      layout != FP8QGG_LAYOUT_TRANSPOSED_PADDED)
    return FP8QGG_ERR_UNSUPPORTED;
  if (!(scale_max >= 0.0f) || scale_max > 3.0e38f) return FP8QGG_ERR_UNSUPPORTED;
  if (layout == FP8QGG_LAYOUT_SAME && ld_q < cols) return FP8QGG_ERR_SHAPE;
  if (layout == FP8QGG_LAYOUT_TRANSPOSED && ld_q < rows_total) return FP8QGG_ERR_SHAPE;
  if (layout == FP8QGG_LAYOUT_TRANSPOSED_PADDED &&
      (ld_q < rows_total + 128 * int64_t(num_groups) ||
       rows_total + 128 * int64_t(num_groups) > INT32_MAX - 4 * kChunkRows))
    return FP8QGG_ERR_SHAPE;
  if (!offsets || !scales) return FP8QGG_ERR_NULL;
  if (rows_total > 0 && (!x || !q)) return FP8QGG_ERR_NULL;
  if (cols % 8 || ld_x % 8) return FP8QGG_ERR_ALIGN;
  if (layout == FP8QGG_LAYOUT_SAME && ld_q % 8) return FP8QGG_ERR_ALIGN;
  if (layout != FP8QGG_LAYOUT_SAME && ld_q % 16) return FP8QGG_ERR_ALIGN;
  if ((x && !aligned(x, 16)) || (q && !aligned(q, 16)) || !aligned(scales, 4) ||
      !aligned(offsets, 4))
    return FP8QGG_ERR_ALIGN;
  if (sat_count && !aligned(sat_count, 8)) return FP8QGG_ERR_ALIGN;
  if (dev_status && !aligned(dev_status, 4)) return FP8QGG_ERR_ALIGN;
  // the task list must stay within int32: amax + cast tasks of the tall
  // units (each group's span is its rows plus at most 15) and whole units
  const int64_t n_ct = (cols + kCW - 1) / kCW;
  const int64_t chunks = (rows_total + 16 * int64_t(num_groups)) / kChunkRows + num_groups;
  if (n_ct * (2 * chunks + num_groups) > INT32_MAX / 2) return FP8QGG_ERR_SHAPE;
  return FP8QGG_OK;
}

// Enqueues the kernel.  The first colwise_scratch(...).bytes of `scratch`
// must already be zero on `stream`.
int colwise_launch(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                   const int32_t *offsets, int32_t num_groups, uint8_t *q, int64_t ld_q,
                   int layout, float *scales, int fmt, float scale_max, uint64_t *sat_count,
                   int32_t *dev_status, void *scratch, cudaStream_t stream) {
  // the padded transposed layout runs on the panel kernel (quant_panels.cu)
  if (layout == FP8QGG_LAYOUT_TRANSPOSED_PADDED)
    return panel_launch(x, rows_total, cols, ld_x, offsets, num_groups, q, ld_q, scales,
                        nullptr, 0, nullptr, fmt, scale_max, sat_count, dev_status, scratch,
                        current_unit_wait(), stream);
  // With no rows no copy is ever issued, so the maps may stay empty.
  CUtensorMap xmap_box, xmap_sub;
  memset(&xmap_box, 0, sizeof xmap_box);
  memset(&xmap_sub, 0, sizeof xmap_sub);
  if (rows_total > 0) {
    const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows_total)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ld_x) * 2};
    const uint32_t box[2] = {kCW, kBoxRows};
    const uint32_t subbox[2] = {kCW, kSubRows};
    if (!encode_tensor_map(&xmap_box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x),
                           dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tensor_map(&xmap_sub, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x),
                           dims, strides, subbox, CU_TENSOR_MAP_SWIZZLE_NONE))
      return FP8QGG_ERR_CUDA;
  }

  DeviceInfo dev;
  if (!device_info(&dev)) return FP8QGG_ERR_CUDA;
  const float smax = effective_scale_max(fmt, scale_max);
  ColKernel kern = col_kernel(fmt, layout, sat_count == nullptr && smax >= format_max(fmt));
  const int smem = static_cast<int>(sizeof(ColSmem)) + 1024;
  if (!set_max_dynamic_smem(reinterpret_cast<const void *>(kern), smem))
    return FP8QGG_ERR_CUDA;
  // at most this many tasks: the grid never exceeds the work
  const int64_t n_ct = (cols + kCW - 1) / kCW;
  const int64_t tasks_max =
      n_ct * (2 * ((rows_total + 16 * int64_t(num_groups)) / kChunkRows + num_groups) + num_groups);
  const int grid = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(tasks_max, int64_t(dev.sm_count) * kBlocksPerSM)));
  const float sat_thr = saturation_threshold(fmt);
  const ColScratch sl = colwise_scratch(rows_total, cols, num_groups);
  uint8_t *base = static_cast<uint8_t *>(scratch);
  kern<<<grid, kColThreads, smem, stream>>>(
      xmap_box, xmap_sub, rows_total, static_cast<int>(cols), offsets,
      static_cast<int>(num_groups), q, ld_q, scales, smax, sat_thr,
      reinterpret_cast<unsigned long long *>(sat_count), dev_status,
      reinterpret_cast<uint32_t *>(base), reinterpret_cast<uint32_t *>(base + sl.arrive_off),
      reinterpret_cast<uint32_t *>(base + sl.amax_off), static_cast<int32_t>(sl.units_cap),
      current_unit_wait());
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}

}  // namespace fp8qgg

using namespace fp8qgg;

extern "C" int fp8qgg_test_unit_wait(uint32_t extra_arrivals, uint64_t limit_ns) {
  if (limit_ns > kWaitLimitNs) return FP8QGG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_unit_wait_mutex);
  g_unit_wait.extra_arrivals = extra_arrivals;
  g_unit_wait.limit_ns = limit_ns ? limit_ns : kWaitLimitNs;
  return FP8QGG_OK;
}

extern "C" size_t fp8_quant_colwise_jagged_workspace_size(int64_t rows_total, int64_t cols,
                                                          int32_t num_groups) {
  // one workspace size serves every layout: the larger of the two kernels' needs
  return std::max(colwise_scratch(rows_total, cols, num_groups).bytes,
                  panel_scratch(rows_total, cols, num_groups, false).bytes);
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
  return colwise_launch(x, rows_total, cols, ld_x, offsets, num_groups, q, ld_q, layout, scales,
                        fmt, scale_max, sat_count, dev_status, workspace, s);
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
struct ScratchAddr {
  CUcontext ctx;  // the context the address belongs to
  void *addr;
};
ScratchAddr g_scratch_addr[kMaxScratchDevices];
std::mutex g_scratch_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);

// The calling thread's current context (nullptr when none is current or the
// driver entry point is missing).
CUcontext current_context() {
  static CtxGetCurrentFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  CUcontext c = nullptr;
  if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}
}  // namespace

// Device address of the fixed scratch array on the current device.  In host
// code `g_noalloc_scratch` only names a host-side stand-in, so the address is
// looked up with the device current and kept per device together with the
// context it belongs to; a call under another context (after
// cudaDeviceReset, for instance, the library's device code is loaded again)
// looks it up again.
static bool noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices) return false;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchAddr &c = g_scratch_addr[dev];
  const CUcontext ctx = current_context();
  if (!c.addr || !ctx || c.ctx != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return false;
    c.addr = p;
    c.ctx = current_context();  // the lookup makes the primary context current if none was
  }
  *out = c.addr;
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
  // the previous call's counters and absmax words must not leak into this one
  if (cudaMemsetAsync(scratch, 0, need, s) != cudaSuccess) return FP8QGG_ERR_CUDA;
  return colwise_launch(x, rows_total, cols, ld_x, offsets, num_groups, q, ld_q, layout, scales,
                        fmt, scale_max, sat_count, dev_status, scratch, s);
}
