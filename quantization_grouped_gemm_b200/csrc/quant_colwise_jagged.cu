// Jagged column-wise FP8 quantisation: for every expert group (rows given by
// the int32 offsets tensor) and every column, absmax -> scale -> clamp -> RNE
// e4m3 cast, with an optional fused transpose.
//
// Sources: "FP8 su GPU AMD: ..." (ai-radar.it) — introduction (one scale per
// column of each expert's weights, an offsets tensor routing tokens), section
// "Il guadagno vero è nel movimento dei dati" (the chain; the backward's
// .t().contiguous().t() copy removed and scale-and-cast fused; the output tile
// of the column-scales kernel transposed on chip so that stores coalesce).
// "AMD Boosts PyTorch FP8 Training on Instinct GPUs", third paragraph.
//
// B200 design.  A unit of work is one (group, 32-column tile): all of the
// group's rows for 32 columns.  One block per SM takes units from an atomic
// counter, largest groups first.  Inside a block one producer warp streams the
// unit's rows with TMA, 256-row boxes, into a 12-slot shared-memory ring; eight
// consumer warps take the column absmax box by box, derive the 32 scales and
// cast.  A unit of at most 12 boxes (3072 rows) stays in the ring between the
// absmax and the cast: one HBM read.  A taller unit is streamed a second time
// for the cast; the units in flight at once belong to the same few groups, so
// the second read is served by L2.  No block ever waits for another block.
// TRANSPOSED output goes through a shared-memory [column][token] tile and is
// written as 16-byte runs along the tokens.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "device_common.cuh"
#include "host_common.h"

namespace fp8qgg {

constexpr int kCW = 32;                   // columns per unit: 64 bytes of bf16 per row
constexpr int kWords = kCW / 2;           // 32-bit words (column pairs) per row
constexpr int kBoxRows = 256;             // rows per TMA box (16 KB)
constexpr int kSlots = 12;                // ring depth = boxes a unit may keep on chip
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kColThreads = kConsumers + 32;  // + one producer warp
constexpr int kMaxGroups = 1024;
constexpr int kStgPitch = kBoxRows + 16;  // [column][token] staging row, bytes
constexpr uint32_t kBoxBytes = kBoxRows * kCW * 2;

enum : int16_t { kLastBox = 1, kResident = 2 };

struct SlotMeta {
  int32_t unit;  // position in the size-sorted unit list; -1 ends the stream
  int32_t y;     // first row of the box (16-aligned)
  int16_t pass;  // 1: absmax, 2: cast of a unit that did not stay on chip
  int16_t flags;
};

struct ColSmem {
  uint32_t ring[kSlots][kBoxRows * kWords];  // [row][16 words]; word = 2 bf16 columns
  uint8_t stg[kCW * kStgPitch];
  SlotMeta meta[kSlots];
  uint32_t red[kConsumers / kWords][kWords];
  float scale[kCW];
  int32_t end[kMaxGroups];
  int32_t order[kMaxGroups];
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  int abort;
};

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

struct Unit {
  int e, ct;
  int32_t gstart, gend;
};

__device__ __forceinline__ Unit decode_unit(const ColSmem &sm, int32_t u, int n_ct) {
  Unit r;
  r.e = sm.order[u / n_ct];
  r.ct = u - (u / n_ct) * n_ct;
  r.gstart = r.e ? sm.end[r.e - 1] : 0;
  r.gend = sm.end[r.e];
  return r;
}

__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory");
}

// Barrier over the consumer warps that ANDs a flag across them, so that a
// wait that gives up is given up by all consumers together.
__device__ __forceinline__ bool consumer_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kConsumers)
      : "memory");
  return r != 0;
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

template <int FMT, bool FAST>
__device__ __forceinline__ uint32_t quant_word(uint32_t w, uint64_t s2, float s0, float s1,
                                               float smax, float sat_thr, uint32_t &sat) {
  if constexpr (FAST)
    return quant_pair_fast<FMT>(w, s2);
  else
    return quant_pair2<FMT>(w, s0, s1, smax, sat_thr, sat);
}

// Cast one box (rows [y, y + 256) of which [v0, v1) belong to the unit) with
// the unit's scales and store it.  Called by the 256 consumer threads.
template <int FMT, int LAYOUT, bool FAST>
__device__ __forceinline__ void cast_box(ColSmem &sm, const uint32_t *box, int32_t y,
                                         int32_t v0, int32_t v1, int c0, int cols,
                                         uint8_t *__restrict__ q, int64_t ld_q, float smax,
                                         float sat_thr, uint32_t &sat) {
  const int tid = threadIdx.x;
  if constexpr (LAYOUT == FP8QGG_LAYOUT_SAME) {
#pragma unroll
    for (int k = 0; k < (kBoxRows * kCW / 8) / kConsumers; ++k) {
      const int idx = tid + k * kConsumers;
      const int rr = idx >> 2;   // row in box
      const int j = idx & 3;     // 8-column vector
      const int32_t row = y + rr;
      if (row < v0 || row >= v1 || c0 + 8 * j >= cols) continue;
      const uint4 v = *reinterpret_cast<const uint4 *>(&box[rr * kWords + 4 * j]);
      const float *sc = &sm.scale[8 * j];
      uint2 o;
      o.x = quant_word<FMT, FAST>(v.x, pack_f32x2(sc[0], sc[1]), sc[0], sc[1], smax, sat_thr, sat) |
            (quant_word<FMT, FAST>(v.y, pack_f32x2(sc[2], sc[3]), sc[2], sc[3], smax, sat_thr,
                                   sat) << 16);
      o.y = quant_word<FMT, FAST>(v.z, pack_f32x2(sc[4], sc[5]), sc[4], sc[5], smax, sat_thr, sat) |
            (quant_word<FMT, FAST>(v.w, pack_f32x2(sc[6], sc[7]), sc[6], sc[7], smax, sat_thr,
                                   sat) << 16);
      *reinterpret_cast<uint2 *>(q + static_cast<int64_t>(row) * ld_q + c0 + 8 * j) = o;
    }
  } else {
    // cast: thread -> column pair cp, 16-row group g
    const int cp = tid & (kWords - 1);
    const int g = tid / kWords;
    const float s0 = sm.scale[2 * cp];
    const float s1 = sm.scale[2 * cp + 1];
    const uint64_t s01 = pack_f32x2(s0, s1);
    uint32_t lo4[4] = {0u, 0u, 0u, 0u};
    uint32_t hi4[4] = {0u, 0u, 0u, 0u};
    const int32_t gb = y + 16 * g;
    if (gb < v1 && gb + 16 > v0) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int32_t row = gb + i;
        const uint32_t w = (row >= v0 && row < v1) ? box[(16 * g + i) * kWords + cp] : 0u;
        const uint32_t c2 = quant_word<FMT, FAST>(w, s01, s0, s1, smax, sat_thr, sat);
        lo4[i >> 2] |= (c2 & 0xFFu) << (8 * (i & 3));
        hi4[i >> 2] |= (c2 >> 8) << (8 * (i & 3));
      }
    }
    *reinterpret_cast<uint4 *>(&sm.stg[(2 * cp) * kStgPitch + 16 * g]) =
        make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
    *reinterpret_cast<uint4 *>(&sm.stg[(2 * cp + 1) * kStgPitch + 16 * g]) =
        make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
    consumer_bar();
    // store: 16 consecutive threads write the 256 tokens of one output row
#pragma unroll
    for (int k = 0; k < (kCW * kBoxRows / 16) / kConsumers; ++k) {
      const int idx = tid + k * kConsumers;
      const int c = idx / (kBoxRows / 16);
      const int sgi = idx % (kBoxRows / 16);
      const int32_t g0 = y + 16 * sgi;
      if (c0 + c >= cols || g0 >= v1 || g0 + 16 <= v0) continue;
      uint8_t *dst = q + static_cast<int64_t>(c0 + c) * ld_q + g0;
      const uint8_t *src = &sm.stg[c * kStgPitch + 16 * sgi];
      if (g0 >= v0 && g0 + 16 <= v1) {
        *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(src);
      } else {
        for (int b = 0; b < 16; ++b)
          if (g0 + b >= v0 && g0 + b < v1) dst[b] = src[b];
      }
    }
    consumer_bar();
  }
}

template <int FMT, int LAYOUT, bool FAST>
__global__ void __launch_bounds__(kColThreads, 1)
    quant_colwise_jagged_kernel(const __grid_constant__ CUtensorMap xmap, int64_t rows_total,
                                int cols, const int32_t *__restrict__ offsets, int num_groups,
                                uint8_t *__restrict__ q, int64_t ld_q,
                                float *__restrict__ scales, float smax, float sat_thr,
                                unsigned long long *sat_count, int32_t *status,
                                uint32_t *__restrict__ work_counter) {
  extern __shared__ uint8_t smem_raw[];
  ColSmem &sm = *reinterpret_cast<ColSmem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_ct = (cols + kCW - 1) / kCW;

  if (tid == kConsumers) {
    prefetch_tensormap(&xmap);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    sm.abort = 0;
    fence_mbarrier_init();
  }
  build_group_ends(sm, offsets, num_groups, rows_total, status);
  __syncthreads();
  // groups ranked by row count, largest first (ties by index)
  for (int e = tid; e < num_groups; e += kColThreads) {
    const int32_t se = sm.end[e] - (e ? sm.end[e - 1] : 0);
    int rank = 0;
    for (int f = 0; f < num_groups; ++f) {
      const int32_t sf = sm.end[f] - (f ? sm.end[f - 1] : 0);
      rank += (sf > se) || (sf == se && f < e);
    }
    sm.order[rank] = e;
  }
  __syncthreads();

  const int32_t total_units = num_groups * n_ct;
  volatile int *abort = &sm.abort;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t slot = 0, phase = 0;
      uint32_t armed = 0;  // slots whose latest phase carries a copy
      uint32_t armed_par[kSlots];
      bool ok = true;
      auto push = [&](int32_t unit, int32_t y, int16_t pass, int16_t flags, bool load,
                      int c0) -> bool {
        if (!mbar_wait(&sm.empty[slot], phase ^ 1, abort)) return false;
        sm.meta[slot] = SlotMeta{unit, y, pass, flags};
        if (load) {
          mbar_arrive_expect_tx(&sm.full[slot], kBoxBytes);
          tma_load_2d(sm.ring[slot], &xmap, &sm.full[slot], c0, y);
          armed |= 1u << slot;
          armed_par[slot] = phase;
        } else {
          mbar_arrive(&sm.full[slot]);
          armed &= ~(1u << slot);
        }
        if (++slot == kSlots) { slot = 0; phase ^= 1; }
        return true;
      };
      int32_t u = static_cast<int32_t>(atomicAdd(work_counter, 1u));
      while (ok && u < total_units) {
        const int32_t next = static_cast<int32_t>(atomicAdd(work_counter, 1u));
        const Unit un = decode_unit(sm, u, n_ct);
        const int c0 = un.ct * kCW;
        if (un.gend <= un.gstart) {
          ok = push(u, un.gstart & ~15, 1, kLastBox | kResident, false, c0);
        } else {
          const int32_t A = un.gstart & ~15;
          const int nbox = (un.gend - A + kBoxRows - 1) / kBoxRows;
          const int16_t res = nbox <= kSlots ? kResident : 0;
          for (int b = 0; ok && b < nbox; ++b)
            ok = push(u, A + b * kBoxRows, 1, (b == nbox - 1 ? kLastBox : 0) | res, true, c0);
          if (!res)
            for (int b = 0; ok && b < nbox; ++b)
              ok = push(u, A + b * kBoxRows, 2, b == nbox - 1 ? kLastBox : 0, true, c0);
        }
        u = next;
      }
      if (ok) ok = push(-1, 0, 0, 0, false, 0);
      if (!ok) {
        *abort = 1;
        status_or(status, FP8QGG_STATUS_TIMEOUT);
        // copies already issued land before the block may exit
        volatile int never = 0;
        for (int s2 = 0; s2 < kSlots; ++s2)
          if (armed & (1u << s2)) (void)mbar_wait(&sm.full[s2], armed_par[s2], &never);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    uint32_t slot = 0, phase = 0;
    uint32_t sat = 0;
    const int cp = tid & (kWords - 1);     // absmax: column pair
    const int rp = tid / kWords;           // absmax: row phase (0..15)
    constexpr int kPhases = kConsumers / kWords;
    uint32_t am = 0;
    uint32_t res_slot = 0, res_phase = 0;  // first ring slot of an on-chip unit
    int res_count = 0;
    while (true) {
      const bool got = mbar_wait(&sm.full[slot], phase, abort);
      if (!consumer_bar_and(got)) {
        *abort = 1;
        if (tid == 0) status_or(status, FP8QGG_STATUS_TIMEOUT);
        break;
      }
      const SlotMeta m = sm.meta[slot];
      if (m.unit < 0) break;
      const Unit un = decode_unit(sm, m.unit, n_ct);
      const int c0 = un.ct * kCW;
      const int32_t v0 = max(un.gstart, m.y);
      const int32_t v1 = min(un.gend, m.y + kBoxRows);
      const uint32_t *box = sm.ring[slot];
      if (m.pass == 1) {
        for (int32_t rr = max(v0 - m.y, 0) + ((rp - max(v0 - m.y, 0)) % kPhases + kPhases) % kPhases;
             rr < v1 - m.y; rr += kPhases)
          am = abs_max_bf16x2(am, box[rr * kWords + cp]);
        if (m.flags & kResident) {
          if (res_count == 0) { res_slot = slot; res_phase = phase; }
          ++res_count;
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.empty[slot]);
        }
        if (m.flags & kLastBox) {
          // column absmax over the row phases -> the unit's 32 scales
          sm.red[rp][cp] = am;
          consumer_bar();
          if (tid < kWords) {
            uint32_t mm = 0;
#pragma unroll
            for (int ph = 0; ph < kPhases; ++ph) mm = __vmaxu2(mm, sm.red[ph][tid]);
            const float sa = scale_from_amax(__uint_as_float((mm & 0xFFFFu) << 16), smax);
            const float sb = scale_from_amax(__uint_as_float(mm & 0xFFFF0000u), smax);
            sm.scale[2 * tid] = sa;
            sm.scale[2 * tid + 1] = sb;
            const int64_t base = static_cast<int64_t>(un.e) * cols + c0 + 2 * tid;
            if (c0 + 2 * tid < cols) scales[base] = sa;
            if (c0 + 2 * tid + 1 < cols) scales[base + 1] = sb;
          }
          consumer_bar();
          am = 0;
          // a unit that stayed on chip is cast now, box by box, from the ring
          uint32_t s2 = res_slot;
          for (int i = 0; i < res_count; ++i) {
            const SlotMeta mi = sm.meta[s2];
            cast_box<FMT, LAYOUT, FAST>(sm, sm.ring[s2], mi.y, max(un.gstart, mi.y),
                                        min(un.gend, mi.y + kBoxRows), c0, cols, q, ld_q, smax,
                                        sat_thr, sat);
            consumer_bar();
            if (lane == 0) mbar_arrive(&sm.empty[s2]);
            if (++s2 == kSlots) s2 = 0;
          }
          res_count = 0;
          (void)res_phase;
        }
      } else {
        cast_box<FMT, LAYOUT, FAST>(sm, box, m.y, v0, v1, c0, cols, q, ld_q, smax, sat_thr, sat);
        consumer_bar();
        if (lane == 0) mbar_arrive(&sm.empty[slot]);
      }
      if (++slot == kSlots) { slot = 0; phase ^= 1; }
    }
    if (!FAST && sat_count) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(0xFFFFFFFFu, sat, off);
      if (lane == 0 && sat) atomicAdd(sat_count, static_cast<unsigned long long>(sat));
    }
  }
}

namespace {

using ColKernel = void (*)(const CUtensorMap, int64_t, int, const int32_t *, int, uint8_t *,
                           int64_t, float *, float, float, unsigned long long *, int32_t *,
                           uint32_t *);

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

}  // namespace

// Bytes of scratch the kernel needs: one work counter, rounded to 256.
constexpr size_t kColwiseScratchBytes = 256;

// Validates the arguments of a jagged column-wise call; returns FP8QGG_OK or
// the error code.
int colwise_check(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                  const int32_t *offsets, int32_t num_groups, uint8_t *q, int64_t ld_q,
                  int layout, float *scales, int fmt, float scale_max, uint64_t *sat_count,
                  int32_t *dev_status) {
  if (rows_total < 0 || rows_total > INT32_MAX - 2 * kBoxRows) return FP8QGG_ERR_SHAPE;
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
  if (int64_t(num_groups) * n_ct > INT32_MAX / 2) return FP8QGG_ERR_SHAPE;
  return FP8QGG_OK;
}

// Enqueues the kernel.  *work_counter must already be zero on `stream`.
int colwise_launch(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                   const int32_t *offsets, int32_t num_groups, uint8_t *q, int64_t ld_q,
                   int layout, float *scales, int fmt, float scale_max, uint64_t *sat_count,
                   int32_t *dev_status, uint32_t *work_counter, cudaStream_t stream) {
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
  const float smax = effective_scale_max(fmt, scale_max);
  ColKernel kern = col_kernel(fmt, layout, sat_count == nullptr && smax >= format_max(fmt));
  const int smem = static_cast<int>(sizeof(ColSmem)) + 1024;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FP8QGG_ERR_CUDA;
  const int64_t n_ct = (cols + kCW - 1) / kCW;
  const int64_t units = int64_t(num_groups) * n_ct;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, dev.sm_count)));
  const float sat_thr = saturation_threshold(fmt);
  kern<<<grid, kColThreads, smem, stream>>>(xmap, rows_total, static_cast<int>(cols), offsets,
                                            static_cast<int>(num_groups), q, ld_q, scales, smax,
                                            sat_thr,
                                            reinterpret_cast<unsigned long long *>(sat_count),
                                            dev_status, work_counter);
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}

}  // namespace fp8qgg

using namespace fp8qgg;

extern "C" size_t fp8_quant_colwise_jagged_workspace_size(int64_t rows_total, int64_t cols,
                                                          int32_t num_groups) {
  (void)rows_total;
  (void)cols;
  (void)num_groups;
  return kColwiseScratchBytes;
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
                        fmt, scale_max, sat_count, dev_status, static_cast<uint32_t *>(workspace),
                        s);
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
  // the previous call's work counter must not leak into this one
  if (cudaMemsetAsync(scratch, 0, need, s) != cudaSuccess) return FP8QGG_ERR_CUDA;
  return colwise_launch(x, rows_total, cols, ld_x, offsets, num_groups, q, ld_q, layout, scales,
                        fmt, scale_max, sat_count, dev_status, static_cast<uint32_t *>(scratch),
                        s);
}
