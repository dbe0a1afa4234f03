// Jagged column-wise FP8 quantisation into the padded transposed layout, and
// the dual-output form that also quantises the same rows rowwise, from one
// read of the input.
//
// Sources: "FP8 su GPU AMD: ..." (ai-radar.it) — introduction (one scale per
// activation row, one per column of each expert's weights, an offsets tensor
// routing tokens to experts), section "Il guadagno vero è nel movimento dei
// dati" (absmax -> scale -> clamp -> cast fused; the backward's
// .t().contiguous().t() copy removed; the output tile of the column-scales
// kernel transposed on chip so that its stores coalesce; relaxed atomics for
// the cross-block reduction).  "AMD Boosts PyTorch FP8 Training on Instinct
// GPUs", second and third paragraphs (the backward fusion).
//
// B200 design.  The input is cut into blocks of 128 rows of one group and
// panels of 256 columns (512-byte row segments: every warp load instruction
// reads one whole segment).  A block of a group with more than one block is
// visited twice:
//  - an "absmax" task: each of the eight warps loads its 16 rows straight into
//    registers (16 loads of 16 bytes in flight per lane), reduces the column
//    absmax, the warps meet in shared memory and the block's partial is merged
//    into the unit's column absmax in global memory with relaxed atomic max
//    (dual form: also every row's partial absmax over the panel); the block
//    is then counted in the unit's arrival counter;
//  - a "cast" task, later in the task list, once the unit's count is full:
//    the scales are derived, the rows are read again (from L2: the list
//    keeps the two visits about one grid-width of tasks apart), cast, and the
//    codes are written transposed into a 32 KB shared-memory tile (256
//    columns x 128 tokens, 128-byte swizzle) that one bulk tensor store sends
//    to the group's 128-token block of the padded layout.  Rows past the
//    group's end are zeros in the tile, so the same store writes the zero
//    codes of the padding.  The dual form also casts every row with its own
//    scale (from the merged row absmax) and stores it in place.
// A single-block unit of the column-wise form is one "whole" task (its
// absmax stays in shared memory).  The unit a cast waits for is one (group,
// panel) in the column-wise form and the whole group in the dual form (a
// row's scale needs every panel).  Tasks come from an atomic counter; the
// absmax tasks run largest group first, and the cast tasks of a unit are
// placed about one grid-width of tasks after the unit's last absmax task, so
// that a cast only waits for a task handed out earlier (to a running block).
#include <algorithm>
#include <cstring>
#include <mutex>

#include "device_common.cuh"
#include "host_common.h"
#include "quant_panels.h"

namespace fp8qgg {

constexpr int kPW = 256;                 // columns per panel
constexpr int kPWords = kPW / 2;         // bf16 pairs per panel row
constexpr int kRB = 128;                 // rows per block = tokens per store tile
constexpr int kPWarps = 8;
constexpr int kPThreads = 32 * kPWarps;
constexpr int kWR = kRB / kPWarps;       // rows per warp: 16
constexpr int kPMaxGroups = 1024;
constexpr uint32_t kTileBytes = kPW * kRB;  // [256 columns][128 tokens] codes
static_assert(kWR == 16, "a lane's tokens of one column fill one 16-byte piece");

enum : int { kTaskAbs = 0, kTaskCast = 1, kTaskWhole = 2 };

struct PanelSmem {
  uint8_t tile[2][kTileBytes];      // transposed code tiles (1024-byte aligned)
  uint32_t red[kPWarps][kPWords];   // per-warp column absmax, bf16 magnitude pairs
  uint32_t colmax[kPWords];         // whole tasks: the unit's column absmax
  float sc[kPW];                    // the panel's column scales
  int32_t end[kPMaxGroups];         // clamped group ends (by group index)
  int32_t pstart[kPMaxGroups];      // padded first token (by group index)
  int32_t order[kPMaxGroups];       // groups by size, largest first
  int32_t nb[kPMaxGroups];          // blocks of ordered group i
  int32_t gpre[kPMaxGroups + 1];    // ordered multi-block groups: blocks before group i
  int32_t n_multi, n_nonempty, a_total, s_total, total, npu;
  int32_t task, flag;
};
static_assert(offsetof(PanelSmem, tile) == 0, "tiles first (1024-byte aligned)");

struct PanelParams {
  const uint4 *x;        // bf16 rows as 16-byte vectors
  int64_t ld_x16;        // row pitch in 16-byte vectors
  int64_t rows_total;
  int cols;
  const int32_t *offsets;
  int num_groups;
  float *scales_col;     // [num_groups, cols]
  uint8_t *q_row;        // dual form: [rows_total, ld_qr] codes
  int64_t ld_qr;
  float *scales_row;     // dual form: [rows_total]
  float smax, sat_thr;
  unsigned long long *sat_count;
  int32_t *status;
  uint32_t *work;        // task counter
  uint32_t *arrive;      // per unit
  uint32_t *amax;        // [num_groups (ordered), cols] column absmax bits
  uint32_t *rowmax;      // dual form: [rows_total] row absmax bits
  int32_t delay;         // tasks between a unit's last absmax task and its casts
  UnitWait uw;
};

// Clamped group ends, padded starts, the size order and the task counts.
template <bool DUAL>
__device__ void panel_prologue(PanelSmem &sm, const PanelParams &p, int np) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int G = p.num_groups;
  const int32_t R = static_cast<int32_t>(p.rows_total);
  if (tid < 32) {
    int32_t carry_end = 0, carry_pad = 0;
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
      const int32_t ps = e < G ? ((endv - prev + kRB - 1) / kRB) * kRB : 0;
      int32_t incl = ps;
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += o;
      }
      if (e < G) {
        sm.end[e] = endv;
        sm.pstart[e] = carry_pad + incl - ps;
      }
      carry_end = __shfl_sync(0xFFFFFFFFu, endv, 31);
      carry_pad += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    bad = __any_sync(0xFFFFFFFFu, bad);
    if (bad && lane == 0 && blockIdx.x == 0) status_or(p.status, FP8QGG_STATUS_BAD_OFFSETS);
  }
  __syncthreads();
  for (int e = tid; e < G; e += kPThreads) {
    const int32_t se = sm.end[e] - (e ? sm.end[e - 1] : 0);
    int rank = 0;
    for (int f = 0; f < G; ++f) {
      const int32_t sf = sm.end[f] - (f ? sm.end[f - 1] : 0);
      rank += (sf > se) || (sf == se && f < e);
    }
    sm.order[rank] = e;
  }
  __syncthreads();
  if (tid < 32) {
    // multi-block groups are a prefix of the order (sizes decrease)
    int32_t carry = 0, n_multi = 0, n_ne = 0;
    for (int base = 0; base < G; base += 32) {
      const int i = base + lane;
      int32_t nbv = 0;
      if (i < G) {
        const int e = sm.order[i];
        const int32_t sz = sm.end[e] - (e ? sm.end[e - 1] : 0);
        nbv = (sz + kRB - 1) / kRB;
        sm.nb[i] = nbv;
      }
      // absmax tasks exist for multi-block groups (every non-empty group in
      // the dual form)
      const bool multi = DUAL ? nbv >= 1 : nbv >= 2;
      int32_t c = multi ? nbv : 0;
      int32_t incl = c;
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += o;
      }
      if (i < G) sm.gpre[i] = carry + incl - c;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
      n_multi += __popc(__ballot_sync(0xFFFFFFFFu, multi));
      n_ne += __popc(__ballot_sync(0xFFFFFFFFu, nbv >= 1));
    }
    if (lane == 0) {
      sm.gpre[G] = carry;
      sm.n_multi = n_multi;
      sm.n_nonempty = n_ne;
      const int32_t npu = DUAL ? 1 : np;  // units per group
      sm.npu = npu;
      // absmax tasks: every (multi group, panel, block); whole tasks: every
      // (single-block group, panel) of the column-wise form
      sm.a_total = carry * np;
      sm.s_total = sm.a_total + (DUAL ? 0 : (n_ne - n_multi) * np);
      sm.total = sm.s_total + sm.a_total;  // + one cast task per absmax task
    }
  }
  __syncthreads();
}

struct PTask {
  int kind;
  int i;      // ordered group
  int e;      // group index
  int p0, p1; // panels
  int b;      // block
  int u;      // unit (arrival counter)
  int32_t need;  // arrivals that complete the unit
};

// Position t of the task list.  The "A stream" holds the absmax tasks of the
// multi-block units (unit-major: group i, then panel p for the column-wise
// form, then block b), then the whole tasks.  The cast block of unit u
// (nbu tasks, same order) is inserted after A-stream index
// d_u = min(first_u + nbu + delay, S); first_u = the unit's first absmax index.
// Since the cast tasks before unit u number first_u as well, the cast block
// starts at list position d_u + first_u.
__device__ PTask decode_panel_task(const PanelSmem &sm, int32_t t, int np, int32_t delay) {
  const int npu = sm.npu;
  const int32_t S = sm.s_total;
  const int n_units = sm.n_multi * npu;
  // unit u = i * npu + q: first absmax index and block count
  auto unit_first = [&](int u, int32_t &first, int32_t &nbu) {
    const int i = u / npu, q = u - (u / npu) * npu;
    const int32_t nbi = sm.nb[i];
    nbu = npu == 1 ? nbi * np : nbi;
    first = sm.gpre[i] * np + q * nbi;
  };
  // largest unit whose cast block starts at or before t
  int lo = -1, hi = n_units - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    int32_t f, n;
    unit_first(mid, f, n);
    const int32_t pos = min(f + n + delay, S) + f;
    if (pos <= t) lo = mid; else hi = mid - 1;
  }
  PTask r;
  int32_t a = t;  // A-stream index, if t is not a cast
  if (lo >= 0) {
    int32_t f, n;
    unit_first(lo, f, n);
    const int32_t pos = min(f + n + delay, S) + f;
    if (t < pos + n) {
      // cast task: block (t - pos) of unit lo, in the unit's absmax order
      const int32_t k = t - pos;
      const int i = lo / npu;
      const int32_t nbi = sm.nb[i];
      r.kind = kTaskCast;
      r.i = i;
      r.u = lo;
      r.need = n;
      if (npu == 1) {
        r.p0 = k / nbi;
        r.b = k - r.p0 * nbi;
      } else {
        r.p0 = lo - i * npu;
        r.b = k;
      }
      r.p1 = r.p0 + 1;
      r.e = sm.order[i];
      return r;
    }
    a = t - (f + n);  // every cast before t belongs to units 0..lo
  }
  if (a < sm.a_total) {
    // absmax task: ordered group by binary search over the block prefix
    int glo = 0, ghi = sm.n_multi - 1;
    while (glo < ghi) {
      const int mid = (glo + ghi + 1) >> 1;
      if (sm.gpre[mid] * np <= a) glo = mid; else ghi = mid - 1;
    }
    const int32_t nbi = sm.nb[glo];
    const int32_t k = a - sm.gpre[glo] * np;
    r.kind = kTaskAbs;
    r.i = glo;
    r.p0 = k / nbi;
    r.p1 = r.p0 + 1;
    r.b = k - r.p0 * nbi;
    r.u = glo * npu + (npu == 1 ? 0 : r.p0);
    r.need = npu == 1 ? nbi * np : nbi;
  } else {
    // whole task (column-wise form only): single-block group, one panel
    const int32_t w = a - sm.a_total;
    r.kind = kTaskWhole;
    r.i = sm.n_multi + w / np;
    r.p0 = w - (w / np) * np;
    r.p1 = r.p0 + 1;
    r.b = 0;
    r.u = -1;
    r.need = 0;
  }
  r.e = sm.order[r.i];
  return r;
}

__device__ __forceinline__ uint32_t hmax_bits(uint32_t acc) {
  const uint32_t m = absmax_bits(acc);
  return max(m & 0xFFFFu, m >> 16);
}

template <int FMT, bool FAST>
__device__ __forceinline__ uint32_t enc_pair(float x0, float x1, float s0, float s1, float smax,
                                             float sat_thr, uint32_t &sat) {
  if constexpr (FAST) {
    uint64_t xx, yy;
    asm("mov.b64 %0, {%1, %2};" : "=l"(xx) : "f"(x0), "f"(x1));
    const uint64_t ss = pack_f32x2(s0, s1);
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(yy) : "l"(xx), "l"(ss));
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

__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t word(const uint4 &v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// Loads the lane's 16 rows x 8 columns (rows [r0, r1) of the block; the rest
// read as zero).  EVICT: the cast's second read, last use of the data.
template <bool SECOND>
__device__ __forceinline__ void load_rows(uint4 (&v)[kWR], const PanelParams &p, int32_t rw0,
                                          int32_t r1, int64_t cvec, bool lane_ok) {
#pragma unroll
  for (int k = 0; k < kWR; ++k) {
    const int32_t row = rw0 + k;
    if (lane_ok && row < r1) {
      const uint4 *src = p.x + static_cast<int64_t>(row) * p.ld_x16 + cvec;
      v[k] = SECOND ? __ldcs(src) : __ldcg(src);
    } else {
      v[k] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

template <int FMT, bool FAST, bool DUAL>
__global__ void __launch_bounds__(kPThreads, 2)
    quant_panel_kernel(const __grid_constant__ CUtensorMap qmap, const PanelParams p) {
  extern __shared__ uint8_t smem_raw[];
  PanelSmem &sm = *align_smem_1024<PanelSmem>(smem_raw);
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int np = (p.cols + kPW - 1) / kPW;
  if (tid == 0 && p.rows_total > 0) prefetch_tensormap(&qmap);
  panel_prologue<DUAL>(sm, p, np);

  // empty groups: scales only (Fmax / 1e-12 in every column), no codes
  for (int i = sm.n_nonempty + static_cast<int>(blockIdx.x); i < p.num_groups;
       i += static_cast<int>(gridDim.x)) {
    const int e = sm.order[i];
    const float s = scale_from_amax(0.0f, p.smax);
    for (int c = tid; c < p.cols; c += kPThreads) p.scales_col[static_cast<int64_t>(e) * p.cols + c] = s;
  }

  uint32_t sat = 0;
  uint32_t tile_parity = 0;
  const int32_t total = sm.total;
  int32_t next = 0;
  if (tid == 0) next = static_cast<int32_t>(atomicAdd(p.work, 1u));
  while (true) {
    if (tid == 0) {
      const int32_t t = next;
      if (t < total) next = static_cast<int32_t>(atomicAdd(p.work, 1u));
      sm.task = t;
    }
    __syncthreads();
    const int32_t t = sm.task;
    if (t >= total) break;
    const PTask tk = decode_panel_task(sm, t, np, p.delay);
    const int e = tk.e;
    const int32_t gs = e ? sm.end[e - 1] : 0;
    const int32_t ge = sm.end[e];
    const int32_t r0 = gs + tk.b * kRB;
    const int32_t r1 = min(ge, r0 + kRB);
    const int32_t rw0 = r0 + kWR * w;
    const int64_t amax_base = static_cast<int64_t>(tk.i) * p.cols;

    if (tk.kind != kTaskCast) {
      // ------------------------------------------------------------ absmax
      for (int pp = tk.p0; pp < tk.p1; ++pp) {
        const int c0 = pp * kPW;
        const bool lane_ok = c0 + 8 * lane < p.cols;
        uint4 v[kWR];
        load_rows<false>(v, p, rw0, r1, (c0 >> 3) + lane, lane_ok);
        uint4 am = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int k = 0; k < kWR; ++k) {
          am.x = absmax_acc(am.x, v[k].x);
          am.y = absmax_acc(am.y, v[k].y);
          am.z = absmax_acc(am.z, v[k].z);
          am.w = absmax_acc(am.w, v[k].w);
        }
        if constexpr (DUAL) {
          // the row's partial absmax over this panel, merged per row
          uint32_t rm[kWR];
#pragma unroll
          for (int k = 0; k < kWR; ++k) {
            uint32_t a2 = absmax_acc(absmax_acc(0u, v[k].x), v[k].y);
            a2 = absmax_acc(absmax_acc(a2, v[k].z), v[k].w);
            rm[k] = hmax_bits(a2);
          }
          // 16 values over 32 lanes: halve four times, then pair lanes
#pragma unroll
          for (int h = 8; h >= 1; h >>= 1) {
            const bool upper = (lane & (2 * h)) != 0;  // partner bits 16, 8, 4, 2
#pragma unroll
            for (int k = 0; k < h; ++k) {
              const uint32_t send = upper ? rm[k] : rm[k + h];
              const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, send, 2 * h);
              rm[k] = max(upper ? rm[k + h] : rm[k], got);
            }
          }
          const uint32_t rmax = max(rm[0], __shfl_xor_sync(0xFFFFFFFFu, rm[0], 1));
          const int32_t row = rw0 + ((lane >> 1) & 15);
          if (!(lane & 1) && row < r1) atomicMax(p.rowmax + row, rmax);
        }
        am = make_uint4(absmax_bits(am.x), absmax_bits(am.y), absmax_bits(am.z),
                        absmax_bits(am.w));
        *reinterpret_cast<uint4 *>(&sm.red[w][4 * lane]) = am;
        __syncthreads();
        if (tid < kPWords) {
          uint32_t m = 0;
#pragma unroll
          for (int ww = 0; ww < kPWarps; ++ww) m = __vmaxu2(m, sm.red[ww][tid]);
          const int c = c0 + 2 * tid;
          if (tk.kind == kTaskWhole) {
            sm.colmax[tid] = m;
          } else if (c < p.cols) {
            atomicMax(p.amax + amax_base + c, m & 0xFFFFu);
            atomicMax(p.amax + amax_base + c + 1, m >> 16);
          }
        }
        __syncthreads();
      }
      if (tk.kind == kTaskAbs) {
        __threadfence();  // this thread's merges are visible before the count
        __syncthreads();
        if (tid == 0) atomicAdd(p.arrive + tk.u, 1u);
        continue;
      }
    }

    // ------------------------------------------------------------ cast
    if (tk.kind == kTaskCast) {
      if (tid == 0) {
        const uint32_t *cnt = p.arrive + tk.u;
        const uint32_t target = static_cast<uint32_t>(tk.need) + p.uw.extra_arrivals;
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
        int ok = 1;
        if (v < target) {
          const uint64_t t0 = global_timer_ns();
          while (true) {
            __nanosleep(128);
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
            if (v >= target) break;
            if (global_timer_ns() - t0 > p.uw.limit_ns) { ok = 0; break; }
          }
        }
        sm.flag = ok;
      }
      __syncthreads();
      if (!sm.flag) {
        if (tid == 0) status_or(p.status, FP8QGG_STATUS_TIMEOUT);
        break;  // this block takes no more tasks; earlier stores complete below
      }
    }
    float rs_lane = 0.0f;  // dual form: the scale of row rw0 + lane (lanes 0..15)
    if constexpr (DUAL) {
      const int32_t row = rw0 + lane;
      if (lane < kWR && row < r1) {
        const uint32_t bits = __ldcg(p.rowmax + row);
        rs_lane = scale_from_amax(bf16_bits_to_float(bits), p.smax);
        if (tk.p0 == 0) p.scales_row[row] = rs_lane;
      }
    }
    for (int pp = tk.p0; pp < tk.p1; ++pp) {
      const int c0 = pp * kPW;
      const bool lane_ok = c0 + 8 * lane < p.cols;
      {  // the panel's column scales, one column per thread
        const int c = c0 + tid;
        if (c < p.cols) {
          uint32_t bits;
          if (tk.kind == kTaskWhole)
            bits = (tid & 1) ? sm.colmax[tid >> 1] >> 16 : sm.colmax[tid >> 1] & 0xFFFFu;
          else
            bits = __ldcg(p.amax + amax_base + c);
          const float s = scale_from_amax(bf16_bits_to_float(bits), p.smax);
          sm.sc[tid] = s;
          if (tk.b == 0) p.scales_col[static_cast<int64_t>(e) * p.cols + c] = s;
        }
        // the tile about to be written was sent two stores ago: its store must
        // have read it
        if (tid == 0) bulk_wait_read<1>();
      }
      __syncthreads();
      float s[8];
      {
        const float4 a = *reinterpret_cast<const float4 *>(&sm.sc[8 * lane]);
        const float4 b = *reinterpret_cast<const float4 *>(&sm.sc[8 * lane + 4]);
        s[0] = a.x; s[1] = a.y; s[2] = a.z; s[3] = a.w;
        s[4] = b.x; s[5] = b.y; s[6] = b.z; s[7] = b.w;
      }
      uint4 v[kWR];
      load_rows<true>(v, p, rw0, r1, (c0 >> 3) + lane, lane_ok);
      if constexpr (DUAL) {
        // rowwise codes in place: 8 columns of each row, one 8-byte store
#pragma unroll
        for (int k = 0; k < kWR; ++k) {
          const float rs = __shfl_sync(0xFFFFFFFFu, rs_lane, k);
          const int32_t row = rw0 + k;
          uint32_t c2[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t wd = word(v[k], j);
            c2[j] = enc_pair<FMT, FAST>(lo_f(wd), hi_f(wd), rs, rs, p.smax, p.sat_thr, sat);
          }
          if (lane_ok && row < r1)
            *reinterpret_cast<uint2 *>(p.q_row + static_cast<int64_t>(row) * p.ld_qr + c0 +
                                       8 * lane) =
                make_uint2(c2[0] | (c2[1] << 16), c2[2] | (c2[3] << 16));
        }
      }
      // column-wise codes: column 8*lane + j, tokens rw0 .. rw0 + 15 as one
      // 16-byte piece
      uint4 tok[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int wj = j >> 1;
        uint32_t c2[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const uint32_t w0 = word(v[2 * m], wj), w1 = word(v[2 * m + 1], wj);
          const float x0 = (j & 1) ? hi_f(w0) : lo_f(w0);
          const float x1 = (j & 1) ? hi_f(w1) : lo_f(w1);
          // rows past the group's end are zero: their codes are the padding
          c2[m] = enc_pair<FMT, FAST>(x0, x1, s[j], s[j], p.smax, p.sat_thr, sat);
        }
        tok[j] = make_uint4(c2[0] | (c2[1] << 16), c2[2] | (c2[3] << 16),
                            c2[4] | (c2[5] << 16), c2[6] | (c2[7] << 16));
      }
      // rotate by lane % 8, so that the eight lanes of a shared-memory phase
      // write eight different 16-byte bank groups of the swizzled tile
      const int rot = lane & 7;
#pragma unroll
      for (int st = 1; st < 8; st <<= 1) {
        if (rot & st) {
          uint4 tmp[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) tmp[j] = tok[(j + st) & 7];
#pragma unroll
          for (int j = 0; j < 8; ++j) tok[j] = tmp[j];
        }
      }
      uint8_t *tile = sm.tile[tile_parity];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int cc = 8 * lane + ((j + rot) & 7);  // tile row = column of the panel
        // 128-byte swizzle: 16-byte piece w of row cc sits at piece w ^ (cc % 8)
        *reinterpret_cast<uint4 *>(tile + cc * kRB + 16 * (w ^ (cc & 7))) = tok[j];
      }
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        tma_store_2d(&qmap, tile, sm.pstart[e] + tk.b * kRB, c0);
        bulk_commit();
      }
      tile_parity ^= 1;
    }
  }
  if (tid == 0) bulk_wait_all();  // the tiles stay valid until their stores have read them
  if (!FAST && p.sat_count) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sat += __shfl_xor_sync(0xFFFFFFFFu, sat, off);
    if (lane == 0 && sat) atomicAdd(p.sat_count, static_cast<unsigned long long>(sat));
  }
}

namespace {

using PanelKernel = void (*)(const CUtensorMap, const PanelParams);

template <bool DUAL>
PanelKernel panel_kernel(int fmt, bool fast) {
  if (fmt == FP8QGG_E4M3FN)
    return fast ? quant_panel_kernel<FP8QGG_E4M3FN, true, DUAL>
                : quant_panel_kernel<FP8QGG_E4M3FN, false, DUAL>;
  return fast ? quant_panel_kernel<FP8QGG_E4M3FNUZ, true, DUAL>
              : quant_panel_kernel<FP8QGG_E4M3FNUZ, false, DUAL>;
}

}  // namespace

PanelScratch panel_scratch(int64_t rows_total, int64_t cols, int32_t num_groups, bool dual) {
  PanelScratch s;
  const int64_t np = (std::max<int64_t>(cols, 1) + kPW - 1) / kPW;
  const int64_t g = std::max<int32_t>(num_groups, 1);
  s.arrive_off = 256;
  s.amax_off = s.arrive_off + (static_cast<size_t>(g * np) * 4 + 255) / 256 * 256;
  s.rowmax_off = s.amax_off + (static_cast<size_t>(g * std::max<int64_t>(cols, 1)) * 4 + 255) /
                                  256 * 256;
  s.bytes = s.rowmax_off +
            (dual ? (static_cast<size_t>(std::max<int64_t>(rows_total, 0)) * 4 + 255) / 256 * 256
                  : 0);
  return s;
}

int panel_launch(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                 const int32_t *offsets, int32_t num_groups, uint8_t *q_col, int64_t ld_qc,
                 float *scales_col, uint8_t *q_row, int64_t ld_qr, float *scales_row, int fmt,
                 float scale_max, uint64_t *sat_count, int32_t *dev_status, void *scratch,
                 UnitWait uw, cudaStream_t stream) {
  const bool dual = q_row != nullptr;
  CUtensorMap qmap;
  memset(&qmap, 0, sizeof qmap);
  if (rows_total > 0) {
    // codes [cols][ld_qc tokens]; boxes of 128 tokens x 256 columns (fewer
    // columns when the tensor has fewer), 128-byte swizzle
    const uint64_t dims[2] = {static_cast<uint64_t>(ld_qc), static_cast<uint64_t>(cols)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ld_qc)};
    const uint32_t box[2] = {kRB, static_cast<uint32_t>(std::min<int64_t>(kPW, cols))};
    if (!encode_tensor_map(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q_col, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return FP8QGG_ERR_CUDA;
  }
  DeviceInfo dev;
  if (!device_info(&dev)) return FP8QGG_ERR_CUDA;
  const float smax = effective_scale_max(fmt, scale_max);
  const bool fast = sat_count == nullptr && smax >= format_max(fmt);
  PanelKernel kern = dual ? panel_kernel<true>(fmt, fast) : panel_kernel<false>(fmt, fast);
  const int smem = static_cast<int>(sizeof(PanelSmem)) + 1024;
  if (!set_max_dynamic_smem(reinterpret_cast<const void *>(kern), smem)) return FP8QGG_ERR_CUDA;
  const PanelScratch sl = panel_scratch(rows_total, cols, num_groups, dual);
  uint8_t *base = static_cast<uint8_t *>(scratch);
  PanelParams prm;
  prm.x = static_cast<const uint4 *>(x);
  prm.ld_x16 = ld_x / 8;
  prm.rows_total = rows_total;
  prm.cols = static_cast<int>(cols);
  prm.offsets = offsets;
  prm.num_groups = num_groups;
  prm.scales_col = scales_col;
  prm.q_row = q_row;
  prm.ld_qr = ld_qr;
  prm.scales_row = scales_row;
  prm.smax = smax;
  prm.sat_thr = saturation_threshold(fmt);
  prm.sat_count = reinterpret_cast<unsigned long long *>(sat_count);
  prm.status = dev_status;
  prm.work = reinterpret_cast<uint32_t *>(base);
  prm.arrive = reinterpret_cast<uint32_t *>(base + sl.arrive_off);
  prm.amax = reinterpret_cast<uint32_t *>(base + sl.amax_off);
  prm.rowmax = reinterpret_cast<uint32_t *>(base + sl.rowmax_off);
  prm.uw = uw;
  // blocks: two per SM, never more than the tasks (at least one, for the
  // scales of empty groups)
  const int64_t np = (cols + kPW - 1) / kPW;
  const int64_t blocks_max = (rows_total + int64_t(kRB) * num_groups) / kRB * np;
  const int grid = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(2 * blocks_max, int64_t(dev.sm_count) * 2)));
  prm.delay = grid;
  kern<<<grid, kPThreads, smem, stream>>>(qmap, prm);
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}

}  // namespace fp8qgg

using namespace fp8qgg;

extern "C" size_t fp8_quant_dual_jagged_workspace_size(int64_t rows_total, int64_t cols,
                                                       int32_t num_groups) {
  return panel_scratch(rows_total, cols, num_groups, true).bytes;
}

extern "C" int fp8_quant_dual_jagged(const void *x, int64_t rows_total, int64_t cols,
                                     int64_t ld_x, const int32_t *offsets, int32_t num_groups,
                                     uint8_t *q_row, int64_t ld_qr, float *scales_row,
                                     uint8_t *q_col, int64_t ld_qc, float *scales_col, int fmt,
                                     float scale_max, uint64_t *sat_count, int32_t *dev_status,
                                     void *workspace, size_t workspace_bytes, void *stream) {
  int rc = colwise_check(x, rows_total, cols, ld_x, offsets, num_groups, q_col, ld_qc,
                         FP8QGG_LAYOUT_TRANSPOSED_PADDED, scales_col, fmt, scale_max, sat_count,
                         dev_status);
  if (rc != FP8QGG_OK) return rc;
  if (ld_qr < cols) return FP8QGG_ERR_SHAPE;
  if (rows_total > 0 && (!q_row || !scales_row)) return FP8QGG_ERR_NULL;
  if (ld_qr % 8) return FP8QGG_ERR_ALIGN;
  if ((q_row && !aligned(q_row, 16)) || (scales_row && !aligned(scales_row, 4)))
    return FP8QGG_ERR_ALIGN;
  if (!workspace) return FP8QGG_ERR_NULL;
  if (!aligned(workspace, 16)) return FP8QGG_ERR_ALIGN;
  const size_t need = fp8_quant_dual_jagged_workspace_size(rows_total, cols, num_groups);
  if (workspace_bytes < need) return FP8QGG_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, need, s) != cudaSuccess) return FP8QGG_ERR_CUDA;
  // a row pointer is needed to select the dual form even when no row exists
  uint8_t *qr = q_row ? q_row : reinterpret_cast<uint8_t *>(workspace);
  return panel_launch(x, rows_total, cols, ld_x, offsets, num_groups, q_col, ld_qc, scales_col,
                      qr, ld_qr, scales_row, fmt, scale_max, sat_count, dev_status, workspace,
                      current_unit_wait(), s);
}
