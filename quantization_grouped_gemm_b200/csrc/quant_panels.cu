// Jagged column-wise FP8 quantisation into the padded transposed layout, and
// the dual-output form that also quantises the same rows rowwise, from one
// read of the input.
//
// Sources: "FP8 su GPU AMD: ..." (ai-radar.it) — introduction (one scale per
// activation row, one per column of each expert's weights, an offsets tensor
// routing tokens to experts), section "Il guadagno vero è nel movimento dei
// dati" (absmax -> scale -> clamp -> cast fused; the backward's
// .t().contiguous().t() copy removed; the column-scales kernel's output
// transposed on chip so that its stores coalesce; relaxed atomics for the
// cross-block reduction).  "AMD Boosts PyTorch FP8 Training on Instinct GPUs",
// second and third paragraphs (the backward fusion).
//
// B200 design.  The input is cut into panels of 256 columns (one warp load
// instruction reads a whole 512-byte row segment; lane l owns columns
// 8l .. 8l + 7) and blocks of 128 rows of one group; a block of a panel is
// one task of a block of eight warps, each warp owning 16 rows.  A block of a
// group with more than one block is visited twice:
//  - an "absmax" task: every warp loads its 16 rows straight into registers
//    (16 loads of 16 bytes in flight per lane) and reduces its column absmax;
//    the warps meet in shared memory, then each warp merges 32 of the
//    panel's columns into the unit's absmax words in global memory with
//    relaxed atomic max and counts itself in the unit's arrival counter (the
//    dual form also merges every row's absmax over the panel);
//  - a "cast" task, later in the task list, once the unit's count is full:
//    every lane derives its 8 scales, reads its rows again (from L2: the
//    list keeps the two visits about one grid-width of tasks apart), encodes
//    two rows of a column per conversion and writes each column's 16 tokens
//    into a 32 KB shared-memory tile (256 columns x 128 tokens, 128-byte
//    swizzle), which one bulk tensor store sends to the group's 128-token
//    block of the padded layout: whole 128-byte lines, zero codes of the
//    padding included (rows past the group's end are zeros).  The dual form
//    also encodes every row with its own scale and stores it in place.
// A single-block unit of the column-wise form is one "whole" task (absmax
// and cast from the same registers).  The unit a cast waits for is one
// (group, panel) in the column-wise form and the whole group in the dual
// form (a row's scale needs every panel).  Tasks come from an atomic counter
// read by warp 0, which also finds the next task (a 32-way search, one
// candidate per lane) while the block works on the current one; each task
// ends with the block's only barrier.  The absmax tasks run largest group
// first, and the casts of a unit are placed about one grid-width of tasks
// after its last absmax task, so that a cast only waits for tasks handed out
// earlier (to running blocks).
#include <algorithm>
#include <cstring>

#include "device_common.cuh"
#include "host_common.h"
#include "quant_panels.h"

namespace fp8qgg {

constexpr int kPW = 256;               // columns per panel
constexpr int kPWords = kPW / 2;       // bf16 pairs per panel row
constexpr int kRB = 128;               // rows per block = tokens per store tile
constexpr int kPWarps = 8;
constexpr int kPThreads = 32 * kPWarps;
constexpr int kWR = kRB / kPWarps;     // rows per warp: 16
constexpr int kPBlocksPerSM = 2;
constexpr int kPMaxGroups = 1024;
constexpr uint32_t kTileBytes = kPW * kRB;
static_assert(kWR == 16, "a lane's tokens of one column fill one 16-byte piece");

enum : int { kTaskAbs = 0, kTaskCast = 1, kTaskWhole = 2, kTaskEnd = 3 };

struct PTask {
  int32_t kind;
  int32_t i, e;   // ordered group, group index
  int32_t q;      // panel
  int32_t b;      // block of the group
  int32_t u;      // unit (arrival counter)
  int32_t need;   // arrivals that complete the unit
  int32_t pad;
};

struct PanelSmem {
  uint8_t tile[2][kTileBytes];          // transposed code tiles (1024-byte aligned)
  uint32_t red[2][kPWarps][kPWords];    // per-warp column absmax (bf16 magnitude pairs)
  PTask tk[2];                          // the current and the next task
  int32_t end[kPMaxGroups];             // clamped group ends (by group index)
  int32_t pstart[kPMaxGroups];          // padded first token (by group index)
  int32_t order[kPMaxGroups];           // groups by size, largest first
  int32_t nb[kPMaxGroups];              // ordered group i: 128-row blocks
  int32_t apre[kPMaxGroups + 1];        // multi-block groups: blocks before group i
  int32_t n_multi, n_nonempty, a_total, s_total, total;
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
  uint32_t *amax;        // [ordered group, cols] column absmax bits
  uint32_t *rowmax;      // dual form: [rows_total] row absmax bits
  int32_t delay;         // list positions between a unit's last absmax task and its casts
  UnitWait uw;
};

__device__ __forceinline__ int32_t warp_scan_incl(int32_t v, int lane) {
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t o = __shfl_up_sync(0xFFFFFFFFu, v, d);
    if (lane >= d) v += o;
  }
  return v;
}

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
      const int32_t incl = warp_scan_incl(ps, lane);
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
    // groups with absmax and cast tasks ("multi") are a prefix of the order:
    // every non-empty group in the dual form, groups of more than one block
    // in the column-wise form (single-block ones are whole tasks)
    int32_t carry = 0, n_multi = 0, n_ne = 0;
    for (int base = 0; base < G; base += 32) {
      const int i = base + lane;
      int32_t nbv = 0;
      if (i < G) {
        const int e = sm.order[i];
        nbv = (sm.end[e] - (e ? sm.end[e - 1] : 0) + kRB - 1) / kRB;
        sm.nb[i] = nbv;
      }
      const bool multi = DUAL ? nbv >= 1 : nbv >= 2;
      const int32_t c = multi ? nbv : 0;
      const int32_t incl = warp_scan_incl(c, lane);
      if (i < G) sm.apre[i] = carry + incl - c;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
      n_multi += __popc(__ballot_sync(0xFFFFFFFFu, multi));
      n_ne += __popc(__ballot_sync(0xFFFFFFFFu, nbv >= 1));
    }
    if (lane == 0) {
      sm.apre[G] = carry;
      sm.n_multi = n_multi;
      sm.n_nonempty = n_ne;
      sm.a_total = carry * np;
      sm.s_total = sm.a_total + (DUAL ? 0 : (n_ne - n_multi) * np);
      sm.total = sm.s_total + sm.a_total;  // one cast per absmax task
    }
  }
  __syncthreads();
}

// Unit u: first absmax index (= cast tasks before its cast block) and count.
template <bool DUAL>
__device__ __forceinline__ void unit_span(const PanelSmem &sm, int np, int u, int32_t &fa,
                                          int32_t &na) {
  if constexpr (DUAL) {
    fa = sm.apre[u] * np;
    na = sm.nb[u] * np;
  } else {
    const int i = u / np, q = u - (u / np) * np;
    fa = sm.apre[i] * np + q * sm.nb[i];
    na = sm.nb[i];
  }
}

// Task at position t of the list (called by a whole warp; every lane gets the
// same task).  The "A stream" holds the absmax tasks of the multi units
// (group i in size order, panel q, block b), then the whole tasks.  The cast
// block of unit u (same blocks, same order) is inserted after A-stream index
// d_u = min(fa_u + na_u + delay, S); the casts before it number fa_u, so it
// starts at list position d_u + fa_u.
template <bool DUAL>
__device__ PTask decode_panel_task(const PanelSmem &sm, int32_t t, int np, int32_t delay,
                                   int lane) {
  PTask r;
  r.pad = 0;
  if (t >= sm.total) {
    r.kind = kTaskEnd;
    r.i = r.e = r.q = r.b = r.u = r.need = 0;
    return r;
  }
  const int32_t S = sm.s_total;
  const int U = DUAL ? sm.n_multi : sm.n_multi * np;
  auto pos_of = [&](int u) -> int32_t {
    int32_t fa, na;
    unit_span<DUAL>(sm, np, u, fa, na);
    return min(fa + na + delay, S) + fa;
  };
  int best = -1;
  if (U > 0 && pos_of(0) <= t) {
    int lo = 0, hi = U;  // pos(lo) <= t; the answer lies in [lo, hi)
    while (hi - lo > 1) {
      const int step = (hi - lo + 31) / 32;
      const int c = lo + lane * step;
      const bool ok = c < hi && pos_of(c) <= t;
      const int n = __popc(__ballot_sync(0xFFFFFFFFu, ok));  // lanes 0 .. n-1
      const int nlo = lo + (n - 1) * step;
      hi = min(hi, nlo + step);
      lo = nlo;
    }
    best = lo;
  }
  int32_t a = t;  // A-stream index, if t is not a cast
  if (best >= 0) {
    int32_t fa, na;
    unit_span<DUAL>(sm, np, best, fa, na);
    const int32_t pos = min(fa + na + delay, S) + fa;
    if (t < pos + na) {
      const int32_t k = t - pos;
      r.kind = kTaskCast;
      r.u = best;
      r.need = kPWarps * na;  // every warp of every absmax task arrives
      if constexpr (DUAL) {
        r.i = best;
        const int32_t per = sm.nb[best];
        r.q = k / per;
        r.b = k - r.q * per;
      } else {
        r.i = best / np;
        r.q = best - r.i * np;
        r.b = k;
      }
      r.e = sm.order[r.i];
      return r;
    }
    a = t - (fa + na);  // every cast before t belongs to units 0 .. best
  }
  if (a < sm.a_total) {
    int lo = 0, hi = sm.n_multi;  // apre[lo] * np <= a
    while (hi - lo > 1) {
      const int step = (hi - lo + 31) / 32;
      const int c = lo + lane * step;
      const bool ok = c < hi && sm.apre[c] * np <= a;
      const int n = __popc(__ballot_sync(0xFFFFFFFFu, ok));
      const int nlo = lo + (n - 1) * step;
      hi = min(hi, nlo + step);
      lo = nlo;
    }
    const int32_t nbi = sm.nb[lo];
    const int32_t rr = a - sm.apre[lo] * np;
    r.kind = kTaskAbs;
    r.i = lo;
    r.q = rr / nbi;
    r.b = rr - r.q * nbi;
    r.u = DUAL ? lo : lo * np + r.q;
    r.need = 0;
  } else {
    const int32_t w = a - sm.a_total;  // whole task: single-block group, one panel
    r.kind = kTaskWhole;
    r.i = sm.n_multi + w / np;
    r.q = w - (w / np) * np;
    r.b = 0;
    r.u = -1;
    r.need = 0;
  }
  r.e = sm.order[r.i];
  return r;
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

// The lane's 16 rows x 8 columns from row rw0 (rows at or past r1 read as
// zero).  SECOND: the cast's re-read, the data's last use.
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

// Dual form: every row's absmax over the lane's 8 columns, reduced over the
// warp (16 values over 32 lanes: halve four times, then pair lanes), merged
// into the row's absmax word.
__device__ __forceinline__ void merge_row_amax(const uint4 (&v)[kWR], uint32_t *rowmax,
                                               int32_t rw0, int32_t r1, int lane) {
  uint32_t rm[kWR];
#pragma unroll
  for (int k = 0; k < kWR; ++k) {
    uint32_t a2 = absmax_acc(absmax_acc(0u, v[k].x), v[k].y);
    a2 = absmax_acc(absmax_acc(a2, v[k].z), v[k].w);
    const uint32_t m = absmax_bits(a2);
    rm[k] = max(m & 0xFFFFu, m >> 16);
  }
#pragma unroll
  for (int h = 8; h >= 1; h >>= 1) {
    const bool upper = (lane & (2 * h)) != 0;
#pragma unroll
    for (int k = 0; k < h; ++k) {
      const uint32_t send = upper ? rm[k] : rm[k + h];
      const uint32_t got = __shfl_xor_sync(0xFFFFFFFFu, send, 2 * h);
      rm[k] = max(upper ? rm[k + h] : rm[k], got);
    }
  }
  const uint32_t rmax = max(rm[0], __shfl_xor_sync(0xFFFFFFFFu, rm[0], 1));
  const int32_t row = rw0 + ((lane >> 1) & 15);  // lanes 2j, 2j+1 hold row rw0 + j
  if (!(lane & 1) && row < r1) atomicMax(rowmax + row, rmax);
}

// The lane's 8 column scales (16-byte stores when the address allows).
__device__ __forceinline__ void store_scales8(float *d, const float (&s)[8]) {
  if ((reinterpret_cast<uintptr_t>(d) & 15) == 0) {
    reinterpret_cast<float4 *>(d)[0] = make_float4(s[0], s[1], s[2], s[3]);
    reinterpret_cast<float4 *>(d)[1] = make_float4(s[4], s[5], s[6], s[7]);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) d[j] = s[j];
  }
}

// Column-wise codes of the lane's 16 rows into the tile: column 8*lane + j as
// one 16-byte piece (adjacent rows of a column share one conversion), at tile
// row 8*lane + j, piece w ^ (row % 8) (128-byte swizzle).  The pieces are
// stored in rotated order (lane % 8 steps), so that the 8 lanes of a
// shared-memory phase hit 8 different 16-byte bank groups.
template <int FMT, bool FAST>
__device__ __forceinline__ void tile_col_codes(const uint4 (&v)[kWR], const float (&s)[8],
                                               uint8_t *tile, int w, int lane, float smax,
                                               float sat_thr, uint32_t &sat) {
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
      c2[m] = enc_pair<FMT, FAST>(x0, x1, s[j], s[j], smax, sat_thr, sat);
    }
    tok[j] = make_uint4(c2[0] | (c2[1] << 16), c2[2] | (c2[3] << 16), c2[4] | (c2[5] << 16),
                        c2[6] | (c2[7] << 16));
  }
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
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int cc = 8 * lane + ((j + rot) & 7);
    *reinterpret_cast<uint4 *>(tile + cc * kRB + 16 * (w ^ (cc & 7))) = tok[j];
  }
}

template <int FMT, bool FAST, bool DUAL>
__global__ void __launch_bounds__(kPThreads, kPBlocksPerSM)
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
    for (int c = tid; c < p.cols; c += kPThreads)
      p.scales_col[static_cast<int64_t>(e) * p.cols + c] = s;
  }

  // warp 0 fetches and decodes the tasks, one ahead of the block
  int32_t next = 0;
  if (w == 0) {
    int32_t t = 0;
    if (lane == 0) {
      t = static_cast<int32_t>(atomicAdd(p.work, 1u));
      next = static_cast<int32_t>(atomicAdd(p.work, 1u));
    }
    t = __shfl_sync(0xFFFFFFFFu, t, 0);
    const PTask tk = decode_panel_task<DUAL>(sm, t, np, p.delay, lane);
    if (lane == 0) sm.tk[0] = tk;
  }
  __syncthreads();

  uint32_t sat = 0;
  bool failed = false;
  for (int n = 0;; ++n) {
    const int cur = n & 1;
    const PTask tk = sm.tk[cur];
    if (tk.kind == kTaskEnd) break;
    const int e = tk.e;
    const int32_t gs = e ? sm.end[e - 1] : 0;
    const int32_t ge = sm.end[e];
    const int32_t r0 = gs + tk.b * kRB;
    const int32_t r1 = min(ge, r0 + kRB);
    const int32_t rw0 = r0 + kWR * w;
    const int c0 = tk.q * kPW;
    const bool lane_ok = c0 + 8 * lane < p.cols;
    const int64_t cvec = (c0 >> 3) + lane;
    const int64_t amax_base = static_cast<int64_t>(tk.i) * p.cols + c0;
    uint8_t *tile = sm.tile[cur];

    uint4 v[kWR];
    float s[8];
    if (tk.kind != kTaskCast) {
      // ---------------------------------------------------------- absmax
      load_rows<false>(v, p, rw0, r1, cvec, lane_ok);
      uint4 am = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int k = 0; k < kWR; ++k) {
        am.x = absmax_acc(am.x, v[k].x);
        am.y = absmax_acc(am.y, v[k].y);
        am.z = absmax_acc(am.z, v[k].z);
        am.w = absmax_acc(am.w, v[k].w);
      }
      if constexpr (DUAL) merge_row_amax(v, p.rowmax, rw0, r1, lane);
      *reinterpret_cast<uint4 *>(&sm.red[cur][w][4 * lane]) =
          make_uint4(absmax_bits(am.x), absmax_bits(am.y), absmax_bits(am.z),
                     absmax_bits(am.w));
      if (tk.kind == kTaskWhole) {
        // single block: the block's column absmax is the unit's; its scales
        // and codes come from the same registers
        __syncthreads();
        uint4 mm = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int ww = 0; ww < kPWarps; ++ww) {
          const uint4 o = *reinterpret_cast<const uint4 *>(&sm.red[cur][ww][4 * lane]);
          mm.x = __vmaxu2(mm.x, o.x);
          mm.y = __vmaxu2(mm.y, o.y);
          mm.z = __vmaxu2(mm.z, o.z);
          mm.w = __vmaxu2(mm.w, o.w);
        }
        const uint32_t a[8] = {mm.x & 0xFFFFu, mm.x >> 16, mm.y & 0xFFFFu, mm.y >> 16,
                               mm.z & 0xFFFFu, mm.z >> 16, mm.w & 0xFFFFu, mm.w >> 16};
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] = scale_from_amax(bf16_bits_to_float(a[j]), p.smax);
        if (w == 0 && lane_ok)
          store_scales8(p.scales_col + static_cast<int64_t>(e) * p.cols + c0 + 8 * lane, s);
        tile_col_codes<FMT, FAST>(v, s, tile, w, lane, p.smax, p.sat_thr, sat);
        fence_proxy_async_smem();
      }
    } else {
      // ---------------------------------------------------------- cast
      int ok = 1;
      if (lane == 0) {  // every warp waits (bounded) for the unit's count
        const uint32_t *cnt = p.arrive + tk.u;
        const uint32_t target = static_cast<uint32_t>(tk.need) + p.uw.extra_arrivals;
        uint32_t c;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(cnt) : "memory");
        if (c < target) {
          const uint64_t t0 = global_timer_ns();
          while (true) {
            __nanosleep(64);
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(cnt) : "memory");
            if (c >= target) break;
            if (global_timer_ns() - t0 > p.uw.limit_ns) { ok = 0; break; }
          }
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (ok) {  // every lane acquires the count it relies on
        uint32_t c;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(p.arrive + tk.u)
                     : "memory");
        (void)c;
      } else {
        failed = true;
      }
      if (!failed) {
        uint4 a0 = make_uint4(0u, 0u, 0u, 0u), a1 = a0;
        if (lane_ok) {
          const uint4 *src = reinterpret_cast<const uint4 *>(p.amax + amax_base + 8 * lane);
          a0 = __ldcg(src);
          a1 = __ldcg(src + 1);
        }
        const uint32_t a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] = scale_from_amax(bf16_bits_to_float(a[j]), p.smax);
        if (tk.b == 0 && w == 0 && lane_ok)
          store_scales8(p.scales_col + static_cast<int64_t>(e) * p.cols + c0 + 8 * lane, s);
        float rs_lane = 0.0f;  // dual form: the scale of row rw0 + lane (lanes 0..15)
        if constexpr (DUAL) {
          const int32_t row = rw0 + lane;
          if (lane < kWR && row < r1) {
            rs_lane = scale_from_amax(bf16_bits_to_float(__ldcg(p.rowmax + row)), p.smax);
            if (tk.q == 0) p.scales_row[row] = rs_lane;
          }
        }
        load_rows<true>(v, p, rw0, r1, cvec, lane_ok);
        if constexpr (DUAL) {
          // rowwise codes in place: 8 columns of a row per lane, one 8-byte store
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
        tile_col_codes<FMT, FAST>(v, s, tile, w, lane, p.smax, p.sat_thr, sat);
        fence_proxy_async_smem();
      }
    }

    // warp 0: the next task; the tile written above may only be reused once
    // the store that read it two tasks ago has finished reading
    if (w == 0) {
      int32_t t = 0;
      if (lane == 0) {
        t = next;
        if (t < sm.total) next = static_cast<int32_t>(atomicAdd(p.work, 1u));
        bulk_wait_read<0>();
      }
      t = __shfl_sync(0xFFFFFFFFu, t, 0);
      const PTask nt = decode_panel_task<DUAL>(sm, t, np, p.delay, lane);
      if (lane == 0) sm.tk[cur ^ 1] = nt;
    }
    // a warp that gave up on its wait stops the block after this task
    if (__syncthreads_or(failed)) {
      if (tid == 0) status_or(p.status, FP8QGG_STATUS_TIMEOUT);
      break;
    }

    if (tk.kind == kTaskAbs) {
      // each warp merges 32 of the panel's columns into the unit's absmax and
      // counts itself: column 32w + lane is half (lane & 1) of word 16w + lane / 2
      const int wd = 16 * w + (lane >> 1);
      uint32_t m = 0;
#pragma unroll
      for (int ww = 0; ww < kPWarps; ++ww) m = __vmaxu2(m, sm.red[cur][ww][wd]);
      const int cc = 32 * w + lane;
      if (c0 + cc < p.cols) atomicMax(p.amax + amax_base + cc, (lane & 1) ? m >> 16 : m & 0xFFFFu);
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(p.arrive + tk.u, 1u);
    } else if (tid == 0) {
      tma_store_2d(&qmap, tile, sm.pstart[e] + tk.b * kRB, c0);
      bulk_commit();
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
  // blocks: kPBlocksPerSM per SM, never more than the tasks need (at least
  // one, for the scales of empty groups)
  const int64_t np = (cols + kPW - 1) / kPW;
  const int64_t blocks = (rows_total + int64_t(kRB) * num_groups) / kRB * np;
  const int grid = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(2 * blocks, int64_t(dev.sm_count) * kPBlocksPerSM)));
  // a cast waits for absmax tasks that the running blocks have taken by then
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
  // a row pointer selects the dual form even when no row exists
  uint8_t *qr = q_row ? q_row : reinterpret_cast<uint8_t *>(workspace);
  return panel_launch(x, rows_total, cols, ld_x, offsets, num_groups, q_col, ld_qc, scales_col,
                      qr, ld_qr, scales_row, fmt, scale_max, sat_count, dev_status, workspace,
                      current_unit_wait(), s);
}
