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
// 8l .. 8l + 7) and blocks of 128 rows of one group (16 rows per warp of an
// eight-warp thread block).  The blocks are listed unit by unit, largest
// group first, where a unit is one (group, panel) in the column-wise form and
// one group (all its panels) in the dual form.  The kernel is a software
// pipeline over that list: the thread block that takes step s from an
// atomic counter
//  - reads block s (HBM), reduces its column absmax (the warps meet in
//    shared memory) and merges it into the unit's absmax words in global
//    memory with relaxed atomic max, then counts it in the unit's arrival
//    counter with one release reduction by the first warp once every warp
//    has merged (the dual form also merges every row's absmax);
//  - reads block s - D again (from L2: D blocks ago is about one grid-width
//    plus the longest unit, so the block is still there and its unit's count
//    is normally full already; the block waits for it, bounded, otherwise),
//    derives the scales from the unit's absmax (once per thread block: each
//    warp 32 of the 256 columns, shared through shared memory), encodes two
//    rows of a column per conversion and writes each column's 16 tokens into
//    a 32 KB tile
//    (256 columns x 128 tokens, 128-byte swizzle) that one bulk tensor store
//    sends to the group's 128-token block of the padded layout: whole
//    128-byte lines, zero codes of the padding included (rows past the
//    group's end are zeros).  The dual form also encodes every row with its
//    own scale and stores it in place.
// A step has two block barriers (after the absmax, which also publishes the
// scales; before the tile's store), and warps 1 and 2 decode the blocks of a
// later step into shared memory while it runs.  Every block is read once from
// HBM.  A step only waits for steps handed out earlier (to running thread
// blocks), so no thread block waits for one that is not running.
#include <algorithm>
#include <cstring>

#include "device_common.cuh"
#include "host_common.h"
#include "quant_panels.h"
#include "quant_tile.cuh"

namespace fp8qgg {

// Build-time knob: the pipeline delay beyond the longest unit, in quarters
// of the grid (the default is the best of the values measured on B200).
#ifndef FP8QGG_PANEL_DELAY_Q
#define FP8QGG_PANEL_DELAY_Q 4
#endif

constexpr int kPW = 256;               // columns per panel
constexpr int kPWords = kPW / 2;       // bf16 pairs per panel row
constexpr int kRB = 128;               // rows per block = tokens per store tile
constexpr int kPWarps = 8;
constexpr int kPThreads = 32 * kPWarps;
constexpr int kWR = kRB / kPWarps;     // rows per warp: 16
constexpr int kPBlocksPerSM = 2;
constexpr int kPMaxGroups = 1024;
constexpr uint32_t kTileBytes = kPW * kRB;
static_assert(kWR == kTileRowsPerWarp && kRB == kTileTokens, "the shared transposed tile");

struct PanelSmem {
  uint8_t tile[kTileBytes];             // transposed code tile (1024-byte aligned)
  uint32_t red[kPWarps][kPWords];       // per-warp column absmax (bf16 magnitude pairs)
  int32_t end[kPMaxGroups];             // clamped group ends (by group index)
  int32_t pstart[kPMaxGroups];          // padded first token (by group index)
  int32_t order[kPMaxGroups];           // groups by size, largest first
  int32_t nb[kPMaxGroups];              // ordered group i: 128-row blocks
  int32_t apre[kPMaxGroups + 1];        // blocks of the groups before ordered group i
  alignas(16) float cscale[kPW];        // the cast's column scales (read as float4)
  int32_t n_nonempty, total, delay;
  int32_t nstep;                        // the step decoded during the current one
  int32_t sidx[3];                      // step index, by slot (step number mod 3)
  int32_t dA[3][6], dC[3][6];           // its decoded blocks (PBlock), by slot
};
static_assert(offsetof(PanelSmem, tile) == 0, "store tile 1024-byte aligned");
static_assert(kPWarps >= 3, "warps 1 and 2 decode the next step");
static_assert(offsetof(PanelSmem, cscale) % 16 == 0 && offsetof(PanelSmem, red) % 16 == 0,
              "16-byte shared-memory accesses");

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
  uint32_t *work;        // step counter
  uint32_t *arrive;      // per unit
  uint32_t *amax;        // [ordered group, cols] column absmax bits
  uint32_t *rowmax;      // dual form: [rows_total] row absmax bits
  UnitWait uw;
};

__device__ __forceinline__ int32_t warp_scan_incl(int32_t v, int lane) {
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t o = __shfl_up_sync(0xFFFFFFFFu, v, d);
    if (lane >= d) v += o;
  }
  return v;
}

// Clamped group ends, padded starts, the size order, the block list and the
// pipeline delay.
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
    int32_t carry = 0, n_ne = 0, nb_max = 0;
    for (int base = 0; base < G; base += 32) {
      const int i = base + lane;
      int32_t nbv = 0;
      if (i < G) {
        const int e = sm.order[i];
        nbv = (sm.end[e] - (e ? sm.end[e - 1] : 0) + kRB - 1) / kRB;
        sm.nb[i] = nbv;
      }
      const int32_t incl = warp_scan_incl(nbv, lane);
      if (i < G) sm.apre[i] = carry + incl - nbv;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
      n_ne += __popc(__ballot_sync(0xFFFFFFFFu, nbv >= 1));
      nb_max = max(nb_max, nbv);
    }
    for (int d = 16; d > 0; d >>= 1) nb_max = max(nb_max, __shfl_xor_sync(0xFFFFFFFFu, nb_max, d));
    if (lane == 0) {
      sm.apre[G] = carry;
      sm.n_nonempty = n_ne;
      sm.total = carry * np;
      // a unit's blocks are consecutive: the delay covers the longest unit and
      // the steps the running blocks hold (one grid width at the default)
      const int32_t span = DUAL ? nb_max * np : nb_max;
      sm.delay = min(sm.total, span + (FP8QGG_PANEL_DELAY_Q * static_cast<int32_t>(gridDim.x)) / 4);
    }
  }
  __syncthreads();
}

struct PBlock {
  int32_t i, e;   // ordered group, group index
  int32_t q, b;   // panel, block of the group
  int32_t u;      // unit (arrival counter)
  int32_t need;   // arrivals that complete the unit
};
static_assert(sizeof(PBlock) == sizeof(PanelSmem::dA[0]), "decoded blocks are kept as six words");

// Block a of the list (the whole warp calls it; every lane gets the same
// answer): the ordered group by a 32-way search over the block prefix.
template <bool DUAL>
__device__ PBlock decode_block(const PanelSmem &sm, int32_t a, int np, int lane) {
  int lo = 0, hi = sm.n_nonempty;  // apre[lo] * np <= a
  while (hi - lo > 1) {
    const int step = (hi - lo + 31) / 32;
    const int c = lo + lane * step;
    const bool ok = c < hi && sm.apre[c] * np <= a;
    const int n = __popc(__ballot_sync(0xFFFFFFFFu, ok));  // lanes 0 .. n-1
    const int nlo = lo + (n - 1) * step;
    hi = min(hi, nlo + step);
    lo = nlo;
  }
  PBlock r;
  const int32_t nbi = sm.nb[lo];
  const int32_t rr = a - sm.apre[lo] * np;
  r.i = lo;
  r.e = sm.order[lo];
  r.q = rr / nbi;
  r.b = rr - r.q * nbi;
  r.u = DUAL ? lo : lo * np + r.q;
  r.need = kPWarps * (DUAL ? nbi * np : nbi);  // each block of the unit adds kPWarps
  return r;
}

// The blocks of step sm.nstep, decoded ahead into slot par: warp 1 takes the
// absmax block (and the index), warp 2 the cast block.
template <bool DUAL>
__device__ __forceinline__ void decode_ahead(PanelSmem &sm, int par, int np, int w, int lane,
                                             int32_t total, int32_t delay, int32_t steps) {
  const int32_t ns = sm.nstep;
  if (w == 1) {
    if (ns < total) {
      const PBlock b = decode_block<DUAL>(sm, ns, np, lane);
      if (lane == 0) memcpy(sm.dA[par], &b, sizeof b);
    }
    if (lane == 0) sm.sidx[par] = ns;
  } else if (w == 2) {
    if (ns >= delay && ns < steps) {
      const PBlock b = decode_block<DUAL>(sm, ns - delay, np, lane);
      if (lane == 0) memcpy(sm.dC[par], &b, sizeof b);
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

  const int32_t total = sm.total, delay = sm.delay;
  const int32_t steps = total + delay;
  uint32_t sat = 0;
  if constexpr (!DUAL) {
    // The column-wise form loads each block where the step needs it (early
    // loads, as in the dual form below, measured 2% slower here); the next
    // step's blocks are decoded one step ahead (two slots).
    int32_t next = 0;  // thread 0: the step after the one being decoded
    if (tid == 0) sm.nstep = static_cast<int32_t>(atomicAdd(p.work, 1u));
    __syncthreads();
    decode_ahead<false>(sm, 0, np, w, lane, total, delay, steps);
    if (tid == 0 && sm.nstep < steps) next = static_cast<int32_t>(atomicAdd(p.work, 1u));
    __syncthreads();
    for (int par = 0;; par ^= 1) {
      // a step is bracketed by two block barriers: the one after the absmax
      // (which also publishes the cast's column scales and the next step's
      // index) and the one before the tile's store
      const int32_t st = sm.sidx[par];
      if (st >= steps) break;
      if (tid == 0) {
        sm.nstep = next;
        if (next < steps) next = static_cast<int32_t>(atomicAdd(p.work, 1u));
      }
      const bool has_a = st < total;
      const bool has_c = st >= delay;
      PBlock A{}, C{};
      if (has_a) memcpy(&A, sm.dA[par], sizeof A);
      if (has_c) memcpy(&C, sm.dC[par], sizeof C);

      // the cast's scale words, early when the unit is complete already: each
      // warp derives the scales of 32 of the panel's columns
      bool c_ready = false;
      uint32_t uword = 0;
      const int cc0 = C.q * kPW;
      const bool c_lane = has_c && cc0 + 8 * lane < p.cols;
      const int ccol = cc0 + 32 * w + lane;  // this lane's scale column
      if (has_c) {
        uint32_t cnt = 0;
        if (lane == 0)
          asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(cnt) : "l"(p.arrive + C.u)
                       : "memory");
        c_ready = __shfl_sync(0xFFFFFFFFu, cnt, 0) >= static_cast<uint32_t>(C.need) +
                                                       p.uw.extra_arrivals;
      }
      if (c_ready)
        uword = ccol < p.cols ? __ldcg(p.amax + static_cast<int64_t>(C.i) * p.cols + ccol) : 0u;

      // ---------------------------------------------------------- absmax of block s
      if (has_a) {
        const int32_t gs = A.e ? sm.end[A.e - 1] : 0;
        const int32_t r0 = gs + A.b * kRB;
        const int32_t r1 = min(sm.end[A.e], r0 + kRB);
        const int32_t rw0 = r0 + kWR * w;
        const int c0 = A.q * kPW;
        const bool lane_ok = c0 + 8 * lane < p.cols;
        const uint4 *src = p.x + static_cast<int64_t>(rw0) * p.ld_x16 + (c0 >> 3) + lane;
        uint4 v[kWR];
#pragma unroll
        for (int k = 0; k < kWR; ++k)
          v[k] = (lane_ok && rw0 + k < r1) ? __ldcg(src + k * p.ld_x16) : make_uint4(0u, 0u, 0u, 0u);
        uint4 am = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int k = 0; k < kWR; ++k) {
          am.x = absmax_acc(am.x, v[k].x);
          am.y = absmax_acc(am.y, v[k].y);
          am.z = absmax_acc(am.z, v[k].z);
          am.w = absmax_acc(am.w, v[k].w);
        }
        *reinterpret_cast<uint4 *>(&sm.red[w][4 * lane]) =
            make_uint4(absmax_bits(am.x), absmax_bits(am.y), absmax_bits(am.z),
                       absmax_bits(am.w));
      }
      if (c_ready) {
        const float sc = scale_from_amax(bf16_bits_to_float(uword), p.smax);
        sm.cscale[32 * w + lane] = sc;
        if (C.b == 0 && ccol < p.cols) p.scales_col[static_cast<int64_t>(C.e) * p.cols + ccol] = sc;
      }
      if (tid == 0) bulk_wait_read<0>();  // the previous store has read the tile
      const bool all_ready = __syncthreads_and(!has_c || c_ready) != 0;
      if (has_a) {
        // each warp merges 32 of the panel's columns into the unit's absmax:
        // column 32w + lane is half (lane & 1) of word 16w + lane / 2
        const int wd = 16 * w + (lane >> 1);
        uint32_t m = 0;
#pragma unroll
        for (int ww = 0; ww < kPWarps; ++ww) m = __vmaxu2(m, sm.red[ww][wd]);
        const int c0 = A.q * kPW;
        const int cc = 32 * w + lane;
        if (c0 + cc < p.cols)
          atomicMax(p.amax + static_cast<int64_t>(A.i) * p.cols + c0 + cc,
                    (lane & 1) ? m >> 16 : m & 0xFFFFu);
        // every warp's merges happen before warp 0's one release of the count
        // (a named barrier: the other warps arrive without waiting and go on to
        // the cast; the release orders their merges too, being cumulative over
        // the barrier)
        __syncwarp();
        if (w != 0) {
          asm volatile("bar.arrive 2, %0;" ::"n"(kPThreads) : "memory");
        } else {
          asm volatile("bar.sync 2, %0;" ::"n"(kPThreads) : "memory");
          if (lane == 0)
            asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p.arrive + A.u),
                         "n"(kPWarps)
                         : "memory");
        }
      }
      decode_ahead<false>(sm, par ^ 1, np, w, lane, total, delay, steps);

      // ---------------------------------------------------------- cast of block s - D
      bool failed = false;
      float s[8];
      if (has_c && all_ready) {
        const float4 s0 = *reinterpret_cast<const float4 *>(&sm.cscale[8 * lane]);
        const float4 s1 = *reinterpret_cast<const float4 *>(&sm.cscale[8 * lane + 4]);
        s[0] = s0.x; s[1] = s0.y; s[2] = s0.z; s[3] = s0.w;
        s[4] = s1.x; s[5] = s1.y; s[6] = s1.z; s[7] = s1.w;
      } else if (has_c) {  // wait (bounded) until every block of the unit is counted
        int ok = 1;
        if (lane == 0) {
          const uint32_t target = static_cast<uint32_t>(C.need) + p.uw.extra_arrivals;
          const uint64_t t0 = global_timer_ns();
          while (true) {
            uint32_t c;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(p.arrive + C.u)
                         : "memory");
            if (c >= target) break;
            if (global_timer_ns() - t0 > p.uw.limit_ns) { ok = 0; break; }
            __nanosleep(64);
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (ok) {
          uint32_t c;  // every lane acquires the count it relies on
          asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(p.arrive + C.u)
                       : "memory");
          (void)c;
          uint4 ua0 = make_uint4(0u, 0u, 0u, 0u), ua1 = ua0;
          if (c_lane) {
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.amax + static_cast<int64_t>(C.i) * p.cols + cc0 + 8 * lane);
            ua0 = __ldcg(src);
            ua1 = __ldcg(src + 1);
          }
          const uint32_t a[8] = {ua0.x, ua0.y, ua0.z, ua0.w, ua1.x, ua1.y, ua1.z, ua1.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) s[j] = scale_from_amax(bf16_bits_to_float(a[j]), p.smax);
          if (C.b == 0 && w == 0 && c_lane)
            store_scales8(p.scales_col + static_cast<int64_t>(C.e) * p.cols + cc0 + 8 * lane, s);
        } else {
          failed = true;
        }
      }
      uint4 v[kWR];
      int32_t c_r1 = 0, c_rw0 = 0;
      if (has_c && !failed) {
        const int32_t gs = C.e ? sm.end[C.e - 1] : 0;
        const int32_t r0 = gs + C.b * kRB;
        c_r1 = min(sm.end[C.e], r0 + kRB);
        c_rw0 = r0 + kWR * w;
        const uint4 *src = p.x + static_cast<int64_t>(c_rw0) * p.ld_x16 + (cc0 >> 3) + lane;
#pragma unroll
        for (int k = 0; k < kWR; ++k)
          v[k] = (c_lane && c_rw0 + k < c_r1) ? __ldcs(src + k * p.ld_x16)
                                              : make_uint4(0u, 0u, 0u, 0u);
      }
      if (has_c && !failed) {
        tile_col_codes<FMT, FAST>(v, s, sm.tile, w, lane, p.smax, p.sat_thr, sat);
        fence_proxy_async_smem();
      }
      if (__syncthreads_or(failed)) {
        if (tid == 0) status_or(p.status, FP8QGG_STATUS_TIMEOUT);
        break;  // this block takes no more steps
      }
      if (has_c && tid == 0) {
        const int32_t ps = sm.pstart[C.e] + C.b * kRB;
        tma_store_2d(&qmap, sm.tile, ps, cc0);
        bulk_commit();
      }
    }
  } else {
    // The dual form loads each block early: the absmax block's rows at the end
    // of the previous step (under the end-of-step barrier and the store), the
    // cast block's as soon as the absmax has read them (under the mid-step
    // barrier); its longer step gains from the overlap (185 -> 177 us on the
    // DeepSeek-MoE-16B grad_out).  Early loads need the next step's blocks a
    // step in advance: they are decoded two steps ahead (three slots).
    constexpr int kSlots = 3;
    // thread 0 claims this block's steps from the counter, in increasing order;
    // each is published in sm.nstep and decoded two steps before it runs
    int32_t next = 0;
    auto claim = [&]() {
      sm.nstep = next;
      if (next < steps) next = static_cast<int32_t>(atomicAdd(p.work, 1u));
    };
    if (tid == 0) {
      next = static_cast<int32_t>(atomicAdd(p.work, 1u));
      claim();
    }
    __syncthreads();
    decode_ahead<DUAL>(sm, 0, np, w, lane, total, delay, steps);
    __syncthreads();
    if (tid == 0) claim();
    __syncthreads();
    decode_ahead<DUAL>(sm, 1, np, w, lane, total, delay, steps);
    __syncthreads();

    // The block's rows, 16 per warp (v lives across steps).
    uint4 v[kWR];
    // (every call defines all of v, zeros when there is no block, so that no
    // earlier contents stay live)
    auto load_rows = [&](uint4 (&dst)[kWR], const PBlock &B, bool has, bool streaming) {
      const int32_t gs = B.e ? sm.end[B.e - 1] : 0;
      const int32_t r0 = gs + B.b * kRB;
      const int32_t r1 = has ? min(sm.end[B.e], r0 + kRB) : 0;
      const int32_t rw0 = r0 + kWR * w;
      const int c0 = B.q * kPW;
      const bool lane_ok = c0 + 8 * lane < p.cols;
      const uint4 *src = p.x + static_cast<int64_t>(rw0) * p.ld_x16 + (c0 >> 3) + lane;
#pragma unroll
      for (int k = 0; k < kWR; ++k) {
        const bool ok = lane_ok && rw0 + k < r1;
        dst[k] = !ok ? make_uint4(0u, 0u, 0u, 0u)
                     : streaming ? __ldcs(src + k * p.ld_x16) : __ldcg(src + k * p.ld_x16);
      }
    };
    auto load_a = [&](int slot) {  // the absmax block of the step in this slot
      PBlock B{};
      const bool has = sm.sidx[slot] < total;
      if (has) memcpy(&B, sm.dA[slot], sizeof B);
      load_rows(v, B, has, false);
    };
    load_a(0);
    for (int slot = 0;; slot = slot == kSlots - 1 ? 0 : slot + 1) {
      // a step is bracketed by two block barriers: the one after the absmax
      // (which also publishes the cast's column scales and the index of the
      // step decoded next) and the one before the tile's store
      const int slot1 = slot == kSlots - 1 ? 0 : slot + 1;
      const int slot_dec = slot1 == 2 ? 0 : slot1 + 1;
      const int32_t st = sm.sidx[slot];
      if (st >= steps) break;
      if (tid == 0) claim();
      const bool has_a = st < total;
      const bool has_c = st >= delay;
      PBlock A{}, C{};
      if (has_a) memcpy(&A, sm.dA[slot], sizeof A);
      if (has_c) memcpy(&C, sm.dC[slot], sizeof C);

      // the cast's scale words, early when the unit is complete already: each
      // warp derives the scales of 32 of the panel's columns
      bool c_ready = false;
      uint32_t uword = 0, urow = 0;
      const int cc0 = C.q * kPW;
      const bool c_lane = has_c && cc0 + 8 * lane < p.cols;
      const int ccol = cc0 + 32 * w + lane;  // this lane's scale column
      if (has_c) {
        uint32_t cnt = 0;
        if (lane == 0)
          asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(cnt) : "l"(p.arrive + C.u)
                       : "memory");
        c_ready = __shfl_sync(0xFFFFFFFFu, cnt, 0) >= static_cast<uint32_t>(C.need) +
                                                       p.uw.extra_arrivals;
      }
      auto load_row_word = [&]() {  // the row absmax word of row rw0 + lane (lanes 0..15)
        const int32_t cgs = C.e ? sm.end[C.e - 1] : 0;
        const int32_t row = cgs + C.b * kRB + kWR * w + lane;
        const int32_t r1 = min(sm.end[C.e], cgs + C.b * kRB + kRB);
        urow = (lane < kWR && row < r1) ? __ldcg(p.rowmax + row) : 0u;
      };
      if (c_ready) {
        uword = ccol < p.cols ? __ldcg(p.amax + static_cast<int64_t>(C.i) * p.cols + ccol) : 0u;
        load_row_word();
      }

      // ---------------------------------------------------------- absmax of block s
      if (has_a) {
        const int32_t gs = A.e ? sm.end[A.e - 1] : 0;
        const int32_t r0 = gs + A.b * kRB;
        const int32_t r1 = min(sm.end[A.e], r0 + kRB);
        const int32_t rw0 = r0 + kWR * w;
        uint4 am = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int k = 0; k < kWR; ++k) {
          am.x = absmax_acc(am.x, v[k].x);
          am.y = absmax_acc(am.y, v[k].y);
          am.z = absmax_acc(am.z, v[k].z);
          am.w = absmax_acc(am.w, v[k].w);
        }
        merge_row_amax(v, p.rowmax, rw0, r1, lane);
        *reinterpret_cast<uint4 *>(&sm.red[w][4 * lane]) =
            make_uint4(absmax_bits(am.x), absmax_bits(am.y), absmax_bits(am.z),
                       absmax_bits(am.w));
      }
      // the cast block's rows (read-only input: no need to wait for its unit)
      load_rows(v, C, has_c, true);
      if (c_ready) {
        const float sc = scale_from_amax(bf16_bits_to_float(uword), p.smax);
        sm.cscale[32 * w + lane] = sc;
        if (C.b == 0 && ccol < p.cols) p.scales_col[static_cast<int64_t>(C.e) * p.cols + ccol] = sc;
      }
      if (tid == 0) bulk_wait_read<0>();  // the previous store has read the tile
      const bool all_ready = __syncthreads_and(!has_c || c_ready) != 0;
      if (has_a) {
        // each warp merges 32 of the panel's columns into the unit's absmax:
        // column 32w + lane is half (lane & 1) of word 16w + lane / 2
        const int wd = 16 * w + (lane >> 1);
        uint32_t m = 0;
#pragma unroll
        for (int ww = 0; ww < kPWarps; ++ww) m = __vmaxu2(m, sm.red[ww][wd]);
        const int c0 = A.q * kPW;
        const int cc = 32 * w + lane;
        if (c0 + cc < p.cols)
          atomicMax(p.amax + static_cast<int64_t>(A.i) * p.cols + c0 + cc,
                    (lane & 1) ? m >> 16 : m & 0xFFFFu);
        // every warp's merges happen before warp 0's one release of the count
        // (a named barrier: the other warps arrive without waiting and go on to
        // the cast; the release orders their merges too, being cumulative over
        // the barrier)
        __syncwarp();
        if (w != 0) {
          asm volatile("bar.arrive 2, %0;" ::"n"(kPThreads) : "memory");
        } else {
          asm volatile("bar.sync 2, %0;" ::"n"(kPThreads) : "memory");
          if (lane == 0)
            asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p.arrive + A.u),
                         "n"(kPWarps)
                         : "memory");
        }
      }
      decode_ahead<DUAL>(sm, slot_dec, np, w, lane, total, delay, steps);

      // ---------------------------------------------------------- cast of block s - D
      bool failed = false;
      float s[8];
      if (has_c && all_ready) {
        const float4 s0 = *reinterpret_cast<const float4 *>(&sm.cscale[8 * lane]);
        const float4 s1 = *reinterpret_cast<const float4 *>(&sm.cscale[8 * lane + 4]);
        s[0] = s0.x; s[1] = s0.y; s[2] = s0.z; s[3] = s0.w;
        s[4] = s1.x; s[5] = s1.y; s[6] = s1.z; s[7] = s1.w;
      } else if (has_c) {  // wait (bounded) until every block of the unit is counted
        int ok = 1;
        if (lane == 0) {
          const uint32_t target = static_cast<uint32_t>(C.need) + p.uw.extra_arrivals;
          const uint64_t t0 = global_timer_ns();
          while (true) {
            uint32_t c;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(p.arrive + C.u)
                         : "memory");
            if (c >= target) break;
            if (global_timer_ns() - t0 > p.uw.limit_ns) { ok = 0; break; }
            __nanosleep(64);
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (ok) {
          uint32_t c;  // every lane acquires the count it relies on
          asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(p.arrive + C.u)
                       : "memory");
          (void)c;
          uint4 ua0 = make_uint4(0u, 0u, 0u, 0u), ua1 = ua0;
          if (c_lane) {
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.amax + static_cast<int64_t>(C.i) * p.cols + cc0 + 8 * lane);
            ua0 = __ldcg(src);
            ua1 = __ldcg(src + 1);
          }
          load_row_word();
          const uint32_t a[8] = {ua0.x, ua0.y, ua0.z, ua0.w, ua1.x, ua1.y, ua1.z, ua1.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) s[j] = scale_from_amax(bf16_bits_to_float(a[j]), p.smax);
          if (C.b == 0 && w == 0 && c_lane)
            store_scales8(p.scales_col + static_cast<int64_t>(C.e) * p.cols + cc0 + 8 * lane, s);
        } else {
          failed = true;
        }
      }
      if (has_c && !failed) {
        const int32_t cgs = C.e ? sm.end[C.e - 1] : 0;
        const int32_t r1 = min(sm.end[C.e], cgs + C.b * kRB + kRB);
        const int32_t rw0 = cgs + C.b * kRB + kWR * w;
        float rs_lane = 0.0f;  // the scale of row rw0 + lane (lanes 0..15)
        if (lane < kWR && rw0 + lane < r1) {
          rs_lane = scale_from_amax(bf16_bits_to_float(urow), p.smax);
          if (C.q == 0) p.scales_row[rw0 + lane] = rs_lane;
        }
        // rowwise codes in place: 8 columns of a row per lane, one 8-byte store
#pragma unroll
        for (int k = 0; k < kWR; ++k) {
          const float rs = __shfl_sync(0xFFFFFFFFu, rs_lane, k);
          uint32_t c2[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t wd = word(v[k], j);
            c2[j] = enc_pair<FMT, FAST>(lo_f(wd), hi_f(wd), rs, rs, p.smax, p.sat_thr, sat);
          }
          if (c_lane && rw0 + k < r1)
            *reinterpret_cast<uint2 *>(p.q_row + static_cast<int64_t>(rw0 + k) * p.ld_qr +
                                       cc0 + 8 * lane) =
                make_uint2(c2[0] | (c2[1] << 16), c2[2] | (c2[3] << 16));
        }
        tile_col_codes<FMT, FAST>(v, s, sm.tile, w, lane, p.smax, p.sat_thr, sat);
        fence_proxy_async_smem();
      }
      if (!failed) load_a(slot1);  // the next step's absmax block
      if (__syncthreads_or(failed)) {
        if (tid == 0) status_or(p.status, FP8QGG_STATUS_TIMEOUT);
        break;  // this block takes no more steps
      }
      if (has_c && tid == 0) {
        const int32_t ps = sm.pstart[C.e] + C.b * kRB;
        tma_store_2d(&qmap, sm.tile, ps, cc0);
        bulk_commit();
      }
    }
  }
  if (tid == 0) bulk_wait_all();  // the tile stays valid until its stores have read it
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
  // thread blocks: kPBlocksPerSM per SM, never more than the steps need (at
  // least one, for the scales of empty groups)
  const int64_t np = (cols + kPW - 1) / kPW;
  const int64_t blocks = (rows_total + int64_t(kRB) * num_groups) / kRB * np;
  const int grid = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(blocks, int64_t(dev.sm_count) * kPBlocksPerSM)));
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
