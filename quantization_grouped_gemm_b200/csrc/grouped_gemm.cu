// FP8 scaled grouped GEMM on the B200 5th-generation tensor cores.
//
// The pages run the MoE expert GEMMs as one grouped GEMM over FP8 operands
// whose groups come from the token offsets ("AMD Boosts PyTorch FP8 Training
// on Instinct GPUs", third paragraph; "AMD Primus adds FP8/MXFP8 kernels ...",
// "What Primus adds for MoE training on MI355X": FP8 grouped GEMM and
// sync-free MoE execution).  This kernel reads the offsets on the device and
// never synchronises with the host.
//
// Structure (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer: A and B tiles, 128 bytes of K per row, 128-byte
//               swizzle, into a 4-stage shared-memory ring (mbarrier full /
//               empty pairs).
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators)
//               and issues tcgen05.mma kind::f8f6f4 (M128 N256 K32) from one
//               lane; tcgen05.commit frees ring stages and publishes finished
//               accumulators.  In the contraction-jagged mode it also zeroes,
//               in shared memory, the token columns of a tile that fall
//               outside the group (group edges need not be 16-aligned, TMA
//               coordinates must be).
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes, multiply by
//               1/scale_a (row) and 1/scale_b (column), masked stores.  With
//               two accumulators the epilogue of tile i overlaps the
//               mainloop of tile i+1.
// Tiles are enumerated group by group; in the token-jagged mode the N tiles
// of one M tile are consecutive so that concurrent CTAs share the A rows in
// L2 and the whole B_e stays L2-resident across the group.
#include <algorithm>

#include "device_common.cuh"
#include "gemm_store.cuh"
#include "host_common.h"

namespace fp8qgg {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // bytes of K per stage row = one 128-byte swizzle atom
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;  // two per TMEM lane quarter: one per 128-column half
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kGemmThreads = 64 + kEpiThreads;
// the one-CTA kernel adds a warp that masks the edge blocks of the
// contraction-jagged mode, off the MMA warp's path
constexpr int kMaskWarp = kGemmThreads / 32;
constexpr int kGemm1Threads = kGemmThreads + 32;
constexpr int kMaxGemmGroups = 1024;
constexpr int kBandRows = 4096;  // rows per raster band of tiles (token-jagged mode)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kStageBytes = (BM + BN) * BK;
constexpr uint32_t kIdesc = idesc_e4m3_f32(BM, BN);

struct GemmSmem {
  uint8_t a[kStages][BM * BK];  // 16 KB each, 1024-aligned (swizzle atoms)
  uint8_t b[kStages][BN * BK];  // 32 KB each
  float stg[kEpiWarps][512];  // per epilogue warp: one 32-row x 64-byte output unit
  float inv_sb[2][BN];
  int32_t end[kMaxGemmGroups];
  int32_t tile_prefix[kMaxGemmGroups + 1];
  int32_t order[kMaxGemmGroups];  // contraction-jagged mode: groups, largest first
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t ready[kStages];  // contraction-jagged mode: edge block masked
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct GemmParams {
  const float *scale_a;
  int64_t sas;  // scale_a group stride (contraction-jagged mode)
  const float *scale_b;
  int64_t sbs;  // scale_b group stride
  const int32_t *offsets;
  int num_groups;
  int64_t m_total, n, k;
  void *out;
  int64_t ld_out;
  int64_t out_gs;  // output group stride (contraction-jagged mode)
  int32_t *status;
  int padded;      // contraction-jagged operands with groups at 128-token boundaries
};

struct TileInfo {
  int e;       // group
  int tm, tn;  // tile coordinates inside the group
  int32_t gstart, gend;
  int nk;  // k blocks
};

template <int MODE, int ROWS = BM, class Smem = GemmSmem>
__device__ __forceinline__ TileInfo decode_tile(const Smem &sm, const GemmParams &p, int32_t t) {
  int lo = 0, hi = p.num_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sm.tile_prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  TileInfo ti;
  ti.e = lo;
  ti.gstart = lo ? sm.end[lo - 1] : 0;
  ti.gend = sm.end[lo];
  const int32_t local = t - sm.tile_prefix[lo];
  if constexpr (MODE == FP8QGG_M_JAGGED) {
    // Bands of kBand M tiles: consecutive tiles walk down a band before moving
    // to the next N tile, so the tiles in flight at once share a few A rows
    // and a few B rows in L2.
    constexpr int kB = kBandRows / ROWS;
    const int nt = static_cast<int>((p.n + BN - 1) / BN);
    const int mt = (ti.gend - ti.gstart + ROWS - 1) / ROWS;
    const int band = local / (kB * nt);
    const int rem = local - band * kB * nt;
    const int bm = min(kB, mt - band * kB);
    ti.tm = band * kB + rem % bm;
    ti.tn = rem / bm;
    ti.nk = static_cast<int>((p.k + BK - 1) / BK);
  } else {
    const int nt = static_cast<int>((p.k + BN - 1) / BN);
    ti.tm = local / nt;
    ti.tn = local % nt;
    ti.nk = ti.gend > ti.gstart ? (ti.gend - (ti.gstart & ~(BK - 1)) + BK - 1) / BK : 0;
  }
  return ti;
}

// Contraction-jagged mode: every group has the same number of tiles, but a
// tile's cost grows with the group's token count.  Position `pos` of the list
// sorted by group size (largest first) maps to group order[pos / tpg].
__device__ __forceinline__ TileInfo decode_tile_sorted(const GemmSmem &sm, const GemmParams &p,
                                                       int32_t pos) {
  const int32_t tpg = sm.tile_prefix[1] - sm.tile_prefix[0];
  const int e = sm.order[pos / tpg];
  const int32_t local = pos - (pos / tpg) * tpg;
  TileInfo ti;
  ti.e = e;
  ti.gstart = e ? sm.end[e - 1] : 0;
  ti.gend = sm.end[e];
  const int nt = static_cast<int>((p.k + BN - 1) / BN);
  ti.tm = local / nt;
  ti.tn = local % nt;
  ti.nk = ti.gend > ti.gstart ? (ti.gend - (ti.gstart & ~(BK - 1)) + BK - 1) / BK : 0;
  return ti;
}

// The i-th tile of this CTA.  Token-jagged mode: plain grid stride (tiles
// cost the same).  Contraction-jagged mode: rounds of gridDim.x tiles taken in
// alternating directions over the size-sorted list, so that every CTA gets a
// similar mix of long and short tiles.  Returns a position >= total when the
// CTA has no i-th tile.
template <int MODE>
__device__ __forceinline__ int32_t tile_position(int32_t i) {
  const int32_t G = static_cast<int32_t>(gridDim.x);
  const int32_t b = static_cast<int32_t>(blockIdx.x);
  if constexpr (MODE == FP8QGG_M_JAGGED) return b + i * G;
  return i * G + ((i & 1) ? (G - 1 - b) : b);
}

template <int MODE>
__device__ __forceinline__ TileInfo tile_at(const GemmSmem &sm, const GemmParams &p,
                                            int32_t pos) {
  if constexpr (MODE == FP8QGG_M_JAGGED)
    return decode_tile<MODE>(sm, p, pos);
  else
    return decode_tile_sorted(sm, p, pos);
}

// Clamped group ends and cumulative tile counts, warp-parallel (one warp).
template <int MODE, int ROWS = BM, class Smem = GemmSmem>
__device__ void build_tile_table(Smem &sm, const GemmParams &p, int lane) {
  const int32_t R = static_cast<int32_t>(p.m_total);
  const int32_t nt_m = static_cast<int32_t>((p.n + BN - 1) / BN);
  const int32_t tiles_k_mode =
      static_cast<int32_t>(((p.n + BM - 1) / BM) * ((p.k + BN - 1) / BN));
  int32_t carry_end = 0, carry_tiles = 0, carry_pend = 0;
  bool bad = false;
  for (int base = 0; base < p.num_groups; base += 32) {
    const int e = base + lane;
    const int32_t raw = e < p.num_groups ? __ldg(p.offsets + e) : INT32_MIN;
    int32_t run = max(raw, 0);
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t o = __shfl_up_sync(0xFFFFFFFFu, run, d);
      if (lane >= d) run = max(run, o);
    }
    const int32_t endv = min(R, max(carry_end, run));
    int32_t prev = __shfl_up_sync(0xFFFFFFFFu, endv, 1);
    if (lane == 0) prev = carry_end;
    if (e < p.num_groups && (raw < prev || raw > R)) bad = true;
    int32_t tiles = 0;
    if (e < p.num_groups) {
      if constexpr (MODE == FP8QGG_M_JAGGED)
        tiles = ((endv - prev + ROWS - 1) / ROWS) * nt_m;
      else
        tiles = tiles_k_mode;
    }
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t o = __shfl_up_sync(0xFFFFFFFFu, tiles, d);
      if (lane >= d) tiles += o;
    }
    // padded contraction-jagged operands: group e's tokens sit at
    // [P_e, P_e + round_up(size_e, BK)), P_e the earlier groups' padded sizes
    int32_t pend = endv;
    if constexpr (MODE == FP8QGG_K_JAGGED) {
      if (p.padded) {
        int32_t psz = e < p.num_groups ? (endv - prev + BK - 1) & ~(BK - 1) : 0;
        for (int d = 1; d < 32; d <<= 1) {
          const int32_t o = __shfl_up_sync(0xFFFFFFFFu, psz, d);
          if (lane >= d) psz += o;
        }
        pend = carry_pend + psz;
        carry_pend += __shfl_sync(0xFFFFFFFFu, psz, 31);
      }
    }
    if (e < p.num_groups) {
      sm.end[e] = pend;
      sm.tile_prefix[e + 1] = carry_tiles + tiles;
    }
    carry_end = __shfl_sync(0xFFFFFFFFu, endv, 31);
    carry_tiles += __shfl_sync(0xFFFFFFFFu, tiles, 31);
  }
  if (lane == 0) sm.tile_prefix[0] = 0;
  bad = __any_sync(0xFFFFFFFFu, bad);
  if (bad && lane == 0 && blockIdx.x == 0) status_or(p.status, FP8QGG_STATUS_BAD_OFFSETS);
}

// Byte mask keeping the bytes [lo, hi) of a 16-byte piece (lo, hi in 0..16).
__device__ __forceinline__ uint4 keep_mask16(int lo, int hi) {
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t m = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int k = 4 * q + b;
      if (k >= lo && k < hi) m |= 0xFFu << (8 * b);
    }
    w[q] = m;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Zero the K columns outside [lo, hi) of a K-major tile written by TMA with
// 128-byte swizzle (logical 16-byte piece j of row r sits at piece j ^ (r & 7)),
// within the 32-column MMA steps that will be issued: those that hold a column
// of [lo, hi), i.e. steps lo / 32 .. ceil(hi / 32) - 1.  So at most four
// pieces per row are touched (two around lo, two around hi).  The piece masks
// are built once per call.
template <int ROWS>
__device__ __forceinline__ void mask_k_edges(uint8_t *tile, int lo, int hi, int lane) {
  // the two pieces of the step holding lo and the two of the step holding
  // hi - 1 (the same two when lo and hi share a step: applying a piece's mask
  // twice changes nothing)
  const int s0 = lo >> 5, s1 = (hi - 1) >> 5;
  int pj[4];
  uint4 pm[4];
  bool act[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    pj[i] = 2 * (i < 2 ? s0 : s1) + (i & 1);
    const int a = max(lo - 16 * pj[i], 0), b = min(hi - 16 * pj[i], 16);
    act[i] = !(a == 0 && b == 16);
    pm[i] = b > a ? keep_mask16(a, b) : make_uint4(0u, 0u, 0u, 0u);
  }
  // all reads first, then all writes: the lane's ROWS / 32 rows are
  // independent, so their shared-memory latencies overlap
  const int sw = lane & 7;  // rows lane, lane + 32, ... share the swizzle phase
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (act[i]) {
      uint4 v[ROWS / 32];
      uint4 *ptr[ROWS / 32];
#pragma unroll
      for (int rr = 0; rr < ROWS / 32; ++rr) {
        ptr[rr] = reinterpret_cast<uint4 *>(tile + (lane + 32 * rr) * BK + ((pj[i] ^ sw) << 4));
        v[rr] = *ptr[rr];
      }
#pragma unroll
      for (int rr = 0; rr < ROWS / 32; ++rr) {
        v[rr].x &= pm[i].x; v[rr].y &= pm[i].y; v[rr].z &= pm[i].z; v[rr].w &= pm[i].w;
        *ptr[rr] = v[rr];
      }
    }
  }
}

// The group's columns [lo, hi) of k-block kb of a contraction-jagged tile
// (blocks start on 128-token boundaries) and whether the block needs masking.
struct KEdge {
  int lo, hi;
  bool masked;
};

__device__ __forceinline__ KEdge k_edge(const TileInfo &ti, int kb) {
  const int32_t kx = (ti.gstart & ~(BK - 1)) + kb * BK;
  KEdge e;
  e.lo = max(0, ti.gstart - kx);
  e.hi = min(BK, ti.gend - kx);
  e.masked = (e.lo & 31) != 0 || (e.hi & 31) != 0;
  return e;
}

// Epilogue of one tile for one warp: TMEM lanes [32*quarter, +32) (the rows
// row0 .. row0+31 of the output), columns [128*chalf, +128) of the tile.
// Two 32-column TMEM loads share one wait.
template <int MODE, int OUT>
__device__ __forceinline__ void epilogue_tile(float *stg, const CUtensorMap *omap,
                                              const GemmParams &p, const TileInfo &ti,
                                              uint32_t taddr, int chalf, int64_t row0,
                                              int valid_rows, float inv_a, const float *inv_sb,
                                              int lane) {
  constexpr int kOutBytes = OUT == FP8QGG_OUT_F32 ? 4 : 2;
  const int64_t ncols = MODE == FP8QGG_M_JAGGED ? p.n : p.k;
  const int64_t row_stride = p.ld_out * kOutBytes;
  char *out_base = static_cast<char *>(p.out) +
                   (MODE == FP8QGG_K_JAGGED ? ti.e * p.out_gs * kOutBytes : 0) + row0 * row_stride;
  // token-jagged windows that cross the group's end are stored row by row
  const bool tma = MODE == FP8QGG_K_JAGGED || valid_rows == 32;
  const int32_t y = static_cast<int32_t>(row0);
#pragma unroll 1
  for (int cp = 0; cp < 2; ++cp) {
    uint32_t r0[32], r1[32];
    const uint32_t ta = taddr + 128 * chalf + 64 * cp;
    if (ti.nk > 0) {
      tmem_ld_32x32b_x32(ta, r0);
      tmem_ld_32x32b_x32(ta + 32, r1);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        r0[i] = 0u;
        r1[i] = 0u;
      }
    }
    if (valid_rows <= 0) continue;
    const int64_t col0 = static_cast<int64_t>(ti.tn) * BN + 128 * chalf + 64 * cp;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t cc = col0 + 32 * h;
      if (cc >= ncols) break;
      const uint32_t *rr = h ? r1 : r0;
      const float *ib = inv_sb + 128 * chalf + 64 * cp + 32 * h;
      emit_unit<MODE, OUT>(stg, omap, rr, inv_a, ib, static_cast<int32_t>(cc), y, ti.e, tma,
                           out_base, row_stride, valid_rows, ncols, lane);
      if constexpr (OUT == FP8QGG_OUT_F32) {
        if (cc + 16 < ncols)
          emit_unit<MODE, OUT>(stg, omap, rr + 16, inv_a, ib + 16,
                               static_cast<int32_t>(cc + 16), y, ti.e, tma, out_base, row_stride,
                               valid_rows, ncols, lane);
      }
    }
  }
}

template <int MODE, int OUT>
__global__ void __launch_bounds__(kGemm1Threads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                        const __grid_constant__ CUtensorMap bmap,
                        const __grid_constant__ CUtensorMap omap, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  GemmSmem &sm = *align_smem_1024<GemmSmem>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&amap);
    prefetch_tensormap(&bmap);
    prefetch_tensormap(&omap);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      // contraction-jagged mode: a stage is free once the MMAs are done AND
      // the mask warp has passed it, so the mask warp never falls a phase
      // behind a stage
      mbar_init(&sm.empty[s], MODE == FP8QGG_K_JAGGED ? 2 : 1);
      mbar_init(&sm.ready[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], kEpiThreads);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2) build_tile_table<MODE>(sm, p, lane);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if constexpr (MODE == FP8QGG_K_JAGGED) {
    // rank of each group by token count (ties by index): order[rank] = group
    for (int e = threadIdx.x; e < p.num_groups; e += kGemm1Threads) {
      const int32_t se = sm.end[e] - (e ? sm.end[e - 1] : 0);
      int rank = 0;
      for (int f = 0; f < p.num_groups; ++f) {
        const int32_t sf = sm.end[f] - (f ? sm.end[f - 1] : 0);
        rank += (sf > se) || (sf == se && f < e);
      }
      sm.order[rank] = e;
    }
    __syncthreads();
  }

  const int32_t total = sm.tile_prefix[p.num_groups];
  volatile int *abort = &sm.abort;
  const uint32_t tmem_base = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t armed = 0;  // stages with a load issued
      uint32_t last_par[kStages] = {0, 0, 0, 0};
      bool ok = true;
      for (int32_t i = 0, t = tile_position<MODE>(0); t < total && ok;
           t = tile_position<MODE>(++i)) {
        const TileInfo ti = tile_at<MODE>(sm, p, t);
        for (int kb = 0; kb < ti.nk; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1, abort)) { ok = false; break; }
          mbar_arrive_expect_tx(&sm.full[stage], kStageBytes);
          if constexpr (MODE == FP8QGG_M_JAGGED) {
            tma_load_2d(sm.a[stage], &amap, &sm.full[stage], kb * BK, ti.gstart + ti.tm * BM);
            tma_load_3d(sm.b[stage], &bmap, &sm.full[stage], kb * BK, ti.tn * BN, ti.e);
          } else {
            const int32_t kx = (ti.gstart & ~(BK - 1)) + kb * BK;
            tma_load_2d(sm.a[stage], &amap, &sm.full[stage], kx, ti.tm * BM);
            tma_load_2d(sm.b[stage], &bmap, &sm.full[stage], kx, ti.tn * BN);
          }
          armed |= 1u << stage;
          last_par[stage] = phase;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        *abort = 1;
        status_or(p.status, FP8QGG_STATUS_TIMEOUT);
        // let copies already in flight land before the CTA can exit
        volatile int never = 0;
        for (int s = 0; s < kStages; ++s)
          if (armed & (1u << s)) (void)mbar_wait(&sm.full[s], last_par[s], &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
    uint32_t rpar = 0;  // bit s: parity of the next phase of ready[s]
    bool ok = true;
    for (int32_t i = 0, t = tile_position<MODE>(0); t < total && ok;
         t = tile_position<MODE>(++i)) {
      const TileInfo ti = tile_at<MODE>(sm, p, t);
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.tempty[acc], acc_phase ^ 1, abort))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < ti.nk; ++kb) {
        int k0 = 0, k1 = BK / 32;  // 32-column MMA steps [k0, k1) of this block
        bool masked = false;
        if constexpr (MODE == FP8QGG_K_JAGGED) {
          // blocks start on 128-token boundaries (aligned copies); the
          // group's columns of this block are [lo, hi): steps wholly outside
          // are not issued, and the mask warp zeroes the columns of the
          // issued steps that lie outside the group
          const KEdge ed = k_edge(ti, kb);
          k0 = ed.lo >> 5;
          k1 = (ed.hi + 31) >> 5;
          masked = ed.masked;
        }
        const bool got = masked ? mbar_wait(&sm.ready[stage], (rpar >> stage) & 1u, abort)
                                : mbar_wait(&sm.full[stage], phase, abort);
        if (!__all_sync(0xFFFFFFFFu, got)) {
          ok = false;
          break;
        }
        if (masked) rpar ^= 1u << stage;
        tc_fence_after_sync();
        if (lane == 0) {
          const uint64_t adesc = smem_desc_k_sw128(smem_addr(sm.a[stage]));
          const uint64_t bdesc = smem_desc_k_sw128(smem_addr(sm.b[stage]));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            if (kk >= k0 && kk < k1)
              mma_f8f6f4(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, kIdesc, kb != 0 || kk != k0);
          mma_commit(&sm.empty[stage]);
        }
        __syncwarp();
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) {
        if (ti.nk > 0) mma_commit(&sm.tfull[acc]); else mbar_arrive(&sm.tfull[acc]);
      }
      __syncwarp();
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (!ok && lane == 0) {
      *abort = 1;
      status_or(p.status, FP8QGG_STATUS_TIMEOUT);
    }
    // every MMA this thread issued has completed before TMEM is released
    if (lane == 0) {
      mma_commit(&sm.drain);
      volatile int never = 0;
      (void)mbar_wait(&sm.drain, 0, &never);
    }
    __syncwarp();
  } else if (warp == kMaskWarp) {
    // ------------------------------------------------------------ edge masks
    // Follows every stage in order, and for each edge block of the
    // contraction-jagged mode zeroes the columns outside the group once the
    // copy has landed, then releases the block to the MMA warp.  It waits for
    // every stage's copy and counts in every stage's release, so it is never
    // more than one phase ahead of or behind a stage.
    if constexpr (MODE == FP8QGG_K_JAGGED) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int32_t i = 0, t = tile_position<MODE>(0); t < total && ok;
           t = tile_position<MODE>(++i)) {
        const TileInfo ti = tile_at<MODE>(sm, p, t);
        for (int kb = 0; kb < ti.nk; ++kb) {
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.full[stage], phase, abort))) {
            ok = false;
            break;
          }
          const KEdge ed = k_edge(ti, kb);
          if (ed.masked) {
            mask_k_edges<BM>(sm.a[stage], ed.lo, ed.hi, lane);
            mask_k_edges<BN>(sm.b[stage], ed.lo, ed.hi, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.ready[stage]);
          }
          if (lane == 0) mbar_arrive(&sm.empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok && lane == 0) {
        *abort = 1;
        status_or(p.status, FP8QGG_STATUS_TIMEOUT);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;    // 0..255
    const int ew = warp - 2;            // epilogue warp 0..7
    const int quarter = warp & 3;       // TMEM lanes [32*quarter, 32*quarter + 32)
    const int chalf = ew >> 2;          // columns [128*chalf, 128*chalf + 128) of the tile
    float *stg = sm.stg[ew];
    uint32_t acc = 0, acc_phase = 0;
    for (int32_t i = 0, t = tile_position<MODE>(0); t < total; t = tile_position<MODE>(++i)) {
      const TileInfo ti = tile_at<MODE>(sm, p, t);
      const int64_t ncols = MODE == FP8QGG_M_JAGGED ? p.n : p.k;
      {  // column reciprocal scales of this tile, one column per thread
        const int64_t col = static_cast<int64_t>(ti.tn) * BN + et;
        sm.inv_sb[acc][et] = col < ncols ? __frcp_rn(__ldg(p.scale_b + ti.e * p.sbs + col)) : 0.0f;
      }
      int64_t row0;    // first output row of the warp's 32-row window
      int valid_rows;  // rows of the window inside the group / matrix
      float inv_a = 0.0f;
      if constexpr (MODE == FP8QGG_M_JAGGED) {
        row0 = static_cast<int64_t>(ti.gstart) + static_cast<int64_t>(ti.tm) * BM + 32 * quarter;
        valid_rows = static_cast<int>(
            ::max(int64_t(0), ::min(int64_t(32), static_cast<int64_t>(ti.gend) - row0)));
        if (lane < valid_rows) inv_a = __frcp_rn(__ldg(p.scale_a + row0 + lane));
      } else {
        row0 = static_cast<int64_t>(ti.tm) * BM + 32 * quarter;
        valid_rows = static_cast<int>(::max(int64_t(0), ::min(int64_t(32), p.n - row0)));
        if (lane < valid_rows) inv_a = __frcp_rn(__ldg(p.scale_a + ti.e * p.sas + row0 + lane));
      }
      const bool got = mbar_wait(&sm.tfull[acc], acc_phase, abort);
      if (!epi_bar_and<kEpiThreads>(got)) {
        *abort = 1;
        if (et == 0) status_or(p.status, FP8QGG_STATUS_TIMEOUT);
        break;
      }
      tc_fence_after_sync();
      epilogue_tile<MODE, OUT>(stg, &omap, p, ti,
                               tmem_base + (static_cast<uint32_t>(32 * quarter) << 16) + acc * BN,
                               chalf, row0, valid_rows, inv_a, sm.inv_sb[acc], lane);
      tc_fence_before_sync();
      mbar_arrive(&sm.tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    // every bulk store has completed before the block exits
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Token-jagged mode on SM pairs (cta_group::2).  A cluster of two CTAs owns a
// 256 x 256 output tile: each CTA loads 128 rows of A and 128 rows of B (its
// half of the tile's N) per k-block, the first CTA of the pair issues
// tcgen05.mma.cta_group::2 (M256 N256 K32) reading both CTAs' shared memory,
// and each CTA's TMEM receives its 128 rows of the accumulator.  Per SM the
// operand stream is 32 KB per 128-deep k-block instead of 48 KB, and the ring
// has 6 stages.  Both CTAs' copies complete on the first CTA's full barriers;
// its commits are multicast to both CTAs' empty and accumulator-full
// barriers; both epilogues release the first CTA's accumulator-empty barrier.
constexpr int kPairRows = 256;
constexpr int kStages2 = 6;
constexpr uint32_t kStage2Bytes = 2u * (128 + 128) * BK;  // both CTAs' copies
constexpr uint32_t kIdesc2 = idesc_e4m3_f32(256, BN);

struct Gemm2Smem {
  uint8_t a[kStages2][128 * BK];
  uint8_t b[kStages2][128 * BK];
  float stg[kEpiWarps][512];
  float inv_sb[2][BN];
  int32_t end[kMaxGemmGroups];
  int32_t tile_prefix[kMaxGemmGroups + 1];
  uint64_t full[kStages2];
  uint64_t empty[kStages2];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap amap,
                            const __grid_constant__ CUtensorMap bmap,
                            const __grid_constant__ CUtensorMap omap, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  Gemm2Smem &sm = *align_smem_1024<Gemm2Smem>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool first = rank == 0;
  constexpr int MODE = FP8QGG_M_JAGGED;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&amap);
    prefetch_tensormap(&bmap);
    prefetch_tensormap(&omap);
    for (int s2 = 0; s2 < kStages2; ++s2) {
      mbar_init(&sm.full[s2], 1);
      mbar_init(&sm.empty[s2], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], 2 * kEpiThreads);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc_2sm(&sm.tmem_base, kTmemCols);
    tmem_relinquish_2sm();
  }
  if (warp == 2) build_tile_table<MODE, kPairRows>(sm, p, lane);
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any copy or arrive crosses the pair
  tc_fence_after_sync();

  const int32_t total = sm.tile_prefix[p.num_groups];
  const int32_t cid = static_cast<int32_t>(blockIdx.x) >> 1;
  const int32_t ncl = static_cast<int32_t>(gridDim.x) >> 1;
  volatile int *abort = &sm.abort;
  const uint32_t tmem_base = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t armed = 0;
      uint32_t last_par[kStages2];
      bool ok = true;
      for (int32_t t = cid; t < total && ok; t += ncl) {
        const TileInfo ti = decode_tile<MODE, kPairRows>(sm, p, t);
        const int32_t arow = ti.gstart + ti.tm * kPairRows + 128 * static_cast<int32_t>(rank);
        const int32_t brow = ti.tn * BN + 128 * static_cast<int32_t>(rank);
        for (int kb = 0; kb < ti.nk; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1, abort)) { ok = false; break; }
          const uint32_t full0 = mapa_shared(smem_addr(&sm.full[stage]), 0);
          if (first) {
            mbar_arrive_expect_tx(&sm.full[stage], kStage2Bytes);
            armed |= 1u << stage;
            last_par[stage] = phase;
          }
          tma_load_2d_2sm(sm.a[stage], &amap, full0, kb * BK, arow);
          tma_load_3d_2sm(sm.b[stage], &bmap, full0, kb * BK, brow, ti.e);
          if (++stage == kStages2) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        *abort = 1;
        status_or(p.status, FP8QGG_STATUS_TIMEOUT);
        volatile int never = 0;
        for (int s2 = 0; s2 < kStages2; ++s2)
          if (armed & (1u << s2)) (void)mbar_wait(&sm.full[s2], last_par[s2], &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (first CTA)
    if (first) {
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int32_t t = cid; t < total && ok; t += ncl) {
        const TileInfo ti = decode_tile<MODE, kPairRows>(sm, p, t);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.tempty[acc], acc_phase ^ 1, abort))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < ti.nk; ++kb) {
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.full[stage], phase, abort))) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          if (lane == 0) {
            const uint64_t adesc = smem_desc_k_sw128(smem_addr(sm.a[stage]));
            const uint64_t bdesc = smem_desc_k_sw128(smem_addr(sm.b[stage]));
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
              mma_f8f6f4_2sm(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, kIdesc2, (kb | kk) != 0);
            mma_commit_2sm_mc(&sm.empty[stage], 0x3);
          }
          __syncwarp();
          if (++stage == kStages2) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (lane == 0) mma_commit_2sm_mc(&sm.tfull[acc], 0x3);
        __syncwarp();
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      if (!ok && lane == 0) {
        *abort = 1;
        status_or(p.status, FP8QGG_STATUS_TIMEOUT);
      }
      if (lane == 0) {
        mma_commit_2sm(&sm.drain);
        volatile int never = 0;
        (void)mbar_wait(&sm.drain, 0, &never);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int et = threadIdx.x - 64;
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int chalf = ew >> 2;
    float *stg = sm.stg[ew];
    uint32_t tempty0[2];
    for (int b = 0; b < 2; ++b) tempty0[b] = mapa_shared(smem_addr(&sm.tempty[b]), 0);
    uint32_t acc = 0, acc_phase = 0;
    for (int32_t t = cid; t < total; t += ncl) {
      const TileInfo ti = decode_tile<MODE, kPairRows>(sm, p, t);
      {
        const int64_t col = static_cast<int64_t>(ti.tn) * BN + et;
        sm.inv_sb[acc][et] = col < p.n ? __frcp_rn(__ldg(p.scale_b + ti.e * p.sbs + col)) : 0.0f;
      }
      const int64_t row0 = static_cast<int64_t>(ti.gstart) + static_cast<int64_t>(ti.tm) * kPairRows +
                           128 * static_cast<int64_t>(rank) + 32 * quarter;
      const int valid_rows = static_cast<int>(
          ::max(int64_t(0), ::min(int64_t(32), static_cast<int64_t>(ti.gend) - row0)));
      float inv_a = 0.0f;
      if (lane < valid_rows) inv_a = __frcp_rn(__ldg(p.scale_a + row0 + lane));
      const bool got = mbar_wait(&sm.tfull[acc], acc_phase, abort);
      if (!epi_bar_and<kEpiThreads>(got)) {
        *abort = 1;
        if (et == 0) status_or(p.status, FP8QGG_STATUS_TIMEOUT);
        break;
      }
      tc_fence_after_sync();
      epilogue_tile<MODE, OUT>(stg, &omap, p, ti,
                               tmem_base + (static_cast<uint32_t>(32 * quarter) << 16) + acc * BN,
                               chalf, row0, valid_rows, inv_a, sm.inv_sb[acc], lane);
      tc_fence_before_sync();
      mbar_arrive_cluster(tempty0[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();  // the pair's MMAs are drained and no peer access is pending
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_2sm(tmem_base, kTmemCols);
  }
}

namespace {
using GemmKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                           const GemmParams);

GemmKernel gemm_kernel(int mode, int out_dtype) {
  if (mode == FP8QGG_M_JAGGED)
    return out_dtype == FP8QGG_OUT_F32 ? grouped_gemm_kernel<FP8QGG_M_JAGGED, FP8QGG_OUT_F32>
                                       : grouped_gemm_kernel<FP8QGG_M_JAGGED, FP8QGG_OUT_BF16>;
  return out_dtype == FP8QGG_OUT_F32 ? grouped_gemm_kernel<FP8QGG_K_JAGGED, FP8QGG_OUT_F32>
                                     : grouped_gemm_kernel<FP8QGG_K_JAGGED, FP8QGG_OUT_BF16>;
}
}  // namespace

}  // namespace fp8qgg

using namespace fp8qgg;

extern "C" int fp8_scaled_grouped_gemm(int mode, const uint8_t *a, int64_t ld_a,
                                       const float *scale_a, int64_t scale_a_group_stride,
                                       const uint8_t *b, int64_t ld_b, int64_t b_group_stride,
                                       const float *scale_b, int64_t scale_b_group_stride,
                                       const int32_t *offsets, int32_t num_groups,
                                       int64_t m_total, int64_t n, int64_t k, void *out,
                                       int64_t ld_out, int64_t out_group_stride, int out_dtype,
                                       int fmt, int32_t *dev_status, void *stream) {
  if (mode != FP8QGG_M_JAGGED && mode != FP8QGG_K_JAGGED && mode != FP8QGG_K_JAGGED_PADDED)
    return FP8QGG_ERR_UNSUPPORTED;
  const bool padded = mode == FP8QGG_K_JAGGED_PADDED;
  if (padded) mode = FP8QGG_K_JAGGED;
  if (out_dtype != FP8QGG_OUT_F32 && out_dtype != FP8QGG_OUT_BF16) return FP8QGG_ERR_UNSUPPORTED;
  if (fmt != FP8QGG_E4M3FN) return FP8QGG_ERR_UNSUPPORTED;
  if (num_groups < 1 || num_groups > kMaxGemmGroups) return FP8QGG_ERR_SHAPE;
  if (m_total < 0 || m_total > INT32_MAX - 2 * BK || n < 1 || k < 1) return FP8QGG_ERR_SHAPE;
  if (n > INT32_MAX / 2 || k > INT32_MAX / 2) return FP8QGG_ERR_SHAPE;
  const int64_t ocols = mode == FP8QGG_M_JAGGED ? n : k;
  const int vec = out_dtype == FP8QGG_OUT_F32 ? 4 : 8;
  if (mode == FP8QGG_M_JAGGED) {
    if (ld_a < k || ld_b < k || ld_out < n || scale_b_group_stride < n) return FP8QGG_ERR_SHAPE;
    if (num_groups > 1 && b_group_stride < n * ld_b) return FP8QGG_ERR_SHAPE;
  } else {
    // padded operands hold up to 128 * num_groups more token columns
    const int64_t tok = m_total + (padded ? int64_t(BK) * num_groups : 0);
    if (tok > INT32_MAX - 2 * BK) return FP8QGG_ERR_SHAPE;
    if (ld_a < tok || ld_b < tok || ld_out < k) return FP8QGG_ERR_SHAPE;
    if (scale_a_group_stride < n || scale_b_group_stride < k) return FP8QGG_ERR_SHAPE;
    if (num_groups > 1 && out_group_stride < n * ld_out) return FP8QGG_ERR_SHAPE;
  }
  if (!a || !b || !scale_a || !scale_b || !offsets || !out) return FP8QGG_ERR_NULL;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16)) return FP8QGG_ERR_ALIGN;
  if (!aligned(scale_a, 4) || !aligned(scale_b, 4) || !aligned(offsets, 4))
    return FP8QGG_ERR_ALIGN;
  if (dev_status && !aligned(dev_status, 4)) return FP8QGG_ERR_ALIGN;
  if (ld_a % 16 || ld_b % 16) return FP8QGG_ERR_ALIGN;
  if (mode == FP8QGG_M_JAGGED && b_group_stride % 16) return FP8QGG_ERR_ALIGN;
  if (ocols % vec || ld_out % vec) return FP8QGG_ERR_ALIGN;
  if (mode == FP8QGG_K_JAGGED && num_groups > 1 && out_group_stride % vec) return FP8QGG_ERR_ALIGN;

  CUtensorMap amap, bmap;
  const uint32_t abox[2] = {BK, BM};
  if (mode == FP8QGG_M_JAGGED) {
    const uint64_t adims[2] = {static_cast<uint64_t>(k),
                               static_cast<uint64_t>(std::max<int64_t>(m_total, 1))};
    const uint64_t astr[1] = {static_cast<uint64_t>(ld_a)};
    const uint64_t bdims[3] = {static_cast<uint64_t>(k), static_cast<uint64_t>(n),
                               static_cast<uint64_t>(num_groups)};
    const uint64_t bstr[2] = {static_cast<uint64_t>(ld_b),
                              static_cast<uint64_t>(num_groups > 1 ? b_group_stride
                                                                   : n * ld_b)};
    const uint32_t bbox[3] = {BK, BN, 1};
    if (!encode_tensor_map(&amap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(a),
                           adims, astr, abox, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(b),
                           bdims, bstr, bbox, CU_TENSOR_MAP_SWIZZLE_128B))
      return FP8QGG_ERR_CUDA;
  } else {
    const uint64_t mt = static_cast<uint64_t>(
        std::max<int64_t>(m_total + (padded ? int64_t(BK) * num_groups : 0), 1));
    const uint64_t adims[2] = {mt, static_cast<uint64_t>(n)};
    const uint64_t astr[1] = {static_cast<uint64_t>(ld_a)};
    const uint64_t bdims[2] = {mt, static_cast<uint64_t>(k)};
    const uint64_t bstr[1] = {static_cast<uint64_t>(ld_b)};
    const uint32_t bbox[2] = {BK, BN};
    if (!encode_tensor_map(&amap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(a),
                           adims, astr, abox, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(b),
                           bdims, bstr, bbox, CU_TENSOR_MAP_SWIZZLE_128B))
      return FP8QGG_ERR_CUDA;
  }

  // output map for the bulk stores: boxes of 32 rows x 64 bytes, 64-byte swizzle
  CUtensorMap omap;
  {
    const CUtensorMapDataType odt = out_dtype == FP8QGG_OUT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                                : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint64_t esz = out_dtype == FP8QGG_OUT_F32 ? 4 : 2;
    const uint32_t box_x = static_cast<uint32_t>(64 / esz);
    if (mode == FP8QGG_M_JAGGED) {
      const uint64_t dims[2] = {static_cast<uint64_t>(n),
                                static_cast<uint64_t>(std::max<int64_t>(m_total, 1))};
      const uint64_t str[1] = {static_cast<uint64_t>(ld_out) * esz};
      const uint32_t box[2] = {box_x, 32};
      if (!encode_tensor_map(&omap, odt, 2, out, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B))
        return FP8QGG_ERR_CUDA;
    } else {
      const uint64_t dims[3] = {static_cast<uint64_t>(k), static_cast<uint64_t>(n),
                                static_cast<uint64_t>(num_groups)};
      const uint64_t gs = num_groups > 1 ? static_cast<uint64_t>(out_group_stride)
                                         : static_cast<uint64_t>(n * ld_out);
      const uint64_t str[2] = {static_cast<uint64_t>(ld_out) * esz, gs * esz};
      const uint32_t box[3] = {box_x, 32, 1};
      if (!encode_tensor_map(&omap, odt, 3, out, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B))
        return FP8QGG_ERR_CUDA;
    }
  }

  DeviceInfo dev;
  if (!device_info(&dev)) return FP8QGG_ERR_CUDA;

  GemmParams prm;
  prm.scale_a = scale_a;
  prm.sas = scale_a_group_stride;
  prm.scale_b = scale_b;
  prm.sbs = scale_b_group_stride;
  prm.offsets = offsets;
  prm.num_groups = num_groups;
  prm.m_total = m_total;
  prm.n = n;
  prm.k = k;
  prm.out = out;
  prm.ld_out = ld_out;
  prm.out_gs = out_group_stride;
  prm.status = dev_status;
  prm.padded = padded ? 1 : 0;

  // Token-jagged problems whose groups average at least one 256-row pair
  // tile run on SM pairs (half the operand stream per SM); smaller groups
  // keep 128-row tiles so that little tensor work is spent on padding.
  if (mode == FP8QGG_M_JAGGED && m_total >= int64_t(kPairRows) * num_groups && dev.sm_count >= 2) {
    CUtensorMap bmap2;
    const uint64_t bdims[3] = {static_cast<uint64_t>(k), static_cast<uint64_t>(n),
                               static_cast<uint64_t>(num_groups)};
    const uint64_t bstr[2] = {static_cast<uint64_t>(ld_b),
                              static_cast<uint64_t>(num_groups > 1 ? b_group_stride : n * ld_b)};
    const uint32_t bbox[3] = {BK, 128, 1};
    if (!encode_tensor_map(&bmap2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(b),
                           bdims, bstr, bbox, CU_TENSOR_MAP_SWIZZLE_128B))
      return FP8QGG_ERR_CUDA;
    auto kern2 = out_dtype == FP8QGG_OUT_F32 ? grouped_gemm_2sm_kernel<FP8QGG_OUT_F32>
                                             : grouped_gemm_2sm_kernel<FP8QGG_OUT_BF16>;
    const int smem2 = static_cast<int>(sizeof(Gemm2Smem)) + 1024;
    if (!set_max_dynamic_smem(reinterpret_cast<const void *>(kern2), smem2))
      return FP8QGG_ERR_CUDA;
    const int64_t pair_tiles =
        ((m_total + kPairRows - 1) / kPairRows + num_groups) * ((n + BN - 1) / BN);
    const int clusters =
        static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(pair_tiles, dev.sm_count / 2)));
    kern2<<<2 * clusters, kGemmThreads, smem2, static_cast<cudaStream_t>(stream)>>>(amap, bmap2,
                                                                                  omap, prm);
    return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
  }

  GemmKernel kern = gemm_kernel(mode, out_dtype);
  const int smem = static_cast<int>(sizeof(GemmSmem)) + 1024;
  if (!set_max_dynamic_smem(reinterpret_cast<const void *>(kern), smem))
    return FP8QGG_ERR_CUDA;
  int64_t max_tiles;
  if (mode == FP8QGG_M_JAGGED)
    max_tiles = ((m_total + BM - 1) / BM + num_groups) * ((n + BN - 1) / BN);
  else
    max_tiles = int64_t(num_groups) * ((n + BM - 1) / BM) * ((k + BN - 1) / BN);
  if (max_tiles > INT32_MAX) return FP8QGG_ERR_SHAPE;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(max_tiles, dev.sm_count)));

  kern<<<grid, kGemm1Threads, smem, static_cast<cudaStream_t>(stream)>>>(amap, bmap, omap, prm);
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}
