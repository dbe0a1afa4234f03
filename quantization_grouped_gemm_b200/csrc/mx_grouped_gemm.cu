// MXFP8 grouped GEMM on the B200 5th-generation tensor cores: block-scaled
// tcgen05.mma (kind::mxf8f6f4, e4m3 operands, one E8M0 scale per 32-element
// block of K for every row of A and of B), fp32 accumulation in TMEM.
//
// The pages name MXFP8 grouped GEMM kernels for MoE training ("AMD Primus
// adds FP8/MXFP8 kernels ...", section "What Primus adds for MoE training on
// MI355X") without defining the format; it is taken from the OCP
// Microscaling (MX) v1.0 definition, so that
//   C[m, n] = sum_k (code_a[m,k] * 2^(sa[m, k/32] - 127)) * (code_b[n,k] * 2^(sb[n, k/32] - 127)).
// The tensor cores apply the two scales of each 32-element block to that
// block's partial products; the epilogue stores the accumulator unscaled.
//
// Modes (group tables from the offsets, read on the device as in the FP8
// grouped GEMM):
//   M_JAGGED         forward / input gradient: rows of A grouped by expert,
//                    B_e = the expert's [n, k] weights.
//   K_JAGGED_PADDED  weight gradient on the padded transposed layout: the
//                    contraction runs over each group's tokens, which start
//                    on 128-token boundaries, so no 32-token block holds two
//                    groups.
//
// Structure (one persistent CTA per SM, 10 warps):
//   warp 0     producer: lane 0 issues the TMA copies of the A and B tiles
//              (128 bytes of K per row, 128-byte swizzle) into a 4-stage ring;
//              all 32 lanes copy the stage's scale words (one 32-bit word per
//              row holds the four block scales of the stage; the words of a
//              stage are contiguous over the rows) with 4-byte cp.async,
//              lane i taking rows i, i + 32, i + 64, i + 96 (each instruction
//              reads one 128-byte line) straight into the layout tcgen05.cp
//              reads (row i + 32j of a 128-row chunk at word 4i + j), whatever
//              row the tile starts on; the stage's full barrier completes when
//              both have landed.
//   warp 1     MMA issuer: per stage, tcgen05.cp moves the scale chunks into
//              TMEM (32x128b, replicated to the four lane quarters), then four
//              block-scaled MMAs (M128 N bn K32), each selecting its block's
//              scale byte through the instruction descriptor.
//   warps 2-9  epilogue: tcgen05.ld of the accumulator, bulk tensor stores.
// TMEM: two accumulators of up to 240 columns at columns 0 and 256, the A
// scales at 496 (4 columns), the B scales at 504 (8 columns).  bn (<= 240, a
// multiple of 16 for fp32 output; <= 224, a multiple of 32, for bf16 output,
// whose 64-byte store units are 32 columns wide) is chosen per call for the
// fewest tiles with little waste.
#include <algorithm>

#include "device_common.cuh"
#include "gemm_store.cuh"
#include "host_common.h"

namespace fp8qgg {

constexpr int kMxBM = 128;
constexpr int kMxBK = 128;       // K bytes per stage = four 32-element blocks
constexpr int kMxMaxBN = 240;
constexpr int kMxStages = 4;
constexpr int kMxEpiWarps = 8;
constexpr int kMxEpiThreads = 32 * kMxEpiWarps;
constexpr int kMxGemmThreads = 64 + kMxEpiThreads;
constexpr int kMxGemmMaxGroups = 1024;
constexpr int kMxBandRows = 4096;
constexpr uint32_t kMxTmemCols = 512;
constexpr uint32_t kMxAccStride = 256;
constexpr uint32_t kMxSfaCol = 496;
constexpr uint32_t kMxSfbCol = 504;
constexpr uint32_t kMxFullCount = 1 + 32;  // lane 0's expect-tx arrive + one per lane's scale copies

struct MxGemmSmem {
  uint8_t a[kMxStages][kMxBM * kMxBK];      // 16 KB each, 1024-aligned
  uint8_t b[kMxStages][kMxMaxBN * kMxBK];   // 30 KB each
  uint8_t sfa[kMxStages][512];              // one 128-row chunk
  uint8_t sfb[kMxStages][1024];             // two 128-row chunks
  float stg[kMxEpiWarps][512];
  int32_t end[kMxGemmMaxGroups];
  int32_t pstart[kMxGemmMaxGroups];
  int32_t tile_prefix[kMxGemmMaxGroups + 1];
  int32_t order[kMxGemmMaxGroups];
  uint64_t full[kMxStages];
  uint64_t empty[kMxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(MxGemmSmem) + 1024 <= 232448, "one thread block's shared memory on sm_100a");
static_assert(kMxMaxBN + kMxAccStride <= kMxSfaCol, "the second accumulator ends below the A scales");

struct MxGemmParams {
  const uint32_t *sfa;  // scale words [stage group, ld_sa]
  int64_t ld_sa;
  const uint32_t *sfb;
  int64_t ld_sb;
  int64_t sbs;  // token-jagged mode: words between the experts' rows of B
  const int32_t *offsets;
  int num_groups;
  int64_t m_total, n, k;
  int bn;
  int b_inter;  // token-jagged: B's experts interleaved in its rows (map dims k, expert, row)
  void *out;
  int64_t ld_out;
  int64_t out_gs;
  int32_t *status;
};

struct MxTile {
  int e, tm, tn;
  int32_t gstart, gend;  // token-jagged: rows; contraction-jagged: the padded start in gstart
  int nk;
};

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// The barrier receives one arrival once every cp.async this thread issued so
// far has completed (no pending-count increment: the arrival is one of those
// the barrier was initialised with).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Shared-memory descriptor of a scale chunk for tcgen05.cp: no swizzle,
// 8-row x 16-byte core matrices, consecutive core matrices 128 bytes apart
// (stride byte offset), a single one along K (leading byte offset unused).
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;  // descriptor version
  return d;                               // layout type 0: no swizzle
}

// 32 rows x 128 bits from shared memory into TMEM columns [taddr, taddr + 4),
// replicated into the four 32-lane quarters.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// D[tmem] (+)= (A * scale_a) (B * scale_b)^T, kind::mxf8f6f4 block-scaled.
__device__ __forceinline__ void mma_mxf8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor, block-scaled kind::mxf8f6f4: A and B e4m3 [7,10)
// and [10,13) = 0, both K-major, N >> 3 at [17,23), scale type E8M0 (bit 23),
// M >> 4 at [24,29); the scale byte of block kk within the 32-bit TMEM word
// of each row: B's at [4,6), A's at [29,31).
__device__ __forceinline__ uint32_t idesc_mx(uint32_t n, uint32_t kk) {
  return (kk << 4) | ((n >> 3) << 17) | (1u << 23) | ((uint32_t(kMxBM) >> 4) << 24) | (kk << 29);
}

// ------------------------------------------------------------ tile tables
template <int MODE>
__device__ void mx_build_tables(MxGemmSmem &sm, const MxGemmParams &p, int lane) {
  const int32_t R = static_cast<int32_t>(p.m_total);
  const int32_t nt = static_cast<int32_t>((p.n + p.bn - 1) / p.bn);
  const int32_t tiles_k = static_cast<int32_t>(((p.n + kMxBM - 1) / kMxBM) *
                                               ((p.k + p.bn - 1) / p.bn));
  int32_t carry_end = 0, carry_tiles = 0, carry_pad = 0;
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
    int32_t tiles = 0, psz = 0;
    if (e < p.num_groups) {
      if constexpr (MODE == FP8QGG_M_JAGGED)
        tiles = ((endv - prev + kMxBM - 1) / kMxBM) * nt;
      else
        tiles = tiles_k;
      psz = (endv - prev + kMxBK - 1) / kMxBK * kMxBK;
    }
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t o1 = __shfl_up_sync(0xFFFFFFFFu, tiles, d);
      const int32_t o2 = __shfl_up_sync(0xFFFFFFFFu, psz, d);
      if (lane >= d) {
        tiles += o1;
        psz += o2;
      }
    }
    if (e < p.num_groups) {
      sm.end[e] = endv;
      sm.tile_prefix[e + 1] = carry_tiles + tiles;
      sm.pstart[e] = carry_pad + psz - (endv - prev + kMxBK - 1) / kMxBK * kMxBK;
    }
    carry_end = __shfl_sync(0xFFFFFFFFu, endv, 31);
    carry_tiles += __shfl_sync(0xFFFFFFFFu, tiles, 31);
    carry_pad += __shfl_sync(0xFFFFFFFFu, psz, 31);
  }
  if (lane == 0) sm.tile_prefix[0] = 0;
  bad = __any_sync(0xFFFFFFFFu, bad);
  if (bad && lane == 0 && blockIdx.x == 0) status_or(p.status, FP8QGG_STATUS_BAD_OFFSETS);
}

template <int MODE>
__device__ __forceinline__ int32_t mx_tile_position(int32_t i) {
  const int32_t G = static_cast<int32_t>(gridDim.x);
  const int32_t b = static_cast<int32_t>(blockIdx.x);
  if constexpr (MODE == FP8QGG_M_JAGGED) return b + i * G;
  return i * G + ((i & 1) ? (G - 1 - b) : b);
}

template <int MODE>
__device__ __forceinline__ MxTile mx_tile_at(const MxGemmSmem &sm, const MxGemmParams &p,
                                             int32_t t) {
  MxTile ti;
  if constexpr (MODE == FP8QGG_M_JAGGED) {
    int lo = 0, hi = p.num_groups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.tile_prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    ti.e = lo;
    ti.gstart = lo ? sm.end[lo - 1] : 0;
    ti.gend = sm.end[lo];
    const int32_t local = t - sm.tile_prefix[lo];
    // bands of M tiles: the tiles in flight share a few A rows and B rows in L2
    constexpr int kB = kMxBandRows / kMxBM;
    const int nt = static_cast<int>((p.n + p.bn - 1) / p.bn);
    const int mt = (ti.gend - ti.gstart + kMxBM - 1) / kMxBM;
    const int band = local / (kB * nt);
    const int rem = local - band * kB * nt;
    const int bm = min(kB, mt - band * kB);
    ti.tm = band * kB + rem % bm;
    ti.tn = rem / bm;
    ti.nk = static_cast<int>((p.k + kMxBK - 1) / kMxBK);
  } else {
    // every group has the same tiles; positions run over the groups sorted
    // by token count, largest first
    const int32_t tpg = sm.tile_prefix[1] - sm.tile_prefix[0];
    const int e = sm.order[t / tpg];
    const int32_t local = t - (t / tpg) * tpg;
    const int nt = static_cast<int>((p.k + p.bn - 1) / p.bn);
    ti.e = e;
    ti.gstart = sm.pstart[e];
    ti.gend = sm.end[e];
    ti.tm = local / nt;
    ti.tn = local % nt;
    const int32_t size = sm.end[e] - (e ? sm.end[e - 1] : 0);
    ti.nk = (size + kMxBK - 1) / kMxBK;
  }
  return ti;
}

template <int MODE, int OUT>
__global__ void __launch_bounds__(kMxGemmThreads, 1)
    mx_grouped_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                           const __grid_constant__ CUtensorMap bmap,
                           const __grid_constant__ CUtensorMap omap, const MxGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  MxGemmSmem &sm = *align_smem_1024<MxGemmSmem>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bn = p.bn;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&amap);
    prefetch_tensormap(&bmap);
    prefetch_tensormap(&omap);
    for (int s = 0; s < kMxStages; ++s) {
      mbar_init(&sm.full[s], kMxFullCount);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], kMxEpiThreads);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kMxTmemCols);
    tmem_relinquish();
  }
  if (warp == 2) mx_build_tables<MODE>(sm, p, lane);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if constexpr (MODE == FP8QGG_K_JAGGED) {
    // rank of each group by token count (ties by index): order[rank] = group
    for (int e = threadIdx.x; e < p.num_groups; e += kMxGemmThreads) {
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
  const uint32_t stage_bytes = static_cast<uint32_t>((kMxBM + bn) * kMxBK);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t stage = 0, phase = 0;
    uint32_t armed = 0;  // stages with copies issued
    uint32_t last_par[kMxStages] = {0, 0, 0, 0};
    bool ok = true;
    for (int32_t i = 0, t = mx_tile_position<MODE>(0); t < total && ok;
         t = mx_tile_position<MODE>(++i)) {
      const MxTile ti = mx_tile_at<MODE>(sm, p, t);
      for (int kb = 0; kb < ti.nk; ++kb) {
        bool got = true;
        if (lane == 0) got = mbar_wait(&sm.empty[stage], phase ^ 1, abort);
        if (!__shfl_sync(0xFFFFFFFFu, got, 0)) {
          ok = false;
          break;
        }
        int32_t ka;  // contraction coordinate of the stage (bytes = elements)
        if constexpr (MODE == FP8QGG_M_JAGGED)
          ka = kb * kMxBK;
        else
          ka = ti.gstart + kb * kMxBK;
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.full[stage], stage_bytes);
          if constexpr (MODE == FP8QGG_M_JAGGED) {
            tma_load_2d(sm.a[stage], &amap, &sm.full[stage], ka, ti.gstart + ti.tm * kMxBM);
            if (p.b_inter)
              tma_load_3d(sm.b[stage], &bmap, &sm.full[stage], ka, ti.e, ti.tn * bn);
            else
              tma_load_3d(sm.b[stage], &bmap, &sm.full[stage], ka, ti.tn * bn, ti.e);
          } else {
            tma_load_2d(sm.a[stage], &amap, &sm.full[stage], ka, ti.tm * kMxBM);
            tma_load_2d(sm.b[stage], &bmap, &sm.full[stage], ka, ti.tn * bn);
          }
        }
        // scale words: row i + 32j of a chunk -> word 4i + j (lane = i)
        const int64_t kg = ka / kMxBK;  // the stage's group of four blocks
        const uint32_t *sa_src = p.sfa + kg * p.ld_sa;
        const uint32_t *sb_src = p.sfb + kg * p.ld_sb +
                                 (MODE == FP8QGG_M_JAGGED ? int64_t(ti.e) * p.sbs : int64_t(0));
        const uint32_t sa_dst = smem_addr(sm.sfa[stage]) + 16 * lane;
        const uint32_t sb_dst = smem_addr(sm.sfb[stage]) + 16 * lane;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          int64_t r;
          int64_t lim;
          if constexpr (MODE == FP8QGG_M_JAGGED) {
            r = int64_t(ti.gstart) + int64_t(ti.tm) * kMxBM + lane + 32 * j;
            lim = p.m_total;
          } else {
            r = int64_t(ti.tm) * kMxBM + lane + 32 * j;
            lim = p.n;
          }
          if (r < lim) cp_async_4(sa_dst + 4 * j, sa_src + r);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int rr = 128 * c + lane + 32 * j;  // row of the B tile
            const int64_t nrow = int64_t(ti.tn) * bn + rr;
            if (rr < bn && nrow < (MODE == FP8QGG_M_JAGGED ? p.n : p.k))
              cp_async_4(sb_dst + 512 * c + 4 * j, sb_src + nrow);
          }
        }
        cp_async_arrive_noinc(&sm.full[stage]);
        armed |= 1u << stage;
        last_par[stage] = phase;
        if (++stage == kMxStages) { stage = 0; phase ^= 1; }
      }
    }
    cp_async_wait_all();
    if (!ok && lane == 0) {
      *abort = 1;
      status_or(p.status, FP8QGG_STATUS_TIMEOUT);
      // let copies already in flight land before the CTA can exit
      volatile int never = 0;
      for (int s = 0; s < kMxStages; ++s)
        if (armed & (1u << s)) (void)mbar_wait(&sm.full[s], last_par[s], &never);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
    bool ok = true;
    const uint32_t sfa_t = tmem_base + kMxSfaCol;
    const uint32_t sfb_t = tmem_base + kMxSfbCol;
    for (int32_t i = 0, t = mx_tile_position<MODE>(0); t < total && ok;
         t = mx_tile_position<MODE>(++i)) {
      const MxTile ti = mx_tile_at<MODE>(sm, p, t);
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.tempty[acc], acc_phase ^ 1, abort))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + acc * kMxAccStride;
      for (int kb = 0; kb < ti.nk; ++kb) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.full[stage], phase, abort))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        if (lane == 0) {
          // the scale bytes came through cp.async (generic proxy); tcgen05.cp
          // reads them through the async proxy
          fence_proxy_async_smem();
          tmem_cp_32x128b_x4(sfa_t, smem_desc_sf(smem_addr(sm.sfa[stage])));
          tmem_cp_32x128b_x4(sfb_t, smem_desc_sf(smem_addr(sm.sfb[stage])));
          if (bn > 128) tmem_cp_32x128b_x4(sfb_t + 4, smem_desc_sf(smem_addr(sm.sfb[stage]) + 512));
          const uint64_t adesc = smem_desc_k_sw128(smem_addr(sm.a[stage]));
          const uint64_t bdesc = smem_desc_k_sw128(smem_addr(sm.b[stage]));
          // blocks past K (token-jagged mode, K not a multiple of 128) are not issued
          int nkk = 4;
          if constexpr (MODE == FP8QGG_M_JAGGED)
            nkk = static_cast<int>(::min(int64_t(4), (p.k - int64_t(kb) * kMxBK) / 32));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            if (kk < nkk)
              mma_mxf8f6f4(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc_mx(bn, kk), sfa_t, sfb_t,
                           kb != 0 || kk != 0);
          mma_commit(&sm.empty[stage]);
        }
        __syncwarp();
        if (++stage == kMxStages) { stage = 0; phase ^= 1; }
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
    // every MMA and copy this thread issued has completed before TMEM is released
    if (lane == 0) {
      mma_commit(&sm.drain);
      volatile int never = 0;
      (void)mbar_wait(&sm.drain, 0, &never);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;       // epilogue warp 0..7
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const int half = ew >> 2;      // 32-column units half, half + 2, ...
    float *stg = sm.stg[ew];
    constexpr int kOutBytes = OUT == FP8QGG_OUT_F32 ? 4 : 2;
    const int64_t ncols = MODE == FP8QGG_M_JAGGED ? p.n : p.k;
    const int64_t row_stride = p.ld_out * kOutBytes;
    const float ones[32] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f,
                            1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f,
                            1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
    uint32_t acc = 0, acc_phase = 0;
    for (int32_t i = 0, t = mx_tile_position<MODE>(0); t < total;
         t = mx_tile_position<MODE>(++i)) {
      const MxTile ti = mx_tile_at<MODE>(sm, p, t);
      int64_t row0;
      int valid_rows;
      if constexpr (MODE == FP8QGG_M_JAGGED) {
        row0 = int64_t(ti.gstart) + int64_t(ti.tm) * kMxBM + 32 * quarter;
        valid_rows = static_cast<int>(
            ::max(int64_t(0), ::min(int64_t(32), int64_t(ti.gend) - row0)));
      } else {
        row0 = int64_t(ti.tm) * kMxBM + 32 * quarter;
        valid_rows = static_cast<int>(::max(int64_t(0), ::min(int64_t(32), p.n - row0)));
      }
      const bool got = mbar_wait(&sm.tfull[acc], acc_phase, abort);
      if (!epi_bar_and<kMxEpiThreads>(got)) {
        *abort = 1;
        if (ew == 0 && lane == 0) status_or(p.status, FP8QGG_STATUS_TIMEOUT);
        break;
      }
      tc_fence_after_sync();
      char *out_base = static_cast<char *>(p.out) +
                       (MODE == FP8QGG_K_JAGGED ? int64_t(ti.e) * p.out_gs * kOutBytes : 0) +
                       row0 * row_stride;
      const bool tma = MODE == FP8QGG_K_JAGGED || valid_rows == 32;
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(32 * quarter) << 16) + acc * kMxAccStride;
      for (int u = half; 32 * u < bn; u += 2) {
        // a 16-column last chunk (fp32 output only) is loaded and stored alone,
        // so that nothing past the tile's bn columns is read or written
        const bool whole = 32 * u + 32 <= bn;
        uint32_t r[32];
        if (ti.nk > 0) {
          if (whole) {
            tmem_ld_32x32b_x32(taddr + 32 * u, r);
          } else {
            uint32_t h[16];
            tmem_ld_32x32b_x16(taddr + 32 * u, h);
#pragma unroll
            for (int c = 0; c < 16; ++c) r[c] = h[c];
#pragma unroll
            for (int c = 16; c < 32; ++c) r[c] = 0u;
          }
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) r[c] = 0u;
        }
        if (valid_rows <= 0) continue;
        const int64_t cc = int64_t(ti.tn) * bn + 32 * u;
        if (cc >= ncols) continue;
        emit_unit<MODE, OUT, false>(stg, &omap, r, 1.f, ones, static_cast<int32_t>(cc),
                                    static_cast<int32_t>(row0), ti.e, tma, out_base, row_stride,
                                    valid_rows, ncols, lane);
        if constexpr (OUT == FP8QGG_OUT_F32) {
          if (whole && cc + 16 < ncols)
            emit_unit<MODE, OUT, false>(stg, &omap, r + 16, 1.f, ones,
                                        static_cast<int32_t>(cc + 16), static_cast<int32_t>(row0),
                                        ti.e, tma, out_base, row_stride, valid_rows, ncols, lane);
        }
      }
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
    tmem_dealloc(tmem_base, kMxTmemCols);
  }
}

using MxGemmKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                              const MxGemmParams);

MxGemmKernel mx_gemm_kernel(int mode, int out_dtype) {
  if (mode == FP8QGG_M_JAGGED)
    return out_dtype == FP8QGG_OUT_F32 ? mx_grouped_gemm_kernel<FP8QGG_M_JAGGED, FP8QGG_OUT_F32>
                                       : mx_grouped_gemm_kernel<FP8QGG_M_JAGGED, FP8QGG_OUT_BF16>;
  return out_dtype == FP8QGG_OUT_F32 ? mx_grouped_gemm_kernel<FP8QGG_K_JAGGED, FP8QGG_OUT_F32>
                                     : mx_grouped_gemm_kernel<FP8QGG_K_JAGGED, FP8QGG_OUT_BF16>;
}

// N tile width: a multiple of `gran` (16 for fp32 output, 32 for bf16) up to
// the widest such width that fits (240 / 224), for the tile count (between the
// fewest possible and four more) of the lowest cost, counting 256 columns of
// fixed cost per tile: on B200 a 128-deep stage takes about the same time at
// any width from 128 to 224 columns (481 us at 224 and 531 us at 192 on the
// Llama3-8B up-projection fit a fixed cost of some 330 columns).
int mx_pick_bn(int64_t n, int gran) {
  const int max_bn = kMxMaxBN / gran * gran;
  const int64_t t0 = (n + max_bn - 1) / max_bn;
  int best_bn = max_bn;
  int64_t best_cost = INT64_MAX;
  for (int64_t t = t0; t <= t0 + 4; ++t) {
    const int64_t w = std::max<int64_t>(32, ((n + t - 1) / t + gran - 1) / gran * gran);
    if (w > max_bn) continue;
    const int64_t tiles = (n + w - 1) / w;
    const int64_t cost = tiles * (w + 256);
    if (cost < best_cost) {
      best_cost = cost;
      best_bn = static_cast<int>(w);
    }
  }
  return best_bn;
}

}  // namespace fp8qgg

using namespace fp8qgg;

extern "C" int fp8_mx_grouped_gemm(int mode, const uint8_t *a, int64_t ld_a,
                                   const uint32_t *scale_a, int64_t ld_sa, const uint8_t *b,
                                   int64_t ld_b, int64_t b_group_stride, const uint32_t *scale_b,
                                   int64_t ld_sb, int64_t scale_b_group_stride,
                                   const int32_t *offsets, int32_t num_groups, int64_t m_total,
                                   int64_t n, int64_t k, void *out, int64_t ld_out,
                                   int64_t out_group_stride, int out_dtype, int32_t *dev_status,
                                   void *stream) {
  if (mode != FP8QGG_M_JAGGED && mode != FP8QGG_K_JAGGED_PADDED) return FP8QGG_ERR_UNSUPPORTED;
  const int kmode = mode == FP8QGG_M_JAGGED ? FP8QGG_M_JAGGED : FP8QGG_K_JAGGED;
  if (out_dtype != FP8QGG_OUT_F32 && out_dtype != FP8QGG_OUT_BF16) return FP8QGG_ERR_UNSUPPORTED;
  if (num_groups < 1 || num_groups > kMxGemmMaxGroups) return FP8QGG_ERR_SHAPE;
  if (m_total < 0 || m_total > INT32_MAX / 2 || n < 1 || k < 1) return FP8QGG_ERR_SHAPE;
  if (n > INT32_MAX / 2 || k > INT32_MAX / 2) return FP8QGG_ERR_SHAPE;
  const int vec = out_dtype == FP8QGG_OUT_F32 ? 4 : 8;
  const int64_t ocols = kmode == FP8QGG_M_JAGGED ? n : k;
  bool interleaved = false;
  if (kmode == FP8QGG_M_JAGGED) {
    if (k % 32) return FP8QGG_ERR_SHAPE;
    if (ld_a < k || ld_out < n || ld_sa < m_total) return FP8QGG_ERR_SHAPE;
    // the experts' B matrices may be stacked (B_e after B_{e-1}) or
    // interleaved (row i of every B_e in row i of one matrix, as the
    // column-wise quantisation of W writes W^T); either way they must not
    // overlap
    const int64_t E = num_groups;
    const bool b_stacked = ld_b >= k && (E == 1 || b_group_stride >= n * ld_b);
    const bool b_inter = E > 1 && b_group_stride >= k && ld_b >= (E - 1) * b_group_stride + k;
    if (!b_stacked && !b_inter) return FP8QGG_ERR_SHAPE;
    interleaved = !b_stacked;
    // scale words likewise: the experts' rows stacked within a 128-column
    // group, or each expert's groups in a block of its own
    const int64_t kgroups = (k + kMxBK - 1) / kMxBK;
    const bool s_stacked = E == 1 ? ld_sb >= n
                                  : scale_b_group_stride >= n &&
                                        ld_sb >= (E - 1) * scale_b_group_stride + n;
    const bool s_blocked = E > 1 && ld_sb >= n && scale_b_group_stride >= kgroups * ld_sb;
    if (!s_stacked && !s_blocked) return FP8QGG_ERR_SHAPE;
  } else {
    const int64_t tok = m_total + int64_t(kMxBK) * num_groups;
    if (tok > INT32_MAX / 2) return FP8QGG_ERR_SHAPE;
    if (ld_a < tok || ld_b < tok || ld_out < k || ld_sa < n || ld_sb < k) return FP8QGG_ERR_SHAPE;
    if (num_groups > 1 && out_group_stride < n * ld_out) return FP8QGG_ERR_SHAPE;
  }
  if (!a || !b || !scale_a || !scale_b || !offsets || !out) return FP8QGG_ERR_NULL;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16)) return FP8QGG_ERR_ALIGN;
  if (!aligned(scale_a, 4) || !aligned(scale_b, 4) || !aligned(offsets, 4)) return FP8QGG_ERR_ALIGN;
  if (dev_status && !aligned(dev_status, 4)) return FP8QGG_ERR_ALIGN;
  if (ld_a % 16 || ld_b % 16) return FP8QGG_ERR_ALIGN;
  if (kmode == FP8QGG_M_JAGGED && b_group_stride % 16) return FP8QGG_ERR_ALIGN;
  if (ocols % vec || ld_out % vec) return FP8QGG_ERR_ALIGN;
  if (kmode == FP8QGG_K_JAGGED && num_groups > 1 && out_group_stride % vec)
    return FP8QGG_ERR_ALIGN;
  if (kmode == FP8QGG_M_JAGGED && m_total == 0) return FP8QGG_OK;  // no rows: nothing to write

  const int bn = mx_pick_bn(kmode == FP8QGG_M_JAGGED ? n : k, out_dtype == FP8QGG_OUT_F32 ? 16 : 32);
  CUtensorMap amap, bmap;
  const uint32_t abox[2] = {kMxBK, kMxBM};
  if (kmode == FP8QGG_M_JAGGED) {
    const uint64_t adims[2] = {static_cast<uint64_t>(k), static_cast<uint64_t>(m_total)};
    const uint64_t astr[1] = {static_cast<uint64_t>(ld_a)};
    // stacked experts: dims (k, row, expert); interleaved: (k, expert, row),
    // so that the strides grow with the dimension either way
    const uint64_t bdims[3] = {
        static_cast<uint64_t>(k),
        static_cast<uint64_t>(interleaved ? num_groups : n),
        static_cast<uint64_t>(interleaved ? n : num_groups)};
    const uint64_t bstr[2] = {
        static_cast<uint64_t>(interleaved ? b_group_stride : ld_b),
        static_cast<uint64_t>(interleaved ? ld_b
                                          : (num_groups > 1 ? b_group_stride : n * ld_b))};
    const uint32_t bbox[3] = {kMxBK, interleaved ? 1u : static_cast<uint32_t>(bn),
                              interleaved ? static_cast<uint32_t>(bn) : 1u};
    if (!encode_tensor_map(&amap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(a),
                           adims, astr, abox, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(b),
                           bdims, bstr, bbox, CU_TENSOR_MAP_SWIZZLE_128B))
      return FP8QGG_ERR_CUDA;
  } else {
    const uint64_t mt = static_cast<uint64_t>(m_total + int64_t(kMxBK) * num_groups);
    const uint64_t adims[2] = {mt, static_cast<uint64_t>(n)};
    const uint64_t astr[1] = {static_cast<uint64_t>(ld_a)};
    const uint64_t bdims[2] = {mt, static_cast<uint64_t>(k)};
    const uint64_t bstr[1] = {static_cast<uint64_t>(ld_b)};
    const uint32_t bbox[2] = {kMxBK, static_cast<uint32_t>(bn)};
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
    if (kmode == FP8QGG_M_JAGGED) {
      const uint64_t dims[2] = {static_cast<uint64_t>(n), static_cast<uint64_t>(m_total)};
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
  MxGemmParams prm;
  prm.sfa = scale_a;
  prm.ld_sa = ld_sa;
  prm.sfb = scale_b;
  prm.ld_sb = ld_sb;
  prm.sbs = scale_b_group_stride;
  prm.offsets = offsets;
  prm.num_groups = num_groups;
  prm.m_total = m_total;
  prm.n = n;
  prm.k = k;
  prm.bn = bn;
  prm.b_inter = interleaved ? 1 : 0;
  prm.out = out;
  prm.ld_out = ld_out;
  prm.out_gs = out_group_stride;
  prm.status = dev_status;
  MxGemmKernel kern = mx_gemm_kernel(kmode, out_dtype);
  const int smem = static_cast<int>(sizeof(MxGemmSmem)) + 1024;
  if (!set_max_dynamic_smem(reinterpret_cast<const void *>(kern), smem)) return FP8QGG_ERR_CUDA;
  int64_t max_tiles;
  if (kmode == FP8QGG_M_JAGGED)
    max_tiles = ((m_total + kMxBM - 1) / kMxBM + num_groups) * ((n + bn - 1) / bn);
  else
    max_tiles = int64_t(num_groups) * ((n + kMxBM - 1) / kMxBM) * ((k + bn - 1) / bn);
  if (max_tiles > INT32_MAX) return FP8QGG_ERR_SHAPE;
  const int grid =
      static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(max_tiles, dev.sm_count)));
  kern<<<grid, kMxGemmThreads, smem, static_cast<cudaStream_t>(stream)>>>(amap, bmap, omap, prm);
  return cudaGetLastError() == cudaSuccess ? FP8QGG_OK : FP8QGG_ERR_CUDA;
}
