// Device-side building blocks shared by the fp8qgg kernels (sm_100a only):
// bounded mbarrier waits, TMA tile loads, tcgen05 (TMEM allocation, MMA,
// commit, loads), e4m3 conversion and the absmax helpers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fp8qgg.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "fp8qgg kernels target sm_100a only"
#endif

namespace fp8qgg {

// A bounded device wait gives up after this many nanoseconds of global time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// The wait of a cast for its unit's merged absmax (jagged column-wise
// kernels): the arrivals it needs beyond the unit's own (0 in every normal
// call) and its time limit.  Only the failure-detection test changes them
// (fp8qgg_test_unit_wait).
struct UnitWait {
  uint32_t extra_arrivals;
  uint64_t limit_ns;
};

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The first 1024-byte aligned address inside a dynamic shared-memory buffer,
// reached by pointer arithmetic on the buffer itself (a detour through an
// integer would hide from the compiler that the result is shared memory, and
// every access through it would become a generic one).
template <class T>
__device__ __forceinline__ T *align_smem_1024(uint8_t *raw) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(raw));
  return reinterpret_cast<T *>(raw + ((1024u - (a & 1023u)) & 1023u));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void status_or(int32_t *status, int32_t bits) {
  if (status) atomicOr(status, bits);
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits for the phase with the given parity.  Gives up (returns false) when
// *abort becomes non-zero or after kWaitLimitNs; never spins forever.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          volatile int *abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// --------------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Bulk tensor stores from shared memory (async proxy; the caller fences its
// shared-memory writes with fence_proxy_async_smem first).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t c0,
                                             int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_addr(src)), "r"(c0), "r"(c1)
               : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int32_t c0,
                                             int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_addr(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// -------------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f8f6f4, both operands K-major.
__device__ __forceinline__ void mma_f8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// TMEM lane (base lane + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns (the same lane mapping).
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------ clusters and 2-SM MMA
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// All threads of all CTAs of the cluster.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (local or peer).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__device__ __forceinline__ void tmem_alloc_2sm(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_2sm() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_2sm(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D (M=256 across the CTA pair) (+)= A * B^T; issued by the pair's first CTA.
__device__ __forceinline__ void mma_f8f6f4_2sm(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the mbarrier at this shared-memory offset in every CTA of `mask`
// once the pair's previously issued MMAs have completed.
__device__ __forceinline__ void mma_commit_2sm_mc(uint64_t *bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_addr(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void mma_commit_2sm(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// TMA tile loads whose completion is counted on an mbarrier that may live in
// the peer CTA of the pair (shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_2sm(void *dst, const CUtensorMap *map,
                                                uint32_t mbar_cluster, int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_2sm(void *dst, const CUtensorMap *map,
                                                uint32_t mbar_cluster, int32_t c0, int32_t c1,
                                                int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 128 bytes, 8-row groups 1024 bytes apart.
// Bits: start address >> 4 [0,14), leading byte offset >> 4 [16,30) (unused
// for swizzled K-major, set to 1), stride byte offset >> 4 [32,46),
// descriptor version 1 [46,48), layout type 2 = 128B swizzle [61,64).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor, kind::f8f6f4: D fp32, A and B e4m3, both K-major,
// dense, no negation.  N >> 3 at [17,23), M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(uint32_t m, uint32_t n) {
  return (1u << 4)            // D format fp32
         | (0u << 7)          // A format e4m3
         | (0u << 10)         // B format e4m3
         | ((n >> 3) << 17)   // N
         | ((m >> 4) << 24);  // M
}

// -------------------------------------------------------------- e4m3 convert
// Two fp32 -> two e4m3fn codes (lo in the low byte), round to nearest even,
// saturating to +-448.
__device__ __forceinline__ uint32_t cvt_e4m3fn_x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// e4m3fnuz from the hardware e4m3fn converter.  Every e4m3fnuz value is
// exactly half the e4m3fn value with the same bits (bias 8 instead of 7, the
// same mantissa and subnormal layout), and doubling an fp32 value is exact,
// so rounding 2y onto the e4m3fn grid is rounding y onto the e4m3fnuz grid.
// Two code points differ: 0x7F (240 in e4m3fnuz, NaN in e4m3fn) is chosen
// when |y| lies above the midpoint 232 between 224 and 240, and the e4m3fn
// negative zero 0x80 (the e4m3fnuz NaN) becomes the single zero 0x00.
__device__ __forceinline__ uint32_t fnuz_fix(uint32_t code, float y) {
  if (y != y) return 0x80u;  // NaN: the format's only NaN code
  if (fabsf(y) > 232.0f) return (y < 0.0f ? 0x80u : 0u) | 0x7Fu;
  return code == 0x80u ? 0u : code;
}

__device__ __forceinline__ uint32_t cvt_e4m3fnuz_x2(float lo, float hi) {
  const uint32_t c = cvt_e4m3fn_x2(__fmul_rn(lo, 2.0f), __fmul_rn(hi, 2.0f));
  return fnuz_fix(c & 0xFFu, lo) | (fnuz_fix(c >> 8, hi) << 8);
}

template <int FMT>
__device__ __forceinline__ uint32_t cvt_x2(float lo, float hi) {
  if constexpr (FMT == FP8QGG_E4M3FNUZ)
    return cvt_e4m3fnuz_x2(lo, hi);
  else
    return cvt_e4m3fn_x2(lo, hi);
}

// Clamp to [-smax, smax] that lets a NaN through (to be encoded as NaN), the
// way two comparisons would; fminf/fmaxf would turn it into -smax.
__device__ __forceinline__ float clamp_keep_nan(float y, float smax) {
  return fabsf(y) > smax ? copysignf(smax, y) : y;
}

// Scale, clamp and encode one pair of bf16 values packed in a 32-bit word.
// Counts saturated elements (pre-clamp |y| above sat_thr) into *sat.
template <int FMT>
__device__ __forceinline__ uint32_t quant_pair(uint32_t packed, float s, float smax,
                                               float sat_thr, uint32_t &sat) {
  const float x0 = __uint_as_float(packed << 16);
  const float x1 = __uint_as_float(packed & 0xFFFF0000u);
  float y0 = __fmul_rn(x0, s);
  float y1 = __fmul_rn(x1, s);
  sat += (fabsf(y0) > sat_thr) + (fabsf(y1) > sat_thr);
  y0 = clamp_keep_nan(y0, smax);
  y1 = clamp_keep_nan(y1, smax);
  return cvt_x2<FMT>(y0, y1);
}

// Fast form of quant_pair for the common case: no saturation count, and no
// clamp because the scaling maximum is at least the format's largest finite
// value.  Then clamping to +-smax before the saturating encode changes no code
// (a value beyond the format maximum saturates to it either way), so the two
// products go straight to the encoder.  Both products come from one packed
// instruction (two IEEE round-to-nearest fp32 multiplies).
template <int FMT>
__device__ __forceinline__ uint32_t quant_pair_fast(uint32_t packed, uint64_t s2) {
  const float x0 = __uint_as_float(packed << 16);
  const float x1 = __uint_as_float(packed & 0xFFFF0000u);
  uint64_t xx, yy;
  asm("mov.b64 %0, {%1, %2};" : "=l"(xx) : "f"(x0), "f"(x1));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(yy) : "l"(xx), "l"(s2));
  float y0, y1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(yy));
  return cvt_x2<FMT>(y0, y1);
}

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

// Running absmax of bf16 pairs: one packed IEEE max of magnitudes per pair
// (max.xorsign.abs: |result| = max(|acc|, |x|); its sign bit carries no
// meaning and is cleared by absmax_bits).  A NaN operand is ignored, as an
// IEEE maxNum does, so a NaN input never decides a scale; the accumulator,
// which starts at zero, never becomes NaN.  Subnormals are kept.
__device__ __forceinline__ uint32_t absmax_acc(uint32_t acc, uint32_t x) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(x));
  return r;
}

// Magnitude bit patterns of a running absmax: for non-NaN bf16 they compare
// like the magnitudes themselves, so halves can be merged with integer max.
__device__ __forceinline__ uint32_t absmax_bits(uint32_t acc) { return acc & 0x7FFF7FFFu; }

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

// s = fp32(smax / max(amax, 1e-12)), IEEE division.
__device__ __forceinline__ float scale_from_amax(float amax, float smax) {
  return __fdiv_rn(smax, fmaxf(amax, 1e-12f));
}

}  // namespace fp8qgg
