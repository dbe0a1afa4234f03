// Output stores of the grouped GEMM epilogues (shared by the scaled FP8 and
// the block-scaled MXFP8 kernels).
#pragma once

#include <cuda_bf16.h>

#include "device_common.cuh"

namespace fp8qgg {

// Barrier (id 1) over the kThreads epilogue threads that also ANDs a flag
// across them, so that an abort is always decided by all of them together.
template <int kThreads>
__device__ __forceinline__ bool epi_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kThreads)
      : "memory");
  return r != 0;
}

// One output unit of an epilogue warp: its 32 rows x 64 bytes (16 fp32 or 32
// bf16 columns starting at column x).  The values are scaled in registers and
// written to the warp's 2 KB buffer in the 64-byte swizzle layout (16-byte
// piece j of row r at piece j ^ ((r >> 1) & 3): conflict-free row-wise
// writes).  Then either one bulk tensor store sends the buffer out (clipped at
// the edges of the output tensor), or, for a window that crosses the end of
// its group, lanes write the valid rows back as coalesced 16-byte pieces.
// Streaming stores keep the output from evicting the operands from L2.
// SCALED = false (block-scaled products, already scaled by the tensor cores)
// stores the accumulator as it is.
template <int MODE, int OUT, bool SCALED = true>
__device__ __forceinline__ void emit_unit(float *buf, const CUtensorMap *omap, const uint32_t *r,
                                          float inv_a, const float *inv_b, int32_t x, int32_t y,
                                          int32_t e, bool tma, char *out_base,
                                          int64_t row_stride, int valid_rows, int64_t ncols,
                                          int lane) {
  constexpr int kOutBytes = OUT == FP8QGG_OUT_F32 ? 4 : 2;
  if (lane == 0) bulk_wait_read<0>();
  __syncwarp();
  uint32_t *bw = reinterpret_cast<uint32_t *>(buf);
  auto val = [&](int c) {
    if constexpr (SCALED)
      return __fmul_rn(__fmul_rn(__uint_as_float(r[c]), inv_a), inv_b[c]);
    else
      return __uint_as_float(r[c]);
  };
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 v;
    if constexpr (OUT == FP8QGG_OUT_F32) {
      v.x = __float_as_uint(val(4 * j + 0));
      v.y = __float_as_uint(val(4 * j + 1));
      v.z = __float_as_uint(val(4 * j + 2));
      v.w = __float_as_uint(val(4 * j + 3));
    } else {
      uint32_t w[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int c = 8 * j + 2 * h;
        const float f0 = val(c);
        const float f1 = val(c + 1);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(f0, f1);
        w[h] = *reinterpret_cast<uint32_t *>(&b2);
      }
      v = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *reinterpret_cast<uint4 *>(bw + lane * 16 + 4 * (j ^ ((lane >> 1) & 3))) = v;
  }
  if (tma) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if constexpr (MODE == FP8QGG_M_JAGGED)
        tma_store_2d(omap, buf, x, y);
      else
        tma_store_3d(omap, buf, x, y, e);
      bulk_commit();
    }
  } else {
    __syncwarp();
    constexpr int kColsPerPiece = 16 / kOutBytes;
#pragma unroll
    for (int pss = 0; pss < 4; ++pss) {
      const int row = pss * 8 + (lane >> 2);
      const int j = lane & 3;
      const uint4 v = *reinterpret_cast<const uint4 *>(bw + row * 16 + 4 * (j ^ ((row >> 1) & 3)));
      const int64_t col = static_cast<int64_t>(x) + kColsPerPiece * j;
      if (row < valid_rows && col < ncols)
        __stcs(reinterpret_cast<uint4 *>(out_base + row * row_stride + col * kOutBytes), v);
    }
    __syncwarp();
  }
}


}  // namespace fp8qgg
