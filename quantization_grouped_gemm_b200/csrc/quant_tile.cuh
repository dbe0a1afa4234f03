// Encoding helpers shared by the column-wise quantisation kernels that
// transpose through a shared-memory tile: 256 columns x 128 tokens of codes,
// 128-byte swizzle, filled by eight warps of 16 rows each and sent out by one
// bulk tensor store.
#pragma once

#include "device_common.cuh"

namespace fp8qgg {

constexpr int kTileTokens = 128;      // tokens per tile row (one 128-byte line)
constexpr int kTileRowsPerWarp = 16;  // a lane's tokens of one column: one 16-byte piece

// Two values times their multipliers, encoded.  FAST: one packed IEEE
// multiply and the saturating encoder (no clamp and no saturation count are
// needed when the scaling maximum is at least the format's largest finite
// value).  Otherwise: multiply, count |y| above sat_thr, clamp, encode.
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

// Column-wise codes of the lane's 16 rows into the tile: column 8*lane + j as
// one 16-byte piece (adjacent rows of a column share one conversion), at tile
// row 8*lane + j, piece w ^ (row % 8) (128-byte swizzle).  The pieces are
// stored in rotated order (lane % 8 steps), so that the 8 lanes of a
// shared-memory phase hit 8 different 16-byte bank groups.
template <int FMT, bool FAST>
__device__ __forceinline__ void tile_col_codes(const uint4 (&v)[kTileRowsPerWarp], const float (&s)[8],
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
    *reinterpret_cast<uint4 *>(tile + cc * kTileTokens + 16 * (w ^ (cc & 7))) = tok[j];
  }
}

}  // namespace fp8qgg
