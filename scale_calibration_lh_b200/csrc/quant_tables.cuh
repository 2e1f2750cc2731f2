// Exact NVFP4 fake-quantization decisions shared by the sweep kernels.
//
// "Add WMSE weight scale search calibration" (PR #2283), How: 126 candidate E4M3 block
// scales; the weights are fake-quantized to FP4 E2M1. Candidate k (0-based) is E4M3 code
// k + 1 and its scale is s_k = fp32(v_{k+1} * g). An element of magnitude a rounds to E2M1
// level j (0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6) by nearest-even rounding of the exact quotient
// a / s_k, clamped at 6. Level j >= 1 is reached iff a >= level_threshold(j, s_k).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lhcal {

constexpr int kCand = 126;
constexpr int kLev = 8;

__device__ __forceinline__ float pow2i(int e) {  // exact 2^e for -126 <= e <= 127
  return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

// E4M3 value of code (1..126), exact in fp32: e = code >> 3, m = code & 7.
__device__ __forceinline__ float e4m3_value(int code) {
  const int e = code >> 3, m = code & 7;
  return e == 0 ? static_cast<float>(m) * pow2i(-9) : static_cast<float>(8 + m) * pow2i(e - 10);
}

__device__ __forceinline__ float candidate_scale(int k, float g) { return __fmul_rn(e4m3_value(k + 1), g); }

__device__ __forceinline__ float e2m1_grid(int j) {
  // 0, 0.5, 1, 1.5, 2, 3, 4, 6
  return j < 5 ? 0.5f * static_cast<float>(j) : (j == 5 ? 3.f : (j == 6 ? 4.f : 6.f));
}

// fp16 bit pattern of e2m1_grid(j).
__device__ __forceinline__ uint32_t e2m1_grid_f16_bits(int j) {
  return j == 0 ? 0u : (j == 1 ? 0x3800u : 0x3800u + 0x200u * static_cast<uint32_t>(j));
}

__device__ __forceinline__ float e2m1_lower_midpoint(int j) {
  // Midpoint between grid[j - 1] and grid[j]: 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.
  return 0.5f * (e2m1_grid(j - 1) + e2m1_grid(j));
}

__device__ __forceinline__ float next_up(float x) {  // x >= 0, finite
  return __uint_as_float(__float_as_uint(x) + 1u);
}

// The smallest fp32 magnitude whose exact quotient by s rounds to a level >= j (j >= 1);
// 0 for j == 0. Computed from the exact residual of the midpoint product, so ties and
// near-ties are decided as on the exact quotient; ties go to the even code (up for even j).
__device__ __forceinline__ float level_threshold(int j, float s) {
  if (j == 0) return 0.f;
  const float m = e2m1_lower_midpoint(j);
  const float prod = __fmul_rn(m, s);
  const float resid = __fmaf_rn(m, s, -prod);  // exact m*s - prod
  const bool tie_up = (j & 1) == 0;
  return (resid < 0.f || (resid == 0.f && tie_up)) ? prod : next_up(prod);
}

}  // namespace lhcal
