// NVFP4 fake quant of bf16 activations: the input quantizer whose output X_q the
// activation-aware capture records ("Add activation-aware local Hessian scale calibration",
// PR #1976, re-review: the input-quantizer hook captures X_q next to the raw X).
//
// Per (token, 16-wide block along cin), with the per-tensor global scale gx (fp32):
//   code c = E4M3(amax_blk / (6 gx)) on the exact quotient: nearest, ties to the even code,
//            saturating at 448 (code 126); code 0 (zero) gives a zero block;
//   s      = fp32(v_c * gx);
//   X_q    = bf16(fp32(q * s)) with the sign of x, q = E2M1(|x| / s) on the exact quotient
//            (nearest, ties to even, clamped at 6).
//
// Both decisions are taken by comparing bf16 bit patterns with exact thresholds: a
// non-negative bf16 value a reaches code >= k iff a >= bound[k], and level >= j + 1 iff
// a >= T_j, where each threshold is the smallest bf16 value on the upper side of the exact
// midpoint (on a tie, the side of the even code). The products behind the thresholds are
// exact in fp64 (at most 31 significant bits), so every rounding decision is the exact one.
// Because gx is one scalar per tensor, the thresholds and level values of all 127 codes fit
// in one 8.6 KB table that each CTA builds in shared memory once.
//
// Level selection, two exact forms. Step sum (act_quant_steps(gx)): with step_j = 1.0 when
// |x| >= T_j (bf16 compare) the value is the sum of step_j * dV_j, dV_j = V_{j+1} - V_j, in
// bf16 FMAs on the FP16/FMA pipe. Consecutive level values are within a factor 2 of each
// other, so every dV_j and every partial sum V_j is exact in bf16 while the values are normal
// numbers, which 2^-100 <= gx <= 2^100 guarantees. Outside that range each compare yields a
// mask that selects V_{j+1} (integer logic); the table then holds V_j instead of dV_j.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "quant_tables.cuh"

namespace lhcal {

struct ActQuantTables {
  // bound[k], k = 1..126: bf16 bits of the smallest |x| whose code is >= k; bound[0] = 0 and
  // bound[127] = +inf (no code above 126).
  uint32_t bound[128];
  // Per code c: words 0..6 = thresholds T_0..T_6 of E2M1 levels 1..7; words 7..13 = dV_0..dV_6
  // (step sum) or the bf16 values V_1..V_7 of levels 1..7 (select), V = bf16(fp32(q s)); each
  // bf16 repeated in both halves of the word.
  uint4 lev[127][4];
};

// Smallest bf16 value >= t (t >= 0), as bits; +inf (0x7F80) if t exceeds the largest bf16.
__device__ __forceinline__ uint32_t bf16_ceil_bits(double t) {
  uint32_t b = __float_as_uint(__double2float_ru(t));  // smallest fp32 >= t
  if (b & 0xFFFFu) b += 0x10000u;                        // then the smallest bf16 >= that
  return b >> 16;
}

// Smallest bf16 a with a > t, or a >= t when a tie at t goes up.
__device__ __forceinline__ uint32_t bf16_threshold(double t, bool up_on_tie) {
  uint32_t b = bf16_ceil_bits(t);
  if (!up_on_tie && b < 0x7F80u && static_cast<double>(__uint_as_float(b << 16)) == t) b += 1;
  return b;
}

__device__ __forceinline__ float e4m3_value_or_zero(int code) { return code == 0 ? 0.f : e4m3_value(code); }

// Whether the step-sum form is exact for global scale gx (all level values normal numbers).
__device__ __forceinline__ bool act_quant_steps(float gx) { return gx >= 0x1p-100f && gx <= 0x1p100f; }

__device__ __forceinline__ float act_level_value(int j, float s) {  // bf16(fp32(q_j s)), as fp32
  return __bfloat162float(__float2bfloat16_rn(__fmul_rn(e2m1_grid(j), s)));
}

// Fills the tables for global scale gx; every thread of the block takes part. The caller
// synchronises before use.
__device__ inline void build_act_tables(ActQuantTables& t, float gx, int tid, int nthreads) {
  const double g = static_cast<double>(gx);
  const bool steps = act_quant_steps(gx);
  for (int k = tid; k < 128; k += nthreads) {
    uint32_t b;
    if (k == 0) {
      b = 0;
    } else if (k == 127) {
      b = 0x7F80u;
    } else {
      // Midpoint of codes k-1 and k (5 significant bits) times 6 gx: exact in fp64. On a tie
      // the even code wins, so reaching code k on the tie needs k even.
      const double mid = 0.5 * (static_cast<double>(e4m3_value_or_zero(k - 1)) + static_cast<double>(e4m3_value(k)));
      b = bf16_threshold(mid * 6.0 * g, (k & 1) == 0);
    }
    t.bound[k] = b;
  }
  uint32_t* words = reinterpret_cast<uint32_t*>(t.lev);
  for (int i = tid; i < 127 * 16; i += nthreads) {
    const int c = i >> 4, j = i & 15;
    const float s = __fmul_rn(e4m3_value_or_zero(c), gx);
    uint32_t h = 0;
    if (j < 7) {
      // Midpoint between E2M1 levels j and j + 1; the tie goes up when level j + 1 is even.
      h = bf16_threshold(static_cast<double>(e2m1_lower_midpoint(j + 1)) * static_cast<double>(s), (j & 1) == 1);
    } else if (j < 14) {
      const float v = act_level_value(j - 6, s);  // V_{j-6}, j - 6 = 1..7
      // dV = V_{j-6} - V_{j-7}: exact in fp32 and in bf16 (Sterbenz, normal values).
      h = __bfloat16_as_ushort(__float2bfloat16_rn(steps ? v - act_level_value(j - 7, s) : v));
    }
    words[i] = h | (h << 16);
  }
}

// Block scale code of a block whose largest magnitude has bf16 bits amax. The hardware E4M3
// conversion of an approximate quotient gives a first guess; the exact bounds then settle it.
// With steps (2^-100 <= gx <= 2^100, so 6 gx and its reciprocal are normal fp32 numbers) the
// guess carries a relative error below 2^-22 while neighbouring code midpoints are at least
// 2^-4 apart (2^-9 absolute below 2^-6), so it is off by at most one code and one pair of
// bound loads settles it; otherwise bounded walks do.
__device__ __forceinline__ int act_scale_code(uint32_t amax, float inv6gx, const ActQuantTables& t, bool steps) {
  const float r = fminf(__uint_as_float(amax << 16) * inv6gx, 448.f);  // a NaN guess becomes 448
  int c = static_cast<int>(__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3) & 0x7F);
  c = c > 126 ? 126 : c;
  if (steps) {
    const uint32_t lo = t.bound[c], hi = t.bound[c + 1];
    return c + (amax >= hi ? 1 : 0) - (amax < lo ? 1 : 0);
  }
  while (c < 126 && amax >= t.bound[c + 1]) ++c;
  while (c > 0 && amax < t.bound[c]) --c;
  return c;
}

// |x| of a 16-value block (8 words of bf16 pairs) and its scale code.
__device__ __forceinline__ int act_block_code(const uint32_t (&x)[8], uint32_t (&a)[8], float inv6gx,
                                              const ActQuantTables& t, bool steps) {
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = x[i] & 0x7FFF7FFFu;  // |x|
  // Largest |x| of the block: bf16x2 max (exact, no NaN here); non-negative bf16 values order
  // like their bit patterns, so the two halves finish with an integer max.
  __nv_bfloat162 m2 = *reinterpret_cast<const __nv_bfloat162*>(&a[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&a[i]));
  const uint32_t m = *reinterpret_cast<const uint32_t*>(&m2);
  return act_scale_code(max(m & 0xFFFFu, m >> 16), inv6gx, t, steps);
}

// X_q of the block from |x| (a), the signs (x) and the block's scale code c.
__device__ __forceinline__ void act_block_apply(const uint32_t (&x)[8], const uint32_t (&a)[8], int c,
                                                uint32_t (&q)[8], const ActQuantTables& t, bool steps) {
  const uint4 w0 = t.lev[c][0], w1 = t.lev[c][1], w2 = t.lev[c][2], w3 = t.lev[c][3];
  const uint32_t thr[7] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z};
  const uint32_t val[7] = {w1.w, w2.x, w2.y, w2.z, w2.w, w3.x, w3.y};
  if (steps) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 ai = *reinterpret_cast<const __nv_bfloat162*>(&a[i]);
      __nv_bfloat162 o = __float2bfloat162_rn(0.f);
#pragma unroll
      for (int j = 0; j < 7; ++j) {  // o = V_0 + dV_0 + ... up to the level reached: exact
        const __nv_bfloat162 st = __hge2(ai, *reinterpret_cast<const __nv_bfloat162*>(&thr[j]));
        o = __hfma2(st, *reinterpret_cast<const __nv_bfloat162*>(&val[j]), o);
      }
      q[i] = *reinterpret_cast<const uint32_t*>(&o) | (x[i] & 0x80008000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 ai = *reinterpret_cast<const __nv_bfloat162*>(&a[i]);
      uint32_t o = 0;
#pragma unroll
      for (int j = 0; j < 7; ++j) {  // levels rise with j: the last threshold met picks the value
        const uint32_t mk = __hge2_mask(ai, *reinterpret_cast<const __nv_bfloat162*>(&thr[j]));
        o = (mk & val[j]) | (~mk & o);
      }
      q[i] = o | (x[i] & 0x80008000u);
    }
  }
}

// Fake-quantizes one 16-value block held as 8 words of bf16 pairs. steps must be
// act_quant_steps(gx) of the gx the tables were built for.
__device__ __forceinline__ void act_quant_block(const uint32_t (&x)[8], uint32_t (&q)[8], float inv6gx,
                                                const ActQuantTables& t, bool steps) {
  uint32_t a[8];
  const int c = act_block_code(x, a, inv6gx, t, steps);
  act_block_apply(x, a, c, q, t, steps);
}

}  // namespace lhcal
