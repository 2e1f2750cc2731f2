// Amax-multiplier search: the non-sweep block-scale search of the MSE calibrator that "add local
// hessian calibration" (PR #788) configures by step size and multipliers, with the losses of the
// 126-candidate sweep (FULL, activation-aware, DIAG, and MSE = H = I).
//
// For each unit (group e, row r, block n) and each caller multiplier m_i in order: the candidate
// amax fp32(m_i * amax_blk) becomes the NVFP4 block scale the quantizer would use, the E4M3 code
// c_i nearest to amax / (6 g) (exact quotient, ties to the even code, saturating at 448; 0 is a
// zero scale), and the unit is scored at s = fp32(v_c g). The first multiplier with the smallest
// loss wins. A multiplier whose code equals the previous one's has the same loss and is skipped.
//
// One thread per unit; a CTA covers 128 rows of one block, with H (or Imp), P and the
// multipliers in shared memory. The losses are evaluated by their definitions in fp32. This is
// a generic kernel: a few dozen multipliers collapse onto a few distinct codes per unit.
#include "common.cuh"
#include "quant_tables.cuh"

#include <cuda_fp8.h>

namespace lhcal {
namespace {

constexpr int kMsThreads = 128;

struct __align__(16) MsShared {
  float h[256];  // FULL/ACT: H of the block; DIAG: Imp in the first 16 (rows read 16 bytes at a time)
  float p[256];  // ACT: P of the block
  float mult[kMaxMultipliers];
};

__device__ __forceinline__ float e4m3_value_or_zero_ms(int code) { return code == 0 ? 0.f : e4m3_value(code); }

// Whether a (>= 0) reaches code k (1..126) of the E4M3 rounding of a / (6 g): a above the exact
// midpoint of codes k-1 and k times 6 g (exact in fp64: at most 31 significant bits), or on it
// with k even.
__device__ __forceinline__ bool reaches_code(float a, int k, double g6) {
  const double t = 0.5 * (static_cast<double>(e4m3_value_or_zero_ms(k - 1)) + static_cast<double>(e4m3_value(k))) * g6;
  const double ad = static_cast<double>(a);
  return ad > t || (ad == t && (k & 1) == 0);
}

// Exact E4M3 code of a / (6 g) for a >= 0 (possibly +inf) and g > 0. A first guess from the
// hardware conversion of an approximate fp32 quotient, then bounded exact walks.
__device__ __forceinline__ int e4m3_code_of(float a, float g) {
  const float r = fminf(a / (6.f * g), 448.f);  // NaN (from inf / inf) becomes 448
  int c = static_cast<int>(__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3) & 0x7F);
  c = c > 126 ? 126 : c;
  const double g6 = 6.0 * static_cast<double>(g);
  while (c < 126 && reaches_code(a, c + 1, g6)) ++c;
  while (c > 0 && !reaches_code(a, c, g6)) --c;
  return c;
}

// Four entries of a shared-memory row. volatile: H is read again for every evaluated scale
// rather than hoisted out of the multiplier loop into 256 registers (which left one CTA's worth
// of warps per SM).
__device__ __forceinline__ float4 lds_row4(const float* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
  return v;
}

template <int MODE>
__device__ __forceinline__ float unit_loss(const float (&w)[16], const float (&pw)[16], float s,
                                           const MsShared& sh, float (&wq)[16]) {
  float thr[kLev], val[kLev];
#pragma unroll
  for (int j = 1; j < kLev; ++j) {
    thr[j] = level_threshold(j, s);
    val[j] = __fmul_rn(e2m1_grid(j), s);
  }
  float dw[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = fabsf(w[i]);
    float m = 0.f;
#pragma unroll
    for (int j = 1; j < kLev; ++j) m = a >= thr[j] ? val[j] : m;
    wq[i] = copysignf(m, w[i]);
    dw[i] = wq[i] - w[i];
  }
  float L = 0.f;
  if (MODE == LHCAL_MSE) {
#pragma unroll
    for (int i = 0; i < 16; ++i) L = fmaf(dw[i], dw[i], L);
  } else if (MODE == LHCAL_DIAG) {
#pragma unroll
    for (int i = 0; i < 16; ++i) L = fmaf(sh.h[i] * dw[i], dw[i], L);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float r = 0.f;
#pragma unroll
      for (int j = 0; j < 16; j += 4) {  // row i of H, in column order
        const float4 hq = lds_row4(sh.h + i * 16 + j);
        r = fmaf(hq.x, dw[j], r);
        r = fmaf(hq.y, dw[j + 1], r);
        r = fmaf(hq.z, dw[j + 2], r);
        r = fmaf(hq.w, dw[j + 3], r);
      }
      L = fmaf(dw[i], r, L);
      if (MODE == LHCAL_ACT_AWARE) L = fmaf(2.f * dw[i], pw[i], L);
    }
  }
  return L;
}

template <int MODE, typename WT>
__global__ void __launch_bounds__(kMsThreads)
msearch_kernel(const WT* __restrict__ w, int64_t rows, int64_t cin, const float* __restrict__ h,
               const float* __restrict__ p, const float* __restrict__ g, const float* __restrict__ mult,
               int n_mult, uint8_t* __restrict__ codes, float* __restrict__ wq_out, float* __restrict__ loss) {
  __shared__ MsShared sh;
  const int64_t nblk = cin / kBlock;
  const int64_t n = blockIdx.y;
  const int64_t e = blockIdx.z;
  const int64_t hblk = e * nblk + n;
  if (MODE == LHCAL_DIAG) {
    if (threadIdx.x < kBlock) sh.h[threadIdx.x] = __ldg(h + hblk * kBlock + threadIdx.x);
  } else if (MODE != LHCAL_MSE) {
    for (int i = threadIdx.x; i < 256; i += kMsThreads) {
      sh.h[i] = __ldg(h + hblk * 256 + i);
      if (MODE == LHCAL_ACT_AWARE) sh.p[i] = __ldg(p + hblk * 256 + i);
    }
  }
  for (int i = threadIdx.x; i < n_mult; i += kMsThreads) sh.mult[i] = __ldg(mult + i);
  __syncthreads();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kMsThreads + threadIdx.x;
  if (row >= rows) return;
  const int64_t unit = (e * rows + row) * nblk + n;
  float wv[16];
  load8<WT>(w + (e * rows + row) * cin + n * kBlock, wv);
  load8<WT>(w + (e * rows + row) * cin + n * kBlock + 8, wv + 8);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(wv[i]));
  float pw[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float r = 0.f;
    if (MODE == LHCAL_ACT_AWARE) {
#pragma unroll
      for (int j = 0; j < 16; ++j) r = fmaf(sh.p[i * 16 + j], wv[j], r);
    }
    pw[i] = r;
  }
  const float gs = __ldg(g + e);
  float best = __int_as_float(0x7f800000);
  int best_c = 0, prev = -1;
  for (int i = 0; i < n_mult; ++i) {
    float am = __fmul_rn(sh.mult[i], amax);
    am = am >= 0.f ? am : 0.f;  // negative or NaN counts as 0
    const int c = gs > 0.f ? e4m3_code_of(am, gs) : 0;
    if (c == prev) continue;  // same scale, same loss: the earlier multiplier keeps it
    prev = c;
    float wq[16];
    const float L = unit_loss<MODE>(wv, pw, __fmul_rn(e4m3_value_or_zero_ms(c), gs), sh, wq);
    if (L < best) {
      best = L;
      best_c = c;
    }
  }
  codes[unit] = static_cast<uint8_t>(best_c);
  if (loss) loss[unit] = best;
  if (wq_out) {
    float wq[16];
    (void)unit_loss<MODE>(wv, pw, __fmul_rn(e4m3_value_or_zero_ms(best_c), gs), sh, wq);
    float4* dst = reinterpret_cast<float4*>(wq_out + unit * kBlock);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_float4(wq[4 * q], wq[4 * q + 1], wq[4 * q + 2], wq[4 * q + 3]);
  }
}

template <int MODE>
lhcal_status launch_ms(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows, int64_t cin, const float* h,
                       const float* p, const float* g, const float* mult, int32_t n_mult, uint8_t* codes, float* wq,
                       float* loss, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(ceil_div(rows, kMsThreads)), static_cast<unsigned>(cin / kBlock),
                  static_cast<unsigned>(groups));
  if (dtype == LHCAL_BF16)
    msearch_kernel<MODE, __nv_bfloat16><<<grid, kMsThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(w), rows, cin, h, p, g, mult, n_mult, codes, wq, loss);
  else
    msearch_kernel<MODE, float><<<grid, kMsThreads, 0, stream>>>(static_cast<const float*>(w), rows, cin, h, p, g,
                                                                 mult, n_mult, codes, wq, loss);
  return check_launch("multiplier search");
}

}  // namespace

lhcal_status launch_multiplier_search(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows,
                                      int64_t cin, const float* h, const float* p, const float* g, const float* mult,
                                      int32_t n_mult, uint8_t* codes, float* wq, float* loss, cudaStream_t stream) {
  switch (mode) {
    case LHCAL_FULL:
      return launch_ms<LHCAL_FULL>(dtype, w, groups, rows, cin, h, p, g, mult, n_mult, codes, wq, loss, stream);
    case LHCAL_ACT_AWARE:
      return launch_ms<LHCAL_ACT_AWARE>(dtype, w, groups, rows, cin, h, p, g, mult, n_mult, codes, wq, loss, stream);
    case LHCAL_DIAG:
      return launch_ms<LHCAL_DIAG>(dtype, w, groups, rows, cin, h, p, g, mult, n_mult, codes, wq, loss, stream);
    default:
      return launch_ms<LHCAL_MSE>(dtype, w, groups, rows, cin, h, p, g, mult, n_mult, codes, wq, loss, stream);
  }
}

}  // namespace lhcal
