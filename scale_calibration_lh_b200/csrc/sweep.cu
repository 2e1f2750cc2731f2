// Exhaustive 126-candidate FP8 (E4M3) block-scale sweep with FP4 (E2M1) fake quantization
// and a Hessian-weighted argmin.
//
// Method: "Add WMSE weight scale search calibration" (PR #2283), "How" (126 candidate
// scales; full-Hessian and diagonal losses); "Add activation-aware local Hessian scale
// calibration" (PR #1976), "What does this PR do?" and reviews (cross term 2 dW^T (P W0),
// dW = quant(w) - w, best loss starts at +inf, negative losses allowed).
//
// Design (sm_100a, FP32 pipe bound):
//  * One thread owns one unit (group e, row r, block n) and keeps everything it needs in
//    registers: |w| (16), the sign-folded symmetric Hessian (16 diagonal + 120 doubled
//    off-diagonal terms), the current E2M1 level of each element, and dW.
//  * A CTA covers 128 rows of one block n of one group, so H_n (and P_n / Imp_n) are read
//    once per CTA through shared memory.
//  * Exact fake quantization without a divide: for each candidate k and E2M1 level j the CTA
//    precomputes, in shared memory, thr[k][j] = the smallest fp32 magnitude whose exact
//    quotient |w| / s_k rounds (nearest, ties to even) to level >= j, and
//    val[k][j] = fp32(grid[j] * s_k). The threshold comes from an exact product residual
//    (fma) so ties and near-ties are decided exactly as on the exact quotient.
//  * Candidates are visited in ascending scale. The level of an element never rises and,
//    from the 4th candidate on, consecutive scales differ by at most 4/3 while consecutive
//    E2M1 rounding midpoints differ by at least 1.4, so it falls by at most one level per
//    step: one shared-memory compare per element and candidate replaces the rounding.
//  * Loss: L = sum_i t_i e_i with t_i = H_ii e_i + sum_{j>i} (H_ij + H_ji) s_i s_j e_j (+ 2 c_i
//    for the cross term), where e_i = |wq_i| - |w_i| and s_i = sign(w_i); dW_i = s_i e_i.
#include "common.cuh"

namespace lhcal {
namespace {

constexpr int kCand = LHCAL_N_CANDIDATES;
constexpr int kLev = 8;
constexpr int kThreads = 128;

__device__ __forceinline__ float pow2i(int e) {  // exact 2^e for -126 <= e <= 127
  return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

// E4M3 value of code (1..126), exact in fp32.
__device__ __forceinline__ float e4m3_value(int code) {
  const int e = code >> 3, m = code & 7;
  return e == 0 ? static_cast<float>(m) * pow2i(-9) : static_cast<float>(8 + m) * pow2i(e - 10);
}

__device__ __forceinline__ float e2m1_grid(int j) {
  // 0, 0.5, 1, 1.5, 2, 3, 4, 6
  return j < 5 ? 0.5f * static_cast<float>(j) : (j == 5 ? 3.f : (j == 6 ? 4.f : 6.f));
}

__device__ __forceinline__ float e2m1_lower_midpoint(int j) {
  // Midpoint between grid[j - 1] and grid[j]: 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.
  return 0.5f * (e2m1_grid(j - 1) + e2m1_grid(j));
}

__device__ __forceinline__ float next_up(float x) {  // x >= 0, finite
  return __uint_as_float(__float_as_uint(x) + 1u);
}

// thr/val tables for one global scale g (see file comment).
__device__ void build_tables(float* thr, float* val, float g) {
  for (int idx = threadIdx.x; idx < kCand * kLev; idx += blockDim.x) {
    const int k = idx >> 3, j = idx & 7;
    const float s = __fmul_rn(e4m3_value(k + 1), g);
    val[idx] = __fmul_rn(e2m1_grid(j), s);
    float t = 0.f;
    if (j > 0) {
      const float m = e2m1_lower_midpoint(j);
      const float prod = __fmul_rn(m, s);
      const float resid = __fmaf_rn(m, s, -prod);  // exact m*s - prod (sign is exact)
      // Ties at the midpoint go to the even code: up for even j, down for odd j.
      const bool tie_up = (j & 1) == 0;
      // |w| >= t  <=>  |w| / s rounds to level >= j.
      t = (resid < 0.f || (resid == 0.f && tie_up)) ? prod : next_up(prod);
    }
    thr[idx] = t;
  }
}

__device__ __forceinline__ int level_direct(const float* thr_k, float a) {
  int lev = 0;
#pragma unroll
  for (int j = 1; j < kLev; ++j) lev += (a >= thr_k[j]) ? 1 : 0;
  return lev;
}

template <typename WT>
__device__ __forceinline__ void load_w16(const WT* src, float* w) {
  load8<WT>(src, w);
  load8<WT>(src + 8, w + 8);
}

template <int MODE, typename WT>
__global__ void __launch_bounds__(kThreads, 2)
sweep_kernel(const WT* __restrict__ w, int64_t rows, int64_t cin, const float* __restrict__ h,
             const float* __restrict__ p, const float* __restrict__ g, uint8_t* __restrict__ codes,
             float* __restrict__ wq, float* __restrict__ loss) {
  __shared__ float thr_s[kCand * kLev];
  __shared__ float val_s[kCand * kLev];
  __shared__ float h_s[256];
  __shared__ float p_s[256];

  const int64_t nblk = cin / kBlock;
  const int64_t n = blockIdx.y;
  const int64_t e = blockIdx.z;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;

  build_tables(thr_s, val_s, __ldg(g + e));
  const int64_t hblk = (e * nblk + n);
  if (MODE == LHCAL_DIAG) {
    if (threadIdx.x < kBlock) h_s[threadIdx.x] = __ldg(h + hblk * kBlock + threadIdx.x);
  } else {
    for (int i = threadIdx.x; i < 256; i += kThreads) {
      h_s[i] = __ldg(h + hblk * 256 + i);
      if (MODE == LHCAL_ACT_AWARE) p_s[i] = __ldg(p + hblk * 256 + i);
    }
  }
  __syncthreads();
  if (r >= rows) return;

  const int64_t unit = (e * rows + r) * nblk + n;
  const int64_t woff = (e * rows + r) * cin + n * kBlock;

  float wv[kBlock];
  load_w16<WT>(w + woff, wv);
  float a[kBlock];
  uint32_t sg[kBlock];
#pragma unroll
  for (int i = 0; i < kBlock; ++i) {
    a[i] = fabsf(wv[i]);
    sg[i] = __float_as_uint(wv[i]) & 0x80000000u;
  }

  // Sign-folded weights of the loss.
  float hd[kBlock];                    // FULL/ACT: H_ii; DIAG: Imp_i
  float ho[kBlock * (kBlock - 1) / 2];  // (H_ij + H_ji) s_i s_j, i < j
  float c2[kBlock];                    // ACT: 2 s_i (P w)_i
  if (MODE == LHCAL_DIAG) {
#pragma unroll
    for (int i = 0; i < kBlock; ++i) hd[i] = h_s[i];
  } else {
    int o = 0;
#pragma unroll
    for (int i = 0; i < kBlock; ++i) {
      hd[i] = h_s[i * 17];
#pragma unroll
      for (int j = i + 1; j < kBlock; ++j, ++o) {
        const float v = h_s[i * 16 + j] + h_s[j * 16 + i];
        ho[o] = __uint_as_float(__float_as_uint(v) ^ sg[i] ^ sg[j]);
      }
    }
    if (MODE == LHCAL_ACT_AWARE) {
#pragma unroll
      for (int i = 0; i < kBlock; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < kBlock; ++j) acc = fmaf(p_s[i * 16 + j], wv[j], acc);
        c2[i] = __uint_as_float(__float_as_uint(2.f * acc) ^ sg[i]);
      }
    }
  }

  int lev[kBlock];
  float best = __int_as_float(0x7f800000);  // +inf
  int best_k = 0;

#pragma unroll 1
  for (int k = 0; k < kCand; ++k) {
    const float* thr_k = thr_s + k * kLev;
    const float* val_k = val_s + k * kLev;
    float ev[kBlock];
    if (k < 3) {
#pragma unroll
      for (int i = 0; i < kBlock; ++i) lev[i] = level_direct(thr_k, a[i]);
    } else {
#pragma unroll
      for (int i = 0; i < kBlock; ++i) lev[i] -= (a[i] < thr_k[lev[i]]) ? 1 : 0;
    }
#pragma unroll
    for (int i = 0; i < kBlock; ++i) ev[i] = val_k[lev[i]] - a[i];

    float L;
    if (MODE == LHCAL_DIAG) {
      float l0 = 0.f, l1 = 0.f;
#pragma unroll
      for (int i = 0; i < kBlock; i += 2) {
        l0 = fmaf(hd[i] * ev[i], ev[i], l0);
        l1 = fmaf(hd[i + 1] * ev[i + 1], ev[i + 1], l1);
      }
      L = l0 + l1;
    } else {
      float l0 = 0.f, l1 = 0.f;
      int o = 0;
#pragma unroll
      for (int i = 0; i < kBlock; ++i) {
        float t = (MODE == LHCAL_ACT_AWARE) ? fmaf(hd[i], ev[i], c2[i]) : hd[i] * ev[i];
#pragma unroll
        for (int j = i + 1; j < kBlock; ++j, ++o) t = fmaf(ho[o], ev[j], t);
        if (i & 1) l1 = fmaf(t, ev[i], l1); else l0 = fmaf(t, ev[i], l0);
      }
      L = l0 + l1;
    }
    if (L < best) {
      best = L;
      best_k = k;
    }
  }

  codes[unit] = static_cast<uint8_t>(best_k + 1);
  if (loss != nullptr) loss[unit] = best;
  if (wq != nullptr) {
    const float* thr_k = thr_s + best_k * kLev;
    const float* val_k = val_s + best_k * kLev;
    float outv[kBlock];
#pragma unroll
    for (int i = 0; i < kBlock; ++i)
      outv[i] = __uint_as_float(__float_as_uint(val_k[level_direct(thr_k, a[i])]) | sg[i]);
    float4* dst = reinterpret_cast<float4*>(wq + woff);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[q] = make_float4(outv[4 * q], outv[4 * q + 1], outv[4 * q + 2], outv[4 * q + 3]);
  }
}

template <int MODE, typename WT>
lhcal_status launch_mode(const void* w, int32_t groups, int64_t rows, int64_t cin, const float* h,
                         const float* p, const float* g, uint8_t* codes, float* wq, float* loss,
                         cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(ceil_div(rows, kThreads)), static_cast<unsigned>(cin / kBlock),
                  static_cast<unsigned>(groups));
  sweep_kernel<MODE, WT><<<grid, kThreads, 0, stream>>>(static_cast<const WT*>(w), rows, cin, h, p, g,
                                                        codes, wq, loss);
  return check_launch("scale sweep");
}

}  // namespace

lhcal_status launch_sweep(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups,
                          int64_t rows, int64_t cin, const float* h, const float* p, const float* g,
                          uint8_t* codes, float* wq, float* loss, cudaStream_t stream) {
  if (rows > static_cast<int64_t>(65535) * kThreads * 1024 || cin / kBlock > 65535 || groups > 65535)
    return fail(LHCAL_ERR_INVALID_ARG, "scale sweep: grid too large (rows %lld, cin %lld, groups %d)",
                (long long)rows, (long long)cin, groups);
#define LHCAL_SWEEP_CASE(M, T)                                                                   \
  return launch_mode<M, T>(w, groups, rows, cin, h, p, g, codes, wq, loss, stream)
  if (dtype == LHCAL_BF16) {
    if (mode == LHCAL_FULL) LHCAL_SWEEP_CASE(LHCAL_FULL, __nv_bfloat16);
    if (mode == LHCAL_ACT_AWARE) LHCAL_SWEEP_CASE(LHCAL_ACT_AWARE, __nv_bfloat16);
    if (mode == LHCAL_DIAG) LHCAL_SWEEP_CASE(LHCAL_DIAG, __nv_bfloat16);
  } else {
    if (mode == LHCAL_FULL) LHCAL_SWEEP_CASE(LHCAL_FULL, float);
    if (mode == LHCAL_ACT_AWARE) LHCAL_SWEEP_CASE(LHCAL_ACT_AWARE, float);
    if (mode == LHCAL_DIAG) LHCAL_SWEEP_CASE(LHCAL_DIAG, float);
  }
#undef LHCAL_SWEEP_CASE
  return fail(LHCAL_ERR_UNSUPPORTED, "scale sweep: unsupported mode/dtype");
}

}  // namespace lhcal
