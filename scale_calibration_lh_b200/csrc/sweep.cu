// Exhaustive 126-candidate FP8 (E4M3) block-scale sweep for the WMSE (diagonal) loss, and the
// dispatch of the sweep entry point.
//
// Method: "Add WMSE weight scale search calibration" (PR #2283), What / How: importance
// Imp_i = ||X[:, i]||^2 replaces the block Hessian, the loss is sum_i Imp_i dW_i^2, and the
// kernel's DIAGONAL specialization uses a weighted sum instead of a matrix product.
// "Add activation-aware local Hessian scale calibration" (PR #1976) reviews: dW = quant(w) - w,
// best loss starts at +inf. FULL and activation-aware losses run in sweep_tc.cu. The plain
// block MSE (LHCAL_MSE, H = I: the "mse" method next to which "Add WMSE weight scale search
// calibration" fingerprints local_hessian) is this kernel with every importance 1.
//
// Design (sm_100a, FP32 pipe):
//  * One thread owns one unit (group e, row r, block n); a CTA covers 128 rows of one block.
//  * Exact fake quantization without a divide (quant_tables.cuh): per-candidate threshold and
//    value tables in shared memory; from the 4th candidate on each element's E2M1 level falls
//    by at most one per candidate, so one shared-memory compare per element and candidate
//    replaces the rounding. Each element keeps a shared-memory address into the interleaved
//    {threshold, value} table that a level drop lowers by one entry; the candidate row is an
//    immediate offset in a loop unrolled by three.
//  * While all 16 weights of a unit sit at the top grid level (6), its loss is the parabola
//    36 s^2 sum Imp - 12 s sum Imp |w| + sum Imp w^2. The CTA stages its rows' weights in
//    shared memory and orders the rows by their first unclamped candidate (a stable counting
//    sort, row_order.cuh), so that each warp's units leave that regime together; below the
//    warp's first candidate with an unclamped element the parabola gives the loss.
//  * Loss: packed f32x2 products, L = sum_i Imp_i (|wq_i| - |w_i|)^2.
#include <cstddef>

#include <cuda_fp8.h>

#include "common.cuh"
#include "quant_tables.cuh"
#include "row_order.cuh"

namespace lhcal {
namespace {

constexpr int kThreads = 128;
constexpr int kRowBytes = 8 * kLev;  // {thr, val} float2 entries per candidate

constexpr int kWStride = kBlock + 4;  // floats per staged weight row (16-byte aligned rows)

struct __align__(16) DiagShared {
  float2 tab[kCand * kLev];  // .x threshold, .y fake-quant value, per (candidate, level)
  alignas(16) float wall[kThreads][kWStride];  // the CTA's rows' weights (fp32)
  float imp[kBlock];
  int kfirst[kThreads];  // per row: first candidate with an element below the top level
  int perm[kThreads];    // rows in ascending kfirst (row_order.cuh)
  int kf_sorted[kThreads];
  int hist[4][kOrderRows];
  int base[kOrderRows];
};
static_assert(kThreads == kOrderRows, "one row per thread");
static_assert(offsetof(DiagShared, wall) % 16 == 0, "16-byte shared-memory accesses need aligned rows");

// Level of magnitude a at candidate row tab_k, by counting thresholds.
__device__ __forceinline__ int level_direct(const float2* tab_k, float a) {
  int lev = 0;
#pragma unroll
  for (int j = 1; j < kLev; ++j) lev += (a >= tab_k[j].x) ? 1 : 0;
  return lev;
}

template <int OFF>
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1+%2];\n" : "=f"(v) : "r"(addr), "n"(OFF));
  return v;
}

template <typename WT>
__device__ __forceinline__ void load_w16(const WT* src, float* w) {
  load8<WT>(src, w);
  load8<WT>(src + 8, w + 8);
}

template <typename WT>
__global__ void __launch_bounds__(kThreads, 7)  // seven CTAs (28 warps) per SM: 72 registers
sweep_diag_kernel(const WT* __restrict__ w, int64_t rows, int64_t cin, const float* __restrict__ imp,  // NULL: all 1
                  const float* __restrict__ g, uint8_t* __restrict__ codes, float* __restrict__ wq,
                  float* __restrict__ loss) {
  __shared__ DiagShared sh;
  const int64_t nblk = cin / kBlock;
  const int64_t n = blockIdx.x;  // blocks fastest: neighbouring CTAs share rows (see sweep_tc.cu)
  const int64_t e = blockIdx.z;
  const int64_t rbase = static_cast<int64_t>(blockIdx.y) * kThreads;

  const float gs = __ldg(g + e);
  for (int idx = threadIdx.x; idx < kCand * kLev; idx += kThreads) {
    const int k = idx >> 3, j = idx & 7;
    const float s = candidate_scale(k, gs);
    sh.tab[idx] = make_float2(level_threshold(j, s), __fmul_rn(e2m1_grid(j), s));
  }
  if (threadIdx.x < kBlock) sh.imp[threadIdx.x] = imp ? __ldg(imp + (e * nblk + n) * kBlock + threadIdx.x) : 1.f;
  for (int i = threadIdx.x; i < 4 * kOrderRows; i += kThreads) (&sh.hist[0][0])[i] = 0;
  __syncthreads();
  // Each row: its weights staged in shared memory, and kfirst, the first candidate at which one
  // of its weights falls below the top E2M1 level; rows past the end get kCand and sort last.
  {
    const int64_t row = rbase + threadIdx.x;
    float m = __int_as_float(0x7f800000);
    float wt[kBlock];
    if (row < rows) {
      load_w16<WT>(w + (e * rows + row) * cin + n * kBlock, wt);
    } else {
#pragma unroll
      for (int i = 0; i < kBlock; ++i) wt[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < kBlock; i += 4) {
      *reinterpret_cast<float4*>(&sh.wall[threadIdx.x][i]) = make_float4(wt[i], wt[i + 1], wt[i + 2], wt[i + 3]);
      m = fminf(fminf(fabsf(wt[i]), fabsf(wt[i + 1])), fminf(fminf(fabsf(wt[i + 2]), fabsf(wt[i + 3])), m));
    }
    int lo = 0, hi = kCand;  // first k with m < thr[k][7]
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (m < sh.tab[kLev * mid + 7].x) hi = mid; else lo = mid + 1;
    }
    const int kf = row < rows ? lo : kCand;
    sh.kfirst[threadIdx.x] = kf;
    row_order_count(kf, sh.hist);
  }
  __syncthreads();
  if (threadIdx.x < 32) row_order_scan(sh.hist, sh.base);
  __syncthreads();
  row_order_place(sh.kfirst[threadIdx.x], sh.hist, sh.base, sh.perm, sh.kf_sorted);
  __syncthreads();

  const int64_t r = rbase + sh.perm[threadIdx.x];
  const bool valid = r < rows;
  const int64_t unit = (e * rows + r) * nblk + n;
  const int64_t woff = (e * rows + (valid ? r : 0)) * cin + n * kBlock;

  float wv[kBlock];
  {
    const float* wr = sh.wall[sh.perm[threadIdx.x]];
#pragma unroll
    for (int i = 0; i < kBlock; i += 4) {
      const float4 q = *reinterpret_cast<const float4*>(wr + i);
      wv[i] = q.x; wv[i + 1] = q.y; wv[i + 2] = q.z; wv[i + 3] = q.w;
    }
  }
  float2 na2[kBlock / 2];  // -|w|, pairs
  float2 wp[kBlock / 2];   // Imp, pairs
  uint32_t neg = 0;        // bit i: w_i has its sign bit set
  float pa = 0.f, pb = 0.f, pc = 0.f;
#pragma unroll
  for (int i = 0; i < kBlock; ++i) {
    const float ai = fabsf(wv[i]), im = sh.imp[i];
    neg |= (__float_as_uint(wv[i]) >> 31) << i;
    pa += im;
    pb = fmaf(im, ai, pb);
    pc = fmaf(im * ai, ai, pc);
  }
#pragma unroll
  for (int q = 0; q < kBlock / 2; ++q) {
    na2[q] = make_float2(-fabsf(wv[2 * q]), -fabsf(wv[2 * q + 1]));
    wp[q] = make_float2(sh.imp[2 * q], sh.imp[2 * q + 1]);
  }
  pa *= 36.f;
  pb *= -12.f;

  float best = __int_as_float(0x7f800000);  // +inf
  int best_k = 0;
  auto consider = [&](const float2 (&e2)[kBlock / 2], int k) {
    float2 l0 = make_float2(0.f, 0.f), l1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < kBlock / 2; q += 2) {
      l0 = __ffma2_rn(__fmul2_rn(wp[q], e2[q]), e2[q], l0);
      l1 = __ffma2_rn(__fmul2_rn(wp[q + 1], e2[q + 1]), e2[q + 1], l1);
    }
    l0 = __fadd2_rn(l0, l1);
    const float L = l0.x + l0.y;
    if (L < best) {
      best = L;
      best_k = k;
    }
  };

  // Clamped prefix: the warp's first full candidate is the smallest kfirst of its 32 rows, the
  // first of its sorted range.
  const int kstart = sh.kf_sorted[threadIdx.x & ~31];
  // The parabola's minimum over the prefix (lowest k on equal values) is at one of the two
  // candidates that bracket its vertex s* = -pb / (2 pa), up to rounding: consecutive candidate
  // scales differ by at least 1/16 (relative), so a candidate two or more places beyond the
  // bracket exceeds the bracket's better one by at least about 0.6% of pa s*^2. With the constant
  // pc in the sum, rounding errors are a few 2^-24 of pc, so the window is taken only where
  // pa s*^2 = pb^2 / (4 pa) is at least 2^-12 pc; the candidates within two places of the E4M3
  // code of s*/g (one of the bracket's codes or next to them) then find the same minimum and
  // index as all of them. Otherwise every candidate of the prefix is evaluated.
  constexpr int kPrefixWin = 2;
  int lo = 0, hi = kstart;
  {
    const float s0 = sh.tab[2].y;  // the smallest candidate scale
    if (kstart > 2 * kPrefixWin + 1 && s0 > 0.f && pa > 0.f && pa < 0x1p100f && fabsf(pb) < 0x1p100f &&
        pc < 0x1p100f && pa * s0 * s0 >= 0x1p-100f && sh.tab[kLev * (kstart - 1) + 2].y < 0x1p40f &&
        pb * pb >= 0x1p-10f * pa * pc) {
      const float q = fmaxf(-pb / (2.f * pa), 0.f) / __ldg(g + e);  // s*/g (0 if the vertex is at s <= 0)
      const int c = static_cast<int>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3) & 0x7F);
      const int k0 = min(max(c - 1, 0), kstart - 1);  // candidate k has code k + 1
      lo = max(0, k0 - kPrefixWin);
      hi = min(kstart, k0 + kPrefixWin + 1);
    }
  }
#pragma unroll 1
  for (int k = lo; k < hi; ++k) {
    const float sk = sh.tab[kLev * k + 2].y;  // grid value 1 times s_k
    const float L = fmaf(fmaf(pa, sk, pb), sk, pc);
    if (L < best) {
      best = L;
      best_k = k;
    }
  }

  int kinc = max(kstart + 1, 3);
  kinc += (kCand - kinc) % 3;
  const uint32_t tab_base = static_cast<uint32_t>(__cvta_generic_to_shared(sh.tab));
  uint32_t addr[kBlock];  // shared address of tab[k][level] per element
#pragma unroll 1
  for (int k = kstart; k < kinc; ++k) {
    const float2* tab_k = sh.tab + kLev * k;
    float2 e2[kBlock / 2];
#pragma unroll
    for (int q = 0; q < kBlock / 2; ++q) {
      const int l0 = level_direct(tab_k, -na2[q].x), l1 = level_direct(tab_k, -na2[q].y);
      addr[2 * q] = tab_base + 8u * static_cast<uint32_t>(kLev * k + l0);
      addr[2 * q + 1] = tab_base + 8u * static_cast<uint32_t>(kLev * k + l1);
      e2[q] = __fadd2_rn(make_float2(tab_k[l0].y, tab_k[l1].y), na2[q]);
    }
    consider(e2, k);
  }
#pragma unroll 1
  for (int k = kinc; k < kCand; k += 3) {
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      float2 e2[kBlock / 2];
#pragma unroll
      for (int q = 0; q < kBlock / 2; ++q) {
        float v[2];
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const int i = 2 * q + b;
          const float a = -(b ? na2[q].y : na2[q].x);
          float t;
          if (u == 0) t = lds_f32<kRowBytes>(addr[i]);
          else if (u == 1) t = lds_f32<2 * kRowBytes>(addr[i]);
          else t = lds_f32<3 * kRowBytes>(addr[i]);
          addr[i] -= (a < t) ? 8u : 0u;
          if (u == 0) v[b] = lds_f32<kRowBytes + 4>(addr[i]);
          else if (u == 1) v[b] = lds_f32<2 * kRowBytes + 4>(addr[i]);
          else v[b] = lds_f32<3 * kRowBytes + 4>(addr[i]);
        }
        e2[q] = __fadd2_rn(make_float2(v[0], v[1]), na2[q]);
      }
      consider(e2, k + u);
    }
#pragma unroll
    for (int i = 0; i < kBlock; ++i) addr[i] += 3 * kRowBytes;
  }

  if (!valid) return;
  // The winner's loss by its definition from the fp32 fake-quant weights.
  const float2* tab_k = sh.tab + kLev * best_k;
  float outv[kBlock];
  float lw = 0.f;
#pragma unroll
  for (int i = 0; i < kBlock; ++i) {
    const float a = fabsf(wv[i]);
    const float mag = tab_k[level_direct(tab_k, a)].y;
    outv[i] = __uint_as_float(__float_as_uint(mag) | (((neg >> i) & 1u) << 31));
    const float d = mag - a;
    lw = fmaf(sh.imp[i] * d, d, lw);
  }
  codes[unit] = static_cast<uint8_t>(best_k + 1);
  if (loss != nullptr) loss[unit] = lw;
  if (wq != nullptr) {
    float4* dst = reinterpret_cast<float4*>(wq + woff);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[q] = make_float4(outv[4 * q], outv[4 * q + 1], outv[4 * q + 2], outv[4 * q + 3]);
  }
}

}  // namespace

lhcal_status launch_sweep(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups,
                          int64_t rows, int64_t cin, const float* h, const float* p, const float* g,
                          uint8_t* codes, float* wq, float* loss, cudaStream_t stream) {
  if (ceil_div(rows, kThreads) > 65535 || cin / kBlock > 65535 || groups > 65535)
    return fail(LHCAL_ERR_INVALID_ARG, "scale sweep: grid too large (rows %lld, cin %lld, groups %d)",
                (long long)rows, (long long)cin, groups);
  // FULL and ACT_AWARE: quadratic form on tensor cores; DIAG: FP32 weighted sum.
  if (mode == LHCAL_FULL || mode == LHCAL_ACT_AWARE)
    return launch_sweep_tc(mode, dtype, w, groups, rows, cin, h, p, g, codes, wq, loss, stream);
  if (mode != LHCAL_DIAG && mode != LHCAL_MSE) return fail(LHCAL_ERR_UNSUPPORTED, "scale sweep: unsupported mode");
  if (mode == LHCAL_MSE) h = nullptr;
  const dim3 grid(static_cast<unsigned>(cin / kBlock), static_cast<unsigned>(ceil_div(rows, kThreads)),
                  static_cast<unsigned>(groups));
  if (dtype == LHCAL_BF16)
    sweep_diag_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(w), rows,
                                                                     cin, h, g, codes, wq, loss);
  else
    sweep_diag_kernel<float><<<grid, kThreads, 0, stream>>>(static_cast<const float*>(w), rows, cin, h, g,
                                                             codes, wq, loss);
  return check_launch("scale sweep (diagonal)");
}

}  // namespace lhcal
