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
#include "quant_tables.cuh"

namespace lhcal {
namespace {

constexpr int kThreads = 128;

// Candidate table for one global scale g, interleaved per (candidate k, level j):
// tab[2 * (8k + j)] = thr[k][j], tab[2 * (8k + j) + 1] = val[k][j] (see file comment).
__device__ void build_tables(float* tab, float g) {
  for (int idx = threadIdx.x; idx < kCand * kLev; idx += blockDim.x) {
    const int k = idx >> 3, j = idx & 7;
    const float s = candidate_scale(k, g);
    tab[2 * idx] = level_threshold(j, s);
    tab[2 * idx + 1] = __fmul_rn(e2m1_grid(j), s);
  }
}

// Level of magnitude a for candidate row tab_k (interleaved table), by counting thresholds.
__device__ __forceinline__ int level_direct(const float* tab_k, float a) {
  int lev = 0;
#pragma unroll
  for (int j = 1; j < kLev; ++j) lev += (a >= tab_k[2 * j]) ? 1 : 0;
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

// Packed weights of the quadratic form for row-pair evaluation with f32x2 FMAs.
// Row i of the upper triangle (diagonal H_ii, off-diagonal (H_ij + H_ji) s_i s_j for j > i) is
// stored as column pairs p = i/2 .. 7 (columns 2p, 2p+1); for odd i the first pair carries a
// zero for column i-1. 72 pairs in total, row 2q and row 2q+1 both starting at pair q.
constexpr int kPairs = 72;

__device__ __forceinline__ int row_first_slot(int i) {  // slot of row i's first pair
  // Rows 0..i-1 use 8 - (r >> 1) pairs each.
  int n = 0;
#pragma unroll
  for (int r = 0; r < 16; ++r)
    if (r < i) n += 8 - (r >> 1);
  return n;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Loss of one candidate from its dequantized errors e2 (pairs of |wq| - |w|).
template <int MODE>
__device__ __forceinline__ float candidate_loss(const float2 (&e2)[kBlock / 2], const float2* wp,
                                                const float2 (&c2p)[kBlock / 2]) {
  float2 lacc = make_float2(0.f, 0.f), lacc1 = make_float2(0.f, 0.f);
  if (MODE == LHCAL_DIAG) {
#pragma unroll
    for (int q = 0; q < kBlock / 2; q += 2) {
      lacc = __ffma2_rn(__fmul2_rn(wp[q], e2[q]), e2[q], lacc);
      lacc1 = __ffma2_rn(__fmul2_rn(wp[q + 1], e2[q + 1]), e2[q + 1], lacc1);
    }
  } else {
#pragma unroll
    for (int q = 0; q < kBlock / 2; ++q) {  // rows 2q and 2q+1
      const int sa = row_first_slot(2 * q), sb = row_first_slot(2 * q + 1);
      float2 ra = __fmul2_rn(wp[sa], e2[q]);
      float2 rb = __fmul2_rn(wp[sb], e2[q]);
#pragma unroll
      for (int c = q + 1; c < 8; ++c) {
        ra = __ffma2_rn(wp[sa + c - q], e2[c], ra);
        rb = __ffma2_rn(wp[sb + c - q], e2[c], rb);
      }
      float2 t = make_float2(ra.x + ra.y, rb.x + rb.y);
      if (MODE == LHCAL_ACT_AWARE) t = __fadd2_rn(t, c2p[q]);
      if (q & 1) lacc1 = __ffma2_rn(t, e2[q], lacc1); else lacc = __ffma2_rn(t, e2[q], lacc);
    }
  }
  lacc = __fadd2_rn(lacc, lacc1);
  return lacc.x + lacc.y;
}

template <int MODE, typename WT>
__global__ void __launch_bounds__(kThreads, 2)
sweep_kernel(const WT* __restrict__ w, int64_t rows, int64_t cin, const float* __restrict__ h,
             const float* __restrict__ p, const float* __restrict__ g, uint8_t* __restrict__ codes,
             float* __restrict__ wq, float* __restrict__ loss) {
  __shared__ __align__(16) float tab_s[2 * kCand * kLev];
  __shared__ float h_s[256];
  __shared__ float p_s[256];

  const int64_t nblk = cin / kBlock;
  const int64_t n = blockIdx.y;
  const int64_t e = blockIdx.z;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;

  build_tables(tab_s, __ldg(g + e));
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
  float2 na2[kBlock / 2];  // -|w|, pairs
  uint32_t neg = 0;        // bit i: w_i has its sign bit set
#pragma unroll
  for (int i = 0; i < kBlock; i += 2) na2[i / 2] = make_float2(-fabsf(wv[i]), -fabsf(wv[i + 1]));
#pragma unroll
  for (int i = 0; i < kBlock; ++i) neg |= (__float_as_uint(wv[i]) >> 31) << i;

  float2 wp[MODE == LHCAL_DIAG ? kBlock / 2 : kPairs];  // packed loss weights
  float2 c2p[kBlock / 2];                               // ACT: 2 s_i (P w)_i, pairs
  if (MODE == LHCAL_DIAG) {
#pragma unroll
    for (int q = 0; q < kBlock / 2; ++q) wp[q] = make_float2(h_s[2 * q], h_s[2 * q + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < kBlock; ++i) {
      const int s0 = row_first_slot(i);
#pragma unroll
      for (int q = i >> 1; q < 8; ++q) {
        float c[2];
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const int j = 2 * q + b;
          if (j < i) {
            c[b] = 0.f;
          } else if (j == i) {
            c[b] = h_s[i * 17];
          } else {
            const float v = h_s[i * 16 + j] + h_s[j * 16 + i];
            c[b] = __uint_as_float(__float_as_uint(v) ^ ((((neg >> i) ^ (neg >> j)) & 1u) << 31));
          }
        }
        wp[s0 + q - (i >> 1)] = make_float2(c[0], c[1]);
      }
    }
    if (MODE == LHCAL_ACT_AWARE) {
      float c2[kBlock];
#pragma unroll
      for (int i = 0; i < kBlock; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < kBlock; ++j) acc = fmaf(p_s[i * 16 + j], wv[j], acc);
        c2[i] = __uint_as_float(__float_as_uint(2.f * acc) ^ (((neg >> i) & 1u) << 31));
      }
#pragma unroll
      for (int q = 0; q < kBlock / 2; ++q) c2p[q] = make_float2(c2[2 * q], c2[2 * q + 1]);
    }
  }

  float best = __int_as_float(0x7f800000);  // +inf
  int best_k = 0;
  auto consider = [&](const float2 (&e2)[kBlock / 2], int k) {
    const float L = candidate_loss<MODE>(e2, wp, c2p);
    if (L < best) {
      best = L;
      best_k = k;
    }
  };

  // Candidates 0..2: levels by counting thresholds (consecutive scales there differ by up to 2x).
  const uint32_t tab_base = smem_addr(tab_s);
  uint32_t addr[kBlock];  // shared address of tab[k][level] for the current k, per element
#pragma unroll 1
  for (int k = 0; k < 3; ++k) {
    const float* tab_k = tab_s + 2 * kLev * k;
    float2 e2[kBlock / 2];
#pragma unroll
    for (int q = 0; q < kBlock / 2; ++q) {
      const int l0 = level_direct(tab_k, -na2[q].x), l1 = level_direct(tab_k, -na2[q].y);
      addr[2 * q] = tab_base + 8u * static_cast<uint32_t>(kLev * k + l0);
      addr[2 * q + 1] = tab_base + 8u * static_cast<uint32_t>(kLev * k + l1);
      e2[q] = __fadd2_rn(make_float2(tab_k[2 * l0 + 1], tab_k[2 * l1 + 1]), na2[q]);
    }
    consider(e2, k);
  }
  // Candidates 3..125: the level falls by at most one per step; the step's table row is an
  // immediate offset from each element's address, which moves on every third candidate.
  constexpr int kRow = 8 * kLev;  // bytes per candidate row
#pragma unroll 1
  for (int k = 3; k < kCand; k += 3) {
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
          if (u == 0) t = lds_f32<kRow>(addr[i]);
          else if (u == 1) t = lds_f32<2 * kRow>(addr[i]);
          else t = lds_f32<3 * kRow>(addr[i]);
          addr[i] -= (a < t) ? 8u : 0u;
          if (u == 0) v[b] = lds_f32<kRow + 4>(addr[i]);
          else if (u == 1) v[b] = lds_f32<2 * kRow + 4>(addr[i]);
          else v[b] = lds_f32<3 * kRow + 4>(addr[i]);
        }
        e2[q] = __fadd2_rn(make_float2(v[0], v[1]), na2[q]);
      }
      consider(e2, k + u);
    }
#pragma unroll
    for (int i = 0; i < kBlock; ++i) addr[i] += 3 * kRow;
  }

  codes[unit] = static_cast<uint8_t>(best_k + 1);
  if (loss != nullptr) loss[unit] = best;
  if (wq != nullptr) {
    const float* tab_k = tab_s + 2 * kLev * best_k;
    float outv[kBlock];
#pragma unroll
    for (int i = 0; i < kBlock; ++i) {
      const float a = -(i & 1 ? na2[i / 2].y : na2[i / 2].x);
      outv[i] = __uint_as_float(__float_as_uint(tab_k[2 * level_direct(tab_k, a) + 1]) | (((neg >> i) & 1u) << 31));
    }
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
  // FULL and ACT_AWARE: quadratic form on tensor cores; DIAG: FP32 weighted sum.
  if (mode == LHCAL_FULL || mode == LHCAL_ACT_AWARE)
    return launch_sweep_tc(mode, dtype, w, groups, rows, cin, h, p, g, codes, wq, loss, stream);
#define LHCAL_SWEEP_CASE(M, T)                                                                   \
  return launch_mode<M, T>(w, groups, rows, cin, h, p, g, codes, wq, loss, stream)
  if (mode == LHCAL_DIAG) {
    if (dtype == LHCAL_BF16) LHCAL_SWEEP_CASE(LHCAL_DIAG, __nv_bfloat16);
    LHCAL_SWEEP_CASE(LHCAL_DIAG, float);
  }
#undef LHCAL_SWEEP_CASE
  return fail(LHCAL_ERR_UNSUPPORTED, "scale sweep: unsupported mode/dtype");
}

}  // namespace lhcal
