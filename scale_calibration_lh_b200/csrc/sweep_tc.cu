// Exhaustive 126-candidate FP8 scale sweep, FULL and activation-aware losses, with the
// Hessian-weighted quadratic form on tensor cores.
//
// Method: "Add WMSE weight scale search calibration" (PR #2283), How (126 candidate E4M3
// scales, full-Hessian loss); "Add activation-aware local Hessian scale calibration"
// (PR #1976), "What does this PR do?" and reviews (loss dW^T H dW + 2 dW^T (P W0),
// dW = quant(w) - w, best loss from +inf, negative losses allowed).
//
// Formulation. For candidate scale s and signed E2M1 values v = sign(w) * q (|v| in
// {0, .5, 1, 1.5, 2, 3, 4, 6}), dW = s v - w, so
//     L(s) = s^2 v^T H v - 2 s v^T U' + C',
//     U' = ((H + H^T) / 2) w - P w,   C' = w^T H w - 2 w^T P w   (P = 0 for FULL).
// U' and C' are per-unit constants. v is exact in fp16, so the matrix part v^T H (all 16
// outputs, for 16 units at once) is one m16n8k16 fp16 MMA per 8 outputs with H split into
// fp16 hi + lo, fp32 accumulation. H is first scaled by a power of two, H' = H 2^eH with the
// largest |H'| in [2^14, 2^15). Then hi = fp16(H') and lo = fp16(H' - hi) represent an entry to
// within 2^-22 of itself while lo is an fp16 normal number (|H'| >= about 2^-3, i.e. within
// 2^17 of the largest entry); smaller entries keep an absolute accuracy of about 2^-25 in H'
// units (lo reaches the fp16 subnormals), i.e. 2^-39 of the block's largest entry. Against
// |v|^T |H| |v| both are far below the fp32 rounding of the 16-term products themselves, so
// the loss differs from the fp32-rounded definition by a few 2^-23 of |w|^T |H| |w|, below the
// 1e-5 decision gaps that matter. A test runs blocks whose H diagonal spans 2^20.
//
// Mapping (mma.sync.m16n8k16, row.col, f16 -> f32): a warp evaluates 16 units (the M rows) of
// one input block for one candidate per step. Lane (g = lane / 4, t = lane % 4) owns units
// g and g + 8 and, of each, the four columns {2t, 2t+1, 2t+8, 2t+9}. Those are exactly its
// A-fragment columns and its accumulator columns, so the epilogue needs no data movement
// except a reduction over the four lanes of a quad.
//
// Quantization. As in the FP32 sweep: per-candidate threshold tables built from exact
// residuals decide the E2M1 level of every element exactly as on the exact quotient, and
// each element's level falls by at most one per candidate from the 4th on. fp32 weights: each
// table entry also carries the fp16 bits of its grid value, pre-placed for the low or the high
// half of a packed pair, so building the A fragment is one OR (and a sign XOR) per pair. bf16
// weights: the levels are tracked per pair (the two halves of an A register) on bf16 copies of
// the thresholds, which decide exactly as the fp32 ones for bf16 magnitudes: one load of the
// pair's two thresholds, one packed compare, one load of the pair's two grid values.
//
// Work per candidate. Candidates below the warp's first unclamped one take a closed form;
// the rest go four per loop trip, and the quad's four lanes share the reduction of four
// candidates (a transposed reduction: lane t ends with candidate k + t) and keep their own
// bests, merged after the loop. The argmin compares 2^eH (L - C') (C' and 2^eH are the same for
// all of a unit's candidates); the winner's loss is then recomputed by its definition.
//
// Set-up per CTA (128 rows of one block). The rows' weights are staged in shared memory once;
// each row's first unclamped candidate kfirst comes from a binary search of the top-level
// thresholds, and a stable counting sort by kfirst (match_any over each warp, per-warp
// histograms, one scan) orders the rows, so that a warp's 16 units leave the clamped regime
// together and its first full candidate is the first of its sorted range. U' and H sign(w)
// are 16-term dot products with rows of (H + H^T) / 2 read four at a time. The grid runs the
// 16-column blocks fastest.
#include <cstddef>
#include <type_traits>

#include <cuda_fp8.h>

#include "common.cuh"
#include "quant_tables.cuh"
#include "row_order.cuh"

namespace lhcal {
namespace {

// Warps per CTA (16 units each) and the CTAs per SM that the register allocation targets.
#ifndef LHCAL_TC_WARPS
#define LHCAL_TC_WARPS 8
#endif
#ifndef LHCAL_TC_MIN_BLOCKS
#define LHCAL_TC_MIN_BLOCKS 3
#endif

constexpr int kTcWarps = LHCAL_TC_WARPS;
constexpr int kTcThreads = 32 * kTcWarps;
constexpr int kUnitsPerWarp = 16;
constexpr int kUnitsPerCta = kUnitsPerWarp * kTcWarps;
constexpr int kEntryBytes = 16;                 // {thr, q16 (low half), q16 << 16, val}
constexpr int kTabRowBytes = kLev * kEntryBytes;  // one candidate

constexpr int kWStride = kBlock + 4;  // floats per staged weight row (16-byte aligned, see below)
static_assert(kTcWarps >= 5 && kUnitsPerCta == 128, "the set-up uses warps 0-4 and 4 warps of rows");

// Arrays read with 16-byte loads are declared 16-byte aligned (a member is otherwise aligned
// only to its element type); the static_asserts after the struct check the offsets.
struct __align__(16) TcShared {
  float4 tab[kCand * kLev];
  alignas(16) float h[256];
  alignas(16) float p[256];
  alignas(16) float hs[256];  // (H + H^T) / 2
  // The CTA's 128 rows' weights (fp32), row stride 20 floats (80 bytes): the 8 rows that a
  // warp's lane groups read at once with 16-byte loads then fall in distinct banks.
  alignas(16) float wall[kUnitsPerCta][kWStride];
  float rho[kCand];  // -2 / (s_k * 2^eH): scale of U' in the MMA accumulator
  float s2[kCand];   // s_k^2 (losses are compared in H' units, 2^eH times the true ones)
  float hscale;  // 2^-eH: H' = H * hscale lies below 2^15
  int kfirst[kUnitsPerCta];     // per row: first candidate with an element below the top level
  int perm[kUnitsPerCta];       // the CTA's rows in ascending kfirst (row_order.cuh)
  int kf_sorted[kUnitsPerCta];
  int hist[4][kOrderRows];
  int base[kOrderRows];
};
static_assert(offsetof(TcShared, tab) % 16 == 0 && offsetof(TcShared, h) % 16 == 0 &&
                  offsetof(TcShared, p) % 16 == 0 && offsetof(TcShared, hs) % 16 == 0 &&
                  offsetof(TcShared, wall) % 16 == 0 && (kWStride * sizeof(float)) % 16 == 0,
              "16-byte shared-memory accesses need 16-byte aligned rows");

// Pair tables (bf16 weights). A bf16 magnitude a lies below an fp32 threshold t iff it lies
// below the smallest bf16 value >= t, so the level decisions can be taken on bf16 thresholds,
// two elements per packed compare. For candidate k and an element pair at levels (l0, l1) (l0
// the A register's low half), thr2[k][8 l1 + l0] holds both elements' thresholds (bf16, l0 in
// the low half) and q2[8 l1 + l0] both grid values as fp16 bits (candidate-independent). thr16
// stages the bf16 thresholds per (k, level) so that a row of eight pairs is one 16-byte load.
constexpr int kPairs = kLev * kLev;  // 64 level pairs
constexpr int kPairRowBytes = kPairs * 4;
struct __align__(16) TcPairShared {
  uint32_t thr2[kCand * kPairs];
  uint32_t q2[kPairs];
  alignas(16) uint16_t thr16[kCand * kLev];
};
static_assert(offsetof(TcPairShared, thr16) % 16 == 0, "thr16 rows are read with 16-byte loads");

// Smallest bf16 >= x (x >= 0; +inf stays +inf), as bits.
__device__ __forceinline__ uint32_t bf16_ceil_bits(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b >> 16) + ((b & 0xffffu) != 0u ? 1u : 0u);
}

// The pair's level step at one candidate: each half of a2 (bf16 magnitudes) below its half of
// t2 (bf16 thresholds of its current level) drops that element one level, i.e. the pair index
// 8 l1 + l0 by 1 (low half) and 8 (high half): 4 and 32 bytes of the table address.
__device__ __forceinline__ void drop_pair(uint32_t& addr, uint32_t a2, uint32_t t2) {
  asm("{\n\t.reg .pred pl, ph;\n\t"
      "setp.lt.bf16x2 pl|ph, %1, %2;\n\t"
      "@pl sub.u32 %0, %0, 4;\n\t"
      "@ph sub.u32 %0, %0, 32;\n\t}\n"
      : "+r"(addr)
      : "r"(a2), "r"(t2));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <int OFF>
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1+%2];\n" : "=f"(v) : "r"(addr), "n"(OFF));
  return v;
}

template <int OFF>
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1+%2];\n" : "=r"(v) : "r"(addr), "n"(OFF));
  return v;
}

// addr - step if a < t (fp32 compare), else addr. Plain C: measured faster than an inline-asm
// predicated select, with the same codes.
__device__ __forceinline__ uint32_t drop_if_below(uint32_t addr, float a, float t, uint32_t step) {
  return a < t ? addr - step : addr;
}

__device__ __forceinline__ void mma_f16(float* d, const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

// Level of magnitude a at candidate row k of the table: the largest j with a >= thr[k][j], by a
// three-step binary search (the thresholds rise with j for s > 0; for s = 0 every level's
// value is 0, so whichever level it returns gives the same fake-quant value).
__device__ __forceinline__ int level_direct_tc(const float4* tab_k, float a) {
  int lev = (a >= tab_k[4].x) ? 4 : 0;
  lev += (a >= tab_k[lev + 2].x) ? 2 : 0;
  lev += (a >= tab_k[lev + 1].x) ? 1 : 0;
  return lev;
}

template <typename WT>
__device__ __forceinline__ void load_row16(const WT* src, bool valid, float* w) {
  if (valid) {
    load8<WT>(src, w);
    load8<WT>(src + 8, w + 8);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = 0.f;
  }
}

template <bool ACT, typename WT>
__global__ void __launch_bounds__(kTcThreads, LHCAL_TC_MIN_BLOCKS)
sweep_tc_kernel(const WT* __restrict__ w, int64_t rows, int64_t cin, const float* __restrict__ h,
                const float* __restrict__ p, const float* __restrict__ g, uint8_t* __restrict__ codes,
                float* __restrict__ wq, float* __restrict__ loss) {
  __shared__ TcShared sh;
  // bf16 weights: the pair tables, in dynamic shared memory (the launch sizes it).
  constexpr bool kPair = std::is_same<WT, __nv_bfloat16>::value;
  extern __shared__ __align__(16) uint8_t tc_dyn[];
  TcPairShared& ps = *reinterpret_cast<TcPairShared*>(tc_dyn);
  const int64_t nblk = cin / kBlock;
  // Blocks vary fastest across the grid: CTAs running together cover neighbouring blocks of the
  // same rows, so their W reads are adjacent and their codes / loss writes share DRAM sectors.
  const int64_t n = blockIdx.x;
  const int64_t e = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;

  // ---- per-CTA set-up: H (and P) of block n, its symmetric part, candidate tables
  const int64_t hblk = e * nblk + n;
  for (int i = threadIdx.x; i < 256; i += kTcThreads) {
    const float hv = __ldg(h + hblk * 256 + i);
    sh.h[i] = hv;
    sh.hs[i] = 0.5f * (hv + __ldg(h + hblk * 256 + (i & 15) * 16 + (i >> 4)));
    if (ACT) sh.p[i] = __ldg(p + hblk * 256 + i);
  }
  const float gs = __ldg(g + e);
  for (int idx = threadIdx.x; idx < kCand * kLev; idx += kTcThreads) {
    const int k = idx >> 3, j = idx & 7;
    const float s = candidate_scale(k, gs);
    const uint32_t q16 = e2m1_grid_f16_bits(j);
    const float thr = level_threshold(j, s);
    sh.tab[idx] = make_float4(thr, __uint_as_float(q16), __uint_as_float(q16 << 16), __fmul_rn(e2m1_grid(j), s));
    if (kPair) ps.thr16[idx] = static_cast<uint16_t>(bf16_ceil_bits(thr));
  }
  if (kPair && threadIdx.x < kPairs)
    ps.q2[threadIdx.x] = e2m1_grid_f16_bits(threadIdx.x & 7) | (e2m1_grid_f16_bits(threadIdx.x >> 3) << 16);
  for (int i = threadIdx.x; i < 4 * kOrderRows; i += kTcThreads) (&sh.hist[0][0])[i] = 0;
  const int64_t rbase = static_cast<int64_t>(blockIdx.y) * kUnitsPerCta;
  __syncthreads();
  // Each of the CTA's rows: weights staged in shared memory, and kfirst, the first candidate at
  // which one of its 16 weights falls below the top E2M1 level (|w| < thr[k][7]); before it the
  // unit's loss has a closed form (below). Rows past the end get kCand and sort last.
  if (threadIdx.x < kUnitsPerCta) {
    const int64_t row = rbase + threadIdx.x;
    const bool ok = row < rows;
    float wt[16];
    load_row16<WT>(w + (e * rows + (ok ? row : 0)) * cin + n * kBlock, ok, wt);
    float m = __int_as_float(0x7f800000);
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
      *reinterpret_cast<float4*>(&sh.wall[threadIdx.x][i]) = make_float4(wt[i], wt[i + 1], wt[i + 2], wt[i + 3]);
      m = fminf(fminf(fabsf(wt[i]), fabsf(wt[i + 1])), fminf(fminf(fabsf(wt[i + 2]), fabsf(wt[i + 3])), m));
    }
    int lo = 0, hi = kCand;  // first k with m < thr[k][7]
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (m < sh.tab[kLev * mid + 7].x) hi = mid; else lo = mid + 1;
    }
    const int kf = ok ? lo : kCand;
    sh.kfirst[threadIdx.x] = kf;
    row_order_count(kf, sh.hist);
  } else if (warp == 4) {
    // Scale H so that its largest |H'| lies in [2^14, 2^15): below the fp16 maximum.
    uint32_t m = 0;
    for (int i = lane; i < 256; i += 32) m = max(m, __float_as_uint(sh.h[i]) & 0x7fffffffu);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) {
      const int ex = (m == 0u) ? 0 : static_cast<int>(m >> 23) - 127;  // floor(log2 max|H|)
      sh.hscale = pow2i(min(127, max(-126, 14 - ex)));
    }
  }
  if (kPair) {
    // Row (k, l1) of the pair table: eight entries (l0 = 0..7), from the bf16 thresholds of
    // candidate k (one 16-byte load) and the threshold of level l1.
    for (int kr = threadIdx.x; kr < kCand * kLev; kr += kTcThreads) {
      const int k = kr >> 3, l1 = kr & 7;
      const uint4 t8 = *reinterpret_cast<const uint4*>(ps.thr16 + k * kLev);
      const uint32_t hi = static_cast<uint32_t>(ps.thr16[kr]) << 16;
      const uint32_t tw[4] = {t8.x, t8.y, t8.z, t8.w};
      uint32_t e[8];
#pragma unroll
      for (int l0 = 0; l0 < 8; ++l0) e[l0] = ((tw[l0 >> 1] >> (16 * (l0 & 1))) & 0xffffu) | hi;
      uint4* dst = reinterpret_cast<uint4*>(ps.thr2 + k * kPairs + l1 * kLev);
      dst[0] = make_uint4(e[0], e[1], e[2], e[3]);
      dst[1] = make_uint4(e[4], e[5], e[6], e[7]);
    }
  }
  __syncthreads();
  if (warp == 0) {
    row_order_scan(sh.hist, sh.base);
  } else if (warp == 1) {
    const float hscale = sh.hscale;
    for (int k = lane; k < kCand; k += 32) {
      const float s = candidate_scale(k, gs);
      sh.rho[k] = -2.f * hscale / s;
      sh.s2[k] = s * s;
    }
  }
  __syncthreads();
  if (threadIdx.x < kUnitsPerCta)
    row_order_place(sh.kfirst[threadIdx.x], sh.hist, sh.base, sh.perm, sh.kf_sorted);
  __syncthreads();
  const float hscale = sh.hscale;

  // ---- B fragments: H' = H * hscale as fp16 hi + lo. B[k][n] = H'[k][n].
  uint32_t bhi[2][2], blo[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int col = gq + 8 * nt;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int k0 = 2 * tq + 8 * half;
      const float x0 = sh.h[k0 * 16 + col] * hscale, x1 = sh.h[(k0 + 1) * 16 + col] * hscale;
      bhi[nt][half] = pack_f16x2(x0, x1);
      const float2 hf = unpack_f16x2(bhi[nt][half]);
      blo[nt][half] = pack_f16x2(x0 - hf.x, x1 - hf.y);
    }
  }

  // ---- the warp's 16 units: sorted positions 16 warp + gq (unit 0) and + 8 (unit 1); the
  // warp's first candidate to evaluate in full is the smallest kfirst of its units, the first
  // of its sorted range.
  const int kstart = sh.kf_sorted[warp * kUnitsPerWarp];
  // Lane element i (0..7): unit i / 4, column col_of(i % 4) with columns {2t, 2t+1, 2t+8, 2t+9}.
  auto col_of = [&](int ci) { return 2 * tq + (ci & 1) + 8 * (ci >> 1); };
  float a[8], up[8];
  uint32_t sgn[8];
  float pa[2], pb[2];
  float pwk[8];  // activation-aware: (P w)_c of each lane element, kept for the epilogue
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    // The unit's 16 weights and their signs (+-1), then per lane column c of the unit:
    // U'_c = (Hs w)_c - (P w)_c and (Hs sign(w))_c, as 16-term dot products with the rows of
    // Hs (and P) read four at a time.
    const float* wr = sh.wall[sh.perm[warp * kUnitsPerWarp + gq + 8 * u]];
    float wv[16], sv[16];
#pragma unroll
    for (int k = 0; k < 16; k += 4) {
      const float4 q = *reinterpret_cast<const float4*>(wr + k);
      wv[k] = q.x; wv[k + 1] = q.y; wv[k + 2] = q.z; wv[k + 3] = q.w;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) sv[k] = copysignf(1.f, wv[k]);
    float qa = 0.f, qb = 0.f;
#pragma unroll
    for (int ci = 0; ci < 4; ++ci) {
      const int c = col_of(ci);
      const int i = 4 * u + ci;
      const float* hr = sh.hs + c * 16;
      float hw = 0.f, hsg = 0.f, pw = 0.f;
#pragma unroll
      for (int k = 0; k < 16; k += 4) {
        const float4 hq = *reinterpret_cast<const float4*>(hr + k);
        hw = fmaf(hq.x, wv[k], hw); hw = fmaf(hq.y, wv[k + 1], hw);
        hw = fmaf(hq.z, wv[k + 2], hw); hw = fmaf(hq.w, wv[k + 3], hw);
        hsg = fmaf(hq.x, sv[k], hsg); hsg = fmaf(hq.y, sv[k + 1], hsg);
        hsg = fmaf(hq.z, sv[k + 2], hsg); hsg = fmaf(hq.w, sv[k + 3], hsg);
        if (ACT) {
          const float4 pq = *reinterpret_cast<const float4*>(sh.p + c * 16 + k);
          pw = fmaf(pq.x, wv[k], pw); pw = fmaf(pq.y, wv[k + 1], pw);
          pw = fmaf(pq.z, wv[k + 2], pw); pw = fmaf(pq.w, wv[k + 3], pw);
        }
      }
      const float x = wr[c];  // from shared memory: c depends on the lane
      const float sc = copysignf(1.f, x);
      a[i] = fabsf(x);
      sgn[i] = __float_as_uint(x) >> 31;
      up[i] = hw - pw;  // U'_c
      pwk[i] = pw;
      qa = fmaf(sc, hsg, qa);
      qb = fmaf(sc, up[i], qb);
    }
    // Over the quad: sign^T Hs sign and sign^T U'. While every element of the unit is clamped
    // at the top of the grid (v = 6 sign(w)), its scale-dependent loss is the parabola
    // 36 s^2 sign^T H sign - 12 s sign^T U'.
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      qa += __shfl_xor_sync(0xffffffffu, qa, o);
      qb += __shfl_xor_sync(0xffffffffu, qb, o);
    }
    // In H' units, as the candidate loop compares: times 2^eH (exact, a power of two).
    pa[u] = 36.f * (qa * hscale);
    pb[u] = -12.f * (qb * hscale);
  }
  if (ACT && kPair) {
    // The epilogue needs (P w)_c again. Rather than keep it in registers through the sweep, each
    // lane stores its eight values over the staged weights of its own units' rows, once every
    // lane of the warp has read those rows (only this warp reads them, and after this only the
    // writing lane reads the entries it wrote). fp32 weights recompute it in the epilogue (the
    // stored form measured a large spill in that build).
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) sh.wall[sh.perm[warp * kUnitsPerWarp + gq + 8 * (i >> 2)]][col_of(i & 3)] = pwk[i];
  }
  // Sign masks of the four packed A registers: a0 = (elems 0,1), a1 = (4,5), a2 = (2,3), a3 = (6,7).
  constexpr int kPairLo[4] = {0, 4, 2, 6};
  uint32_t smask[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) smask[r] = (sgn[kPairLo[r]] << 15) | (sgn[kPairLo[r] + 1] << 31);

  float best[2] = {__int_as_float(0x7f800000), __int_as_float(0x7f800000)};
  int best_k[2] = {0, 0};

  // U' pairs in accumulator order: d0 = (unit0 col 2t, 2t+1, unit1 col 2t, 2t+1), d1 = same at 2t+8.
  const float2 u0a = make_float2(up[0], up[1]), u0b = make_float2(up[4], up[5]);
  const float2 u1a = make_float2(up[2], up[3]), u1b = make_float2(up[6], up[7]);

  // One candidate: A fragment from the elements' packed fp16 grid values; the accumulator starts
  // at rho_k U', so after the 4 MMAs D = v^T H' + rho_k U' and
  //   s2_k * sum_n v_n D_n = 2^eH (s^2 v^T H v - 2 s v^T U') = 2^eH (L - C').
  // C' and 2^eH are the same for every candidate of a unit, so the argmin compares these values
  // (normalised to H', they stay in range whatever H's magnitude); the winner's loss is
  // recomputed by its definition after the sweep.
  // The lane's share of t for units 0 and 1 (its 4 columns), before the reduction over the quad.
  auto partials_afr = [&](const uint32_t (&afr)[4], int k, float (&tp)[2]) {
    const float rk = sh.rho[k];
    const float2 rr = make_float2(rk, rk);
    float2 c0a = __fmul2_rn(rr, u0a), c0b = __fmul2_rn(rr, u0b);
    float2 c1a = __fmul2_rn(rr, u1a), c1b = __fmul2_rn(rr, u1b);
    float d0[4] = {c0a.x, c0a.y, c0b.x, c0b.y}, d1[4] = {c1a.x, c1a.y, c1b.x, c1b.y};
    mma_f16(d0, afr, bhi[0][0], bhi[0][1]);
    mma_f16(d1, afr, bhi[1][0], bhi[1][1]);
    mma_f16(d0, afr, blo[0][0], blo[0][1]);
    mma_f16(d1, afr, blo[1][0], blo[1][1]);
    // v values as fp32: element pairs (0,1) (4,5) (2,3) (6,7).
    const float2 v01 = unpack_f16x2(afr[0]), v45 = unpack_f16x2(afr[1]);
    const float2 v23 = unpack_f16x2(afr[2]), v67 = unpack_f16x2(afr[3]);
    const float2 p0 = __ffma2_rn(v23, make_float2(d1[0], d1[1]), __fmul2_rn(v01, make_float2(d0[0], d0[1])));
    const float2 p1 = __ffma2_rn(v67, make_float2(d1[2], d1[3]), __fmul2_rn(v45, make_float2(d0[2], d0[3])));
    tp[0] = p0.x + p0.y;
    tp[1] = p1.x + p1.y;
  };
  auto partials = [&](const uint32_t (&q)[8], int k, float (&tp)[2]) {
    uint32_t afr[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) afr[r] = (q[kPairLo[r]] | q[kPairLo[r] + 1]) ^ smask[r];
    partials_afr(afr, k, tp);
  };
  auto evaluate = [&](const uint32_t (&q)[8], int k) {
    float tp[2];
    partials(q, k, tp);
    float t0 = tp[0], t1 = tp[1];
    t0 += __shfl_xor_sync(0xffffffffu, t0, 1);
    t1 += __shfl_xor_sync(0xffffffffu, t1, 1);
    t0 += __shfl_xor_sync(0xffffffffu, t0, 2);
    t1 += __shfl_xor_sync(0xffffffffu, t1, 2);
    const float s2 = sh.s2[k];
    const float L0 = s2 * t0, L1 = s2 * t1;
    if (L0 < best[0]) {
      best[0] = L0;
      best_k[0] = k;
    }
    if (L1 < best[1]) {
      best[1] = L1;
      best_k[1] = k;
    }
  };

  // Candidates below kstart: every unit of the warp is fully clamped, and its loss is the
  // parabola f(k) = (pa s_k + pb) s_k, evaluated in fp32 exactly as written. For pa > 0 its
  // minimum over the prefix (lowest k on equal values) is at one of the two candidates that
  // bracket the vertex s* = -pb / (2 pa), up to rounding: consecutive candidate scales differ by
  // at least 1/16 (relative), so a candidate two or more places beyond the bracket exceeds the
  // bracket's better one by at least about 0.6% of pa s*^2, against rounding errors of a few
  // 2^-24 of the same. The E4M3 code of s*/g, rounded to nearest, is one of the bracketing
  // candidates' codes or next to them, so the candidates within two places of it find the
  // same minimum and index as all of them. Short prefixes, pa <= 0 and values near the ends of
  // the fp32 range take every candidate.
  constexpr int kPrefixWin = 2;
  const float s0 = sh.tab[2].w;  // the smallest candidate scale (grid value 1 times s_0)
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    int lo = 0, hi = kstart;
    const float a = pa[u], b = pb[u];
    if (kstart > 2 * kPrefixWin + 1 && s0 > 0.f && a > 0.f && a < 0x1p100f && fabsf(b) < 0x1p100f &&
        a * s0 * s0 >= 0x1p-100f && sh.tab[kLev * (kstart - 1) + 2].w < 0x1p40f) {
      const float q = fmaxf(-b / (2.f * a), 0.f) / __ldg(g + e);  // s*/g, or 0 if the vertex is at s <= 0
      const int c = static_cast<int>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3) & 0x7F);
      const int k0 = min(max(c - 1, 0), kstart - 1);  // candidate k has code k + 1
      lo = max(0, k0 - kPrefixWin);
      hi = min(kstart, k0 + kPrefixWin + 1);
    }
    float bu = best[u];
    int bk = best_k[u];
#pragma unroll 1
    for (int k = lo; k < hi; ++k) {
      const float sk = sh.tab[kLev * k + 2].w;  // grid value 1 times s_k
      const float L = fmaf(a, sk, b) * sk;
      if (L < bu) {
        bu = L;
        bk = k;
      }
    }
    best[u] = bu;
    best_k[u] = bk;
  }
  // From kstart: levels by counting thresholds until the 4th candidate and until the rest is a
  // multiple of four, then by single-step drops (consecutive scales differ by at most 4/3).
  int kinc = max(kstart + 1, 3);
  kinc += (kCand - kinc) % 4;
  const uint32_t tab_base = smem_u32(sh.tab);
  uint32_t addr[8];  // shared address of the table entry (k, level) of each element
#pragma unroll 1
  for (int k = kstart; k < kinc; ++k) {
    const float4* tab_k = sh.tab + kLev * k;
    uint32_t q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int lev = level_direct_tc(tab_k, a[i]);
      addr[i] = tab_base + static_cast<uint32_t>((kLev * k + lev) * kEntryBytes);
      q[i] = __float_as_uint((i & 1) ? tab_k[lev].z : tab_k[lev].y);
    }
    evaluate(q, k);
  }
  // Four candidates at a time. A transposed reduction over the quad leaves lane tq with the
  // full sums of candidate k + tq (the same additions as the per-candidate reduction, so the
  // same values): after each pair of candidates the lanes tq and tq ^ 1 swap halves (lane tq
  // keeps the pair's candidate with index bit tq & 1), and after the second pair lanes tq and
  // tq ^ 2 finish. Each lane tracks the best of its own candidates; the quad merges them after
  // the loop.
  const bool b0 = (tq & 1) != 0, b1 = (tq & 2) != 0;
  // One loop trip's bookkeeping after the four candidates: the reductions' second stage and the
  // best of the lane's candidate k + tq.
  auto finish4 = [&](int k, const float (&spair)[2][2]) {
    const int kk = k + tq;
    const float s2 = sh.s2[kk];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float t = (b1 ? spair[1][u] : spair[0][u]) + __shfl_xor_sync(0xffffffffu, b1 ? spair[0][u] : spair[1][u], 2);
      const float L = s2 * t;
      if (L < best[u]) {
        best[u] = L;
        best_k[u] = kk;
      }
    }
  };
  auto stage_pair = [&](int c, const float (&tp)[2], float (&hold)[2], float (&spair)[2][2]) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if ((c & 1) == 0) {
        hold[u] = tp[u];
      } else {  // candidates (c - 1, c): keep the one with index bit b0, hand over the other
        spair[c >> 1][u] = (b0 ? tp[u] : hold[u]) + __shfl_xor_sync(0xffffffffu, b0 ? hold[u] : tp[u], 1);
      }
    }
  };
  // bf16 magnitudes of the A registers' element pairs (exact: the weights are bf16).
  uint32_t a2[4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
    a2[r] = (__float_as_uint(a[kPairLo[r]]) >> 16) | (__float_as_uint(a[kPairLo[r] + 1]) & 0xffff0000u);
  if constexpr (kPair) {
    // Pair addresses in the row of candidate kinc - 1, from the levels the direct loop left.
    const uint32_t thr2_base = smem_u32(ps.thr2), q2_base = smem_u32(ps.q2);
    uint32_t pa[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const uint32_t l0 = ((addr[kPairLo[r]] - tab_base) >> 4) & 7u;
      const uint32_t l1 = ((addr[kPairLo[r] + 1] - tab_base) >> 4) & 7u;
      pa[r] = thr2_base + static_cast<uint32_t>((kinc - 1) * kPairRowBytes) + (8u * l1 + l0) * 4u;
    }
    // pa - qoff is the pair's grid-value entry: qoff removes the row and the table base.
    uint32_t qoff = thr2_base + static_cast<uint32_t>((kinc - 1) * kPairRowBytes) - q2_base;
#pragma unroll 1
    for (int k = kinc; k < kCand; k += 4) {
      float hold[2], spair[2][2];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t afr[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          uint32_t t2;
          if (c == 0) t2 = lds_u32<kPairRowBytes>(pa[r]);
          else if (c == 1) t2 = lds_u32<2 * kPairRowBytes>(pa[r]);
          else if (c == 2) t2 = lds_u32<3 * kPairRowBytes>(pa[r]);
          else t2 = lds_u32<4 * kPairRowBytes>(pa[r]);
          drop_pair(pa[r], a2[r], t2);
          afr[r] = lds_u32<0>(pa[r] - qoff) ^ smask[r];
        }
        float tp[2];
        partials_afr(afr, k + c, tp);
        stage_pair(c, tp, hold, spair);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) pa[r] += 4 * kPairRowBytes;
      qoff += 4 * kPairRowBytes;
      finish4(k, spair);
    }
  } else {
#pragma unroll 1
    for (int k = kinc; k < kCand; k += 4) {
      float hold[2], spair[2][2];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float t;
          if (c == 0) t = lds_f32<kTabRowBytes>(addr[i]);
          else if (c == 1) t = lds_f32<2 * kTabRowBytes>(addr[i]);
          else if (c == 2) t = lds_f32<3 * kTabRowBytes>(addr[i]);
          else t = lds_f32<4 * kTabRowBytes>(addr[i]);
          addr[i] = drop_if_below(addr[i], a[i], t, static_cast<uint32_t>(kEntryBytes));
          constexpr int kQ0 = 4, kQ1 = 8;  // byte offsets of the low- and high-half fp16 words
          if (i & 1) {
            if (c == 0) q[i] = lds_u32<kTabRowBytes + kQ1>(addr[i]);
            else if (c == 1) q[i] = lds_u32<2 * kTabRowBytes + kQ1>(addr[i]);
            else if (c == 2) q[i] = lds_u32<3 * kTabRowBytes + kQ1>(addr[i]);
            else q[i] = lds_u32<4 * kTabRowBytes + kQ1>(addr[i]);
          } else {
            if (c == 0) q[i] = lds_u32<kTabRowBytes + kQ0>(addr[i]);
            else if (c == 1) q[i] = lds_u32<2 * kTabRowBytes + kQ0>(addr[i]);
            else if (c == 2) q[i] = lds_u32<3 * kTabRowBytes + kQ0>(addr[i]);
            else q[i] = lds_u32<4 * kTabRowBytes + kQ0>(addr[i]);
          }
        }
        float tp[2];
        partials(q, k + c, tp);
        stage_pair(c, tp, hold, spair);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) addr[i] += 4 * kTabRowBytes;
      finish4(k, spair);
    }
  }
  // Merge the quad's bests: the smallest loss, and on equal losses the lowest candidate.
#pragma unroll
  for (int u = 0; u < 2; ++u) {
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      const float ol = __shfl_xor_sync(0xffffffffu, best[u], o);
      const int ok = __shfl_xor_sync(0xffffffffu, best_k[u], o);
      if (ol < best[u] || (ol == best[u] && ok < best_k[u])) {
        best[u] = ol;
        best_k[u] = ok;
      }
    }
  }

  // ---- outputs. The winner's loss is recomputed from its fp32 fake-quant weights by the
  // definition, dW^T H dW (+ 2 dW^T P w), so that it is accurate relative to itself.
  float wqv[8], dwv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4* tab_k = sh.tab + kLev * best_k[i >> 2];
    // The sign bit of element i, from the packed A-register masks (not kept live through the sweep).
    constexpr int kPairOf[8] = {0, 0, 2, 2, 1, 1, 3, 3};
    const uint32_t sbit = (smask[kPairOf[i]] >> ((i & 1) ? 31 : 15)) & 1u;
    // bf16 weights: |w| from the packed pairs, so that a[] need not stay live through the sweep.
    constexpr int kRegOf[8] = {0, 0, 2, 2, 1, 1, 3, 3};
    const float ai = kPair ? __uint_as_float((i & 1) ? (a2[kRegOf[i]] & 0xffff0000u) : (a2[kRegOf[i]] << 16)) : a[i];
    wqv[i] = __uint_as_float(__float_as_uint(tab_k[level_direct_tc(tab_k, ai)].w) | (sbit << 31));
    dwv[i] = wqv[i] - __uint_as_float(__float_as_uint(ai) | (sbit << 31));
  }
#pragma unroll 1
  for (int u = 0; u < 2; ++u) {
    float dw[4], wq4[4];
#pragma unroll
    for (int ci = 0; ci < 4; ++ci) {
      dw[ci] = u ? dwv[4 + ci] : dwv[ci];
      wq4[ci] = u ? wqv[4 + ci] : wqv[ci];
    }
    float dfull[16];  // all 16 dW of the unit, gathered from the quad
#pragma unroll
    for (int t2 = 0; t2 < 4; ++t2) {
#pragma unroll
      for (int ci = 0; ci < 4; ++ci)
        dfull[2 * t2 + (ci & 1) + 8 * (ci >> 1)] = __shfl_sync(0xffffffffu, dw[ci], (lane & ~3) | t2);
    }
    // The unit's row, read again from the CTA's ordering (not kept live through the sweep).
    const int64_t row = rbase + sh.perm[warp * kUnitsPerWarp + gq + 8 * u];
    const bool ok = row < rows;
    float part = 0.f;
#pragma unroll
    for (int ci = 0; ci < 4; ++ci) {
      const int c = col_of(ci);
      float hd = 0.f;
#pragma unroll
      for (int k = 0; k < 16; k += 4) {  // row c of H, four entries at a time
        const float4 hq = *reinterpret_cast<const float4*>(sh.h + c * 16 + k);
        hd = fmaf(hq.x, dfull[k], hd);
        hd = fmaf(hq.y, dfull[k + 1], hd);
        hd = fmaf(hq.z, dfull[k + 2], hd);
        hd = fmaf(hq.w, dfull[k + 3], hd);
      }
      if (ACT) {  // + 2 (P w)_c
        const float* wr = sh.wall[sh.perm[warp * kUnitsPerWarp + gq + 8 * u]];
        float pw = 0.f;
        if (kPair) {
          pw = wr[c];  // as the set-up computed it, stored over the unit's staged row
        } else {  // from the staged weights, in the set-up's order
#pragma unroll
          for (int k = 0; k < 16; k += 4) {
            const float4 pq = *reinterpret_cast<const float4*>(sh.p + c * 16 + k);
            const float4 wq4v = *reinterpret_cast<const float4*>(wr + k);
            pw = fmaf(pq.x, wq4v.x, pw);
            pw = fmaf(pq.y, wq4v.y, pw);
            pw = fmaf(pq.z, wq4v.z, pw);
            pw = fmaf(pq.w, wq4v.w, pw);
          }
        }
        hd = fmaf(2.f, pw, hd);
      }
      part = fmaf(dw[ci], hd, part);
    }
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    if (!ok) continue;
    const int64_t unit = (e * rows + row) * nblk + n;
    if (tq == 0) {
      codes[unit] = static_cast<uint8_t>((u ? best_k[1] : best_k[0]) + 1);
      if (loss != nullptr) loss[unit] = part;
    }
    if (wq != nullptr) {
      float* dst = wq + (e * rows + row) * cin + n * kBlock + 2 * tq;
      *reinterpret_cast<float2*>(dst) = make_float2(wq4[0], wq4[1]);
      *reinterpret_cast<float2*>(dst + 8) = make_float2(wq4[2], wq4[3]);
    }
  }
}

}  // namespace

lhcal_status launch_sweep_tc(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows,
                             int64_t cin, const float* h, const float* p, const float* g, uint8_t* codes,
                             float* wq, float* loss, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(cin / kBlock), static_cast<unsigned>(ceil_div(rows, kUnitsPerCta)),
                  static_cast<unsigned>(groups));
  if (dtype == LHCAL_BF16) {
    // The pair tables live in dynamic shared memory; with the static part a CTA holds about 69 KB,
    // three per SM. Set on every call with the same values: cheap, and right for any device.
    constexpr int kDyn = static_cast<int>(sizeof(TcPairShared));
    for (const void* fn : {reinterpret_cast<const void*>(sweep_tc_kernel<true, __nv_bfloat16>),
                           reinterpret_cast<const void*>(sweep_tc_kernel<false, __nv_bfloat16>)}) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kDyn);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return fail(LHCAL_ERR_CUDA, "scale sweep: %s", cudaGetErrorString(e));
    }
    if (mode == LHCAL_ACT_AWARE)
      sweep_tc_kernel<true, __nv_bfloat16><<<grid, kTcThreads, kDyn, stream>>>(
          static_cast<const __nv_bfloat16*>(w), rows, cin, h, p, g, codes, wq, loss);
    else
      sweep_tc_kernel<false, __nv_bfloat16><<<grid, kTcThreads, kDyn, stream>>>(
          static_cast<const __nv_bfloat16*>(w), rows, cin, h, p, g, codes, wq, loss);
  } else {
    if (mode == LHCAL_ACT_AWARE)
      sweep_tc_kernel<true, float><<<grid, kTcThreads, 0, stream>>>(static_cast<const float*>(w), rows, cin, h, p,
                                                                     g, codes, wq, loss);
    else
      sweep_tc_kernel<false, float><<<grid, kTcThreads, 0, stream>>>(static_cast<const float*>(w), rows, cin, h,
                                                                      p, g, codes, wq, loss);
  }
  return check_launch("scale sweep (tensor cores)");
}

}  // namespace lhcal
