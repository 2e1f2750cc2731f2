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
// fp16 hi + lo (H scaled by a power of two into fp16 range): relative error <= 2^-23 per H
// entry, fp32 accumulation. The loss then differs from the fp32-rounded definition by at most
// a few 2^-23 of |w|^T |H| |w|, far below the 1e-5 decision gaps that matter.
//
// Mapping (mma.sync.m16n8k16, row.col, f16 -> f32): a warp evaluates 16 units (the M rows) of
// one input block for one candidate per step. Lane (g = lane / 4, t = lane % 4) owns units
// g and g + 8 and, of each, the four columns {2t, 2t+1, 2t+8, 2t+9}. Those are exactly its
// A-fragment columns and its accumulator columns, so the epilogue needs no data movement
// except a reduction over the four lanes of a quad.
//
// Quantization. As in the FP32 sweep: per-candidate threshold tables built from exact
// residuals decide the E2M1 level of every element exactly as on the exact quotient, and
// each element's level falls by at most one per candidate from the 4th on. Each table entry
// also carries the fp16 bits of its grid value, pre-placed for the low or the high half of
// a packed pair, so building the A fragment is one OR (and a sign XOR) per pair.
//
// Work per candidate. Candidates below the warp's first unclamped one take a closed form;
// the rest go four per loop trip, and the quad's four lanes share the reduction of four
// candidates (a transposed reduction: lane t ends with candidate k + t) and keep their own
// bests, merged after the loop. The per-unit set-up reads the units' weights from shared
// memory, and the grid runs the 16-column blocks fastest.
#include "common.cuh"
#include "quant_tables.cuh"

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

struct __align__(16) TcShared {
  float4 tab[kCand * kLev];
  float rho[kCand];  // -2 / (s_k * 2^eH): scale of U' in the MMA accumulator
  float s2[kCand];   // s_k^2 * 2^eH
  float h[256];
  float p[256];
  float hscale;  // 2^-eH: H' = H * hscale lies below 2^15
  float key[kUnitsPerCta];  // min |w| of each of the CTA's units (rows)
  int perm[kUnitsPerCta];   // the CTA's rows ordered by key
  // Each warp's 16 units' weights (fp32), rows padded to 17 floats so that the 8 units a warp
  // reads at once fall in distinct banks. Read by the per-unit set-up and the ACT epilogue.
  float wst[kTcWarps][kUnitsPerWarp][kBlock + 1];
};

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

// Level of magnitude a at candidate row k of the table, by counting thresholds.
__device__ __forceinline__ int level_direct_tc(const float4* tab_k, float a) {
  int lev = 0;
#pragma unroll
  for (int j = 1; j < kLev; ++j) lev += (a >= tab_k[j].x) ? 1 : 0;
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
  const int64_t nblk = cin / kBlock;
  // Blocks vary fastest across the grid: CTAs running together cover neighbouring blocks of the
  // same rows, so their W reads are adjacent and their codes / loss writes share DRAM sectors.
  const int64_t n = blockIdx.x;
  const int64_t e = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;

  // ---- per-CTA set-up: H (and P) of block n, the H scale, candidate tables
  const int64_t hblk = e * nblk + n;
  for (int i = threadIdx.x; i < 256; i += kTcThreads) {
    sh.h[i] = __ldg(h + hblk * 256 + i);
    if (ACT) sh.p[i] = __ldg(p + hblk * 256 + i);
  }
  const float gs = __ldg(g + e);
  for (int idx = threadIdx.x; idx < kCand * kLev; idx += kTcThreads) {
    const int k = idx >> 3, j = idx & 7;
    const float s = candidate_scale(k, gs);
    const uint32_t q16 = e2m1_grid_f16_bits(j);
    sh.tab[idx] = make_float4(level_threshold(j, s), __uint_as_float(q16), __uint_as_float(q16 << 16),
                              __fmul_rn(e2m1_grid(j), s));
  }
  // Order the CTA's rows by their smallest |w|, so that the units a warp evaluates together
  // leave the all-clamped candidates at similar scales (see the clamped prefix below).
  const int64_t rbase = static_cast<int64_t>(blockIdx.y) * kUnitsPerCta;
  if (threadIdx.x < kUnitsPerCta) {
    const int64_t row = rbase + threadIdx.x;
    float m = __int_as_float(0x7f800000);
    if (row < rows) {
      float wt[16];
      load_row16<WT>(w + (e * rows + row) * cin + n * kBlock, true, wt);
#pragma unroll
      for (int i = 0; i < 16; ++i) m = fminf(m, fabsf(wt[i]));
    }
    sh.key[threadIdx.x] = m;
  }
  __syncthreads();
  if (threadIdx.x < kUnitsPerCta) {
    const float my = sh.key[threadIdx.x];
    int rank = 0;
    for (int j = 0; j < kUnitsPerCta; ++j) {
      const float kj = sh.key[j];
      rank += (kj < my || (kj == my && j < static_cast<int>(threadIdx.x))) ? 1 : 0;
    }
    sh.perm[rank] = threadIdx.x;
  }
  if (warp == 0) {
    uint32_t m = 0;
    for (int i = lane; i < 256; i += 32) m = max(m, __float_as_uint(sh.h[i]) & 0x7fffffffu);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) {
      // Scale so that the largest |H'| lies in [2^14, 2^15): below the fp16 maximum.
      const int ex = (m == 0u) ? 0 : static_cast<int>(m >> 23) - 127;  // floor(log2 max|H|)
      const int sh_exp = min(127, max(-126, 14 - ex));
      sh.hscale = pow2i(sh_exp);
    }
  }
  __syncthreads();
  const float hscale = sh.hscale;
  const float inv_hscale = 1.0f / hscale;  // exact: a power of two
  for (int k = threadIdx.x; k < kCand; k += kTcThreads) {
    const float s = candidate_scale(k, gs);
    sh.rho[k] = -2.f * hscale / s;
    sh.s2[k] = (s * s) * inv_hscale;
  }
  __syncthreads();

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

  // ---- the warp's 16 units: sorted positions 16 warp + gq (unit 0) and + 8 (unit 1). Their
  // weights go to shared memory (lane l loads half l & 1 of unit l / 2), so that the set-up
  // below reads them instead of holding 32 of them in registers.
  float (*wst)[kBlock + 1] = sh.wst[warp];
  {
    const int j = lane >> 1, h8 = (lane & 1) * 8;
    const int64_t row = rbase + sh.perm[warp * kUnitsPerWarp + j];
    const bool ok = row < rows;
    float w8[8];
    if (ok) load8<WT>(w + (e * rows + row) * cin + n * kBlock + h8, w8);
#pragma unroll
    for (int k = 0; k < 8; ++k) wst[j][h8 + k] = ok ? w8[k] : 0.f;
  }
  __syncwarp();
  bool valid[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) valid[u] = rbase + sh.perm[warp * kUnitsPerWarp + gq + 8 * u] < rows;
  // Lane element i (0..7): unit i / 4, column col_of(i % 4) with columns {2t, 2t+1, 2t+8, 2t+9}.
  auto col_of = [&](int ci) { return 2 * tq + (ci & 1) + 8 * (ci >> 1); };
  float a[8], up[8];
  uint32_t sgn[8];
  float cpart[2] = {0.f, 0.f};
  float pqa[2] = {0.f, 0.f}, pqb[2] = {0.f, 0.f}, amin[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    amin[u] = __int_as_float(0x7f800000);
#pragma unroll
    for (int ci = 0; ci < 4; ++ci) {
      const int c = col_of(ci);
      const int i = 4 * u + ci;
      const float* wr = wst[gq + 8 * u];
      const float x = wr[c];
      a[i] = fabsf(x);
      amin[u] = fminf(amin[u], a[i]);
      sgn[i] = __float_as_uint(x) >> 31;
      float hw_sym = 0.f, hw_row = 0.f, pw = 0.f, hsg = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float hck = sh.h[c * 16 + k];
        const float wk = wr[k];
        hw_sym = fmaf(0.5f * (hck + sh.h[k * 16 + c]), wk, hw_sym);
        hw_row = fmaf(hck, wk, hw_row);
        hsg += (__float_as_uint(wk) >> 31) ? -hck : hck;  // (H sign(w))_c
        if (ACT) pw = fmaf(sh.p[c * 16 + k], wk, pw);
      }
      up[i] = hw_sym - pw;                               // U'_c
      cpart[u] = fmaf(x, hw_row - 2.f * pw, cpart[u]);  // w_c ((H w)_c - 2 (P w)_c)
      const float sc = sgn[i] ? -1.f : 1.f;
      pqa[u] = fmaf(sc, hsg, pqa[u]);
      pqb[u] = fmaf(sc, up[i], pqb[u]);
    }
  }
  float cconst[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    float v = cpart[u];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    cconst[u] = v;  // C' of the unit
  }
  // While every element of a unit is clamped at the top of the grid (|w_i| >= thr[k][7], so
  // v = 6 sign(w)), its loss is the parabola 36 s^2 sign^T H sign - 12 s sign^T U' + C'.
  // kfirst = first candidate at which some element of the unit is below the top level.
  float pa[2], pb[2];
  int kfirst_lane = kCand;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    float m = amin[u], qa = pqa[u], qb = pqb[u];
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      m = fminf(m, __shfl_xor_sync(0xffffffffu, m, o));
      qa += __shfl_xor_sync(0xffffffffu, qa, o);
      qb += __shfl_xor_sync(0xffffffffu, qb, o);
    }
    pa[u] = 36.f * qa;
    pb[u] = -12.f * qb;
    if (valid[u]) {
      int lo = 0, hi = kCand;  // first k with m < thr[k][7]
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (m < sh.tab[kLev * mid + 7].x) hi = mid; else lo = mid + 1;
      }
      kfirst_lane = min(kfirst_lane, lo);
    }
  }
  int kstart = kfirst_lane;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) kstart = min(kstart, __shfl_xor_sync(0xffffffffu, kstart, o));
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
  //   L = s2_k * sum_n v_n D_n + C' = s^2 v^T H v - 2 s v^T U' + C'.
  // The lane's share of t for units 0 and 1 (its 4 columns), before the reduction over the quad.
  auto partials = [&](const uint32_t (&q)[8], int k, float (&tp)[2]) {
    uint32_t afr[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) afr[r] = (q[kPairLo[r]] | q[kPairLo[r] + 1]) ^ smask[r];
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
  auto evaluate = [&](const uint32_t (&q)[8], int k) {
    float tp[2];
    partials(q, k, tp);
    float t0 = tp[0], t1 = tp[1];
    t0 += __shfl_xor_sync(0xffffffffu, t0, 1);
    t1 += __shfl_xor_sync(0xffffffffu, t1, 1);
    t0 += __shfl_xor_sync(0xffffffffu, t0, 2);
    t1 += __shfl_xor_sync(0xffffffffu, t1, 2);
    const float s2 = sh.s2[k];
    const float L0 = fmaf(s2, t0, cconst[0]), L1 = fmaf(s2, t1, cconst[1]);
    if (L0 < best[0]) {
      best[0] = L0;
      best_k[0] = k;
    }
    if (L1 < best[1]) {
      best[1] = L1;
      best_k[1] = k;
    }
  };

  // Candidates below kstart: every unit of the warp is fully clamped; closed-form losses.
#pragma unroll 1
  for (int k = 0; k < kstart; ++k) {
    const float sk = sh.tab[kLev * k + 2].w;  // grid value 1 times s_k
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float L = fmaf(fmaf(pa[u], sk, pb[u]), sk, cconst[u]);
      if (L < best[u]) {
        best[u] = L;
        best_k[u] = k;
      }
    }
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
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if ((c & 1) == 0) {
          hold[u] = tp[u];
        } else {  // candidates (c - 1, c): keep the one with index bit b0, hand over the other
          spair[c >> 1][u] = (b0 ? tp[u] : hold[u]) + __shfl_xor_sync(0xffffffffu, b0 ? hold[u] : tp[u], 1);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) addr[i] += 4 * kTabRowBytes;
    const int kk = k + tq;
    const float s2 = sh.s2[kk];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float t = (b1 ? spair[1][u] : spair[0][u]) + __shfl_xor_sync(0xffffffffu, b1 ? spair[0][u] : spair[1][u], 2);
      const float L = fmaf(s2, t, cconst[u]);
      if (L < best[u]) {
        best[u] = L;
        best_k[u] = kk;
      }
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
    wqv[i] = __uint_as_float(__float_as_uint(tab_k[level_direct_tc(tab_k, a[i])].w) | (sbit << 31));
    dwv[i] = wqv[i] - __uint_as_float(__float_as_uint(a[i]) | (sbit << 31));
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
      for (int k = 0; k < 16; ++k) hd = fmaf(sh.h[c * 16 + k], dfull[k], hd);
      if (ACT) {  // + 2 (P w)_c, with w from the warp's shared copy
        const float* wr = wst[gq + 8 * u];
        float pw = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) pw = fmaf(sh.p[c * 16 + k], wr[k], pw);
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
    if (mode == LHCAL_ACT_AWARE)
      sweep_tc_kernel<true, __nv_bfloat16><<<grid, kTcThreads, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(w), rows, cin, h, p, g, codes, wq, loss);
    else
      sweep_tc_kernel<false, __nv_bfloat16><<<grid, kTcThreads, 0, stream>>>(
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
