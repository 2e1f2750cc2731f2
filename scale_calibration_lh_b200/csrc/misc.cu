// Token counts, finalisation (/B and the zero-token fallback) and the per-group global scale.
//
// "Add activation-aware local Hessian scale calibration" (PR #1976), "What does this PR do?":
// H and P are divided by the number of accumulated rows B. "[2/3] Speed up layerwise GPTQ on
// MoE models" (PR #2864), embedded #2840: an expert that no token reaches gets the plain
// search (here H = I, P = 0, Imp = 1). "Add composable scale calibration to GPTQ" (PR #2004):
// 448-normalized NVFP4 global scale g = amax / (6 * 448), and 256-normalized for the page's
// NVFP4 "4/6" variant. The output epilogue (apply_scales) writes the fake-quantized weights in
// fp32 and bf16 and the per-block amax, the quantizer state "Add WMSE weight scale search
// calibration" (PR #2283) fingerprints (amax, _amax, the fake-quantized weights).
#include "common.cuh"
#include "quant_tables.cuh"

namespace lhcal {
namespace {

__global__ void count_tokens_kernel(int32_t groups, int64_t tokens, const int32_t* __restrict__ offs,
                                    int accumulate_into, int64_t* __restrict__ counts) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= groups) return;
  const int64_t c = offs ? static_cast<int64_t>(offs[e + 1]) - offs[e] : tokens;
  counts[e] = accumulate_into ? counts[e] + c : c;
}

template <int MODE>
__global__ void finalize_kernel(int32_t groups, int64_t per_group, const int64_t* __restrict__ counts,
                                float* __restrict__ h, float* __restrict__ p) {
  const int64_t total = static_cast<int64_t>(groups) * per_group;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = i / per_group;
    const int64_t b = __ldg(counts + e);
    if (MODE == LHCAL_DIAG) {
      if (b == 0) h[i] = 1.f;  // plain block MSE
      continue;
    }
    if (b == 0) {
      const int ij = static_cast<int>(i & 255);
      h[i] = ((ij >> 4) == (ij & 15)) ? 1.f : 0.f;
      if (MODE == LHCAL_ACT_AWARE) p[i] = 0.f;
    } else {
      // Correctly rounded quotient of the fp32 sum by the exact integer count.
      const double bd = static_cast<double>(b);
      h[i] = static_cast<float>(static_cast<double>(h[i]) / bd);
      if (MODE == LHCAL_ACT_AWARE) p[i] = static_cast<float>(static_cast<double>(p[i]) / bd);
    }
  }
}

// amax as the bit pattern of |w| (non-negative floats order like unsigned integers).
template <typename T>
__device__ __forceinline__ uint32_t abs_bits8(const T* src);

template <>
__device__ __forceinline__ uint32_t abs_bits8<float>(const float* src) {
  const uint4 a = __ldcs(reinterpret_cast<const uint4*>(src));
  const uint4 b = __ldcs(reinterpret_cast<const uint4*>(src) + 1);
  const uint32_t m = 0x7fffffffu;
  uint32_t r = max(max(a.x & m, a.y & m), max(a.z & m, a.w & m));
  return max(r, max(max(b.x & m, b.y & m), max(b.z & m, b.w & m)));
}

template <>
__device__ __forceinline__ uint32_t abs_bits8<__nv_bfloat16>(const __nv_bfloat16* src) {
  const uint4 v = __ldcs(reinterpret_cast<const uint4*>(src));
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  uint32_t r = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) r = max(r, max((u[i] << 16) & 0x7fffffffu, u[i] & 0x7fff0000u));
  return r;
}

constexpr int kAmaxThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kAmaxThreads)
amax_kernel(const T* __restrict__ w, int64_t per_group, uint32_t* __restrict__ amax_bits) {
  const int64_t e = blockIdx.y;
  const T* base = w + e * per_group;
  const int64_t n8 = per_group / 8;
  uint32_t m = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n8; i += 4 * stride) {  // four independent 16-byte loads in flight
    const uint32_t a = abs_bits8<T>(base + i * 8), b = abs_bits8<T>(base + (i + stride) * 8);
    const uint32_t c = abs_bits8<T>(base + (i + 2 * stride) * 8), d = abs_bits8<T>(base + (i + 3 * stride) * 8);
    m = max(m, max(max(a, b), max(c, d)));
  }
  for (; i < n8; i += stride) m = max(m, abs_bits8<T>(base + i * 8));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t red[kAmaxThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < kAmaxThreads / 32; ++k) m = max(m, red[k]);
    atomicMax(amax_bits + e, m);
  }
}

// g = RN(amax / divisor), divisor = 6 * fp8_max exactly (2688 for 448, 1536 for 256).
__global__ void scale_from_amax_kernel(int32_t groups, float divisor, float* __restrict__ g) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= groups) return;
  const float amax = __uint_as_float(reinterpret_cast<const uint32_t*>(g)[e]);
  g[e] = __fdiv_rn(amax, divisor);
}

// Outputs for chosen codes: one thread per unit (group, row, block). s = fp32(v_c g) with the
// exact E2M1 thresholds of quant_tables.cuh; wq = copysign(fp32(q s), w); the bf16 copy rounds
// that fp32 value to nearest even; amax = fp32(6 v_c g). Code 0 is a zero scale; codes above
// 126 are taken as 126.
template <typename T>
__global__ void __launch_bounds__(256)
apply_scales_kernel(const T* __restrict__ w, int64_t units, int64_t nblk, int64_t rows_x_nblk,
                    const float* __restrict__ g, const uint8_t* __restrict__ codes, float* __restrict__ wq,
                    __nv_bfloat16* __restrict__ wq16, float* __restrict__ amax) {
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = u / rows_x_nblk;
    const int c = min(static_cast<int>(codes[u]), kCand);
    const float gv = __ldg(g + e);
    const float v = c == 0 ? 0.f : e4m3_value(c);
    const float s = __fmul_rn(v, gv);
    if (amax) amax[u] = __fmul_rn(6.f * v, gv);  // 6 v is exact
    if (!wq && !wq16) continue;
    float thr[kLev], val[kLev];
#pragma unroll
    for (int j = 0; j < kLev; ++j) {
      thr[j] = level_threshold(j, s);
      val[j] = __fmul_rn(e2m1_grid(j), s);
    }
    float x[kBlock];
    load8<T>(w + u * kBlock, x);
    load8<T>(w + u * kBlock + 8, x + 8);
    float out[kBlock];
#pragma unroll
    for (int i = 0; i < kBlock; ++i) {
      const float a = fabsf(x[i]);
      float m = 0.f;  // s == 0: every threshold is 0 and every value 0
#pragma unroll
      for (int j = 1; j < kLev; ++j) m = a >= thr[j] ? val[j] : m;
      out[i] = copysignf(m, x[i]);
    }
    if (wq) {
      float4* dst = reinterpret_cast<float4*>(wq + u * kBlock);
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
    }
    if (wq16) {
      uint32_t pk[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(out[2 * q], out[2 * q + 1]);
        pk[q] = *reinterpret_cast<const uint32_t*>(&b);
      }
      uint4* dst = reinterpret_cast<uint4*>(wq16 + u * kBlock);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
  }
}

}  // namespace

lhcal_status launch_count_tokens(int32_t groups, int64_t tokens, const int32_t* group_offsets,
                                 int32_t flags, int64_t* counts, cudaStream_t stream) {
  const int acc = (flags & LHCAL_ACCUM_OVERWRITE) ? 0 : 1;
  count_tokens_kernel<<<static_cast<unsigned>(ceil_div(groups, 256)), 256, 0, stream>>>(
      groups, tokens, group_offsets, acc, counts);
  return check_launch("count tokens");
}

lhcal_status launch_finalize(lhcal_mode mode, int32_t groups, int64_t cin, const int64_t* counts,
                             float* h, float* p, cudaStream_t stream) {
  const int64_t nblk = cin / kBlock;
  const int64_t per_group = mode == LHCAL_DIAG ? cin : nblk * 256;
  const int64_t total = static_cast<int64_t>(groups) * per_group;
  const unsigned blocks = static_cast<unsigned>(imin64(ceil_div(total, 256), 8 * kNumSms));
  if (mode == LHCAL_FULL)
    finalize_kernel<LHCAL_FULL><<<blocks, 256, 0, stream>>>(groups, per_group, counts, h, p);
  else if (mode == LHCAL_ACT_AWARE)
    finalize_kernel<LHCAL_ACT_AWARE><<<blocks, 256, 0, stream>>>(groups, per_group, counts, h, p);
  else
    finalize_kernel<LHCAL_DIAG><<<blocks, 256, 0, stream>>>(groups, per_group, counts, h, p);
  return check_launch("finalize");
}

lhcal_status launch_global_scale(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows,
                                 int64_t cin, float* g, cudaStream_t stream, float fp8_max) {
  // g doubles as the amax accumulator (bit patterns), then is converted in place.
  cudaError_t e = cudaMemsetAsync(g, 0, sizeof(float) * static_cast<size_t>(groups), stream);
  if (e != cudaSuccess) return fail(LHCAL_ERR_CUDA, "global scale: %s", cudaGetErrorString(e));
  const int64_t per_group = rows * cin;
  const int64_t n8 = per_group / 8;
  const int64_t want = imax64(1, ceil_div(8 * kNumSms, groups));
  const int64_t bx = imax64(1, imin64(want, ceil_div(n8, kAmaxThreads)));
  const dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(groups));
  auto* bits = reinterpret_cast<uint32_t*>(g);
  if (dtype == LHCAL_BF16)
    amax_kernel<__nv_bfloat16><<<grid, kAmaxThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(w), per_group, bits);
  else
    amax_kernel<float><<<grid, kAmaxThreads, 0, stream>>>(static_cast<const float*>(w), per_group, bits);
  lhcal_status st = check_launch("global scale (amax)");
  if (st != LHCAL_OK) return st;
  scale_from_amax_kernel<<<static_cast<unsigned>(ceil_div(groups, 256)), 256, 0, stream>>>(groups, 6.f * fp8_max,
                                                                                              g);
  return check_launch("global scale");
}

lhcal_status launch_apply_scales(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows, int64_t cin,
                                 const float* g, const uint8_t* codes, float* wq, void* wq16, float* amax,
                                 cudaStream_t stream) {
  const int64_t nblk = cin / kBlock;
  const int64_t units = static_cast<int64_t>(groups) * rows * nblk;
  const unsigned blocks = static_cast<unsigned>(imin64(ceil_div(units, 256), 8 * kNumSms));
  auto* w16 = static_cast<__nv_bfloat16*>(wq16);
  if (dtype == LHCAL_BF16)
    apply_scales_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(w), units, nblk,
                                                                    rows * nblk, g, codes, wq, w16, amax);
  else
    apply_scales_kernel<float><<<blocks, 256, 0, stream>>>(static_cast<const float*>(w), units, nblk, rows * nblk,
                                                           g, codes, wq, w16, amax);
  return check_launch("apply scales");
}

}  // namespace lhcal
