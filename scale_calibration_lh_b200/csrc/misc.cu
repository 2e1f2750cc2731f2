// Token counts, finalisation (/B and the zero-token fallback) and the per-group global scale.
//
// "Add activation-aware local Hessian scale calibration" (PR #1976), "What does this PR do?":
// H and P are divided by the number of accumulated rows B. "[2/3] Speed up layerwise GPTQ on
// MoE models" (PR #2864), embedded #2840: an expert that no token reaches gets the plain
// search (here H = I, P = 0, Imp = 1). "Add composable scale calibration to GPTQ" (PR #2004):
// 448-normalized NVFP4 global scale g = amax / (6 * 448).
#include "common.cuh"

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
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    m = max(m, abs_bits8<T>(base + i * 8));
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

__global__ void scale_from_amax_kernel(int32_t groups, float* __restrict__ g) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= groups) return;
  const float amax = __uint_as_float(reinterpret_cast<const uint32_t*>(g)[e]);
  g[e] = __fdiv_rn(amax, 2688.f);  // 6 * 448
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
                                 int64_t cin, float* g, cudaStream_t stream) {
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
  scale_from_amax_kernel<<<static_cast<unsigned>(ceil_div(groups, 256)), 256, 0, stream>>>(groups, g);
  return check_launch("global scale");
}

}  // namespace lhcal
