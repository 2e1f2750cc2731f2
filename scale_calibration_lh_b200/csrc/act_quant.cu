// Standalone NVFP4 activation fake quant: X [tokens, cin] bf16 -> X_q bf16, the input
// quantizer of "Add activation-aware local Hessian scale calibration" (PR #1976, re-review).
// The same block quantizer runs inside the fused activation-aware accumulation; this kernel
// materialises X_q for callers that want it.
#include "common.cuh"
#include "act_quant.cuh"

namespace lhcal {
namespace {

constexpr int kQuantThreads = 256;

constexpr int kQuantRows = 4;  // (token, block) rows per thread and iteration, loads in flight together

// Each thread takes kQuantRows (token, block) rows per iteration: two 16-byte loads each, all
// issued before the first quantization, then the block quantizer and two 16-byte stores per
// row. Consecutive threads take consecutive blocks, so a warp moves 1 KB contiguously.
__global__ void __launch_bounds__(kQuantThreads)
act_quant_kernel(const __nv_bfloat16* __restrict__ x, int64_t tokens, int64_t nblk, int64_t ldx,
                 const float* __restrict__ gx_ptr, __nv_bfloat16* __restrict__ xq, int64_t ldq) {
  __shared__ ActQuantTables tab;
  const float gx = __ldg(gx_ptr);
  build_act_tables(tab, gx, threadIdx.x, blockDim.x);
  __syncthreads();
  const float inv6gx = 1.f / (6.f * gx);
  const bool steps = act_quant_steps(gx);
  const int64_t units = tokens * nblk;
  const int64_t span = static_cast<int64_t>(gridDim.x) * blockDim.x;  // distance between a thread's rows
  const int64_t span_tok = span / nblk, span_b = span - span_tok * nblk;
  for (int64_t u0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u0 < units;
       u0 += span * kQuantRows) {
    uint32_t xv[kQuantRows][8];
    int64_t tok[kQuantRows], b[kQuantRows];
    tok[0] = u0 / nblk;  // one division per kQuantRows rows; the others step by span
    b[0] = u0 - tok[0] * nblk;
#pragma unroll
    for (int r = 0; r < kQuantRows; ++r) {
      if (r > 0) {
        tok[r] = tok[r - 1] + span_tok;
        b[r] = b[r - 1] + span_b;
        if (b[r] >= nblk) {
          b[r] -= nblk;
          ++tok[r];
        }
      }
      const int64_t u = u0 + r * span;
      if (u < units) {
        const uint4* src = reinterpret_cast<const uint4*>(x + tok[r] * ldx + b[r] * kBlock);
        const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
        xv[r][0] = v0.x; xv[r][1] = v0.y; xv[r][2] = v0.z; xv[r][3] = v0.w;
        xv[r][4] = v1.x; xv[r][5] = v1.y; xv[r][6] = v1.z; xv[r][7] = v1.w;
      }
    }
#pragma unroll
    for (int r = 0; r < kQuantRows; ++r) {
      if (u0 + r * span >= units) break;
      uint32_t qv[8];
      act_quant_block(xv[r], qv, inv6gx, tab, steps);
      uint4* dst = reinterpret_cast<uint4*>(xq + tok[r] * ldq + b[r] * kBlock);
      dst[0] = make_uint4(qv[0], qv[1], qv[2], qv[3]);
      dst[1] = make_uint4(qv[4], qv[5], qv[6], qv[7]);
    }
  }
}

}  // namespace

lhcal_status launch_act_fake_quant(const void* x, int64_t tokens, int64_t cin, int64_t ldx, const float* gx,
                                   void* xq, int64_t ldq, cudaStream_t stream) {
  if (tokens == 0) return LHCAL_OK;
  const int64_t nblk = cin / kBlock;
  // 104 registers a thread (ptxas): two CTAs per SM; one wave of them loops over the rows.
  const int64_t blocks = imin64(ceil_div(tokens * nblk, kQuantThreads * kQuantRows), 2 * kNumSms);
  act_quant_kernel<<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), tokens, nblk, ldx, gx, static_cast<__nv_bfloat16*>(xq), ldq);
  return check_launch("activation fake quant");
}

}  // namespace lhcal
