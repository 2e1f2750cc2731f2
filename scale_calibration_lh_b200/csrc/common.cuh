// Internal helpers shared by the liblhcal translation units (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <string>

#include "lhcal.h"

namespace lhcal {

// B200: 148 SMs. Work splits are a pure function of the problem size (not of the device
// queried at run time) so that results and workspace sizes are reproducible.
constexpr int kNumSms = 148;
constexpr int kBlock = LHCAL_BLOCK;
constexpr int kMaxMultipliers = LHCAL_MAX_MULTIPLIERS;

// Thread-local last-error message (lhcal_last_error_string).
void set_error(const char* fmt, ...);
void clear_error();

lhcal_status fail(lhcal_status st, const char* fmt, ...);

// Validates that `p` is device (or managed) memory of the current device, aligned to
// `align` bytes. `what` names the argument in the error message.
lhcal_status check_device_ptr(const void* p, size_t align, const char* what);

lhcal_status check_launch(const char* what);

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t imax64(int64_t a, int64_t b) { return a > b ? a : b; }
__host__ __device__ inline int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// ---- device helpers ---------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Loads 8 consecutive elements as fp32 (16-byte aligned source for bf16, 32-byte for fp32).
template <typename T>
__device__ __forceinline__ void load8(const T* src, float* out);

template <>
__device__ __forceinline__ void load8<float>(const float* src, float* out) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* src, float* out) {
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = __uint_as_float(u[i] << 16);
    out[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

// ---- launchers implemented in the kernel translation units --------------------------------

lhcal_status launch_sweep(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups,
                          int64_t rows, int64_t cin, const float* h, const float* p, const float* g,
                          uint8_t* codes, float* wq, float* loss, cudaStream_t stream);

lhcal_status launch_sweep_tc(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups,
                             int64_t rows, int64_t cin, const float* h, const float* p, const float* g,
                             uint8_t* codes, float* wq, float* loss, cudaStream_t stream);

// quant: the activation-aware variant with the input quantizer fused (X_q derived from x).
size_t accumulate_workspace_bytes(lhcal_mode mode, lhcal_dtype dtype, int64_t tokens, int64_t cin,
                                  int32_t groups, bool quant = false);

// act_gx != NULL (ACT_AWARE, bf16 only): X_q is not read but derived from x in the kernel by the
// NVFP4 activation fake quant with global scale *act_gx (xq must then be NULL).
lhcal_status launch_accumulate(lhcal_mode mode, lhcal_dtype dtype, const void* x, const void* xq,
                               int64_t tokens, int64_t cin, int64_t ldx, int32_t groups,
                               const int32_t* group_offsets, const int32_t* token_ids, int32_t flags,
                               float* h, float* p, void* workspace, cudaStream_t stream,
                               const float* act_gx = nullptr);

lhcal_status launch_act_fake_quant(const void* x, int64_t tokens, int64_t cin, int64_t ldx, const float* gx,
                                   void* xq, int64_t ldq, cudaStream_t stream);

lhcal_status launch_count_tokens(int32_t groups, int64_t tokens, const int32_t* group_offsets,
                                 int32_t flags, int64_t* counts, cudaStream_t stream);

lhcal_status launch_finalize(lhcal_mode mode, int32_t groups, int64_t cin, const int64_t* counts,
                             float* h, float* p, cudaStream_t stream);

lhcal_status launch_global_scale(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows,
                                 int64_t cin, float* g, cudaStream_t stream, float fp8_max = 448.f);

lhcal_status launch_multiplier_search(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows,
                                      int64_t cin, const float* h, const float* p, const float* g, const float* mult,
                                      int32_t n_mult, uint8_t* codes, float* wq, float* loss, cudaStream_t stream);

lhcal_status launch_apply_scales(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows, int64_t cin,
                                 const float* g, const uint8_t* codes, float* wq, void* wq16, float* amax,
                                 cudaStream_t stream);

}  // namespace lhcal
