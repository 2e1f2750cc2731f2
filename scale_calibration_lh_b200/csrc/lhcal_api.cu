// C ABI of liblhcal.so: argument validation and dispatch to the kernel launchers.
//
// Validation follows the kernel contract stated in "Add activation-aware local Hessian scale
// calibration" (PR #1976), review comments (CUDA placement and numel validation), and the
// device fix embedded in "[2/3] Speed up layerwise GPTQ on MoE models" (#2877: a kernel
// launched on the current device with another device's pointers faults, so every pointer
// must belong to the current device).
#include <cstdarg>
#include <cstring>

#include "common.cuh"

namespace lhcal {

namespace {
thread_local char g_error[512] = "";
thread_local int64_t g_launches = 0;
}

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_error, sizeof(g_error), fmt, ap);
  va_end(ap);
}

void clear_error() { g_error[0] = '\0'; }

lhcal_status fail(lhcal_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_error, sizeof(g_error), fmt, ap);
  va_end(ap);
  return st;
}

lhcal_status check_device_ptr(const void* p, size_t align, const char* what) {
  if (p == nullptr) return fail(LHCAL_ERR_INVALID_ARG, "%s is NULL", what);
  if (!aligned(p, align)) return fail(LHCAL_ERR_INVALID_ARG, "%s is not %zu-byte aligned", what, align);
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error state of the runtime
    return fail(LHCAL_ERR_INVALID_ARG, "%s: cannot query pointer (%s)", what, cudaGetErrorString(e));
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(LHCAL_ERR_INVALID_ARG, "%s is not device memory", what);
  int dev = -1;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(LHCAL_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (attr.type == cudaMemoryTypeDevice && attr.device != dev)
    return fail(LHCAL_ERR_DEVICE_MISMATCH, "%s lives on device %d but device %d is current", what,
                attr.device, dev);
  return LHCAL_OK;
}

lhcal_status check_launch(const char* what) {
  ++g_launches;
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(LHCAL_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  return LHCAL_OK;
}

namespace {

// Modes with activation statistics (accumulate / finalize); the sweep also takes LHCAL_MSE.
bool valid_mode(lhcal_mode m) { return m == LHCAL_FULL || m == LHCAL_ACT_AWARE || m == LHCAL_DIAG; }
bool valid_sweep_mode(lhcal_mode m) { return valid_mode(m) || m == LHCAL_MSE; }
bool valid_dtype(lhcal_dtype d) { return d == LHCAL_F32 || d == LHCAL_BF16; }
size_t elt_size(lhcal_dtype d) { return d == LHCAL_F32 ? 4 : 2; }

lhcal_status check_cin(int64_t cin) {
  if (cin <= 0 || cin % LHCAL_BLOCK != 0)
    return fail(LHCAL_ERR_INVALID_ARG, "cin (%lld) must be a positive multiple of 16", (long long)cin);
  if (cin / LHCAL_BLOCK > 65535)
    return fail(LHCAL_ERR_INVALID_ARG, "cin (%lld) too large (at most 65535 blocks)", (long long)cin);
  return LHCAL_OK;
}

lhcal_status check_groups(int32_t groups) {
  if (groups < 1 || groups > 65535)
    return fail(LHCAL_ERR_INVALID_ARG, "groups (%d) must be in [1, 65535]", groups);
  return LHCAL_OK;
}

#define LHCAL_TRY(expr)                         \
  do {                                          \
    const lhcal_status st_ = (expr);            \
    if (st_ != LHCAL_OK) return st_;            \
  } while (0)

// Validation shared by lhcal_accumulate and lhcal_accumulate_act_quant (act_gx != NULL: X_q is
// derived from x in the kernel, xq must be NULL).
lhcal_status accumulate_checked(lhcal_mode mode, lhcal_dtype dtype, const void* x, const void* xq, int64_t tokens,
                                int64_t cin, int64_t ldx, int32_t groups, const int32_t* group_offsets,
                                const int32_t* token_ids, int32_t flags, float* h, float* p, void* workspace,
                                size_t workspace_bytes, void* stream, const float* act_gx) {
  if (!valid_mode(mode) || !valid_dtype(dtype)) return fail(LHCAL_ERR_UNSUPPORTED, "unknown mode or dtype");
  LHCAL_TRY(check_cin(cin));
  LHCAL_TRY(check_groups(groups));
  if (tokens < 0) return fail(LHCAL_ERR_INVALID_ARG, "tokens (%lld) is negative", (long long)tokens);
  if (tokens > (int64_t)INT32_MAX)
    return fail(LHCAL_ERR_INVALID_ARG, "tokens (%lld) must fit in int32", (long long)tokens);
  if (ldx < cin) return fail(LHCAL_ERR_INVALID_ARG, "ldx (%lld) < cin (%lld)", (long long)ldx, (long long)cin);
  if ((ldx * (int64_t)elt_size(dtype)) % 16 != 0)
    return fail(LHCAL_ERR_INVALID_ARG, "ldx * element size must be a multiple of 16 bytes");
  if (flags != LHCAL_ACCUM_ADD && flags != LHCAL_ACCUM_OVERWRITE)
    return fail(LHCAL_ERR_INVALID_ARG, "unknown flags %d", flags);
  const bool grouped = group_offsets != nullptr || token_ids != nullptr;
  if (grouped && (group_offsets == nullptr || token_ids == nullptr))
    return fail(LHCAL_ERR_INVALID_ARG, "group_offsets and token_ids must both be set or both be NULL");
  if (!grouped && groups != 1) return fail(LHCAL_ERR_INVALID_ARG, "groups > 1 needs group_offsets and token_ids");
  if (mode == LHCAL_ACT_AWARE && xq == nullptr && act_gx == nullptr)
    return fail(LHCAL_ERR_INVALID_ARG, "ACT_AWARE needs xq");
  if (mode != LHCAL_ACT_AWARE && (xq != nullptr || p != nullptr))
    return fail(LHCAL_ERR_INVALID_ARG, "xq and p are only for ACT_AWARE");
  const size_t need = accumulate_workspace_bytes(mode, dtype, tokens, cin, groups, act_gx != nullptr);
  if (workspace_bytes < need)
    return fail(LHCAL_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
  if (tokens > 0 || grouped) {
    LHCAL_TRY(check_device_ptr(x, 16, "x"));
    if (mode == LHCAL_ACT_AWARE && act_gx == nullptr) LHCAL_TRY(check_device_ptr(xq, 16, "xq"));
  }
  if (act_gx != nullptr) LHCAL_TRY(check_device_ptr(act_gx, 4, "act_gx"));
  if (grouped) {
    LHCAL_TRY(check_device_ptr(group_offsets, 4, "group_offsets"));
    LHCAL_TRY(check_device_ptr(token_ids, 4, "token_ids"));
  }
  LHCAL_TRY(check_device_ptr(h, 16, "h"));
  if (mode == LHCAL_ACT_AWARE) LHCAL_TRY(check_device_ptr(p, 16, "p"));
  if (need > 0) LHCAL_TRY(check_device_ptr(workspace, 256, "workspace"));
  return launch_accumulate(mode, dtype, x, xq, tokens, cin, ldx, groups, group_offsets, token_ids, flags, h, p,
                           workspace, static_cast<cudaStream_t>(stream), act_gx);
}

}  // namespace
}  // namespace lhcal

using namespace lhcal;

extern "C" {

int32_t lhcal_version(void) { return 100; }

const char* lhcal_last_error_string(void) { return g_error; }

int64_t lhcal_launch_count(int32_t reset) {
  const int64_t n = g_launches;
  if (reset) g_launches = 0;
  return n;
}

lhcal_status lhcal_accumulate_workspace(lhcal_mode mode, lhcal_dtype dtype, int64_t tokens, int64_t cin,
                                        int32_t groups, size_t* bytes) {
  clear_error();
  if (bytes == nullptr) return fail(LHCAL_ERR_INVALID_ARG, "bytes is NULL");
  if (!valid_mode(mode) || !valid_dtype(dtype)) return fail(LHCAL_ERR_UNSUPPORTED, "unknown mode or dtype");
  LHCAL_TRY(check_cin(cin));
  LHCAL_TRY(check_groups(groups));
  if (tokens < 0) return fail(LHCAL_ERR_INVALID_ARG, "tokens (%lld) is negative", (long long)tokens);
  *bytes = accumulate_workspace_bytes(mode, dtype, tokens, cin, groups);
  return LHCAL_OK;
}

lhcal_status lhcal_accumulate(lhcal_mode mode, lhcal_dtype dtype, const void* x, const void* xq,
                              int64_t tokens, int64_t cin, int64_t ldx, int32_t groups,
                              const int32_t* group_offsets, const int32_t* token_ids, int32_t flags,
                              float* h, float* p, void* workspace, size_t workspace_bytes, void* stream) {
  clear_error();
  return accumulate_checked(mode, dtype, x, xq, tokens, cin, ldx, groups, group_offsets, token_ids, flags, h, p,
                            workspace, workspace_bytes, stream, nullptr);
}

lhcal_status lhcal_accumulate_act_quant_workspace(lhcal_dtype dtype, int64_t tokens, int64_t cin, int32_t groups,
                                                  size_t* bytes) {
  clear_error();
  if (bytes == nullptr) return fail(LHCAL_ERR_INVALID_ARG, "bytes is NULL");
  if (dtype != LHCAL_BF16) return fail(LHCAL_ERR_UNSUPPORTED, "the fused input quantizer takes bf16 activations");
  LHCAL_TRY(check_cin(cin));
  LHCAL_TRY(check_groups(groups));
  if (tokens < 0) return fail(LHCAL_ERR_INVALID_ARG, "tokens (%lld) is negative", (long long)tokens);
  *bytes = accumulate_workspace_bytes(LHCAL_ACT_AWARE, dtype, tokens, cin, groups, true);
  return LHCAL_OK;
}

lhcal_status lhcal_accumulate_act_quant(lhcal_dtype dtype, const void* x, int64_t tokens, int64_t cin,
                                        int64_t ldx, int32_t groups, const int32_t* group_offsets,
                                        const int32_t* token_ids, const float* act_gx, int32_t flags,
                                        float* h, float* p, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  clear_error();
  if (dtype != LHCAL_BF16) return fail(LHCAL_ERR_UNSUPPORTED, "the fused input quantizer takes bf16 activations");
  if (act_gx == nullptr) return fail(LHCAL_ERR_INVALID_ARG, "act_gx is NULL");
  return accumulate_checked(LHCAL_ACT_AWARE, dtype, x, nullptr, tokens, cin, ldx, groups, group_offsets, token_ids,
                            flags, h, p, workspace, workspace_bytes, stream, act_gx);
}

lhcal_status lhcal_act_fake_quant(lhcal_dtype dtype, const void* x, int64_t tokens, int64_t cin, int64_t ldx,
                                  const float* act_gx, void* xq, int64_t ldxq, void* stream) {
  clear_error();
  if (dtype != LHCAL_BF16) return fail(LHCAL_ERR_UNSUPPORTED, "the activation quantizer takes bf16");
  LHCAL_TRY(check_cin(cin));
  if (tokens < 0) return fail(LHCAL_ERR_INVALID_ARG, "tokens (%lld) is negative", (long long)tokens);
  if (ldx < cin || ldxq < cin)
    return fail(LHCAL_ERR_INVALID_ARG, "row strides (%lld, %lld) must be >= cin (%lld)", (long long)ldx,
                (long long)ldxq, (long long)cin);
  if ((ldx * 2) % 16 != 0 || (ldxq * 2) % 16 != 0)
    return fail(LHCAL_ERR_INVALID_ARG, "row strides * 2 must be multiples of 16 bytes");
  LHCAL_TRY(check_device_ptr(act_gx, 4, "act_gx"));
  if (tokens == 0) return LHCAL_OK;
  LHCAL_TRY(check_device_ptr(x, 16, "x"));
  LHCAL_TRY(check_device_ptr(xq, 16, "xq"));
  return launch_act_fake_quant(x, tokens, cin, ldx, act_gx, xq, ldxq, static_cast<cudaStream_t>(stream));
}

lhcal_status lhcal_count_tokens(int32_t groups, int64_t tokens, const int32_t* group_offsets, int32_t flags,
                                int64_t* counts, void* stream) {
  clear_error();
  LHCAL_TRY(check_groups(groups));
  if (tokens < 0) return fail(LHCAL_ERR_INVALID_ARG, "tokens (%lld) is negative", (long long)tokens);
  if (flags != LHCAL_ACCUM_ADD && flags != LHCAL_ACCUM_OVERWRITE)
    return fail(LHCAL_ERR_INVALID_ARG, "unknown flags %d", flags);
  if (group_offsets == nullptr && groups != 1)
    return fail(LHCAL_ERR_INVALID_ARG, "groups > 1 needs group_offsets");
  if (group_offsets != nullptr) LHCAL_TRY(check_device_ptr(group_offsets, 4, "group_offsets"));
  LHCAL_TRY(check_device_ptr(counts, 8, "counts"));
  return launch_count_tokens(groups, tokens, group_offsets, flags, counts, static_cast<cudaStream_t>(stream));
}

lhcal_status lhcal_finalize(lhcal_mode mode, int32_t groups, int64_t cin, const int64_t* counts, float* h,
                            float* p, void* stream) {
  clear_error();
  if (!valid_mode(mode)) return fail(LHCAL_ERR_UNSUPPORTED, "unknown mode");
  LHCAL_TRY(check_cin(cin));
  LHCAL_TRY(check_groups(groups));
  if (mode != LHCAL_ACT_AWARE && p != nullptr) return fail(LHCAL_ERR_INVALID_ARG, "p is only for ACT_AWARE");
  LHCAL_TRY(check_device_ptr(counts, 8, "counts"));
  LHCAL_TRY(check_device_ptr(h, 16, "h"));
  if (mode == LHCAL_ACT_AWARE) LHCAL_TRY(check_device_ptr(p, 16, "p"));
  return launch_finalize(mode, groups, cin, counts, h, p, static_cast<cudaStream_t>(stream));
}

lhcal_status lhcal_global_scale(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows, int64_t cin,
                                float* g, void* stream) {
  clear_error();
  if (!valid_dtype(dtype)) return fail(LHCAL_ERR_UNSUPPORTED, "unknown dtype");
  LHCAL_TRY(check_cin(cin));
  LHCAL_TRY(check_groups(groups));
  if (rows <= 0) return fail(LHCAL_ERR_INVALID_ARG, "rows (%lld) must be positive", (long long)rows);
  LHCAL_TRY(check_device_ptr(w, 16, "w"));
  LHCAL_TRY(check_device_ptr(g, 4, "g"));
  return launch_global_scale(dtype, w, groups, rows, cin, g, static_cast<cudaStream_t>(stream));
}

lhcal_status lhcal_global_scale_ex(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows, int64_t cin,
                                   float fp8_max, float* g, void* stream) {
  clear_error();
  if (!valid_dtype(dtype)) return fail(LHCAL_ERR_UNSUPPORTED, "unknown dtype");
  if (!(fp8_max > 0.f && fp8_max <= 448.f) || static_cast<double>(6.f * fp8_max) != 6.0 * fp8_max)
    return fail(LHCAL_ERR_INVALID_ARG, "fp8_max (%g) must be in (0, 448] with 6 * fp8_max exact in fp32",
                static_cast<double>(fp8_max));
  LHCAL_TRY(check_cin(cin));
  LHCAL_TRY(check_groups(groups));
  if (rows <= 0) return fail(LHCAL_ERR_INVALID_ARG, "rows (%lld) must be positive", (long long)rows);
  LHCAL_TRY(check_device_ptr(w, 16, "w"));
  LHCAL_TRY(check_device_ptr(g, 4, "g"));
  return launch_global_scale(dtype, w, groups, rows, cin, g, static_cast<cudaStream_t>(stream), fp8_max);
}

lhcal_status lhcal_apply_scales(lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows, int64_t cin,
                                const float* g, const uint8_t* codes, float* wq, void* wq16, float* amax,
                                void* stream) {
  clear_error();
  if (!valid_dtype(dtype)) return fail(LHCAL_ERR_UNSUPPORTED, "unknown dtype");
  LHCAL_TRY(check_cin(cin));
  LHCAL_TRY(check_groups(groups));
  if (rows <= 0) return fail(LHCAL_ERR_INVALID_ARG, "rows (%lld) must be positive", (long long)rows);
  LHCAL_TRY(check_device_ptr(w, 16, "w"));
  LHCAL_TRY(check_device_ptr(g, 4, "g"));
  LHCAL_TRY(check_device_ptr(codes, 1, "codes"));
  if (wq != nullptr) LHCAL_TRY(check_device_ptr(wq, 16, "wq"));
  if (wq16 != nullptr) LHCAL_TRY(check_device_ptr(wq16, 16, "wq16"));
  if (amax != nullptr) LHCAL_TRY(check_device_ptr(amax, 4, "amax"));
  return launch_apply_scales(dtype, w, groups, rows, cin, g, codes, wq, wq16, amax, static_cast<cudaStream_t>(stream));
}

lhcal_status lhcal_multiplier_search(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups,
                                     int64_t rows, int64_t cin, const float* h, const float* p, const float* g,
                                     const float* multipliers, int32_t n_multipliers, uint8_t* codes, float* wq,
                                     float* loss, void* stream) {
  clear_error();
  if (!valid_sweep_mode(mode) || !valid_dtype(dtype)) return fail(LHCAL_ERR_UNSUPPORTED, "unknown mode or dtype");
  LHCAL_TRY(check_cin(cin));
  LHCAL_TRY(check_groups(groups));
  if (rows <= 0) return fail(LHCAL_ERR_INVALID_ARG, "rows (%lld) must be positive", (long long)rows);
  if (n_multipliers < 1 || n_multipliers > LHCAL_MAX_MULTIPLIERS)
    return fail(LHCAL_ERR_INVALID_ARG, "n_multipliers (%d) must be in [1, %d]", n_multipliers, LHCAL_MAX_MULTIPLIERS);
  if (mode == LHCAL_MSE && (h != nullptr || p != nullptr)) return fail(LHCAL_ERR_INVALID_ARG, "MSE takes no h or p");
  if (mode == LHCAL_ACT_AWARE && p == nullptr) return fail(LHCAL_ERR_INVALID_ARG, "ACT_AWARE needs p");
  if (mode != LHCAL_ACT_AWARE && p != nullptr) return fail(LHCAL_ERR_INVALID_ARG, "p is only for ACT_AWARE");
  LHCAL_TRY(check_device_ptr(w, 16, "w"));
  if (mode != LHCAL_MSE) LHCAL_TRY(check_device_ptr(h, 16, "h"));
  if (mode == LHCAL_ACT_AWARE) LHCAL_TRY(check_device_ptr(p, 16, "p"));
  LHCAL_TRY(check_device_ptr(g, 4, "g"));
  LHCAL_TRY(check_device_ptr(multipliers, 4, "multipliers"));
  LHCAL_TRY(check_device_ptr(codes, 1, "codes"));
  if (wq != nullptr) LHCAL_TRY(check_device_ptr(wq, 16, "wq"));
  if (loss != nullptr) LHCAL_TRY(check_device_ptr(loss, 4, "loss"));
  if (ceil_div(rows, 128) > 0x7fffffff) return fail(LHCAL_ERR_INVALID_ARG, "rows (%lld) too large", (long long)rows);
  return launch_multiplier_search(mode, dtype, w, groups, rows, cin, h, p, g, multipliers, n_multipliers, codes, wq,
                                  loss, static_cast<cudaStream_t>(stream));
}

lhcal_status lhcal_scale_sweep(lhcal_mode mode, lhcal_dtype dtype, const void* w, int32_t groups, int64_t rows,
                               int64_t cin, const float* h, const float* p, const float* g, uint8_t* codes,
                               float* wq, float* loss, void* stream) {
  clear_error();
  if (!valid_sweep_mode(mode) || !valid_dtype(dtype)) return fail(LHCAL_ERR_UNSUPPORTED, "unknown mode or dtype");
  if (mode == LHCAL_MSE && (h != nullptr || p != nullptr))
    return fail(LHCAL_ERR_INVALID_ARG, "MSE takes no h or p");
  LHCAL_TRY(check_cin(cin));
  LHCAL_TRY(check_groups(groups));
  if (rows <= 0) return fail(LHCAL_ERR_INVALID_ARG, "rows (%lld) must be positive", (long long)rows);
  if (rows > (int64_t)INT32_MAX) return fail(LHCAL_ERR_INVALID_ARG, "rows (%lld) too large", (long long)rows);
  if (mode == LHCAL_ACT_AWARE && p == nullptr) return fail(LHCAL_ERR_INVALID_ARG, "ACT_AWARE needs p");
  if (mode != LHCAL_ACT_AWARE && p != nullptr) return fail(LHCAL_ERR_INVALID_ARG, "p is only for ACT_AWARE");
  LHCAL_TRY(check_device_ptr(w, 16, "w"));
  if (mode != LHCAL_MSE) LHCAL_TRY(check_device_ptr(h, 16, "h"));
  if (mode == LHCAL_ACT_AWARE) LHCAL_TRY(check_device_ptr(p, 16, "p"));
  LHCAL_TRY(check_device_ptr(g, 4, "g"));
  LHCAL_TRY(check_device_ptr(codes, 1, "codes"));
  if (wq != nullptr) LHCAL_TRY(check_device_ptr(wq, 16, "wq"));
  if (loss != nullptr) LHCAL_TRY(check_device_ptr(loss, 4, "loss"));
  return launch_sweep(mode, dtype, w, groups, rows, cin, h, p, g, codes, wq, loss, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
