// lhcal_accumulate_noalloc: Hessian accumulation for callers that cannot allocate device
// memory. The split-partial workspace that lhcal_accumulate takes from its caller lives here
// in a fixed, file-scope device array instead, so the call needs nothing but its inputs and
// outputs. The calibration method itself has no such entry point; this is a deployment aid.
#include <mutex>

#include "common.cuh"

namespace lhcal {
namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(LHCAL_NOALLOC_SCRATCH_BYTES);

// Loaded into every device that uses this library and kept until the process exits.
static __device__ __align__(256) float g_noalloc_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code the symbol's name
// is only a host-side stand-in, so the address must come from the runtime, once per device,
// with that device current. It is cached for the life of the process: a cudaDeviceReset after
// the first call would reload the module elsewhere, which the header states is unsupported.
lhcal_status scratch_for_current_device(float** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(LHCAL_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(LHCAL_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(LHCAL_ERR_CUDA, "cudaGetSymbolAddress(scratch) on device %d: %s", dev, cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<float*>(g_scratch_addr[dev]);
  return LHCAL_OK;
}

}  // namespace
}  // namespace lhcal

using namespace lhcal;

extern "C" lhcal_status lhcal_accumulate_noalloc(lhcal_mode mode, lhcal_dtype dtype, const void* x, const void* xq,
                                                 int64_t tokens, int64_t cin, int64_t ldx, int32_t groups,
                                                 const int32_t* group_offsets, const int32_t* token_ids,
                                                 int32_t flags, float* h, float* p, void* stream) {
  clear_error();
  size_t need = 0;
  // Validates mode, dtype, cin, groups and tokens, and sizes the scratch exactly as
  // lhcal_accumulate sizes its workspace.
  const lhcal_status st = lhcal_accumulate_workspace(mode, dtype, tokens, cin, groups, &need);
  if (st != LHCAL_OK) return st;
  if (need > kScratchBytes)
    return fail(LHCAL_ERR_INVALID_ARG,
                "accumulate_noalloc: these sizes need %zu bytes of scratch, more than the fixed %zu bytes "
                "(LHCAL_NOALLOC_SCRATCH_BYTES); use lhcal_accumulate with a caller workspace",
                need, kScratchBytes);
  float* scratch = nullptr;
  if (need > 0) {
    const lhcal_status s2 = scratch_for_current_device(&scratch);
    if (s2 != LHCAL_OK) return s2;
  }
  // The kernels overwrite every partial they later reduce, so the scratch needs no clearing.
  return lhcal_accumulate(mode, dtype, x, xq, tokens, cin, ldx, groups, group_offsets, token_ids, flags, h, p,
                          scratch, need > 0 ? kScratchBytes : 0, stream);
}
