// dd_verify_logits_static: the vocabulary verification pass without a caller
// workspace, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or hand us a buffer from their own
// allocator): code embedded in another runtime whose device memory is owned and
// budgeted by that runtime, latency-critical serving loops where cudaMalloc's
// implicit device synchronisation is not acceptable, or code that must not be
// able to fail with an out-of-memory error in the middle of a step. For them the
// per-row partial states that dd_verify_logits keeps in its workspace live in
// a fixed array in this library's own device memory instead.
#include <mutex>

#include "dd_common.cuh"
#include "dd_internal.h"

// The library's own scratch for dd_verify_logits_static. Every GPU that loads
// libdd holds this array until the process exits. In host code the name is
// only a stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_verify_scratch[DD_STATIC_SCRATCH_BYTES];

namespace dd {

namespace {

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {};

// Device address of the scratch array on the current device (set up on the
// first call on that device, with that device current).
dd_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_verify_scratch) != cudaSuccess || ptr == nullptr)
      return DD_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return DD_OK;
}

}  // namespace

}  // namespace dd

extern "C" dd_status dd_verify_logits_static(const void* logits_t, const void* logits_d,
                                             dd_dtype dtype, int B, int R, int V, int64_t ld,
                                             int pos_offset, float temperature, uint64_t seed,
                                             uint64_t step, const dd_row_stats* out,
                                             void* stream) {
  using namespace dd;
  if (!logits_t || !logits_d || !out) return DD_ERR_INVALID_ARG;
  if (dtype != DD_F32 && dtype != DD_BF16) return DD_ERR_INVALID_ARG;
  if (B < 1 || R < 1 || V < 1 || ld < V || pos_offset < 0) return DD_ERR_INVALID_ARG;
  if ((int64_t)B * R > (1ll << 27)) return DD_ERR_UNSUPPORTED;
  if (!(temperature >= 0.f) || isinf(temperature)) return DD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(logits_t) & 15u) || (reinterpret_cast<uintptr_t>(logits_d) & 15u))
    return DD_ERR_INVALID_ARG;
  const int64_t esize = dtype == DD_BF16 ? 2 : 4;
  if ((ld * esize) % 16 != 0) return DD_ERR_INVALID_ARG;
  // the partial states of this call must fit the fixed array
  if (verify_workspace_bytes(B, R, V, dtype) > (size_t)DD_STATIC_SCRATCH_BYTES)
    return DD_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const dd_status st = scratch_for_current_device(&scratch);
  if (st != DD_OK) return st;
  // Nothing in the scratch needs to start at zero: every partial the merge
  // kernel reads is written earlier in the same call.
  return launch_verify_logits(logits_t, logits_d, dtype, B, R, V, ld, pos_offset, temperature,
                              seed, step, *out, scratch, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? DD_OK
             : DD_ERR_CUDA;
}
