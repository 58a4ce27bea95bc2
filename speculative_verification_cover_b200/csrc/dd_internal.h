// Internal launcher interface between the C ABI (dd_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dd.h"

namespace dd {

struct DeviceInfo {
  int device;
  int sm_count;
  int cc_major, cc_minor;
  size_t smem_optin;
};
// Properties of the current device, cached per device.
const DeviceInfo& device_info();

// Bound of every device-side wait (iterations).
uint32_t spin_limit();

struct AttnArgs {
  const void *q, *k_cur, *v_cur, *k_prev, *v_prev;
  const uint8_t *is_seed, *is_masked, *is_new;
  int B, L, Hq, Hkv, d;
  float scale;          // softmax scale (natural units)
  dd_dtype dtype;
  int accumulate;
  int q_begin;          // first query row computed (rows before it: a cached prefix)
  float stats_weight;   // this call's d_in / d_out are added with this weight
  void* out;
  float* lse;
  float *d_in, *d_out;
  // workspace carve-up
  float* dout_part;     // [B, Hq, L]
  float* din_part;      // [B, Hq, L]
  int32_t* mrows;       // [B, L] masked rows of each sequence, ascending
  int32_t* mcount;      // [B]
  uint32_t* newbits;    // [B, ceil(L/32)] packed is_new
  int32_t* mrank;       // [B, L] rank of a masked row among its sequence's masked rows, else -1
  // tensor-core path only (bf16)
  void *k_view, *v_view;  // [B, L, Hkv, d] drafting view: seed rows from the cache, others current
  void* q_m;              // [B, L, Hq, d] masked query rows in rank order (rows >= count unset)
  float* lse2_m;          // [B, Hq, Lp] lse (log2 units) of masked rows in rank order
  int Lp;                 // L rounded up to 128
};

// Workspace layout shared by the entry point and the kernels.
struct AttnWorkspace {
  size_t dout_off, din_off, mrows_off, mcount_off, newbits_off, mrank_off;
  size_t kview_off, vview_off, qm_off, lse2m_off, total;
  int Lp;
};
AttnWorkspace attn_workspace_layout(int B, int L, int Hq, int Hkv, int d);

// prep_done (may be null) is recorded on the stream right after the mask preparation.
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t stream, cudaEvent_t prep_done);

// Launch `kernel` so that it may start while the previous kernel on `stream` is still
// finishing (programmatic stream serialization); the kernel calls pdl_wait() before
// it touches that kernel's data.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_verify_logits(const void* lt, const void* lm, dd_dtype dtype, int B, int R,
                                 int V, int64_t ld, int pos_offset, float temperature,
                                 uint64_t seed, uint64_t step, const dd_row_stats& out,
                                 void* workspace, cudaStream_t stream);
size_t verify_workspace_bytes(int B, int R, int V, dd_dtype dtype);

cudaError_t launch_coupled_gumbel(uint64_t seed, uint64_t step, int B, int R, int V, int64_t ld,
                                  int pos_offset, float* g, cudaStream_t stream);

cudaError_t launch_select_seeds(const float* entropy, int R, int pos_offset, const float* d_in,
                                const float* d_out, const uint8_t* eligible, int B, int L, int k,
                                float min_score, int32_t* seeds, uint8_t* is_seed, float* score,
                                int32_t* count, cudaStream_t stream);

cudaError_t launch_decide(const dd_decide_params& p, const int32_t* tokens,
                          const uint8_t* is_seed, const uint8_t* eligible,
                          const dd_row_stats& stats, int B, int L, int R, int pos_offset,
                          uint8_t* decision, int32_t* new_tokens, uint8_t* accepted,
                          cudaStream_t stream);

cudaError_t launch_selftest_wait(uint32_t limit, cudaStream_t stream);
cudaError_t launch_selftest_bounds(int n, int index, int* value, cudaStream_t stream);
cudaError_t launch_selftest_gumbel(float* g_of_k, float* j_of_k, const float* g_req,
                                   float* limit, int n, cudaStream_t stream);
float gumbel_max_constant();

// Largest L dd_select_seeds handles (keys of one sequence live in shared memory).
constexpr int kSelectMaxL = 24576;
// Longest sequence the tensor-core attention handles (a sequence's packed newly-written
// flags live in shared memory).
constexpr int kTcMaxL = 32768;
constexpr int kSelectMaxK = 1024;

}  // namespace dd
