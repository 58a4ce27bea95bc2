// C ABI of libdd (include/dd.h): argument validation, workspace carve-up and
// kernel launches. No entry point allocates device memory.
#include <math.h>
#include <stdlib.h>

#include <mutex>

#include "dd_common.cuh"
#include "dd_internal.h"

namespace dd {

const DeviceInfo& device_info() {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    DeviceInfo d{};
    d.device = dev;
    cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    d.smem_optin = (size_t)optin;
    if (d.sm_count <= 0) d.sm_count = 1;
    cache[dev] = d;
    have[dev] = true;
  }
  return cache[dev];
}

static uint32_t g_spin_limit = [] {
  const char* e = getenv("DD_SPIN_LIMIT");
  if (e && *e) {
    const unsigned long v = strtoul(e, nullptr, 0);
    if (v > 0 && v <= 0xffffffffUL) return (uint32_t)v;
  }
  return (uint32_t)(1u << 26);
}();

uint32_t spin_limit() { return g_spin_limit; }

}  // namespace dd

using namespace dd;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dd_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DD_OK : DD_ERR_CUDA; }

size_t elem_size(dd_dtype t) { return t == DD_BF16 ? 2 : 4; }

bool valid_dtype(dd_dtype t) { return t == DD_F32 || t == DD_BF16; }

}  // namespace

extern "C" {

size_t dd_dualview_attention_workspace_size(int B, int L, int Hq, int Hkv, int d) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || d < 1) return 0;
  return attn_workspace_layout(B, L, Hq, Hkv, d).total;
}

dd_status dd_dualview_attention_ex2(const void* q, const void* k_cur, const void* v_cur,
                                    const void* k_prev, const void* v_prev, const uint8_t* is_seed,
                                    const uint8_t* is_masked, const uint8_t* is_new, int B, int L,
                                    int Hq, int Hkv, int d, float softmax_scale, dd_dtype dtype,
                                    int q_begin, int accumulate_stats, float stats_weight,
                                    void* out, float* lse, float* d_in, float* d_out,
                                    void* workspace, size_t workspace_bytes, void* prep_done,
                                    void* stream) {
  if (!q || !k_cur || !v_cur || !out || !lse) return DD_ERR_INVALID_ARG;
  if (q_begin < 0 || q_begin >= L) return DD_ERR_INVALID_ARG;
  if (!(stats_weight == stats_weight) || isinf(stats_weight)) return DD_ERR_INVALID_ARG;
  if (is_seed && (!k_prev || !v_prev)) return DD_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return DD_ERR_INVALID_ARG;
  if (B > 65535 || Hq > 65535) return DD_ERR_UNSUPPORTED;
  if (!valid_dtype(dtype)) return DD_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return DD_ERR_UNSUPPORTED;
  if (!(softmax_scale == softmax_scale) || isinf(softmax_scale)) return DD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(out) ||
      (k_prev && !aligned16(k_prev)) || (v_prev && !aligned16(v_prev)))
    return DD_ERR_INVALID_ARG;
  if (dtype == DD_BF16 && L > kTcMaxL) return DD_ERR_UNSUPPORTED;
  const AttnWorkspace ws = attn_workspace_layout(B, L, Hq, Hkv, d);
  if (!workspace || workspace_bytes < ws.total) return DD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DD_ERR_INVALID_ARG;
  AttnArgs a{};
  a.q = q; a.k_cur = k_cur; a.v_cur = v_cur; a.k_prev = k_prev; a.v_prev = v_prev;
  a.is_seed = is_seed; a.is_masked = is_masked; a.is_new = is_new;
  a.B = B; a.L = L; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.f / sqrtf((float)d);
  a.dtype = dtype;
  a.accumulate = accumulate_stats ? 1 : 0;
  a.q_begin = q_begin;
  a.stats_weight = stats_weight;
  a.out = out; a.lse = lse; a.d_in = d_in; a.d_out = d_out;
  char* w = static_cast<char*>(workspace);
  a.dout_part = reinterpret_cast<float*>(w + ws.dout_off);
  a.din_part = reinterpret_cast<float*>(w + ws.din_off);
  a.mrows = reinterpret_cast<int32_t*>(w + ws.mrows_off);
  a.mcount = reinterpret_cast<int32_t*>(w + ws.mcount_off);
  a.newbits = reinterpret_cast<uint32_t*>(w + ws.newbits_off);
  a.mrank = reinterpret_cast<int32_t*>(w + ws.mrank_off);
  a.k_view = w + ws.kview_off;
  a.v_view = w + ws.vview_off;
  a.q_m = w + ws.qm_off;
  a.lse2_m = reinterpret_cast<float*>(w + ws.lse2m_off);
  a.Lp = ws.Lp;
  return from_cuda(launch_attention(a, static_cast<cudaStream_t>(stream),
                                    static_cast<cudaEvent_t>(prep_done)));
}

dd_status dd_dualview_attention_ex(const void* q, const void* k_cur, const void* v_cur,
                                   const void* k_prev, const void* v_prev, const uint8_t* is_seed,
                                   const uint8_t* is_masked, const uint8_t* is_new, int B, int L,
                                   int Hq, int Hkv, int d, float softmax_scale, dd_dtype dtype,
                                   int q_begin, int accumulate_stats, float stats_weight,
                                   void* out, float* lse, float* d_in, float* d_out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  return dd_dualview_attention_ex2(q, k_cur, v_cur, k_prev, v_prev, is_seed, is_masked, is_new,
                                   B, L, Hq, Hkv, d, softmax_scale, dtype, q_begin,
                                   accumulate_stats, stats_weight, out, lse, d_in, d_out,
                                   workspace, workspace_bytes, nullptr, stream);
}

dd_status dd_dualview_attention(const void* q, const void* k_cur, const void* v_cur,
                                const void* k_prev, const void* v_prev, const uint8_t* is_seed,
                                const uint8_t* is_masked, const uint8_t* is_new, int B, int L,
                                int Hq, int Hkv, int d, float softmax_scale, dd_dtype dtype,
                                int accumulate_stats, void* out, float* lse, float* d_in,
                                float* d_out, void* workspace, size_t workspace_bytes,
                                void* stream) {
  if (L < 1) return DD_ERR_INVALID_ARG;
  return dd_dualview_attention_ex(q, k_cur, v_cur, k_prev, v_prev, is_seed, is_masked, is_new, B,
                                  L, Hq, Hkv, d, softmax_scale, dtype, 0, accumulate_stats, 1.f,
                                  out, lse, d_in, d_out, workspace, workspace_bytes, stream);
}

size_t dd_verify_logits_workspace_size(int B, int R, int V, dd_dtype dtype) {
  if (B < 1 || R < 1 || V < 1 || !valid_dtype(dtype)) return 0;
  if ((int64_t)B * R > (1ll << 27)) return 0;
  return verify_workspace_bytes(B, R, V, dtype);
}

dd_status dd_verify_logits(const void* logits_t, const void* logits_d, dd_dtype dtype, int B,
                           int R, int V, int64_t ld, int pos_offset, float temperature,
                           uint64_t seed, uint64_t step, const dd_row_stats* out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!logits_t || !logits_d || !out) return DD_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return DD_ERR_INVALID_ARG;
  if (B < 1 || R < 1 || V < 1 || ld < V || pos_offset < 0) return DD_ERR_INVALID_ARG;
  if ((int64_t)B * R > (1ll << 27)) return DD_ERR_UNSUPPORTED;
  if (!(temperature >= 0.f) || isinf(temperature)) return DD_ERR_INVALID_ARG;
  if (!aligned16(logits_t) || !aligned16(logits_d)) return DD_ERR_INVALID_ARG;
  if ((ld * (int64_t)elem_size(dtype)) % 16 != 0) return DD_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < verify_workspace_bytes(B, R, V, dtype))
    return DD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DD_ERR_INVALID_ARG;
  return from_cuda(launch_verify_logits(logits_t, logits_d, dtype, B, R, V, ld, pos_offset,
                                        temperature, seed, step, *out, workspace,
                                        static_cast<cudaStream_t>(stream)));
}

dd_status dd_coupled_gumbel(uint64_t seed, uint64_t step, int B, int R, int V, int64_t ld,
                            int pos_offset, float* g, void* stream) {
  if (!g || B < 1 || R < 1 || V < 1 || ld < V || pos_offset < 0) return DD_ERR_INVALID_ARG;
  return from_cuda(
      launch_coupled_gumbel(seed, step, B, R, V, ld, pos_offset, g, static_cast<cudaStream_t>(stream)));
}

dd_status dd_select_seeds_ex(const float* entropy, int R, int pos_offset, const float* d_in,
                             const float* d_out, const uint8_t* eligible, int B, int L, int k,
                             float min_score, int32_t* seeds, uint8_t* is_seed, float* score,
                             int32_t* count, void* stream) {
  if (!d_in || !d_out || !eligible) return DD_ERR_INVALID_ARG;
  if (!(min_score == min_score)) return DD_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || k < 0 || R < 0 || pos_offset < 0) return DD_ERR_INVALID_ARG;
  if (R > 0 && !entropy) return DD_ERR_INVALID_ARG;
  if (k > 0 && !seeds) return DD_ERR_INVALID_ARG;
  if (k > kSelectMaxK || L > kSelectMaxL) return DD_ERR_UNSUPPORTED;
  if (B > 2147483647 / 1) return DD_ERR_UNSUPPORTED;
  return from_cuda(launch_select_seeds(entropy, R, pos_offset, d_in, d_out, eligible, B, L, k,
                                       min_score, seeds, is_seed, score, count,
                                       static_cast<cudaStream_t>(stream)));
}

dd_status dd_select_seeds(const float* entropy, int R, int pos_offset, const float* d_in,
                          const float* d_out, const uint8_t* eligible, int B, int L, int k,
                          int32_t* seeds, uint8_t* is_seed, float* score, void* stream) {
  return dd_select_seeds_ex(entropy, R, pos_offset, d_in, d_out, eligible, B, L, k, -INFINITY,
                            seeds, is_seed, score, nullptr, stream);
}

dd_status dd_decide(const dd_decide_params* params, const int32_t* tokens,
                    const uint8_t* is_seed, const uint8_t* eligible, const dd_row_stats* stats,
                    int B, int L, int R, int pos_offset, uint8_t* decision, int32_t* new_tokens,
                    uint8_t* accepted, void* stream) {
  if (!params || !tokens || !stats || !decision || !new_tokens) return DD_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || R < 0 || pos_offset < 0) return DD_ERR_INVALID_ARG;
  const dd_decide_params& p = *params;
  if (!(p.temperature >= 0.f)) return DD_ERR_INVALID_ARG;
  if (!(p.tau_commit == p.tau_commit) || p.min_commit < 0 || p.min_commit > 1)
    return DD_ERR_INVALID_ARG;
  if (p.tau_commit > 0.f && !stats->p_sample_t) return DD_ERR_INVALID_ARG;
  const bool sampled = p.temperature > 0.f;
  if (sampled ? !stats->sample_t : !stats->argmax_t) return DD_ERR_INVALID_ARG;
  switch (p.policy) {
    case DD_POLICY_TRUST:
      if (!eligible) return DD_ERR_INVALID_ARG;
      break;
    case DD_POLICY_KL:
      if (!eligible || !stats->kl_dt) return DD_ERR_INVALID_ARG;
      break;
    case DD_POLICY_CONF:
      if (!eligible || !stats->conf_t) return DD_ERR_INVALID_ARG;
      break;
    case DD_POLICY_COVER:
      if (!is_seed || !stats->p_sample_t) return DD_ERR_INVALID_ARG;
      break;
    case DD_POLICY_COUPLED:
      if (!eligible || (sampled ? !stats->sample_d : !stats->argmax_d)) return DD_ERR_INVALID_ARG;
      if (p.tau_kl > 0.f && !stats->kl_dt) return DD_ERR_INVALID_ARG;
      break;
    case DD_POLICY_KL_STOCHASTIC:
      if (!eligible || !stats->kl_dt || !(p.tau_kl > 0.f)) return DD_ERR_INVALID_ARG;
      break;
    default:
      return DD_ERR_INVALID_ARG;
  }
  return from_cuda(launch_decide(p, tokens, is_seed, eligible, *stats, B, L, R, pos_offset,
                                 decision, new_tokens, accepted,
                                 static_cast<cudaStream_t>(stream)));
}

const char* dd_status_string(dd_status s) {
  switch (s) {
    case DD_OK: return "DD_OK";
    case DD_ERR_INVALID_ARG: return "DD_ERR_INVALID_ARG";
    case DD_ERR_UNSUPPORTED: return "DD_ERR_UNSUPPORTED";
    case DD_ERR_CUDA: return "DD_ERR_CUDA";
    case DD_ERR_TIMEOUT: return "DD_ERR_TIMEOUT";
    case DD_ERR_BOUNDS: return "DD_ERR_BOUNDS";
  }
  return "DD_UNKNOWN_STATUS";
}

dd_status dd_get_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DD_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return DD_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return DD_ERR_CUDA;
  return static_cast<dd_status>(v);
}

uint32_t dd_set_spin_limit(uint32_t limit) {
  const uint32_t old = g_spin_limit;
  if (limit > 0) g_spin_limit = limit;
  return old;
}

dd_status dd_selftest_bounded_wait(uint32_t limit, void* stream) {
  if (limit == 0) return DD_ERR_INVALID_ARG;
  return from_cuda(launch_selftest_wait(limit, static_cast<cudaStream_t>(stream)));
}

int dd_bounds_checked(void) {
#ifdef DD_CHECK_BOUNDS
  return 1;
#else
  return 0;
#endif
}

dd_status dd_selftest_bounds_check(int n, int index, int* value, void* stream) {
  if (!value || n < 0 || n > 64) return DD_ERR_INVALID_ARG;
  if (!dd_bounds_checked()) return DD_ERR_UNSUPPORTED;
  return from_cuda(launch_selftest_bounds(n, index, value, static_cast<cudaStream_t>(stream)));
}

dd_status dd_selftest_gumbel_screen(float* g_of_level, float* j_of_level, const float* g_req,
                                    float* limit, int n, float* gumbel_max, void* stream) {
  if (!g_of_level || !j_of_level || n < 0 || (n > 0 && (!g_req || !limit)))
    return DD_ERR_INVALID_ARG;
  if (gumbel_max) *gumbel_max = gumbel_max_constant();
  return from_cuda(launch_selftest_gumbel(g_of_level, j_of_level, g_req, limit, n,
                                          static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
