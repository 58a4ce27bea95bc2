// Stability-aware seed selection (dd_select_seeds), the verification
// decisions (dd_decide) and the bounded-wait self-test.
#include "dd_common.cuh"
#include "dd_internal.h"

namespace dd {

namespace {

constexpr int kSelThreads = 512;

// Order-preserving map of a float onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t orderable(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum of one int per thread (blockDim.x multiple of 32).
__device__ __forceinline__ int block_exclusive_sum(int x, int* warp_tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = lane < nw ? warp_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    if (lane < nw) warp_tmp[lane] = v;  // inclusive over warps
    if (lane == nw - 1) *total = v;
  }
  __syncthreads();
  const int before = warp > 0 ? warp_tmp[warp - 1] : 0;
  const int r = before + incl - x;
  __syncthreads();
  return r;
}

// One CTA per sequence.
//   score_i = u_i (1 + d_in_i) / (1 + d_out_i) on eligible positions with a row.
// The k-th largest score (as an order-preserving 32-bit key) is found by an
// MSB-first radix select, 8 bits per pass; positions tied with it are taken in
// ascending order up to k (a block prefix count); the chosen positions are
// ranked by (score descending, position ascending).
__global__ void __launch_bounds__(kSelThreads)
select_seeds_kernel(const float* __restrict__ entropy, int R, int pos_offset,
                    const float* __restrict__ d_in, const float* __restrict__ d_out,
                    const uint8_t* __restrict__ eligible, int L, int k, float min_score,
                    int32_t* __restrict__ seeds, uint8_t* __restrict__ is_seed,
                    float* __restrict__ score, int32_t* __restrict__ count) {
  pdl_wait();  // launched as a dependent of the previous kernel
  extern __shared__ uint32_t skey[];  // [L] orderable score; 0 = not a candidate
  __shared__ unsigned int hist[256];
  __shared__ int warp_tmp[32];
  __shared__ int total_s, nsel_s, ncand_s;
  __shared__ uint32_t prefix_s;
  __shared__ int need_s;
  __shared__ unsigned long long chosen[kSelectMaxK];
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) { ncand_s = 0; nsel_s = 0; }
  for (int t = threadIdx.x; t < 256; t += blockDim.x) hist[t] = 0u;
  __syncthreads();
  int my_cand = 0;
  for (int i = threadIdx.x; i < L; i += blockDim.x) {
    const int64_t bi = (int64_t)b * L + i;
    const int r = i - pos_offset;
    const bool has_row = r >= 0 && r < R;
    // all four loads at once (one memory round trip); positions without a row read
    // row 0 (entropy may be NULL only when R = 0)
    const uint8_t el = eligible[bi];
    const float u = R > 0 ? entropy[(int64_t)b * R + (has_row ? r : 0)] : 0.f;
    const float di = d_in[bi], dout = d_out[bi];
    float s = -INFINITY;
    uint32_t key = 0u;
    if (el && has_row) {
      s = u * (1.f + di) / (1.f + dout);
      if (s >= min_score) {  // the adaptive set: only scores reaching the floor compete
        key = orderable(s);
        ++my_cand;
      }
    }
    skey[i] = key;
    if (score) score[bi] = s;
  }
  if (my_cand) atomicAdd(&ncand_s, my_cand);
  __syncthreads();
  const int ncand = ncand_s;
  const int kk = k < ncand ? k : ncand;
  // ---- the kk-th largest key (keys are > 0 for candidates)
  uint32_t thresh = 1u;
  int need = 0;  // how many keys equal to thresh are taken
  if (kk > 0 && kk < ncand) {
    uint32_t prefix = 0u;
    int want = kk;
    for (int shift = 24; shift >= 0; shift -= 8) {
      const uint32_t hmask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
      for (int i = threadIdx.x; i < L; i += blockDim.x) {
        const uint32_t key = skey[i];
        if (key != 0u && (key & hmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (threadIdx.x < 32) {
        // lane handles digits 255-8*lane .. 248-8*lane (descending)
        unsigned int c[8], sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { c[e] = hist[255 - 8 * lane - e]; sum += c[e]; }
        unsigned int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        unsigned int run = incl - sum;  // keys with a larger digit than this lane's first
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (run < (unsigned)want && run + c[e] >= (unsigned)want) {
            prefix_s = prefix | ((uint32_t)(255 - 8 * lane - e) << shift);
            need_s = want - (int)run;
          }
          run += c[e];
        }
      }
      __syncthreads();
      prefix = prefix_s;
      want = need_s;
      for (int t = threadIdx.x; t < 256; t += blockDim.x) hist[t] = 0u;
      __syncthreads();
    }
    thresh = prefix;
    need = want;
  }
  // ---- choose: keys above the threshold, then the first `need` ties by position
  for (int i0 = 0; i0 < L; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    const uint32_t key = i < L ? skey[i] : 0u;
    const bool tie = kk > 0 && key != 0u && key == thresh && kk < ncand;
    const int before = block_exclusive_sum(tie ? 1 : 0, warp_tmp, &total_s);
    if (i < L) {
      const bool sel = kk > 0 && key != 0u && (kk >= ncand ? true : (key > thresh ||
                                                                     (tie && before < need)));
      if (sel) {
        const int slot = atomicAdd(&nsel_s, 1);
        if (DD_IN_BOUNDS(slot < kSelectMaxK))
          chosen[slot] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)i);
      }
      if (is_seed) is_seed[(int64_t)b * L + i] = sel ? 1 : 0;
    }
    if (kk < ncand) {
      need -= total_s;
      if (need < 0) need = 0;
    }
  }
  __syncthreads();
  const int nsel = DD_IN_BOUNDS(nsel_s <= kSelectMaxK && nsel_s <= k) ? nsel_s : 0;
  for (int t = threadIdx.x; t < nsel; t += blockDim.x) {
    const unsigned long long key = chosen[t];
    int rank = 0;
    for (int u = 0; u < nsel; ++u) rank += chosen[u] > key;
    if (DD_IN_BOUNDS(rank < k))
      seeds[(int64_t)b * k + rank] = (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
  }
  for (int t = nsel + threadIdx.x; t < k; t += blockDim.x) seeds[(int64_t)b * k + t] = -1;
  if (count && threadIdx.x == 0) count[b] = nsel;
}

// One CTA per sequence; accepted[b] = all decided positions of the policy's domain
// KEEP. Dynamic threshold decoding commits masked positions with p(pred) >= tau_commit;
// with min_commit, a sequence where none does commits its most confident one (a
// block-wide max of (p, -position) keys).
__global__ void __launch_bounds__(1024)
decide_kernel(dd_decide_params p, const int32_t* __restrict__ tokens,
              const uint8_t* __restrict__ is_seed, const uint8_t* __restrict__ eligible,
              dd_row_stats st, int L, int R, int pos_offset, uint8_t* __restrict__ decision,
              int32_t* __restrict__ new_tokens, uint8_t* __restrict__ accepted) {
  pdl_wait();  // launched as a dependent of the previous kernel
  const int b = blockIdx.x;
  const bool sampled = p.temperature > 0.f;
  const bool commit_on = p.tau_commit > 0.f;
  __shared__ unsigned long long best_key;  // most confident masked position: (p, -pos)
  if (threadIdx.x == 0) best_key = 0ull;
  __syncthreads();
  int all_keep = 1, committed = 0;
  for (int i = threadIdx.x; i < L; i += blockDim.x) {
    const int64_t bi = (int64_t)b * L + i;
    const int r = i - pos_offset;
    const int32_t cur = tokens[bi];
    const uint8_t* domain = p.policy == DD_POLICY_COVER ? is_seed : eligible;
    const bool in = r >= 0 && r < R && domain != nullptr && domain[bi];
    uint8_t dcs = DD_NONE;
    int32_t tok = cur;
    if (in) {
      const int64_t row = (int64_t)b * R + r;
      const int32_t pred = sampled ? st.sample_t[row] : st.argmax_t[row];
      switch (p.policy) {
        case DD_POLICY_TRUST:
          dcs = DD_KEEP;
          break;
        case DD_POLICY_KL:
          dcs = st.kl_dt[row] > p.tau_kl ? DD_REMASK : DD_KEEP;
          break;
        case DD_POLICY_CONF:
          dcs = st.conf_t[row] < p.tau_conf ? DD_REMASK : DD_KEEP;
          break;
        case DD_POLICY_COVER:
          if (pred == cur) dcs = DD_KEEP;
          else dcs = st.p_sample_t[row] >= p.tau_conf ? DD_REPLACE : DD_REMASK;
          break;
        case DD_POLICY_COUPLED: {
          const int32_t sd = sampled ? st.sample_d[row] : st.argmax_d[row];
          if (sd == pred) dcs = DD_KEEP;
          else if (p.tau_kl > 0.f && st.kl_dt[row] > p.tau_kl) dcs = DD_REMASK;
          else dcs = DD_REPLACE;
          break;
        }
        case DD_POLICY_KL_STOCHASTIC: {
          // REMASK with probability min(1, KL / tau), decided as U * tau < KL in fp32
          const PhiloxOut o = philox4x32_10(0x80000000u, (uint32_t)i, (uint32_t)b,
                                            (uint32_t)p.step, (uint32_t)p.seed,
                                            (uint32_t)(p.seed >> 32));
          const float u = uniform_from_word(o.w[0]);
          dcs = __fmul_rn(u, p.tau_kl) < st.kl_dt[row] ? DD_REMASK : DD_KEEP;
          break;
        }
        default:
          break;
      }
      if (dcs == DD_REPLACE || (dcs == DD_KEEP && p.policy == DD_POLICY_COUPLED)) tok = pred;
      else if (dcs == DD_REMASK) tok = DD_MASK_TOKEN;
      if (dcs != DD_KEEP) all_keep = 0;
    } else if (commit_on && cur == DD_MASK_TOKEN && r >= 0 && r < R) {
      const int64_t row = (int64_t)b * R + r;
      const float pp = st.p_sample_t[row];
      if (pp >= p.tau_commit) {
        dcs = DD_COMMIT;
        tok = sampled ? st.sample_t[row] : st.argmax_t[row];
        committed = 1;
      } else if (p.min_commit) {
        atomicMax(&best_key, ((unsigned long long)orderable(pp) << 32) | (0xFFFFFFFFu - (uint32_t)i));
      }
    }
    decision[bi] = dcs;
    new_tokens[bi] = tok;
  }
  const int acc = __syncthreads_and(all_keep);
  const int any_commit = __syncthreads_or(committed);
  if (accepted && threadIdx.x == 0) accepted[b] = (uint8_t)acc;
  if (p.min_commit && !any_commit && threadIdx.x == 0 && best_key != 0ull) {
    // progress: nothing passed the threshold, so the most confident masked position commits
    const int i = (int)(0xFFFFFFFFu - (uint32_t)(best_key & 0xFFFFFFFFull));
    const int64_t row = (int64_t)b * R + (i - pos_offset);
    if (DD_IN_BOUNDS(i >= 0 && i < L && i - pos_offset >= 0 && i - pos_offset < R)) {
      decision[(int64_t)b * L + i] = DD_COMMIT;
      new_tokens[(int64_t)b * L + i] = sampled ? st.sample_t[row] : st.argmax_t[row];
    }
  }
}

// Failure-detection self-test: wait on an mbarrier that nobody arrives on.
__global__ void selftest_wait_kernel(uint32_t limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, limit);
  __syncthreads();
}

}  // namespace

cudaError_t launch_select_seeds(const float* entropy, int R, int pos_offset, const float* d_in,
                                const float* d_out, const uint8_t* eligible, int B, int L, int k,
                                float min_score, int32_t* seeds, uint8_t* is_seed, float* score,
                                int32_t* count, cudaStream_t stream) {
  const size_t smem = (size_t)L * sizeof(uint32_t);
  static thread_local int configured_for = -1;
  const DeviceInfo& dev = device_info();
  if (configured_for != dev.device) {
    cudaError_t e = cudaFuncSetAttribute(select_seeds_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(kSelectMaxL * sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    configured_for = dev.device;
  }
  return launch_dependent(select_seeds_kernel, dim3(B), dim3(kSelThreads), smem, stream, entropy, R,
                          pos_offset, d_in, d_out, eligible, L, k, min_score, seeds, is_seed,
                          score, count);
}

cudaError_t launch_decide(const dd_decide_params& p, const int32_t* tokens,
                          const uint8_t* is_seed, const uint8_t* eligible,
                          const dd_row_stats& stats, int B, int L, int R, int pos_offset,
                          uint8_t* decision, int32_t* new_tokens, uint8_t* accepted,
                          cudaStream_t stream) {
  return launch_dependent(decide_kernel, dim3(B), dim3(1024), 0, stream, p, tokens, is_seed, eligible,
                          stats, L, R, pos_offset, decision, new_tokens, accepted);
}

// Self-test of the checked build: fill a 64-int array, then read element `index`
// of its first n through the checked path (-1 when the check skips the read).
// Without DD_CHECK_BOUNDS the read is not compiled at all.
__device__ int g_bounds_probe[64];
__device__ int g_bounds_probe_out;
__global__ void selftest_bounds_kernel(int n, int index) {
  for (int t = threadIdx.x; t < 64; t += blockDim.x) g_bounds_probe[t] = 3 * t + 1;
  __syncthreads();
  if (threadIdx.x != 0) return;
  int v = -1;
#ifdef DD_CHECK_BOUNDS
  if (DD_IN_BOUNDS(index >= 0 && index < n)) v = g_bounds_probe[index];
#else
  (void)n;
  (void)index;
#endif
  g_bounds_probe_out = v;
}

cudaError_t launch_selftest_bounds(int n, int index, int* value, cudaStream_t stream) {
  selftest_bounds_kernel<<<1, 64, 0, stream>>>(n, index);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbolAsync(value, g_bounds_probe_out, sizeof(int), 0,
                                cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(stream);
}

cudaError_t launch_selftest_wait(uint32_t limit, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(limit);
  return cudaGetLastError();
}

}  // namespace dd
