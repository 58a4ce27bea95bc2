// Fused vocabulary verification pass (dd_verify_logits) and the shared
// Gumbel noise writer (dd_coupled_gumbel).
//
// One streaming read of the verifier logits l and the drafter logits m of each
// verified row produces: LSE of both, argmax of both, the verifier's max
// probability, its entropy (the uncertainty u of COVER's seed score),
// KL(drafter || verifier), and at T > 0 the coupled Gumbel-max samples of
// both with the same Philox noise.
//
// Work decomposition: a row is split into C contiguous segments, one CTA each;
// the C CTAs of a row form a thread-block cluster and merge their partial
// states through distributed shared memory, so no global scratch is needed.
// Each thread streams 16-byte vectors with no-L1-allocate loads, four vectors
// of each matrix in flight, and keeps an online (running-max rescaled) state:
//   s1 = sum e^{x - M},  s2 = sum e^{x - M} (x - M) log2(e),  sk = sum e^{m - Md}(m - l)
// from which LSE = M + ln s1, H = ln s1 - s2 ln2 / s1, conf = 1 / s1,
// KL = sk_d / s1_d + (M_t - M_d) + ln(s1_t / s1_d).
#include <cooperative_groups.h>

#include "dd_common.cuh"
#include "dd_internal.h"

namespace cg = cooperative_groups;

namespace dd {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct Partial {
  float mt, s1t, s2t;  // verifier: max, sum e, sum e*y (log2 units)
  float md, s1d, skd;  // drafter: max, sum e, sum e*(m - l)
  int at, ad;          // argmaxes
  float bt, lt_at;     // best coupled score of l, and l at that index
  float bd;            // best coupled score of m
  int it, id;          // their indices
};

__device__ __forceinline__ void init(Partial& p) {
  p.mt = p.md = -INFINITY;
  p.s1t = p.s2t = p.s1d = p.skd = 0.f;
  p.at = p.ad = 0x7fffffff;
  p.bt = p.bd = -INFINITY;
  p.lt_at = 0.f;
  p.it = p.id = 0x7fffffff;
}

// Accumulate N consecutive vocabulary entries starting at index v0.
template <int N, bool SAMPLE>
__device__ __forceinline__ void accumulate(Partial& p, const float (&l)[N], const float (&m)[N],
                                           const float (&g)[N], int v0, float invT) {
  // --- verifier: maximum, argmax (lowest index), online rescale
  float cm = l[0];
#pragma unroll
  for (int i = 1; i < N; ++i) cm = fmaxf(cm, l[i]);
  if (cm > p.mt) {
    int a = v0 + N - 1;
#pragma unroll
    for (int i = N - 1; i >= 0; --i)
      if (l[i] == cm) a = v0 + i;
    if (p.mt != -INFINITY) {
      const float dl = (p.mt - cm) * kLog2e;
      const float f = exp2f(dl);
      p.s2t = f * (p.s2t + dl * p.s1t);
      p.s1t = f * p.s1t;
    }
    p.mt = cm;
    p.at = a;
  }
  const float mt2 = p.mt * kLog2e;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float y = fmaf(l[i], kLog2e, -mt2);
    const float e = fast_exp2(y);
    p.s1t += e;
    p.s2t = fmaf(e, y, p.s2t);
  }
  // --- drafter
  float dm = m[0];
#pragma unroll
  for (int i = 1; i < N; ++i) dm = fmaxf(dm, m[i]);
  if (dm > p.md) {
    int a = v0 + N - 1;
#pragma unroll
    for (int i = N - 1; i >= 0; --i)
      if (m[i] == dm) a = v0 + i;
    if (p.md != -INFINITY) {
      const float f = exp2f((p.md - dm) * kLog2e);
      p.s1d *= f;
      p.skd *= f;
    }
    p.md = dm;
    p.ad = a;
  }
  const float md2 = p.md * kLog2e;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float e = fast_exp2(fmaf(m[i], kLog2e, -md2));
    p.s1d += e;
    p.skd = fmaf(e, m[i] - l[i], p.skd);
  }
  // --- coupled Gumbel-max samples (same noise g for both)
  if constexpr (SAMPLE) {
    float st[N], sd[N];
    float bt = -INFINITY, bd = -INFINITY;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      st[i] = fmaf(l[i], invT, g[i]);
      sd[i] = fmaf(m[i], invT, g[i]);
      bt = fmaxf(bt, st[i]);
      bd = fmaxf(bd, sd[i]);
    }
    if (bt > p.bt) {
      int a = 0;
      float la = l[0];
#pragma unroll
      for (int i = N - 1; i >= 0; --i)
        if (st[i] == bt) { a = i; la = l[i]; }
      p.bt = bt;
      p.it = v0 + a;
      p.lt_at = la;
    }
    if (bd > p.bd) {
      int a = 0;
#pragma unroll
      for (int i = N - 1; i >= 0; --i)
        if (sd[i] == bd) a = i;
      p.bd = bd;
      p.id = v0 + a;
    }
  }
}

// Merge partial b into a (both cover disjoint vocabulary ranges).
template <bool SAMPLE>
__device__ __forceinline__ void merge(Partial& a, const Partial& b) {
  // verifier
  if (b.mt != -INFINITY) {
    if (a.mt == -INFINITY) {
      a.mt = b.mt; a.s1t = b.s1t; a.s2t = b.s2t; a.at = b.at;
    } else {
      const float M = fmaxf(a.mt, b.mt);
      const float da = (a.mt - M) * kLog2e, db = (b.mt - M) * kLog2e;
      const float fa = exp2f(da), fb = exp2f(db);
      a.s2t = fa * (a.s2t + da * a.s1t) + fb * (b.s2t + db * b.s1t);
      a.s1t = fa * a.s1t + fb * b.s1t;
      if (b.mt > a.mt || (b.mt == a.mt && b.at < a.at)) a.at = b.at;
      a.mt = M;
    }
  }
  // drafter
  if (b.md != -INFINITY) {
    if (a.md == -INFINITY) {
      a.md = b.md; a.s1d = b.s1d; a.skd = b.skd; a.ad = b.ad;
    } else {
      const float M = fmaxf(a.md, b.md);
      const float fa = exp2f((a.md - M) * kLog2e), fb = exp2f((b.md - M) * kLog2e);
      a.s1d = fa * a.s1d + fb * b.s1d;
      a.skd = fa * a.skd + fb * b.skd;
      if (b.md > a.md || (b.md == a.md && b.ad < a.ad)) a.ad = b.ad;
      a.md = M;
    }
  }
  if constexpr (SAMPLE) {
    if (b.bt > a.bt || (b.bt == a.bt && b.it < a.it)) { a.bt = b.bt; a.it = b.it; a.lt_at = b.lt_at; }
    if (b.bd > a.bd || (b.bd == a.bd && b.id < a.id)) { a.bd = b.bd; a.id = b.id; }
  }
}

__device__ __forceinline__ Partial shfl_down(const Partial& p, int delta) {
  Partial q;
  q.mt = __shfl_down_sync(0xffffffffu, p.mt, delta);
  q.s1t = __shfl_down_sync(0xffffffffu, p.s1t, delta);
  q.s2t = __shfl_down_sync(0xffffffffu, p.s2t, delta);
  q.md = __shfl_down_sync(0xffffffffu, p.md, delta);
  q.s1d = __shfl_down_sync(0xffffffffu, p.s1d, delta);
  q.skd = __shfl_down_sync(0xffffffffu, p.skd, delta);
  q.at = __shfl_down_sync(0xffffffffu, p.at, delta);
  q.ad = __shfl_down_sync(0xffffffffu, p.ad, delta);
  q.bt = __shfl_down_sync(0xffffffffu, p.bt, delta);
  q.lt_at = __shfl_down_sync(0xffffffffu, p.lt_at, delta);
  q.bd = __shfl_down_sync(0xffffffffu, p.bd, delta);
  q.it = __shfl_down_sync(0xffffffffu, p.it, delta);
  q.id = __shfl_down_sync(0xffffffffu, p.id, delta);
  return q;
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& u, float (&x)[8]) {
    x[0] = bf16lo(u.x); x[1] = bf16hi(u.x); x[2] = bf16lo(u.y); x[3] = bf16hi(u.y);
    x[4] = bf16lo(u.z); x[5] = bf16hi(u.z); x[6] = bf16lo(u.w); x[7] = bf16hi(u.w);
  }
  __device__ static float scalar(const __nv_bfloat16* p) { return __bfloat162float(*p); }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& u, float (&x)[4]) {
    x[0] = __uint_as_float(u.x); x[1] = __uint_as_float(u.y);
    x[2] = __uint_as_float(u.z); x[3] = __uint_as_float(u.w);
  }
  __device__ static float scalar(const float* p) { return *p; }
};

struct NoiseKey {
  uint32_t k0, k1, step;
};

// Gumbel noise of N consecutive entries starting at v0 (v0 % 4 == 0 when N >= 4).
template <int N>
__device__ __forceinline__ void noise(float (&g)[N], int v0, int pos, int b, const NoiseKey& key) {
  if constexpr (N >= 4) {
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
      const PhiloxOut o = philox4x32_10((uint32_t)(v0 >> 2) + q, (uint32_t)pos, (uint32_t)b,
                                        key.step, key.k0, key.k1);
#pragma unroll
      for (int w = 0; w < 4; ++w) g[4 * q + w] = gumbel_from_word(o.w[w]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const int v = v0 + i;
      const PhiloxOut o = philox4x32_10((uint32_t)(v >> 2), (uint32_t)pos, (uint32_t)b, key.step,
                                        key.k0, key.k1);
      g[i] = gumbel_from_word(o.w[v & 3]);
    }
  }
}

template <typename T, bool SAMPLE>
__global__ void __launch_bounds__(kThreads)
verify_logits_kernel(const T* __restrict__ lt, const T* __restrict__ lm, int R, int V,
                     int64_t ld, int pos_offset, float invT, NoiseKey key, int seg_len,
                     dd_row_stats out) {
  constexpr int VEC = Vec<T>::N;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / C;
  const int b = row / R;
  const int pos = pos_offset + row % R;
  const int seg0 = rank * seg_len;
  const int seg1 = min(V, seg0 + seg_len);
  const T* lrow = lt + (int64_t)row * ld;
  const T* mrow = lm + (int64_t)row * ld;

  Partial p;
  init(p);
  float gz[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) gz[i] = 0.f;

  if (seg0 < seg1) {
    const int nvec = (seg1 - seg0) / VEC;  // full vectors (seg0 is a multiple of 64)
    const uint4* lv = reinterpret_cast<const uint4*>(lrow + seg0);
    const uint4* mv = reinterpret_cast<const uint4*>(mrow + seg0);
    for (int base = threadIdx.x; base < nvec; base += kUnroll * kThreads) {
      uint4 a[kUnroll], c[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int idx = base + u * kThreads;
        if (idx < nvec) { a[u] = ld_stream(lv + idx); c[u] = ld_stream(mv + idx); }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int idx = base + u * kThreads;
        if (idx < nvec) {
          float x[VEC], y[VEC];
          Vec<T>::unpack(a[u], x);
          Vec<T>::unpack(c[u], y);
          const int v0 = seg0 + idx * VEC;
          if constexpr (SAMPLE) {
            float g[VEC];
            noise<VEC>(g, v0, pos, b, key);
            accumulate<VEC, SAMPLE>(p, x, y, g, v0, invT);
          } else {
            accumulate<VEC, SAMPLE>(p, x, y, gz, v0, invT);
          }
        }
      }
    }
    // ragged tail of the row (fewer than VEC entries), one entry per thread
    const int tail0 = seg0 + nvec * VEC;
    const int v = tail0 + threadIdx.x;
    if (v < seg1) {
      float x[1] = {Vec<T>::scalar(lrow + v)};
      float y[1] = {Vec<T>::scalar(mrow + v)};
      float g[1] = {0.f};
      if constexpr (SAMPLE) noise<1>(g, v, pos, b, key);
      accumulate<1, SAMPLE>(p, x, y, g, v, invT);
    }
  }

  // --- CTA reduction: warp shuffles, then across warps through shared memory
#pragma unroll
  for (int delta = 16; delta > 0; delta >>= 1) {
    const Partial q = shfl_down(p, delta);
    merge<SAMPLE>(p, q);
  }
  __shared__ Partial warp_part[kThreads / 32];
  __shared__ Partial cta_part;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) warp_part[warp] = p;
  __syncthreads();
  if (threadIdx.x == 0) {
    Partial acc = warp_part[0];
    for (int w = 1; w < kThreads / 32; ++w) merge<SAMPLE>(acc, warp_part[w]);
    cta_part = acc;
  }
  // --- cluster reduction through distributed shared memory
  cluster.sync();
  if (rank == 0 && threadIdx.x == 0) {
    Partial acc = cta_part;
    for (int r = 1; r < C; ++r) {
      const Partial* remote = cluster.map_shared_rank(&cta_part, r);
      merge<SAMPLE>(acc, *remote);
    }
    const float ln_s1t = logf(acc.s1t);
    const float lse_t = acc.mt + ln_s1t;
    const float lse_d = acc.md + logf(acc.s1d);
    const float conf = 1.f / acc.s1t;
    const float ent = ln_s1t - acc.s2t * kLn2 / acc.s1t;
    const float kl = acc.skd / acc.s1d + (acc.mt - acc.md) + logf(acc.s1t / acc.s1d);
    int st = acc.at, sd = acc.ad;
    float psamp = conf;
    if constexpr (SAMPLE) {
      st = acc.it;
      sd = acc.id;
      psamp = expf(acc.lt_at - lse_t);
    }
    if (out.lse_t) out.lse_t[row] = lse_t;
    if (out.lse_d) out.lse_d[row] = lse_d;
    if (out.conf_t) out.conf_t[row] = conf;
    if (out.p_sample_t) out.p_sample_t[row] = psamp;
    if (out.entropy_t) out.entropy_t[row] = ent;
    if (out.kl_dt) out.kl_dt[row] = kl;
    if (out.argmax_t) out.argmax_t[row] = acc.at;
    if (out.argmax_d) out.argmax_d[row] = acc.ad;
    if (out.sample_t) out.sample_t[row] = st;
    if (out.sample_d) out.sample_d[row] = sd;
  }
  cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
}

__global__ void coupled_gumbel_kernel(NoiseKey key, int R, int V, int64_t ld, int pos_offset,
                                      int64_t nquads_per_row, int64_t total_quads, float* g) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total_quads;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = t / nquads_per_row;
    const int qd = (int)(t % nquads_per_row);
    const int b = (int)(row / R);
    const int pos = pos_offset + (int)(row % R);
    const PhiloxOut o = philox4x32_10((uint32_t)qd, (uint32_t)pos, (uint32_t)b, key.step,
                                      key.k0, key.k1);
    float* dst = g + row * ld + 4 * (int64_t)qd;
#pragma unroll
    for (int w = 0; w < 4; ++w)
      if (4 * qd + w < V) dst[w] = gumbel_from_word(o.w[w]);
  }
}

template <typename T, bool SAMPLE>
cudaError_t launch_verify(const void* lt, const void* lm, int B, int R, int V, int64_t ld,
                          int pos_offset, float temperature, NoiseKey key,
                          const dd_row_stats& out, cudaStream_t stream) {
  auto kern = verify_logits_kernel<T, SAMPLE>;
  const int rows = B * R;
  const DeviceInfo& dev = device_info();
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0);
  if (err != cudaSuccess) return err;
  const int64_t slots = (int64_t)dev.sm_count * (per_sm > 0 ? per_sm : 1);
  // Split rows into C segments (a power of two <= 8) while the whole grid
  // still fits in one wave and every thread keeps at least 2 vectors per matrix.
  constexpr int VEC = Vec<T>::N;
  int C = 1;
  while (C < 8 && (int64_t)rows * (2 * C) <= slots &&
         (int64_t)V >= (int64_t)(2 * C) * kThreads * VEC * 2)
    C *= 2;
  int seg_len = (V + C - 1) / C;
  seg_len = (seg_len + 63) / 64 * 64;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float invT = temperature > 0.f ? 1.f / temperature : 0.f;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(lt), static_cast<const T*>(lm), R,
                            V, ld, pos_offset, invT, key, seg_len, out);
}

}  // namespace

cudaError_t launch_verify_logits(const void* lt, const void* lm, dd_dtype dtype, int B, int R,
                                 int V, int64_t ld, int pos_offset, float temperature,
                                 uint64_t seed, uint64_t step, const dd_row_stats& out,
                                 cudaStream_t stream) {
  NoiseKey key{(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32),
               (uint32_t)(step & 0xffffffffu)};
  const bool sample = temperature > 0.f;
  if (dtype == DD_BF16)
    return sample ? launch_verify<__nv_bfloat16, true>(lt, lm, B, R, V, ld, pos_offset,
                                                       temperature, key, out, stream)
                  : launch_verify<__nv_bfloat16, false>(lt, lm, B, R, V, ld, pos_offset,
                                                        temperature, key, out, stream);
  return sample ? launch_verify<float, true>(lt, lm, B, R, V, ld, pos_offset, temperature, key,
                                             out, stream)
                : launch_verify<float, false>(lt, lm, B, R, V, ld, pos_offset, temperature, key,
                                              out, stream);
}

cudaError_t launch_coupled_gumbel(uint64_t seed, uint64_t step, int B, int R, int V, int64_t ld,
                                  int pos_offset, float* g, cudaStream_t stream) {
  NoiseKey key{(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32),
               (uint32_t)(step & 0xffffffffu)};
  const int64_t nq = (V + 3) / 4;
  const int64_t total = (int64_t)B * R * nq;
  const DeviceInfo& dev = device_info();
  const int64_t want = (total + 255) / 256;
  const int grid = (int)(want < (int64_t)dev.sm_count * 8 ? want : (int64_t)dev.sm_count * 8);
  coupled_gumbel_kernel<<<grid > 0 ? grid : 1, 256, 0, stream>>>(key, R, V, ld, pos_offset, nq,
                                                                 total, g);
  return cudaGetLastError();
}

}  // namespace dd
