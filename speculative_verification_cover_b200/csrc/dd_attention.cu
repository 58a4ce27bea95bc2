// Dual-view attention (dd_dualview_attention): pass 1 (out, lse, d_out) and
// pass 2 (d_in), plus the small kernels around them.
//
// Dual view of COVER (cache override + leave-one-out): for query i, column j,
//   (k~, v~)_ij = (k_prev[j], v_prev[j]) if j is a seed and j != i, else (k_cur[j], v_cur[j]).
// Both passes stage a "view" tile in which every seed column already holds the
// step t-1 cache; the one element that differs per query -- a seed query's own
// column -- is skipped in the tile loop and merged back from k_cur / v_cur
// afterwards (one extra term of the online softmax).
//
// This file holds the CUDA-core (SIMT) implementation used for fp32 inputs,
// where the benchmark spec's tolerance (1e-4) rules out tf32 tensor cores, and the
// pieces shared with the tensor-core path in dd_attention_tc.cu.
#include "dd_common.cuh"
#include "dd_internal.h"

namespace dd {

AttnWorkspace attn_workspace_layout(int B, int L, int Hq, int Hkv, int d) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  AttnWorkspace w;
  const size_t part = (size_t)B * Hq * L * sizeof(float);
  w.dout_off = 0;
  w.din_off = up(w.dout_off + part);
  w.mrows_off = up(w.din_off + part);
  w.mcount_off = up(w.mrows_off + (size_t)B * L * sizeof(int32_t));
  const size_t words = (size_t)B * ((L + 31) / 32) * sizeof(uint32_t);
  w.newbits_off = up(w.mcount_off + (size_t)B * sizeof(int32_t));
  w.mrank_off = up(w.newbits_off + words);
  // tensor-core path: bf16 views and the compacted masked rows for pass 2
  w.Lp = (L + 127) / 128 * 128;
  const size_t kv = (size_t)B * L * Hkv * d * 2;
  w.kview_off = up(w.mrank_off + (size_t)B * L * sizeof(int32_t));
  w.vview_off = up(w.kview_off + kv);
  w.qm_off = up(w.vview_off + kv);
  w.lse2m_off = up(w.qm_off + (size_t)B * L * Hq * d * 2);
  w.total = up(w.lse2m_off + (size_t)B * Hq * w.Lp * sizeof(float));
  return w;
}

namespace {

// ---------------------------------------------------------------------------
// Everything the passes need from the flags, one launch, grid (1 + copy blocks, B):
//   block 0 of sequence b: the newly-written flags packed 32 to a word, the
//     masked query rows in ascending order (stable compaction), their count, and
//     each row's rank among them (-1 for a row that is not masked);
//   blocks 1.. (tensor-core path with seeds): the drafting view of K and V --
//     row j of the step t-1 cache where j is a seed, of the current input
//     otherwise -- so the attention passes stream plain tiles of it.
struct PrepArgs {
  const uint8_t *is_masked, *is_seed, *is_new;
  int L;
  int32_t *mrows, *mcount, *mrank;  // mrows == nullptr: no compaction
  uint32_t* newbits;
  // drafting view (view_units == 0: none); rows of row_units 16-byte units
  const uint4 *k_cur, *v_cur, *k_prev, *v_prev;
  uint4 *k_view, *v_view;
  int64_t view_units;  // per sequence: L * row_units
  int row_units;       // Hkv * d * 2 / 16
};
constexpr int kPrepThreads = 1024;
constexpr int kPrepUnitsPerThread = 4;

__global__ void __launch_bounds__(kPrepThreads) prep_kernel(const PrepArgs a) {
  // Pass 1 may take its SMs (and set up its barriers and tensor memory) while this
  // kernel runs; it reads nothing of ours before its pdl_wait().
  pdl_release();
  const int b = blockIdx.y;
  const int L = a.L;
  if (blockIdx.x > 0) {
    const int64_t base = (int64_t)b * a.view_units;
    const int64_t u0 = (int64_t)(blockIdx.x - 1) * (kPrepThreads * kPrepUnitsPerThread) + threadIdx.x;
    uint4 kv[kPrepUnitsPerThread], vv[kPrepUnitsPerThread];
#pragma unroll
    for (int e = 0; e < kPrepUnitsPerThread; ++e) {
      const int64_t u = u0 + e * kPrepThreads;
      if (u < a.view_units) {
        const int pos = (int)(u / a.row_units);
        const bool seed = a.is_seed[(int64_t)b * L + pos] != 0;
        kv[e] = (seed ? a.k_prev : a.k_cur)[base + u];
        vv[e] = (seed ? a.v_prev : a.v_cur)[base + u];
      }
    }
#pragma unroll
    for (int e = 0; e < kPrepUnitsPerThread; ++e) {
      const int64_t u = u0 + e * kPrepThreads;
      if (u < a.view_units) {
        a.k_view[base + u] = kv[e];
        a.v_view[base + u] = vv[e];
      }
    }
    return;
  }
  const int W = (L + 31) / 32;
  for (int i0 = threadIdx.x & ~31; i0 < W * 32; i0 += blockDim.x) {
    const int i = i0 + (threadIdx.x & 31);
    const bool fn = a.is_new != nullptr && i < L && a.is_new[(int64_t)b * L + i];
    const uint32_t wn = __ballot_sync(0xffffffffu, fn);
    if ((threadIdx.x & 31) == 0 && a.newbits) a.newbits[(int64_t)b * W + i0 / 32] = wn;
  }
  if (a.mrows == nullptr) return;
  __shared__ int warp_sums[32];
  __shared__ int base;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int c0 = 0; c0 < L; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    const int f = (a.is_masked != nullptr && i < L && a.is_masked[(int64_t)b * L + i]) ? 1 : 0;
    int incl = f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_sums[w];
    const int rank = base + before + incl - 1;
    if (f && DD_IN_BOUNDS(rank >= 0 && rank < L)) a.mrows[(int64_t)b * L + rank] = i;
    if (i < L) a.mrank[(int64_t)b * L + i] = f ? rank : -1;
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w = 0; w < nwarps; ++w) tot += warp_sums[w];
      base += tot;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) a.mcount[b] = base;
}

// d_x[b, j] = (accumulate ? d_x[b, j] : 0) + (1/Hq) sum_s part[b, s, j], s < nslices,
// for both statistics in one launch (part == nullptr skips one). Eight lanes per
// position, each summing every eighth slice, then a shuffle reduction: one
// round of memory latency whatever the head count.
struct HeadReduce {
  const float* part;
  int nslices;
  float* dst;
  int begin;  // positions before it have no partials: they contribute 0
};
__global__ void __launch_bounds__(256) head_reduce_kernel(HeadReduce r0, HeadReduce r1, int B, int L,
                                                          float inv_hq, int accumulate) {
  pdl_wait();  // launched as a dependent of the previous kernel
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t pos = t >> 3;
  const int sub = (int)(t & 7);
  if (pos >= (int64_t)B * L) return;  // whole groups of eight leave together
  const unsigned mask = 0xFFu << (threadIdx.x & 24);
  const int64_t b = pos / L;
  const int j = (int)(pos % L);
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const HeadReduce& r = which ? r1 : r0;
    if (r.part == nullptr) continue;
    const float* p = r.part + b * r.nslices * L + j;
    float acc = 0.f;
    if (j >= r.begin)
      for (int h = sub; h < r.nslices; h += 8) acc += p[(int64_t)h * L];
    acc += __shfl_xor_sync(mask, acc, 4);
    acc += __shfl_xor_sync(mask, acc, 2);
    acc += __shfl_xor_sync(mask, acc, 1);
    if (sub == 0) {
      const float v = acc * inv_hq;
      r.dst[pos] = accumulate ? r.dst[pos] + v : v;
    }
  }
}

// ---------------------------------------------------------------------------
// SIMT pass 1. Block: 32 query rows of one (b, h), 4 threads per row; thread q
// of a row owns 16-byte chunks q, q+4, q+8, ... of the head dimension.
template <typename T>
struct Ld;
template <>
struct Ld<float> {
  __device__ static float4 chunk(const float* p, int c) {
    return reinterpret_cast<const float4*>(p)[c];
  }
  __device__ static void store(float* p, int c, float4 v) { reinterpret_cast<float4*>(p)[c] = v; }
};
template <>
struct Ld<__nv_bfloat16> {
  // chunk c = elements 4c..4c+3
  __device__ static float4 chunk(const __nv_bfloat16* p, int c) {
    const uint2 u = reinterpret_cast<const uint2*>(p)[c];
    return make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
  }
  __device__ static void store(__nv_bfloat16* p, int c, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    reinterpret_cast<uint2*>(p)[c] = u;
  }
};

constexpr int kRows = 32;   // query rows per block
constexpr int kCols = 32;   // columns per staged tile

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

// Same, for code that only the four threads of one row execute together.
__device__ __forceinline__ float quad_sum_local(float x) {
  const unsigned mask = 0xFu << (threadIdx.x & 28);
  x += __shfl_xor_sync(mask, x, 1);
  x += __shfl_xor_sync(mask, x, 2);
  return x;
}

template <typename T, int D>
__global__ void __launch_bounds__(128) simt_pass1_kernel(AttnArgs a) {
  constexpr int NC = D / 16;  // float4 chunks per thread
  __shared__ float4 Ks[kCols][D / 4];
  __shared__ float4 Vs[kCols][D / 4];
  __shared__ uint8_t newflag[kCols];

  const int b = blockIdx.z, h = blockIdx.y;
  const int G = a.Hq / a.Hkv, g = h / G;
  const int r = threadIdx.x >> 2, qd = threadIdx.x & 3;
  const int i = a.q_begin + blockIdx.x * kRows + r;
  const bool valid = i < a.L;
  const int L = a.L;
  const T* qp = static_cast<const T*>(a.q);
  const T* kc = static_cast<const T*>(a.k_cur);
  const T* vc = static_cast<const T*>(a.v_cur);
  const T* kp = static_cast<const T*>(a.k_prev);
  const T* vp = static_cast<const T*>(a.v_prev);
  const float sl2 = a.scale * kLog2e;  // scores in log2 units

  float4 q[NC], o[NC];
  const T* qrow = qp + (((int64_t)b * L + (valid ? i : 0)) * a.Hq + h) * D;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    float4 x = Ld<T>::chunk(qrow, qd + 4 * c);
    q[c] = make_float4(x.x * sl2, x.y * sl2, x.z * sl2, x.w * sl2);
    o[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const bool seed_row = valid && a.is_seed != nullptr && a.is_seed[(int64_t)b * L + i];
  float m = -INFINITY, l = 0.f, ln = 0.f;

  for (int j0 = 0; j0 < L; j0 += kCols) {
    __syncthreads();
    // stage the view tile: seed columns from the cache
    for (int t = threadIdx.x; t < kCols * (D / 4); t += blockDim.x) {
      const int c = t / (D / 4), e = t % (D / 4);
      const int j = j0 + c;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (j < L) {
        const bool sj = a.is_seed != nullptr && a.is_seed[(int64_t)b * L + j];
        const int64_t off = (((int64_t)b * L + j) * a.Hkv + g) * D;
        kv = Ld<T>::chunk((sj ? kp : kc) + off, e);
        vv = Ld<T>::chunk((sj ? vp : vc) + off, e);
      }
      Ks[c][e] = kv;
      Vs[c][e] = vv;
    }
    for (int c = threadIdx.x; c < kCols; c += blockDim.x) {
      const int j = j0 + c;
      newflag[c] = (j < L && a.is_new != nullptr) ? a.is_new[(int64_t)b * L + j] : 0;
    }
    __syncthreads();
    float s[kCols];
    float tmax = -INFINITY;
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < NC; ++e) {
        const float4 kk = Ks[c][qd + 4 * e];
        part = fmaf(q[e].x, kk.x, part);
        part = fmaf(q[e].y, kk.y, part);
        part = fmaf(q[e].z, kk.z, part);
        part = fmaf(q[e].w, kk.w, part);
      }
      float sc = quad_sum(part);
      const int j = j0 + c;
      if (j >= L || (seed_row && j == i)) sc = -INFINITY;  // out of range / seed's own column
      s[c] = sc;
      tmax = fmaxf(tmax, sc);
    }
    if (tmax > m) {
      const float f = (m == -INFINITY) ? 0.f : exp2f(m - tmax);
      l *= f;
      ln *= f;
#pragma unroll
      for (int e = 0; e < NC; ++e) {
        o[e].x *= f; o[e].y *= f; o[e].z *= f; o[e].w *= f;
      }
      m = tmax;
    }
    if (m == -INFINITY) continue;
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      const float p = exp2f(s[c] - m);
      l += p;
      if (newflag[c]) ln += p;
#pragma unroll
      for (int e = 0; e < NC; ++e) {
        const float4 vv = Vs[c][qd + 4 * e];
        o[e].x = fmaf(p, vv.x, o[e].x);
        o[e].y = fmaf(p, vv.y, o[e].y);
        o[e].z = fmaf(p, vv.z, o[e].z);
        o[e].w = fmaf(p, vv.w, o[e].w);
      }
    }
  }

  // Leave-one-out diagonal of a seed query: its own column from the masked input.
  if (seed_row) {
    const int64_t off = (((int64_t)b * L + i) * a.Hkv + g) * D;
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < NC; ++e) {
      const float4 kk = Ld<T>::chunk(kc + off, qd + 4 * e);
      part += q[e].x * kk.x + q[e].y * kk.y + q[e].z * kk.z + q[e].w * kk.w;
    }
    const float sd = quad_sum_local(part);
    const float mn = fmaxf(m, sd);
    const float f = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    const float p = exp2f(sd - mn);
    l = l * f + p;
    const bool self_new = a.is_new != nullptr && a.is_new[(int64_t)b * L + i];
    ln = ln * f + (self_new ? p : 0.f);
#pragma unroll
    for (int e = 0; e < NC; ++e) {
      const float4 vv = Ld<T>::chunk(vc + off, qd + 4 * e);
      o[e].x = fmaf(p, vv.x, o[e].x * f);
      o[e].y = fmaf(p, vv.y, o[e].y * f);
      o[e].z = fmaf(p, vv.z, o[e].z * f);
      o[e].w = fmaf(p, vv.w, o[e].w * f);
    }
    m = mn;
  }
  if (!valid) return;
  const float inv = 1.f / l;
  T* orow = static_cast<T*>(a.out) + (((int64_t)b * L + i) * a.Hq + h) * D;
#pragma unroll
  for (int e = 0; e < NC; ++e)
    Ld<T>::store(orow, qd + 4 * e, make_float4(o[e].x * inv, o[e].y * inv, o[e].z * inv,
                                               o[e].w * inv));
  if (qd == 0) {
    a.lse[((int64_t)b * a.Hq + h) * L + i] = (m + log2f(l)) * kLn2;
    if (a.dout_part) a.dout_part[((int64_t)b * a.Hq + h) * L + i] = ln * inv;
  }
}

// SIMT pass 2: column masses of the masked queries. Block: 32 columns of one
// (b, h), 4 threads per column; loops over the masked rows of the sequence.
template <typename T, int D>
__global__ void __launch_bounds__(128) simt_pass2_kernel(AttnArgs a) {
  constexpr int NC = D / 16;
  constexpr int QR = 32;  // masked query rows staged per step
  __shared__ float4 Qs[QR][D / 4];
  __shared__ float lse2[QR];
  const int b = blockIdx.z, h = blockIdx.y;
  const int G = a.Hq / a.Hkv, g = h / G;
  const int L = a.L;
  const int c = threadIdx.x >> 2, qd = threadIdx.x & 3;
  const int j = blockIdx.x * kCols + c;
  const bool valid = j < L;
  const T* qp = static_cast<const T*>(a.q);
  const bool sj = valid && a.is_seed != nullptr && a.is_seed[(int64_t)b * L + j];
  const T* kbase = static_cast<const T*>(sj ? a.k_prev : a.k_cur);
  const float sl2 = a.scale * kLog2e;
  float4 k[NC];
  const T* krow = kbase + (((int64_t)b * L + (valid ? j : 0)) * a.Hkv + g) * D;
#pragma unroll
  for (int e = 0; e < NC; ++e) {
    const float4 x = Ld<T>::chunk(krow, qd + 4 * e);
    k[e] = make_float4(x.x * sl2, x.y * sl2, x.z * sl2, x.w * sl2);
  }
  const int nm0 = a.mcount[b];
  const int nm = DD_IN_BOUNDS(nm0 >= 0 && nm0 <= L) ? nm0 : 0;
  const int32_t* rows = a.mrows + (int64_t)b * L;
  const float* lse = a.lse + ((int64_t)b * a.Hq + h) * L;
  float acc = 0.f;
  for (int r0 = 0; r0 < nm; r0 += QR) {
    __syncthreads();
    for (int t = threadIdx.x; t < QR * (D / 4); t += blockDim.x) {
      const int rr = t / (D / 4), e = t % (D / 4);
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r0 + rr < nm) {
        const int row = rows[r0 + rr];
        if (DD_IN_BOUNDS(row >= 0 && row < L))
          x = Ld<T>::chunk(qp + (((int64_t)b * L + row) * a.Hq + h) * D, e);
      }
      Qs[rr][e] = x;
    }
    for (int t = threadIdx.x; t < QR; t += blockDim.x)
      lse2[t] = (r0 + t < nm && DD_IN_BOUNDS(rows[r0 + t] >= 0 && rows[r0 + t] < L))
                    ? lse[rows[r0 + t]] * kLog2e
                    : INFINITY;
    __syncthreads();
    const int nr = min(QR, nm - r0);
    for (int rr = 0; rr < nr; ++rr) {
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < NC; ++e) {
        const float4 qq = Qs[rr][qd + 4 * e];
        part = fmaf(qq.x, k[e].x, part);
        part = fmaf(qq.y, k[e].y, part);
        part = fmaf(qq.z, k[e].z, part);
        part = fmaf(qq.w, k[e].w, part);
      }
      acc += exp2f(quad_sum(part) - lse2[rr]);
    }
  }
  if (valid && qd == 0) a.din_part[((int64_t)b * a.Hq + h) * L + j] = acc;
}

template <typename T, int D>
cudaError_t launch_simt(const AttnArgs& a, cudaStream_t stream) {
  dim3 g1((a.L - a.q_begin + kRows - 1) / kRows, a.Hq, a.B);
  simt_pass1_kernel<T, D><<<g1, 128, 0, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (a.d_in && a.is_masked) {
    dim3 g2((a.L + kCols - 1) / kCols, a.Hq, a.B);
    simt_pass2_kernel<T, D><<<g2, 128, 0, stream>>>(a);
    err = cudaGetLastError();
  }
  return err;
}

}  // namespace

cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t stream, bool* handled,
                                int* din_slices);

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t stream, cudaEvent_t prep_done) {
  cudaError_t err;
  const bool need_din = a.d_in != nullptr && a.is_masked != nullptr;
  PrepArgs pa{};
  pa.is_masked = a.is_masked;
  pa.is_seed = a.is_seed;
  pa.is_new = a.is_new;
  pa.L = a.L;
  pa.mrows = need_din ? a.mrows : nullptr;
  pa.mcount = a.mcount;
  pa.mrank = a.mrank;
  pa.newbits = a.newbits;
  unsigned copy_blocks = 0;
  if (a.dtype == DD_BF16 && a.is_seed != nullptr) {
    // the tensor-core passes read the drafting view instead of patching tiles
    pa.k_cur = static_cast<const uint4*>(a.k_cur);
    pa.v_cur = static_cast<const uint4*>(a.v_cur);
    pa.k_prev = static_cast<const uint4*>(a.k_prev);
    pa.v_prev = static_cast<const uint4*>(a.v_prev);
    pa.k_view = static_cast<uint4*>(a.k_view);
    pa.v_view = static_cast<uint4*>(a.v_view);
    pa.row_units = a.Hkv * a.d * 2 / 16;
    pa.view_units = (int64_t)a.L * pa.row_units;
    const int64_t per_block = kPrepThreads * kPrepUnitsPerThread;
    copy_blocks = (unsigned)((pa.view_units + per_block - 1) / per_block);
  }
  prep_kernel<<<dim3(1 + copy_blocks, a.B), kPrepThreads, 0, stream>>>(pa);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if (prep_done != nullptr && (err = cudaEventRecord(prep_done, stream)) != cudaSuccess) return err;
  bool handled = false;
  int din_slices = a.Hq;  // d_in partials: per query head (CUDA-core pass 2) or per kv head
  if (a.dtype == DD_BF16) {
    err = launch_attention_tc(a, stream, &handled, &din_slices);
    if (err != cudaSuccess) return err;
  }
  if (!handled) {
    if (a.dtype == DD_F32)
      err = a.d == 64 ? launch_simt<float, 64>(a, stream) : launch_simt<float, 128>(a, stream);
    else
      err = a.d == 64 ? launch_simt<__nv_bfloat16, 64>(a, stream)
                      : launch_simt<__nv_bfloat16, 128>(a, stream);
    if (err != cudaSuccess) return err;
  }
  const int64_t total = (int64_t)a.B * a.L;
  HeadReduce rin{nullptr, 0, nullptr, 0}, rout{nullptr, 0, nullptr, 0};
  if (a.d_out) {
    if (a.is_new) rout = HeadReduce{a.dout_part, a.Hq, a.d_out, a.q_begin};
    else if (!a.accumulate) cudaMemsetAsync(a.d_out, 0, total * sizeof(float), stream);
  }
  if (a.d_in) {
    if (need_din) rin = HeadReduce{a.din_part, din_slices, a.d_in, 0};
    else if (!a.accumulate) cudaMemsetAsync(a.d_in, 0, total * sizeof(float), stream);
  }
  if (rin.part || rout.part) {
    err = launch_dependent(head_reduce_kernel, dim3((unsigned)((total * 8 + 255) / 256)), dim3(256),
                           0, stream, rin, rout, a.B, a.L, a.stats_weight / a.Hq, a.accumulate);
    if (err != cudaSuccess) return err;
  }
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  return cudaSuccess;
}

}  // namespace dd
