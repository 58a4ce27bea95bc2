// Fused vocabulary verification pass (dd_verify_logits) and the shared
// Gumbel noise writer (dd_coupled_gumbel).
//
// One streaming read of the verifier logits l and the drafter logits m of each
// verified row produces: LSE of both, argmax of both, the verifier's max
// probability, its entropy (the uncertainty u of COVER's seed score),
// KL(drafter || verifier), and at T > 0 the coupled Gumbel-max samples of both
// with the same Philox noise. The exact Gumbel value of an entry is computed only
// where the entry could still be sampled: a 16-byte vector whose logits cannot
// reach the best score its warp holds even with the largest possible noise draws
// no noise at all, and one whose generator words all lie below the level it would
// need is dropped after an integer comparison (see fold()).
//
// Work decomposition: the 16-byte vectors of all rows form one index space
// (rows x vectors per row); it is split into equal contiguous ranges, one per
// persistent CTA (several per SM), so every SM streams the same number of bytes
// whatever B, R and V are. A CTA's range is one to a few row pieces; in each
// piece its 128 threads stride over the vectors, two per matrix per half-step,
// each thread staging its own 16-byte vectors through a ring of three half-steps
// in shared memory (cp.async), and fold each into an online (running-max
// rescaled) state kept in float2 lanes so pairs of entries use the packed fp32
// pipe:
//   s1 = sum e^{x - M},  s2 = sum e^{x - M} (x - M) log2(e),  sk = sum e^{m - Md}(m - l).
// At the end of a piece the CTA reduces its state to one partial per
// (row, CTA) in the workspace; a small second kernel merges a row's partials:
//   LSE = M + ln s1, H = ln s1 - s2 ln2 / s1, conf = 1 / s1,
//   KL = sk_d / s1_d + (M_t - M_d) + ln(s1_t / s1_d).
#include "dd_common.cuh"
#include "dd_internal.h"
#include "dd_tc.cuh"

namespace dd {

namespace {

constexpr int kVThreads = 128;
// Launch shape. Each thread stages its own vectors in a shared-memory ring of
// kStages half-steps (cp.async), so loads in flight cost no registers. CTAs are
// small -- 128 threads, about 10 K registers and 24 KB of shared memory at T = 0 --
// so that one fits on an SM beside a CTA of the attention's pass 1 (the two calls of a
// verification step run side by side) and the SM's several CTAs share its bandwidth
// in fine steps. The sampling pass needs about 120 registers: 4 CTAs per SM.
template <bool SAMPLE>
struct VCfg {
  static constexpr int kMinBlocks = SAMPLE ? 4 : 6;  // resident CTAs per SM
  static constexpr int kStages = 3;
  static constexpr int kRingBytes = kStages * 4 * kVThreads * 16;  // [stage][l0 l1 m0 m1][thread]
};
constexpr int kMaxGridPerSm = 6;  // bounds the grid for workspace sizing

struct Partial {
  float mt, s1t, s2t;  // verifier: max, sum e, sum e*y (log2 units)
  float md, s1d, skd;  // drafter: max, sum e, sum e*(m - l)
  int at, ad;          // argmaxes
  float bt, lt_at;     // best coupled score of l, and l at that index
  float bd;            // best coupled score of m
  int it, id;          // their indices
  int pad[3];
};
static_assert(sizeof(Partial) == 64, "partial record is 64 bytes");

struct NoiseKey {
  uint32_t k0, k1, step;
};

__device__ __forceinline__ void init(Partial& p) {
  p.mt = p.md = -INFINITY;
  p.s1t = p.s2t = p.s1d = p.skd = 0.f;
  p.at = p.ad = 0x7fffffff;
  p.bt = p.bd = -INFINITY;
  p.lt_at = 0.f;
  p.it = p.id = 0x7fffffff;
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

// Per-thread accumulator: the sums are float2 so that pairs of vocabulary
// entries go through the packed fp32 pipe (FFMA2 / FADD2) and each sum has two
// independent dependency chains. The exponentials are taken against a
// reference (ref_t / ref_d) that is moved only when the running maximum grows
// by more than kRefMargin, so rescaling is rare; the exact maxima (mt / md) and
// the 16-byte vector where each first appeared (vt / vd) are tracked with two
// selects, and the element index inside that vector is recovered at flush time.
// A negative vt / vd encodes an exact element index (-1 - index).
constexpr float kRefMargin = 20.f;  // e^20 headroom: sums stay far from fp32 overflow

struct Acc {
  float mt, md;        // exact running maxima of l and m
  float ref_t, ref_d;  // exponent references
  float2 s1t, s2t, s1d, skd;
  int vt, vd;          // where the maxima were first seen
  float bt, bd;        // best coupled scores
  int vbt, vbd;        // where they were first seen
};

__device__ __forceinline__ void init(Acc& a) {
  a.mt = a.md = a.ref_t = a.ref_d = -INFINITY;
  a.s1t = a.s2t = a.s1d = a.skd = make_float2(0.f, 0.f);
  a.vt = a.vd = a.vbt = a.vbd = 0x7fffffff;
  a.bt = a.bd = -INFINITY;
}

__device__ __forceinline__ float2 ex2x2(float2 y) {
  return make_float2(fast_exp2(y.x), fast_exp2(y.y));
}

__device__ __forceinline__ uint32_t hmax2_bits(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a);
  __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&b);
  __nv_bfloat162 r = __hmax2(x, y);
  return *reinterpret_cast<uint32_t*>(&r);
}

// Fold NV 16-byte vectors of each matrix (vector k starts at vocabulary index v0[k],
// indices increasing with k). l/m: the unpacked values; lw/mw: the raw words.

template <typename T>
struct Unpack;
template <>
struct Unpack<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void run(const uint4& u, float2 (&x)[4]) {
    x[0] = make_float2(bf16lo(u.x), bf16hi(u.x));
    x[1] = make_float2(bf16lo(u.y), bf16hi(u.y));
    x[2] = make_float2(bf16lo(u.z), bf16hi(u.z));
    x[3] = make_float2(bf16lo(u.w), bf16hi(u.w));
  }
  __device__ static float vmax(const uint4& u) {
    const uint32_t h = hmax2_bits(hmax2_bits(u.x, u.y), hmax2_bits(u.z, u.w));
    return fmaxf(bf16lo(h), bf16hi(h));
  }
  // entries 2e, 2e + 1 of the vector
  __device__ static float2 pair(const uint4& u, int e) {
    const uint32_t w = e == 0 ? u.x : e == 1 ? u.y : e == 2 ? u.z : u.w;
    return make_float2(bf16lo(w), bf16hi(w));
  }
};
template <>
struct Unpack<float> {
  static constexpr int N = 4;
  __device__ static void run(const uint4& u, float2 (&x)[2]) {
    x[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
    x[1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
  }
  __device__ static float vmax(const uint4& u) {
    return fmaxf(fmaxf(__uint_as_float(u.x), __uint_as_float(u.y)),
                 fmaxf(__uint_as_float(u.z), __uint_as_float(u.w)));
  }
  __device__ static float2 pair(const uint4& u, int e) {
    return e == 0 ? make_float2(__uint_as_float(u.x), __uint_as_float(u.y))
                  : make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
  }
};

// ---------------------------------------------------------------------------
// Exact coupled scores, evaluated by the warp together.
//
// A lane whose 16-byte vector passes the noise screen does not evaluate it on its
// own (that would hold the whole warp for the few lanes that need it); it pushes
// the vector into its warp's queue in shared memory, and once a few vectors are
// queued every lane of the warp takes one generator counter (four consecutive
// entries) at a time: the words, their exact fp32 Gumbel values and the scores.
// Entries are kept by exact vocabulary index (encoded -1 - v), ties going to the
// lower index.
constexpr int kQueueCap = 80;    // vectors per warp
constexpr int kQueueDrain = 16;  // evaluate once this many vectors are queued

struct NoiseQueue {
  int v[kQueueCap];             // first vocabulary index of the vector
  uint4 l[kQueueCap], m[kQueueCap];
};

__device__ __forceinline__ void keep_best(float& best, int& code, float s, int v) {
  if (s > best || (s == best && v < -1 - code)) {
    best = s;
    code = -1 - v;
  }
}

template <typename T>
__device__ __forceinline__ float vec_entry(const uint4& u, int e) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w = (e >> 1) == 0 ? u.x : (e >> 1) == 1 ? u.y : (e >> 1) == 2 ? u.z : u.w;
    return (e & 1) ? bf16hi(w) : bf16lo(w);
  } else {
    const uint32_t w = e == 0 ? u.x : e == 1 ? u.y : e == 2 ? u.z : u.w;
    return __uint_as_float(w);
  }
}

// The best exact coupled scores any lane in `act` holds (the screen's thresholds).
__device__ __forceinline__ void warp_thresholds(const Acc& a, unsigned act, float& tht,
                                                float& thd) {
  tht = ordered_to_float(__reduce_max_sync(act, float_to_ordered(a.bt)));
  thd = ordered_to_float(__reduce_max_sync(act, float_to_ordered(a.bd)));
}

// The warp's thresholds, raised to the CTA-wide best (every warp of a CTA works on the
// same row piece). A threshold from any entry of the row keeps the screen exact: a
// screened-out entry scores strictly below it (the slack), so it cannot be sampled.
__device__ __forceinline__ void publish_thresholds(const Acc& a, unsigned act, float& tht,
                                                   float& thd, int* cta_thr) {
  warp_thresholds(a, act, tht, thd);
  int ot = 0, od = 0;
  const int lead = __ffs(act) - 1;
  if ((int)(threadIdx.x & 31) == lead) {
    ot = atomicMax(&cta_thr[0], float_to_ordered(tht));
    od = atomicMax(&cta_thr[1], float_to_ordered(thd));
  }
  tht = fmaxf(tht, ordered_to_float(__shfl_sync(act, ot, lead)));
  thd = fmaxf(thd, ordered_to_float(__shfl_sync(act, od, lead)));
}

// Every queued entry, spread over the lanes in `act`; empties the queue.
template <typename T>
__device__ __forceinline__ void drain_queue(Acc& a, NoiseQueue* q, int& qn, unsigned act,
                                         const PhiloxRow& pr, NoiseKey key, float invT) {
  constexpr int VEC = Unpack<T>::N;
  __syncwarp(act);  // the pushes are visible
  const int lane = threadIdx.x & 31;
  const int nact = __popc(act), rank = __popc(act & ((1u << lane) - 1u));
  // one generator counter (four consecutive entries) per lane and round
  constexpr int NC = VEC / 4;  // counters per 16-byte vector
  for (int i = rank; i < qn * NC; i += nact) {
    const int s = i / NC, c = i % NC;
    const int v = q->v[s] + 4 * c;
    const uint4 lw = q->l[s], mw = q->m[s];
    const PhiloxOut o = philox_row_counter(pr, (uint32_t)(v >> 2), key.k0, key.k1);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float g = gumbel_from_word(o.w[w]);
      keep_best(a.bt, a.vbt, fmaf(vec_entry<T>(lw, 4 * c + w), invT, g), v + w);
      keep_best(a.bd, a.vbd, fmaf(vec_entry<T>(mw, 4 * c + w), invT, g), v + w);
    }
  }
  __syncwarp(act);  // every lane is done reading before the queue is reused
  qn = 0;
}

template <typename T, bool SAMPLE, int NV>
__device__ __forceinline__ void fold(Acc& a, const uint4 (&lw)[NV], const uint4 (&mw)[NV],
                                     const int (&v0)[NV], const PhiloxRow& pr,
                                     const NoiseKey& key, float invT, NoiseQueue* q, int& qn,
                                     float& tht, float& thd, int* cta_thr) {
  constexpr int VEC = Unpack<T>::N, NP = VEC / 2;
  float xm[NV], ym[NV];  // per-vector maxima of l and m
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    xm[k] = Unpack<T>::vmax(lw[k]);
    ym[k] = Unpack<T>::vmax(mw[k]);
  }
  // --- exact maxima and the first vector holding them (selects, no branch)
  float cm = xm[0], dm = ym[0];
  int cv = v0[0], dv = v0[0];
#pragma unroll
  for (int k = 1; k < NV; ++k) {
    if (xm[k] > cm) { cm = xm[k]; cv = v0[k]; }
    if (ym[k] > dm) { dm = ym[k]; dv = v0[k]; }
  }
  if (cm > a.mt) { a.mt = cm; a.vt = cv; }
  if (dm > a.md) { a.md = dm; a.vd = dv; }
  // --- move an exponent reference only when its maximum outgrew it (rare)
  const bool rt = a.mt > a.ref_t + kRefMargin, rd = a.md > a.ref_d + kRefMargin;
  if (__any_sync(__activemask(), rt || rd)) {
    if (rt) {
      if (a.ref_t != -INFINITY) {
        const float dl = (a.ref_t - a.mt) * kLog2e;
        const float f = exp2f(dl);
        const float2 f2 = make_float2(f, f), dl2 = make_float2(dl, dl);
        a.s2t = __fmul2_rn(f2, __ffma2_rn(dl2, a.s1t, a.s2t));
        a.s1t = __fmul2_rn(f2, a.s1t);
      }
      a.ref_t = a.mt;
    }
    if (rd) {
      if (a.ref_d != -INFINITY) {
        const float f = exp2f((a.ref_d - a.md) * kLog2e);
        const float2 f2 = make_float2(f, f);
        a.s1d = __fmul2_rn(f2, a.s1d);
        a.skd = __fmul2_rn(f2, a.skd);
      }
      a.ref_d = a.md;
    }
  }
  const float2 l2e = make_float2(kLog2e, kLog2e);
  const float2 nmt = make_float2(-a.ref_t * kLog2e, -a.ref_t * kLog2e);
  const float2 nmd = make_float2(-a.ref_d * kLog2e, -a.ref_d * kLog2e);
  const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int k = 0; k < NV; ++k)
#pragma unroll
    for (int e = 0; e < NP; ++e) {
      const float2 lp = Unpack<T>::pair(lw[k], e), mp = Unpack<T>::pair(mw[k], e);
      const float2 y = __ffma2_rn(lp, l2e, nmt);
      const float2 et = ex2x2(y);
      a.s1t = __fadd2_rn(a.s1t, et);
      a.s2t = __ffma2_rn(et, y, a.s2t);
      const float2 z = __ffma2_rn(mp, l2e, nmd);
      const float2 ed = ex2x2(z);
      a.s1d = __fadd2_rn(a.s1d, ed);
      a.skd = __ffma2_rn(ed, __ffma2_rn(lp, neg1, mp), a.skd);
    }
  // --- coupled Gumbel-max samples (same noise for both).
  // Screening, per 16-byte vector: tht / thd are the best exact scores any lane of
  // the warp holds for this row (all lanes work on one row, and every vector of
  // this fold lies above every entry evaluated so far, so such a score wins a tie
  // against any entry here). They change only when exact scores are added, so the
  // caller keeps them and they are refreshed after each evaluation of the queue. An entry with noise g scores at most x_max / T + g; it
  // can only matter if g exceeds G = min over the two matrices of (thr - x_max / T),
  // minus a rounding slack. If G >= kGumbelMax no noise value can do that and the
  // vector's generator words are not even drawn; otherwise the words are drawn and
  // compared, as integers, with the limit that g > G implies (gumbel_screen_limit).
  // A vector that passes goes to the warp's queue (drain_queue): its entries get
  // exactly the fp32 noise and scores the unscreened pass would compute.
  if constexpr (SAMPLE) {
    const unsigned act = __activemask();
    // the best the CTA's other warps have published for this row
    tht = fmaxf(tht, ordered_to_float(*(volatile int*)&cta_thr[0]));
    thd = fmaxf(thd, ordered_to_float(*(volatile int*)&cta_thr[1]));
    // slack for the fp32 rounding of thr - x/T (about 1e-7 relative)
    const float slt = fmaf(fabsf(tht), 1e-5f, 1e-5f), sld = fmaf(fabsf(thd), 1e-5f, 1e-5f);
    const float is = invT * 1e-5f;
    const int lane = threadIdx.x & 31;
    bool cand[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const float gt = fmaf(-xm[k], invT, tht) - fmaf(fabsf(xm[k]), is, slt);
      const float gd = fmaf(-ym[k], invT, thd) - fmaf(fabsf(ym[k]), is, sld);
      const float G = fminf(gt, gd);
      cand[k] = false;
      if (G < kGumbelMax) {
        uint32_t wm = 0u;
#pragma unroll
        for (int qq = 0; qq < VEC / 4; ++qq) {
          const PhiloxOut o = philox_row_counter(pr, (uint32_t)(v0[k] >> 2) + qq, key.k0, key.k1);
          wm = max(wm, max(max(o.w[0], o.w[1]), max(o.w[2], o.w[3])));
        }
        cand[k] = gumbel_screen_j(wm) + 0.5f < gumbel_screen_limit(G);
      }
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const unsigned bal = __ballot_sync(act, cand[k]);
      if (bal) {
        if (cand[k]) {
          const int slot = qn + __popc(bal & ((1u << lane) - 1u));
          q->v[slot] = v0[k];
          q->l[slot] = lw[k];
          q->m[slot] = mw[k];
        }
        qn += __popc(bal);
      }
    }
    if (qn >= kQueueDrain) {
      drain_queue<T>(a, q, qn, act, pr, key, invT);
      publish_thresholds(a, act, tht, thd, cta_thr);
    }
  }
}

// One vocabulary entry (the ragged end of a row); exact indices encoded -1 - v.
template <bool SAMPLE>
__device__ __forceinline__ void fold_one(Acc& a, float l, float m, float g, int v, float invT) {
  if (l > a.mt) { a.mt = l; a.vt = -1 - v; }
  if (m > a.md) { a.md = m; a.vd = -1 - v; }
  if (a.mt > a.ref_t + kRefMargin) {
    if (a.ref_t != -INFINITY) {
      const float dl = (a.ref_t - a.mt) * kLog2e;
      const float f = exp2f(dl);
      a.s2t = make_float2(f * (a.s2t.x + dl * a.s1t.x), f * (a.s2t.y + dl * a.s1t.y));
      a.s1t = make_float2(f * a.s1t.x, f * a.s1t.y);
    }
    a.ref_t = a.mt;
  }
  if (a.md > a.ref_d + kRefMargin) {
    if (a.ref_d != -INFINITY) {
      const float f = exp2f((a.ref_d - a.md) * kLog2e);
      a.s1d = make_float2(f * a.s1d.x, f * a.s1d.y);
      a.skd = make_float2(f * a.skd.x, f * a.skd.y);
    }
    a.ref_d = a.md;
  }
  const float y = fmaf(l, kLog2e, -a.ref_t * kLog2e);
  const float et = fast_exp2(y);
  a.s1t.x += et;
  a.s2t.x = fmaf(et, y, a.s2t.x);
  const float ed = fast_exp2(fmaf(m, kLog2e, -a.ref_d * kLog2e));
  a.s1d.x += ed;
  a.skd.x = fmaf(ed, m - l, a.skd.x);
  if constexpr (SAMPLE) {
    const float st = fmaf(l, invT, g), sd = fmaf(m, invT, g);
    if (st > a.bt) { a.bt = st; a.vbt = -1 - v; }
    if (sd > a.bd) { a.bd = sd; a.vbd = -1 - v; }
  }
}

// Turn a thread's state for one row piece into a Partial: sums re-expressed
// relative to the exact maximum, exact indices recovered by re-reading the one
// 16-byte vector where each maximum / best score first appeared.
template <typename T, bool SAMPLE>
__device__ Partial resolve(const Acc& a, const T* lrow, const T* mrow, int pos, int b,
                           const NoiseKey& key, float invT) {
  constexpr int VEC = Unpack<T>::N;
  Partial p;
  p.mt = a.mt;
  p.md = a.md;
  p.s1t = p.s2t = p.s1d = p.skd = 0.f;
  p.at = p.ad = p.it = p.id = 0x7fffffff;
  p.bt = a.bt;
  p.bd = a.bd;
  p.lt_at = 0.f;
  if (a.mt != -INFINITY) {
    const float dl = (a.ref_t - a.mt) * kLog2e;  // <= 0
    const float f = exp2f(dl);
    const float s1 = a.s1t.x + a.s1t.y, s2 = a.s2t.x + a.s2t.y;
    p.s1t = f * s1;
    p.s2t = f * (s2 + dl * s1);
    if (a.vt < 0) {
      p.at = -1 - a.vt;
    } else {
      float x[VEC];
      Vec<T>::unpack(*reinterpret_cast<const uint4*>(lrow + a.vt), x);
      for (int e = VEC - 1; e >= 0; --e)
        if (x[e] == a.mt) p.at = a.vt + e;
    }
  }
  if (a.md != -INFINITY) {
    const float f = exp2f((a.ref_d - a.md) * kLog2e);
    p.s1d = f * (a.s1d.x + a.s1d.y);
    p.skd = f * (a.skd.x + a.skd.y);
    if (a.vd < 0) {
      p.ad = -1 - a.vd;
    } else {
      float x[VEC];
      Vec<T>::unpack(*reinterpret_cast<const uint4*>(mrow + a.vd), x);
      for (int e = VEC - 1; e >= 0; --e)
        if (x[e] == a.md) p.ad = a.vd + e;
    }
  }
  if constexpr (SAMPLE) {
    auto find = [&](int vb, float best, const T* row, int& idx, float* lval) {
      if (best == -INFINITY) return;
      if (vb < 0) {
        idx = -1 - vb;
        if (lval) *lval = Vec<T>::scalar(lrow + idx);
        return;
      }
      float x[VEC], l[VEC], g[VEC];
      Vec<T>::unpack(*reinterpret_cast<const uint4*>(row + vb), x);
      Vec<T>::unpack(*reinterpret_cast<const uint4*>(lrow + vb), l);
      #pragma unroll
      for (int q = 0; q < VEC / 4; ++q) {
        const PhiloxOut o = philox4x32_10((uint32_t)(vb >> 2) + q, (uint32_t)pos, (uint32_t)b,
                                          key.step, key.k0, key.k1);
        #pragma unroll
        for (int w = 0; w < 4; ++w) g[4 * q + w] = gumbel_from_word(o.w[w]);
      }
      #pragma unroll
      for (int e = VEC - 1; e >= 0; --e)
        if (fmaf(x[e], invT, g[e]) == best) {
          idx = vb + e;
          if (lval) *lval = l[e];
        }
    };
    find(a.vbt, a.bt, lrow, p.it, &p.lt_at);
    find(a.vbd, a.bd, mrow, p.id, nullptr);
  }
  return p;
}

// Merge partial b into a (both cover disjoint vocabulary ranges of one row).
template <bool SAMPLE>
__device__ __forceinline__ void merge(Partial& a, const Partial& b) {
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

__device__ __forceinline__ Partial shfl_xor(const Partial& p, int mask) {
  Partial q;
  q.mt = __shfl_xor_sync(0xffffffffu, p.mt, mask);
  q.s1t = __shfl_xor_sync(0xffffffffu, p.s1t, mask);
  q.s2t = __shfl_xor_sync(0xffffffffu, p.s2t, mask);
  q.md = __shfl_xor_sync(0xffffffffu, p.md, mask);
  q.s1d = __shfl_xor_sync(0xffffffffu, p.s1d, mask);
  q.skd = __shfl_xor_sync(0xffffffffu, p.skd, mask);
  q.at = __shfl_xor_sync(0xffffffffu, p.at, mask);
  q.ad = __shfl_xor_sync(0xffffffffu, p.ad, mask);
  q.bt = __shfl_xor_sync(0xffffffffu, p.bt, mask);
  q.lt_at = __shfl_xor_sync(0xffffffffu, p.lt_at, mask);
  q.bd = __shfl_xor_sync(0xffffffffu, p.bd, mask);
  q.it = __shfl_xor_sync(0xffffffffu, p.it, mask);
  q.id = __shfl_xor_sync(0xffffffffu, p.id, mask);
  return q;
}

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
      const uint32_t w = (v & 3) == 0 ? o.w[0] : (v & 3) == 1 ? o.w[1] : (v & 3) == 2 ? o.w[2]
                                                                                        : o.w[3];
      g[i] = gumbel_from_word(w);
    }
  }
}

// Work partition: U units split into G ranges, the first `rem` of size q + 1.
struct Split {
  int64_t q, rem;
  __host__ __device__ int64_t begin(int64_t c) const {
    return c < rem ? c * (q + 1) : rem * (q + 1) + (c - rem) * q;
  }
  __host__ __device__ int64_t size(int64_t c) const { return c < rem ? q + 1 : q; }
  __host__ __device__ int64_t cta_of(int64_t u) const {
    return u < rem * (q + 1) ? u / (q + 1) : rem + (u - rem * (q + 1)) / (q > 0 ? q : 1);
  }
};

struct VerifyArgs {
  const void *lt, *lm;
  int R, V;
  int64_t ld;
  int pos_offset;
  float invT;
  NoiseKey key;
  int nchunk;  // chunks per row
  Split split;
  Partial* parts;  // [rows, maxparts]
  int maxparts;
  uint32_t spin;
};

// 16 bytes global -> this thread's own shared-memory slot, asynchronously, caching in
// L2 only (with a 256-byte L2 prefetch); completion is per thread (commit / wait groups).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename T, bool SAMPLE>
__global__ void __launch_bounds__(kVThreads, VCfg<SAMPLE>::kMinBlocks)
verify_stream_kernel(const VerifyArgs a) {
  constexpr int VEC = Vec<T>::N;
  constexpr int kStages = VCfg<SAMPLE>::kStages;
  __shared__ Partial red[kVThreads / 32];

  const int c = blockIdx.x;
  const int ct = threadIdx.x, lane = ct & 31, cw = ct >> 5;
  const T* LT = static_cast<const T*>(a.lt);
  const T* LM = static_cast<const T*>(a.lm);
  const int spr = a.nchunk;                       // vector slots per row
  const int nvr = (int)(((int64_t)a.V * (int)sizeof(T)) >> 4);  // full vectors per row
  const int64_t s0 = a.split.begin(c), s1 = s0 + a.split.size(c);

  Acc acc;
  init(acc);
  // sampling: this warp's queue of vectors awaiting exact noise (see drain_queue)
  NoiseQueue* q = nullptr;
  int* cta_thr = nullptr;  // the CTA's best exact scores of the current row (ordered ints)
  if constexpr (SAMPLE) {
    __shared__ NoiseQueue queues[kVThreads / 32];
    __shared__ int thr_s[2];
    q = &queues[cw];
    cta_thr = thr_s;
    if (ct == 0) thr_s[0] = thr_s[1] = float_to_ordered(-INFINITY);
    __syncthreads();
  }
  int qn = 0;
  auto flush = [&](int64_t row, Partial p) {
#pragma unroll
    for (int mask = 16; mask > 0; mask >>= 1) {
      const Partial q = shfl_xor(p, mask);
      merge<SAMPLE>(p, q);
    }
    if (lane == 0) red[cw] = p;
    __syncthreads();
    if (cw == 0) {
      Partial r;
      if (lane < kVThreads / 32) {
        r = red[lane];
      } else {
        r = p;  // an empty partial (no entries)
        r.mt = r.md = r.bt = r.bd = -INFINITY;
        r.s1t = r.s2t = r.s1d = r.skd = 0.f;
      }
#pragma unroll
      for (int mask = 16; mask > 0; mask >>= 1) {
        const Partial q = shfl_xor(r, mask);
        merge<SAMPLE>(r, q);
      }
      if (lane == 0) {
        const int64_t slot = c - a.split.cta_of(row * spr);
        if (DD_IN_BOUNDS(slot >= 0 && slot < a.maxparts)) a.parts[row * a.maxparts + slot] = r;
      }
      // every warp is past the row: its thresholds start over for the next one
      if (SAMPLE && lane == 0) cta_thr[0] = cta_thr[1] = float_to_ordered(-INFINITY);
    }
    __syncthreads();
    init(acc);
  };

  for (int64_t sidx = s0; sidx < s1;) {
    const int64_t row = sidx / spr;
    const int vbeg = (int)(sidx - row * spr);
    const int64_t rest = s1 - sidx;
    const int vend = rest < (int64_t)(spr - vbeg) ? vbeg + (int)rest : spr;
    const int b = (int)(row / a.R);
    const int pos = a.pos_offset + (int)(row - (int64_t)b * a.R);
    const uint4* lv = reinterpret_cast<const uint4*>(LT + row * a.ld);
    const uint4* mv = reinterpret_cast<const uint4*>(LM + row * a.ld);
    const int vlim = min(vend, nvr);  // slots past nvr carry no full vector
    // per-row parts of the noise generator (only used when sampling)
    const PhiloxRow pr = philox_row((uint32_t)pos, (uint32_t)b, a.key.step, a.key.k0, a.key.k1);
    float tht = -INFINITY, thd = -INFINITY;  // the screen's thresholds (warp-uniform)
    // both vectors of a half-step in one fold where both exist (one warp-wide
    // screening threshold per pair), else the one that does
    auto fold2 = [&](int bs, const uint4 (&l)[2], const uint4 (&m)[2]) {
      // Both vectors in one fold (one maximum update and rescale check for the pair)
      // where both exist. When sampling, only if every active lane of the warp has
      // both: the warp's lanes share one queue and one count, so two groups of a warp
      // must never fold (and push) at the same time.
      const bool both = SAMPLE ? __all_sync(__activemask(), bs + kVThreads < vlim)
                               : bs + kVThreads < vlim;
      if (both) {
        const int vv[2] = {bs * VEC, (bs + kVThreads) * VEC};
        fold<T, SAMPLE, 2>(acc, l, m, vv, pr, a.key, a.invT, q, qn, tht, thd, cta_thr);
        return;
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int idx = bs + k * kVThreads;
        if (idx < vlim) {
          const uint4 l1[1] = {l[k]}, m1[1] = {m[k]};
          const int vv[1] = {idx * VEC};
          fold<T, SAMPLE, 1>(acc, l1, m1, vv, pr, a.key, a.invT, q, qn, tht, thd, cta_thr);
        }
      }
    };
    constexpr int kStep = 2 * kVThreads;
    {
      extern __shared__ uint4 ring[];  // kRingBytes: [stage][4][kVThreads]
      constexpr int kStageStride = 4 * kVThreads;  // uint4s per stage
      uint4* const mine = ring + ct;               // this thread's slot 0 of stage 0
      // the issue cursor: next half-step's stage and the index of its first vector
      int ist = 0, ibs = vbeg + ct;
      auto issue = [&]() {
        uint4* const sp = mine + ist * kStageStride;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int idx = ibs + k * kVThreads;
          if (idx < vlim) {
            cp_async16(sp + k * kVThreads, lv + idx);
            cp_async16(sp + (2 + k) * kVThreads, mv + idx);
          }
        }
        cp_async_commit();  // a group per half-step, empty or not
        ist = ist + 1 == kStages ? 0 : ist + 1;
        ibs += kStep;
      };
#pragma unroll
      for (int hh = 0; hh < kStages - 1; ++hh) issue();
      int h = 0, cst = 0;
      for (int bs = vbeg + ct; bs < vlim; bs += kStep, ++h) {
        cp_async_wait<kStages - 2>();  // half-step h has landed (this thread's copies)
        const uint4* const sp = mine + cst * kStageStride;
        const uint4 l[2] = {sp[0], sp[kVThreads]}, m[2] = {sp[2 * kVThreads], sp[3 * kVThreads]};
        cst = cst + 1 == kStages ? 0 : cst + 1;
        issue();  // into the stage read one half-step ago
        if constexpr (SAMPLE) {
          if (h == 0) {
            // a first exact score per lane (the four entries of its first vector's first
            // generator counter), so the screen has a threshold from the start
            const int v = bs * VEC;
            const PhiloxOut o = philox_row_counter(pr, (uint32_t)(v >> 2), a.key.k0, a.key.k1);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float g = gumbel_from_word(o.w[e]);
              keep_best(acc.bt, acc.vbt, fmaf(vec_entry<T>(l[0], e), a.invT, g), v + e);
              keep_best(acc.bd, acc.vbd, fmaf(vec_entry<T>(m[0], e), a.invT, g), v + e);
            }
            publish_thresholds(acc, __activemask(), tht, thd, cta_thr);
          }
        }
        fold2(bs, l, m);
      }
      cp_async_wait<0>();  // nothing of this row piece left in flight
    }
    if (vend == spr) {
      // ragged end of the row (fewer than 16 bytes): one entry per thread
      const int e = nvr * VEC + ct;
      if (e < a.V) {
        float g = 0.f;
        if constexpr (SAMPLE) {
          float gg[1];
          noise<1>(gg, e, pos, b, a.key);
          g = gg[0];
        }
        fold_one<SAMPLE>(acc, Vec<T>::scalar(LT + row * a.ld + e),
                         Vec<T>::scalar(LM + row * a.ld + e), g, e, a.invT);
      }
    }
    if constexpr (SAMPLE) {
      // Lanes leave a row piece's last folds in lane order (a lane's vectors lie above
      // those of the lanes before it), so lane 0 took part in every push: its count
      // is the warp's. Evaluate what is still queued.
      __syncwarp();
      qn = __shfl_sync(0xffffffffu, qn, 0);
      if (qn > 0) drain_queue<T>(acc, q, qn, 0xffffffffu, pr, a.key, a.invT);
    }
    flush(row, resolve<T, SAMPLE>(acc, LT + row * a.ld, LM + row * a.ld, pos, b, a.key, a.invT));
    sidx += vend - vbeg;
  }
}

// One warp per row: merge the row's partials and write the statistics.
template <bool SAMPLE>
__global__ void __launch_bounds__(256) verify_merge_kernel(const VerifyArgs a, int rows,
                                                           dd_row_stats out) {
  pdl_wait();  // launched as a dependent of the previous kernel
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int64_t c0 = a.split.cta_of(row * a.nchunk);
  const int np0 = (int)(a.split.cta_of(row * a.nchunk + a.nchunk - 1) - c0 + 1);
  const int nparts = DD_IN_BOUNDS(np0 >= 1 && np0 <= a.maxparts) ? np0 : 0;
  Partial acc;
  init(acc);
  for (int k = lane; k < nparts; k += 32) merge<SAMPLE>(acc, a.parts[row * a.maxparts + k]);
#pragma unroll
  for (int mask = 16; mask > 0; mask >>= 1) {
    const Partial q = shfl_xor(acc, mask);
    merge<SAMPLE>(acc, q);
  }
  if (lane != 0) return;
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

__global__ void coupled_gumbel_kernel(NoiseKey key, int R, int V, int64_t ld, int pos_offset,
                                      int64_t nquads_per_row, int64_t total_quads, float* g) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total_quads;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = t / nquads_per_row;
    const int qd = (int)(t % nquads_per_row);
    const int b = (int)(row / R);
    const int pos = pos_offset + (int)(row % R);
    // the row-split generator of the streaming pass, so its words are what the
    // noise written here is checked against
    const PhiloxRow pr = philox_row((uint32_t)pos, (uint32_t)b, key.step, key.k0, key.k1);
    const PhiloxOut o = philox_row_counter(pr, (uint32_t)qd, key.k0, key.k1);
    float* dst = g + row * ld + 4 * (int64_t)qd;
#pragma unroll
    for (int w = 0; w < 4; ++w)
      if (4 * qd + w < V) dst[w] = gumbel_from_word(o.w[w]);
  }
}

// Self-test of the noise screen: the fp32 Gumbel value of every noise level
// k = w >> 9 (2^23 of them), the screen's exact-float j of a word at that level,
// and the screen limit for each requested noise level.
__global__ void selftest_gumbel_kernel(float* g_of_k, float* j_of_k, const float* g_req,
                                       float* limit, int n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < (1 << 23); t += stride) {
    const uint32_t k = (uint32_t)t;
    const uint32_t w = (k << 9) | (k & 511u);  // low bits play no part; mix them anyway
    g_of_k[t] = gumbel_from_word(w);
    j_of_k[t] = gumbel_screen_j(w);
  }
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n; t += stride)
    limit[t] = gumbel_screen_limit(g_req[t]);
}

// Grid and partition for a call (also sizes the workspace).
struct VerifyPlan {
  int grid, nchunk, maxparts;
  Split split;
};

VerifyPlan plan_verify(int rows, int V, int esize, int sm_count, int per_sm) {
  VerifyPlan pl;
  const int64_t nvr = ((int64_t)V * esize) >> 4;
  pl.nchunk = (int)(nvr > 0 ? nvr : 1);  // vector slots per row
  const int64_t units = (int64_t)rows * pl.nchunk;
  // at least 2048 vectors per CTA, so a piece is long enough to stream
  int64_t g = (int64_t)sm_count * per_sm;
  const int64_t gmin = (units + 2047) / 2048;
  if (g > gmin) g = gmin > 0 ? gmin : 1;
  pl.grid = (int)g;
  pl.split.q = units / pl.grid;
  pl.split.rem = units % pl.grid;
  // a row's slots overlap at most ceil(nchunk / q) + 1 ranges
  const int64_t q = pl.split.q > 0 ? pl.split.q : 1;
  pl.maxparts = (int)((pl.nchunk + q - 1) / q + 1);
  return pl;
}

// The workspace bound must hold on any device: plan for up to 512 SMs.
constexpr int kPlanSmBound = 512;

template <typename T, bool SAMPLE>
cudaError_t launch_verify(const void* lt, const void* lm, int B, int R, int V, int64_t ld,
                          int pos_offset, float temperature, NoiseKey key,
                          const dd_row_stats& out, void* workspace, cudaStream_t stream) {
  const int rows = B * R;
  const DeviceInfo& dev = device_info();
  VerifyPlan pl = plan_verify(rows, V, (int)sizeof(T), dev.sm_count, VCfg<SAMPLE>::kMinBlocks);
  const VerifyPlan bound = plan_verify(rows, V, (int)sizeof(T), kPlanSmBound, kMaxGridPerSm);
  VerifyArgs a;
  a.lt = lt;
  a.lm = lm;
  a.R = R;
  a.V = V;
  a.ld = ld;
  a.pos_offset = pos_offset;
  a.invT = temperature > 0.f ? 1.f / temperature : 0.f;
  a.key = key;
  a.nchunk = pl.nchunk;
  a.split = pl.split;
  a.parts = static_cast<Partial*>(workspace);
  a.maxparts = bound.maxparts > pl.maxparts ? bound.maxparts : pl.maxparts;
  a.spin = spin_limit();
  const int smem = VCfg<SAMPLE>::kRingBytes;
  {
    static int configured[64] = {};
    if (!configured[dev.device & 63]) {
      cudaError_t e = cudaFuncSetAttribute(verify_stream_kernel<T, SAMPLE>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      configured[dev.device & 63] = 1;
    }
  }
  verify_stream_kernel<T, SAMPLE><<<pl.grid, kVThreads, smem, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_dependent(verify_merge_kernel<SAMPLE>, dim3((rows + 7) / 8), dim3(256), 0, stream, a,
                          rows, out);
}

}  // namespace

size_t verify_workspace_bytes(int B, int R, int V, dd_dtype dtype) {
  const int esize = dtype == DD_BF16 ? 2 : 4;
  const int rows = B * R;
  const VerifyPlan bound = plan_verify(rows, V, esize, kPlanSmBound, kMaxGridPerSm);
  // any real device has at most kPlanSmBound SMs, so its maxparts is no larger
  return (size_t)rows * bound.maxparts * sizeof(Partial);
}

cudaError_t launch_verify_logits(const void* lt, const void* lm, dd_dtype dtype, int B, int R,
                                 int V, int64_t ld, int pos_offset, float temperature,
                                 uint64_t seed, uint64_t step, const dd_row_stats& out,
                                 void* workspace, cudaStream_t stream) {
  NoiseKey key{(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32),
               (uint32_t)(step & 0xffffffffu)};
  const bool sample = temperature > 0.f;
  if (dtype == DD_BF16)
    return sample ? launch_verify<__nv_bfloat16, true>(lt, lm, B, R, V, ld, pos_offset,
                                                       temperature, key, out, workspace, stream)
                  : launch_verify<__nv_bfloat16, false>(lt, lm, B, R, V, ld, pos_offset,
                                                        temperature, key, out, workspace, stream);
  return sample ? launch_verify<float, true>(lt, lm, B, R, V, ld, pos_offset, temperature, key,
                                             out, workspace, stream)
                : launch_verify<float, false>(lt, lm, B, R, V, ld, pos_offset, temperature, key,
                                              out, workspace, stream);
}

cudaError_t launch_selftest_gumbel(float* g_of_k, float* j_of_k, const float* g_req,
                                   float* limit, int n, cudaStream_t stream) {
  selftest_gumbel_kernel<<<device_info().sm_count * 4, 256, 0, stream>>>(g_of_k, j_of_k, g_req,
                                                                        limit, n);
  return cudaGetLastError();
}

float gumbel_max_constant() { return kGumbelMax; }

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
