// Tensor-core (sm_100a, tcgen05) dual-view attention for bf16 inputs.
//
// The drafting view -- seed rows of K and V taken from the step t-1 cache --
// is materialised once per call by the prep kernel, so both passes stream
// plain TMA tiles of it and no tile is patched on the way in.
//
// Pass 1, one CTA per (128 query rows, head, sequence), warp-specialised:
//   warp 0      producer: TMA loads of the Q tile and of K / V tiles of the
//               view (128 columns; K and V have their own stage rings), and the
//               tile's "newly written" flags into a 16-column block next to the
//               V tile whose key rows read [1, is_new(key), 0, ...].
//   warp 1      MMA issuer (one thread): S = Q K^T into a double-buffered TMEM
//               accumulator; [O | l | l_new] += P [V | 1 | is_new] as one MMA of
//               N = D + 16 with P read from TMEM, i.e. the row sum and the mass on
//               newly written columns come out of the tensor core with the same
//               bf16 P that weights V, at the cost of 16 extra output columns.
//   warps 2-5   softmax (one thread per query row = TMEM lane): online max with
//               a lazy rescale (O is rescaled in TMEM only when the running max
//               grows by more than 2^8), P = exp2(S*scale*log2e - m) as bf16
//               pairs written over the S columns they came from. A seed query's
//               own column is masked in the loop and merged back afterwards from
//               k_cur / v_cur (leave-one-out diagonal). Epilogue: out = O / l,
//               lse, d_out partial = l_new / l, and for a still-masked row its Q
//               row and lse (log2 units) in rank order, the inputs of pass 2.
// Every wait is bounded; on expiry the kernel records DD_ERR_TIMEOUT and winds down.
#include <cudaTypedefs.h>

#include "dd_internal.h"
#include "dd_tc.cuh"

namespace dd {

namespace {

using namespace tc;

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kSK = 2;  // K stages
constexpr int kSV = 2;  // V stages
constexpr int kP1Threads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kAtom = 128 * 128;  // one 128-row x 128-byte swizzle atom column

template <int D>
struct P1Layout {
  static constexpr int kTile = (D / 64) * kAtom;  // 128 x D bf16
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;
  // A V stage is the V tile plus one more 64-column swizzle atom whose first
  // 16 columns are [1, is_new(key), 0...]: PV with N = D + 16 then yields O and
  // the statistics [l, l_new] together.
  static constexpr int kVStage = kTile + kAtom;
  static constexpr int kV = kK + kSK * kTile;
  // packed newly-written flags of the whole sequence
  static constexpr int kNew = kV + kSV * kVStage;
  static constexpr int kNewWords = kTcMaxL / 32;
  static constexpr int kBar = kNew + kNewWords * 4;
  static constexpr int kBytes = kBar + 256;
  // TMEM columns
  static constexpr uint32_t kS0 = 0, kS1 = 128, kO = 256, kSt = 256 + D;
};

struct P1Bars {
  uint64_t q_full;
  uint64_t k_full[kSK], k_empty[kSK];
  uint64_t v_full[kSV], v_empty[kSV];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct P1Params {
  const __nv_bfloat16 *q, *k_cur, *v_cur;
  const uint8_t *is_seed, *is_new;
  const uint32_t* newbits;  // [B, ceil(L/32)]
  const int32_t* mrank;     // [B, L]
  int L, Hq, Hkv, Lp;
  int q_begin;  // first query row (rows before it are a cached prefix, not computed)
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  float* dout_part;
  __nv_bfloat16* q_m;  // nullptr: pass 2 does not run
  float* lse2_m;
  uint32_t spin;
};

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}

template <int D>
__global__ void __launch_bounds__(kP1Threads, 1)
attn_p1_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const P1Params p) {
  using Lay = P1Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  P1Bars* bars = reinterpret_cast<P1Bars*>(smem + Lay::kBar);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int L = p.L;
  const int g = h / (p.Hq / p.Hkv);
  const int q0 = p.q_begin + qt * kBM;
  const int T = (L + kBN - 1) / kBN;
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kSK; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kSV; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->s_full[0], 1);
    mbar_init(&bars->s_full[1], 1);
    mbar_init(&bars->p_full[0], 4);
    mbar_init(&bars->p_full[1], 4);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // the statistics atoms start at zero (chunk 0 of each row is rewritten per tile)
  if (warp >= 2) {
    const int t = threadIdx.x - 64;  // 0..127
    for (int idx = t; idx < kSV * 128 * 8; idx += 128) {
      const int s = idx / (128 * 8), row = (idx / 8) % 128, c = idx % 8;
      st_shared_v4(sbase + Lay::kV + s * Lay::kVStage + Lay::kTile + sw128(row, c), 0u, 0u, 0u, 0u);
    }
    fence_proxy_async();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  // set-up above touches only shared and tensor memory; the previous kernel's
  // outputs are read from here on
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(&bars->q_full, Lay::kTile);
#pragma unroll
      for (int ac = 0; ac < D / 64; ++ac)
        tma_load_4d(smem + Lay::kQ + ac * kAtom, &tmQ, ac * 64, h, q0, b, &bars->q_full);
    }
    uint32_t* neww = reinterpret_cast<uint32_t*>(smem + Lay::kNew);
    const int W = (L + 31) / 32;
    // K(j) may reuse its stage once QK(j - kSK) is done, V(j) once PV(j - kSV) is.
    auto issue_k = [&](int j) -> bool {
      const int s = j % kSK;
      if (j >= kSK && !wait_bounded(&bars->k_empty[s], ((j / kSK) - 1) & 1, p.spin, abort_flag))
        return false;
      if (lane == 0) {
        mbar_expect_tx(&bars->k_full[s], Lay::kTile);
#pragma unroll
        for (int ac = 0; ac < D / 64; ++ac)
          tma_load_4d(smem + Lay::kK + s * Lay::kTile + ac * kAtom, &tmK, ac * 64, g, j * kBN, b,
                      &bars->k_full[s]);
      }
      return true;
    };
    auto issue_v = [&](int j) -> bool {
      const int s = j % kSV;
      if (j >= kSV && !wait_bounded(&bars->v_empty[s], ((j / kSV) - 1) & 1, p.spin, abort_flag))
        return false;
      {
        // statistics columns of key row r: [1, is_new(r), 0, ...] (rows = keys)
        const uint32_t atom = sbase + Lay::kV + s * Lay::kVStage + Lay::kTile;
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int wi = j * 4 + rr;
          const bool nw = wi < W && ((neww[wi] >> lane) & 1u);
          st_shared_v4(atom + sw128(rr * 32 + lane, 0), nw ? 0x3F803F80u : 0x00003F80u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        mbar_expect_tx(&bars->v_full[s], Lay::kTile);
#pragma unroll
        for (int ac = 0; ac < D / 64; ++ac)
          tma_load_4d(smem + Lay::kV + s * Lay::kVStage + ac * kAtom, &tmV, ac * 64, g, j * kBN, b,
                      &bars->v_full[s]);
      }
      return true;
    };
    // the order the MMA issuer consumes them: K0, K1, V0, K2, V1, K3, V2, ...
    // The newly-written flags (for V's statistics columns) are read from global
    // memory after the first K copies are on their way, not before.
    int nk = 0, nv = 0;
    bool ok = issue_k(0);
    if (ok) nk = 1;
    for (int j = 0; ok && j < T; ++j) {
      if (j + 1 < T) {
        if (!(ok = issue_k(j + 1))) break;
        nk = j + 2;
      }
      if (j == 0) {
        for (int w = lane; w < W; w += 32) neww[w] = p.newbits[(int64_t)b * W + w];
        __syncwarp();
      }
      if (!(ok = issue_v(j))) break;
      nv = j + 1;
    }
    // never leave with TMA writes in flight: the last load of every stage has landed
    for (int s = 0; s < kSK && s < nk; ++s) {
      const int j = nk - 1 - ((nk - 1 - s) % kSK + kSK) % kSK;  // last tile issued to stage s
      if (j >= 0) wait_bounded(&bars->k_full[s], (j / kSK) & 1, p.spin, abort_flag);
    }
    for (int s = 0; s < kSV && s < nv; ++s) {
      const int j = nv - 1 - ((nv - 1 - s) % kSV + kSV) % kSV;
      if (j >= 0) wait_bounded(&bars->v_full[s], (j / kSV) & 1, p.spin, abort_flag);
    }
    wait_bounded(&bars->q_full, 0, p.spin, abort_flag);
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(kBM, kBN, false);
      const uint32_t idO = idesc_bf16(kBM, D + 16, true);  // O and [l, l_new]
      const uint32_t sQ = sbase + Lay::kQ;
      auto qk = [&](int j) {
        const int s = j % kSK;
        const uint32_t sK = sbase + Lay::kK + s * Lay::kTile;
        const uint32_t dS = tmem + ((j & 1) ? Lay::kS1 : Lay::kS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kAtom + (kk % 4) * 32;
          mma_bf16(dS, desc_kmajor_sw128(sQ + off), desc_kmajor_sw128(sK + off), idS, kk > 0);
        }
        mma_commit(&bars->s_full[j & 1]);
        mma_commit(&bars->k_empty[s]);
      };
      bool ok = wait_bounded(&bars->q_full, 0, p.spin, abort_flag);
      ok = ok && wait_bounded(&bars->k_full[0], 0, p.spin, abort_flag);
      if (ok) {
        fence_after_sync();
        qk(0);
      }
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) {
          ok = wait_bounded(&bars->k_full[(j + 1) % kSK], ((j + 1) / kSK) & 1, p.spin, abort_flag);
          // S(j+1) overwrites the buffer that held P(j-1): PV(j-1) must be done
          if (ok && j >= 1) ok = wait_bounded(&bars->pv_done, (j - 1) & 1, p.spin, abort_flag);
          if (!ok) break;
          fence_after_sync();
          qk(j + 1);
        }
        const int s = j % kSV;
        ok = wait_bounded(&bars->p_full[j & 1], (j >> 1) & 1, p.spin, abort_flag) &&
             wait_bounded(&bars->v_full[s], (j / kSV) & 1, p.spin, abort_flag);
        if (!ok) break;
        fence_after_sync();
        const uint32_t tP = tmem + ((j & 1) ? Lay::kS1 : Lay::kS0);  // P(j), bf16 pairs
        const uint32_t sV = sbase + Lay::kV + s * Lay::kVStage;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_bf16_ts(tmem + Lay::kO, tP + kk * 8, desc_mnmajor_sw128(sV + kk * 16 * 128, kAtom),
                      idO, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->pv_done);
        mma_commit(&bars->v_empty[s]);
      }
      // all issued tensor-core work done before TMEM is released
      mma_commit(&bars->drain);
      wait_bounded(&bars->drain, 0, p.spin, abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int i = q0 + r;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool seed_row =
        i < L && p.is_seed != nullptr && p.is_seed[(int64_t)b * L + i] != 0;
    // rank among the sequence's masked rows (-1: not masked or no pass 2)
    const int rank = (p.q_m != nullptr && i < L) ? p.mrank[(int64_t)b * L + i] : -1;
    const float c2 = p.scale_log2;
    if (seed_row) {
      // the epilogue's diagonal term reads this row of q, k_cur and v_cur: bring them
      // into L2 while the tiles stream
      const int64_t qoff = (((int64_t)b * L + i) * p.Hq + h) * D;
      const int64_t koff = (((int64_t)b * L + i) * p.Hkv + g) * D;
#pragma unroll
      for (int c = 0; c < D * 2; c += 128) {
        prefetch_l2(reinterpret_cast<const char*>(p.q + qoff) + c);
        prefetch_l2(reinterpret_cast<const char*>(p.k_cur + koff) + c);
        prefetch_l2(reinterpret_cast<const char*>(p.v_cur + koff) + c);
      }
    }
    float m = -INFINITY;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      // warp-uniform outcome: the tcgen05 loads below are warp-wide
      ok = __all_sync(0xffffffffu,
                      wait_bounded(&bars->s_full[j & 1], (j >> 1) & 1, p.spin, abort_flag));
      if (!ok) break;
      fence_after_sync();
      float s[kBN];
      {
        const uint32_t scol = (j & 1) ? Lay::kS1 : Lay::kS0;
#pragma unroll
        for (int q = 0; q < kBN / 32; ++q) {
          float t[32];
          tmem_ld32(tl + scol + q * 32, t);
#pragma unroll
          for (int e = 0; e < 32; ++e) s[q * 32 + e] = t[e];
        }
        tmem_wait_ld();
      }
      if ((j + 1) * kBN > L) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (j * kBN + c >= L) s[c] = -INFINITY;
      }
      if (seed_row && j == i / kBN) {
        // the seed's own column (query tiles need not line up with key tiles)
        const int sc = i & (kBN - 1);
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c == sc) s[c] = -INFINITY;
      }
      // row maximum: eight independent chains of three-input maxima, then a tree
      float pm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pm[e] = fmax3(s[e], s[8 + e], s[16 + e]);
      static_assert((kBN - 24) % 16 == 8, "chain schedule assumes 128 columns");
#pragma unroll
      for (int c = 24; c + 16 <= kBN; c += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e) pm[e] = fmax3(pm[e], s[c + e], s[c + 8 + e]);
#pragma unroll
      for (int e = 0; e < 8; ++e) pm[e] = fmaxf(pm[e], s[kBN - 8 + e]);
      float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
      mx *= c2;
      const bool need = mx > m + 8.f;
      const float m_new = need ? mx : m;
      const bool resc = need && j > 0 && m != -INFINITY;
      if (__any_sync(0xffffffffu, resc)) {
        // O (and the statistics columns) may only be rescaled once PV(j-1) is done
        ok = __all_sync(0xffffffffu,
                        wait_bounded(&bars->pv_done, (j - 1) & 1, p.spin, abort_flag));
        if (!ok) break;
        fence_after_sync();
        const float f = resc ? exp2f(m - m_new) : 1.f;
#pragma unroll 1
        for (int q = 0; q < D / 32 + 1; ++q) {
          float o[32];
          tmem_ld32(tl + Lay::kO + q * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= f;
          tmem_st32(tl + Lay::kO + q * 32, o);
        }
        tmem_wait_st();
      }
      m = m_new;
      // P = exp2(S * scale * log2e - m) as bf16 pairs over the first 64 columns of
      // this tile's S buffer (already read into registers): the A operand of PV.
      // While every score so far is masked (m = -inf) all of S is -inf and a zero
      // reference gives exp2(-inf) = 0 without a per-element select.
      const float mref = m == -INFINITY ? 0.f : m;
      const uint32_t scol = (j & 1) ? Lay::kS1 : Lay::kS0;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = half * 64 + 2 * e;
          const float a = fast_exp2(fmaf(s[c], c2, -mref));
          const float bb = fast_exp2(fmaf(s[c + 1], c2, -mref));
          w[e] = pack_bf16(a, bb);
        }
        tmem_st32u(tl + scol + half * 32, w);
      }
      tmem_wait_st();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[j & 1]);
    }
    // Warps may be a tile apart, so pv_done's parity cannot tell PV(T-1) from
    // PV(T-3) here; drain completes once, after every tensor-core operation.
    if (ok) ok = __all_sync(0xffffffffu, wait_bounded(&bars->drain, 0, p.spin, abort_flag));
    if (ok) {
      fence_after_sync();
      float o[D];
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        float t[32];
        tmem_ld32(tl + Lay::kO + q * 32, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[q * 32 + e] = t[e];
      }
      float st[32];
      tmem_ld32(tl + Lay::kSt, st);
      tmem_wait_ld();
      float l = st[0], ln = st[1];
      if (seed_row) {
        // leave-one-out diagonal: the seed's own column from the masked input
        const int64_t qoff = (((int64_t)b * L + i) * p.Hq + h) * D;
        const int64_t koff = (((int64_t)b * L + i) * p.Hkv + g) * D;
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 qa = ldg16(p.q + qoff + c * 8), ka = ldg16(p.k_cur + koff + c * 8);
          dot += bf16lo(qa.x) * bf16lo(ka.x) + bf16hi(qa.x) * bf16hi(ka.x) +
                 bf16lo(qa.y) * bf16lo(ka.y) + bf16hi(qa.y) * bf16hi(ka.y) +
                 bf16lo(qa.z) * bf16lo(ka.z) + bf16hi(qa.z) * bf16hi(ka.z) +
                 bf16lo(qa.w) * bf16lo(ka.w) + bf16hi(qa.w) * bf16hi(ka.w);
        }
        const float sd = dot * c2;
        const float mn = fmaxf(m, sd);
        const float f = m == -INFINITY ? 0.f : exp2f(m - mn);
        const float pd = exp2f(sd - mn);
        const bool self_new = p.is_new != nullptr && p.is_new[(int64_t)b * L + i] != 0;
        l = l * f + pd;
        ln = ln * f + (self_new ? pd : 0.f);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 va = ldg16(p.v_cur + koff + c * 8);
          o[c * 8 + 0] = fmaf(pd, bf16lo(va.x), o[c * 8 + 0] * f);
          o[c * 8 + 1] = fmaf(pd, bf16hi(va.x), o[c * 8 + 1] * f);
          o[c * 8 + 2] = fmaf(pd, bf16lo(va.y), o[c * 8 + 2] * f);
          o[c * 8 + 3] = fmaf(pd, bf16hi(va.y), o[c * 8 + 3] * f);
          o[c * 8 + 4] = fmaf(pd, bf16lo(va.z), o[c * 8 + 4] * f);
          o[c * 8 + 5] = fmaf(pd, bf16hi(va.z), o[c * 8 + 5] * f);
          o[c * 8 + 6] = fmaf(pd, bf16lo(va.w), o[c * 8 + 6] * f);
          o[c * 8 + 7] = fmaf(pd, bf16hi(va.w), o[c * 8 + 7] * f);
        }
        m = mn;
      }
      if (i < L) {
        const float inv = 1.f / l;
        uint4* dst = reinterpret_cast<uint4*>(p.out + (((int64_t)b * L + i) * p.Hq + h) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          uint4 v;
          v.x = pack_bf16(o[c * 8 + 0] * inv, o[c * 8 + 1] * inv);
          v.y = pack_bf16(o[c * 8 + 2] * inv, o[c * 8 + 3] * inv);
          v.z = pack_bf16(o[c * 8 + 4] * inv, o[c * 8 + 5] * inv);
          v.w = pack_bf16(o[c * 8 + 6] * inv, o[c * 8 + 7] * inv);
          dst[c] = v;
        }
        const float lse2 = m + log2f(l);
        p.lse[((int64_t)b * p.Hq + h) * L + i] = lse2 * kLn2;
        if (p.dout_part) p.dout_part[((int64_t)b * p.Hq + h) * L + i] = ln * inv;
        if (rank >= 0 && DD_IN_BOUNDS(rank < L)) {
          // pass 2's inputs for a still-masked row: its Q row (from the staged,
          // swizzled tile; q_full completed long before) and its lse in log2 units
          wait_bounded(&bars->q_full, 0, p.spin, abort_flag);
          uint4* qd = reinterpret_cast<uint4*>(p.q_m + (((int64_t)b * L + rank) * p.Hq + h) * D);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(sbase + Lay::kQ + (c / 8) * kAtom + sw128(r, c & 7)));
            qd[c] = v;
          }
          p.lse2_m[((int64_t)b * p.Hq + h) * p.Lp + rank] = lse2;
        }
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------------------- pass 2
// d_in partials: one CTA per (128 key columns, kv head, sequence). The key tile
// of the drafting view stays in shared memory; the CTA loops over the G query
// heads sharing this kv head and over tiles of 128 still-masked query rows,
// which pass 1 left in rank order (q_m) together with their lse (lse2_m, log2
// units). S^T = K Q_m^T puts one key column per TMEM lane, so each consumer
// thread sums exp2(S * scale * log2e - lse2) over its own column without any
// cross-thread reduction.
//   warp 0     producer: TMA of the key tile, then per row tile a TMA of the
//              Q_m tile and a bulk copy of its 128 lse values (double buffer)
//   warp 1     MMA issuer
//   warps 2-5  consumers (one key column each)
constexpr int kP2Threads = 192;

template <int D>
struct P2Layout {
  static constexpr int kTile = (D / 64) * kAtom;
  static constexpr int kK = 0;
  static constexpr int kQ = kK + kTile;        // two buffers
  static constexpr int kLse = kQ + 2 * kTile;  // two buffers of 128 floats
  static constexpr int kBar = kLse + 2 * 128 * 4;
  static constexpr int kBytes = kBar + 128;
};

struct P2Bars {
  uint64_t k_full;
  uint64_t q_full[2];
  uint64_t s_full[2];
  uint64_t c_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct P2Params {
  const int32_t* mcount;
  const float* lse2_m;  // [B, Hq, Lp]
  int L, Hq, Hkv, Lp;
  float scale_log2;
  float* din_part;  // [B, Hkv, L]
  uint32_t spin;
};

template <int D>
__global__ void __launch_bounds__(kP2Threads, 2)
attn_p2_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQm,
               const P2Params p) {
  using Lay = P2Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  P2Bars* bars = reinterpret_cast<P2Bars*>(smem + Lay::kBar);
  const uint32_t sbase = smem_u32(smem);
  const float* lse2 = reinterpret_cast<const float*>(smem + Lay::kLse);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int L = p.L;
  const int G = p.Hq / p.Hkv;
  const int col0 = kt * kBN;
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars->k_full, 1);
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bars->q_full[u], 1);
      mbar_init(&bars->s_full[u], 1);
      mbar_init(&bars->c_done[u], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  // set-up above touches only shared and tensor memory; the previous kernel's
  // outputs (the masked-row count, Q_m, lse) are read from here on
  pdl_wait();
  const int M0 = p.mcount[b];
  // (the lse window of the last row tile, [m0, m0 + 128), then stays inside Lp)
  const int M = DD_IN_BOUNDS(M0 >= 0 && M0 <= L) ? M0 : 0;
  const int nrt = (M + 127) / 128;
  const int NT = G * nrt;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      if (NT > 0) {
        mbar_expect_tx(&bars->k_full, Lay::kTile);
#pragma unroll
        for (int ac = 0; ac < D / 64; ++ac)
          tma_load_4d(smem + Lay::kK + ac * kAtom, &tmK, ac * 64, g, col0, b, &bars->k_full);
      }
      int issued = 0;
      for (int t = 0; t < NT; ++t) {
        const int u = t & 1;
        // buffer u is free once the consumers are done with tile t-2 (its QK is done too)
        if (t >= 2 && !wait_bounded(&bars->c_done[u], ((t >> 1) - 1) & 1, p.spin, abort_flag)) break;
        const int hh = g * G + t / nrt;
        const int m0 = (t % nrt) * 128;
        mbar_expect_tx(&bars->q_full[u], Lay::kTile + 128 * 4);
#pragma unroll
        for (int ac = 0; ac < D / 64; ++ac)
          tma_load_4d(smem + Lay::kQ + u * Lay::kTile + ac * kAtom, &tmQm, ac * 64, hh, m0, b,
                      &bars->q_full[u]);
        bulk_load(smem + Lay::kLse + u * 512, p.lse2_m + ((int64_t)b * p.Hq + hh) * p.Lp + m0, 512,
                  &bars->q_full[u]);
        issued = t + 1;
      }
      // never leave with copies in flight
      if (NT > 0) wait_bounded(&bars->k_full, 0, p.spin, abort_flag);
      for (int t = issued - 2 < 0 ? 0 : issued - 2; t < issued; ++t)
        wait_bounded(&bars->q_full[t & 1], (t >> 1) & 1, p.spin, abort_flag);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(kBM, kBN, false);
      const uint32_t sK = sbase + Lay::kK;
      bool ok = NT == 0 || wait_bounded(&bars->k_full, 0, p.spin, abort_flag);
      for (int t = 0; ok && t < NT; ++t) {
        const int u = t & 1;
        ok = wait_bounded(&bars->q_full[u], (t >> 1) & 1, p.spin, abort_flag);
        // S buffer u held tile t-2: its consumers must be done with it
        if (ok && t >= 2) ok = wait_bounded(&bars->c_done[u], ((t >> 1) - 1) & 1, p.spin, abort_flag);
        if (!ok) break;
        fence_after_sync();
        const uint32_t sQ = sbase + Lay::kQ + u * Lay::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kAtom + (kk % 4) * 32;
          mma_bf16(tmem + u * 128, desc_kmajor_sw128(sK + off), desc_kmajor_sw128(sQ + off), idS,
                   kk > 0);
        }
        mma_commit(&bars->s_full[u]);
      }
      mma_commit(&bars->drain);
      wait_bounded(&bars->drain, 0, p.spin, abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ consumers
    const int quarter = warp & 3;
    const int j = quarter * 32 + lane;  // key column within the tile
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float c2 = p.scale_log2;
    float acc = 0.f;
    bool ok = true;
    for (int t = 0; t < NT; ++t) {
      const int u = t & 1;
      // lse values land with the Q tile; S(t) done implies q_full(t) completed
      ok = __all_sync(0xffffffffu,
                      wait_bounded(&bars->s_full[u], (t >> 1) & 1, p.spin, abort_flag) &&
                          wait_bounded(&bars->q_full[u], (t >> 1) & 1, p.spin, abort_flag));
      if (!ok) break;
      fence_after_sync();
      const int nvalid = min(128, M - (t % nrt) * 128);  // rows past the count are unset
      float a0 = 0.f, a1 = 0.f;
      // two halves of 64 query rows (TMEM columns) each, to keep registers down
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        float s[64];
        {
          float t0[32], t1[32];
          tmem_ld32(tl + u * 128 + hq * 64, t0);
          tmem_ld32(tl + u * 128 + hq * 64 + 32, t1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            s[e] = t0[e];
            s[32 + e] = t1[e];
          }
        }
        const float4* lv = reinterpret_cast<const float4*>(lse2 + u * 128 + hq * 64);
        if (nvalid == 128) {
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            const float4 l4 = lv[c4];
            a0 += fast_exp2(fmaf(s[4 * c4 + 0], c2, -l4.x));
            a1 += fast_exp2(fmaf(s[4 * c4 + 1], c2, -l4.y));
            a0 += fast_exp2(fmaf(s[4 * c4 + 2], c2, -l4.z));
            a1 += fast_exp2(fmaf(s[4 * c4 + 3], c2, -l4.w));
          }
        } else {
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            const float4 l4 = lv[c4];
            const float l[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = hq * 64 + 4 * c4 + e;
              const float x = c < nvalid ? fmaf(s[4 * c4 + e], c2, -l[e]) : -INFINITY;
              if (e & 1) a1 += fast_exp2(x);
              else a0 += fast_exp2(x);
            }
          }
        }
      }
      acc += a0 + a1;
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->c_done[u]);
    }
    if (col0 + j < L) p.din_part[((int64_t)b * p.Hkv + g) * L + col0 + j] = acc;
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, 256);
  }
}

// --------------------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }();
  return fn;
}

// 4-D map over a [B, L, H, D] bf16 tensor, dims innermost first {D, H, L, B};
// box = 64 head-dim elements (128 bytes) x 1 head x 128 positions x 1 sequence.
bool make_map(CUtensorMap* map, const void* base, int D, int H, int L, int B, int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)L * H * D * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

P1Params p1_params(const AttnArgs& a, bool pass2) {
  P1Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k_cur = static_cast<const __nv_bfloat16*>(a.k_cur);
  p.v_cur = static_cast<const __nv_bfloat16*>(a.v_cur);
  p.is_seed = a.is_seed;
  p.is_new = a.is_new;
  p.newbits = a.newbits;
  p.mrank = a.mrank;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Lp = a.Lp;
  p.q_begin = a.q_begin;
  p.scale_log2 = a.scale * kLog2e;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.dout_part = a.dout_part;
  p.q_m = pass2 ? static_cast<__nv_bfloat16*>(a.q_m) : nullptr;
  p.lse2_m = a.lse2_m;
  p.spin = spin_limit();
  return p;
}

template <int D>
cudaError_t launch_p1(const AttnArgs& a, bool pass2, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  // without seeds the drafting view is the current input itself
  const void* kv = a.is_seed ? a.k_view : a.k_cur;
  const void* vv = a.is_seed ? a.v_view : a.v_cur;
  if (!make_map(&tq, a.q, D, a.Hq, a.L, a.B) || !make_map(&tk, kv, D, a.Hkv, a.L, a.B) ||
      !make_map(&tv, vv, D, a.Hkv, a.L, a.B))
    return cudaErrorInvalidValue;
  const P1Params p = p1_params(a, pass2);
  const DeviceInfo& di = device_info();
  const int smem = P1Layout<D>::kBytes + 1024;
  static int configured[64] = {};
  if (!configured[di.device & 63]) {
    cudaError_t e = cudaFuncSetAttribute(attn_p1_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[di.device & 63] = 1;
  }
  dim3 grid((a.L - a.q_begin + kBM - 1) / kBM, a.Hq, a.B);
  return launch_dependent(attn_p1_kernel<D>, grid, dim3(kP1Threads), smem, stream, tq, tk, tv, p);
}

template <int D>
cudaError_t launch_p2(const AttnArgs& a, cudaStream_t stream) {
  CUtensorMap tk, tqm;
  const void* kv = a.is_seed ? a.k_view : a.k_cur;
  if (!make_map(&tk, kv, D, a.Hkv, a.L, a.B) || !make_map(&tqm, a.q_m, D, a.Hq, a.L, a.B))
    return cudaErrorInvalidValue;
  const int smem = P2Layout<D>::kBytes + 1024;
  static int configured[64] = {};
  const int dev = device_info().device;
  if (!configured[dev & 63]) {
    cudaError_t e = cudaFuncSetAttribute(attn_p2_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[dev & 63] = 1;
  }
  P2Params p;
  p.mcount = a.mcount;
  p.lse2_m = a.lse2_m;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.Lp = a.Lp;
  p.scale_log2 = a.scale * kLog2e;
  p.din_part = a.din_part;
  p.spin = spin_limit();
  dim3 grid((a.L + kBN - 1) / kBN, a.Hkv, a.B);
  return launch_dependent(attn_p2_kernel<D>, grid, dim3(kP2Threads), smem, stream, tk, tqm, p);
}

}  // namespace

template <int D>
cudaError_t launch_p1x2(const AttnArgs& a, bool pass2, cudaStream_t stream);

// Both passes on tensor cores. d_in partials are per kv head ([B, Hkv, L]).
// Pass 1 takes two query tiles per CTA where that still gives every SM a few CTAs
// (the tiles then share K / V and the tensor core alternates between them), one
// tile per CTA otherwise (short sequences, where a 256-row CTA would leave SMs idle).
cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t stream, bool* handled,
                                int* din_slices) {
  *handled = true;
  const bool pass2 = a.d_in != nullptr && a.is_masked != nullptr;
  const int64_t ctas2 = (int64_t)((a.L - a.q_begin + 2 * kBM - 1) / (2 * kBM)) * a.Hq * a.B;
  const bool two = ctas2 >= 2 * (int64_t)device_info().sm_count;
  cudaError_t err = two ? (a.d == 64 ? launch_p1x2<64>(a, pass2, stream)
                                     : launch_p1x2<128>(a, pass2, stream))
                        : (a.d == 64 ? launch_p1<64>(a, pass2, stream)
                                     : launch_p1<128>(a, pass2, stream));
  if (err != cudaSuccess) return err;
  if (pass2) {
    err = a.d == 64 ? launch_p2<64>(a, stream) : launch_p2<128>(a, stream);
    *din_slices = a.Hkv;
  }
  return err;
}

}  // namespace dd
