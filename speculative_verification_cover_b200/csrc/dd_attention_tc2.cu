// Pass 1 of the tensor-core dual-view attention with two query tiles per CTA.
//
// One CTA owns 256 query rows of a head as two 128-row tiles, A and B, that
// share every K / V tile the CTA streams. The tensor core alternates between
// them -- PV(A, j), QK(A, j+1), PV(B, j), QK(B, j+1), ... -- so while one tile's
// softmax warps turn S into P the tensor core works on the other tile, and each
// K / V tile read from shared memory feeds twice the MMA work. Everything a row
// computes is as in the single-tile pass 1 (dd_attention_tc.cu): dual view from
// the materialised drafting view, the seed's own column masked and merged back
// in the epilogue, [O | l | l_new] from one PV MMA of N = D + 16.
//
// TMEM holds both tiles' S (P written over it as bf16 pairs) and both [O | l |
// l_new] accumulators: 2 kBN + 2 (D + 16) columns, which is exactly the 512 of
// an SM with 112-column key tiles at D = 128 (128-column tiles at D = 64).
//
//   warp 0      producer: TMA of both Q tiles, K / V tiles in 2-stage rings, the
//               [1, is_new] statistics block of each V stage
//   warp 1      MMA issuer (one thread)
//   warps 2-5   softmax of tile A (one query row per TMEM lane)
//   warps 6-9   softmax of tile B
// Every wait is bounded; on expiry the kernel records DD_ERR_TIMEOUT and winds down.

namespace dd {

namespace {

constexpr int kP1x2Threads = 320;

template <int D>
struct P1x2Layout {
  static constexpr int kBN = D == 128 ? 112 : 128;      // key columns per tile
  static constexpr int kQAtom = 128 * 128;              // 128 rows x 128 bytes
  static constexpr int kKAtom = kBN * 128;              // kBN rows x 128 bytes
  static constexpr int kQTile = (D / 64) * kQAtom;
  static constexpr int kKTile = (D / 64) * kKAtom;
  static constexpr int kVStage = kKTile + kKAtom;       // V tile + [1, is_new] block
  static constexpr int kQ = 0;                          // tile A, then tile B
  static constexpr int kK = kQ + 2 * kQTile;
  static constexpr int kV = kK + kSK * kKTile;
  static constexpr int kNew = kV + kSV * kVStage;
  static constexpr int kNewWords = kTcMaxL / 32;
  static constexpr int kBar = kNew + kNewWords * 4;
  static constexpr int kBytes = kBar + 256;
  // TMEM columns
  static constexpr uint32_t kOW = D + 16;               // [O | l | l_new | 0...]
  static constexpr uint32_t kSA = 0, kSB = kBN, kOA = 2 * kBN, kOB = 2 * kBN + kOW;
  static_assert(kOB + kOW <= kTmemCols, "two tiles' S and O must fit TMEM");
  static_assert(kKAtom % 1024 == 0 && kVStage % 1024 == 0, "swizzle atoms are 1 KB aligned");
  static_assert(kBytes + 1024 <= 232448, "shared memory per CTA");
  static_assert(kBN % 16 == 0 && kBN >= 96 && kBN <= 128, "key tile width");
};

struct P1x2Bars {
  uint64_t q_full;
  uint64_t k_full[kSK], k_empty[kSK];
  uint64_t v_full[kSV], v_empty[kSV];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// S columns [c0, c0 + N) of this thread's lane into s[c0 ...] (N a multiple of 16).
template <int N>
__device__ __forceinline__ void load_s(uint32_t taddr, float* s) {
#pragma unroll
  for (int q = 0; q < N / 32; ++q) {
    float t[32];
    tmem_ld32(taddr + q * 32, t);
#pragma unroll
    for (int e = 0; e < 32; ++e) s[q * 32 + e] = t[e];
  }
  if constexpr (N % 32 == 16) {
    float t[16];
    tmem_ld16(taddr + (N / 32) * 32, t);
#pragma unroll
    for (int e = 0; e < 16; ++e) s[(N / 32) * 32 + e] = t[e];
  }
}

// Multiply `ncols` (a multiple of 16) TMEM columns of this lane by f.
template <int NCOLS>
__device__ __forceinline__ void rescale_cols(uint32_t taddr, float f) {
#pragma unroll 1
  for (int q = 0; q < NCOLS / 32; ++q) {
    float o[32];
    tmem_ld32(taddr + q * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) o[e] *= f;
    tmem_st32(taddr + q * 32, o);
  }
  if constexpr (NCOLS % 32 == 16) {
    float o[16];
    tmem_ld16(taddr + (NCOLS / 32) * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; ++e) o[e] *= f;
    tmem_st16(taddr + (NCOLS / 32) * 32, o);
  }
}

template <int D>
__global__ void __launch_bounds__(kP1x2Threads, 1)
attn_p1x2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const P1Params p) {
  using Lay = P1x2Layout<D>;
  constexpr int kBN = Lay::kBN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  P1x2Bars* bars = reinterpret_cast<P1x2Bars*>(smem + Lay::kBar);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int L = p.L;
  const int g = h / (p.Hq / p.Hkv);
  const int q0 = p.q_begin + qt * 2 * kBM;  // tile A: q0.., tile B: q0 + 128..
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
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 4);
      mbar_init(&bars->pv_done[t], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // the statistics blocks start at zero (column 0 of each key row is rewritten per tile)
  if (warp >= 2) {
    const int t = threadIdx.x - 64;  // 0..255
    for (int idx = t; idx < kSV * kBN * 8; idx += kP1x2Threads - 64) {
      const int s = idx / (kBN * 8), row = (idx / 8) % kBN, c = idx % 8;
      st_shared_v4(sbase + Lay::kV + s * Lay::kVStage + Lay::kKTile + sw128(row, c), 0u, 0u, 0u,
                   0u);
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
      mbar_expect_tx(&bars->q_full, 2 * Lay::kQTile);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int ac = 0; ac < D / 64; ++ac)
          tma_load_4d(smem + Lay::kQ + t * Lay::kQTile + ac * Lay::kQAtom, &tmQ, ac * 64, h,
                      q0 + t * kBM, b, &bars->q_full);
    }
    uint32_t* neww = reinterpret_cast<uint32_t*>(smem + Lay::kNew);
    const int W = (L + 31) / 32;
    // K(j) may reuse its stage once QK(B, j - kSK) is done, V(j) once PV(B, j - kSV) is.
    auto issue_k = [&](int j) -> bool {
      const int s = j % kSK;
      if (j >= kSK && !wait_bounded(&bars->k_empty[s], ((j / kSK) - 1) & 1, p.spin, abort_flag))
        return false;
      if (lane == 0) {
        mbar_expect_tx(&bars->k_full[s], Lay::kKTile);
#pragma unroll
        for (int ac = 0; ac < D / 64; ++ac)
          tma_load_4d(smem + Lay::kK + s * Lay::kKTile + ac * Lay::kKAtom, &tmK, ac * 64, g,
                      j * kBN, b, &bars->k_full[s]);
      }
      return true;
    };
    auto issue_v = [&](int j) -> bool {
      const int s = j % kSV;
      if (j >= kSV && !wait_bounded(&bars->v_empty[s], ((j / kSV) - 1) & 1, p.spin, abort_flag))
        return false;
      {
        // statistics columns of key row r: [1, is_new(key), 0, ...]
        const uint32_t atom = sbase + Lay::kV + s * Lay::kVStage + Lay::kKTile;
#pragma unroll
        for (int rr0 = 0; rr0 < kBN; rr0 += 32) {
          const int rr = rr0 + lane;
          const int pos = j * kBN + rr;
          const bool nw = pos < L && ((neww[pos >> 5] >> (pos & 31)) & 1u);
          if (rr < kBN)
            st_shared_v4(atom + sw128(rr, 0), nw ? 0x3F803F80u : 0x00003F80u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        mbar_expect_tx(&bars->v_full[s], Lay::kKTile);
#pragma unroll
        for (int ac = 0; ac < D / 64; ++ac)
          tma_load_4d(smem + Lay::kV + s * Lay::kVStage + ac * Lay::kKAtom, &tmV, ac * 64, g,
                      j * kBN, b, &bars->v_full[s]);
      }
      return true;
    };
    // the order the MMA issuer consumes them: K0, V0, K1, V1, ...
    // The newly-written flags (for V's statistics columns) are read from global
    // memory after K0's copy is on its way, not before.
    int nk = 0, nv = 0;
    bool ok = issue_k(0);
    if (ok) nk = 1;
    for (int w = lane; w < W; w += 32) neww[w] = p.newbits[(int64_t)b * W + w];
    __syncwarp();
    for (int j = 0; ok && j < T; ++j) {
      if (!(ok = issue_v(j))) break;
      nv = j + 1;
      if (j + 1 < T) {
        if (!(ok = issue_k(j + 1))) break;
        nk = j + 2;
      }
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
  }
  else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // Order: QK(A,0) QK(B,0) | PV(A,j) QK(A,j+1) PV(B,j) QK(B,j+1) | ... A tile's S
    // buffer holds its P until that tile's PV has read it, so QK(t, j+1) waits for
    // PV(t, j) (pv_done[t]); the other tile's work keeps the tensor core busy meanwhile.
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(kBM, kBN, false);
      const uint32_t idO = idesc_bf16(kBM, D + 16, true);  // O and [l, l_new]
      auto qk = [&](int t, int j) {
        const uint32_t sQ = sbase + Lay::kQ + t * Lay::kQTile;
        const uint32_t sK = sbase + Lay::kK + (j % kSK) * Lay::kKTile;
        const uint32_t dS = tmem + (t ? Lay::kSB : Lay::kSA);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = (kk / 4) * Lay::kQAtom + (kk % 4) * 32;
          const uint32_t koff = (kk / 4) * Lay::kKAtom + (kk % 4) * 32;
          mma_bf16(dS, desc_kmajor_sw128(sQ + qoff), desc_kmajor_sw128(sK + koff), idS, kk > 0);
        }
        mma_commit(&bars->s_full[t]);
      };
      auto pv = [&](int t, int j) {
        const uint32_t tP = tmem + (t ? Lay::kSB : Lay::kSA);  // P(t, j), bf16 pairs
        const uint32_t sV = sbase + Lay::kV + (j % kSV) * Lay::kVStage;
        const uint32_t dO = tmem + (t ? Lay::kOB : Lay::kOA);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_bf16_ts(dO, tP + kk * 8, desc_mnmajor_sw128(sV + kk * 16 * 128, Lay::kKAtom), idO,
                      (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->pv_done[t]);
      };
      bool ok = wait_bounded(&bars->q_full, 0, p.spin, abort_flag) &&
                wait_bounded(&bars->k_full[0], 0, p.spin, abort_flag);
      if (ok) {
        fence_after_sync();
        qk(0, 0);
        qk(1, 0);
        mma_commit(&bars->k_empty[0]);
      }
      for (int j = 0; ok && j < T; ++j) {
        const int sv = j % kSV;
        const bool more = j + 1 < T;
        ok = wait_bounded(&bars->v_full[sv], (j / kSV) & 1, p.spin, abort_flag) &&
             wait_bounded(&bars->p_full[0], j & 1, p.spin, abort_flag);
        if (!ok) break;
        fence_after_sync();
        pv(0, j);
        if (more) {
          ok = wait_bounded(&bars->k_full[(j + 1) % kSK], ((j + 1) / kSK) & 1, p.spin,
                            abort_flag) &&
               wait_bounded(&bars->pv_done[0], j & 1, p.spin, abort_flag);
          if (!ok) break;
          fence_after_sync();
          qk(0, j + 1);
        }
        ok = wait_bounded(&bars->p_full[1], j & 1, p.spin, abort_flag);
        if (!ok) break;
        fence_after_sync();
        pv(1, j);
        mma_commit(&bars->v_empty[sv]);
        if (more) {
          ok = wait_bounded(&bars->pv_done[1], j & 1, p.spin, abort_flag);
          if (!ok) break;
          fence_after_sync();
          qk(1, j + 1);
          mma_commit(&bars->k_empty[(j + 1) % kSK]);
        }
      }
      // all issued tensor-core work done before TMEM is released
      mma_commit(&bars->drain);
      wait_bounded(&bars->drain, 0, p.spin, abort_flag);
    }
    __syncwarp();
  }
  else {
    // ------------------------------------------------------------------ softmax, tile t
    const int t = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int i = q0 + t * kBM + r;
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t scol = t ? Lay::kSB : Lay::kSA;
    const uint32_t ocol = t ? Lay::kOB : Lay::kOA;
    const bool seed_row = i < L && p.is_seed != nullptr && p.is_seed[(int64_t)b * L + i] != 0;
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
                      wait_bounded(&bars->s_full[t], j & 1, p.spin, abort_flag));
      if (!ok) break;
      fence_after_sync();
      float s[kBN];
      load_s<kBN>(tl + scol, s);
      tmem_wait_ld();
      if ((j + 1) * kBN > L) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (j * kBN + c >= L) s[c] = -INFINITY;
      }
      if (seed_row && j == i / kBN) {
        const int sc = i - j * kBN;  // the seed's own column
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c == sc) s[c] = -INFINITY;
      }
      // row maximum: eight independent chains of three-input maxima, then a tree
      float pm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pm[e] = fmax3(s[e], s[8 + e], s[16 + e]);
      static_assert((kBN - 24) % 16 == 8, "chain schedule");
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
      const float fres = resc ? exp2f(m - m_new) : 1.f;
      m = m_new;
      // P = exp2(S * scale * log2e - m) as bf16 pairs over the first kBN/2 columns of
      // this tile's S buffer (already read into registers): the A operand of PV.
      const float mref = m == -INFINITY ? 0.f : m;
      // packed and stored chunk by chunk, so S values die as they are consumed
      {
        constexpr int NW = kBN / 2;
#pragma unroll
        for (int c = 0; c + 32 <= NW; c += 32) {
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e)
            w[e] = pack_bf16(fast_exp2(fmaf(s[2 * (c + e)], c2, -mref)),
                             fast_exp2(fmaf(s[2 * (c + e) + 1], c2, -mref)));
          tmem_st32u(tl + scol + c, w);
        }
        if constexpr (NW % 32 >= 16) {
          constexpr int c = (NW / 32) * 32;
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16(fast_exp2(fmaf(s[2 * (c + e)], c2, -mref)),
                             fast_exp2(fmaf(s[2 * (c + e) + 1], c2, -mref)));
          tmem_st16u(tl + scol + c, w);
        }
        if constexpr (NW % 16 == 8) {
          constexpr int c = NW - 8;
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            w[e] = pack_bf16(fast_exp2(fmaf(s[2 * (c + e)], c2, -mref)),
                             fast_exp2(fmaf(s[2 * (c + e) + 1], c2, -mref)));
          tmem_st8u(tl + scol + c, w);
        }
      }
      tmem_wait_st();
      // With P(t, j) stored (S is dead), a grown maximum rescales O and the statistics
      // columns -- once PV(t, j-1) is done, and before PV(t, j), which waits for p_full.
      if (__any_sync(0xffffffffu, resc)) {
        ok = __all_sync(0xffffffffu,
                        wait_bounded(&bars->pv_done[t], (j - 1) & 1, p.spin, abort_flag));
        if (!ok) break;
        fence_after_sync();
        rescale_cols<D + 16>(tl + ocol, fres);
        tmem_wait_st();
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[t]);
    }
    // drain completes once, after every tensor-core operation
    if (ok) ok = __all_sync(0xffffffffu, wait_bounded(&bars->drain, 0, p.spin, abort_flag));
    if (ok) {
      fence_after_sync();
      float o[D];
      load_s<D>(tl + ocol, o);
      float st[16];
      tmem_ld16(tl + ocol + D, st);
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
          const uint32_t qbase = sbase + Lay::kQ + t * Lay::kQTile;
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(qbase + (c / 8) * Lay::kQAtom + sw128(r, c & 7)));
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

}  // namespace

template <int D>
cudaError_t launch_p1x2(const AttnArgs& a, bool pass2, cudaStream_t stream) {
  using Lay = P1x2Layout<D>;
  CUtensorMap tq, tk, tv;
  const void* kv = a.is_seed ? a.k_view : a.k_cur;
  const void* vv = a.is_seed ? a.v_view : a.v_cur;
  if (!make_map(&tq, a.q, D, a.Hq, a.L, a.B) ||
      !make_map(&tk, kv, D, a.Hkv, a.L, a.B, Lay::kBN) ||
      !make_map(&tv, vv, D, a.Hkv, a.L, a.B, Lay::kBN))
    return cudaErrorInvalidValue;
  const P1Params p = p1_params(a, pass2);
  const int smem = Lay::kBytes + 1024;
  static int configured[64] = {};
  const int dev = device_info().device;
  if (!configured[dev & 63]) {
    cudaError_t e = cudaFuncSetAttribute(attn_p1x2_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[dev & 63] = 1;
  }
  dim3 grid((a.L - a.q_begin + 2 * kBM - 1) / (2 * kBM), a.Hq, a.B);
  return launch_dependent(attn_p1x2_kernel<D>, grid, dim3(kP1x2Threads), smem, stream, tq, tk, tv,
                          p);
}

template cudaError_t launch_p1x2<64>(const AttnArgs&, bool, cudaStream_t);
template cudaError_t launch_p1x2<128>(const AttnArgs&, bool, cudaStream_t);

}  // namespace dd
