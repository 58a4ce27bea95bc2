// Tensor-core (sm_100a, tcgen05) dual-view attention for bf16 inputs.
//
// Pass 1, one CTA per (128 query rows, head, sequence), warp-specialised:
//   warp 0      producer: TMA loads of the Q tile and of K/V tiles (128 columns,
//               two stages) from k_cur / v_cur; then, per tile, overwrites the
//               rows of seed columns with the step t-1 cache (k_prev / v_prev,
//               plain loads + swizzled shared stores) -- the drafting view; and
//               writes the tile's "newly written" flags into a small B operand
//               whose rows are [1, is_new, 0, ...].
//   warp 1      MMA issuer (one thread): S = Q K^T into a double-buffered TMEM
//               accumulator; O += P V and [l, l_new] += P [1, is_new]^T, i.e. the
//               row sum and the mass on newly written columns come out of the
//               tensor core with the same bf16 P that weights V.
//   warps 2-5   softmax (one thread per query row = TMEM lane): online max with
//               a lazy rescale (O is rescaled in TMEM only when the running max
//               grows by more than 2^8), P = exp2(S*scale*log2e - m) as bf16 into
//               shared memory. A seed query's own column is masked in the loop and
//               merged back afterwards from k_cur / v_cur (leave-one-out
//               diagonal). Epilogue: out = O / l, lse, d_out partial = l_new / l.
// Every wait is bounded; on expiry the kernel records DD_ERR_TIMEOUT and winds down.
#include <cudaTypedefs.h>

#include "dd_internal.h"
#include "dd_tc.cuh"

namespace dd {

namespace {

using namespace tc;

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kStages = 2;
constexpr int kP1Threads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kAtom = 128 * 128;  // one 128-row x 128-byte swizzle atom column

template <int D>
struct P1Layout {
  static constexpr int kTile = (D / 64) * kAtom;  // 128 x D bf16
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kB2 = kV + kStages * kTile;
  static constexpr int kB2Bytes = 2 * 16 * 128;       // 16 rows x 128 columns bf16
  // staging for up to kStaged seed rows of the step t-1 cache per stage (K then V rows)
  static constexpr int kStaged = 16;
  static constexpr int kRowBytes = D * 2;
  static constexpr int kStage = kB2 + kStages * kB2Bytes;
  static constexpr int kStageBytes = 2 * kStaged * kRowBytes;
  // packed seed / newly-written flags of the whole sequence
  static constexpr int kMask = kStage + kStages * kStageBytes;
  static constexpr int kMaskWords = kTcMaxL / 32;
  static constexpr int kBar = kMask + 2 * kMaskWords * 4;
  static constexpr int kBytes = kBar + 256;
  // TMEM columns
  static constexpr uint32_t kS0 = 0, kS1 = 128, kO = 256, kSt = 256 + D;
};

struct P1Bars {
  uint64_t q_full;
  uint64_t k_full[kStages], k_ready[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_ready[kStages], v_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct P1Params {
  const __nv_bfloat16 *q, *k_cur, *v_cur, *k_prev, *v_prev;
  const uint8_t *is_seed, *is_new;
  const uint32_t *seedbits, *newbits;  // [B, ceil(L/32)]
  int L, Hq, Hkv;
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  float* dout_part;
  uint32_t spin;
};

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}

template <int D>
__global__ void __launch_bounds__(kP1Threads, 1)
attn_p1_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKp,
               const __grid_constant__ CUtensorMap tmVp, const P1Params p) {
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
  const int q0 = qt * kBM;
  const int T = (L + kBN - 1) / kBN;
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_ready[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_ready[s], 1);
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
  // constant rows of the [1, is_new, 0...] operand: row 0 = ones, rows 2..15 = 0
  if (warp >= 2) {
    const int t = threadIdx.x - 64;  // 0..127
    for (int idx = t; idx < kStages * 2 * 16 * 8; idx += 128) {
      const int s = idx / (2 * 16 * 8), rem = idx % (2 * 16 * 8);
      const int ac = rem / (16 * 8), row = (rem / 8) % 16, c = rem % 8;
      const uint32_t one = 0x3F803F80u;  // two bf16 1.0
      const uint32_t v = row == 0 ? one : 0u;
      st_shared_v4(sbase + Lay::kB2 + s * Lay::kB2Bytes + ac * 2048 + sw128(row, c), v, v, v, v);
    }
    fence_proxy_async();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    constexpr uint32_t kTxQ = Lay::kTile, kTxKV = 2 * Lay::kTile;
    if (lane == 0) {
      mbar_expect_tx(&bars->q_full, kTxQ);
#pragma unroll
      for (int ac = 0; ac < D / 64; ++ac)
        tma_load_4d(smem + Lay::kQ + ac * kAtom, &tmQ, ac * 64, h, q0, b, &bars->q_full);
    }
    // the sequence's packed flags into shared memory
    uint32_t* seedw = reinterpret_cast<uint32_t*>(smem + Lay::kMask);
    uint32_t* neww = seedw + Lay::kMaskWords;
    const int W = (L + 31) / 32;
    for (int w = lane; w < W; w += 32) {
      seedw[w] = p.seedbits[(int64_t)b * W + w];
      neww[w] = p.newbits[(int64_t)b * W + w];
    }
    __syncwarp();
    // Tile j of K (resp. V): the current input's rows, plus (same barrier) up to
    // kStaged seed rows of the step t-1 cache into the stage's staging area. K
    // and V have their own stages so K(j+2) can load as soon as QK(j) is done.
    auto seeds_in_tile = [&](int j) {
      int n = 0;
      for (int w = 0; w < 4; ++w) {
        const int wi = j * 4 + w;
        n += wi < W ? __popc(seedw[wi]) : 0;
      }
      return min(n, Lay::kStaged);
    };
    auto issue = [&](int j, bool is_v) {
      const int s = j % kStages;
      if (lane == 0) {
        const int n = seeds_in_tile(j);
        uint64_t* bar = is_v ? &bars->v_full[s] : &bars->k_full[s];
        mbar_expect_tx(bar, Lay::kTile + (uint32_t)n * Lay::kRowBytes);
        const CUtensorMap* tm = is_v ? &tmV : &tmK;
        const CUtensorMap* tmp = is_v ? &tmVp : &tmKp;
        uint8_t* tile = smem + (is_v ? Lay::kV : Lay::kK) + s * Lay::kTile;
#pragma unroll
        for (int ac = 0; ac < D / 64; ++ac)
          tma_load_4d(tile + ac * kAtom, tm, ac * 64, g, j * kBN, b, bar);
        uint8_t* stg = smem + Lay::kStage + s * Lay::kStageBytes +
                       (is_v ? Lay::kStaged * Lay::kRowBytes : 0);
        int slot = 0;
        for (int w = 0; w < 4 && slot < n; ++w) {
          const int wi = j * 4 + w;
          uint32_t bits = wi < W ? seedw[wi] : 0u;
          while (bits && slot < n) {
            const int r = w * 32 + __ffs(bits) - 1;
            bits &= bits - 1;
            tma_load_4d(stg + slot * Lay::kRowBytes, tmp, 0, g, j * kBN + r, b, bar);
            ++slot;
          }
        }
      }
    };
    auto finalize = [&](int j, bool is_v) -> bool {
      const int s = j % kStages;
      uint64_t* full = is_v ? &bars->v_full[s] : &bars->k_full[s];
      if (!wait_bounded(full, (j / kStages) & 1, p.spin, abort_flag)) return false;
      const int col0 = j * kBN;
      const uint32_t stg = sbase + Lay::kStage + s * Lay::kStageBytes +
                           (is_v ? Lay::kStaged * Lay::kRowBytes : 0);
      const uint32_t tile = sbase + (is_v ? Lay::kV : Lay::kK) + s * Lay::kTile;
      const __nv_bfloat16* prev = is_v ? p.v_prev : p.k_prev;
      // two seed rows at a time: lanes 0-15 and 16-31
      const int half = lane >> 4, ch = lane & 15;
      int slot = 0;
      for (int w = 0; w < 4; ++w) {
        const int wi = j * 4 + w;
        uint32_t bits = wi < W ? seedw[wi] : 0u;
        while (bits) {
          int r0 = w * 32 + __ffs(bits) - 1;
          bits &= bits - 1;
          int r1 = -1;
          if (bits) {
            r1 = w * 32 + __ffs(bits) - 1;
            bits &= bits - 1;
          }
          const int r = half ? r1 : r0;
          const int sl = slot + half;
          if (r >= 0 && ch < D / 8) {
            uint4 val;
            if (sl < Lay::kStaged) {
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                           : "r"(stg + sl * Lay::kRowBytes + ch * 16));
            } else {
              val = ldg16(prev + (((int64_t)b * L + col0 + r) * p.Hkv + g) * D + ch * 8);
            }
            st_shared_v4(tile + (ch / 8) * kAtom + sw128(r, ch & 7), val.x, val.y, val.z, val.w);
          }
          slot += r1 >= 0 ? 2 : 1;
        }
      }
      if (is_v && lane < 16) {
        // row 1 of the statistics operand: the tile's newly-written flags
        const int wi = j * 4 + lane / 4;
        const uint32_t byte = ((wi < W ? neww[wi] : 0u) >> ((lane & 3) * 8)) & 0xFFu;
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w4[e] = ((byte >> (2 * e)) & 1u ? 0x3F80u : 0u) |
                  ((byte >> (2 * e + 1)) & 1u ? 0x3F800000u : 0u);
        st_shared_v4(sbase + Lay::kB2 + s * Lay::kB2Bytes + (lane / 8) * 2048 + sw128(1, lane & 7),
                     w4[0], w4[1], w4[2], w4[3]);
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(is_v ? &bars->v_ready[s] : &bars->k_ready[s]);
      return true;
    };
    int issued_k = 0, issued_v = 0, fin_k = 0, fin_v = 0;
    for (int j = 0; j < T && j < kStages; ++j) {
      issue(j, false);
      ++issued_k;
      issue(j, true);
      ++issued_v;
    }
    bool ok = finalize(0, false);
    if (ok) fin_k = 1;
    ok = ok && finalize(0, true);
    if (ok) fin_v = 1;
    for (int j = 0; ok && j < T; ++j) {
      if (j + 1 < T) {
        if (!(ok = finalize(j + 1, false))) break;
        fin_k = j + 2;
      }
      if (j + kStages < T) {
        // K stage of tile j is free once QK(j) is done
        if (!(ok = wait_bounded(&bars->k_empty[j % kStages], (j / kStages) & 1, p.spin,
                                abort_flag)))
          break;
        issue(j + kStages, false);
        ++issued_k;
      }
      if (j + 1 < T) {
        if (!(ok = finalize(j + 1, true))) break;
        fin_v = j + 2;
      }
      if (j + kStages < T) {
        // V stage of tile j is free once PV(j) is done
        if (!(ok = wait_bounded(&bars->v_empty[j % kStages], (j / kStages) & 1, p.spin,
                                abort_flag)))
          break;
        issue(j + kStages, true);
        ++issued_v;
      }
    }
    // never leave with TMA writes in flight
    for (int j = fin_k; j < issued_k; ++j)
      wait_bounded(&bars->k_full[j % kStages], (j / kStages) & 1, p.spin, abort_flag);
    for (int j = fin_v; j < issued_v; ++j)
      wait_bounded(&bars->v_full[j % kStages], (j / kStages) & 1, p.spin, abort_flag);
    wait_bounded(&bars->q_full, 0, p.spin, abort_flag);
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(kBM, kBN, false);
      const uint32_t idO = idesc_bf16(kBM, D, true);
      const uint32_t idSt = idesc_bf16(kBM, 16, false);
      const uint32_t sQ = sbase + Lay::kQ;
      auto qk = [&](int j) {
        const int s = j % kStages;
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
      ok = ok && wait_bounded(&bars->k_ready[0], 0, p.spin, abort_flag);
      if (ok) {
        fence_after_sync();
        qk(0);
      }
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) {
          const int s1 = (j + 1) % kStages;
          ok = wait_bounded(&bars->k_ready[s1], ((j + 1) / kStages) & 1, p.spin, abort_flag);
          // S(j+1) overwrites the buffer that held P(j-1): PV(j-1) must be done
          if (ok && j >= 1) ok = wait_bounded(&bars->pv_done, (j - 1) & 1, p.spin, abort_flag);
          if (!ok) break;
          fence_after_sync();
          qk(j + 1);
        }
        const int s = j % kStages;
        ok = wait_bounded(&bars->p_full[j & 1], (j >> 1) & 1, p.spin, abort_flag) &&
             wait_bounded(&bars->v_ready[s], (j / kStages) & 1, p.spin, abort_flag);
        if (!ok) break;
        fence_after_sync();
        const uint32_t tP = tmem + ((j & 1) ? Lay::kS1 : Lay::kS0);  // P(j), bf16 pairs
        const uint32_t sV = sbase + Lay::kV + s * Lay::kTile;
        const uint32_t sB2 = sbase + Lay::kB2 + s * Lay::kB2Bytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          mma_bf16_ts(tmem + Lay::kO, tP + kk * 8, desc_mnmajor_sw128(sV + kk * 16 * 128, kAtom),
                      idO, acc);
          mma_bf16_ts(tmem + Lay::kSt, tP + kk * 8,
                      desc_kmajor_sw128(sB2 + (kk / 4) * 2048 + (kk % 4) * 32), idSt, acc);
        }
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
    const float c2 = p.scale_log2;
    float m = -INFINITY;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      ok = wait_bounded(&bars->s_full[j & 1], (j >> 1) & 1, p.spin, abort_flag);
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
      if (seed_row && j == qt) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c == r) s[c] = -INFINITY;
      }
      // row maximum: eight independent chains, then a tree (short dependency chain)
      float pm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pm[e] = s[e];
#pragma unroll
      for (int c = 8; c < kBN; c += 8)
#pragma unroll
        for (int e = 0; e < 8; ++e) pm[e] = fmaxf(pm[e], s[c + e]);
      float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                       fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      mx *= c2;
      const bool need = mx > m + 8.f;
      const float m_new = need ? mx : m;
      const bool resc = need && j > 0 && m != -INFINITY;
      if (__any_sync(0xffffffffu, resc)) {
        // O (and the statistics columns) may only be rescaled once PV(j-1) is done
        ok = wait_bounded(&bars->pv_done, (j - 1) & 1, p.spin, abort_flag);
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
      const bool live = m != -INFINITY;
      // P = exp2(S * scale * log2e - m) as bf16 pairs over the first 64 columns of
      // this tile's S buffer (already read into registers): the A operand of PV.
      const uint32_t scol = (j & 1) ? Lay::kS1 : Lay::kS0;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = half * 64 + 2 * e;
          const float a = live ? fast_exp2(fmaf(s[c], c2, -m)) : 0.f;
          const float bb = live ? fast_exp2(fmaf(s[c + 1], c2, -m)) : 0.f;
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
    if (ok) ok = wait_bounded(&bars->drain, 0, p.spin, abort_flag);
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
        p.lse[((int64_t)b * p.Hq + h) * L + i] = (m + log2f(l)) * kLn2;
        if (p.dout_part) p.dout_part[((int64_t)b * p.Hq + h) * L + i] = ln * inv;
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
// (drafting view: seed columns from the cache) stays in shared memory; the CTA
// loops over the G query heads sharing this kv head and over tiles of 128
// still-masked query rows (gathered). S^T = K Q_m^T puts one key column per
// TMEM lane, so each consumer thread sums exp2(S * scale * log2e - lse2) over
// its own column without any cross-thread reduction.
//   warps 0-3  producers: warp 0 issues the key TMA and patches seed rows; all
//              four gather masked query rows (plain loads, swizzled stores) and
//              their lse (natural log -> log2 units) into a double buffer
//   warp 4     MMA issuer
//   warps 5-8  consumers (one key column each)
constexpr int kP2Threads = 288;

template <int D>
struct P2Layout {
  static constexpr int kTile = (D / 64) * kAtom;
  static constexpr int kK = 0;
  static constexpr int kQ = kK + kTile;               // two buffers
  static constexpr int kLse = kQ + 2 * kTile;         // two buffers of 128 floats
  static constexpr int kBar = kLse + 2 * 128 * 4;
  static constexpr int kBytes = kBar + 256;
};

struct P2Bars {
  uint64_t k_full, k_ready;
  uint64_t q_full[2];
  uint64_t s_full[2];
  uint64_t c_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct P2Params {
  const __nv_bfloat16 *q, *k_prev;
  const uint32_t* seedbits;
  const float* lse;
  const int32_t *mrows, *mcount;
  int L, Hq, Hkv;
  float scale_log2;
  float* din_part;  // [B, Hkv, L]
  uint32_t spin;
};

template <int D>
__global__ void __launch_bounds__(kP2Threads, 1)
attn_p2_kernel(const __grid_constant__ CUtensorMap tmK, const P2Params p) {
  using Lay = P2Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  P2Bars* bars = reinterpret_cast<P2Bars*>(smem + Lay::kBar);
  const uint32_t sbase = smem_u32(smem);
  float* lse2 = reinterpret_cast<float*>(smem + Lay::kLse);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int L = p.L;
  const int G = p.Hq / p.Hkv;
  const int col0 = kt * kBN;
  const int M = p.mcount[b];
  const int nrt = (M + 127) / 128;
  const int NT = G * nrt;
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars->k_full, 1);
    mbar_init(&bars->k_ready, 1);
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bars->q_full[u], 128);
      mbar_init(&bars->s_full[u], 1);
      mbar_init(&bars->c_done[u], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
    // ------------------------------------------------------------------ producers
    const int pt = threadIdx.x;  // 0..127: the masked row this thread gathers
    if (warp == 0) {
      if (lane == 0) {
        mbar_expect_tx(&bars->k_full, Lay::kTile);
#pragma unroll
        for (int ac = 0; ac < D / 64; ++ac)
          tma_load_4d(smem + Lay::kK + ac * kAtom, &tmK, ac * 64, g, col0, b, &bars->k_full);
      }
      const int W = (L + 31) / 32;
      uint32_t seedword = 0;
      if (lane < 4 && kt * 4 + lane < W) seedword = p.seedbits[(int64_t)b * W + kt * 4 + lane];
      if (wait_bounded(&bars->k_full, 0, p.spin, abort_flag)) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t bits = __shfl_sync(0xffffffffu, seedword, w);
          while (bits) {
            const int r = w * 32 + __ffs(bits) - 1;
            bits &= bits - 1;
            if (lane < D / 8) {
              const uint4 val =
                  ldg16(p.k_prev + (((int64_t)b * L + col0 + r) * p.Hkv + g) * D + lane * 8);
              st_shared_v4(sbase + Lay::kK + (lane / 8) * kAtom + sw128(r, lane & 7), val.x,
                           val.y, val.z, val.w);
            }
          }
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->k_ready);
      }
    }
    for (int t = 0; t < NT; ++t) {
      const int u = t & 1;
      if (t >= 2 && !wait_bounded(&bars->c_done[u], ((t >> 1) - 1) & 1, p.spin, abort_flag)) break;
      const int hh = g * G + t / nrt;
      const int m = (t % nrt) * 128 + pt;
      const uint32_t qb = sbase + Lay::kQ + u * Lay::kTile;
      if (m < M) {
        const int pos = p.mrows[(int64_t)b * L + m];
        const __nv_bfloat16* src = p.q + (((int64_t)b * L + pos) * p.Hq + hh) * D;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 val = ldg16(src + c * 8);
          st_shared_v4(qb + (c / 8) * kAtom + sw128(pt, c & 7), val.x, val.y, val.z, val.w);
        }
        lse2[u * 128 + pt] = p.lse[((int64_t)b * p.Hq + hh) * L + pos] * kLog2e;
      } else {
#pragma unroll
        for (int c = 0; c < D / 8; ++c)
          st_shared_v4(qb + (c / 8) * kAtom + sw128(pt, c & 7), 0u, 0u, 0u, 0u);
        lse2[u * 128 + pt] = INFINITY;
      }
      fence_proxy_async();
      mbar_arrive(&bars->q_full[u]);
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(kBM, kBN, false);
      const uint32_t sK = sbase + Lay::kK;
      bool ok = NT == 0 || wait_bounded(&bars->k_ready, 0, p.spin, abort_flag);
      for (int t = 0; ok && t < NT; ++t) {
        const int u = t & 1;
        ok = wait_bounded(&bars->q_full[u], (t >> 1) & 1, p.spin, abort_flag);
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
      ok = wait_bounded(&bars->s_full[u], (t >> 1) & 1, p.spin, abort_flag);
      if (!ok) break;
      fence_after_sync();
      float s[kBN];
#pragma unroll
      for (int q = 0; q < kBN / 32; ++q) {
        float tt[32];
        tmem_ld32(tl + u * 128 + q * 32, tt);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[q * 32 + e] = tt[e];
      }
      tmem_wait_ld();
      const float4* lv = reinterpret_cast<const float4*>(lse2 + u * 128);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int c4 = 0; c4 < kBN / 4; ++c4) {
        const float4 l4 = lv[c4];
        a0 += fast_exp2(fmaf(s[4 * c4 + 0], c2, -l4.x));
        a1 += fast_exp2(fmaf(s[4 * c4 + 1], c2, -l4.y));
        a0 += fast_exp2(fmaf(s[4 * c4 + 2], c2, -l4.z));
        a1 += fast_exp2(fmaf(s[4 * c4 + 3], c2, -l4.w));
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
  if (warp == 4) {
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
bool make_map(CUtensorMap* map, const void* base, int D, int H, int L, int B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)L * H * D * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rows of the step t-1 cache: box = one whole head row (D elements), no swizzle.
bool make_row_map(CUtensorMap* map, const void* base, int D, int H, int L, int B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)L * H * D * 2};
  cuuint32_t box[4] = {(cuuint32_t)D, 1, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_p1(const AttnArgs& a, cudaStream_t stream) {
  CUtensorMap tq, tk, tv, tkp, tvp;
  // without seeds the cache maps are never read; point them at the current K/V
  const void* kp = a.is_seed ? a.k_prev : a.k_cur;
  const void* vp = a.is_seed ? a.v_prev : a.v_cur;
  if (!make_map(&tq, a.q, D, a.Hq, a.L, a.B) || !make_map(&tk, a.k_cur, D, a.Hkv, a.L, a.B) ||
      !make_map(&tv, a.v_cur, D, a.Hkv, a.L, a.B) ||
      !make_row_map(&tkp, kp, D, a.Hkv, a.L, a.B) || !make_row_map(&tvp, vp, D, a.Hkv, a.L, a.B))
    return cudaErrorInvalidValue;
  const int smem = P1Layout<D>::kBytes + 1024;
  static int configured[64] = {};
  const int dev = device_info().device;
  if (!configured[dev & 63]) {
    cudaError_t e = cudaFuncSetAttribute(attn_p1_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[dev & 63] = 1;
  }
  P1Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k_cur = static_cast<const __nv_bfloat16*>(a.k_cur);
  p.v_cur = static_cast<const __nv_bfloat16*>(a.v_cur);
  p.k_prev = static_cast<const __nv_bfloat16*>(a.k_prev);
  p.v_prev = static_cast<const __nv_bfloat16*>(a.v_prev);
  p.is_seed = a.is_seed;
  p.is_new = a.is_new;
  p.seedbits = a.seedbits;
  p.newbits = a.newbits;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.scale_log2 = a.scale * kLog2e;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.dout_part = a.dout_part;
  p.spin = spin_limit();
  dim3 grid((a.L + kBM - 1) / kBM, a.Hq, a.B);
  attn_p1_kernel<D><<<grid, kP1Threads, smem, stream>>>(tq, tk, tv, tkp, tvp, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_p2(const AttnArgs& a, cudaStream_t stream) {
  CUtensorMap tk;
  if (!make_map(&tk, a.k_cur, D, a.Hkv, a.L, a.B)) return cudaErrorInvalidValue;
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
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k_prev = static_cast<const __nv_bfloat16*>(a.k_prev);
  p.seedbits = a.seedbits;
  p.lse = a.lse;
  p.mrows = a.mrows;
  p.mcount = a.mcount;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.scale_log2 = a.scale * kLog2e;
  p.din_part = a.din_part;
  p.spin = spin_limit();
  dim3 grid((a.L + kBN - 1) / kBN, a.Hkv, a.B);
  attn_p2_kernel<D><<<grid, kP2Threads, smem, stream>>>(tk, p);
  return cudaGetLastError();
}

}  // namespace

// Both passes on tensor cores. d_in partials are per kv head ([B, Hkv, L]).
cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t stream, bool* handled,
                                int* din_slices) {
  *handled = true;
  cudaError_t err = a.d == 64 ? launch_p1<64>(a, stream) : launch_p1<128>(a, stream);
  if (err != cudaSuccess) return err;
  if (a.d_in && a.is_masked) {
    err = a.d == 64 ? launch_p2<64>(a, stream) : launch_p2<128>(a, stream);
    *din_slices = a.Hkv;
  }
  return err;
}

}  // namespace dd
