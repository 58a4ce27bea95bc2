/*
 * dd.h -- C ABI of the B200 (sm_100a) verification-step library libdd.so.
 *
 * One verification step of speculative / revocable decoding for masked
 * diffusion language models, as described on three pages:
 *
 *   [COVER] "Stop the Flip-Flop: Context-Preserving Verification for Fast
 *           Revocable Diffusion Decoding" -- Methodology: COVER, sections
 *           1 (Dual-View Feed Forward via KV cache override), 2 (Stability-Aware
 *           Seed Selection, the Score equation), 3 (Adaptive Revision Outcomes).
 *   [DD]    "DualDiffusion: A Speculative Decoding Strategy for Masked Diffusion
 *           Models" -- section 2 Methodology, Verification Algorithms (Trust
 *           Verifier, KL Divergence-based Remasking, Confidence-based Remasking).
 *   [SPOT]  "[Review] On the SPOT: Enhancing Speculative Decoding for Diffusion
 *           Language Models via Commit-Order Prediction" -- section 1 Key Terms
 *           (Coupled-Noise Verification), section 3 Method (one batched
 *           verification of a candidate tree).
 *
 * Conventions (all entry points):
 *   - Tensor pointers are DEVICE memory owned by the caller unless stated.
 *     The library never allocates device memory inside a call; scratch
 *     memory comes from the caller through `workspace`.
 *   - Layouts are row-major and contiguous unless a stride is given:
 *       q [B,L,Hq,d]; k_cur, v_cur, k_prev, v_prev [B,L,Hkv,d];
 *       per-position arrays [B,L]; logits [B,R,V] with row stride ld >= V;
 *       per-row statistics [B,R].
 *     Row r of a logits matrix is sequence position pos_offset + r.
 *   - Every device pointer to a vector-loaded operand (q, k_*, v_*, out,
 *     logits) must be 16-byte aligned; ld * sizeof(element) must be a
 *     multiple of 16.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). They return DD_OK after host-side validation and a
 *     successful launch, DD_ERR_INVALID_ARG / DD_ERR_UNSUPPORTED without
 *     touching the GPU, or DD_ERR_CUDA if a launch failed. Faults found on
 *     the device (a bounded wait that ran out) are recorded in a device
 *     error word read by dd_get_device_error().
 *   - No C++ exception crosses this interface.
 *   - Supported: d in {64, 128}; Hq % Hkv == 0; L >= 1; V >= 1; B >= 1.
 */
#ifndef DD_VERIFY_H_
#define DD_VERIFY_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DD_OK = 0,
  DD_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, short workspace */
  DD_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d = 96) */
  DD_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  DD_ERR_TIMEOUT = 4,       /* device: a bounded wait ran out (see dd_get_device_error) */
  DD_ERR_BOUNDS = 5         /* device, checked builds only: an index check failed and the
                               access was skipped (see dd_bounds_checked) */
} dd_status;

typedef enum { DD_F32 = 0, DD_BF16 = 1 } dd_dtype;

/* Verification policies (see dd_decide). */
typedef enum {
  DD_POLICY_TRUST = 0,    /* [DD] Trust Verifier */
  DD_POLICY_KL = 1,       /* [DD] KL Divergence-based Remasking */
  DD_POLICY_CONF = 2,     /* [DD] Confidence-based Remasking */
  DD_POLICY_COVER = 3,    /* [COVER] section 3, KEEP / REPLACE / REMASK on seeds */
  DD_POLICY_COUPLED = 4,  /* [SPOT] Coupled-Noise Verification */
  DD_POLICY_KL_STOCHASTIC = 5  /* [DD] KL remasking, "or probabilistically high" */
} dd_policy;

/* Decision codes written by dd_decide. */
enum { DD_NONE = 0, DD_KEEP = 1, DD_REPLACE = 2, DD_REMASK = 3, DD_COMMIT = 4 };
#define DD_MASK_TOKEN (-1)

/*
 * dd_dualview_attention -- one layer of COVER's dual-view attention plus the
 * attention-mass statistics of the seed score ([COVER] sections 1 and 2).
 *
 * For query i and column j of sequence b, head h (kv head h / (Hq/Hkv)):
 *   (k~, v~)_ij = (k_prev[j], v_prev[j])  if j is a seed and j != i
 *               = (k_cur[j],  v_cur[j])   otherwise
 * so non-seed queries read seed columns from the step t-1 cache, and a seed
 * query's own column is the one computed from its [MASK] input (diagonal
 * correction, no self-leakage). Attention is bidirectional (no mask):
 *   out_i = sum_j softmax_j(scale * q_i . k~_ij) v~_ij,  lse_i = log sum_j e^{scale q_i.k~_ij}
 * Statistics of the same (row-normalised) attention A, averaged over heads:
 *   d_out_i = (1/Hq) sum_h sum_{j new}    A^h_ij   (drift sensitivity)
 *   d_in_j  = (1/Hq) sum_h sum_{i masked} A^h_ij   (influence on masked positions)
 *
 * q, k_cur, v_cur   [B,L,Hq,d] / [B,L,Hkv,d], dtype (DD_F32 or DD_BF16)
 * k_prev, v_prev    [B,L,Hkv,d] step t-1 cache; may be NULL when is_seed is NULL
 * is_seed           [B,L] u8 (nonzero = seed); NULL = no seeds (plain attention)
 * is_masked         [B,L] u8, still-masked positions; NULL = none (d_in = 0)
 * is_new            [B,L] u8, newly written positions; NULL = none (d_out = 0)
 * softmax_scale     <= 0 selects 1/sqrt(d)
 * accumulate_stats  0: d_in/d_out are overwritten; 1: this layer's values are
 *                   added (the caller averages over layers)
 * out               [B,L,Hq,d] same dtype as q (required)
 * lse               [B,Hq,L] fp32 natural-log LSE (required)
 * d_in, d_out       [B,L] fp32, each may be NULL to skip it
 * workspace         device scratch (required) of at least
 *                   dd_dualview_attention_workspace_size(B,L,Hq,Hkv,d) bytes,
 *                   256-byte aligned; contents on entry are ignored. Calls that
 *                   share a workspace must not overlap on the GPU.
 * Preconditions: is_seed and is_masked are disjoint (seeds are previously
 * unmasked tokens); K/V/Q values are finite.
 * Errors: DD_ERR_INVALID_ARG for null required pointers, non-positive sizes,
 * Hq % Hkv != 0, misalignment or a short workspace; DD_ERR_UNSUPPORTED for
 * d not in {64,128}, or L > 32768 with DD_BF16.
 */
dd_status dd_dualview_attention(
    const void* q, const void* k_cur, const void* v_cur,
    const void* k_prev, const void* v_prev,
    const uint8_t* is_seed, const uint8_t* is_masked, const uint8_t* is_new,
    int B, int L, int Hq, int Hkv, int d, float softmax_scale, dd_dtype dtype,
    int accumulate_stats,
    void* out, float* lse, float* d_in, float* d_out,
    void* workspace, size_t workspace_bytes, void* stream);

/*
 * dd_dualview_attention_ex -- dd_dualview_attention for one layer of a
 * multi-layer verification pass with a prefix cache ([COVER] Results: COVER
 * composes with Fast-dLLM-style prefix caching; section 2's statistics are
 * taken over the whole pass).
 *   q_begin       first query row computed, 0 <= q_begin < L. Rows before it are
 *                 a cached prefix (the prompt): their K/V rows in k_cur / v_cur
 *                 (and k_prev / v_prev) were filled once from the cache and are
 *                 read as keys, but their queries are not computed -- out and lse
 *                 rows before q_begin are not written (q rows there are not read),
 *                 and they contribute 0 to d_out. Seeds and masked positions must
 *                 lie at or after q_begin.
 *   stats_weight  this layer's d_in / d_out are multiplied by it before they are
 *                 written (accumulate_stats = 0) or added (accumulate_stats = 1):
 *                 1 / n_layers on every layer of an n-layer pass, with
 *                 accumulate_stats = 0 on the first and 1 on the rest, leaves the
 *                 layer average. Finite.
 * Every other argument as dd_dualview_attention, which is this call with
 * q_begin = 0 and stats_weight = 1.
 * Errors: as dd_dualview_attention; DD_ERR_INVALID_ARG for q_begin outside
 * [0, L) or a non-finite stats_weight.
 */
dd_status dd_dualview_attention_ex(
    const void* q, const void* k_cur, const void* v_cur,
    const void* k_prev, const void* v_prev,
    const uint8_t* is_seed, const uint8_t* is_masked, const uint8_t* is_new,
    int B, int L, int Hq, int Hkv, int d, float softmax_scale, dd_dtype dtype,
    int q_begin, int accumulate_stats, float stats_weight,
    void* out, float* lse, float* d_in, float* d_out,
    void* workspace, size_t workspace_bytes, void* stream);

/*
 * dd_dualview_attention_ex2 -- dd_dualview_attention_ex that also records
 * `prep_done` (a cudaEvent_t created by the caller; NULL: none) on `stream` right
 * after the call's first kernel, the mask preparation. That kernel lets the first
 * attention pass take its SMs while it runs, so by the time the event completes
 * the pass is resident. A caller that runs a bandwidth-bound kernel beside this
 * call on another stream (the vocabulary pass of the same verification step) makes
 * that stream wait on the event: the other kernel then fills the SMs the pass
 * leaves free instead of taking every SM before the pass can start. The event
 * says nothing about the call's outputs; wait for the call itself before reading
 * them. Every other argument, and the errors, as dd_dualview_attention_ex (plus
 * DD_ERR_CUDA if the event cannot be recorded).
 */
dd_status dd_dualview_attention_ex2(
    const void* q, const void* k_cur, const void* v_cur,
    const void* k_prev, const void* v_prev,
    const uint8_t* is_seed, const uint8_t* is_masked, const uint8_t* is_new,
    int B, int L, int Hq, int Hkv, int d, float softmax_scale, dd_dtype dtype,
    int q_begin, int accumulate_stats, float stats_weight,
    void* out, float* lse, float* d_in, float* d_out,
    void* workspace, size_t workspace_bytes, void* prep_done, void* stream);

/* Bytes of device scratch dd_dualview_attention needs for these sizes
 * (0 on invalid sizes). Pure host function. Dominant terms: a bf16 copy of K
 * and V with the seed rows taken from the cache (2*B*L*Hkv*d*2 bytes) and room
 * for every query row of the second pass (B*L*Hq*d*2 bytes: how many rows are
 * still masked is only known on the device), plus per-head fp32 partials of
 * the statistics (2*B*Hq*L*4 bytes). */
size_t dd_dualview_attention_workspace_size(int B, int L, int Hq, int Hkv, int d);

/* Per-row outputs of dd_verify_logits, each [B*R] (row-major [B,R]).
 * Any pointer may be NULL to skip that output. */
typedef struct {
  float* lse_t;       /* log sum_v e^{l_v}            (verifier) */
  float* lse_d;       /* log sum_v e^{m_v}            (drafter) */
  float* conf_t;      /* max_v p_t(v)                 ([DD] confidence) */
  float* p_sample_t;  /* p_t(sample_t) */
  float* entropy_t;   /* -sum_v p_t log p_t           ([COVER] uncertainty u) */
  float* kl_dt;       /* KL(p_d || p_t)               ([DD] KL remasking) */
  int32_t* argmax_t;  /* lowest index among the maxima of l */
  int32_t* argmax_d;
  int32_t* sample_t;  /* T > 0: argmax_v(l_v/T + g_v); T == 0: argmax_t */
  int32_t* sample_d;  /* T > 0: argmax_v(m_v/T + g_v); T == 0: argmax_d */
} dd_row_stats;

/*
 * dd_verify_logits -- the fused per-position vocabulary verification pass:
 * one streaming read of the verifier logits l and drafter logits m of every
 * verified row, producing dd_row_stats ([DD] section 2; [COVER] section 2's
 * uncertainty u; [SPOT] Coupled-Noise Verification).
 *
 * logits_t, logits_d  [B,R,V] with row stride ld (elements), dtype DD_F32 or DD_BF16
 * pos_offset          row r is sequence position pos_offset + r (Gumbel counter)
 * temperature         0: samples are argmaxes (no noise); > 0: coupled Gumbel-max
 *                     with the SAME noise g_v for drafter and verifier:
 *                       key = (seed lo32, seed hi32),
 *                       counter = (v >> 2, pos_offset + r, b, step lo32),
 *                       word = Philox4x32-10 output word (v & 3),
 *                       U = (2*(word >> 9) + 1) * 2^-24,  g = -ln(-ln U)
 * Statistics (lse, conf, entropy, kl) use the T = 1 distributions.
 * Ties in argmax / samples go to the lowest vocabulary index. Logits must be
 * finite.
 * workspace           device scratch (required) of at least
 *                     dd_verify_logits_workspace_size(B,R,V,dtype) bytes, 256-byte
 *                     aligned; holds per-row partial states; contents on entry are
 *                     ignored. Calls sharing a workspace must not overlap on the GPU.
 * Errors: DD_ERR_INVALID_ARG for null logits/out/workspace, B/R/V < 1, ld < V,
 * temperature < 0, misaligned logits or ld, a short workspace.
 */
dd_status dd_verify_logits(
    const void* logits_t, const void* logits_d, dd_dtype dtype,
    int B, int R, int V, int64_t ld, int pos_offset,
    float temperature, uint64_t seed, uint64_t step,
    const dd_row_stats* out, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device scratch dd_verify_logits needs (0 on invalid sizes). Pure host
 * function; the bound holds on any device. */
size_t dd_verify_logits_workspace_size(int B, int R, int V, dd_dtype dtype);

/*
 * dd_verify_logits_static -- dd_verify_logits for callers that cannot allocate
 * device memory. (The pages have no counterpart: this is a library convenience.)
 *
 * Some callers cannot call cudaMalloc or supply a workspace: code embedded in a
 * runtime that owns and budgets all device memory, latency-critical loops where
 * an allocation's implicit device synchronisation is unacceptable, or code that
 * must not hit out-of-memory mid-step. This entry point allocates nothing: the
 * per-row partial states live in a fixed array of DD_STATIC_SCRATCH_BYTES inside
 * libdd's own device memory, which every GPU that loads the library holds until
 * the process exits. Same arguments, semantics and outputs as dd_verify_logits,
 * without the workspace.
 *   - The first call on a device looks up that array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: after cudaDeviceReset (or
 *     anything else that tears the device's context down) this entry point must
 *     not be called again on that device.
 *   - Every call shares the one array and leaves its contents behind; nothing in
 *     it needs to start at zero. Calls that overlap on the GPU (e.g. on two
 *     streams, or two threads) race on it: serialise them.
 * Errors: as dd_verify_logits; DD_ERR_UNSUPPORTED when the call would need more
 * than DD_STATIC_SCRATCH_BYTES of scratch (dd_verify_logits_workspace_size(...)
 * > DD_STATIC_SCRATCH_BYTES) -- use dd_verify_logits with a workspace then;
 * DD_ERR_CUDA if the array's address cannot be obtained.
 */
#define DD_STATIC_SCRATCH_BYTES (4u << 20)
dd_status dd_verify_logits_static(
    const void* logits_t, const void* logits_d, dd_dtype dtype,
    int B, int R, int V, int64_t ld, int pos_offset,
    float temperature, uint64_t seed, uint64_t step,
    const dd_row_stats* out, void* stream);

/*
 * dd_coupled_gumbel -- write the shared Gumbel noise g[b, r, v] (fp32, row
 * stride ld) that dd_verify_logits uses for row r = position pos_offset + r,
 * so that a drafter can sample with the very same noise ([SPOT] Coupled-Noise
 * Verification). Same counter layout and mapping as dd_verify_logits.
 */
dd_status dd_coupled_gumbel(uint64_t seed, uint64_t step, int B, int R, int V, int64_t ld,
                            int pos_offset, float* g, void* stream);

/*
 * dd_select_seeds -- stability-aware seed selection ([COVER] section 2):
 *   score_i = u_i * (1 + d_in_i) / (1 + d_out_i)
 * on eligible positions that have a verified row (u_i = entropy[b, i - pos_offset]);
 * every other position scores -inf. The k highest scores per sequence are
 * chosen, ties going to the lower position.
 * entropy        [B,R] fp32 (dd_row_stats.entropy_t)
 * d_in, d_out    [B,L] fp32 (dd_dualview_attention)
 * eligible       [B,L] u8 (previously unmasked generated positions)
 * seeds          [B,k] int32 out, in rank order, -1 padded when fewer than k
 * is_seed        [B,L] u8 out (may be NULL)
 * score          [B,L] fp32 out (may be NULL)
 * Errors: DD_ERR_INVALID_ARG for null inputs/seeds, B, L < 1, k < 0,
 * R < 0, k > 1024.
 */
dd_status dd_select_seeds(
    const float* entropy, int R, int pos_offset,
    const float* d_in, const float* d_out, const uint8_t* eligible,
    int B, int L, int k, int32_t* seeds, uint8_t* is_seed, float* score, void* stream);

typedef struct {
  dd_policy policy;
  float tau_kl;       /* KL threshold (REMASK if KL > tau_kl); <= 0 disables it for COUPLED */
  float tau_conf;     /* confidence threshold (CONF: REMASK if conf < tau; COVER: REPLACE if p >= tau) */
  float temperature;  /* > 0: pred = sample_t; 0: pred = argmax_t */
  float tau_commit;   /* > 0: dynamic threshold decoding on masked positions (see dd_decide) */
  int min_commit;     /* 1: commit at least one masked position per sequence (see dd_decide) */
  uint64_t seed;      /* key of the stochastic decisions' draws (KL_STOCHASTIC) */
  uint64_t step;      /* their step counter (low 32 bits used) */
} dd_decide_params;

/*
 * dd_decide -- KEEP / REPLACE / REMASK per position ([COVER] section 3;
 * [DD] section 2; [SPOT] section 1).
 *   TRUST   eligible: KEEP
 *   KL      eligible: REMASK if kl_dt > tau_kl else KEEP
 *   CONF    eligible: REMASK if conf_t < tau_conf else KEEP
 *   COVER   seeds:    pred == token -> KEEP; p_t(pred) >= tau_conf -> REPLACE(pred); else REMASK
 *   COUPLED eligible: sample_d == pred -> KEEP(pred); else tau_kl > 0 and
 *                     kl_dt > tau_kl -> REMASK; else REPLACE(pred)
 *   KL_STOCHASTIC eligible: REMASK if U * tau_kl < kl_dt (fp32), else KEEP: certain
 *                     when kl_dt > tau_kl, else with probability kl_dt / tau_kl. U is
 *                     the uniform of Philox4x32-10 word 0 at counter
 *                     (2^31, position, b, step lo32), key (seed lo32, seed hi32),
 *                     U = (2*(word >> 9) + 1) * 2^-24 (the mapping of the sampling
 *                     noise; counter word 2^31 is never a vocabulary counter).
 * Dynamic threshold decoding ([SPOT] section 3, SPOT-Sets with dynamic threshold
 * decoding), on still-masked positions (token DD_MASK_TOKEN) with a verified row,
 * whatever the policy: with tau_commit > 0, p_sample_t >= tau_commit -> DD_COMMIT
 * with new token pred; with min_commit = 1, a sequence none of whose masked
 * positions passes commits its single most confident one (lowest position on a
 * tie), so every step unmasks something. COMMIT does not enter accepted[b].
 * Only positions with a verified row are decided; others get DD_NONE and keep
 * their token. new_tokens: KEEP keeps the token (COUPLED: the agreed sample),
 * REPLACE writes pred, REMASK writes DD_MASK_TOKEN.
 * tokens [B,L] int32 (DD_MASK_TOKEN for masked); is_seed, eligible [B,L] u8
 * (is_seed only read by COVER, eligible by the others; the unused one may be NULL)
 * stats  dd_row_stats from dd_verify_logits (argmax_t, argmax_d, sample_t,
 *        sample_d, conf_t, p_sample_t, kl_dt as the policy needs)
 * decision [B,L] u8 out; new_tokens [B,L] int32 out;
 * accepted [B] u8 out or NULL: 1 iff every decided position of b is KEEP.
 */
dd_status dd_decide(
    const dd_decide_params* params, const int32_t* tokens,
    const uint8_t* is_seed, const uint8_t* eligible,
    const dd_row_stats* stats, int B, int L, int R, int pos_offset,
    uint8_t* decision, int32_t* new_tokens, uint8_t* accepted, void* stream);

/* Human-readable name of a status. */
/*
 * dd_select_seeds_ex -- dd_select_seeds with an adaptive set size ([COVER]
 * section 2 calls the seed set "small and adaptive"; the page gives no rule).
 * Only positions whose fp32 score reaches min_score compete, so each sequence
 * gets min(k, #{score >= min_score}) seeds; -INFINITY gives dd_select_seeds.
 * count  [B] int32 out (may be NULL): seeds chosen per sequence.
 * Errors: as dd_select_seeds; DD_ERR_INVALID_ARG for a NaN min_score.
 */
dd_status dd_select_seeds_ex(
    const float* entropy, int R, int pos_offset,
    const float* d_in, const float* d_out, const uint8_t* eligible,
    int B, int L, int k, float min_score, int32_t* seeds, uint8_t* is_seed, float* score,
    int32_t* count, void* stream);

const char* dd_status_string(dd_status s);

/* Synchronises `stream`, then returns and clears the device error word
 * (DD_OK if no kernel recorded a fault). DD_ERR_CUDA if the sync failed. */
dd_status dd_get_device_error(void* stream);

/* Iteration limit of every bounded device-side wait (default 1<<26, also
 * settable through the DD_SPIN_LIMIT environment variable at load time).
 * Returns the previous limit. */
uint32_t dd_set_spin_limit(uint32_t limit);

/*
 * dd_selftest_bounded_wait -- failure-detection self-test: launches one CTA
 * that waits on an mbarrier nobody arrives on, bounded by `spin_limit`
 * iterations. The wait gives up, records DD_ERR_TIMEOUT in the device error
 * word and the kernel returns; the context stays usable. Read the result with
 * dd_get_device_error().
 */
dd_status dd_selftest_bounded_wait(uint32_t spin_limit, void* stream);

/*
 * dd_selftest_gumbel_screen -- self-test of the screen dd_verify_logits uses to
 * skip the exact Gumbel noise of entries that cannot be sampled ([SPOT]
 * Coupled-Noise Verification; the screen itself is this library's, the pages
 * have no counterpart). For every noise level k = word >> 9 (2^23 levels) it
 * writes the library's fp32 noise g_of_level[k] = -ln(-ln U) and the screen's
 * exact-float j_of_level[k] = 2^23 - 1 - k; for each of the n requested levels
 * G = g_req[i] it writes limit[i], the screen's bound: a word is screened out at
 * level G iff its j + 1/2 >= limit. The screen is sound iff every level with
 * g_of_level[k] > G has j + 1/2 < limit. *gumbel_max (host pointer, may be NULL)
 * receives the constant above which a required level skips the noise entirely;
 * sound iff no g_of_level exceeds it.
 * g_of_level, j_of_level  device, 2^23 floats each
 * g_req, limit            device, n floats each (may be NULL when n == 0)
 * Errors: DD_ERR_INVALID_ARG for NULL buffers or n < 0.
 */
dd_status dd_selftest_gumbel_screen(float* g_of_level, float* j_of_level, const float* g_req,
                                    float* limit, int n, float* gumbel_max, void* stream);

/*
 * Checked builds. libdd_checked.so is this library compiled with DD_CHECK_BOUNDS
 * defined (the Python binding loads it instead of libdd.so when the environment
 * sets DD_CHECK_BOUNDS=1). In it every index the kernels derive from device data
 * or from a layout invariant -- a masked row's rank, a partial record's slot, a
 * seed's rank, the masked-row count, the rows of pass 2's staged inputs -- is
 * tested before the access. A failed test records DD_ERR_BOUNDS in the device
 * error word (read by dd_get_device_error; the first error recorded wins), the
 * access is skipped, and the kernel runs to its end: no trap, no fault, the
 * context stays usable. Outputs of a call that recorded DD_ERR_BOUNDS are
 * undefined. Results of calls that record nothing are bit-identical to libdd.so.
 *
 * dd_bounds_checked -- 1 in a checked build, 0 otherwise. Pure host function.
 */
int dd_bounds_checked(void);

/*
 * dd_selftest_bounds_check -- self-test of the checked build: one CTA fills a
 * library-owned device array of 64 ints with 3*i + 1 and reads element `index`
 * of its first n through the checked path; *value (host pointer) receives the
 * element, or -1 when the check skipped the read (the device error word then
 * holds DD_ERR_BOUNDS). Synchronises `stream`.
 * Errors: DD_ERR_UNSUPPORTED in a build without the checks (nothing is launched,
 * so no out-of-range read can happen); DD_ERR_INVALID_ARG for value == NULL or n
 * outside [0, 64].
 */
dd_status dd_selftest_bounds_check(int n, int index, int* value, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DD_VERIFY_H_ */
