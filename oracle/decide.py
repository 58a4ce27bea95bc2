"""Verification decisions per position (oracle).

Test infrastructure only (see the package docstring).

Decision codes: NONE (not decided), KEEP, REPLACE, REMASK, COMMIT.
Policies, each restating one verification rule of the pages:

  TRUST   [DD] section 2, Trust Verifier: accept the drafter's tokens as they are.
  KL      [DD] section 2, KL Divergence-based Remasking: remask a drafted token
          when KL(drafter || verifier) exceeds tau_KL (strictly); the page's
          "or probabilistically high" alternative is KL_STOCHASTIC below.
  CONF    [DD] section 2, Confidence-based Remasking: remask when the
          verifier's max probability is below tau_conf.
  COVER   [COVER] section 3, Adaptive Revision Outcomes, on seed positions:
          re-predicted token equals the current one -> KEEP; differs and the
          verifier is confident (p_t(pred) >= tau_conf) -> REPLACE in place;
          otherwise (uncertain and likely wrong) -> REMASK.
  COUPLED [SPOT] sections 1 and 3, Coupled-Noise Verification: with shared
          Gumbel noise the drafted token is the drafter's coupled sample
          sample_d; the target accepts it iff its own coupled sample agrees
          (KEEP). On a mismatch, our reading: REMASK if a KL threshold is set
          and KL > tau_KL, else REPLACE with the target's sample.

  KL_STOCHASTIC  [DD] section 2, KL Divergence-based Remasking, with its "or
          probabilistically high" clause. Our reading: REMASK when KL > tau_KL, or
          else with probability KL / tau_KL; the draw is U of the shared generator
          (philox.decision_uniform) at the position, decided as U * tau_KL < KL in
          fp32 (which also covers KL > tau_KL, as U < 1).

COMMIT (dynamic threshold decoding, [SPOT] section 3 "SPOT-Sets with dynamic
threshold decoding"): with tau_commit > 0, every still-masked position (token
MASK) with a verified row whose p_t(pred) >= tau_commit is unmasked with pred.
Our reading adds a progress rule (min_commit): if no masked position of a
sequence passes, its single most confident one (lowest position on a tie) is
committed, so that every step unmasks something. COMMIT does not enter
accepted[b] (that flag is about the policy's own domain).

pred is the verifier's coupled sample at T > 0 and its argmax at T = 0.
Only positions with a verified row (pos_offset <= pos < pos_offset + R) are
decided; the domain is the seed set for COVER and the eligible (drafted)
positions otherwise. accepted[b] = every decided position of b is KEEP
(the per-candidate acceptance of a SPOT candidate batch; 1 if none is decided).
new_tokens: KEEP keeps the current token (COUPLED: the agreed sample),
REPLACE writes pred, REMASK writes MASK (-1), NONE leaves the token.
"""
from __future__ import annotations

import numpy as np

from . import philox

NONE, KEEP, REPLACE, REMASK, COMMIT = 0, 1, 2, 3, 4
POLICIES = {"trust": 0, "kl": 1, "conf": 2, "cover": 3, "coupled": 4, "kl_stochastic": 5}
MASK_TOKEN = -1


def decide(policy, tokens, is_seed, eligible, stats, pos_offset, R, temperature,
           tau_kl, tau_conf, tie_eps=1e-4, tau_commit=0.0, min_commit=0, seed=0, step=0, b=0):
    """One sequence (batch index b). stats: per-row dict (vocab.verify_rows of rows 0..R-1).

    Returns decision [L] u8, new_tokens [L] i32, accepted (0/1), near [L] bool
    (positions whose decision rests on a statistic within tie_eps of a
    threshold or of a tie)."""
    tokens = np.asarray(tokens, dtype=np.int64)
    L = tokens.shape[0]
    decision = np.zeros(L, dtype=np.uint8)
    new_tokens = tokens.copy()
    near = np.zeros(L, dtype=bool)
    dom = np.asarray(is_seed if policy == "cover" else eligible).astype(bool).copy()
    rowed = np.zeros(L, dtype=bool)
    rowed[pos_offset:pos_offset + R] = True
    dom &= rowed
    sampled = temperature > 0
    for pos in np.nonzero(dom)[0]:
        r = pos - pos_offset
        kl = stats["kl_dt"][r]
        conf = stats["conf_t"][r]
        pred = int(stats["sample_t"][r] if sampled else stats["argmax_t"][r])
        pred_margin = stats["margin_t"][r] if sampled else np.inf
        if policy == "trust":
            dcs = KEEP
        elif policy == "kl":
            dcs = REMASK if kl > tau_kl else KEEP
            near[pos] = abs(kl - tau_kl) < tie_eps
        elif policy == "conf":
            dcs = REMASK if conf < tau_conf else KEEP
            near[pos] = abs(conf - tau_conf) < tie_eps
        elif policy == "cover":
            near[pos] = pred_margin < tie_eps
            if pred == tokens[pos]:
                dcs = KEEP
            else:
                p = stats["p_sample_t"][r]
                near[pos] |= abs(p - tau_conf) < tie_eps
                dcs = REPLACE if p >= tau_conf else REMASK
        elif policy == "kl_stochastic":
            u = np.float32(philox.decision_uniform(seed, step, b, pos))
            lhs = np.float32(u * np.float32(tau_kl))  # the decision, taken in fp32
            dcs = REMASK if lhs < np.float32(kl) else KEEP
            near[pos] = abs(float(lhs) - kl) < tie_eps
        elif policy == "coupled":
            sd = int(stats["sample_d"][r] if sampled else stats["argmax_d"][r])
            md = stats["margin_d"][r] if sampled else np.inf
            near[pos] = min(pred_margin, md) < tie_eps
            if sd == pred:
                dcs = KEEP
            elif tau_kl > 0 and kl > tau_kl:
                near[pos] |= abs(kl - tau_kl) < tie_eps
                dcs = REMASK
            else:
                near[pos] |= tau_kl > 0 and abs(kl - tau_kl) < tie_eps
                dcs = REPLACE
        else:
            raise ValueError(policy)
        decision[pos] = dcs
        if dcs == REPLACE or (dcs == KEEP and policy == "coupled"):
            new_tokens[pos] = pred
        elif dcs == REMASK:
            new_tokens[pos] = MASK_TOKEN
    accepted = int(all(decision[p] == KEEP for p in np.nonzero(dom)[0]))
    if tau_commit > 0:
        masked = (tokens == MASK_TOKEN) & rowed
        cand = []
        for pos in np.nonzero(masked)[0]:
            r = pos - pos_offset
            pred = int(stats["sample_t"][r] if sampled else stats["argmax_t"][r])
            p = float(stats["p_sample_t"][r])
            cand.append((p, pos, pred))
            near[pos] = abs(p - tau_commit) < tie_eps
            if p >= tau_commit:
                decision[pos] = COMMIT
                new_tokens[pos] = pred
        if min_commit and cand and not any(p >= tau_commit for p, _, _ in cand):
            order = sorted(cand, key=lambda c: (-c[0], c[1]))
            p, pos, pred = order[0]
            decision[pos] = COMMIT
            new_tokens[pos] = pred
            if len(order) > 1 and p - order[1][0] < tie_eps:
                near[pos] = near[order[1][1]] = True
    return decision, new_tokens.astype(np.int32), accepted, near
