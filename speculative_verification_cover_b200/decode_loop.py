"""A multi-step decode loop over the verification step, with the revision diagnostics
of the COVER page (problem statement: revocable decoders flip-flop -- a remasked
token comes back unchanged; results: the share of revisions that change the token).

Each step t runs the library's four calls on synthetic inputs drawn by a
workloads.DecodeDynamics from the current tokens:
  * attention: the seeds chosen at step t-1 are [MASK] in the verification view
    (their K / V rows are looked up as [MASK]); the drafting view reads their
    columns from the cache, which is the previous step's K / V (tokens unmasked);
  * the vocabulary pass, seed selection for step t+1, and the decisions: the
    policy on its domain plus dynamic threshold commits of masked positions;
  * tokens(t+1) = new_tokens(t) -- the decisions' own output.
The trace (tokens before, decisions, tokens after) feeds revision_metrics.

The loop is host orchestration of library calls; the dynamics are a workload
stand-in for the drafter and verifier models, not part of the method.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

from . import dd
from .workloads import DecodeDynamics, WorkloadSpec

REVISIONS = (dd.DD_REPLACE, dd.DD_REMASK)


@dataclass
class LoopConfig:
    policy: str = "cover"        # the revision policy ("cover" on seeds, or "conf", "kl", ...)
    use_seeds: bool = True       # dual view with stability-selected seeds (COVER) or none
    k: int = 16                  # seed-set size (its cap, with min_score)
    min_score: float = float("-inf")
    tau_kl: float = 0.5
    tau_conf: float = 0.9
    tau_commit: float = 0.9
    min_commit: int = 1
    temperature: float = 0.0
    seed: int = 2024


@dataclass
class Trace:
    tokens_before: list = field(default_factory=list)  # [B, L] int32 per step
    decision: list = field(default_factory=list)       # [B, L] u8 per step
    tokens_after: list = field(default_factory=list)
    is_seed: list = field(default_factory=list)
    lib_ms: list = field(default_factory=list)         # device time of the four calls


class DecodeLoop:
    def __init__(self, spec: WorkloadSpec, dyn: DecodeDynamics, cfg: LoopConfig):
        self.spec, self.dyn, self.cfg = spec, dyn, cfg
        dev = dyn.device
        B, L, Hq, Hkv, d, R = spec.B, spec.L, spec.Hq, spec.Hkv, spec.d, spec.R
        self.tokens = dyn.initial.clone()
        self.is_seed = torch.zeros(B, L, dtype=torch.uint8, device=dev)
        self.cache = None  # previous step's (k, v)
        self.out = torch.empty(B, L, Hq, d, dtype=dyn.dtype, device=dev)
        self.lse = torch.empty(B, Hq, L, device=dev)
        self.d_in = torch.empty(B, L, device=dev)
        self.d_out = torch.empty(B, L, device=dev)
        self.ws = torch.empty(dd.dd_dualview_attention_workspace_size(B, L, Hq, Hkv, d),
                              dtype=torch.uint8, device=dev)
        self.stats = dd.RowStats.empty(B, R, dev)
        self.k = max(cfg.k, 1)
        self.next_seeds = torch.empty(B, self.k, dtype=torch.int32, device=dev)
        self.next_is_seed = torch.empty(B, L, dtype=torch.uint8, device=dev)
        self.score = torch.empty(B, L, device=dev)
        self.count = torch.empty(B, dtype=torch.int32, device=dev)
        self.decision = torch.empty(B, L, dtype=torch.uint8, device=dev)
        self.new_tokens = torch.empty(B, L, dtype=torch.int32, device=dev)
        self.accepted = torch.empty(B, dtype=torch.uint8, device=dev)
        self.prev_new = torch.zeros(B, L, dtype=torch.uint8, device=dev)
        self.t = 0

    def inputs(self):
        """Everything step t reads, drawn from the current state (the model stand-in)."""
        s, dyn, cfg = self.spec, self.dyn, self.cfg
        seeds = self.is_seed.clone() if cfg.use_seeds else None  # the step rewrites is_seed
        q, k, v = dyn.operands(self.tokens, masked_view=seeds)
        _, k_full, v_full = dyn.operands(self.tokens)
        kp, vp = self.cache if self.cache is not None else (k_full, v_full)
        lt, lm = dyn.logits(self.tokens)
        is_masked = (self.tokens < 0).to(torch.uint8)
        gen = torch.zeros_like(is_masked)
        gen[:, s.prompt:] = 1
        eligible = (1 - is_masked) * gen
        return dict(q=q, k_cur=k, v_cur=v, k_prev=kp, v_prev=vp, k_full=k_full, v_full=v_full,
                    logits_t=lt, logits_d=lm, is_masked=is_masked, eligible=eligible,
                    is_new=self.prev_new, is_seed=seeds)

    def step(self, x=None, trace: Trace | None = None):
        """One decode step; returns the inputs it used (for checking)."""
        s, cfg = self.spec, self.cfg
        x = self.inputs() if x is None else x
        seeds = x["is_seed"]
        before = self.tokens.clone()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        dd.dd_dualview_attention(x["q"], x["k_cur"], x["v_cur"],
                                 x["k_prev"] if seeds is not None else None,
                                 x["v_prev"] if seeds is not None else None, seeds,
                                 x["is_masked"], x["is_new"], self.out, self.lse, self.d_in,
                                 self.d_out, self.ws)
        dd.dd_verify_logits(x["logits_t"], x["logits_d"], self.stats, pos_offset=s.prompt,
                            temperature=cfg.temperature, seed=cfg.seed, step=self.t)
        dd.dd_select_seeds_ex(self.stats.entropy_t, s.prompt, self.d_in, self.d_out,
                              x["eligible"], self.next_seeds, self.next_is_seed, self.score,
                              self.count, min_score=cfg.min_score)
        dom_seed = seeds if seeds is not None else x["eligible"]
        dd.dd_decide(cfg.policy, self.tokens, dom_seed, x["eligible"], self.stats, s.prompt,
                     self.decision, self.new_tokens, self.accepted, tau_kl=cfg.tau_kl,
                     tau_conf=cfg.tau_conf, temperature=cfg.temperature,
                     tau_commit=cfg.tau_commit, min_commit=cfg.min_commit, seed=cfg.seed,
                     step=self.t)
        ev[1].record()
        # the state of step t+1
        self.cache = (x["k_full"], x["v_full"])
        self.prev_new = (self.decision == dd.DD_COMMIT).to(torch.uint8) | \
                        (self.decision == dd.DD_REPLACE).to(torch.uint8)
        self.tokens.copy_(self.new_tokens)
        if cfg.use_seeds:
            # a position chosen as a seed but remasked by this step's decisions is masked
            # now, and seeds are previously unmasked tokens: it drops out of the set
            self.is_seed.copy_(self.next_is_seed * (self.tokens >= 0).to(torch.uint8))
        if trace is not None:
            torch.cuda.synchronize()
            trace.tokens_before.append(before.cpu().numpy())
            trace.decision.append(self.decision.cpu().numpy())
            trace.tokens_after.append(self.tokens.cpu().numpy())
            trace.is_seed.append(seeds.cpu().numpy() if seeds is not None else None)
            trace.lib_ms.append(ev[0].elapsed_time(ev[1]))
        self.t += 1
        return x

    def done(self):
        return bool((self.tokens[:, self.spec.prompt:] >= 0).all())

    def run(self, max_steps: int) -> Trace:
        """Steps until every generated position holds a token (a REMASK leaves its
        position masked, so no revision is left pending then) or max_steps."""
        trace = Trace()
        while self.t < max_steps and not self.done():
            self.step(trace=trace)
        return trace


def revision_metrics(trace: Trace, mask_token: int = dd.DD_MASK_TOKEN) -> dict:
    """Revisions and their outcome over a decode trace.

    A revision is a REPLACE or REMASK decision on a position holding a token x. It is
    effective if the next token the position holds afterwards (the first non-MASK
    token at the end of a step from that step on) differs from x, and a flip-flop if
    it is x again; if the position is still masked at the end of the trace the
    revision is pending. effective_ratio = effective / (effective + flip-flops)."""
    before = np.stack(trace.tokens_before)   # [T, B, L]
    dec = np.stack(trace.decision)
    after = np.stack(trace.tokens_after)
    T = before.shape[0]
    eff = flip = pend = 0
    for t, b, i in zip(*np.nonzero(np.isin(dec, REVISIONS) & (before != mask_token))):
        x = before[t, b, i]
        later = after[t:, b, i]
        held = later[later != mask_token]
        if held.size == 0:
            pend += 1
        elif held[0] == x:
            flip += 1
        else:
            eff += 1
    n = eff + flip
    return {"steps": int(T), "revisions": int(eff + flip + pend), "effective": int(eff),
            "flip_flops": int(flip), "pending": int(pend),
            "effective_ratio": (eff / n) if n else None,
            "commits": int((dec == dd.DD_COMMIT).sum())}
