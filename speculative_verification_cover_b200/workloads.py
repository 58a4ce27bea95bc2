"""Seeded synthetic workloads for one verification step of a masked diffusion LM.

This module only *draws* inputs: attention operands, the step t-1 K/V cache,
position masks, verifier/drafter logits and the current token assignment,
with the shapes and value distributions of the models the pages evaluate
(LLaDA-8B, Dream-7B, SDAR-8B). It computes no part of the verification step
itself, so both the CUDA path's tests and benchmark and the CPU oracle's
tests take their inputs from here without sharing any of the method's
arithmetic.

The model weights and benchmark datasets the pages use (MMLU, GSM8K,
HumanEval, MBPP, MATH500) are not available; these tensors stand in for one
verification step of those models on those benchmarks.

Layouts (row-major):
  q                [B, L, Hq, d]
  k_cur, v_cur     [B, L, Hkv, d]   K/V computed from the current input (seeds -> [MASK])
  k_prev, v_prev   [B, L, Hkv, d]   step t-1 cache
  is_masked, is_new, eligible, is_seed, is_prompt   [B, L] uint8
  tokens           [B, L] int32, MASK = -1
  logits_t, logits_d  [B, R, V]      row r is sequence position pos_offset + r
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import torch

MASK_TOKEN = -1


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    B: int
    L: int
    prompt: int          # prompt (or fixed context) positions at the start of each sequence
    Hq: int
    Hkv: int
    d: int
    dtype: str           # "f32" or "bf16": storage type of attention operands and logits
    qkv_std: float       # Q/K/V entries ~ N(0, qkv_std)
    drift_std: float     # cache = current + N(0, drift_std)
    masked: int          # still-masked generated positions per sequence
    new: int             # newly written positions per sequence (unmasked by the current draft)
    k: int               # seed-set size per sequence
    V: int
    logit_std: float     # verifier logits ~ N(0, logit_std)
    peak: float          # + peak on one seeded token ...
    peak_rate: float     # ... at this fraction of rows
    drafter_std: float   # drafter = verifier + N(0, drafter_std)
    temperature: float
    tau_kl: float        # <= 0 means "no KL threshold"
    tau_conf: float
    policy: str          # "trust" | "kl" | "conf" | "cover" | "coupled"
    tree: bool = False   # SPOT candidate batch: B candidates of one block
    block: int = 0       # block length for tree workloads
    max_commit: int = 0  # tree: each candidate commits 1..max_commit block positions

    @property
    def gen(self) -> int:
        return self.L - self.prompt

    @property
    def R(self) -> int:
        """Verified rows per sequence: every generated position."""
        return self.L - self.prompt

    @property
    def pos_offset(self) -> int:
        return self.prompt

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def replace(self, **kw) -> "WorkloadSpec":
        return dataclasses.replace(self, **kw)


# The five workloads. Sizes follow the models' published shapes; the masked,
# newly-written and seed counts are the stated fractions rounded down.
TINY_F32 = WorkloadSpec(
    name="tiny_f32_B1_L64_H2_d64_V1000", B=1, L=64, prompt=16, Hq=2, Hkv=2, d=64,
    dtype="f32", qkv_std=1.0, drift_std=0.1, masked=24, new=8, k=6, V=1000,
    logit_std=3.0, peak=8.0, peak_rate=0.7, drafter_std=1.0,
    temperature=0.0, tau_kl=0.5, tau_conf=0.9, policy="cover")

LLADA8B_L512 = WorkloadSpec(
    name="llada8b_B1_L512_H32_d128_V126464", B=1, L=512, prompt=128, Hq=32, Hkv=32,
    d=128, dtype="bf16", qkv_std=1.0 / math.sqrt(128), drift_std=0.05, masked=192,
    new=64, k=16, V=126464, logit_std=3.0, peak=8.0, peak_rate=0.7, drafter_std=1.0,
    temperature=0.0, tau_kl=0.5, tau_conf=0.9, policy="cover")

LLADA8B_B16_L1024 = WorkloadSpec(
    name="llada8b_B16_L1024_H32_d128_V126464", B=16, L=1024, prompt=256, Hq=32, Hkv=32,
    d=128, dtype="bf16", qkv_std=1.0 / math.sqrt(128), drift_std=0.05, masked=230,
    new=179, k=32, V=126464, logit_std=3.0, peak=8.0, peak_rate=0.7, drafter_std=1.0,
    temperature=1.0, tau_kl=0.5, tau_conf=0.9, policy="coupled")

DREAM7B_GQA_L2048 = WorkloadSpec(
    name="dream7b_B8_L2048_H28kv4_d128_V152064", B=8, L=2048, prompt=512, Hq=28, Hkv=4,
    d=128, dtype="bf16", qkv_std=1.0 / math.sqrt(128), drift_std=0.1, masked=614,
    new=307, k=64, V=152064, logit_std=4.0, peak=6.0, peak_rate=0.6, drafter_std=1.5,
    temperature=0.0, tau_kl=0.5, tau_conf=0.9, policy="cover")

SDAR8B_TREE = WorkloadSpec(
    name="sdar8b_tree_B16_L1024_H32kv8_d128_V151936", B=16, L=1024, prompt=992, Hq=32,
    Hkv=8, d=128, dtype="bf16", qkv_std=1.0 / math.sqrt(128), drift_std=0.0, masked=0,
    new=0, k=0, V=151936, logit_std=3.0, peak=8.0, peak_rate=0.7, drafter_std=1.0,
    temperature=0.7, tau_kl=0.5, tau_conf=0.9, policy="coupled", tree=True, block=32,
    max_commit=8)

WORKLOADS = [TINY_F32, LLADA8B_L512, LLADA8B_B16_L1024, DREAM7B_GQA_L2048, SDAR8B_TREE]


def default_seed(spec: WorkloadSpec) -> int:
    return 1000 + [w.name for w in WORKLOADS].index(spec.name) if spec in WORKLOADS else 1000


def _torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _randn(gen, shape, std, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std


def _position_masks(spec: WorkloadSpec, gen, device):
    """Masks per sequence: which generated positions are still masked, which were
    newly written by the current draft, which may be re-verified (seed-eligible),
    and a random seed set of size k among the eligible ones."""
    B, L, P = spec.B, spec.L, spec.prompt
    is_masked = torch.zeros(B, L, dtype=torch.uint8, device=device)
    is_new = torch.zeros_like(is_masked)
    eligible = torch.zeros_like(is_masked)
    is_seed = torch.zeros_like(is_masked)
    is_prompt = torch.zeros_like(is_masked)
    is_prompt[:, :P] = 1
    for b in range(B):
        if spec.tree:
            # One block of `block` positions after the context; this candidate
            # commits 1..max_commit of them, the rest of the block stays masked.
            c = int(torch.randint(1, spec.max_commit + 1, (1,), generator=gen, device=device))
            perm = torch.randperm(spec.block, generator=gen, device=device) + P
            committed, rest = perm[:c], perm[c:]
            is_masked[b, rest] = 1
            is_new[b, committed] = 1
            eligible[b, committed] = 1
            continue
        perm = torch.randperm(spec.gen, generator=gen, device=device) + P
        masked, unmasked = perm[:spec.masked], perm[spec.masked:]
        is_masked[b, masked] = 1
        eligible[b, unmasked] = 1
        sub = torch.randperm(unmasked.numel(), generator=gen, device=device)
        is_new[b, unmasked[sub[:spec.new]]] = 1
        sub2 = torch.randperm(unmasked.numel(), generator=gen, device=device)
        is_seed[b, unmasked[sub2[:spec.k]]] = 1
    return is_masked, is_new, eligible, is_seed, is_prompt


def _attention_operands(spec: WorkloadSpec, gen, device, is_new):
    B, L, Hq, Hkv, d = spec.B, spec.L, spec.Hq, spec.Hkv, spec.d
    dt = _torch_dtype(spec.dtype)
    if spec.tree:
        # Candidates share the context; each candidate's committed block
        # positions get their own rows.
        q = _randn(gen, (1, L, Hq, d), spec.qkv_std, device).expand(B, -1, -1, -1).clone()
        k = _randn(gen, (1, L, Hkv, d), spec.qkv_std, device).expand(B, -1, -1, -1).clone()
        v = _randn(gen, (1, L, Hkv, d), spec.qkv_std, device).expand(B, -1, -1, -1).clone()
        sel = is_new.bool()
        n = int(sel.sum())
        q[sel] = _randn(gen, (n, Hq, d), spec.qkv_std, device)
        k[sel] = _randn(gen, (n, Hkv, d), spec.qkv_std, device)
        v[sel] = _randn(gen, (n, Hkv, d), spec.qkv_std, device)
        kp, vp = k.clone(), v.clone()
    else:
        q = _randn(gen, (B, L, Hq, d), spec.qkv_std, device)
        k = _randn(gen, (B, L, Hkv, d), spec.qkv_std, device)
        v = _randn(gen, (B, L, Hkv, d), spec.qkv_std, device)
        kp = k + _randn(gen, (B, L, Hkv, d), spec.drift_std, device)
        vp = v + _randn(gen, (B, L, Hkv, d), spec.drift_std, device)
    return [x.to(dt).contiguous() for x in (q, k, v, kp, vp)]


def _logits(spec: WorkloadSpec, gen, device, rows=None):
    """Verifier logits N(0, logit_std) with +peak on a seeded token at a
    peak_rate fraction of rows; drafter = verifier + N(0, drafter_std).
    Returns (logits_t, logits_d, peak_token[B,R] (-1 where no peak))."""
    B, R, V = spec.B, spec.R, spec.V
    dt = _torch_dtype(spec.dtype)
    lt = torch.empty(B, R, V, dtype=dt, device=device)
    ld = torch.empty(B, R, V, dtype=dt, device=device)
    has_peak = torch.rand(B, R, generator=gen, device=device) < spec.peak_rate
    peak_tok = torch.randint(0, V, (B, R), generator=gen, device=device)
    peak_tok = torch.where(has_peak, peak_tok, torch.full_like(peak_tok, -1))
    chunk = max(1, (1 << 28) // V)  # rows per chunk, bounds the fp32 temporaries
    flat_t, flat_d = lt.view(B * R, V), ld.view(B * R, V)
    pt = peak_tok.view(-1)
    for r0 in range(0, B * R, chunk):
        r1 = min(B * R, r0 + chunk)
        x = _randn(gen, (r1 - r0, V), spec.logit_std, device)
        rows_with_peak = (pt[r0:r1] >= 0).nonzero().squeeze(1)
        x[rows_with_peak, pt[r0:r1][rows_with_peak]] += spec.peak
        flat_t[r0:r1] = x.to(dt)
        x += _randn(gen, (r1 - r0, V), spec.drafter_std, device)
        flat_d[r0:r1] = x.to(dt)
    return lt, ld, peak_tok


def _tokens(spec: WorkloadSpec, gen, device, is_masked, peak_tok):
    """Current token assignment: the planted peak token at generated positions
    whose row has one (a draft the verifier agrees with), a random token
    elsewhere, MASK at masked positions."""
    B, L, P, V = spec.B, spec.L, spec.prompt, spec.V
    tok = torch.randint(0, V, (B, L), generator=gen, device=device, dtype=torch.int64)
    gen_tok = tok[:, P:]
    gen_tok = torch.where(peak_tok >= 0, peak_tok, gen_tok)
    tok[:, P:] = gen_tok
    tok = torch.where(is_masked.bool(), torch.full_like(tok, MASK_TOKEN), tok)
    return tok.to(torch.int32).contiguous()


def make_inputs(spec: WorkloadSpec, device="cpu", seed: int | None = None,
                with_logits: bool = True) -> dict:
    """Draw one verification step's inputs for `spec` on `device`.

    The same (spec, seed, device type) always gives the same tensors."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(default_seed(spec) if seed is None else seed)
    is_masked, is_new, eligible, is_seed, is_prompt = _position_masks(spec, gen, device)
    q, k, v, kp, vp = _attention_operands(spec, gen, device, is_new)
    out = dict(spec=spec, q=q, k_cur=k, v_cur=v, k_prev=kp, v_prev=vp,
               is_masked=is_masked, is_new=is_new, eligible=eligible, is_seed=is_seed,
               is_prompt=is_prompt)
    if with_logits:
        lt, ld, peak_tok = _logits(spec, gen, device)
        out.update(logits_t=lt, logits_d=ld, peak_token=peak_tok)
        out["tokens"] = _tokens(spec, gen, device, is_masked, peak_tok)
    return out


def random_logit_rows(n: int, V: int, gen: torch.Generator, logit_std=3.0, peak=8.0,
                      peak_rate=0.7, drafter_std=1.0, dtype=torch.float32, device="cpu"):
    """Small batches of logit rows with the workloads' distributions (for tests)."""
    spec = TINY_F32.replace(B=1, L=n, prompt=0, V=V, logit_std=logit_std, peak=peak,
                            peak_rate=peak_rate, drafter_std=drafter_std,
                            dtype={torch.float32: "f32", torch.bfloat16: "bf16"}[dtype])
    lt, ld, pk = _logits(spec, gen, torch.device(device))
    return lt[0], ld[0], pk[0]


def layer_operands(spec: WorkloadSpec, device="cpu", seed: int = 0, n_layers: int = 1) -> list:
    """Attention operands (q, k_cur, v_cur, k_prev, v_prev) of n_layers further layers of
    one verification step, with the distributions of spec (a separate seeded stream per
    call). Sequences share the position masks of make_inputs; only the operands differ
    from layer to layer."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    is_new = torch.zeros(spec.B, spec.L, dtype=torch.uint8, device=device)
    out = []
    for _ in range(n_layers):
        q, k, v, kp, vp = _attention_operands(spec, gen, device, is_new)
        out.append(dict(q=q, k_cur=k, v_cur=v, k_prev=kp, v_prev=vp))
    return out


class DecodeDynamics:
    """Seeded synthetic stand-in for the models of a multi-step decode: it draws, from
    the current token assignment, the attention operands and the verifier / drafter
    logits of the next verification step. It holds none of the method's arithmetic.

    * Every sequence has a hidden target token per generated position.
    * Q / K / V rows are looked up by the position's current token (a table of
      `table` rows, [MASK] its own row) plus a positional row, so a token that
      changes changes its K / V, and the previous step's K / V act as a cache.
    * Verifier logits of a generated position: N(0, logit_std) plus a peak of
      height ln V + 4 + 8 c on the target with probability 0.5 + 0.45 c, else on a
      fixed confusable wrong token, where c is the fraction of the sequence's
      generated positions that currently hold their target (more correct context,
      a more confident and more accurate verifier; the ln V term makes the peak's
      probability independent of the vocabulary size). Drafter = verifier +
      N(0, drafter_std).
    """

    def __init__(self, spec: WorkloadSpec, device="cpu", seed: int = 0, table: int = 4096):
        device = torch.device(device)
        self.spec, self.device, self.table = spec, device, table
        self.gen = torch.Generator(device=device)
        self.gen.manual_seed(seed)
        g, B, L, V = self.gen, spec.B, spec.L, spec.V
        dt = _torch_dtype(spec.dtype)
        self.dtype = dt
        std = spec.qkv_std
        self.Eq = _randn(g, (table + 1, spec.Hq, spec.d), std, device)
        self.Ek = _randn(g, (table + 1, spec.Hkv, spec.d), std, device)
        self.Ev = _randn(g, (table + 1, spec.Hkv, spec.d), std, device)
        self.Pq = _randn(g, (L, spec.Hq, spec.d), std, device)
        self.Pk = _randn(g, (L, spec.Hkv, spec.d), std, device)
        self.Pv = _randn(g, (L, spec.Hkv, spec.d), std, device)
        self.target = torch.randint(0, V, (B, L), generator=g, device=device)
        self.wrong = (self.target + 1 + torch.randint(0, V - 1, (B, L), generator=g,
                                                      device=device)) % V
        prompt_tok = torch.randint(0, V, (B, spec.prompt), generator=g, device=device)
        self.initial = torch.full((B, L), MASK_TOKEN, dtype=torch.int32, device=device)
        self.initial[:, :spec.prompt] = prompt_tok.to(torch.int32)
        self.target[:, :spec.prompt] = prompt_tok

    def _rows(self, tokens):
        return torch.where(tokens < 0, torch.full_like(tokens, self.table),
                           tokens.long() % self.table)

    def operands(self, tokens, masked_view=None):
        """q, k, v [B, L, H, d] for `tokens`; positions in masked_view (u8 [B, L], or None)
        are looked up as [MASK] (the verification view of seeds)."""
        rows = self._rows(tokens)
        if masked_view is not None:
            rows = torch.where(masked_view.bool(), torch.full_like(rows, self.table), rows)
        q = self.Eq[rows] + self.Pq
        k = self.Ek[rows] + self.Pk
        v = self.Ev[rows] + self.Pv
        return [x.to(self.dtype).contiguous() for x in (q, k, v)]

    def logits(self, tokens):
        """Verifier and drafter logits [B, R, V] of the generated rows for `tokens`."""
        s, g, dev = self.spec, self.gen, self.device
        B, R, V, P = s.B, s.R, s.V, s.prompt
        correct = (tokens[:, P:].long() == self.target[:, P:]).float().mean(dim=1)  # [B]
        c = correct[:, None]
        right = torch.rand(B, R, generator=g, device=dev) < (0.5 + 0.45 * c)
        peak_tok = torch.where(right, self.target[:, P:], self.wrong[:, P:])
        x = _randn(g, (B, R, V), s.logit_std, dev)
        height = math.log(V) + 4.0 + 8.0 * c
        x.scatter_add_(2, peak_tok[..., None], height.expand(B, R)[..., None])
        lt = x.to(self.dtype)
        x += _randn(g, (B, R, V), s.drafter_std, dev)
        return lt, x.to(self.dtype)
