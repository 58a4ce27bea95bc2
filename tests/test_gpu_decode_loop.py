"""The multi-step decode loop (GPU): every step of a short decode against the oracle,
along the GPU's own trajectory, and the revision diagnostics over the whole run.

[COVER] problem statement and results: flip-flops (a revised token restored) and
the share of effective revisions are measured over a decode. Each step here feeds
the oracle the very inputs the library received (tokens, seeds, cache, logits),
so a near-tie at one step cannot make the comparison drift at the next."""
import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import decide as OD
from oracle import seeds as OS
from oracle import vocab as OV
from speculative_verification_cover_b200 import dd
from speculative_verification_cover_b200 import workloads as W
from speculative_verification_cover_b200.decode_loop import (DecodeLoop, LoopConfig, Trace,
                                                             revision_metrics)
from tests import parity as PA

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("policy,T", [("cover", 0.0), ("cover", 1.0), ("conf", 0.0)])
def test_loop_steps_match_the_oracle(policy, T):
    spec = W.TINY_F32.replace(B=2)
    dyn = W.DecodeDynamics(spec, "cuda", seed=17)
    cfg = LoopConfig(policy=policy, use_seeds=policy == "cover", k=6, temperature=T,
                     tau_commit=0.9, min_commit=1, tau_conf=0.6)
    loop = DecodeLoop(spec, dyn, cfg)
    trace = Trace()
    near_total = 0
    for t in range(8):
        x = loop.inputs()
        tokens = PA.npi(loop.tokens)
        loop.step(x, trace)
        for b in range(spec.B):
            f = lambda key: PA.np64(x[key][b])
            seeds = PA.npi(x["is_seed"][b]) if x["is_seed"] is not None else np.zeros(spec.L)
            masked = PA.npi(x["is_masked"][b]).astype(bool)
            new = PA.npi(x["is_new"][b])
            assert not np.any(seeds.astype(bool) & masked)
            out, lse, A = OA.dualview_attention(f("q"), f("k_cur"), f("v_cur"), f("k_prev"),
                                                f("v_prev"), seeds)
            PA.assert_close("out", PA.np64(loop.out[b]), out, 0, 1e-4)
            PA.assert_close("d_in", PA.np64(loop.d_in[b]), OA.d_in(A[:, masked, :], spec.Hq),
                            PA.MASS_RTOL, PA.MASS_ATOL)
            PA.assert_close("d_out", PA.np64(loop.d_out[b]), OA.d_out(A, new, spec.Hq),
                            PA.MASS_RTOL, PA.MASS_ATOL)
            rows = np.arange(spec.R)
            st = OV.verify_rows(f("logits_t"), f("logits_d"), T, cfg.seed, t, b,
                                rows + spec.pos_offset)
            near_total += PA.compare_verify(
                dd.RowStats(**{k: getattr(loop.stats, k)[b:b + 1] for k in
                               dd.RowStats.__dataclass_fields__}), st, rows, T)
            # the decisions in the kernel's precision, on the kernel's statistics
            gst = {k: PA.np64(getattr(loop.stats, k)[b]) if getattr(loop.stats, k).dtype ==
                   torch.float32 else PA.npi(getattr(loop.stats, k)[b])
                   for k in dd.RowStats.__dataclass_fields__}
            gst["margin_t"] = gst["margin_d"] = np.full(spec.R, np.inf)
            elig = PA.npi(x["eligible"][b])
            f32 = lambda v: float(np.float32(v))
            dom = seeds if cfg.use_seeds else elig
            wd, wt, _, _ = OD.decide(policy, tokens[b], dom, elig, gst, spec.pos_offset, spec.R,
                                     T, f32(cfg.tau_kl), f32(cfg.tau_conf), PA.TIE_EPS,
                                     f32(cfg.tau_commit), cfg.min_commit, cfg.seed, t, b)
            assert np.array_equal(trace.decision[-1][b], wd), (t, b)
            assert np.array_equal(trace.tokens_after[-1][b], wt), (t, b)
            # next seeds: the oracle's choice on the kernel's fp32 scores
            s32 = PA.np64(loop.score[b])
            ks, kis = OS.select(np.where(PA.npi(x["eligible"][b]).astype(bool), s32, -np.inf),
                                cfg.k)
            assert np.array_equal(PA.npi(loop.next_seeds[b]), ks), (t, b)
    assert near_total <= 2
    m = revision_metrics(trace)
    assert m["steps"] == 8 and m["commits"] > 0
    assert m["revisions"] == m["effective"] + m["flip_flops"] + m["pending"]
    assert dd.dd_get_device_error() == dd.DD_OK


def test_loop_decodes_to_completion():
    spec = W.LLADA8B_L512.replace(B=2, L=256, prompt=64, Hq=8, Hkv=8, V=8192)
    dyn = W.DecodeDynamics(spec, "cuda", seed=5)
    loop = DecodeLoop(spec, dyn, LoopConfig(k=8))
    trace = loop.run(200)
    assert loop.done()
    m = revision_metrics(trace)
    assert m["commits"] >= spec.B * spec.R  # every generated position committed at least once
    acc = float((loop.tokens[:, spec.prompt:].long() == dyn.target[:, spec.prompt:]).float().mean())
    assert acc > 0.5, acc
