"""dd_dualview_attention against the oracle (GPU)."""
import numpy as np
import pytest
import torch

from speculative_verification_cover_b200 import dd
from speculative_verification_cover_b200 import workloads as W
from tests import parity as PA

pytestmark = pytest.mark.gpu


def _run(x, with_seeds=True, accumulate=False, d_in=None, d_out=None, guard=0):
    q = x["q"]
    B, L, Hq, d = q.shape
    Hkv = x["k_cur"].shape[2]
    out_buf = torch.full((q.numel() + 2 * guard,), 77.0, dtype=q.dtype, device=q.device)
    lse_buf = torch.full((B * Hq * L + 2 * guard,), 77.0, device=q.device)
    out = out_buf[guard:guard + q.numel()].view_as(q)
    lse = lse_buf[guard:guard + B * Hq * L].view(B, Hq, L)
    d_in = torch.zeros(B, L, device=q.device) if d_in is None else d_in
    d_out = torch.zeros(B, L, device=q.device) if d_out is None else d_out
    ws = torch.empty(dd.dd_dualview_attention_workspace_size(B, L, Hq, Hkv, d), dtype=torch.uint8,
                     device=q.device)
    seeds = x["is_seed"] if with_seeds else None
    dd.dd_dualview_attention(q, x["k_cur"], x["v_cur"], x["k_prev"] if with_seeds else None,
                             x["v_prev"] if with_seeds else None, seeds, x["is_masked"],
                             x["is_new"], out, lse, d_in, d_out, ws,
                             accumulate_stats=accumulate)
    torch.cuda.synchronize()
    assert dd.dd_get_device_error() == dd.DD_OK
    if guard:
        for buf in (out_buf, lse_buf):
            assert bool((buf[:guard] == 77.0).all()) and bool((buf[-guard:] == 77.0).all())
    return out, lse, d_in, d_out


def _check_seq(x, res, b, heads=None, out_atol=None):
    out, lse, d_in, d_out = res
    want_out, want_lse, want_din, want_dout = PA.oracle_attention_seq(x, b, heads=heads)
    got_out = PA.np64(out[b])
    got_lse = PA.np64(lse[b])
    if heads is not None:
        got_out, got_lse = got_out[:, heads], got_lse[heads]
    tol = out_atol if out_atol is not None else (1e-4 if x["q"].dtype == torch.float32 else 2e-2)
    PA.assert_close("out", got_out, want_out, 0.0, tol)
    PA.assert_close("lse", got_lse, want_lse, PA.STAT_RTOL, PA.STAT_ATOL)
    PA.assert_close("d_in", PA.np64(d_in[b]), want_din, PA.MASS_RTOL, PA.MASS_ATOL)
    PA.assert_close("d_out", PA.np64(d_out[b]), want_dout, PA.MASS_RTOL, PA.MASS_ATOL)


def _small(B, L, Hq, Hkv, d, dtype, seed, prompt=None, k=None):
    prompt = L // 4 if prompt is None else prompt
    gen = L - prompt
    masked = gen // 3
    unmasked = gen - masked
    spec = W.TINY_F32.replace(B=B, L=L, prompt=prompt, Hq=Hq, Hkv=Hkv, d=d,
                              dtype="f32" if dtype == torch.float32 else "bf16",
                              qkv_std=1.0 if dtype == torch.float32 else 1.0 / np.sqrt(d),
                              masked=masked, new=unmasked // 3,
                              k=min(unmasked, 5) if k is None else k, V=64)
    return W.make_inputs(spec, "cuda", seed=seed, with_logits=False)


CASES = [
    # B, L, Hq, Hkv, d, dtype
    (1, 64, 2, 2, 64, torch.float32),
    (2, 200, 4, 2, 64, torch.float32),
    (1, 130, 2, 1, 128, torch.float32),
    (2, 200, 4, 2, 64, torch.bfloat16),
    (1, 130, 2, 1, 128, torch.bfloat16),
    (3, 257, 8, 8, 128, torch.bfloat16),
    (1, 1, 1, 1, 128, torch.bfloat16),
    (1, 2, 2, 1, 64, torch.float32),
    # many heads per kv head with a ragged L (rows past L in the last query
    # tile of every head), and d = 64 with 16-way grouping
    (2, 333, 80, 8, 128, torch.bfloat16),
    (1, 600, 128, 16, 64, torch.bfloat16),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%d_L%d_H%d_%d_d%d_%s" % (
    *c[:5], str(c[5]).split(".")[-1]))
def test_small_shapes(case):
    B, L, Hq, Hkv, d, dtype = case
    x = _small(B, L, Hq, Hkv, d, dtype, seed=L * 31 + Hq)
    res = _run(x, guard=16)
    for b in range(B):
        _check_seq(x, res, b)


def test_no_seeds_is_plain_attention():
    x = _small(2, 150, 4, 2, 128, torch.bfloat16, seed=3)
    x["is_seed"].zero_()
    out, lse, _, _ = _run(x, with_seeds=False)
    ref = torch.nn.functional.scaled_dot_product_attention(
        x["q"].float().transpose(1, 2), x["k_cur"].float().repeat_interleave(2, 2).transpose(1, 2),
        x["v_cur"].float().repeat_interleave(2, 2).transpose(1, 2)).transpose(1, 2)
    PA.assert_close("out", PA.np64(out), PA.np64(ref), 0.0, 2e-2)
    res = _run(x, with_seeds=True)  # an all-zero seed mask gives the same answer
    PA.assert_close("out", PA.np64(res[0]), PA.np64(out), 0.0, 1e-6)


def test_every_generated_position_a_seed():
    x = _small(1, 96, 2, 2, 64, torch.float32, seed=4)
    x["is_seed"].copy_(x["eligible"])
    res = _run(x)
    _check_seq(x, res, 0)


def test_accumulate_stats_adds():
    x = _small(1, 100, 2, 2, 64, torch.float32, seed=5)
    _, _, d_in1, d_out1 = _run(x)
    d_in = torch.full_like(d_in1, 0.25)
    d_out = torch.full_like(d_out1, 0.5)
    _run(x, accumulate=True, d_in=d_in, d_out=d_out)
    PA.assert_close("d_in acc", PA.np64(d_in), PA.np64(d_in1) + 0.25, 1e-6, 1e-6)
    PA.assert_close("d_out acc", PA.np64(d_out), PA.np64(d_out1) + 0.5, 1e-6, 1e-6)


@pytest.mark.parametrize("spec,seqs,heads", [
    (W.TINY_F32, [0], None),
    (W.LLADA8B_L512, [0], None),
    (W.LLADA8B_B16_L1024, [0, 15], None),
    (W.DREAM7B_GQA_L2048, [0, 7], None),
    (W.SDAR8B_TREE, [0, 9], None),
], ids=lambda s: s.name if hasattr(s, "name") else str(s))
def test_workloads(spec, seqs, heads):
    x = W.make_inputs(spec, "cuda", with_logits=False)
    res = _run(x)
    for b in seqs:
        _check_seq(x, res, b, heads=heads)
    torch.cuda.empty_cache()
