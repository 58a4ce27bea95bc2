"""dd_dualview_attention_ex over a stack of layers with a prefix cache, against the
oracle's layer_stack (GPU).

[COVER] Results: COVER composes with Fast-dLLM-style prefix caching. Each layer
computes the query rows after the cached prefix only, and d_in / d_out are
averaged over the layers (stats_weight = 1 / n_layers, accumulated)."""
import numpy as np
import pytest
import torch

from oracle import attention as OA
from speculative_verification_cover_b200 import dd
from speculative_verification_cover_b200 import workloads as W
from tests import parity as PA

pytestmark = pytest.mark.gpu


def _run_stack(x, layers, q_begin, with_seeds=True):
    spec = x["spec"]
    B, L, Hq, Hkv, d = spec.B, spec.L, spec.Hq, spec.Hkv, spec.d
    n = len(layers)
    ws = torch.empty(dd.dd_dualview_attention_workspace_size(B, L, Hq, Hkv, d),
                     dtype=torch.uint8, device="cuda")
    d_in = torch.full((B, L), 7.0, device="cuda")
    d_out = torch.full((B, L), 7.0, device="cuda")
    outs, lses = [], []
    for li, y in enumerate(layers):
        out = torch.full_like(y["q"], 3.0)  # prefix rows must stay untouched
        lse = torch.full((B, Hq, L), 5.0, device="cuda")
        dd.dd_dualview_attention_ex(
            y["q"], y["k_cur"], y["v_cur"], y["k_prev"] if with_seeds else None,
            y["v_prev"] if with_seeds else None, x["is_seed"] if with_seeds else None,
            x["is_masked"], x["is_new"], out, lse, d_in, d_out, ws, q_begin=q_begin,
            accumulate_stats=li > 0, stats_weight=1.0 / n)
        outs.append(out)
        lses.append(lse)
    torch.cuda.synchronize()
    assert dd.dd_get_device_error() == dd.DD_OK
    return outs, lses, d_in, d_out


def _check(x, layers, outs, lses, d_in, d_out, q_begin, b, heads, tol, with_seeds=True):
    spec = x["spec"]
    f = PA.np64
    seed = PA.npi(x["is_seed"][b]) if with_seeds else np.zeros(spec.L, np.int64)
    lay = [{k: f(y[k][b]) for k in ("q", "k_cur", "v_cur", "k_prev", "v_prev")} for y in layers]
    wo, wl, wdin, wdout = OA.layer_stack(lay, seed, PA.npi(x["is_masked"][b]),
                                         PA.npi(x["is_new"][b]), q_begin=q_begin)
    for li in range(len(layers)):
        PA.assert_close(f"out[{li}]", f(outs[li][b, q_begin:])[:, heads], wo[li][:, heads], 0, tol)
        PA.assert_close(f"lse[{li}]", f(lses[li][b, :, q_begin:])[heads], wl[li][heads],
                        PA.STAT_RTOL, PA.STAT_ATOL)
        assert bool((outs[li][b, :q_begin] == 3.0).all()), "prefix rows of out were written"
        assert bool((lses[li][b, :, :q_begin] == 5.0).all()), "prefix rows of lse were written"
    PA.assert_close("d_in", f(d_in[b]), wdin, PA.MASS_RTOL, PA.MASS_ATOL)
    PA.assert_close("d_out", f(d_out[b]), wdout, PA.MASS_RTOL, PA.MASS_ATOL)
    assert np.all(f(d_out[b])[:q_begin] == 0.0)


@pytest.mark.parametrize("dtype,q_begin,n_layers", [
    ("f32", 0, 1), ("f32", 16, 3), ("f32", 23, 2),
    ("bf16", 0, 1), ("bf16", 100, 3), ("bf16", 128, 2), ("bf16", 250, 2),
])
def test_small_stacks(dtype, q_begin, n_layers):
    base = W.TINY_F32 if dtype == "f32" else W.LLADA8B_L512
    prompt = max(q_begin, 16)
    spec = base.replace(B=2, L=300, prompt=prompt, Hq=4, Hkv=2, d=64 if dtype == "f32" else 128,
                        masked=min(40, (300 - prompt) // 3), new=min(20, (300 - prompt) // 4),
                        k=min(8, (300 - prompt) // 6), V=64, dtype=dtype)
    x = W.make_inputs(spec, "cuda", seed=31 + q_begin)
    layers = [{k: x[k] for k in ("q", "k_cur", "v_cur", "k_prev", "v_prev")}]
    layers += W.layer_operands(spec, "cuda", seed=99, n_layers=n_layers - 1)
    outs, lses, d_in, d_out = _run_stack(x, layers, q_begin)
    tol = 1e-4 if dtype == "f32" else 2e-2
    for b in range(spec.B):
        _check(x, layers, outs, lses, d_in, d_out, q_begin, b, list(range(spec.Hq)), tol)


@pytest.mark.parametrize("spec,n_layers,heads", [
    (W.LLADA8B_L512, 4, [0, 17, 31]),
    (W.SDAR8B_TREE.replace(B=2), 2, [0, 9, 31]),   # prefix of 992: not a tile multiple
], ids=lambda v: v.name if hasattr(v, "name") else str(v))
def test_workload_stacks(spec, n_layers, heads):
    x = W.make_inputs(spec, "cuda", with_logits=False)
    layers = [{k: x[k] for k in ("q", "k_cur", "v_cur", "k_prev", "v_prev")}]
    layers += W.layer_operands(spec, "cuda", seed=5, n_layers=n_layers - 1)
    with_seeds = spec.k > 0
    outs, lses, d_in, d_out = _run_stack(x, layers, spec.prompt, with_seeds)
    _check(x, layers, outs, lses, d_in, d_out, spec.prompt, 0, heads, 2e-2, with_seeds)
    # one layer with the prefix cache equals the same rows of the full call
    q_begin = spec.prompt
    B, L, Hq = spec.B, spec.L, spec.Hq
    ws = torch.empty(dd.dd_dualview_attention_workspace_size(B, L, Hq, spec.Hkv, spec.d),
                     dtype=torch.uint8, device="cuda")
    full = torch.empty_like(x["q"])
    lse = torch.empty(B, Hq, L, device="cuda")
    di, do = torch.empty(B, L, device="cuda"), torch.empty(B, L, device="cuda")
    y = layers[0]
    dd.dd_dualview_attention(y["q"], y["k_cur"], y["v_cur"], y["k_prev"] if with_seeds else None,
                             y["v_prev"] if with_seeds else None,
                             x["is_seed"] if with_seeds else None, x["is_masked"], x["is_new"],
                             full, lse, di, do, ws)
    o1, l1, _, _ = _run_stack(x, layers[:1], q_begin, with_seeds)
    torch.cuda.synchronize()
    assert torch.equal(o1[0][:, q_begin:], full[:, q_begin:])
    assert torch.equal(l1[0][:, :, q_begin:], lse[:, :, q_begin:])


@pytest.mark.parametrize("spec", [W.LLADA8B_L512, W.TINY_F32], ids=lambda s: s.name)
def test_prep_done_event_leaves_the_outputs_unchanged(spec):
    """dd_dualview_attention_ex2 records the caller's event after the mask preparation:
    a stream that waits on it runs beside the rest of the call, and the call's outputs are
    bit-identical to dd_dualview_attention_ex's."""
    x = W.make_inputs(spec, "cuda", with_logits=False)
    B, L, Hq = spec.B, spec.L, spec.Hq
    ws = torch.empty(dd.dd_dualview_attention_workspace_size(B, L, Hq, spec.Hkv, spec.d),
                     dtype=torch.uint8, device="cuda")

    def run(prep_done=None):
        out = torch.empty_like(x["q"])
        lse = torch.empty(B, Hq, L, device="cuda")
        d_in, d_out = torch.empty(B, L, device="cuda"), torch.empty(B, L, device="cuda")
        dd.dd_dualview_attention_ex(x["q"], x["k_cur"], x["v_cur"], x["k_prev"], x["v_prev"],
                                    x["is_seed"], x["is_masked"], x["is_new"], out, lse, d_in,
                                    d_out, ws, prep_done=prep_done)
        return out, lse, d_in, d_out

    ref = run()
    torch.cuda.synchronize()
    ev = torch.cuda.Event()
    ev.record()  # creates the event
    side = torch.cuda.Stream()
    flag = torch.zeros(1, device="cuda")
    got = run(prep_done=ev)
    with torch.cuda.stream(side):
        side.wait_event(ev)
        flag.fill_(1.0)  # runs once the preparation is done
    torch.cuda.synchronize()
    assert dd.dd_get_device_error() == dd.DD_OK
    assert ev.query() and float(flag) == 1.0
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
