"""One whole verification step through the C ABI against the oracle (GPU):
dual-view attention -> vocabulary verification -> seed selection -> decisions."""
import numpy as np
import pytest
import torch

from speculative_verification_cover_b200 import dd
from speculative_verification_cover_b200 import workloads as W
from tests import parity as PA

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,policy", [(0.0, "cover"), (1.0, "cover"), (0.0, "kl"),
                                      (0.0, "conf"), (1.0, "coupled"), (0.0, "trust")])
def test_tiny_step(T, policy):
    spec = W.TINY_F32.replace(temperature=T, policy=policy)
    x = W.make_inputs(spec, "cpu")
    xg = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    B, L, Hq, Hkv, d, R, off = spec.B, spec.L, spec.Hq, spec.Hkv, spec.d, spec.R, spec.pos_offset
    out = torch.empty_like(xg["q"])
    lse = torch.empty(B, Hq, L, device="cuda")
    d_in = torch.empty(B, L, device="cuda")
    d_out = torch.empty(B, L, device="cuda")
    ws = torch.empty(dd.dd_dualview_attention_workspace_size(B, L, Hq, Hkv, d),
                     dtype=torch.uint8, device="cuda")
    dd.dd_dualview_attention(xg["q"], xg["k_cur"], xg["v_cur"], xg["k_prev"], xg["v_prev"],
                             xg["is_seed"], xg["is_masked"], xg["is_new"], out, lse, d_in, d_out,
                             ws)
    stats = dd.RowStats.empty(B, R)
    dd.dd_verify_logits(xg["logits_t"], xg["logits_d"], stats, pos_offset=off, temperature=T,
                        seed=0, step=0)
    seeds = torch.empty(B, spec.k, dtype=torch.int32, device="cuda")
    next_seed = torch.empty(B, L, dtype=torch.uint8, device="cuda")
    dd.dd_select_seeds(stats.entropy_t, off, d_in, d_out, xg["eligible"], seeds, next_seed)
    dec = torch.empty(B, L, dtype=torch.uint8, device="cuda")
    newt = torch.empty(B, L, dtype=torch.int32, device="cuda")
    acc = torch.empty(B, dtype=torch.uint8, device="cuda")
    dd.dd_decide(policy, xg["tokens"], xg["is_seed"], xg["eligible"], stats, off, dec, newt, acc,
                 tau_kl=spec.tau_kl, tau_conf=spec.tau_conf, temperature=T)
    torch.cuda.synchronize()
    assert dd.dd_get_device_error() == dd.DD_OK

    # oracle, step by step, on the same inputs
    wo, wl, wdin, wdout = PA.oracle_attention_seq(x, 0)
    PA.assert_close("out", PA.np64(out[0]), wo, 0, 1e-4)
    PA.assert_close("d_in", PA.np64(d_in[0]), wdin, PA.MASS_RTOL, PA.MASS_ATOL)
    PA.assert_close("d_out", PA.np64(d_out[0]), wdout, PA.MASS_RTOL, PA.MASS_ATOL)
    rows = np.arange(R)
    ws_ = PA.oracle_verify(x["logits_t"], x["logits_d"], rows, R, off, T, 0, 0)
    near_rows = PA.compare_verify(stats, ws_, rows, T)
    u = np.zeros(L)
    u[off:] = ws_["entropy_t"]
    elig = PA.npi(x["eligible"][0])
    want_seeds, want_is, want_score, _ = PA.oracle_select(u, wdin, wdout, elig, spec.k)
    # The GPU's scores come from the GPU's statistics (entropy, d_in, d_out, each within
    # its tolerance), so its set may differ from the oracle's only by positions whose
    # oracle score lies within that tolerance of the k-th boundary.
    got_is = PA.npi(next_seed[0]).astype(bool)
    fin = np.sort(want_score[np.isfinite(want_score)])[::-1]
    mid = 0.5 * (fin[spec.k - 1] + fin[spec.k])
    band = 4e-3 * (1.0 + abs(mid))
    diff = got_is != want_is.astype(bool)
    assert np.all(np.abs(want_score[diff] - mid) <= band), np.nonzero(diff)
    assert int(diff.sum()) <= 2
    wd, wt, wa, near = PA.oracle_decide(policy, PA.npi(x["tokens"][0]), PA.npi(x["is_seed"][0]),
                                        PA.npi(x["eligible"][0]), ws_, off, R, T, spec.tau_kl,
                                        spec.tau_conf)
    ok = ~near
    assert np.array_equal(PA.npi(dec[0])[ok], wd[ok].astype(np.int64))
    assert np.array_equal(PA.npi(newt[0])[ok], wt[ok].astype(np.int64))
    assert near_rows + int(near.sum()) <= 2


@pytest.mark.parametrize("spec", [W.LLADA8B_L512, W.SDAR8B_TREE], ids=lambda s: s.name)
def test_one_graph_step_matches_the_serial_calls(spec):
    """The step as one CUDA graph, with the vocabulary pass on a side stream beside the
    attention call, gives bit-identical results to the four calls made in order."""
    from speculative_verification_cover_b200.step import VerifyStep
    x = W.make_inputs(spec, "cuda")
    step = VerifyStep(spec, x)
    step.choose_initial_seeds()
    step()  # serial, eager
    torch.cuda.synchronize()
    names = ("lse_t", "lse_d", "conf_t", "entropy_t", "kl_dt", "argmax_t", "sample_t", "sample_d")
    ref = [t.clone() for t in step.result_tensors()] + [getattr(step.stats, n).clone() for n in names]
    ref += [step.out.clone(), step.d_in.clone(), step.d_out.clone()]
    step.capture()
    for t in step.result_tensors():
        t.fill_(0x55)
    step.replay()  # the one-graph step
    torch.cuda.synchronize()
    assert dd.dd_get_device_error() == dd.DD_OK
    got = [t for t in step.result_tensors()] + [getattr(step.stats, n) for n in names]
    got += [step.out, step.d_in, step.d_out]
    for a, b in zip(ref, got):
        assert torch.equal(a, b)


@pytest.mark.parametrize("prefix_cache", [False, True])
def test_multilayer_graph_step_matches_the_serial_calls(prefix_cache):
    """A three-layer step as one CUDA graph (the vocabulary pass starting once the first
    layer's mask preparation is done) gives bit-identical results to the calls made in
    order; with the prefix cache, each layer computes the rows after the prompt only."""
    from speculative_verification_cover_b200.step import VerifyStep
    spec = W.LLADA8B_L512
    x = W.make_inputs(spec, "cuda")
    extra = W.layer_operands(spec, "cuda", seed=11, n_layers=2)
    step = VerifyStep(spec, x, extra_layers=extra, prefix_cache=prefix_cache)
    step.choose_initial_seeds()
    step()  # serial, eager
    torch.cuda.synchronize()
    names = ("lse_t", "entropy_t", "kl_dt", "argmax_t", "sample_t")
    ref = [t.clone() for t in step.result_tensors()] + [getattr(step.stats, n).clone() for n in names]
    ref += [step.d_in.clone(), step.d_out.clone(), step.score.clone()]
    step.capture()
    for t in step.result_tensors():
        t.fill_(0x55)
    step.d_in.fill_(7.0)
    step.replay()
    torch.cuda.synchronize()
    assert dd.dd_get_device_error() == dd.DD_OK
    got = [t for t in step.result_tensors()] + [getattr(step.stats, n) for n in names]
    got += [step.d_in, step.d_out, step.score]
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
    step.graphs = None
