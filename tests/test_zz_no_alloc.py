"""dd_verify_logits_static: the vocabulary pass for callers that cannot allocate.

Some callers cannot call cudaMalloc or hand the library a workspace -- code that
runs inside a runtime owning all device memory, latency-critical loops where an
allocation's implicit synchronisation is not acceptable, code that must not run
out of memory mid-step. dd_verify_logits_static serves them: its scratch is a
fixed array inside libdd. Here it is checked against dd_verify_logits with a
caller workspace, on two calls in a row (the array keeps the previous call's
contents), and for its refusal of problems whose scratch would not fit.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

from speculative_verification_cover_b200 import dd
from speculative_verification_cover_b200 import workloads as W
from tests import parity as PA


def _inputs(seed, B, R, V, dtype):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    lt = torch.empty(B, R, V, dtype=dtype, device="cuda")
    lm = torch.empty_like(lt)
    for b in range(B):
        x, y, _ = W.random_logit_rows(R, V, gen, dtype=dtype, device="cuda")
        lt[b], lm[b] = x, y
    return lt, lm


def _same(a: dd.RowStats, b: dd.RowStats):
    for name in ("lse_t", "lse_d", "conf_t", "p_sample_t", "entropy_t", "kl_dt"):
        PA.assert_close(name, PA.np64(getattr(a, name)), PA.np64(getattr(b, name)),
                        PA.STAT_RTOL, 1e-6)
    for name in ("argmax_t", "argmax_d", "sample_t", "sample_d"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


@pytest.mark.gpu
def test_static_scratch_matches_workspace_variant_two_calls_in_a_row():
    cases = [  # (seed, B, R, V, dtype, temperature, pos_offset)
        (11, 3, 40, 32000, torch.bfloat16, 0.0, 5),
        (12, 2, 64, 50257, torch.bfloat16, 1.0, 0),
        (13, 4, 64, 50257, torch.float32, 0.7, 3),     # fp32 logits
        (14, 16, 2000, 64, torch.bfloat16, 1.0, 0),    # scratch just under the 4 MiB array
    ]
    for seed, B, R, V, dtype, T, off in cases:
        need = dd.dd_verify_logits_workspace_size(B, R, V, dtype)
        assert need <= 4 << 20
        if seed == 14:
            assert need > 0.95 * (4 << 20)  # the array is nearly full
        V_pad = (V + 7) // 8 * 8
        lt_full, lm_full = _inputs(seed, B, R, V_pad, dtype)
        lt, lm = lt_full[..., :V], lm_full[..., :V]
        ref = dd.RowStats.empty(B, R)
        dd.dd_verify_logits(lt, lm, ref, pos_offset=off, temperature=T, seed=seed, step=3)
        got = dd.RowStats.empty(B, R)
        dd.dd_verify_logits_static(lt, lm, got, pos_offset=off, temperature=T, seed=seed, step=3)
        torch.cuda.synchronize()
        assert dd.dd_get_device_error() == dd.DD_OK
        _same(got, ref)


def test_static_scratch_refuses_problems_that_do_not_fit():
    # Host-side check: no device memory is touched before the size is accepted.
    lib = dd.lib()
    assert lib.dd_verify_logits_workspace_size(1, 100000, 152064, dd.DD_BF16) > (4 << 20)
    fake = ctypes.c_void_p(0x10000)
    stats = dd._RowStats()
    st = lib.dd_verify_logits_static(fake, fake, dd.DD_BF16, 1, 100000, 152064, 152064, 0, 0.0,
                                     0, 0, ctypes.byref(stats), None)
    assert st == dd.DD_ERR_UNSUPPORTED
    assert lib.dd_verify_logits_static(None, fake, dd.DD_BF16, 1, 4, 64, 64, 0, 0.0, 0, 0,
                                       ctypes.byref(stats), None) == dd.DD_ERR_INVALID_ARG
