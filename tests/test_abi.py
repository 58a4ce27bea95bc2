"""The C-ABI library: loads on a machine without a GPU, exports every entry
point include/dd.h declares, and rejects bad arguments on the host before any
device work (CPU only; no compute call is made)."""
import ctypes
import os
import re

import pytest

from speculative_verification_cover_b200 import build, dd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dd.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return dd.lib()


def declared_symbols():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dd_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("dd_dualview_attention", "dd_verify_logits", "dd_select_seeds", "dd_decide"):
        assert name in syms
    assert sorted(dd.EXPORTED) == syms


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert dd.status_string(0) == "DD_OK"
    assert dd.status_string(4) == "DD_ERR_TIMEOUT"
    assert dd.status_string(99) == "DD_UNKNOWN_STATUS"


def test_workspace_size_is_host_only(lib):
    n = dd.dd_dualview_attention_workspace_size(8, 2048, 28, 4, 128)
    assert n >= 2 * 8 * 28 * 2048 * 4 + 8 * 2048 * 4
    assert n % 256 == 0
    assert dd.dd_dualview_attention_workspace_size(0, 2048, 28, 4, 128) == 0


@pytest.mark.parametrize("B,L,Hq,Hkv,d", [(1, 512, 32, 32, 128), (8, 2048, 28, 4, 128),
                                          (2, 333, 80, 8, 128), (1, 1, 1, 1, 64)])
def test_attention_workspace_holds_the_documented_terms(lib, B, L, Hq, Hkv, d):
    # the header's dominant terms: the drafting view of K and V, room for every query
    # row of pass 2, per-head fp32 partials of d_in / d_out; the rest is per-position
    # bookkeeping (row lists, ranks, packed flags, lse of the masked rows) and padding
    n = dd.dd_dualview_attention_workspace_size(B, L, Hq, Hkv, d)
    dominant = 2 * B * L * Hkv * d * 2 + B * L * Hq * d * 2 + 2 * B * Hq * L * 4
    lp = (L + 127) // 128 * 128
    small = B * L * 4 * 2 + B * 4 + B * ((L + 31) // 32) * 4 + B * Hq * lp * 4
    assert dominant <= n <= dominant + small + 16 * 256


P = ctypes.c_void_p
FAKE = P(0x10000)      # never dereferenced: validation fails first
MISALIGNED = P(0x10008)


def _attn(lib, **over):
    args = dict(q=FAKE, kc=FAKE, vc=FAKE, kp=None, vp=None, seed=None, masked=None, new=None,
                B=1, L=8, Hq=2, Hkv=2, d=64, scale=0.0, dtype=1, acc=0, out=FAKE, lse=FAKE,
                din=None, dout=None, ws=None, wsb=0)
    args.update(over)
    a = args
    return lib.dd_dualview_attention(a["q"], a["kc"], a["vc"], a["kp"], a["vp"], a["seed"],
                                     a["masked"], a["new"], a["B"], a["L"], a["Hq"], a["Hkv"],
                                     a["d"], a["scale"], a["dtype"], a["acc"], a["out"], a["lse"],
                                     a["din"], a["dout"], a["ws"], a["wsb"], None)


def test_attention_validation(lib):
    assert _attn(lib, q=None) == dd.DD_ERR_INVALID_ARG
    assert _attn(lib, lse=None) == dd.DD_ERR_INVALID_ARG
    assert _attn(lib, seed=FAKE) == dd.DD_ERR_INVALID_ARG          # seeds without a cache
    assert _attn(lib, Hq=3, Hkv=2) == dd.DD_ERR_INVALID_ARG        # Hq % Hkv
    assert _attn(lib, L=0) == dd.DD_ERR_INVALID_ARG
    assert _attn(lib, d=96) == dd.DD_ERR_UNSUPPORTED
    assert _attn(lib, dtype=7) == dd.DD_ERR_INVALID_ARG
    assert _attn(lib, q=MISALIGNED) == dd.DD_ERR_INVALID_ARG
    assert _attn(lib, scale=float("nan")) == dd.DD_ERR_INVALID_ARG
    # statistics requested without (enough) workspace
    assert _attn(lib, din=FAKE, masked=FAKE) == dd.DD_ERR_INVALID_ARG
    assert _attn(lib, din=FAKE, masked=FAKE, ws=P(0x100000), wsb=16) == dd.DD_ERR_INVALID_ARG
    n = dd.dd_dualview_attention_workspace_size(1, 8, 2, 2, 64)
    assert _attn(lib, dout=FAKE, new=FAKE, ws=P(0x100080), wsb=n) == dd.DD_ERR_INVALID_ARG


def _verify(lib, **over):
    a = dict(lt=FAKE, lm=FAKE, dtype=1, B=1, R=4, V=100, ld=104, off=0, T=0.0)
    a.update(over)
    stats = dd._RowStats()
    ws = a.get("ws", P(0x100000))
    wsb = a.get("wsb", 1 << 20)
    return lib.dd_verify_logits(a["lt"], a["lm"], a["dtype"], a["B"], a["R"], a["V"], a["ld"],
                                a["off"], a["T"], 0, 0, ctypes.byref(stats), ws, wsb, None)


def test_verify_validation(lib):
    assert _verify(lib, lt=None) == dd.DD_ERR_INVALID_ARG
    assert _verify(lib, V=0) == dd.DD_ERR_INVALID_ARG
    assert _verify(lib, ld=99) == dd.DD_ERR_INVALID_ARG             # ld < V
    assert _verify(lib, ld=101) == dd.DD_ERR_INVALID_ARG            # 202 bytes, not 16-aligned
    assert _verify(lib, T=-1.0) == dd.DD_ERR_INVALID_ARG
    assert _verify(lib, T=float("inf")) == dd.DD_ERR_INVALID_ARG
    assert _verify(lib, lm=MISALIGNED) == dd.DD_ERR_INVALID_ARG
    assert _verify(lib, dtype=0, ld=102) == dd.DD_ERR_INVALID_ARG   # fp32: 408 bytes
    assert lib.dd_verify_logits(FAKE, FAKE, 1, 1, 4, 100, 104, 0, 0.0, 0, 0, None, P(0x100000),
                                1 << 20, None) == dd.DD_ERR_INVALID_ARG
    assert _verify(lib, ws=None) == dd.DD_ERR_INVALID_ARG
    assert _verify(lib, wsb=16) == dd.DD_ERR_INVALID_ARG
    assert _verify(lib, ws=P(0x100010)) == dd.DD_ERR_INVALID_ARG    # not 256-aligned
    n = dd.dd_verify_logits_workspace_size(16, 768, 126464, 1)
    assert n > 0 and n % 64 == 0
    assert dd.dd_verify_logits_workspace_size(0, 768, 126464, 1) == 0


def test_select_and_decide_validation(lib):
    assert lib.dd_select_seeds(FAKE, 4, 0, None, FAKE, FAKE, 1, 8, 2, FAKE, None, None,
                               None) == dd.DD_ERR_INVALID_ARG
    assert lib.dd_select_seeds(FAKE, 4, 0, FAKE, FAKE, FAKE, 1, 8, 2000, FAKE, None, None,
                               None) == dd.DD_ERR_UNSUPPORTED
    assert lib.dd_select_seeds(FAKE, 4, 0, FAKE, FAKE, FAKE, 1, 8, 2, None, None, None,
                               None) == dd.DD_ERR_INVALID_ARG
    stats = dd._RowStats()
    params = dd._DecideParams(3, 0.5, 0.9, 0.0)
    # COVER needs is_seed and argmax_t / p_sample_t
    assert lib.dd_decide(ctypes.byref(params), FAKE, None, FAKE, ctypes.byref(stats), 1, 8, 4, 0,
                         FAKE, FAKE, None, None) == dd.DD_ERR_INVALID_ARG
    params = dd._DecideParams(9, 0.5, 0.9, 0.0)
    stats.argmax_t = FAKE
    assert lib.dd_decide(ctypes.byref(params), FAKE, FAKE, FAKE, ctypes.byref(stats), 1, 8, 4, 0,
                         FAKE, FAKE, None, None) == dd.DD_ERR_INVALID_ARG


def test_selftest_rejects_zero_limit(lib):
    assert lib.dd_selftest_bounded_wait(0, None) == dd.DD_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        dd.dd_verify_logits(x, x, dd.RowStats())


def test_attention_ex_validation(lib):
    def ex(q_begin=0, weight=1.0, L=8):
        return lib.dd_dualview_attention_ex(FAKE, FAKE, FAKE, None, None, None, None, None, 1, L,
                                            2, 2, 64, 0.0, 1, q_begin, 0, weight, FAKE, FAKE,
                                            None, None, None, 0, None)
    assert ex(q_begin=-1) == dd.DD_ERR_INVALID_ARG
    assert ex(q_begin=8) == dd.DD_ERR_INVALID_ARG          # q_begin must be < L
    assert ex(weight=float("nan")) == dd.DD_ERR_INVALID_ARG
    assert ex(weight=float("inf")) == dd.DD_ERR_INVALID_ARG
    assert ex(L=0) == dd.DD_ERR_INVALID_ARG
    # the variant with a scheduling event validates the same way, before it records anything
    def ex2(q_begin=0, ws=None):
        return lib.dd_dualview_attention_ex2(FAKE, FAKE, FAKE, None, None, None, None, None, 1, 8,
                                             2, 2, 64, 0.0, 1, q_begin, 0, 1.0, FAKE, FAKE,
                                             None, None, ws, 0, FAKE, None)
    assert ex2(q_begin=8) == dd.DD_ERR_INVALID_ARG
    assert ex2() == dd.DD_ERR_INVALID_ARG                   # no workspace


def test_select_ex_and_decide_extension_validation(lib):
    nan = float("nan")
    assert lib.dd_select_seeds_ex(FAKE, 4, 0, FAKE, FAKE, FAKE, 1, 8, 2, nan, FAKE, None, None,
                                  None, None) == dd.DD_ERR_INVALID_ARG
    stats = dd._RowStats()
    stats.argmax_t = FAKE
    stats.kl_dt = FAKE
    # the stochastic KL rule needs a positive threshold
    p = dd._DecideParams(5, 0.0, 0.9, 0.0, 0.0, 0, 1, 2)
    assert lib.dd_decide(ctypes.byref(p), FAKE, FAKE, FAKE, ctypes.byref(stats), 1, 8, 4, 0,
                         FAKE, FAKE, None, None) == dd.DD_ERR_INVALID_ARG
    # min_commit is 0 or 1; commit needs p_sample_t
    p = dd._DecideParams(0, 0.5, 0.9, 0.0, 0.5, 2, 0, 0)
    assert lib.dd_decide(ctypes.byref(p), FAKE, FAKE, FAKE, ctypes.byref(stats), 1, 8, 4, 0,
                         FAKE, FAKE, None, None) == dd.DD_ERR_INVALID_ARG
    p = dd._DecideParams(0, 0.5, 0.9, 0.0, 0.5, 1, 0, 0)
    assert lib.dd_decide(ctypes.byref(p), FAKE, FAKE, FAKE, ctypes.byref(stats), 1, 8, 4, 0,
                         FAKE, FAKE, None, None) == dd.DD_ERR_INVALID_ARG


def test_checked_build_exports_the_same_boundary(lib):
    checked = ctypes.CDLL(build.OUT_CHECKED)
    for name in declared_symbols():
        assert hasattr(checked, name), name
    checked.dd_bounds_checked.restype = ctypes.c_int
    assert checked.dd_bounds_checked() == 1
    assert dd.dd_bounds_checked() is False


def test_bounds_selftest_refused_without_the_checks(lib):
    # the normal build launches nothing, so no out-of-range read can happen
    v = ctypes.c_int(7)
    assert lib.dd_selftest_bounds_check(64, 100, ctypes.byref(v), None) == dd.DD_ERR_UNSUPPORTED
    assert v.value == 7
    assert lib.dd_selftest_bounds_check(65, 0, ctypes.byref(v), None) == dd.DD_ERR_INVALID_ARG
    assert lib.dd_selftest_bounds_check(64, 0, None, None) == dd.DD_ERR_INVALID_ARG
    assert lib.dd_status_string(dd.DD_ERR_BOUNDS) == b"DD_ERR_BOUNDS"
