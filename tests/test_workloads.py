"""The seeded input generator: shapes, counts, determinism (CPU only)."""
import torch

from speculative_verification_cover_b200 import workloads as W


def test_tiny_workload_shapes_and_counts():
    spec = W.TINY_F32
    x = W.make_inputs(spec, "cpu")
    assert x["q"].shape == (1, 64, 2, 64) and x["q"].dtype == torch.float32
    assert x["k_prev"].shape == (1, 64, 2, 64)
    assert x["logits_t"].shape == (1, 48, 1000)
    assert int(x["is_masked"].sum()) == 24
    assert int(x["is_new"].sum()) == 8
    assert int(x["is_seed"].sum()) == 6
    assert int(x["eligible"].sum()) == 24
    # seeds and new positions are unmasked generated positions
    assert int((x["is_seed"] & x["is_masked"]).sum()) == 0
    assert int(x["is_seed"][:, :16].sum()) == 0
    assert bool((x["tokens"][x["is_masked"].bool()] == -1).all())
    assert bool((x["tokens"][~x["is_masked"].bool()] >= 0).all())


def test_deterministic():
    a = W.make_inputs(W.TINY_F32, "cpu")
    b = W.make_inputs(W.TINY_F32, "cpu")
    for key in ("q", "k_prev", "logits_d", "tokens", "is_seed"):
        assert torch.equal(a[key], b[key])


def test_tree_workload_small():
    spec = W.SDAR8B_TREE.replace(L=80, prompt=48, block=32, V=300, Hq=4, Hkv=2, d=64)
    x = W.make_inputs(spec, "cpu")
    new = x["is_new"].sum(1)
    assert bool(((new >= 1) & (new <= 8)).all())
    assert bool((x["is_masked"].sum(1) + new == 32).all())
    # candidates share the context rows
    assert torch.equal(x["k_cur"][0, :48], x["k_cur"][3, :48])
    assert x["logits_t"].shape == (16, 32, 300)
