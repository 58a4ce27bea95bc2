"""dd_verify_logits / dd_coupled_gumbel against the oracle (GPU)."""
import numpy as np
import pytest
import torch

from oracle import philox as OP
from speculative_verification_cover_b200 import dd
from speculative_verification_cover_b200 import workloads as W
from tests import oracle_pool as OP_POOL
from tests import parity as PA

pytestmark = pytest.mark.gpu


def _run(lt, lm, pos_offset, T, seed, step):
    B, R, _ = lt.shape
    stats = dd.RowStats.empty(B, R, lt.device)
    dd.dd_verify_logits(lt, lm, stats, pos_offset=pos_offset, temperature=T, seed=seed, step=step)
    torch.cuda.synchronize()
    return stats


def _padded(B, R, V, dtype, gen):
    """[B, R, V] views of buffers whose rows are padded to a 16-byte multiple."""
    per16 = 16 // torch.tensor([], dtype=dtype).element_size()
    ld = (V + per16 - 1) // per16 * per16
    bt = torch.full((B, R, ld), 55.0, dtype=dtype, device="cuda")  # padding must be ignored
    bm = torch.full((B, R, ld), 55.0, dtype=dtype, device="cuda")
    for b in range(B):
        x, y, _ = W.random_logit_rows(R, V, gen, dtype=dtype, device="cuda")
        bt[b, :, :V], bm[b, :, :V] = x, y
    return bt[..., :V], bm[..., :V]


@pytest.mark.parametrize("V", [1, 3, 8, 1000, 1001, 4099, 126464])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [0.0, 1.0, 0.7])
def test_small_rows(V, dtype, T):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(V * 7 + int(T * 10))
    B, R = 2, 5
    lt, lm = _padded(B, R, V, dtype, gen)
    seed, step, off = 0x1234_5678_9ABC_DEF0, 3, 11
    stats = _run(lt, lm, off, T, seed, step)
    rows = np.arange(B * R)
    want = PA.oracle_verify(lt.contiguous(), lm.contiguous(), rows, R, off, T, seed, step)
    near = PA.compare_verify(stats, want, rows, T)
    # a sample within 1e-4 of a tie would be excluded; these rows have none
    assert near == 0, near


def test_identical_logits_agree_and_zero_kl():
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    x, _, _ = W.random_logit_rows(16, 5000, gen, dtype=torch.bfloat16, device="cuda")
    lt = x[None].contiguous()
    stats = _run(lt, lt.clone(), 0, 1.0, 77, 1)
    assert torch.equal(stats.sample_t, stats.sample_d)
    assert torch.equal(stats.argmax_t, stats.argmax_d)
    assert float(stats.kl_dt.abs().max()) <= 1e-5


def test_constant_rows_closed_form():
    V = 4096
    lt = torch.full((1, 3, V), 2.5, device="cuda")
    stats = _run(lt, lt.clone(), 0, 0.0, 0, 0)
    assert torch.allclose(stats.entropy_t, torch.full_like(stats.entropy_t, float(np.log(V))),
                          rtol=1e-5)
    assert torch.allclose(stats.conf_t, torch.full_like(stats.conf_t, 1 / V), rtol=1e-5)
    assert int(stats.argmax_t.max()) == 0  # all tied: lowest index


def test_no_out_of_bounds_writes():
    gen = torch.Generator(device="cuda")
    gen.manual_seed(9)
    B, R, V = 3, 4, 1003
    lt, lm = _padded(B, R, V, torch.bfloat16, gen)
    guard = 8
    names = [f.name for f in dd.RowStats.__dataclass_fields__.values()]
    big = {}
    for k in names:
        dt = torch.int32 if k.startswith(("argmax", "sample")) else torch.float32
        big[k] = torch.full((B * R + 2 * guard,), -7, dtype=dt, device="cuda")
    stats = dd.RowStats(**{k: v[guard:guard + B * R].view(B, R) for k, v in big.items()})
    dd.dd_verify_logits(lt, lm, stats, pos_offset=2, temperature=0.5, seed=3, step=4)
    torch.cuda.synchronize()
    for k, v in big.items():
        assert bool((v[:guard] == -7).all()) and bool((v[-guard:] == -7).all()), k
    rows = np.arange(B * R)
    want = PA.oracle_verify(lt.contiguous(), lm.contiguous(), rows, R, 2, 0.5, 3, 4)
    PA.compare_verify(stats, want, rows, 0.5)


def test_coupled_gumbel_matches_oracle_noise():
    B, R, V, off, seed, step = 2, 3, 1001, 17, 0xFEDC_BA98_7654_3210, 12
    g = torch.empty(B, R, V, device="cuda")
    dd.dd_coupled_gumbel(g, seed=seed, step=step, pos_offset=off)
    torch.cuda.synchronize()
    gg = PA.np64(g)
    for b in range(B):
        for r in range(R):
            want = OP.gumbel(seed, step, b, off + r, np.arange(V))
            PA.assert_close(f"g[{b},{r}]", gg[b, r], want, 2e-6, 2e-6)


def _host_rows(t):
    """Rows of a device logits tensor as host arrays the oracle pool takes: bf16 as its
    bit patterns (uint16), fp32 as is."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


@pytest.mark.parametrize("spec", W.WORKLOADS, ids=lambda s: s.name)
def test_workloads_every_row(spec):
    """Every row of every workload, against the oracle run row-parallel on the host."""
    x = W.make_inputs(spec, "cuda")
    B, R = spec.B, spec.R
    seed, step = 2024, 1
    stats = _run(x["logits_t"], x["logits_d"], spec.pos_offset, spec.temperature, seed, step)
    lt, lm = x["logits_t"], x["logits_d"]
    kind = "bf16" if lt.dtype == torch.bfloat16 else "f32"
    fetch = lambda b, r0, r1: (_host_rows(lt[b, r0:r1]), _host_rows(lm[b, r0:r1]))
    want = OP_POOL.verify_all_rows(fetch, B, R, kind, spec.temperature, seed, step,
                                   spec.pos_offset)
    rows = np.arange(B * R)
    near = PA.compare_verify(stats, want, rows, spec.temperature)
    # near-ties (a sample within 1e-4 of the runner-up) are excluded and counted
    assert near <= max(1, len(rows) // 1000), f"{near} near-tie rows of {len(rows)}"
    print(f"{spec.name}: {len(rows)} rows compared, {near} near-tie rows excluded")
    del x, stats
    torch.cuda.empty_cache()
