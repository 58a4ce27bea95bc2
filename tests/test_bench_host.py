"""Host-side pieces of bench.py and of the ncu traffic records that need no GPU."""
import json

import numpy as np
import pytest

import bench
from speculative_verification_cover_b200 import profiling
from speculative_verification_cover_b200 import workloads as W


def test_derived_figures_follow_the_algorithmic_work():
    spec = W.LLADA8B_L512
    t = dict(ms=0.1, a_ms=0.04, v_ms=0.05, s_ms=0.01, clocks={})
    d = bench.derived(spec, t, world=1)
    vbytes = 2 * 1 * 384 * 126464 * 2
    assert d["verify"]["algorithmic_bytes"] == vbytes
    assert d["verify"]["achieved_gbs"] == pytest.approx(vbytes / 0.05e-3 / 1e9)
    flop = 4 * 32 * 512 ** 2 * 128 + 2 * 32 * 192 * 512 * 128
    assert d["attention"]["algorithmic_flop"] == flop
    assert d["attention"]["achieved_tflops"] == pytest.approx(flop / 0.04e-3 / 1e12)
    assert d["steps_per_s"] == pytest.approx(10000.0)
    assert d["positions_per_s"] == pytest.approx(10000.0 * 384)
    # weak scaling: N ranks each doing a batch
    assert bench.derived(spec, t, world=4)["steps_per_s"] == pytest.approx(40000.0)


CSV = '''==PROF== Connected to process 1
"ID","Kernel Name","dram__bytes_read.sum","dram__bytes_write.sum","gpu__time_duration.sum"
"","","Mbyte","Kbyte","usecond"
"0","void dd::verify_stream_kernel<bf16, false>(VerifyArgs)","200.5","3,450.0","49.7"
"1","void dd::attn_p1_kernel<128>(...)","12.9","4.0","19.7"
"2","void dd::verify_stream_kernel<bf16, false>(VerifyArgs)","199.5","3,550.0","49.1"
'''


def test_traffic_record_parses_ncu_raw_csv_and_goes_stale(tmp_path):
    raw = tmp_path / "raw.csv"
    raw.write_text(CSV)
    per, n = profiling.dram_bytes_per_launch(str(raw), "verify_stream_kernel")
    assert n == 2
    assert per == pytest.approx((200.5e6 + 3.45e6 + 199.5e6 + 3.55e6) / 2)
    src = tmp_path / "k.cu"
    src.write_text("// kernel v1\nint a = 1;\n")
    out = tmp_path / "traffic.json"
    rec = profiling.record(str(raw), "verify_stream_kernel", "wl", str(src), "ncu ...",
                           out=str(out))
    assert rec["launches"] == 2
    db = json.loads(out.read_text())
    assert "verify_stream_kernel@wl" in db
    # lookup resolves the source relative to the repository root: point it at ours
    db["verify_stream_kernel@wl"]["source"] = str(src)
    out.write_text(json.dumps(db))
    assert profiling.lookup("verify_stream_kernel", "wl", path=str(out)) == pytest.approx(per)
    assert profiling.lookup("verify_stream_kernel", "other", path=str(out)) is None
    # comments and layout are not the kernel: the record still holds
    src.write_text("/* the same kernel,\n   re-commented */ int  a =\n 1; // v1.1\n")
    assert profiling.lookup("verify_stream_kernel", "wl", path=str(out)) == pytest.approx(per)
    src.write_text("// kernel v2\nint a = 2;\n")  # the kernel changed since the capture
    assert profiling.lookup("verify_stream_kernel", "wl", path=str(out)) is None
    with pytest.raises(ValueError):
        profiling.dram_bytes_per_launch(str(raw), "no_such_kernel")


def test_oracle_near_tie_counts_on_a_small_sample():
    spec = W.TINY_F32.replace(temperature=1.0, policy="coupled")
    x = W.make_inputs(spec, "cpu")
    near = bench.oracle_near_ties(x, spec, nrows=16)
    assert near["rows"] == 16
    assert 0 <= near["near_rows"] <= near["rows"]
    assert 0 <= near["near_decisions"] <= near["decisions"] <= near["rows"]
    # the full-step counter of the CPU-baseline leg
    counts = {}
    bench.oracle_step(x, spec, 0, near=counts)
    assert counts["rows"] == spec.R and "seed_boundary_near" in counts
    assert np.isscalar(counts["near_decisions"])


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints one JSON line
    with the contract's keys, on the arm's own config, and exits 0 without a GPU."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", W.TINY_F32.name, "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["unit"] == "steps/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == W.TINY_F32.name
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "steps/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_kernel_count_per_step():
    """gpu_launches counts our kernels: per attention layer the preparation, the two passes
    and the head reduction; then the vocabulary stream and merge, selection, decisions."""
    from speculative_verification_cover_b200 import step
    assert step.KERNELS_PER_STEP == 8
