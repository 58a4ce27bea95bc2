"""Host-side arithmetic of bench.py that needs no GPU."""
import bench


def test_projection_composes_phases_per_layer():
    p = bench.projection("llada8b_B1_L512_H32_d128_V126464", 0.04, 0.06, 0.015)
    assert p["layers"] == 32
    assert abs(p["ms_per_step"] - (32 * 0.04 + 0.06 + 0.015)) < 1e-12
    assert abs(p["steps_per_s"] * p["ms_per_step"] - 1000.0) < 1e-9
    assert "projection" in p["note"]
    assert bench.projection("dream7b_B8_L2048_H28kv4_d128_V152064", 1, 0, 0)["layers"] == 28
    assert bench.projection("sdar8b_tree_B16_L1024_H32kv8_d128_V151936", 1, 0, 0)["layers"] == 36
    assert bench.projection("tiny_f32_B1_L64_H2_d64_V1000", 1, 1, 1) is None
