"""The checked build (DD_CHECK_BOUNDS): a failed device index check records
DD_ERR_BOUNDS and skips the access, with no fault; on valid inputs no check fires
and every output is bit-identical to libdd.so. Each library runs in a process of
its own (the binding loads one library per process)."""
import os
import subprocess
import sys

import pytest
import torch

from speculative_verification_cover_b200 import build, dd

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def _child(tmp_path, checked):
    build.build()
    env = dict(os.environ)
    env["DD_CHECK_BOUNDS"] = "1" if checked else "0"
    path = str(tmp_path / ("checked.pt" if checked else "plain.pt"))
    subprocess.run([sys.executable, os.path.join(HERE, "checked_child.py"), path], env=env,
                   check=True, timeout=600)
    return torch.load(path)


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    tmp = tmp_path_factory.mktemp("checked")
    return _child(tmp, True), _child(tmp, False)


def test_children_loaded_the_builds_asked_for(results):
    checked, plain = results
    assert checked["checked"] == 1 and plain["checked"] == 0


def test_out_of_range_read_is_recorded_not_faulted(results):
    rows = {(n, i): (v, s) for n, i, v, s in results[0]["selftest"]}
    assert rows[(64, 5)] == (16, dd.DD_OK)
    for bad in ((64, 64), (8, -1), (0, 0)):
        assert rows[bad] == (-1, dd.DD_ERR_BOUNDS), bad
    # the context stays usable after the recorded errors
    assert rows[(64, 63)] == (190, dd.DD_OK)


def test_no_check_fires_on_valid_steps(results):
    for name, r in results[0]["steps"].items():
        assert int(r["status"]) == dd.DD_OK, name


def test_checked_outputs_bit_identical(results):
    checked, plain = results
    assert checked["steps"].keys() == plain["steps"].keys()
    for name in plain["steps"]:
        a, b = checked["steps"][name], plain["steps"][name]
        for k in b:
            assert torch.equal(a[k], b[k]), (name, k)
