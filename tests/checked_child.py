"""Child process of test_gpu_checked.py (not collected by pytest): runs the
bounds-check self-test and full verification steps on the library the binding
loads -- the checked build when the parent sets DD_CHECK_BOUNDS=1, libdd.so
otherwise -- and saves every output to the path given as argv[1]."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from speculative_verification_cover_b200 import dd, workloads as W  # noqa: E402
from speculative_verification_cover_b200.step import VerifyStep  # noqa: E402

# one shape per attention path: CUDA-core (fp32), one-tile and two-tile pass 1,
# argmax and sampled vocabulary passes
SPECS = (W.TINY_F32, W.LLADA8B_L512, W.SDAR8B_TREE.replace(B=2), W.DREAM7B_GQA_L2048.replace(B=2))


def run_steps():
    out = {}
    for spec in SPECS:
        x = W.make_inputs(spec, "cuda")
        st = VerifyStep(spec, x)
        st.choose_initial_seeds()
        st()
        status = dd.dd_get_device_error()
        res = {"status": torch.tensor(status),
               "out": st.out, "lse": st.lse, "d_in": st.d_in, "d_out": st.d_out,
               "next_seeds": st.next_seeds, "next_is_seed": st.next_is_seed, "score": st.score,
               "decision": st.decision, "new_tokens": st.new_tokens, "accepted": st.accepted}
        for f in ("lse_t", "lse_d", "conf_t", "p_sample_t", "entropy_t", "kl_dt", "argmax_t",
                  "argmax_d", "sample_t", "sample_d"):
            res["stats." + f] = getattr(st.stats, f)
        out[spec.name] = {k: v.detach().cpu() for k, v in res.items()}
    return out


def selftest():
    """(n, index, value read, device status) for in-range and out-of-range reads;
    the last in-range read shows the context is still usable."""
    rows = []
    for n, index in ((64, 5), (64, 64), (8, -1), (0, 0), (64, 63)):
        v = dd.dd_selftest_bounds_check(n, index)
        rows.append((n, index, v, dd.dd_get_device_error()))
    return rows


def main(path):
    checked = dd.dd_bounds_checked()
    result = {"checked": checked, "selftest": selftest() if checked else None,
              "steps": run_steps()}
    torch.save(result, path)


if __name__ == "__main__":
    main(sys.argv[1])
