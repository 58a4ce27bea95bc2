"""The decode loop's revision diagnostics on hand-built traces (CPU only).

Golden cases in tests/golden/revision_trace.txt (hand-worked, citing the COVER
page's problem statement and results), and an independent per-position scan on
random traces."""
import os

import numpy as np
import pytest

from speculative_verification_cover_b200 import dd
from speculative_verification_cover_b200.decode_loop import Trace, revision_metrics

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "revision_trace.txt")
CODES = {"N": dd.DD_NONE, "K": dd.DD_KEEP, "R": dd.DD_REPLACE, "D": dd.DD_REMASK,
         "C": dd.DD_COMMIT}


def _tok(s):
    return dd.DD_MASK_TOKEN if s == "M" else int(s)


def _trace(steps):
    tr = Trace()
    for before, d, after in steps:
        tr.tokens_before.append(np.array([[before]], np.int32))
        tr.decision.append(np.array([[d]], np.uint8))
        tr.tokens_after.append(np.array([[after]], np.int32))
    return tr


def _cases():
    for line in open(GOLDEN):
        if not line.startswith("case"):
            continue
        parts = line.split()
        k = parts.index("expect")
        steps = [(_tok(a), CODES[b], _tok(c)) for a, b, c in (p.split(":") for p in parts[1:k])]
        yield steps, [int(v) for v in parts[k + 1:]]


@pytest.mark.parametrize("steps,want", list(_cases()))
def test_golden_traces(steps, want):
    m = revision_metrics(_trace(steps))
    assert [m["effective"], m["flip_flops"], m["pending"], m["commits"]] == want
    n = m["effective"] + m["flip_flops"]
    assert m["effective_ratio"] == (m["effective"] / n if n else None)


def _scan(tokens_before, decision, tokens_after):
    """Per position: walk the steps, remembering the token each open revision removed."""
    eff = flip = pend = 0
    T, B, L = decision.shape
    for b in range(B):
        for i in range(L):
            open_rev = []  # tokens revised and not yet followed by a held token
            for t in range(T):
                if decision[t, b, i] in (dd.DD_REPLACE, dd.DD_REMASK) and \
                        tokens_before[t, b, i] != dd.DD_MASK_TOKEN:
                    open_rev.append(tokens_before[t, b, i])
                y = tokens_after[t, b, i]
                if y != dd.DD_MASK_TOKEN and open_rev:
                    for x in open_rev:
                        if x == y:
                            flip += 1
                        else:
                            eff += 1
                    open_rev = []
            pend += len(open_rev)
    return eff, flip, pend


@pytest.mark.parametrize("trial", range(10))
def test_random_traces_match_a_per_position_scan(trial):
    rng = np.random.default_rng(trial)
    T, B, L = 12, 2, 9
    tok = rng.integers(0, 3, (B, L)).astype(np.int32)
    tok[rng.random((B, L)) < 0.5] = -1
    tr = Trace()
    for _ in range(T):
        d = np.zeros((B, L), np.uint8)
        new = tok.copy()
        held = tok >= 0
        r = rng.random((B, L))
        d[held & (r < 0.2)] = dd.DD_REMASK
        new[held & (r < 0.2)] = -1
        rep = held & (r >= 0.2) & (r < 0.35)
        d[rep] = dd.DD_REPLACE
        new[rep] = (tok[rep] + 1 + rng.integers(0, 2, int(rep.sum()))) % 3
        com = ~held & (r < 0.5)
        d[com] = dd.DD_COMMIT
        new[com] = rng.integers(0, 3, int(com.sum()))
        d[held & (r >= 0.35)] = dd.DD_KEEP
        tr.tokens_before.append(tok.copy())
        tr.decision.append(d)
        tr.tokens_after.append(new.copy())
        tok = new
    m = revision_metrics(tr)
    e, f, p = _scan(np.stack(tr.tokens_before), np.stack(tr.decision), np.stack(tr.tokens_after))
    assert (m["effective"], m["flip_flops"], m["pending"]) == (e, f, p)
