"""Row-parallel runs of the vocabulary oracle, for parity over every row of the
large workloads (test infrastructure; imports numpy and the oracle only, so
worker processes start quickly).

Workers are started with the "spawn" method: a process forked after the parent
has initialised CUDA can hang.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

from oracle import vocab as OV


def _widen(bits, kind):
    """Exact fp64 values of bf16 bit patterns (uint16) or fp32 values."""
    if kind == "bf16":
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return bits.astype(np.float64)


def _verify_chunk(job):
    lt, lm, kind, T, seed, step, b, positions = job
    return OV.verify_rows(_widen(lt, kind), _widen(lm, kind), T, seed, step, b, positions)


def workers():
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, 16))


def verify_all_rows(fetch, B, R, kind, T, seed, step, pos_offset, chunk=128):
    """Oracle statistics of every row of [B, R] logits.

    fetch(b, r0, r1) -> (l, m): host arrays of rows r0..r1 of sequence b (uint16 bf16
    bits or float32). Rows are handed to a spawn pool a few chunks at a time, so host
    memory stays bounded whatever the workload. Returns a dict of [B * R] arrays."""
    jobs = [(b, r0, min(R, r0 + chunk)) for b in range(B) for r0 in range(0, R, chunk)]
    out = {}
    ctx = mp.get_context("spawn")
    nw = workers()
    with ctx.Pool(nw) as pool:
        pending = []

        def drain(limit):
            while len(pending) > limit:
                (b, r0, r1), res = pending.pop(0)
                o = res.get()
                sl = slice(b * R + r0, b * R + r1)
                for key, val in o.items():
                    out.setdefault(key, np.zeros(B * R, dtype=val.dtype))[sl] = val

        for b, r0, r1 in jobs:
            l, m = fetch(b, r0, r1)
            pos = pos_offset + np.arange(r0, r1)
            pending.append(((b, r0, r1), pool.apply_async(
                _verify_chunk, ((l, m, kind, T, seed, step, b, pos),))))
            drain(2 * nw)
        drain(0)
    return out
