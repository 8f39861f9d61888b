"""Shared helpers for the tests: seeded workloads with the per-row gap rule.

Exact index parity needs a clear K-th/(K+1)-th score gap.  Per (token, group)
row whose oracle gap is below ``GAP_MIN``, the row's selection query is
redrawn from the next attempt's counter-based stream (at most 64 attempts).
Rows with no more than K eligible chunks need no check.  The gap itself is the
oracle's number: no method arithmetic lives here or in the generator.
"""
from __future__ import annotations

import functools

import numpy as np

import oracle
from chunked_hierarchical_sparse_b200 import synth

GAP_MIN = 1e-3
MAX_ATTEMPTS = 64


def gap_ruled(wl: synth.Workload):
    """Draw ``wl``'s inputs and apply the gap rule.

    Returns (inputs dict, kbar fp32, selection) where selection is the oracle's
    (idx, w, s, gap) over all rows (fwd/train) or (o, idx, w, gap) (decode).
    """
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    if wl.kind == "decode":
        for attempt in range(1, MAX_ATTEMPTS + 2):
            res = oracle.decode(x["q"], x["q_slc"], x["k"], x["v"], kbar, wl.S, wl.K)
            bad = np.argwhere(res[3] < GAP_MIN)
            if len(bad) == 0:
                return x, kbar, res
            if attempt > MAX_ATTEMPTS:
                break
            synth.redraw_q_slc(wl, x["q_slc"], bad, attempt)
        raise RuntimeError("gap rule: no clear top-K after 64 attempts")
    idx, w, s, gap = oracle.select(x["q_slc"], kbar, wl.S, wl.K)
    bad = np.argwhere(gap < GAP_MIN)
    attempt = 0
    while len(bad):
        attempt += 1
        if attempt > MAX_ATTEMPTS:
            raise RuntimeError("gap rule: no clear top-K after 64 attempts")
        synth.redraw_q_slc(wl, x["q_slc"], bad, attempt)
        rows = np.unique(bad[:, 0])
        i2, w2, s2, g2 = oracle.select(x["q_slc"], kbar, wl.S, wl.K, rows=rows)
        idx[rows], w[rows], s[rows], gap[rows] = i2, w2, s2, g2
        bad = np.argwhere(gap < GAP_MIN)
    return x, kbar, (idx, w, s, gap)


@functools.lru_cache(maxsize=4)
def cached_workload(name: str, **overrides):
    wl = synth.WORKLOADS[name]
    if overrides:
        wl = wl.scaled(**overrides)
    return wl, gap_ruled(wl)


def tiny(B=1, L=96, h_q=4, h_kv=2, d=8, S=8, K=3, dtype="f32", structure="iid", seed=7,
         kind="fwd"):
    return synth.Workload("tiny", B, L, h_q, h_kv, d, S, K, dtype, structure, kind, seed)
