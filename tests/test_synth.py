"""The seeded input generators shared by the tests, the benchmark and the oracle
runs: deterministic, distinct per tensor and per layer, dtype-rounded, and shaped
as the workloads state.  They hold none of the method's arithmetic."""
from __future__ import annotations

import numpy as np
import torch

from chunked_hierarchical_sparse_b200 import synth


def _wl(**kw):
    base = dict(name="t", B=2, L=200, h_q=8, h_kv=2, d=64, S=64, K=4, dtype="bf16", structure="iid",
                kind="decode", seed=11)
    base.update(kw)
    return synth.Workload(**base)


def test_make_inputs_is_deterministic_and_shaped():
    for kind in ("fwd", "train", "decode"):
        wl = _wl(kind=kind)
        a, b = synth.make_inputs(wl), synth.make_inputs(wl)
        assert a.keys() == b.keys()
        for n in a:
            assert np.array_equal(a[n], b[n]), n
        assert a["k"].shape == (wl.B, wl.h_kv, wl.L, wl.d) == a["v"].shape
        if kind == "decode":
            assert a["q"].shape == (wl.B, wl.h_q, wl.d) and a["q_slc"].shape == (wl.B, wl.h_kv, wl.d)
        else:
            assert a["q"].shape == (wl.B, wl.L, wl.h_q, wl.d)
            assert a["q_slc"].shape == (wl.B, wl.L, wl.h_kv, wl.d)
        assert ("dO" in a) == (kind == "train")
    # another seed gives other values
    assert not np.array_equal(synth.make_inputs(_wl())["k"], synth.make_inputs(_wl(seed=12))["k"])


def test_values_are_rounded_to_the_workload_dtype():
    x = synth.make_inputs(_wl(dtype="bf16"))
    for n, a in x.items():
        t = torch.from_numpy(a)
        assert torch.equal(t.to(torch.bfloat16).to(torch.float64), t), n
    x = synth.make_inputs(_wl(dtype="f32"))
    for n, a in x.items():
        assert np.array_equal(a.astype(np.float32).astype(np.float64), a), n


def test_layer_queries_extend_the_workload_query():
    wl = _wl()
    q = synth.layer_queries(wl, 4)
    assert q.shape == (4, wl.B, wl.h_q, wl.d)
    assert np.array_equal(q[0], synth.make_inputs(wl)["q"])  # layer 0 is the workload's own query
    for i in range(4):
        for j in range(i + 1, 4):
            assert not np.array_equal(q[i], q[j])
    assert np.array_equal(q, synth.layer_queries(wl, 4))
    assert np.array_equal(q[:2], synth.layer_queries(wl, 2))  # a layer's draw does not depend on the count


def test_planted_and_offset_structures():
    wl = _wl(kind="fwd", L=64 * 12, structure="planted")
    x, base = synth.make_inputs(wl), synth.make_inputs(wl.scaled(structure="iid"))
    for b, c in enumerate(synth.planted_chunks(wl)):
        sl = slice(c * wl.S, (c + 1) * wl.S)
        np.testing.assert_allclose(x["k"][b, :, sl], 4.0 * base["k"][b, :, sl], rtol=2 ** -7)
    wl = _wl(kind="fwd", L=64 * 12 + 5, structure="offsets")
    x = synth.make_inputs(wl)
    assert x["k"].shape == (wl.B, wl.h_kv, wl.L, wl.d)
    # the chunk means carry the offsets: their spread across chunks exceeds that of iid keys
    means = x["k"][:, :, : 12 * wl.S].reshape(wl.B, wl.h_kv, 12, wl.S, wl.d).mean(3)
    assert means.std() > 0.3


def test_redraw_changes_only_the_listed_rows():
    wl = _wl(kind="fwd")
    x = synth.make_inputs(wl)
    qs = x["q_slc"].copy()
    rows = np.array([[3, 0], [150, 1]])
    synth.redraw_q_slc(wl, qs, rows, attempt=1)
    flat0, flat1 = x["q_slc"].reshape(-1, wl.h_kv, wl.d), qs.reshape(-1, wl.h_kv, wl.d)
    changed = np.argwhere(np.any(flat0 != flat1, axis=2))
    assert sorted(map(tuple, changed)) == [(3, 0), (150, 1)]
