"""Pins for the fp64 CPU oracle, none of which re-types the oracle's own formulas.

Each test ties the oracle to something else: a closed form, an invariant, a
special case that reduces to a library routine, or brute force on tiny inputs.
They are arranged so that a dropped term, a flipped sign, a wrong index or a
transposed operand anywhere in the oracle fails at least one of them.

Cited pages: [P1] "Hardware-aligned Hierarchical Sparse Attention for
Efficient Long-term Memory Access" (paper notes), sections HSA and kernel.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from chunked_hierarchical_sparse_b200 import synth
from hsa_testutil import gap_ruled, tiny

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def sig(x):
    return 1.0 / (1.0 + math.exp(-x))


# --------------------------------------------------------------------------- pool
def test_pool_constant_chunks_exact():
    """[P1 §HSA, Chunk Selection]: a chunk whose keys are all equal pools to that key."""
    rng = np.random.default_rng(0)
    B, hk, S, nc, d = 2, 3, 8, 5, 6
    L = nc * S + 3  # trailing partial chunk is not pooled
    const = synth.round_to(rng.standard_normal((B, hk, nc, d)), "bf16")
    k = np.zeros((B, hk, L, d))
    k[:, :, :nc * S] = np.repeat(const, S, axis=2)
    k[:, :, nc * S:] = 1e6  # the partial chunk must not leak into any pooled row
    kbar = oracle.pool(k, S)
    assert kbar.shape == (B, hk, nc, d)
    assert np.array_equal(kbar, const.astype(np.float32))


def test_pool_matches_library_mean():
    """Pooling is a plain mean: numpy's mean over the chunk axis, stored as fp32."""
    rng = np.random.default_rng(1)
    B, hk, S, L, d = 2, 2, 16, 100, 8
    k = synth.round_to(rng.standard_normal((B, hk, L, d)), "bf16")
    nc = L // S
    ref = k[:, :, :nc * S].reshape(B, hk, nc, S, d).mean(axis=3).astype(np.float32)
    assert np.array_equal(oracle.pool(k, S), ref)


# --------------------------------------------------------------------------- select
def _scores_np(q_slc, kbar, d):
    # q_slc [B,L,hk,d], kbar [B,hk,nc,d] -> [B,L,hk,nc]
    return np.einsum("blgd,bgcd->blgc", q_slc, kbar.astype(np.float64)) / math.sqrt(d)


def test_select_is_max_sum_subset_bruteforce():
    """The top-K set is the K-subset of eligible chunks with the largest total
    score (brute force over all subsets); slots are ordered most-recent-first."""
    wl = tiny(B=2, L=64, h_q=2, h_kv=2, d=4, S=4, K=3, seed=11)
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    idx, w, s, gap = oracle.select(x["q_slc"], kbar, wl.S, wl.K)
    sc = _scores_np(x["q_slc"], kbar, wl.d)
    for b in range(wl.B):
        for t in range(wl.L):
            r = b * wl.L + t
            ne = min(t // wl.S, wl.n_c)
            for g in range(wl.h_kv):
                got = [c for c in idx[r, g] if c >= 0]
                n_sel = min(ne, wl.K)
                assert len(got) == n_sel
                assert list(idx[r, g, n_sel:]) == [-1] * (wl.K - n_sel)
                assert got == sorted(got, reverse=True)
                if ne == 0:
                    continue
                best = max(itertools.combinations(range(ne), n_sel),
                           key=lambda sub: sum(sc[b, t, g, c] for c in sub))
                assert set(got) == set(best)


def test_select_matches_library_argsort():
    """Same top-K as numpy's stable sort of (-score) on the eligible prefix."""
    wl = tiny(B=1, L=512, h_q=2, h_kv=2, d=16, S=8, K=5, seed=12)
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    idx, w, s, gap = oracle.select(x["q_slc"], kbar, wl.S, wl.K)
    sc = _scores_np(x["q_slc"], kbar, wl.d)
    for t in range(wl.L):
        ne = t // wl.S
        for g in range(wl.h_kv):
            order = np.argsort(-sc[0, t, g, :ne], kind="stable")
            want = sorted(order[:wl.K].tolist(), reverse=True)
            got = [c for c in idx[t, g] if c >= 0]
            assert got == want
            if ne > wl.K:
                srt = np.sort(sc[0, t, g, :ne])[::-1]
                assert gap[t, g] == pytest.approx(srt[wl.K - 1] - srt[wl.K], abs=1e-12)
            else:
                assert math.isinf(gap[t, g])


def test_select_zero_query_ties_pick_most_recent_and_weights_halve():
    """All scores tie at 0: ties go to the higher index, so each token takes its
    K most recent eligible chunks, and with sig(0)=1/2 the stick-breaking
    weights are 1/2, 1/4, 1/8, ..."""
    wl = tiny(B=1, L=80, h_q=2, h_kv=1, d=8, S=8, K=4)
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    idx, w, s, gap = oracle.select(np.zeros_like(x["q_slc"]), kbar, wl.S, wl.K)
    for t in range(wl.L):
        ne = t // wl.S
        n_sel = min(ne, wl.K)
        want = [ne - 1 - j for j in range(n_sel)] + [-1] * (wl.K - n_sel)
        assert list(idx[t, 0]) == want
        for j in range(wl.K):
            assert w[t, 0, j] == (0.5 ** (j + 1) if j < n_sel else 0.0)


def test_select_causality_and_planted_chunk():
    """A chunk is eligible only if it ends before t's own chunk starts: a huge
    key planted in t's own chunk is never picked, one planted in an earlier
    chunk always is (in its most-recent-first slot)."""
    S, d, K = 8, 8, 3
    L = 12 * S
    rng = np.random.default_rng(3)
    k = synth.round_to(rng.standard_normal((1, 1, L, d)), "f32")
    q_slc = np.abs(synth.round_to(rng.standard_normal((1, L, 1, d)), "f32"))
    planted = 6
    k[0, 0, planted * S:(planted + 1) * S, :] = 50.0  # aligned with the positive q_slc
    kbar = oracle.pool(k, S)
    idx, w, s, gap = oracle.select(q_slc, kbar, S, K)
    for t in range(L):
        ct = t // S
        sel = [c for c in idx[t, 0] if c >= 0]
        assert all(c < ct for c in sel)
        assert (planted in sel) == (ct > planted)
    assert list(idx[:S, 0].ravel()) == [-1] * (S * K)  # chunk-0 tokens select nothing


# --------------------------------------------------------------------------- stick-breaking
def test_stick_breaking_closed_forms():
    """w_k >= 0; sum_k w_k = 1 - prod_k (1 - sig(s_k)); K = 1 gives sig(s_max);
    the first slot (most recent) carries sig(s) with nothing broken off."""
    wl = tiny(B=1, L=256, h_q=2, h_kv=2, d=16, S=8, K=6, seed=5)
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    idx, w, s, gap = oracle.select(x["q_slc"], kbar, wl.S, wl.K)
    assert (w >= 0).all()
    for r in range(wl.L):
        for g in range(wl.h_kv):
            n = int((idx[r, g] >= 0).sum())
            prod = 1.0
            for j in range(n):
                prod *= 1.0 - sig(s[r, g, j])
            assert w[r, g].sum() == pytest.approx(1.0 - prod, abs=1e-12)
            assert w[r, g].sum() <= 1.0 + 1e-15
            if n:
                assert w[r, g, 0] == pytest.approx(sig(s[r, g, 0]), abs=1e-15)
    i1, w1, s1, _ = oracle.select(x["q_slc"], kbar, wl.S, 1)
    sc = _scores_np(x["q_slc"], kbar, wl.d)
    for t in range(wl.S, wl.L):
        for g in range(wl.h_kv):
            c = int(np.argmax(sc[0, t, g, :t // wl.S]))
            assert i1[t, g, 0] == c
            assert w1[t, g, 0] == pytest.approx(sig(sc[0, t, g, c]), abs=1e-12)


def test_stick_breaking_two_chunk_hand_case():
    """Two eligible chunks with hand-set pooled keys: scores are s0 = -0.5 (chunk
    0) and s1 = 1.0 (chunk 1); most-recent-first gives w = [sig(1),
    sig(-0.5) * (1 - sig(1))] and idx = [1, 0]."""
    S, d, K = 2, 4, 2
    L = 3 * S
    k = np.zeros((1, 1, L, d))
    k[0, 0, 0:2, 0] = -1.0   # kbar_0 = (-1, 0, 0, 0)
    k[0, 0, 2:4, 1] = 2.0    # kbar_1 = ( 0, 2, 0, 0)
    q_slc = np.zeros((1, L, 1, d))
    q_slc[0, 5, 0] = [1.0, 1.0, 0, 0]  # s0 = -1/2, s1 = 2/2 = 1  (sqrt(d) = 2)
    kbar = oracle.pool(k, S)
    idx, w, s, gap = oracle.select(q_slc, kbar, S, K, rows=[5])
    assert list(idx[0, 0]) == [1, 0]
    assert w[0, 0, 0] == pytest.approx(1 / (1 + math.exp(-1.0)), abs=1e-15)
    assert w[0, 0, 1] == pytest.approx((1 / (1 + math.exp(0.5))) * (1 - 1 / (1 + math.exp(-1.0))),
                                       abs=1e-15)


# --------------------------------------------------------------------------- attention
def test_attention_zero_query_uniform_off_by_one():
    """q = 0: every logit is 0, so p_i = 1/(1+S), O_k = sum_i v_i/(S+1), lse = log(1+S)."""
    wl = tiny(B=1, L=64, h_q=4, h_kv=2, d=8, S=8, K=3, seed=9)
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    q0 = np.zeros_like(x["q"])
    o, lse, idx, w = oracle.fwd(q0, x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
    G = wl.h_q // wl.h_kv
    for t in range(wl.L):
        for h in range(wl.h_q):
            g = h // G
            want = np.zeros(wl.d)
            for j in range(wl.K):
                c = idx[t, g, j]
                if c < 0:
                    continue
                want += w[t, g, j] * x["v"][0, g, c * wl.S:(c + 1) * wl.S].sum(0) / (wl.S + 1)
                assert lse[t, h, j] == pytest.approx(math.log(1 + wl.S), abs=1e-14)
            np.testing.assert_allclose(o[t, h], want, atol=1e-14)


def test_attention_constant_values_and_very_negative_logits():
    """v = u constant: O_k = u * (1 - 1/(1 + sum e^x)) < u; logits -> -inf: O -> 0, finite."""
    wl = tiny(B=1, L=48, h_q=2, h_kv=1, d=8, S=8, K=2, seed=10)
    x = synth.make_inputs(wl)
    v = np.full_like(x["v"], 0.75)
    kbar = oracle.pool(x["k"], wl.S)
    o, lse, idx, w = oracle.fwd(x["q"], x["k"], v, x["q_slc"], kbar, wl.S, wl.K)
    for t in range(wl.L):
        for h in range(wl.h_q):
            want = sum(w[t, 0, j] * 0.75 * (1 - math.exp(-lse[t, h, j]))
                       for j in range(wl.K) if idx[t, 0, j] >= 0)
            np.testing.assert_allclose(o[t, h], want, atol=1e-14)
    # all keys equal to +u, query = -big * u: x_i -> -inf, output must vanish, no NaN
    k = np.ones_like(x["k"])
    q = -1e3 * np.ones_like(x["q"])
    o2, lse2, _, _ = oracle.fwd(q, k, x["v"], x["q_slc"], oracle.pool(k, wl.S), wl.S, wl.K)
    assert np.isfinite(o2).all() and np.isfinite(lse2).all()
    assert np.abs(o2).max() < 1e-300
    assert np.abs(lse2).max() < 1e-300


def test_k1_closed_form():
    """K = 1: o = sig(s*) * softmax1-attention over c* = argmax_c s (library argmax)."""
    wl = tiny(B=1, L=128, h_q=4, h_kv=2, d=8, S=8, K=1, seed=21)
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    o, lse, idx, w = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, 1)
    sc = _scores_np(x["q_slc"], kbar, wl.d)
    G = wl.h_q // wl.h_kv
    for t in range(wl.L):
        for h in range(wl.h_q):
            g = h // G
            ne = t // wl.S
            if ne == 0:
                assert not o[t, h].any()
                continue
            c = int(np.argmax(sc[0, t, g, :ne]))
            kc = x["k"][0, g, c * wl.S:(c + 1) * wl.S]
            vc = x["v"][0, g, c * wl.S:(c + 1) * wl.S]
            e = np.exp(kc @ x["q"][0, t, h] / math.sqrt(wl.d))
            want = sig(sc[0, t, g, c]) * (e @ vc) / (1.0 + e.sum())
            np.testing.assert_allclose(o[t, h], want, atol=1e-13)


@pytest.mark.parametrize("S", [4, 8])
def test_dense_masked_bruteforce(S):
    """Brute force: the full L x L logit matrix (library matmul), a block mask from
    the selection, and o_t = sum_c [c selected] w_c (sum_{i in c} e^X v_i)/(1 + sum_{i in c} e^X)."""
    wl = tiny(B=2, L=256 if S == 4 else 512, h_q=4, h_kv=2, d=8, S=S, K=3, seed=30 + S)
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    o, lse, idx, w = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
    o = o.reshape(wl.B, wl.L, wl.h_q, wl.d)
    idx = idx.reshape(wl.B, wl.L, wl.h_kv, wl.K)
    w = w.reshape(wl.B, wl.L, wl.h_kv, wl.K)
    G = wl.h_q // wl.h_kv
    chunk_of = np.arange(wl.L) // wl.S
    for b in range(wl.B):
        for h in range(wl.h_q):
            g = h // G
            X = x["q"][b, :, h, :] @ x["k"][b, g].T / math.sqrt(wl.d)  # [L, L]
            E = np.exp(X)
            want = np.zeros((wl.L, wl.d))
            for t in range(wl.L):
                for j in range(wl.K):
                    c = idx[b, t, g, j]
                    if c < 0:
                        continue
                    m = chunk_of == c
                    want[t] += w[b, t, g, j] * (E[t, m] @ x["v"][b, g][m]) / (1.0 + E[t, m].sum())
            np.testing.assert_allclose(o[b, :, h], want, atol=1e-12, rtol=1e-12)


# --------------------------------------------------------------------------- shared selection
def _random_causal_selection(rng, B, L, h_kv, K, S):
    """Any causal selection: complete past chunks, empty slots (-1), repeats, any weights."""
    idx = np.full((B * L, h_kv, K), -1, dtype=np.int32)
    for r in range(B * L):
        ne = min((r % L) // S, L // S)
        if ne:
            idx[r] = rng.integers(0, ne, size=(h_kv, K))
    idx[rng.random(idx.shape) < 0.2] = -1
    w = rng.normal(size=idx.shape)
    return idx, w


def test_attend_given_selection_dense_masked_bruteforce():
    """attend(idx, w) for an arbitrary causal selection against the dense L x L
    logit matrix (library matmul) with a block mask per listed chunk."""
    wl = tiny(B=2, L=96, h_q=4, h_kv=2, d=8, S=8, K=4, seed=41)
    x = synth.make_inputs(wl)
    idx, w = _random_causal_selection(np.random.default_rng(5), wl.B, wl.L, wl.h_kv, wl.K, wl.S)
    idx[3 * wl.S + 1, 0, :2] = 1  # a chunk listed twice for one row
    o, lse = oracle.attend(x["q"], x["k"], x["v"], idx, w, wl.S)
    o = o.reshape(wl.B, wl.L, wl.h_q, wl.d)
    idx4, w4 = idx.reshape(wl.B, wl.L, wl.h_kv, wl.K), w.reshape(wl.B, wl.L, wl.h_kv, wl.K)
    G = wl.h_q // wl.h_kv
    chunk_of = np.arange(wl.L) // wl.S
    for b in range(wl.B):
        for h in range(wl.h_q):
            g = h // G
            E = np.exp(x["q"][b, :, h, :] @ x["k"][b, g].T / math.sqrt(wl.d))
            want = np.zeros((wl.L, wl.d))
            for t in range(wl.L):
                for j in range(wl.K):
                    c = idx4[b, t, g, j]
                    if c < 0:
                        continue
                    m = chunk_of == c
                    want[t] += w4[b, t, g, j] * (E[t, m] @ x["v"][b, g][m]) / (1.0 + E[t, m].sum())
            np.testing.assert_allclose(o[b, :, h], want, atol=1e-12, rtol=1e-12)


def test_attend_with_own_selection_is_forward():
    """attend over select's (idx, w) is the forward pass exactly (same rows, bit for bit)."""
    wl = tiny(B=1, L=128, h_q=4, h_kv=2, d=8, S=8, K=3, seed=42)
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    o, lse, idx, w = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
    o2, lse2 = oracle.attend(x["q"], x["k"], x["v"], idx, w, wl.S)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
    rows = np.array([5, 64, 127])
    o3, _ = oracle.attend(x["q"], x["k"], x["v"], idx[rows], w[rows], wl.S, rows=rows)
    assert np.array_equal(o3, o[rows])


def test_attend_rejects_non_causal_entries():
    wl = tiny(B=1, L=64, h_q=2, h_kv=1, d=8, S=8, K=2, seed=43)
    x = synth.make_inputs(wl)
    idx = np.full((wl.L, 1, wl.K), -1, dtype=np.int32)
    w = np.ones(idx.shape)
    idx[20, 0, 0] = 2  # token 20 sees chunks 0, 1 only
    with pytest.raises(RuntimeError, match="code -4"):
        oracle.attend(x["q"], x["k"], x["v"], idx, w, wl.S)
    idx[20, 0, 0] = 1
    idx[20, 0, 1] = -7  # any negative entry is an empty slot
    o, _ = oracle.attend(x["q"], x["k"], x["v"], idx, w, wl.S)
    idx[20, 0, 1] = -1
    o2, _ = oracle.attend(x["q"], x["k"], x["v"], idx, w, wl.S)
    assert np.array_equal(o, o2) and o[20].any()


# --------------------------------------------------------------------------- decode
def test_decode_equals_forward_last_row():
    """The decode step at position P is forward row t = P of the prompt plus one token."""
    P, S = 96, 8
    wl = tiny(B=3, L=P + 1, h_q=4, h_kv=2, d=8, S=S, K=3, seed=41)
    x = synth.make_inputs(wl)
    kbar_full = oracle.pool(x["k"], S)
    o, lse, idx, w = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar_full, S, wl.K,
                                rows=[b * (P + 1) + P for b in range(wl.B)])
    kc, vc = x["k"][:, :, :P], x["v"][:, :, :P]
    od, idd, wd, gap = oracle.decode(x["q"][:, P], x["q_slc"][:, P], kc, vc, oracle.pool(kc, S),
                                     S, wl.K)
    np.testing.assert_array_equal(idd, idx)
    np.testing.assert_allclose(od, o, atol=1e-15)
    np.testing.assert_allclose(wd, w, atol=1e-15)


# --------------------------------------------------------------------------- backward
def _loss(x, kbar0, dO, wl, **over):
    xx = dict(x)
    xx.update(over)
    kb = over.get("kbar", kbar0)
    o, *_ = oracle.fwd(xx["q"], xx["k"], xx["v"], xx["q_slc"], kb, wl.S, wl.K)
    return float((o.reshape(dO.shape) * dO).sum())


def test_backward_central_differences():
    """Central differences of L = sum dO*o in fp64: q, v, q_slc directly; k with the
    pooled index held fixed (the attention path of dk); the pooled index itself
    (fp32 input, step representable in fp32) for dkbar.  The gap rule keeps the
    selection fixed under the steps."""
    wl = tiny(B=1, L=64, h_q=4, h_kv=2, d=8, S=8, K=3, seed=51, kind="train")
    x, kbar, _ = gap_ruled(wl)
    dO = x["dO"]
    dq, dk, dv, dqs, dkbar = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, dO, wl.S, wl.K)
    rng = np.random.default_rng(0)
    eps = 1e-6

    def fd(name, pos):
        a = x[name].copy()
        a[pos] += eps
        lp = _loss(x, kbar, dO, wl, **{name: a})
        a[pos] -= 2 * eps
        lm = _loss(x, kbar, dO, wl, **{name: a})
        return (lp - lm) / (2 * eps)

    for name, grad in (("q", dq), ("v", dv), ("q_slc", dqs)):
        for _ in range(12):
            pos = tuple(rng.integers(0, n) for n in x[name].shape)
            assert fd(name, pos) == pytest.approx(grad[pos], abs=2e-7, rel=1e-5), (name, pos)
    # k: attention path only (kbar held fixed) -> dk minus the pooled share dkbar/S
    dk_attn = dk - np.repeat(dkbar, wl.S, axis=2) / wl.S
    for _ in range(12):
        pos = tuple(rng.integers(0, n) for n in x["k"].shape)
        assert fd("k", pos) == pytest.approx(dk_attn[pos], abs=2e-7, rel=1e-5), pos
    # kbar: fp32 input; use a step that fp32 represents exactly relative to the value
    for _ in range(12):
        pos = tuple(rng.integers(0, n) for n in kbar.shape)
        kp, km = kbar.copy(), kbar.copy()
        kp[pos] = np.float32(kbar[pos] + np.float32(2 ** -10))
        km[pos] = np.float32(kbar[pos] - np.float32(2 ** -10))
        num = (_loss(x, kbar, dO, wl, kbar=kp) - _loss(x, kbar, dO, wl, kbar=km)) / (
            float(kp[pos]) - float(km[pos]))
        assert num == pytest.approx(dkbar[pos], abs=1e-6, rel=1e-4), pos


def test_backward_matches_autograd_dense_restatement():
    """torch.autograd (fp64) through a dense masked restatement: chunk means by
    reshape/mean, scores by einsum, the oracle's chosen slots as a fixed mask,
    stick-breaking by cumprod, attention as masked exp sums over the full L x L
    logits.  Gradients must match the oracle's per-token loops."""
    wl = tiny(B=2, L=96, h_q=4, h_kv=2, d=8, S=8, K=3, seed=61, kind="train")
    x, kbar, (idx, w, s, gap) = gap_ruled(wl)
    T = {n: torch.tensor(x[n], dtype=torch.float64, requires_grad=True)
         for n in ("q", "k", "v", "q_slc")}
    B, L, hq, hk, d, S, K = wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, wl.S, wl.K
    G = hq // hk
    nc = L // S
    kb = T["k"][:, :, :nc * S].reshape(B, hk, nc, S, d).mean(3)             # [B,hk,nc,d]
    kb = kb + (kb.float().double() - kb).detach()  # stored as fp32, gradient of the mean
    sc = torch.einsum("blgd,bgcd->blgc", T["q_slc"], kb) / math.sqrt(d)      # [B,L,hk,nc]
    idx_t = torch.tensor(idx.reshape(B, L, hk, K), dtype=torch.long)
    valid = idx_t >= 0
    s_sel = torch.gather(sc, 3, idx_t.clamp(min=0)) * valid
    sg = torch.sigmoid(s_sel) * valid
    keep = torch.cumprod(torch.cat([torch.ones_like(sg[..., :1]), 1 - sg[..., :-1]], -1), -1)
    wt = sg * keep                                                          # [B,L,hk,K]
    X = torch.einsum("blhd,bgmd->blhgm", T["q"], T["k"]) / math.sqrt(d)     # all logits
    hidx = torch.arange(hq) // G
    X = X[:, :, torch.arange(hq), hidx, :]                                   # [B,L,hq,L]
    E = torch.exp(X)
    chunk_of = torch.arange(L) // S
    o = torch.zeros(B, L, hq, d, dtype=torch.float64)
    for j in range(K):
        c = idx_t[:, :, hidx, j]                                            # [B,L,hq]
        m = (chunk_of.view(1, 1, 1, L) == c.unsqueeze(-1)).to(torch.float64)
        num = torch.einsum("blhm,bhmd->blhd", E * m, T["v"][:, hidx])
        den = 1.0 + (E * m).sum(-1, keepdim=True)
        o = o + wt[:, :, hidx, j].unsqueeze(-1) * num / den
    dO = torch.tensor(x["dO"])
    (o * dO).sum().backward()
    dq, dk, dv, dqs, _ = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"], S, K)
    np.testing.assert_allclose(dq, T["q"].grad.numpy(), atol=1e-9, rtol=1e-7)
    np.testing.assert_allclose(dv, T["v"].grad.numpy(), atol=1e-9, rtol=1e-7)
    np.testing.assert_allclose(dqs, T["q_slc"].grad.numpy(), atol=1e-7, rtol=1e-5)
    np.testing.assert_allclose(dk, T["k"].grad.numpy(), atol=1e-7, rtol=1e-5)


def test_backward_dv_chunk_sum_invariant():
    """Summed over a chunk's keys, dv equals the sum over (t, h, slot) selecting
    the chunk of w * (sum_i p_i) * dO[t, h], with sum_i p_i = 1 - exp(-lse)."""
    wl = tiny(B=1, L=128, h_q=4, h_kv=2, d=8, S=8, K=3, seed=71, kind="train")
    x, kbar, _ = gap_ruled(wl)
    o, lse, idx, w = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
    dq, dk, dv, dqs, dkbar = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"],
                                        wl.S, wl.K)
    G = wl.h_q // wl.h_kv
    want = np.zeros((wl.h_kv, wl.n_c, wl.d))
    for t in range(wl.L):
        for h in range(wl.h_q):
            g = h // G
            for j in range(wl.K):
                c = idx[t, g, j]
                if c >= 0:
                    want[g, c] += w[t, g, j] * (1 - math.exp(-lse[t, h, j])) * x["dO"][0, t, h]
    got = dv[0, :, :wl.n_c * wl.S].reshape(wl.h_kv, wl.n_c, wl.S, wl.d).sum(2)
    np.testing.assert_allclose(got, want, atol=1e-12)


def test_backward_token_mask_completes_selected_chunks():
    """With a token mask that holds every token selecting chunk c, dk/dv of chunk c
    and dq of those tokens equal the unmasked run."""
    wl = tiny(B=1, L=128, h_q=4, h_kv=2, d=8, S=8, K=3, seed=72, kind="train")
    x, kbar, (idx, w, s, gap) = gap_ruled(wl)
    full = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"], wl.S, wl.K)
    g, c = 1, 3
    mask = (idx[:, g, :] == c).any(-1).reshape(1, wl.L)
    part = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"], wl.S, wl.K, tok_mask=mask)
    sl = slice(c * wl.S, (c + 1) * wl.S)
    np.testing.assert_allclose(part[1][0, g, sl], full[1][0, g, sl], atol=1e-15)
    np.testing.assert_allclose(part[2][0, g, sl], full[2][0, g, sl], atol=1e-15)
    toks = np.nonzero(mask[0])[0]
    np.testing.assert_allclose(part[0][0, toks], full[0][0, toks], atol=1e-15)


# --------------------------------------------------------------------------- generator / gap rule
def test_gap_rule_leaves_clear_gaps_and_is_deterministic():
    wl = tiny(B=2, L=512, h_q=4, h_kv=2, d=16, S=8, K=4, dtype="bf16", seed=81)
    x1, kb1, sel1 = gap_ruled(wl)
    x2, kb2, sel2 = gap_ruled(wl)
    gap = sel1[3]
    assert (gap >= 1e-3).all()
    assert np.array_equal(x1["q_slc"], x2["q_slc"]) and np.array_equal(sel1[0], sel2[0])
    # bf16 rounding: every value is representable in bf16 (low 16 fp32 bits zero)
    f = x1["q"].astype(np.float32).view(np.uint32)
    assert not (f & 0xFFFF).any()


def test_oracle_regression_snapshot():
    """The oracle still produces the committed snapshot (tests/golden/oracle_tiny.txt)."""
    import os
    import sys
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    sys.path.insert(0, here)
    import make_golden
    got = dict(zip(("kbar", "o", "lse", "idx", "w"), make_golden.compute()))
    lines = [ln for ln in open(os.path.join(here, "oracle_tiny.txt")) if not ln.startswith("#")]
    for hdr, body in zip(lines[0::2], lines[1::2]):
        name, *shape = hdr.split()
        want = np.array([float(v) for v in body.split()]).reshape([int(n) for n in shape])
        np.testing.assert_allclose(got[name], want, rtol=0, atol=1e-15, err_msg=name)
