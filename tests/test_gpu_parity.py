"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle.

Bars (fixed in advance, not tuned to results):
  chunk indices           bit-exact (the gap rule leaves no near-ties)
  pooled keys             bit-exact (fp64 sum of bf16/fp32 values, one fp32 rounding)
  fp32 outputs            max |err| <= 1e-5 (forward and gradients)
  bf16 outputs            max |err| <= 2e-2 and relative L2 <= 5e-3
  bf16 gradients          relative L2 <= 5e-3 and, element by element,
                          |err| <= 2e-2 + 2^-8 |ref|: the stated 2e-2 bounds the
                          arithmetic; rounding an element x to bf16 (8 significant
                          bits) moves it by up to 2^-8 |x| on top, and gradients
                          reach magnitudes where that alone exceeds 2e-2 (for
                          |x| >= 8 the bf16 spacing is 2^-4)
  selection weights w     |err| <= 1e-5 (fp32 sigmoid products of fp32 scores)

Every comparison prints its achieved max |err| and relative L2 error.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from chunked_hierarchical_sparse_b200 import synth
from hsa_testutil import cached_workload, gap_ruled

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def hsa():
    import chunked_hierarchical_sparse_b200 as m
    m.load_library()
    return m


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device=DEV, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def _errors(got: np.ndarray, want: np.ndarray, block: int = 1 << 24):
    """max |got - want|, relative L2 error, and for the gradient bar the largest
    |got - want| - 2^-8 |want| (computed in blocks: full-size arrays are large)."""
    g, w = got.reshape(-1), want.reshape(-1)
    mx, ex, num, den = 0.0, -np.inf, 0.0, 0.0
    for i in range(0, g.size, block):
        d = g[i:i + block] - w[i:i + block]
        a = np.abs(d)
        mx = max(mx, float(a.max()))
        ex = max(ex, float((a - 2.0 ** -8 * np.abs(w[i:i + block])).max()))
        num += float(np.dot(d, d))
        den += float(np.dot(w[i:i + block], w[i:i + block]))
    return mx, np.sqrt(num) / max(np.sqrt(den), 1e-30), ex


def assert_out(got: np.ndarray, want: np.ndarray, dtype: str, what: str, grad: bool = False):
    mx, rel, ex = _errors(np.asarray(got, dtype=np.float64), np.asarray(want, dtype=np.float64))
    print(f"[parity] {what} ({dtype}{', gradient' if grad else ''}, {want.size} elements): "
          f"max|err| {mx:.3e}  rel L2 {rel:.3e}" + (f"  max(|err| - 2^-8|ref|) {ex:.3e}" if grad else ""))
    if dtype == "f32":
        assert mx <= 1e-5, f"{what}: max abs err {mx:.3e} > 1e-5"
        return
    if grad:
        assert ex <= 2e-2, f"{what}: |err| - 2^-8 |ref| reaches {ex:.3e} > 2e-2"
    else:
        assert mx <= 2e-2, f"{what}: max abs err {mx:.3e} > 2e-2"
    assert rel <= 5e-3, f"{what}: rel L2 err {rel:.3e}"


def small(name="s", B=2, L=1000, h_q=8, h_kv=2, d=128, K=4, dtype="bf16", structure="iid",
          seed=123, kind="fwd"):
    return synth.Workload(name, B, L, h_q, h_kv, d, 64, K, dtype, structure, kind, seed)


def run_fwd(wl, x):
    m = hsa()
    q, k, v, qs = (to_dev(x[n], wl.dtype) for n in ("q", "k", "v", "q_slc"))
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    ws = torch.empty(m.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, 64, wl.K, tdt, m.OP_FWD),
                     dtype=torch.uint8, device=DEV)
    o, lse, idx, w, kbar = m.hsa_fwd(q, k, v, qs, wl.K, ws=ws)
    torch.cuda.synchronize()
    assert m.hsa_device_status(ws) == 0, "device status word set"
    return o, lse, idx, w, kbar


# --------------------------------------------------------------------------- pool / select
@pytest.mark.parametrize("wl", [small(dtype="f32", d=64), small(), small(L=64 * 40 + 17, B=1)],
                         ids=["f32", "bf16", "ragged"])
def test_pool_bit_exact(wl):
    x = synth.make_inputs(wl)
    kb = hsa().hsa_pool(to_dev(x["k"], wl.dtype))
    assert np.array_equal(kb.cpu().numpy(), oracle.pool(x["k"], wl.S))


@pytest.mark.parametrize("wl", [small(dtype="f32", d=64, K=3), small(K=8, L=4096),
                                small(K=16, L=2048, h_kv=4, h_q=8), small(K=1, L=700)],
                         ids=["f32", "bf16-k8", "k16", "k1-ragged"])
def test_select_indices_exact(wl):
    x, kbar, (idx, w, s, gap) = gap_ruled(wl)
    kb, gi, gw = hsa().hsa_select(to_dev(x["q_slc"], wl.dtype), to_dev(x["k"], wl.dtype), wl.K)
    assert np.array_equal(kb.cpu().numpy(), kbar)
    gi = gi.cpu().numpy().reshape(idx.shape)
    assert np.array_equal(gi, idx), f"{(gi != idx).sum()} index mismatches"
    assert np.abs(gw.cpu().numpy().reshape(w.shape) - w).max() <= 1e-5


# --------------------------------------------------------------------------- forward
FWD_SMALL = [small(dtype="f32", d=64, K=4, L=1024, h_q=4, h_kv=1),
             small(), small(L=64 * 37 + 5, K=8, h_q=16, h_kv=2),
             small(h_q=4, h_kv=4, K=2, L=640), small(d=64, L=1500, K=5),
             small(L=60, K=4), small(L=128, K=8)]


@pytest.mark.parametrize("wl", FWD_SMALL, ids=["f32", "bf16", "ragged-g8", "g1", "d64", "one-chunk",
                                               "K>n_c"])
def test_fwd_small_full(wl):
    x, kbar, sel = gap_ruled(wl)
    o_ref, lse_ref, idx_ref, w_ref = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
    o, lse, idx, w, kb = run_fwd(wl, x)
    assert np.array_equal(idx.cpu().numpy().reshape(idx_ref.shape), idx_ref)
    assert_out(f64(o).reshape(o_ref.shape), o_ref, wl.dtype, "o")
    assert np.abs(f64(lse).reshape(lse_ref.shape) - lse_ref).max() <= (1e-5 if wl.dtype == "f32" else 2e-3)
    # tokens of chunk 0 output exactly zero
    assert not f64(o)[:, :wl.S].any()


# chunk-major tensor-core path: bf16 with G = h_q / h_kv in {8, 16}
FWD_TC = [small(h_q=16, h_kv=2, K=8, L=1000), small(h_q=16, h_kv=1, K=4, L=64 * 45 + 3, B=1),
          small(h_q=16, h_kv=2, d=64, K=8, L=64 * 70 + 30), small(h_q=16, h_kv=2, K=16, L=2048),
          small(h_q=16, h_kv=2, K=1, L=777, B=3),
          small(h_q=16, h_kv=2, K=8, L=64 * 100 + 17, B=2, seed=9)]


@pytest.mark.parametrize("wl", FWD_TC, ids=["g8", "g16-ragged", "g8-d64", "g8-k16", "g8-k1-b3",
                                            "g8-multiwindow"])
def test_fwd_tensor_core_path_full(wl):
    x, kbar, sel = gap_ruled(wl)
    o_ref, lse_ref, idx_ref, w_ref = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
    m = hsa()
    m.hsa_timing_enable(True)
    o, lse, idx, w, kb = run_fwd(wl, x)
    ms, n = m.hsa_timing_read("attend_tc")
    m.hsa_timing_enable(False)
    assert n == 1, "the tensor-core kernel did not run"
    assert np.array_equal(idx.cpu().numpy().reshape(idx_ref.shape), idx_ref)
    assert_out(f64(o).reshape(o_ref.shape), o_ref, "bf16", "o")
    assert np.abs(f64(lse).reshape(lse_ref.shape) - lse_ref).max() <= 2e-3
    assert not f64(o)[:, :wl.S].any()


@pytest.mark.parametrize("factor", [2.0 ** 12, 2.0 ** -12], ids=["v-x4096", "v-x1/4096"])
def test_fwd_tensor_core_value_scale(factor):
    """The chunk-major forward sums chunk outputs in fp16 scaled by a power of two
    >= max|v|.  Scaling v by an exact power of two scales o exactly, so o / factor
    must match the unscaled oracle at the same bar."""
    wl = FWD_TC[0]
    x, kbar, sel = gap_ruled(wl)
    o_ref, lse_ref, idx_ref, w_ref = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
    xs = dict(x)
    xs["v"] = x["v"] * factor
    o, lse, idx, w, kb = run_fwd(wl, xs)
    assert np.array_equal(idx.cpu().numpy().reshape(idx_ref.shape), idx_ref)
    assert_out(f64(o).reshape(o_ref.shape) / factor, o_ref, "bf16", "o")


# --------------------------------------------------------------------------- shared selection
def run_attend(wl, x, idx, w):
    """hsa_attend with the given selection (device tensors); returns (o, lse, status)."""
    m = hsa()
    q, k, v = (to_dev(x[n], wl.dtype) for n in ("q", "k", "v"))
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    ws = torch.empty(m.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, 64, wl.K, tdt, m.OP_FWD),
                     dtype=torch.uint8, device=DEV)
    o, lse = m.hsa_attend(q, k, v, idx, w, ws=ws)
    torch.cuda.synchronize()
    return o, lse, m.hsa_device_status(ws)


def random_selection(wl, seed, w_scale=1.0):
    """Any causal selection (not a top-K): past complete chunks, empty slots,
    repeated chunks and weights of either sign; [B, L, h_kv, K]."""
    rng = np.random.default_rng(seed)
    t = np.arange(wl.L)
    ne = np.minimum(t // wl.S, wl.L // wl.S)[None, :, None, None]
    shape = (wl.B, wl.L, wl.h_kv, wl.K)
    idx = np.floor(rng.random(shape) * ne).astype(np.int32)
    idx[(ne == 0) | (rng.random(shape) < 0.15)] = -1
    w = (rng.normal(size=shape) * w_scale).astype(np.float32)
    return idx, w


ATTEND = [small(dtype="f32", d=64, K=4, L=1024, h_q=4, h_kv=1), small(L=64 * 37 + 5, K=8, h_q=8, h_kv=2),
          small(h_q=16, h_kv=2, K=8, L=1000), small(h_q=16, h_kv=1, K=4, L=64 * 45 + 3, B=1)]
ATTEND_IDS = ["f32-simt", "bf16-g4-simt", "g8-tc", "g16-tc-ragged"]


def tc_ran(wl):
    return wl.dtype == "bf16" and wl.h_q // wl.h_kv in (8, 16)


@pytest.mark.parametrize("wl", ATTEND, ids=ATTEND_IDS)
def test_shared_selection_across_layers(wl):
    """Layer 1 selects (hsa_select on its q_slc, k); layer 2 attends with its own
    q, k, v over layer 1's chunks.  The oracle's forward with layer 2's q, k, v and
    layer 1's q_slc, kbar is the same computation."""
    x1, kbar1, (idx_ref, w_ref, s_ref, gap) = gap_ruled(wl)
    x2 = synth.make_inputs(wl.scaled(seed=wl.seed + 7))
    o_ref, lse_ref, i2, _ = oracle.fwd(x2["q"], x2["k"], x2["v"], x1["q_slc"], kbar1, wl.S, wl.K)
    assert np.array_equal(i2, idx_ref)
    m = hsa()
    kb, idx, w = m.hsa_select(to_dev(x1["q_slc"], wl.dtype), to_dev(x1["k"], wl.dtype), wl.K)
    assert np.array_equal(idx.cpu().numpy().reshape(idx_ref.shape), idx_ref)
    m.hsa_timing_enable(True)
    o, lse, status = run_attend(wl, x2, idx, w)
    _, n_tc = m.hsa_timing_read("attend_tc")
    m.hsa_timing_enable(False)
    assert status == 0
    assert n_tc == (1 if tc_ran(wl) else 0)
    assert_out(f64(o).reshape(o_ref.shape), o_ref, wl.dtype, "o")
    assert np.abs(f64(lse).reshape(lse_ref.shape) - lse_ref).max() <= (1e-5 if wl.dtype == "f32" else 2e-3)


@pytest.mark.parametrize("wl", ATTEND, ids=ATTEND_IDS)
def test_attend_arbitrary_selection(wl):
    """Any causal selection with empty slots, repeats and signed weights."""
    x = synth.make_inputs(wl)
    idx, w = random_selection(wl, wl.seed)
    o_ref, lse_ref = oracle.attend(x["q"], x["k"], x["v"], idx, w, wl.S)
    o, lse, status = run_attend(wl, x, torch.from_numpy(idx).to(DEV), torch.from_numpy(w).to(DEV))
    assert status == 0
    scale = max(1.0, np.abs(o_ref).max())
    got = f64(o).reshape(o_ref.shape)
    assert_out(got / scale, o_ref / scale, wl.dtype, "o")
    assert np.abs(f64(lse).reshape(lse_ref.shape) - lse_ref).max() <= (1e-5 if wl.dtype == "f32" else 2e-3)


def test_attend_large_weights_scale_the_accumulators():
    """Weights of size 2^16 would overflow fp16 cross-chunk sums scaled by max|v|
    alone; the scale takes the row sums of |w| in, so o / 2^16 matches."""
    wl = ATTEND[2]
    x = synth.make_inputs(wl)
    idx, w = random_selection(wl, wl.seed + 1)
    o_ref, _ = oracle.attend(x["q"], x["k"], x["v"], idx, w, wl.S)
    big = torch.from_numpy(w * np.float32(2.0 ** 16)).to(DEV)
    o, _, status = run_attend(wl, x, torch.from_numpy(idx).to(DEV), big)
    assert status == 0
    got = f64(o).reshape(o_ref.shape) / 2.0 ** 16
    assert np.isfinite(got).all()
    scale = max(1.0, np.abs(o_ref).max())
    assert_out(got / scale, o_ref / scale, "bf16", "o")


@pytest.mark.parametrize("wl", [ATTEND[0], ATTEND[2]], ids=["simt", "tc"])
def test_attend_reports_non_causal_index(wl):
    """An entry that is not a causal complete chunk is skipped and reported in the
    status word; every other entry is still attended."""
    x = synth.make_inputs(wl)
    idx, w = random_selection(wl, wl.seed + 2)
    t_bad = 3 * wl.S + 5
    idx[0, t_bad, 0, 0] = 3  # token t_bad sees chunks 0, 1, 2 only
    o, _, status = run_attend(wl, x, torch.from_numpy(idx).to(DEV), torch.from_numpy(w).to(DEV))
    assert status == 6  # HSA_ERR_DEVICE_CHECK
    idx[0, t_bad, 0, 0] = -1
    o_ref, _ = oracle.attend(x["q"], x["k"], x["v"], idx, w, wl.S)
    scale = max(1.0, np.abs(o_ref).max())
    assert_out(f64(o).reshape(o_ref.shape) / scale, o_ref / scale, wl.dtype, "o")


def test_fwd_tiny_fp32_workload():
    """The tiny fp32 workload in full: indices exact, max |err| <= 1e-5."""
    wl, (x, kbar, sel) = cached_workload("tiny_fp32")
    o_ref, lse_ref, idx_ref, w_ref = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
    o, lse, idx, w, kb = run_fwd(wl, x)
    assert np.array_equal(idx.cpu().numpy().reshape(idx_ref.shape), idx_ref)
    assert_out(f64(o).reshape(o_ref.shape), o_ref, "f32", "o")


@pytest.mark.parametrize("name", ["fwd16k", "fwd64k"])
def test_fwd_full_size(name):
    """Full-size workloads in the launch configuration the benchmark times: the
    pooled keys and every chunk index exact, every element of o and lse against
    the oracle's forward over all rows."""
    wl, (x, kbar, (idx_ref, w_ref, s_ref, gap)) = cached_workload(name)
    o, lse, idx, w, kb = run_fwd(wl, x)
    assert np.array_equal(kb.cpu().numpy(), kbar)
    gi = idx.cpu().numpy().reshape(idx_ref.shape)
    assert np.array_equal(gi, idx_ref), f"{(gi != idx_ref).sum()} index mismatches"
    assert np.abs(w.cpu().numpy().reshape(w_ref.shape) - w_ref).max() <= 1e-5
    o_ref, lse_ref, i2, _ = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
    assert np.array_equal(i2, idx_ref)
    assert_out(f64(o).reshape(o_ref.shape), o_ref, wl.dtype, f"o[{name}]")
    del o_ref
    lerr = np.abs(f64(lse).reshape(lse_ref.shape) - lse_ref).max()
    print(f"[parity] lse[{name}]: max|err| {lerr:.3e}")
    assert lerr <= 2e-3


@pytest.mark.parametrize("name", ["fwd64k"])
def test_fwd_repeated_runs_agree(name):
    """The persistent attention kernel hands buffers between roles and CTAs through
    barriers and counters; a missed hand-off shows up as a run that differs from the
    others by far more than the fp16 summation-order noise.  Five runs on the full-size
    workload, compared on every output element (sampled rows against the oracle are
    covered above)."""
    wl, (x, kbar, _) = cached_workload(name)
    m = hsa()
    q, k, v, qs = (to_dev(x[n], wl.dtype) for n in ("q", "k", "v", "q_slc"))
    ws = torch.empty(m.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, 64, wl.K, torch.bfloat16, m.OP_FWD),
                     dtype=torch.uint8, device=DEV)
    outs = []
    for _ in range(5):
        o, _, _, _, _ = m.hsa_fwd(q, k, v, qs, wl.K, want_lse=False, want_sel=False, ws=ws)
        torch.cuda.synchronize()
        assert m.hsa_device_status(ws) == 0
        outs.append(o.float())
    scale = max(1.0, float(outs[0].abs().max()))
    for i in range(1, len(outs)):
        diff = float((outs[i] - outs[0]).abs().max())
        assert diff <= 2e-2 * scale, f"run {i} differs from run 0 by {diff:.3e}"


def test_bwd_repeated_runs_agree():
    """The same for the backward's persistent kernel (three runs, every gradient element)."""
    wl = BWD_TC[1]
    x = synth.make_inputs(wl)
    runs = [run_bwd(wl, x) for _ in range(3)]
    for i in range(1, len(runs)):
        for name, a, b in zip(("dq", "dk", "dv", "dq_slc"), runs[i], runs[0]):
            scale = max(1.0, float(b.float().abs().max()))
            diff = float((a.float() - b.float()).abs().max())
            assert diff <= 2e-2 * scale, f"{name}: run {i} differs from run 0 by {diff:.3e}"


# --------------------------------------------------------------------------- decode
def test_decode_workload():
    wl, (x, kbar, (o_ref, idx_ref, w_ref, gap)) = cached_workload("decode16k")
    m = hsa()
    kc, vc = to_dev(x["k"], "bf16"), to_dev(x["v"], "bf16")
    kb = m.hsa_pool(kc)
    assert np.array_equal(kb.cpu().numpy(), kbar)
    o, idx, w = m.hsa_decode(to_dev(x["q"], "bf16"), to_dev(x["q_slc"], "bf16"), kc, vc, kb, wl.K)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.abs(w.cpu().numpy() - w_ref).max() <= 1e-5
    assert_out(f64(o), o_ref, "bf16", "o")


@pytest.mark.parametrize("P", [0, 63, 64, 640 + 7])
def test_decode_small_edges(P):
    wl = synth.Workload("dec", 3, P, 8, 2, 64, 64, 4, "f32", "iid", "decode", 77 + P)
    x, kbar, (o_ref, idx_ref, w_ref, gap) = gap_ruled(wl)
    m = hsa()
    kc, vc = to_dev(x["k"], "f32"), to_dev(x["v"], "f32")
    o, idx, w = m.hsa_decode(to_dev(x["q"], "f32"), to_dev(x["q_slc"], "f32"), kc, vc,
                             torch.from_numpy(kbar).to(DEV), wl.K)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert_out(f64(o), o_ref, "f32", "o")


# the cluster kernel's other shapes: bf16 d = 64 (tensor-core chunk attention at d = 64),
# 16 query heads per group (the MMA's 16 rows all used), fp32 with 16 heads; one and two layers
DEC_SHAPES = [("bf16", 64, 16, 2), ("bf16", 128, 16, 1), ("f32", 128, 16, 1), ("bf16", 64, 8, 1)]


@pytest.mark.parametrize("dtype,d,h_q,h_kv", DEC_SHAPES, ids=["bf16-d64-g8", "bf16-d128-g16", "f32-d128-g16",
                                                             "bf16-d64-g8-hkv1"])
@pytest.mark.parametrize("NL", [1, 2])
def test_decode_cluster_shapes(dtype, d, h_q, h_kv, NL):
    wl = synth.Workload("decs", 3, 64 * 57 + 21, h_q, h_kv, d, 64, 8, dtype, "iid", "decode", 60 + d + h_q)
    x, kbar, (o_ref, idx_ref, w_ref, gap) = gap_ruled(wl)
    m = hsa()
    kc, vc = to_dev(x["k"], dtype), to_dev(x["v"], dtype)
    kb = torch.from_numpy(kbar).to(DEV)
    qsl = to_dev(x["q_slc"], dtype)
    qs_np = synth.layer_queries(wl, NL)
    m.hsa_timing_enable(True)
    o, idx, w = m.hsa_decode_multi(to_dev(qs_np, dtype), qsl, kc, vc, kb, wl.K)
    _, n_launch = m.hsa_timing_read("decode")
    m.hsa_timing_enable(False)
    torch.cuda.synchronize()
    assert n_launch == 1, "the cluster kernel did not take the call"
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.abs(w.cpu().numpy() - w_ref).max() <= 1e-5
    for l in range(NL):
        o_l, i_l, _, _ = oracle.decode(qs_np[l], x["q_slc"], x["k"], x["v"], kbar, wl.S, wl.K)
        assert np.array_equal(i_l, idx_ref)
        assert_out(f64(o[l]), o_l, dtype, f"decode o[layer {l}] ({dtype} d={d} G={h_q // h_kv})")


def test_decode_offloaded_cache_workload():
    """KV cache in page-locked host memory: only the selected chunks cross the host
    link.  Same kernel and data as the device-cache run, so the same bits."""
    wl, (x, kbar, (o_ref, idx_ref, w_ref, gap)) = cached_workload("decode16k")
    m = hsa()
    kh = torch.from_numpy(x["k"]).to(torch.bfloat16).pin_memory()
    vh = torch.from_numpy(x["v"]).to(torch.bfloat16).pin_memory()
    kb = torch.from_numpy(kbar).to(DEV)
    q, qs = to_dev(x["q"], "bf16"), to_dev(x["q_slc"], "bf16")
    o, idx, w = m.hsa_decode(q, qs, kh, vh, kb, wl.K)
    o_dev, _, _ = m.hsa_decode(q, qs, kh.to(DEV), vh.to(DEV), kb, wl.K)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert_out(f64(o), o_ref, "bf16", "o")
    assert torch.equal(o, o_dev)


def test_decode_refuses_pageable_host_cache():
    """Pageable host memory has no device address: the binding and the C ABI
    both refuse it before any launch."""
    import ctypes
    wl = synth.Workload("dec", 2, 640, 8, 2, 64, 64, 4, "f32", "iid", "decode", 5)
    x = synth.make_inputs(wl)
    m = hsa()
    kh = torch.from_numpy(x["k"]).float()  # ordinary (pageable) host memory
    vh = kh.clone()
    q, qs = to_dev(x["q"], "f32"), to_dev(x["q_slc"], "f32")
    kb = torch.from_numpy(oracle.pool(x["k"], 64)).to(DEV)
    with pytest.raises(ValueError, match="page-locked"):
        m.hsa_decode(q, qs, kh, vh, kb, wl.K)
    o = torch.empty_like(q)
    sh = m.HsaShape(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, 64, wl.K, 0)
    n = m.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, 64, wl.K, torch.float32, m.OP_DECODE)
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    P = ctypes.c_void_p
    rc = m.load_library().hsa_decode(ctypes.byref(sh), P(q.data_ptr()), P(qs.data_ptr()), P(kh.data_ptr()),
                                     P(vh.data_ptr()), P(kb.data_ptr()), P(o.data_ptr()), None, None,
                                     P(ws.data_ptr()), n, None)
    assert rc == 1  # HSA_ERR_INVALID_ARG
    torch.cuda.synchronize()


# (workload, layers, cache memory, launches): the last case, 16 heads per group x 8
# layers x d=128 over a long cache, does not fit the cluster kernel's shared memory
# and runs one launch per layer
DEC_MULTI = [("decode16k", 3, "dev", 1), ("decode16k", 4, "host", 1),
             (synth.Workload("decf32", 3, 64 * 50 + 9, 8, 2, 128, 64, 16, "f32", "iid", "decode", 31), 8, "dev", 1),
             (synth.Workload("decbig", 1, 64 * 5200, 16, 1, 128, 64, 8, "f32", "iid", "decode", 32), 8, "dev", 8)]


@pytest.mark.parametrize("case", DEC_MULTI, ids=["bf16-3-dev", "bf16-4-host", "f32-k16-8", "f32-long-8"])
def test_decode_multi_layer_shared_selection(case):
    """n_layers queries share one selection and one read of each selected chunk.
    Each layer matches the oracle's decode with that layer's query, and equals
    (bit for bit) a single-layer call with the same query."""
    name, NL, where, launches = case
    if isinstance(name, str):
        wl, (x, kbar, (o_ref0, idx_ref, w_ref, gap)) = cached_workload(name)
    else:
        wl = name
        x, kbar, (o_ref0, idx_ref, w_ref, gap) = gap_ruled(wl)
    qs_np = synth.layer_queries(wl, NL)
    m = hsa()
    kc, vc = to_dev(x["k"], wl.dtype), to_dev(x["v"], wl.dtype)
    if where == "host":
        kc, vc = kc.cpu().pin_memory(), vc.cpu().pin_memory()
    kb = torch.from_numpy(kbar).to(DEV)
    qsl = to_dev(x["q_slc"], wl.dtype)
    q = to_dev(qs_np, wl.dtype)
    m.hsa_timing_enable(True)
    o, idx, w = m.hsa_decode_multi(q, qsl, kc, vc, kb, wl.K)
    _, n_launch = m.hsa_timing_read("decode")
    m.hsa_timing_enable(False)
    torch.cuda.synchronize()
    assert n_launch == launches
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    for l in range(NL):
        o_ref, i_l, _, _ = oracle.decode(qs_np[l], x["q_slc"], x["k"], x["v"], kbar, wl.S, wl.K)
        assert np.array_equal(i_l, idx_ref)
        assert_out(f64(o[l]), o_ref, wl.dtype, f"o[layer {l}]")
        if n_launch == 1:  # the cluster kernel for both calls: identical arithmetic per layer
            o1, _, _ = m.hsa_decode(q[l].contiguous(), qsl, kc, vc, kb, wl.K)
            assert torch.equal(o[l], o1), f"layer {l} differs from its single-layer call"


def test_decode_multi_layer_count_bounds():
    wl = synth.Workload("dec", 1, 640, 8, 2, 64, 64, 4, "f32", "iid", "decode", 6)
    x = synth.make_inputs(wl)
    m = hsa()
    kc, vc = to_dev(x["k"], "f32"), to_dev(x["v"], "f32")
    kb = torch.from_numpy(oracle.pool(x["k"], 64)).to(DEV)
    q9 = to_dev(np.stack([x["q"]] * 9), "f32")
    with pytest.raises(m.HsaError):
        m.hsa_decode_multi(q9, to_dev(x["q_slc"], "f32"), kc, vc, kb, wl.K)


# --------------------------------------------------------------------------- backward
def run_bwd(wl, x, kbar_np=None):
    m = hsa()
    q, k, v, qs, dO = (to_dev(x[n], wl.dtype) for n in ("q", "k", "v", "q_slc", "dO"))
    o, lse, idx, w, kbar = m.hsa_fwd(q, k, v, qs, wl.K)
    dq, dk, dv, dqs = m.hsa_bwd(q, k, v, qs, dO, lse, idx, w, kbar, wl.K)
    torch.cuda.synchronize()
    return dq, dk, dv, dqs


BWD_SMALL = [small(dtype="f32", d=64, L=512, K=3, kind="train"),
             small(L=64 * 21 + 9, K=4, kind="train"),
             small(L=1024, K=8, h_q=16, h_kv=2, kind="train")]


@pytest.mark.parametrize("wl", BWD_SMALL, ids=["f32", "bf16-ragged", "bf16-g8"])
def test_bwd_small_full(wl):
    x, kbar, sel = gap_ruled(wl)
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"], wl.S, wl.K)
    got = run_bwd(wl, x)
    for name, g, r in zip(("dq", "dk", "dv", "dq_slc"), got, ref[:4]):
        assert_out(f64(g), r, wl.dtype, name, grad=True)


# chunk-major tensor-core backward: bf16, d in {64, 128}, G in {8, 16}
BWD_TC = [small(h_q=16, h_kv=1, K=4, L=64 * 45 + 3, B=1, kind="train"),
          small(h_q=16, h_kv=2, K=8, L=64 * 100 + 17, B=2, seed=9, kind="train"),
          small(h_q=16, h_kv=2, K=16, L=2048, kind="train"),
          small(h_q=16, h_kv=2, K=1, L=777, B=3, kind="train"),
          small(h_q=16, h_kv=1, d=64, K=4, L=64 * 45 + 3, B=1, seed=21, kind="train"),
          small(h_q=16, h_kv=2, d=64, K=8, L=64 * 100 + 17, B=2, seed=22, kind="train"),
          small(h_q=16, h_kv=2, d=64, K=16, L=2048, seed=23, kind="train")]


@pytest.mark.parametrize("wl", BWD_TC, ids=["g16-ragged", "g8-multiwindow", "g8-k16", "g8-k1-b3",
                                            "d64-g16-ragged", "d64-g8-b2", "d64-g8-k16"])
def test_bwd_tensor_core_path_full(wl):
    x, kbar, sel = gap_ruled(wl)
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"], wl.S, wl.K)
    m = hsa()
    m.hsa_timing_enable(True)
    got = run_bwd(wl, x)
    ms, n = m.hsa_timing_read("bwd_tc")
    m.hsa_timing_enable(False)
    assert n == 1, "the tensor-core backward did not run"
    for name, g, r in zip(("dq", "dk", "dv", "dq_slc"), got, ref[:4]):
        assert_out(f64(g), r, "bf16", name, grad=True)


@pytest.mark.parametrize("wl", [BWD_TC[0], BWD_TC[4]], ids=["d128", "d64"])
@pytest.mark.parametrize("factor", [2.0 ** 12, 2.0 ** -12], ids=["dO-x4096", "dO-x1/4096"])
def test_bwd_tensor_core_grad_scale(factor, wl):
    """The tensor-core backward sums dq in fp16 scaled by a power of two at or above a
    bound computed from max row norms of dO and v and max|k|.  Every gradient is
    linear in dO and scaling dO by a power of two is exact, so grads / factor must
    match the unscaled oracle at the same bar."""
    x, kbar, sel = gap_ruled(wl)
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"], wl.S, wl.K)
    xs = dict(x)
    xs["dO"] = x["dO"] * factor
    got = run_bwd(wl, xs)
    for name, g, r in zip(("dq", "dk", "dv", "dq_slc"), got, ref[:4]):
        assert_out(f64(g) / factor, r, "bf16", name, grad=True)


def test_bwd_train_workload_full():
    """Full-size training workload: every element of dq, dk, dv and dq_slc against
    the oracle's backward over all tokens."""
    wl, (x, kbar, (idx, w, s, gap)) = cached_workload("train16k")
    got = run_bwd(wl, x)
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"], wl.S, wl.K)
    for name, g, r in zip(("dq", "dk", "dv", "dq_slc"), got, ref[:4]):
        assert_out(f64(g), r, "bf16", f"{name}[train16k]", grad=True)


# --------------------------------------------------------------------------- other chunk sizes
# The tensor-core kernels are built around the pages' 64-key chunk; S in {16, 32, 128}
# runs on the CUDA-core kernels (pooling, selection, token-major attention, the decode
# step and the two-phase backward).  (S, dtype, d, h_q, h_kv)
S_CASES = [(16, "f32", 64, 8, 2), (32, "bf16", 128, 16, 2), (128, "bf16", 64, 8, 2),
           (16, "bf16", 128, 4, 1), (128, "f32", 128, 8, 4)]


@pytest.mark.parametrize("S,dtype,d,h_q,h_kv", S_CASES, ids=[f"S{c[0]}-{c[1]}-d{c[2]}" for c in S_CASES])
def test_other_chunk_sizes_fwd_bwd(S, dtype, d, h_q, h_kv):
    K = 4
    wl = synth.Workload(f"s{S}", 2, S * 21 + 5, h_q, h_kv, d, S, K, dtype, "iid", "train", 300 + S + d)
    x, kbar, sel = gap_ruled(wl)
    m = hsa()
    q, k, v, qs, dO = (to_dev(x[n], dtype) for n in ("q", "k", "v", "q_slc", "dO"))
    assert np.array_equal(m.hsa_pool(k, S=S).cpu().numpy(), kbar)
    o_ref, lse_ref, idx_ref, w_ref = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, S, K)
    o, lse, idx, w, kb = m.hsa_fwd(q, k, v, qs, K, S=S)
    torch.cuda.synchronize()
    assert np.array_equal(kb.cpu().numpy(), kbar)
    assert np.array_equal(idx.cpu().numpy().reshape(idx_ref.shape), idx_ref)
    assert np.abs(w.cpu().numpy().reshape(w_ref.shape) - w_ref).max() <= 1e-5
    assert_out(f64(o).reshape(o_ref.shape), o_ref, dtype, f"o (S={S})")
    assert np.abs(f64(lse).reshape(lse_ref.shape) - lse_ref).max() <= (1e-5 if dtype == "f32" else 2e-3)
    assert not f64(o)[:, :S].any()
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"], S, K)
    got = m.hsa_bwd(q, k, v, qs, dO, lse, idx, w, kb, K, S=S)
    torch.cuda.synchronize()
    for name, g, r in zip(("dq", "dk", "dv", "dq_slc"), got, ref[:4]):
        assert_out(f64(g), r, dtype, f"{name} (S={S})", grad=True)


@pytest.mark.parametrize("S", [16, 32, 128])
def test_decode_other_chunk_sizes(S):
    wl = synth.Workload("dec", 3, S * 20 + 3, 8, 2, 64, S, 4, "bf16", "iid", "decode", 90 + S)
    x, kbar, (o_ref, idx_ref, w_ref, gap) = gap_ruled(wl)
    m = hsa()
    kc, vc = to_dev(x["k"], "bf16"), to_dev(x["v"], "bf16")
    kb = m.hsa_pool(kc, S=S)
    assert np.array_equal(kb.cpu().numpy(), kbar)
    o, idx, w = m.hsa_decode(to_dev(x["q"], "bf16"), to_dev(x["q_slc"], "bf16"), kc, vc, kb, wl.K, S=S)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.abs(w.cpu().numpy() - w_ref).max() <= 1e-5
    assert_out(f64(o), o_ref, "bf16", f"decode o (S={S})")


# --------------------------------------------------------------------------- status / errors
def test_device_status_clean_and_bad_index_reported():
    """A corrupted chunk index (one that is not causally eligible) is caught on
    the device: the kernel skips it and sets HSA_ERR_DEVICE_CHECK; nothing traps."""
    m = hsa()
    wl = small(L=512, K=4, kind="train")
    x, kbar, sel = gap_ruled(wl)
    q, k, v, qs, dO = (to_dev(x[n], wl.dtype) for n in ("q", "k", "v", "q_slc", "dO"))
    o, lse, idx, w, kb = m.hsa_fwd(q, k, v, qs, wl.K)
    ws = torch.empty(m.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, 64, wl.K, torch.bfloat16,
                                          m.OP_BWD), dtype=torch.uint8, device=DEV)
    m.hsa_bwd(q, k, v, qs, dO, lse, idx, w, kb, wl.K, ws=ws)
    assert m.hsa_device_status(ws) == 0
    bad = idx.clone()
    bad[0, 100, 0, 0] = 7   # token 100 is in chunk 1: chunk 7 is not eligible
    m.hsa_bwd(q, k, v, qs, dO, lse, bad, w, kb, wl.K, ws=ws)
    assert m.hsa_device_status(ws) == 6
    m.hsa_bwd(q, k, v, qs, dO, lse, idx, w, kb, wl.K, ws=ws)   # cleared by the next call
    assert m.hsa_device_status(ws) == 0


@pytest.mark.parametrize("what", ["fwd", "bwd"])
def test_wait_limit_runs_out_is_reported_and_the_next_call_is_clean(what):
    """The failure path of the persistent kernels, exercised on purpose: with every wait
    bounded at 1 ns some wait runs out, the kernel records HSA_ERR_TIMEOUT in the status
    word, unwinds (its issued copies and MMAs finish, its tensor memory is freed) and
    returns.  The next call with the default bound runs normally and matches the oracle."""
    m = hsa()
    wl = small(h_q=16, h_kv=2, K=8, L=64 * 40 + 7, B=2, kind="train")
    x, kbar, sel = gap_ruled(wl)
    q, k, v, qs, dO = (to_dev(x[n], wl.dtype) for n in ("q", "k", "v", "q_slc", "dO"))
    nf = m.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, 64, wl.K, torch.bfloat16, m.OP_FWD)
    nb = m.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, 64, wl.K, torch.bfloat16, m.OP_BWD)
    wsf = torch.empty(nf, dtype=torch.uint8, device=DEV)
    wsb = torch.empty(nb, dtype=torch.uint8, device=DEV)
    o, lse, idx, w, kb = m.hsa_fwd(q, k, v, qs, wl.K, ws=wsf)
    torch.cuda.synchronize()
    assert m.hsa_device_status(wsf) == 0
    m.hsa_set_wait_limit_ns(1)
    try:
        if what == "fwd":
            m.hsa_fwd(q, k, v, qs, wl.K, ws=wsf)
            code = m.hsa_device_status(wsf)
        else:
            m.hsa_bwd(q, k, v, qs, dO, lse, idx, w, kb, wl.K, ws=wsb)
            code = m.hsa_device_status(wsb)
    finally:
        m.hsa_set_wait_limit_ns(0)
    torch.cuda.synchronize()
    assert code == 5, f"expected HSA_ERR_TIMEOUT, got {code}"
    if what == "fwd":
        o, lse, idx, w, kb = m.hsa_fwd(q, k, v, qs, wl.K, ws=wsf)
        torch.cuda.synchronize()
        assert m.hsa_device_status(wsf) == 0
        o_ref, _, idx_ref, _ = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
        assert np.array_equal(idx.cpu().numpy().reshape(idx_ref.shape), idx_ref)
        assert_out(f64(o).reshape(o_ref.shape), o_ref, "bf16", "o after a timed-out call")
    else:
        dq, dk, dv, dqs = m.hsa_bwd(q, k, v, qs, dO, lse, idx, w, kb, wl.K, ws=wsb)
        torch.cuda.synchronize()
        assert m.hsa_device_status(wsb) == 0
        ref = oracle.bwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, x["dO"], wl.S, wl.K)
        for name, g, r in zip(("dq", "dk", "dv", "dq_slc"), (dq, dk, dv, dqs), ref[:4]):
            assert_out(f64(g), r, "bf16", f"{name} after a timed-out call", grad=True)


def test_empty_inputs():
    m = hsa()
    for L in (0, 30):
        wl = small(L=L, B=1, K=4)
        x = synth.make_inputs(wl)
        o, lse, idx, w, kb = run_fwd(wl, x)
        assert not f64(o).any()
        assert (idx.cpu().numpy() == -1).all() and not w.cpu().numpy().any()
