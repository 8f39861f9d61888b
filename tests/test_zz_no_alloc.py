"""hsa_fwd_noalloc: the forward pass for callers that cannot allocate device
memory (e.g. plug-ins inside a runtime that owns all allocations, or
latency-critical loops where cudaMalloc may synchronise the device).

It is called here straight through the C ABI and checked against the fp64
oracle's forward (chunk indices exact, outputs within the same tolerances as
the other parity tests) on two calls in a row with different inputs: the
shared scratch keeps the previous call's contents, so the second call must not
depend on them.  Each call's result is also compared with hsa_fwd's.  This
file is named to be collected last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
from chunked_hierarchical_sparse_b200 import synth
from hsa_testutil import gap_ruled

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _fn():
    import chunked_hierarchical_sparse_b200 as m
    lib = m.load_library()
    f = lib.hsa_fwd_noalloc
    P = ctypes.c_void_p
    f.argtypes = [ctypes.POINTER(m.HsaShape), P, P, P, P, P, P, P, P, P, P]
    f.restype = ctypes.c_int
    return m, f


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(got, ref, dtype, what):
    err = np.abs(got - ref).max()
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    print(f"[parity] no-alloc {what} ({dtype}): max|err| {err:.3e} rel L2 {rel:.3e}")
    if dtype == "f32":
        assert err <= 1e-5, (what, err)
    else:
        assert err <= 2e-2 and rel <= 5e-3, (what, err, rel)


@pytest.mark.parametrize("tdtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_noalloc_matches_oracle_on_two_calls(tdtype):
    m, f = _fn()
    dt = "bf16" if tdtype == torch.bfloat16 else "f32"
    for call, seed in enumerate((501, 502)):
        wl = synth.Workload("na", 2, 64 * 30 + 11, 8, 2, 128, 64, 4, dt, "iid", "fwd", seed)
        x, kbar, sel = gap_ruled(wl)
        o_ref, lse_ref, idx_ref, w_ref = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K)
        q, k, v, qs = (torch.from_numpy(x[n]).to(DEV, tdtype) for n in ("q", "k", "v", "q_slc"))
        o = torch.empty_like(q)
        lse = torch.empty((wl.B, wl.L, wl.h_q, wl.K), dtype=torch.float32, device=DEV)
        sh = m.HsaShape(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, wl.S, wl.K, 1 if dt == "bf16" else 0)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        # intermediates left to the library's scratch on the first call, returned on the second
        idx = torch.empty((wl.B, wl.L, wl.h_kv, wl.K), dtype=torch.int32, device=DEV) if call else None
        w = torch.empty((wl.B, wl.L, wl.h_kv, wl.K), dtype=torch.float32, device=DEV) if call else None
        rc = f(ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), _ptr(qs), _ptr(o), _ptr(lse), _ptr(idx),
               _ptr(w), None, stream)
        assert rc == 0
        torch.cuda.synchronize()
        _check(o.double().cpu().numpy().reshape(o_ref.shape), o_ref, dt, f"o (call {call + 1})")
        lerr = np.abs(lse.double().cpu().numpy().reshape(lse_ref.shape) - lse_ref).max()
        assert lerr <= (1e-5 if dt == "f32" else 2e-3), lerr
        if call:
            assert np.array_equal(idx.cpu().numpy().reshape(idx_ref.shape), idx_ref)
            assert np.abs(w.cpu().numpy().reshape(w_ref.shape) - w_ref).max() <= 1e-5
        # the same call through hsa_fwd (caller workspace) gives the same result
        o2 = m.hsa_fwd(q, k, v, qs, wl.K)[0]
        torch.cuda.synchronize()
        _check(o.double().cpu().numpy(), o2.double().cpu().numpy(), dt, f"o vs hsa_fwd (call {call + 1})")


def test_noalloc_rejects_problems_beyond_its_scratch():
    m, f = _fn()
    # 2^20 tokens x 2 groups x K=16: the chunk indices alone need 128 MiB > 32 MiB
    sh = m.HsaShape(1, 1 << 20, 16, 2, 128, 64, 16, 1)
    P = ctypes.c_void_p(1 << 20)
    assert f(ctypes.byref(sh), P, P, P, P, P, None, None, None, None, None) == 3
