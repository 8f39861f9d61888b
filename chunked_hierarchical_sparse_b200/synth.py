"""Seeded synthetic workloads for Hierarchical Sparse Attention (HSA).

This module only draws random numbers: it holds none of the method's
arithmetic.  Every tensor comes from a counter-based generator (numpy's
Philox) keyed by (seed, tensor id, attempt), so the same call gives the same
values on any host.  Values are drawn in fp64 and rounded once to the
workload's dtype; the returned fp64 arrays hold exactly the rounded values.

Workloads (shapes from the HSA paper's 16K-64K long-context settings):
  tiny_fp32   B=1  L=1024  S=64 K=4 h_q=4  h_kv=1 d=64   fp32, N(0,1)
  fwd16k      B=2  L=16384 S=64 K=8 h_q=16 h_kv=2 d=128  bf16, N(0,1); one key
              chunk per sequence (index ~ U[1, n_c/2)) scaled x4 on every KV head
  fwd64k      B=1  L=65536 S=64 K=8 h_q=16 h_kv=2 d=128  bf16, N(0,1) plus a
              per-(b, g, chunk) key offset vector ~ N(0, 0.5^2 I) on every key
  decode16k   B=16 P=16384 S=64 K=8 h_q=16 h_kv=2 d=128  bf16 cache, N(0,1)
  train16k    B=4  L=16384 S=64 K=8 h_q=16 h_kv=2 d=128  bf16, N(0,1); dO N(0,1)
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

# tensor ids for the generator key
_TID = {"q": 1, "k": 2, "v": 3, "q_slc": 4, "dO": 5, "plant": 6, "offset": 7,
        "q_dec": 8, "q_slc_dec": 9, "q_layer": 10}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int            # sequence length (decode: cached prompt length P)
    h_q: int
    h_kv: int
    d: int
    S: int
    K: int
    dtype: str        # "f32" or "bf16"
    structure: str    # "iid", "planted", "offsets"
    kind: str         # "fwd", "decode", "train"
    seed: int

    @property
    def n_c(self) -> int:
        return self.L // self.S

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 1024, 4, 1, 64, 64, 4, "f32", "iid", "fwd", 1001),
    "fwd16k": Workload("fwd16k", 2, 16384, 16, 2, 128, 64, 8, "bf16", "planted", "fwd", 1002),
    "fwd64k": Workload("fwd64k", 1, 65536, 16, 2, 128, 64, 8, "bf16", "offsets", "fwd", 1003),
    "decode16k": Workload("decode16k", 16, 16384, 16, 2, 128, 64, 8, "bf16", "iid", "decode", 1004),
    "train16k": Workload("train16k", 4, 16384, 16, 2, 128, 64, 8, "bf16", "iid", "train", 1005),
}


def _rng(seed: int, tensor: str, attempt: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[seed, (_TID[tensor] << 16) | attempt]))


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values to the workload dtype (fp64 -> fp32 -> bf16, each step
    round-to-nearest-even); return them widened back to fp64."""
    import torch
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        f = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        return f.to(torch.bfloat16).to(torch.float64).numpy()
    raise ValueError(dtype)


def normal(seed: int, tensor: str, shape, attempt: int = 0) -> np.ndarray:
    return _rng(seed, tensor, attempt).standard_normal(size=shape)


def planted_chunks(wl: Workload) -> np.ndarray:
    """Per sequence b, the index of the chunk whose keys are scaled x4."""
    g = _rng(wl.seed, "plant")
    hi = max(2, wl.n_c // 2)
    return g.integers(1, hi, size=wl.B) if wl.n_c >= 2 else np.zeros(wl.B, dtype=np.int64)


def make_inputs(wl: Workload, with_dO: bool | None = None) -> dict:
    """Draw a workload's inputs (fp64 arrays holding dtype-rounded values).

    fwd/train: q [B,L,h_q,d], k, v [B,h_kv,L,d], q_slc [B,L,h_kv,d] (+ dO).
    decode:    q [B,h_q,d], q_slc [B,h_kv,d], k, v caches [B,h_kv,P,d].
    """
    B, L, hq, hk, d, S = wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, wl.S
    out = {}
    k = normal(wl.seed, "k", (B, hk, L, d))
    if wl.structure == "planted":
        for b, c in enumerate(planted_chunks(wl)):
            k[b, :, c * S:(c + 1) * S, :] *= 4.0
    elif wl.structure == "offsets":
        mu = 0.5 * normal(wl.seed, "offset", (B, hk, wl.n_c, d))
        nfull = wl.n_c * S
        k[:, :, :nfull, :] += np.repeat(mu, S, axis=2)
    out["k"] = round_to(k, wl.dtype)
    out["v"] = round_to(normal(wl.seed, "v", (B, hk, L, d)), wl.dtype)
    if wl.kind == "decode":
        out["q"] = round_to(normal(wl.seed, "q_dec", (B, hq, d)), wl.dtype)
        out["q_slc"] = round_to(normal(wl.seed, "q_slc_dec", (B, hk, d)), wl.dtype)
    else:
        out["q"] = round_to(normal(wl.seed, "q", (B, L, hq, d)), wl.dtype)
        out["q_slc"] = round_to(normal(wl.seed, "q_slc", (B, L, hk, d)), wl.dtype)
    if with_dO or (with_dO is None and wl.kind == "train"):
        out["dO"] = round_to(normal(wl.seed, "dO", (B, L, hq, d)), wl.dtype)
    return out


def layer_queries(wl: Workload, n_layers: int) -> np.ndarray:
    """Decode queries of n_layers HSA layers that share one selection and KV
    cache: [n_layers, B, h_q, d]; layer 0 is make_inputs' q, layer l >= 1 is
    drawn from its own stream."""
    shape = (wl.B, wl.h_q, wl.d)
    qs = [round_to(normal(wl.seed, "q_dec", shape), wl.dtype)]
    qs += [round_to(normal(wl.seed, "q_layer", shape, attempt=l), wl.dtype) for l in range(1, n_layers)]
    return np.stack(qs)


def redraw_q_slc(wl: Workload, q_slc: np.ndarray, rows_bg: np.ndarray, attempt: int) -> None:
    """Replace selected selection-query rows with fresh draws, in place.

    rows_bg: int array [n, 2] of (flat token row r = b*L + t, group g) for the
    fwd/train layout [B, L, h_kv, d], or [n, 2] of (b, g) for the decode layout
    [B, h_kv, d].  The new values come from the stream keyed by ``attempt``
    (attempt >= 1), read at the row's own position, so the result does not
    depend on which other rows are redrawn.
    """
    if len(rows_bg) == 0:
        return
    tensor = "q_slc_dec" if wl.kind == "decode" else "q_slc"
    fresh = round_to(normal(wl.seed, tensor, q_slc.shape, attempt=attempt), wl.dtype)
    flat = q_slc.reshape(-1, wl.h_kv, wl.d)
    fflat = fresh.reshape(-1, wl.h_kv, wl.d)
    r, g = rows_bg[:, 0], rows_bg[:, 1]
    flat[r, g, :] = fflat[r, g, :]
