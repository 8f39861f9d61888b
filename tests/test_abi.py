"""The C-ABI library builds, loads without a GPU, exports every declared entry
point, and rejects bad arguments on the host before touching CUDA."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hsa.h")


@pytest.fixture(scope="session")
def lib():
    from chunked_hierarchical_sparse_b200 import build, load_library
    build.build()
    return load_library()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"HSA_API\s+[\w\s\*]*?\b(hsa_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    assert {"hsa_pool", "hsa_select", "hsa_fwd", "hsa_attend", "hsa_decode", "hsa_bwd", "hsa_workspace_size",
            "hsa_device_status", "hsa_status_string"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_library_exports_nothing_else(lib):
    import subprocess
    from chunked_hierarchical_sparse_b200 import lib_path
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True).stdout
    ours = {ln.split()[-1] for ln in out.splitlines() if " T " in ln and ln.split()[-1].startswith("hsa_")}
    assert ours == set(declared_symbols())


def _shape(**kw):
    from chunked_hierarchical_sparse_b200 import HsaShape
    d = dict(B=1, L=1024, h_q=16, h_kv=2, d=128, S=64, K=8, dtype=1)
    d.update(kw)
    return HsaShape(**d)


def test_workspace_size_host_only(lib):
    from chunked_hierarchical_sparse_b200 import OP_BWD, OP_DECODE, OP_FWD, OP_POOL
    sh = _shape()
    assert lib.hsa_workspace_size(ctypes.byref(sh), OP_POOL) == 256
    assert lib.hsa_workspace_size(ctypes.byref(sh), OP_DECODE) >= 256
    fwd = lib.hsa_workspace_size(ctypes.byref(sh), OP_FWD)
    assert fwd >= 256 + 1 * 2 * 16 * 128 * 4 + 2 * 1024 * 2 * 8 * 4
    assert lib.hsa_workspace_size(ctypes.byref(sh), OP_BWD) > fwd
    for bad in (dict(S=48), dict(S=8), dict(d=96), dict(K=17), dict(h_q=15), dict(h_kv=0), dict(dtype=7)):
        assert lib.hsa_workspace_size(ctypes.byref(_shape(**bad)), OP_FWD) == 0, bad
    for S in (16, 32, 128):  # other chunk sizes run on the CUDA-core kernels
        assert lib.hsa_workspace_size(ctypes.byref(_shape(S=S)), OP_FWD) > 256, S
    assert lib.hsa_workspace_size(ctypes.byref(sh), 99) == 0


def test_host_validation_without_gpu(lib):
    """Bad arguments return a status before any CUDA call (no GPU needed)."""
    sh = _shape()
    P = ctypes.c_void_p
    good = P(1 << 20)          # aligned, never dereferenced: validation fails first
    odd = P((1 << 20) + 8)     # not 16-byte aligned
    ws = P(1 << 24)
    # null input
    assert lib.hsa_pool(ctypes.byref(sh), None, good, ws, 1 << 20, None) == 1
    # misaligned input
    assert lib.hsa_pool(ctypes.byref(sh), odd, good, ws, 1 << 20, None) == 1
    # unsupported chunk size / head dim
    assert lib.hsa_pool(ctypes.byref(_shape(S=48)), good, good, ws, 1 << 20, None) == 2
    assert lib.hsa_fwd(ctypes.byref(_shape(d=80)), good, good, good, good, good, None, None, None,
                       None, ws, 1 << 30, None) == 2
    # h_q not a multiple of h_kv
    assert lib.hsa_fwd(ctypes.byref(_shape(h_q=15)), good, good, good, good, good, None, None, None,
                       None, ws, 1 << 30, None) == 1
    # workspace too small / misaligned
    assert lib.hsa_fwd(ctypes.byref(sh), good, good, good, good, good, None, None, None, None, ws, 300,
                       None) == 3
    assert lib.hsa_fwd(ctypes.byref(sh), good, good, good, good, good, None, None, None, None,
                       P((1 << 24) + 16), 1 << 30, None) == 1
    # bwd needs every gradient output
    assert lib.hsa_bwd(ctypes.byref(sh), good, good, good, good, good, good, good, good, good, None,
                       good, good, good, ws, 1 << 30, None) == 1
    # shared-selection attend needs idx and w; workspace is the forward's
    assert lib.hsa_attend(ctypes.byref(sh), good, good, good, None, good, good, None, ws, 1 << 30, None) == 1
    assert lib.hsa_attend(ctypes.byref(sh), good, good, good, good, good, good, None, ws, 300, None) == 3
    # decode for several layers: 1 <= n_layers <= HSA_MAX_LAYERS
    dsh = _shape()
    for nl in (0, 9):
        assert lib.hsa_decode_multi(ctypes.byref(dsh), nl, good, good, good, good, good, good, None, None,
                                    ws, 1 << 30, None) == 1
    assert lib.hsa_device_status(None, None, None) == 1
    assert lib.hsa_status_string(3) == b"workspace too small"


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import chunked_hierarchical_sparse_b200 as hsa
    monkeypatch.setattr(hsa, "_lib", None)
    monkeypatch.setattr(hsa, "lib_path", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        hsa.load_library()


def _prototypes():
    """name -> (return type, [parameter declarations]) for every HSA_API prototype."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"HSA_API\s+([\w\s\*]*?)\b(hsa_\w+)\s*\(([^)]*)\)\s*;", text):
        params = [p.strip() for p in m.group(3).split(",") if p.strip() and p.strip() != "void"]
        out[m.group(2)] = (" ".join(m.group(1).split()), params)
    return out


def _ctype_kind(t):
    if t is None:
        return None
    if t in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(t, "_type_") and isinstance(t._type_, type):
        return "ptr"
    if t is ctypes.c_size_t:  # on LP64 also c_uint64
        return "u64"
    if t in (ctypes.c_int, ctypes.c_int32):
        return "int32"
    return repr(t)


def _decl_kind(decl):
    if "*" in decl:
        return "ptr"
    if decl.split()[0] in ("size_t", "uint64_t"):
        return "u64"
    if decl.split()[0] in ("int", "int32_t", "hsa_status_t"):
        return "int32"
    return decl


def test_binding_signatures_match_the_header(lib):
    protos = _prototypes()
    assert set(protos) == set(declared_symbols())
    checked = 0
    for name, (ret, params) in protos.items():
        fn = getattr(lib, name)
        if fn.argtypes is None:  # not bound in Python (C callers only)
            continue
        assert [_ctype_kind(t) for t in fn.argtypes] == [_decl_kind(p) for p in params], name
        assert _ctype_kind(fn.restype) == _decl_kind(ret), name
        checked += 1
    assert checked >= 10
