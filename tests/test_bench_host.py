"""Host-side logic of bench.py that needs no GPU: the source key that ties a stored
DRAM-traffic figure to the kernel code it was measured on, and the reference arm (the
oracle timed on the host cores), whose JSON line must carry the contract's keys."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_source_key_ignores_comments_but_not_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = "int f(int x) {\n    return x + 1;  // add one\n}\n"
    variants = {
        "a.cu": base,
        "b.cu": "/* header\n   block */\n" + base.replace("// add one", "// plus one") + "\n\n",
        "c.cu": base.replace("x + 1", "x + 2"),
    }
    for n, src in variants.items():
        (tmp_path / n).write_text(src)
    ha, hb, hc = (bench.source_hash([n]) for n in ("a.cu", "b.cu", "c.cu"))
    assert ha == hb
    assert ha != hc
    # the key covers every file listed, in order
    assert bench.source_hash(["a.cu", "c.cu"]) != bench.source_hash(["c.cu", "a.cu"])


def test_traffic_record_is_dropped_when_the_code_changes(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "chunked_hierarchical_sparse_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in ("k.cu", "hsa_internal.cuh", "sm100.cuh"):
        (csrc / n).write_text(f"int {n.split('.')[0]}_v = 1;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rel = "chunked_hierarchical_sparse_b200/csrc/k.cu"
    key = bench.source_hash([rel, "chunked_hierarchical_sparse_b200/csrc/hsa_internal.cuh",
                             "chunked_hierarchical_sparse_b200/csrc/sm100.cuh"])
    (tmp_path / "profiles" / "traffic.txt").write_text(f"# header\nk.cu source={key} bytes_per_launch=12345\n")
    assert bench.read_traffic(rel) == 12345
    (csrc / "k.cu").write_text("int k_v = 1;  // a comment changes nothing\n")
    assert bench.read_traffic(rel) == 12345
    (csrc / "k.cu").write_text("int k_v = 2;\n")
    assert bench.read_traffic(rel) is None


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "fwd16k",
                        "--steps", "1", "--warmup", "0", "--ref-rows", "16"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "fwd16k"
