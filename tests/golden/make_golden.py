"""Write the oracle regression fixture ``oracle_tiny.txt``.

The source pages print no worked example with numbers, so no fixture here holds
page values.  This fixture is a snapshot of the fp64 oracle on one tiny seeded
input; it exists so that any later change to the oracle's arithmetic shows up
as a failing test and has to be justified.  Only ``oracle`` and the seeded
generator are called.

Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from chunked_hierarchical_sparse_b200 import synth  # noqa: E402

WL = synth.Workload("golden", 1, 40, 2, 1, 4, 8, 2, "bf16", "iid", "fwd", 4242)


def compute():
    x = synth.make_inputs(WL)
    kbar = oracle.pool(x["k"], WL.S)
    o, lse, idx, w = oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, WL.S, WL.K)
    return kbar, o, lse, idx, w


def main():
    kbar, o, lse, idx, w = compute()
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.txt")
    with open(path, "w") as f:
        f.write("# oracle snapshot, workload B=1 L=40 h_q=2 h_kv=1 d=4 S=8 K=2 bf16 seed=4242\n")
        f.write("# written by tests/golden/make_golden.py (calls only oracle/ and the generator)\n")
        for name, a in (("kbar", kbar), ("o", o), ("lse", lse), ("idx", idx), ("w", w)):
            f.write(f"{name} {' '.join(str(n) for n in a.shape)}\n")
            f.write(" ".join(repr(float(v)) if a.dtype.kind == "f" else str(int(v))
                             for v in a.ravel()) + "\n")


if __name__ == "__main__":
    main()
