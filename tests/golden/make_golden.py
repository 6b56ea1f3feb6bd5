"""Writes tests/golden/tiny_oracle.txt from the CPU oracle alone.

The pages print no worked example for the state update, so the only stored
expected values in this repository are the oracle's own results on the tiny
seeded workload (B=1, Hk=Hv=1, dk=dv=16, eight chained single-token calls
through a 4-slot pool).  They serve as a regression fixture: the CPU suite
checks that the oracle still reproduces them, and the GPU suite compares the
CUDA path against them.  Run:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from hybrid_linear_attention_step_b200 import workloads  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.txt")


def compute():
    w = workloads.tiny(0)
    pool = w.pool.copy()
    outs = []
    for s in w.steps:
        out = np.zeros((s.B, s.T, s.Hv, s.dv), np.float32)
        oracle.decode_step(pool, s.src_idx, s.dst_idx, s.q, s.k, s.v, s.alpha, s.beta, out)
        outs.append(out.reshape(-1))
    return np.stack(outs), pool


def main():
    outs, pool = compute()
    with open(OUT, "w") as f:
        f.write("# tiny workload (seed 0): oracle outputs of 8 chained T=1 calls, then the final pool.\n")
        f.write("# written by tests/golden/make_golden.py (oracle only); float32 values as %.9g\n")
        f.write(f"outputs {outs.shape[0]} {outs.shape[1]}\n")
        for row in outs:
            f.write(" ".join(f"{x:.9g}" for x in row) + "\n")
        p = pool.reshape(pool.shape[0], -1)
        f.write(f"pool {p.shape[0]} {p.shape[1]} shape {' '.join(map(str, pool.shape))}\n")
        for row in p:
            f.write(" ".join(f"{x:.9g}" for x in row) + "\n")


def load(path=OUT):
    with open(path) as f:
        lines = [ln for ln in f if not ln.startswith("#")]
    n, m = map(int, lines[0].split()[1:3])
    outs = np.array([[float(x) for x in ln.split()] for ln in lines[1:1 + n]], np.float32)
    hdr = lines[1 + n].split()
    shape = tuple(int(x) for x in hdr[4:])
    rows = lines[2 + n:2 + n + int(hdr[1])]
    pool = np.array([[float(x) for x in ln.split()] for ln in rows], np.float32).reshape(shape)
    return outs, pool


if __name__ == "__main__":
    main()
