"""Writes the regression fixtures in this folder.  Calls only the oracle and
the seeded input generator; run from the repository root:

    python tests/golden/make_fixtures.py

n4_reshape_l1024_samples.txt: sampled states S_t of the small reshape
workload (n = 4, L = 1024, X_t = I + 0.05 * reshape(x_t), x ~ N(0, 1) from
seed 1001), the definition being the cumulative product of the lifted token
matrices ("MRU Update: An independent developer's alternative to Attention is
now running successfully", section "What MRU Actually Does").
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from linear_rnn_scan_b200 import inputs as gen  # noqa: E402

SAMPLE_T = [1, 2, 3, 10, 100, 512, 1023, 1024]   # 1-based positions


def main():
    w = gen.WORKLOADS["n4_reshape_l1024"]
    x = gen.make_x(w)
    p = oracle.make_problem(w.B, w.H, w.L, w.n, mode=w.mode, alpha=w.alpha, add_identity=1)
    S = oracle.scan(p, x)
    path = os.path.join(HERE, "n4_reshape_l1024_samples.txt")
    with open(path, "w") as f:
        f.write("# S_t (1-based t) of the n=4 reshape workload, seed 1001, alpha=float32(0.05)\n")
        f.write("# written by tests/golden/make_fixtures.py from the fp64 oracle\n")
        f.write("# t  then the 16 entries of S_t, row-major\n")
        for t in SAMPLE_T:
            vals = " ".join(repr(float(v)) for v in S[0, t - 1, 0].ravel())
            f.write(f"{t} {vals}\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
