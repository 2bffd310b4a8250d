"""Regression fixtures under tests/golden/ (written by make_fixtures.py from
the oracle): the oracle must keep reproducing them."""
import os

import numpy as np

from linear_rnn_scan_b200 import inputs as gen

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_samples(name):
    rows = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            rows[int(parts[0])] = np.array([float(v) for v in parts[1:]])
    return rows


def test_n4_fixture_reproduced(oracle_mod):
    w = gen.WORKLOADS["n4_reshape_l1024"]
    x = gen.make_x(w)
    p = oracle_mod.make_problem(w.B, w.H, w.L, w.n, mode=w.mode, alpha=w.alpha, add_identity=1)
    S = oracle_mod.scan(p, x)
    rows = load_samples("n4_reshape_l1024_samples.txt")
    assert len(rows) == 8
    for t, ref in rows.items():
        np.testing.assert_allclose(S[0, t - 1, 0].ravel(), ref, rtol=1e-15, atol=1e-300)
