"""Full-size workloads, in the launch configuration bench.py times (library
chunk choice, fused entry point), against the fp64 oracle.  The oracle
recomputes each listed (b, h) sequence serially over the whole length and
compares every state (or every readout vector and snapshot) on the way; the
largest workloads compare a spread subset of their sequences."""
from __future__ import annotations

import numpy as np
import pytest

from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

from gpu_helpers import compare_readout, compare_S, run_fused, tol_for_problem, torch

pytestmark = pytest.mark.gpu

# sequences compared per workload (None = all)
SAMPLE = {"n4_reshape_l1024": None, "n16_detnorm_b8h8l4096": None, "n32_ldu_bf16_b4h16l8192": 16,
          "n16_detnorm_b1h8l262144": None, "n64_detnorm_readout_b2h4l16384": 2,
          "n64_detnorm_readout_q8_b2h4l16384": 2, "n16_cayley_b8h8l4096": 8, "n16_expm_b8h8l4096": 8}


@pytest.mark.parametrize("name", gen.WORKLOAD_ORDER)
def test_full_workload_against_oracle(name):
    t = torch()
    if not t.cuda.is_available():
        pytest.fail("CUDA device required")
    w = gen.WORKLOADS[name]
    x = gen.make_x(w)
    nbh = w.B * w.H
    k = SAMPLE[name]
    bh = None if k is None else np.unique(np.linspace(0, nbh - 1, k).round().astype(np.int64))
    tol = tol_for_problem(w)
    if w.readout:
        u = gen.make_u(w)
        (o, snaps), st = run_fused(w, x, u=u, every=w.snapshot_every)
        assert st == mru.OK
        e = compare_readout(w, x, o, snaps, u, w.snapshot_every, bh=bh)
        print(name, e)
        assert e["o"]["max"] <= tol and e["snap"]["max"] <= tol, e
        assert np.isfinite(o).all()
    else:
        S, st = run_fused(w, x)
        assert st == mru.OK
        e = compare_S(w, x, S, bh=bh)
        print(name, e)
        assert e["count"] == (nbh if bh is None else len(bh)) * w.L
        assert e["max"] <= tol, e
