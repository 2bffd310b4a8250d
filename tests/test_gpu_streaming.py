"""Streaming use of the scan: a sequence processed in segments, each started
from the previous segment's last state (S0), and token-by-token decoding
(L = 1 calls), both against the oracle's whole-sequence result.  S0 enters
on the left: S_t = S0 X_1 ... X_t, so segment two started from S_{t0} of
segment one continues the same product."""
from __future__ import annotations

import numpy as np
import pytest

from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

from gpu_helpers import compare_readout, compare_S, run_fused, tol_for_problem, torch

pytestmark = pytest.mark.gpu

CASES = [(4, gen.MODE_RESHAPE, "f32", 0.05), (16, gen.MODE_DETNORM, "f32", 0.0125),
         (32, gen.MODE_LDU, "bf16", None), (64, gen.MODE_DETNORM, "f32", 0.00375)]


def _workload(n, mode, dtype, alpha, B, H, L, seed):
    kw = {} if alpha is None else {"alpha": alpha}
    return gen.Workload(f"s{n}", B=B, H=H, L=L, n=n, x_dtype=dtype, mode=mode, seed=seed, **kw)


def _segment(w, x, t0, t1):
    """The workload and input of tokens [t0, t1)."""
    ws = gen.Workload(w.name, B=w.B, H=w.H, L=t1 - t0, n=w.n, x_dtype=w.x_dtype, mode=w.mode, alpha=w.alpha,
                      add_identity=w.add_identity, ldu_offdiag=w.ldu_offdiag, ldu_diag=w.ldu_diag, seed=w.seed)
    return ws, np.ascontiguousarray(x[:, t0:t1])


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch().cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    mru.load()
    yield


@pytest.mark.parametrize("n,mode,dtype,alpha", CASES)
def test_segmented_resume_matches_whole_sequence(n, mode, dtype, alpha):
    w = _workload(n, mode, dtype, alpha, B=2, H=2, L=301, seed=1200 + n)
    x = gen.make_x(w)
    cuts = [0, 137, 200, 301]
    parts, S0 = [], None
    for t0, t1 in zip(cuts[:-1], cuts[1:]):
        ws, xs = _segment(w, x, t0, t1)
        S, st = run_fused(ws, xs, S0=S0)
        assert st == mru.OK
        parts.append(S)
        S0 = np.ascontiguousarray(S[:, -1])                # [B, H, n, n]: the segment's last state
    S_cat = np.concatenate(parts, axis=1)
    e = compare_S(w, x, S_cat)
    assert e["count"] == w.B * w.H * w.L
    assert e["max"] <= tol_for_problem(w), e
    S_whole, st = run_fused(w, x)
    assert st == mru.OK
    rel = np.linalg.norm((S_cat - S_whole).reshape(-1, n * n), axis=1) / \
        np.linalg.norm(S_whole.reshape(-1, n * n), axis=1)
    assert rel.max() <= 2 * tol_for_problem(w)


@pytest.mark.parametrize("n,mode,dtype,alpha", CASES)
def test_token_by_token_decode(n, mode, dtype, alpha):
    w = _workload(n, mode, dtype, alpha, B=1, H=3, L=12, seed=1300 + n)
    x = gen.make_x(w)
    S0, steps = None, []
    for t in range(w.L):
        ws, xs = _segment(w, x, t, t + 1)
        S, st = run_fused(ws, xs, S0=S0)
        assert st == mru.OK
        steps.append(S)
        S0 = np.ascontiguousarray(S[:, -1])
    e = compare_S(w, x, np.concatenate(steps, axis=1))
    assert e["count"] == w.B * w.H * w.L
    assert e["max"] <= tol_for_problem(w), e


@pytest.mark.parametrize("n", [4, 8, 16, 32, 64])
def test_single_chunk_readout_from_S0(n):
    """A segment no longer than one chunk runs as one launch started from S0
    (the decode path); with the readout its outputs are final there too:
    o_t = S_t U with S_t = S0 X_1 ... X_t, and the snapshots."""
    w = _workload(n, gen.MODE_DETNORM, "f32", 0.3 / np.sqrt(n), B=2, H=3, L=12, seed=1400 + n)
    w = w.with_(readout=True, snapshot_every=4)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=1401)
    U = (np.random.default_rng(1402).standard_normal((w.H, n, 3)) / np.sqrt(n)).astype(np.float32)
    p = mru.problem_from_workload(w, chunk=16)
    assert mru.launch_count(p, True) == 1 and mru.kernel_names(p, True) == ["k_chunk_prefix"]
    (o, snaps), st = run_fused(w, x, S0=S0, u=U, every=4, chunk=16)
    assert st == mru.OK
    e = compare_readout(w, x, o, snaps, U, 4, S0=S0)
    assert e["o"]["max"] <= tol_for_problem(w, chunk=16) and e["snap"]["max"] <= tol_for_problem(w, chunk=16), e
