"""GPU parity of the n = 64 chunk phase on tcgen05 (k64_chunk_readout_tc,
opt-in with MRU_N64_TCGEN05=1: the chain's Q M and the determinant series'
M M and M^2 M as tcgen05.mma kind::tf32 into tensor memory, read back with
tcgen05.ld) against the fp64 oracle, on the cases the mma.sync kernel is
held to: tokens whose scale comes from the trace series, from the
near-identity LU and from the pivoted LU in one sequence; q query columns,
one U for every head or one per head, over chunk boundaries and a ragged
tail; permutation products read out through unit columns (exact); and the
full n = 64 readout workload on sampled sequences."""
from __future__ import annotations

import os

import numpy as np
import pytest

from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

from gpu_helpers import compare_readout, oracle_problem, run_fused, tol_for_problem, torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    mru.load()
    old = os.environ.get("MRU_N64_TCGEN05")
    os.environ["MRU_N64_TCGEN05"] = "1"          # read by the library at every call
    yield
    if old is None:
        os.environ.pop("MRU_N64_TCGEN05", None)
    else:
        os.environ["MRU_N64_TCGEN05"] = old


def small(mode, *, B=1, H=1, L=37, alpha=0.3 / 8, add_identity=1, seed=7):
    return gen.Workload("tc64", B=B, H=H, L=L, n=64, x_dtype="f32", mode=mode, alpha=float(alpha),
                        add_identity=add_identity, seed=seed)


def test_kernel_is_the_tcgen05_one():
    p = mru.problem_from_workload(gen.WORKLOADS["n64_detnorm_readout_b2h4l16384"])
    assert mru.kernel_names(p, True)[0] == "k64_chunk_readout_tc"


@pytest.mark.parametrize("chunk", [16, 32])
def test_series_and_lu_tokens_mixed(chunk):
    """Tokens t = 1 mod 3 (slice scaled by 6) fail the series' certificate and
    take the near-identity LU; tokens t = 2 mod 5 (scaled by 60) need the
    pivoted LU, on a row-major copy in the operand buffers."""
    w = small(gen.MODE_DETNORM, B=1, H=2, L=90, alpha=0.03 / 8, seed=660).with_(readout=True, snapshot_every=8)
    x = gen.make_x(w).reshape(w.B, w.L, w.H * 64 * 64).copy()
    x[:, 1::3] *= 6.0
    x[:, 2::5] *= 60.0
    u = gen.make_u(w)
    (o, snaps), st = run_fused(w, x, u=u, every=8, chunk=chunk)
    assert st == mru.OK
    e = compare_readout(w, x, o, snaps, u, 8)
    tol = tol_for_problem(w, chunk=chunk)
    assert e["o"]["count"] == w.B * w.L * w.H
    assert e["o"]["max"] <= tol and e["snap"]["max"] <= tol, e


@pytest.mark.parametrize("q,per_head,chunk", [(1, False, 16), (3, True, 16), (64, True, 0)])
def test_readout_query_columns(q, per_head, chunk):
    w = small(gen.MODE_DETNORM, B=2, H=3, L=53, seed=704 + q).with_(readout=True, snapshot_every=8)
    x = gen.make_x(w)
    rng = np.random.default_rng(705 + q)
    U = (rng.standard_normal((w.H, 64, q) if per_head else (64, q)) / 8.0).astype(np.float32)
    (o, snaps), st = run_fused(w, x, u=U, every=8, chunk=chunk)
    assert st == mru.OK
    e = compare_readout(w, x, o, snaps, U, 8)
    tol = tol_for_problem(w, chunk=chunk)
    assert e["o"]["count"] == w.B * w.L * w.H
    assert e["o"]["max"] <= tol and e["snap"]["max"] <= tol, e


def test_reshape_without_identity_and_unit_columns_exact():
    """Permutation matrices (reshape mode, no identity): every product and
    every tf32 operand is exact, so unit query columns read out picked
    columns of S_t bit for bit."""
    B, H, L, n = 2, 2, 37, 64
    w = small(gen.MODE_RESHAPE, B=B, H=H, L=L, alpha=1.0, add_identity=0).with_(readout=True)
    r = np.random.default_rng(711)
    x = np.zeros((B, L, H, n, n), np.float32)
    for b in range(B):
        for t in range(L):
            for h in range(H):
                x[b, t, h, np.arange(n), r.permutation(n)] = 1.0
    x = x.reshape(B, L, H * n * n)
    S_ref = oracle.scan(oracle_problem(w), x)
    cols = [[n - 1, 0, n // 2], [1, 1, n - 2]]
    U = np.stack([np.eye(n, dtype=np.float32)[:, c] for c in cols])
    (o, _), st = run_fused(w, x, u=U, chunk=16)
    assert st == mru.OK
    for h in range(H):
        assert np.array_equal(o[:, :, h].astype(np.float64), S_ref[:, :, h][..., cols[h]])


def test_full_readout_workload_sampled():
    w = gen.WORKLOADS["n64_detnorm_readout_b2h4l16384"]
    x = gen.make_x(w)
    u = gen.make_u(w)
    (o, snaps), st = run_fused(w, x, u=u, every=w.snapshot_every)
    assert st == mru.OK
    bh = np.array([0, w.B * w.H - 1])
    e = compare_readout(w, x, o, snaps, u, w.snapshot_every, bh=bh)
    tol = tol_for_problem(w)
    assert e["o"]["max"] <= tol and e["snap"]["max"] <= tol, e
    assert np.isfinite(o).all()
