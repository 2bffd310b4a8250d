"""The host-buffer entry point (mru_scan_fused_host): uploads, scans and
downloads pipelined over pieces of the problem on three streams.  Cut along
the batch it must reproduce mru_scan_fused bit for bit (every sequence runs
the same kernels with the same chunks); cut along the sequence (B = 1) each
piece starts from the previous piece's last state, which stays within the
oracle's gate."""
from __future__ import annotations

import numpy as np
import pytest

from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

from gpu_helpers import compare_readout, compare_S, run_fused, to_device_x, tol_for_problem, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch().cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    mru.load()
    yield


def _host_x(x_np):
    t = torch()
    if x_np.dtype == np.uint16:
        return t.from_numpy(x_np.view(np.int16)).view(t.bfloat16).pin_memory()
    return t.from_numpy(np.ascontiguousarray(x_np)).pin_memory()


def _run_host(w, x_np, pieces, *, S0=None, u=None, every=0):
    t = torch()
    p = mru.problem_from_workload(w)
    xh = _host_x(x_np)
    xd = t.empty(xh.shape, dtype=xh.dtype, device="cuda")
    ws = mru.workspace_t(p)
    S0_t = None if S0 is None else t.from_numpy(np.ascontiguousarray(S0, np.float32)).cuda()
    if u is None:
        shape, ro, snaps_d, snaps_h = (w.B, w.L, w.H, w.n, w.n), None, None, None
    else:
        u_t = t.from_numpy(np.ascontiguousarray(u, np.float32)).cuda()
        q, per_head = (1, 0) if u.ndim == 1 else (u.shape[-1], int(u.ndim == 3))
        shape = (w.B, w.L, w.H, w.n) + ((q,) if u.ndim > 1 else ())
        snaps_d = t.empty((w.B, w.L // every, w.H, w.n, w.n), dtype=t.float32, device="cuda") if every else None
        snaps_h = t.empty(snaps_d.shape, dtype=t.float32, pin_memory=True) if every else None
        ro = mru.Readout(u_t.data_ptr(), every, snaps_d.data_ptr() if every else None, q, per_head)
    out_h = t.full(shape, float("nan"), dtype=t.float32, pin_memory=True)
    out_d = t.empty(shape, dtype=t.float32, device="cuda")
    sc, si, so = t.cuda.current_stream(), t.cuda.Stream(), t.cuda.Stream()
    rc = mru.scan_fused_host(p, xh.data_ptr(), None if S0_t is None else S0_t.data_ptr(), ro, out_h.data_ptr(),
                             None if snaps_h is None else snaps_h.data_ptr(), xd.data_ptr(), out_d.data_ptr(),
                             ws.data_ptr(), ws.numel(), pieces, sc.cuda_stream, si.cuda_stream, so.cuda_stream)
    assert rc == mru.OK
    sc.synchronize()
    st = mru.last_device_status(ws.data_ptr(), sc.cuda_stream)
    return out_h.numpy().copy(), (None if snaps_h is None else snaps_h.numpy().copy()), st


@pytest.mark.parametrize("n,mode,dtype", [(16, gen.MODE_DETNORM, "f32"), (32, gen.MODE_LDU, "bf16"),
                                          (8, gen.MODE_RESHAPE, "f32"), (64, gen.MODE_CAYLEY, "f32")])
@pytest.mark.parametrize("pieces", [0, 2, 3, 16])
def test_along_batch_matches_device_call_exactly(n, mode, dtype, pieces):
    w = gen.Workload(f"h{n}", B=5, H=2, L=70, n=n, x_dtype=dtype, mode=mode, alpha=0.3 / np.sqrt(n), seed=1500 + n)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=1501)
    S_dev, st = run_fused(w, x, S0=S0)
    assert st == mru.OK
    S_host, _, st = _run_host(w, x, pieces, S0=S0)
    assert st == mru.OK
    assert np.array_equal(S_host, S_dev)
    e = compare_S(w, x, S_host, S0=S0)                 # and against the oracle directly
    assert e["count"] == w.B * w.H * w.L and e["max"] <= tol_for_problem(w), e


@pytest.mark.parametrize("n,mode", [(16, gen.MODE_DETNORM), (4, gen.MODE_RESHAPE), (32, gen.MODE_EXPM)])
def test_along_sequence_within_gate(n, mode):
    w = gen.Workload(f"l{n}", B=1, H=3, L=301, n=n, x_dtype="f32", mode=mode, alpha=0.3 / np.sqrt(n),
                     seed=1600 + n)
    x = gen.make_x(w)
    S_host, _, st = _run_host(w, x, 4)
    assert st == mru.OK and np.isfinite(S_host).all()
    e = compare_S(w, x, S_host)
    assert e["count"] == w.H * w.L and e["max"] <= tol_for_problem(w), e


def test_readout_along_batch_matches_device_call_exactly():
    w = gen.Workload("r64", B=3, H=2, L=512, n=64, x_dtype="f32", mode=gen.MODE_DETNORM, alpha=0.03 / 8,
                     readout=True, snapshot_every=128, math="tf32", seed=1700)
    x = gen.make_x(w)
    U = (np.random.default_rng(1701).standard_normal((w.H, 64, 2)) / 8).astype(np.float32)
    (o_dev, sn_dev), st = run_fused(w, x, u=U, every=128)
    assert st == mru.OK
    o_host, sn_host, st = _run_host(w, x, 0, u=U, every=128)
    assert st == mru.OK
    assert np.array_equal(o_host, o_dev) and np.array_equal(sn_host, sn_dev)
    e = compare_readout(w, x, o_host, sn_host, U, 128)  # and against the oracle directly
    tol = tol_for_problem(w)
    assert e["o"]["max"] <= tol and e["snap"]["max"] <= tol, e


def test_single_batch_readout_is_one_piece():
    w = gen.Workload("r1", B=1, H=2, L=90, n=16, x_dtype="f32", mode=gen.MODE_DETNORM, alpha=0.05,
                     readout=True, seed=1800)
    x = gen.make_x(w)
    u = gen.make_u(w)
    (o_dev, _), st = run_fused(w, x, u=u)
    o_host, _, st2 = _run_host(w, x, 8, u=u)
    assert st == mru.OK and st2 == mru.OK and np.array_equal(o_host, o_dev)


def test_singular_status_survives_later_pieces():
    """A singular matrix in the first piece is still reported after the last."""
    w = gen.Workload("sg", B=4, H=1, L=20, n=8, x_dtype="f32", mode=gen.MODE_DETNORM, alpha=1.0,
                     add_identity=0, seed=1900)
    x = gen.make_x(w)
    x[0, 3] = 0.0
    _, _, st = _run_host(w, x, 4)
    assert st == mru.ERR_SINGULAR
