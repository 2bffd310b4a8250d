"""mru_scan_fused_noalloc: the fused scan for callers that may not allocate
device memory (a plugin inside a framework that owns every device
allocation, a service that reserves its memory budget at start-up).  Its
scratch is the library's fixed device array instead of a caller workspace.

The GPU tests call it through the C-ABI twice in a row, on two different
inputs, and check each result against the fp64 oracle and against
mru_scan_fused (which uses a caller workspace) on the same input, within the
fp32 relative Frobenius gate of the other parity tests.  The second call
shows that nothing the first call left in the shared scratch leaks into the
next result.  One case is too large for the scratch at the library's chunk:
the entry point doubles the chunk, and its result equals mru_scan_fused's at
that chunk bit for bit.  This file is collected last on purpose.
"""
import numpy as np
import pytest

from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

from gpu_helpers import TOL_FP32, compare_S, to_device_x, torch


def _rel_frobenius(a, b):
    d = np.linalg.norm((a - b).reshape(-1, a.shape[-2] * a.shape[-1]), axis=1)
    r = np.linalg.norm(b.reshape(-1, b.shape[-2] * b.shape[-1]), axis=1)
    return float((d / r).max())


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    t = torch()
    if not t.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    w = gen.Workload("noalloc_n16", B=2, H=3, L=333, n=16, x_dtype="f32", mode=gen.MODE_DETNORM,
                     alpha=0.05 / 4, seed=9001)
    p = mru.problem_from_workload(w)
    assert mru.workspace_size(p) <= mru.NOALLOC_SCRATCH_BYTES
    stream = t.cuda.current_stream().cuda_stream
    for seed in (9001, 9002):                      # two calls in a row, different inputs
        x = to_device_x(gen.make_x(w, seed=seed))
        S_ref = mru.scan_fused_t(p, x)            # existing entry point, caller workspace
        S = t.full_like(S_ref, float("nan"))
        status = t.full((1,), 7, dtype=t.int32, device="cuda")
        rc = mru.scan_fused_noalloc(p, x.data_ptr(), None, None, S.data_ptr(), None, status.data_ptr(), stream)
        assert rc == mru.OK, mru.status_string(rc)
        t.cuda.synchronize()
        assert int(status.item()) == 0
        got, ref = S.cpu().numpy(), S_ref.cpu().numpy()
        assert np.isfinite(got).all()
        assert _rel_frobenius(got, ref) <= TOL_FP32
        e = compare_S(w, gen.make_x(w, seed=seed), got)            # and against the oracle directly
        assert e["count"] == w.B * w.L * w.H and e["max"] <= TOL_FP32, e

    # the readout form, twice as well (o_t = S_t u and snapshots)
    wr = w.with_(readout=True, snapshot_every=32)
    u = t.from_numpy(gen.make_u(wr)).cuda()
    for seed in (9003, 9004):
        x = to_device_x(gen.make_x(wr, seed=seed))
        o_ref, sn_ref = mru.scan_fused_t(p, x, u=u, snapshot_every=32)
        o = t.full_like(o_ref, float("nan"))
        sn = t.full_like(sn_ref, float("nan"))
        ro = mru.Readout(u.data_ptr(), 32, sn.data_ptr())
        rc = mru.scan_fused_noalloc(p, x.data_ptr(), None, ro, None, o.data_ptr(), None, stream)
        assert rc == mru.OK
        t.cuda.synchronize()
        o_h, or_h = o.cpu().numpy(), o_ref.cpu().numpy()
        rel_o = np.linalg.norm(o_h - or_h, axis=-1) / np.linalg.norm(or_h, axis=-1)
        assert float(rel_o.max()) <= TOL_FP32
        assert _rel_frobenius(sn.cpu().numpy(), sn_ref.cpu().numpy()) <= TOL_FP32


@pytest.mark.gpu
def test_noalloc_doubles_the_chunk_when_the_default_does_not_fit():
    """B4 H8 L4096, n = 16: at the library's chunk (16 tokens, 8192 chains)
    the call's own workspace is about 17 MB, above the 16 MiB scratch.  The
    entry point doubles the chunk until it fits, so its result equals
    mru_scan_fused run with that chunk exactly (same kernels, same chunking),
    and the oracle within the fp32 gate; twice in a row."""
    t = torch()
    if not t.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    w = gen.Workload("noalloc_big", B=4, H=8, L=4096, n=16, x_dtype="f32", mode=gen.MODE_DETNORM,
                     alpha=0.05 / 4, seed=9005)
    p = mru.problem_from_workload(w)
    c0 = mru.chosen_chunk(p)
    assert mru.workspace_size(mru.problem_from_workload(w, chunk=c0)) > mru.NOALLOC_SCRATCH_BYTES
    stream = t.cuda.current_stream().cuda_stream
    for seed in (9005, 9006):
        x_np = gen.make_x(w, seed=seed)
        x = to_device_x(x_np)
        S = t.full((w.B, w.L, w.H, 16, 16), float("nan"), device="cuda")
        status = t.full((1,), 7, dtype=t.int32, device="cuda")
        rc = mru.scan_fused_noalloc(p, x.data_ptr(), None, None, S.data_ptr(), None, status.data_ptr(), stream)
        assert rc == mru.OK, mru.status_string(rc)
        t.cuda.synchronize()
        assert int(status.item()) == 0
        got = S.cpu().numpy()
        used = None
        for c in (2 * c0, 4 * c0, 8 * c0):
            ref = mru.scan_fused_t(mru.problem_from_workload(w, chunk=c), x).cpu().numpy()
            if np.array_equal(got, ref):
                used = c
                break
        assert used is not None, "no doubled chunk reproduces the no-alloc result"
        e = compare_S(w, x_np, got)
        assert e["count"] == w.B * w.L * w.H and e["max"] <= TOL_FP32, e


def test_noalloc_rejects_problems_beyond_the_scratch():
    """Host-side: a problem whose workspace cannot fit the fixed scratch even
    with one chunk per sequence is refused before anything is launched."""
    mru.load()
    p = mru.problem(64, 64, 1, 64, mode=gen.MODE_DETNORM, alpha=0.01)
    assert mru.workspace_size(p) > mru.NOALLOC_SCRATCH_BYTES
    fake = 1 << 20
    rc = mru.scan_fused_noalloc(p, fake, None, None, 2 * fake, None, None, 0)
    assert rc == mru.ERR_WORKSPACE
    bad = mru.problem(1, 1, 8, 12)
    assert mru.scan_fused_noalloc(bad, fake, None, None, 2 * fake, None, None, 0) == mru.ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [gen.MODE_CAYLEY, gen.MODE_EXPM])
def test_orthogonal_maps_form_F_once_or_twice_alike(mode):
    """At n = 16 the Cayley map and the exponential keep every token's
    F = X - I in the workspace when it fits (the reduce pass writes it, the
    apply pass reads it); in the fixed scratch it does not fit here (32 MiB
    of F), so the passes form F twice.  Both form it with the same code on
    the same slice: the states agree bit for bit, and with the oracle."""
    t = torch()
    if not t.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    w = gen.Workload("noalloc_orth", B=4, H=4, L=2048, n=16, x_dtype="f32", mode=mode, alpha=0.0125, seed=9101)
    p = mru.problem_from_workload(w, chunk=32)
    assert w.B * w.L * w.H * 16 * 16 * 4 > mru.NOALLOC_SCRATCH_BYTES
    x_np = gen.make_x(w)
    x = to_device_x(x_np)
    S_ref = mru.scan_fused_t(p, x)                 # caller workspace: F kept
    S = t.full_like(S_ref, float("nan"))
    status = t.full((1,), 7, dtype=t.int32, device="cuda")
    stream = t.cuda.current_stream().cuda_stream
    rc = mru.scan_fused_noalloc(p, x.data_ptr(), None, None, S.data_ptr(), None, status.data_ptr(), stream)
    assert rc == mru.OK, mru.status_string(rc)
    t.cuda.synchronize()
    assert int(status.item()) == 0
    got, ref = S.cpu().numpy(), S_ref.cpu().numpy()
    assert np.array_equal(got, ref)
    bh = np.array([0, 7, 15])
    e = compare_S(w, x_np, got, bh=bh)
    assert e["max"] <= TOL_FP32, e
