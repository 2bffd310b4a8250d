"""GPU backward (mru_scan_backward) against the oracle's fp64 backward on the
same inputs and upstream gradients: every n, every construction mode, f32
and bf16 inputs, with S0 and several chunks (ragged last chunk), plus the
full-size default workload on sampled sequences."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

from gpu_helpers import oracle_problem, to_device_x, torch

pytestmark = pytest.mark.gpu

# Relative Frobenius gate per token-head for the fp32 backward (max over every
# compared (b, t, h)): the forward's fp32 gate.  Measured on B200: below 1e-6
# near the identity; 1.8e-5 for the determinant-corrected mode without the
# identity, whose chain rule subtracts <dX, Xr> Xr^-T / n from dX.
TOL_BWD = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch().cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    mru.load()
    yield


def _rel(a, b, axis):
    num = np.sqrt(np.sum((a - b) ** 2, axis=axis))
    den = np.sqrt(np.sum(b ** 2, axis=axis))
    return num / np.maximum(den, 1e-300)


def _run(w, x, S0, dS, chunk):
    t = torch()
    p = mru.problem_from_workload(w, chunk=chunk)
    xd = to_device_x(x)
    S0d = t.from_numpy(np.ascontiguousarray(S0, np.float32)).cuda()
    S = mru.scan_fused_t(p, xd, S0=S0d)
    dx, dS0, ws = mru.scan_backward_t(p, xd, S, t.from_numpy(np.ascontiguousarray(dS, np.float32)).cuda(), S0=S0d)
    st = mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream)
    return dx.cpu().numpy().astype(np.float64), dS0.cpu().numpy().astype(np.float64), st


CASES = []
for n in (4, 8, 16, 32, 64):
    CASES += [(n, gen.MODE_RESHAPE, 1, "f32"), (n, gen.MODE_DETNORM, 1, "f32"), (n, gen.MODE_LDU, 1, "bf16")]
CASES += [(16, gen.MODE_RESHAPE, 0, "f32"), (8, gen.MODE_DETNORM, 0, "f32"), (16, gen.MODE_LDU, 1, "f32")]
for n in (4, 16, 64):
    CASES += [(n, gen.MODE_CAYLEY, 1, "f32"), (n, gen.MODE_EXPM, 1, "f32")]
# orthogonal modes with the larger alpha (the exponential squares twice)
CASES += [(8, gen.MODE_CAYLEY, 0, "f32"), (8, gen.MODE_EXPM, 0, "bf16"), (32, gen.MODE_EXPM, 0, "f32")]


@pytest.mark.parametrize("n,mode,add_identity,dtype", CASES)
def test_backward_small(n, mode, add_identity, dtype):
    """fp32 arithmetic (fp64 only for the right-to-left scan of the chunk
    gradients); the measured errors are in the assertion message."""
    rng = np.random.default_rng(500 + 10 * n + mode + 3 * add_identity)
    if mode == gen.MODE_LDU:
        alpha = 1.0
    elif add_identity:
        alpha = 0.3 / np.sqrt(n)
    else:
        alpha = 1.0 / np.sqrt(n)
    L = 37 if add_identity else 13
    w = gen.Workload(f"b{n}", B=2, H=2, L=L, n=n, x_dtype=dtype, mode=mode, alpha=float(alpha),
                     add_identity=add_identity, seed=600 + n)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=601)
    dS = rng.standard_normal((w.B, w.L, w.H, n, n)).astype(np.float32)
    dx, dS0, st = _run(w, x, S0, dS, chunk=8)
    assert st == mru.OK
    dx_o, dS0_o = oracle.backward(oracle_problem(w), x, dS.astype(np.float64), S0=S0.astype(np.float64))
    e_dx = _rel(dx.reshape(w.B, w.L, w.H, n * n), dx_o.reshape(w.B, w.L, w.H, n * n), axis=-1)
    e_s0 = _rel(dS0.reshape(w.B, w.H, n * n), dS0_o.reshape(w.B, w.H, n * n), axis=-1)
    assert e_dx.max() <= TOL_BWD and e_s0.max() <= TOL_BWD, (e_dx.max(), np.median(e_dx), e_s0.max())


@pytest.mark.parametrize("chunk", [1, 5, 16, 64])
def test_backward_chunk_sizes_agree(chunk):
    w = gen.Workload("bc", B=1, H=2, L=50, n=16, x_dtype="f32", mode=gen.MODE_DETNORM, alpha=0.05 / 4, seed=77)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=78)
    dS = np.random.default_rng(79).standard_normal((w.B, w.L, w.H, 16, 16)).astype(np.float32)
    dx, dS0, st = _run(w, x, S0, dS, chunk=chunk)
    assert st == mru.OK
    dx_o, dS0_o = oracle.backward(oracle_problem(w), x, dS.astype(np.float64), S0=S0.astype(np.float64))
    e = _rel(dx.reshape(w.B, w.L, w.H, 256), dx_o.reshape(w.B, w.L, w.H, 256), axis=-1)
    assert e.max() <= TOL_BWD, e.max()


def test_backward_default_workload_sampled():
    """The bench's default workload (B8 H8 L4096, n = 16, determinant
    corrected) end to end; the oracle recomputes two sequences."""
    t = torch()
    w = gen.WORKLOADS["n16_detnorm_b8h8l4096"]
    x = gen.make_x(w)
    rng = np.random.default_rng(5)
    dS = rng.standard_normal((w.B, w.L, w.H, 16, 16)).astype(np.float32)
    p = mru.problem_from_workload(w)
    xd = to_device_x(x)
    S = mru.scan_fused_t(p, xd)
    dx, _, ws = mru.scan_backward_t(p, xd, S, t.from_numpy(dS).cuda())
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx = dx.cpu().numpy().astype(np.float64).reshape(w.B, w.L, w.H, 256)
    for b, h in [(0, 0), (7, 5)]:
        ws1 = gen.Workload("one", B=1, H=1, L=w.L, n=16, x_dtype="f32", mode=w.mode, alpha=w.alpha, seed=0)
        x1 = np.ascontiguousarray(x.reshape(w.B, w.L, w.H, 256)[b:b + 1, :, h])
        dS1 = dS[b:b + 1, :, h:h + 1].astype(np.float64)
        dx_o, _ = oracle.backward(oracle_problem(ws1), x1, dS1)
        e = _rel(dx[b, :, h], dx_o.reshape(w.L, 256), axis=-1)
        assert e.max() <= TOL_BWD, (b, h, e.max(), np.median(e))


@pytest.mark.parametrize("alpha", [0.002, 0.0125, 0.04, 0.055, 0.1])
def test_backward_n16_inverse_regimes(alpha):
    """n = 16 determinant-corrected backward on the tensor cores: the Xr^-T of
    its chain rule takes 1 to 6 Newton-Schulz steps as |alpha M|_F grows, and
    Gauss-Jordan with pivoting beyond (alpha 0.1: |alpha M|_F near 1.6).  (At
    alpha 0.2 some I + alpha M are ill-conditioned enough that the fp32
    inverse alone moves dx by about 1e-4, on any path.)"""
    rng = np.random.default_rng(int(alpha * 1e4))
    w = gen.Workload("ns", B=1, H=2, L=37, n=16, x_dtype="f32", mode=gen.MODE_DETNORM, alpha=alpha, seed=610)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=611)
    dS = rng.standard_normal((w.B, w.L, w.H, 16, 16)).astype(np.float32)
    dx, dS0, st = _run(w, x, S0, dS, chunk=8)
    assert st == mru.OK
    dx_o, dS0_o = oracle.backward(oracle_problem(w), x, dS.astype(np.float64), S0=S0.astype(np.float64))
    e_dx = _rel(dx.reshape(w.B, w.L, w.H, 256), dx_o.reshape(w.B, w.L, w.H, 256), axis=-1)
    e_s0 = _rel(dS0.reshape(w.B, w.H, 256), dS0_o.reshape(w.B, w.H, 256), axis=-1)
    assert e_dx.max() <= TOL_BWD and e_s0.max() <= TOL_BWD, (e_dx.max(), np.median(e_dx), e_s0.max())


@pytest.mark.parametrize("chunk", [1, 3, 8, 16])
@pytest.mark.parametrize("with_s0", [False, True])
def test_backward_n32_ldu_tensor_cores(chunk, with_s0):
    """The n = 32 LDU backward on the tensor cores (bf16 embeddings): chunks
    of 1, 3, 8 and 16 tokens over L = 45 (a ragged last chunk), with and
    without S0 (then the first token's S_{-1} is I and no dS0 is asked)."""
    t = torch()
    n = 32
    w = gen.Workload("b32", B=2, H=2, L=45, n=n, x_dtype="bf16", mode=gen.MODE_LDU, alpha=1.0, seed=620)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=621) if with_s0 else None
    dS = np.random.default_rng(622 + chunk).standard_normal((w.B, w.L, w.H, n, n)).astype(np.float32)
    p = mru.problem_from_workload(w, chunk=chunk)
    xd = to_device_x(x)
    S0d = None if S0 is None else t.from_numpy(np.ascontiguousarray(S0, np.float32)).cuda()
    S = mru.scan_fused_t(p, xd, S0=S0d)
    dx, dS0, ws = mru.scan_backward_t(p, xd, S, t.from_numpy(dS).cuda(), S0=S0d)
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx_o, dS0_o = oracle.backward(oracle_problem(w), x, dS.astype(np.float64),
                                  S0=None if S0 is None else S0.astype(np.float64))
    dx = dx.cpu().numpy().astype(np.float64)
    e_dx = _rel(dx.reshape(w.B, w.L, w.H, n * n), dx_o.reshape(w.B, w.L, w.H, n * n), axis=-1)
    assert e_dx.max() <= TOL_BWD, (e_dx.max(), np.median(e_dx))
    if with_s0:
        e_s0 = _rel(dS0.cpu().numpy().astype(np.float64).reshape(w.B, w.H, n * n), dS0_o.reshape(w.B, w.H, n * n),
                    axis=-1)
        assert e_s0.max() <= TOL_BWD, e_s0.max()


def test_backward_n32_ldu_workload_sampled():
    """The n = 32 LDU workload (B4 H16 L8192, bf16) end to end on the tensor
    cores; the oracle recomputes two sequences."""
    t = torch()
    w = gen.WORKLOADS["n32_ldu_bf16_b4h16l8192"]
    n = w.n
    x = gen.make_x(w)
    dS = np.random.default_rng(6).standard_normal((w.B, w.L, w.H, n, n)).astype(np.float32)
    p = mru.problem_from_workload(w)
    xd = to_device_x(x)
    S = mru.scan_fused_t(p, xd)
    dx, _, ws = mru.scan_backward_t(p, xd, S, t.from_numpy(dS).cuda())
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx = dx.cpu().numpy().astype(np.float64).reshape(w.B, w.L, w.H, n * n)
    for b, h in [(0, 0), (3, 11)]:
        w1 = gen.Workload("one", B=1, H=1, L=w.L, n=n, x_dtype=w.x_dtype, mode=w.mode, alpha=w.alpha,
                          ldu_offdiag=w.ldu_offdiag, ldu_diag=w.ldu_diag, seed=0)
        x1 = np.ascontiguousarray(x.reshape(w.B, w.L, w.H, n * n)[b:b + 1, :, h])
        dS1 = dS[b:b + 1, :, h:h + 1].astype(np.float64)
        dx_o, _ = oracle.backward(oracle_problem(w1), x1, dS1)
        e = _rel(dx[b, :, h], dx_o.reshape(w.L, n * n), axis=-1)
        assert e.max() <= TOL_BWD, (b, h, e.max(), np.median(e))


READOUT_CASES = [  # n, mode, x_dtype, ushape, every, with_s0
    (4, gen.MODE_RESHAPE, "f32", "vector", 8, False),
    (16, gen.MODE_DETNORM, "f32", "shared", 16, True),
    (16, gen.MODE_CAYLEY, "f32", "per_head", 0, False),
    (32, gen.MODE_LDU, "bf16", "vector", 16, True),
    (64, gen.MODE_DETNORM, "f32", "per_head", 8, False),
]


@pytest.mark.parametrize("n,mode,x_dtype,ushape,every,with_s0", READOUT_CASES)
def test_backward_readout_against_oracle(n, mode, x_dtype, ushape, every, with_s0):
    """mru_scan_backward_readout: gradients of the readout's outputs (o_t =
    S_t U with one vector, shared or per-head query columns; snapshots every
    `every` steps) to the embeddings and S0, through the C-ABI, against the
    oracle's readout backward; several chunks with a ragged tail."""
    t = torch()
    B, H, L = 2, 3, 53
    alpha = 0.3 / np.sqrt(n) if mode != gen.MODE_LDU else 1.0
    w = gen.Workload("bro", B=B, H=H, L=L, n=n, x_dtype=x_dtype, mode=mode, alpha=float(alpha), seed=31 + n)
    x = gen.make_x(w)
    r = np.random.default_rng(n + every)
    q = 1 if ushape == "vector" else 3
    u = {"vector": r.standard_normal(n), "shared": r.standard_normal((n, q)),
         "per_head": r.standard_normal((H, n, q))}[ushape].astype(np.float32)
    d_o = r.standard_normal((B, L, H, n, q)).astype(np.float32)
    d_snap = r.standard_normal((B, L // every, H, n, n)).astype(np.float32) if every else None
    S0 = (np.eye(n) + 0.1 * r.standard_normal((B, H, n, n))).astype(np.float32) if with_s0 else None
    p = mru.problem_from_workload(w, chunk=16)
    dx, dS0, ws = mru.scan_backward_readout_t(
        p, to_device_x(x), t.from_numpy(u).cuda(), t.from_numpy(d_o).cuda(), snapshot_every=every,
        d_snaps=None if d_snap is None else t.from_numpy(d_snap).cuda(),
        S0=None if S0 is None else t.from_numpy(S0).cuda(), q=0 if ushape == "vector" else q,
        u_per_head=1 if ushape == "per_head" else 0)
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx_o, dS0_o = oracle.backward_readout(oracle_problem(w), x, u.astype(np.float64) if ushape != "vector" else
                                          u.astype(np.float64), d_o[..., 0] if ushape == "vector" else d_o,
                                          snapshot_every=every, d_snap=d_snap,
                                          S0=None if S0 is None else S0.astype(np.float64))
    e = _rel(dx.cpu().numpy().astype(np.float64).reshape(B, L, H, n * n), dx_o.reshape(B, L, H, n * n), axis=-1)
    assert e.max() <= TOL_BWD, (e.max(), np.median(e))
    if with_s0:
        e0 = _rel(dS0.cpu().numpy().astype(np.float64).reshape(B, H, n * n), dS0_o.reshape(B, H, n * n), axis=-1)
        assert e0.max() <= TOL_BWD, e0.max()


@pytest.mark.parametrize("n,mode,dtype,L,chunk", [
    (16, gen.MODE_DETNORM, "f32", 530 * 2 + 3, 2),   # K = 532: groups of 32, the last one ragged
    (8, gen.MODE_DETNORM, "f32", 4200, 1),           # K = 4200 at n = 8: groups of 128
    (32, gen.MODE_LDU, "bf16", 77 * 2, 2),           # K = 77 at n = 32: groups of 16, the last one ragged
])
def test_backward_grouped_chunk_gradient_scan(n, mode, dtype, L, chunk):
    """Problems large enough (K n^3 > 2^20) for the chunk-gradient scan to run
    in groups (group suffix compositions, a scan over the groups, a fix-up per
    chunk) instead of serially: the gradients still match the oracle's fp64
    backward, with S0, over ragged last groups (determinant-corrected, alpha
    small: the states stay in range over thousands of tokens)."""
    alpha = 1.0 if mode == gen.MODE_LDU else 0.05 / np.sqrt(n)
    w = gen.Workload(f"g{n}", B=1, H=2, L=L, n=n, x_dtype=dtype, mode=mode, alpha=float(alpha), seed=900 + n)
    K = -(-L // chunk)
    assert K * n ** 3 > 2 ** 20
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=901)
    dS = np.random.default_rng(902).standard_normal((w.B, w.L, w.H, n, n)).astype(np.float32)
    dx, dS0, st = _run(w, x, S0, dS, chunk=chunk)
    assert st == mru.OK
    dx_o, dS0_o = oracle.backward(oracle_problem(w), x, dS.astype(np.float64), S0=S0.astype(np.float64))
    e_dx = _rel(dx.reshape(w.B, w.L, w.H, n * n), dx_o.reshape(w.B, w.L, w.H, n * n), axis=-1)
    e_s0 = _rel(dS0.reshape(w.B, w.H, n * n), dS0_o.reshape(w.B, w.H, n * n), axis=-1)
    assert e_dx.max() <= TOL_BWD and e_s0.max() <= TOL_BWD, (e_dx.max(), np.median(e_dx), e_s0.max())


# n = 64 on the tensor cores when tf32 is asked for (k64b_local / k64b_apply):
# the tf32 gate of the forward.
TOL_BWD_TF32 = 1e-2

N64_TC_CASES = [  # mode, add_identity, alpha, with_s0, L, chunk
    (gen.MODE_DETNORM, 1, 0.03 / 8, True, 53, 16),    # trace series and its three-term inverse
    (gen.MODE_DETNORM, 1, 0.03 / 8, False, 40, 1),    # one-token chunks
    (gen.MODE_DETNORM, 1, 0.3 / 8, False, 37, 8),     # far from the identity: pivoted elimination
    (gen.MODE_DETNORM, 0, 1.0 / 8, True, 21, 8),      # no identity: pivoted elimination
    (gen.MODE_RESHAPE, 1, 0.3 / 8, True, 53, 16),
    (gen.MODE_RESHAPE, 0, 1.0 / 8, False, 13, 4),
    (gen.MODE_DETNORM, 1, 0.03 / 8, True, 1, 64),     # a single token
    (gen.MODE_DETNORM, 1, 0.03 / 8, True, 5, 0),      # a single chunk (the default chunk for this size)
    (gen.MODE_RESHAPE, 1, 0.3 / 8, False, 2, 1),      # two one-token chunks
]


@pytest.mark.parametrize("mode,add_identity,alpha,with_s0,L,chunk", N64_TC_CASES)
def test_backward_n64_tensor_cores(mode, add_identity, alpha, with_s0, L, chunk):
    """mru_scan_backward at n = 64 with math = tf32 (the tensor-core local and
    apply passes) against the oracle's fp64 backward: several chunks with a
    ragged tail, with and without S0, near and far from the identity."""
    t = torch()
    n = 64
    w = gen.Workload("b64tc", B=2, H=2, L=L, n=n, x_dtype="f32", mode=mode, alpha=float(alpha),
                     add_identity=add_identity, math="tf32", seed=640 + L)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=641) if with_s0 else None
    dS = np.random.default_rng(642 + L).standard_normal((w.B, w.L, w.H, n, n)).astype(np.float32)
    p = mru.problem_from_workload(w, chunk=chunk)
    xd = to_device_x(x)
    S0d = None if S0 is None else t.from_numpy(np.ascontiguousarray(S0, np.float32)).cuda()
    S = mru.scan_fused_t(p, xd, S0=S0d)
    dx, dS0, ws = mru.scan_backward_t(p, xd, S, t.from_numpy(dS).cuda(), S0=S0d)
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx_o, dS0_o = oracle.backward(oracle_problem(w), x, dS.astype(np.float64),
                                  S0=None if S0 is None else S0.astype(np.float64))
    e = _rel(dx.cpu().numpy().astype(np.float64).reshape(w.B, w.L, w.H, n * n), dx_o.reshape(w.B, w.L, w.H, n * n),
             axis=-1)
    print("n64 tensor-core backward: max", e.max(), "median", np.median(e))
    assert e.max() <= TOL_BWD_TF32, (e.max(), np.median(e))
    if with_s0:
        e0 = _rel(dS0.cpu().numpy().astype(np.float64).reshape(w.B, w.H, n * n), dS0_o.reshape(w.B, w.H, n * n),
                  axis=-1)
        assert e0.max() <= TOL_BWD_TF32, e0.max()


def test_backward_readout_n64_tensor_cores_workload_shape():
    """The readout backward of the n = 64 workload's construction (alpha =
    0.03 / 8, corrected with the identity, one query vector, snapshots every
    256 steps, tf32) on a shorter sequence (automatic chunking):
    k64b_local / k64b_apply behind mru_scan_backward_readout, against the
    oracle's readout backward."""
    t = torch()
    B, H, L, n = 1, 2, 1024, 64
    w = gen.Workload("bro64", B=B, H=H, L=L, n=n, x_dtype="f32", mode=gen.MODE_DETNORM, alpha=0.03 / 8,
                     math="tf32", seed=1005)
    x = gen.make_x(w)
    r = np.random.default_rng(77)
    u = r.standard_normal(n).astype(np.float32)
    d_o = r.standard_normal((B, L, H, n, 1)).astype(np.float32)
    d_snap = r.standard_normal((B, L // 256, H, n, n)).astype(np.float32)
    p = mru.problem_from_workload(w)
    dx, _, ws = mru.scan_backward_readout_t(p, to_device_x(x), t.from_numpy(u).cuda(), t.from_numpy(d_o).cuda(),
                                            snapshot_every=256, d_snaps=t.from_numpy(d_snap).cuda())
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx_o, _ = oracle.backward_readout(oracle_problem(w), x, u.astype(np.float64), d_o[..., 0],
                                      snapshot_every=256, d_snap=d_snap)
    e = _rel(dx.cpu().numpy().astype(np.float64).reshape(B, L, H, n * n), dx_o.reshape(B, L, H, n * n), axis=-1)
    print("n64 tensor-core readout backward: max", e.max(), "median", np.median(e))
    assert e.max() <= TOL_BWD_TF32, (e.max(), np.median(e))


def test_backward_readout_many_query_columns():
    """The readout gradient when the heads' query columns are too many to
    stage in shared memory (H n q floats above 48 KB: read through the cache
    instead): 16 heads of n = 32 with 32 columns each, against the oracle."""
    t = torch()
    B, H, L, n, q = 1, 16, 9, 32, 32
    w = gen.Workload("brq", B=B, H=H, L=L, n=n, x_dtype="f32", mode=gen.MODE_DETNORM, alpha=float(0.3 / np.sqrt(n)),
                     seed=91)
    x = gen.make_x(w)
    r = np.random.default_rng(92)
    u = r.standard_normal((H, n, q)).astype(np.float32)
    d_o = r.standard_normal((B, L, H, n, q)).astype(np.float32)
    p = mru.problem_from_workload(w, chunk=4)
    dx, _, ws = mru.scan_backward_readout_t(p, to_device_x(x), t.from_numpy(u).cuda(), t.from_numpy(d_o).cuda(),
                                            q=q, u_per_head=1)
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx_o, _ = oracle.backward_readout(oracle_problem(w), x, u.astype(np.float64), d_o)
    e = _rel(dx.cpu().numpy().astype(np.float64).reshape(B, L, H, n * n), dx_o.reshape(B, L, H, n * n), axis=-1)
    assert e.max() <= TOL_BWD, (e.max(), np.median(e))


@pytest.mark.parametrize("alpha,chunk,with_s0", [(0.0125, 8, True), (0.3 / 4, 16, False), (1.0 / 4, 1, True),
                                                 (0.0125, 3, False)])
def test_backward_n16_cayley_tensor_cores(alpha, chunk, with_s0):
    """The n = 16 Cayley map's backward on the tensor cores: F formed per
    stage as in the forward, dA = 2 T + T F^T with T = dX + F^T dX / 2, dM =
    alpha (dA - dA^T) / 2, all in split tf32; chunks of 1, 3, 8 and 16 over
    L = 45 (ragged), near and far from the identity, with and without S0."""
    t = torch()
    n = 16
    w = gen.Workload("b16c", B=2, H=2, L=45, n=n, x_dtype="f32", mode=gen.MODE_CAYLEY, alpha=float(alpha), seed=630)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=631) if with_s0 else None
    dS = np.random.default_rng(632 + chunk).standard_normal((w.B, w.L, w.H, n, n)).astype(np.float32)
    p = mru.problem_from_workload(w, chunk=chunk)
    xd = to_device_x(x)
    S0d = None if S0 is None else t.from_numpy(np.ascontiguousarray(S0, np.float32)).cuda()
    S = mru.scan_fused_t(p, xd, S0=S0d)
    dx, dS0, ws = mru.scan_backward_t(p, xd, S, t.from_numpy(dS).cuda(), S0=S0d)
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx_o, dS0_o = oracle.backward(oracle_problem(w), x, dS.astype(np.float64),
                                  S0=None if S0 is None else S0.astype(np.float64))
    e = _rel(dx.cpu().numpy().astype(np.float64).reshape(w.B, w.L, w.H, n * n), dx_o.reshape(w.B, w.L, w.H, n * n),
             axis=-1)
    print("n16 Cayley backward: max", e.max(), "median", np.median(e))
    assert e.max() <= TOL_BWD, (e.max(), np.median(e))
    if with_s0:
        e0 = _rel(dS0.cpu().numpy().astype(np.float64).reshape(w.B, w.H, n * n), dS0_o.reshape(w.B, w.H, n * n),
                  axis=-1)
        assert e0.max() <= TOL_BWD, e0.max()


def test_backward_n16_cayley_workload_sampled():
    """The n = 16 Cayley workload (B8 H8 L4096) end to end on the tensor
    cores; the oracle recomputes two sequences."""
    t = torch()
    w = gen.WORKLOADS["n16_cayley_b8h8l4096"]
    x = gen.make_x(w)
    dS = np.random.default_rng(7).standard_normal((w.B, w.L, w.H, 16, 16)).astype(np.float32)
    p = mru.problem_from_workload(w)
    xd = to_device_x(x)
    S = mru.scan_fused_t(p, xd)
    dx, _, ws = mru.scan_backward_t(p, xd, S, t.from_numpy(dS).cuda())
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx = dx.cpu().numpy().astype(np.float64).reshape(w.B, w.L, w.H, 256)
    for b, h in [(0, 0), (6, 3)]:
        w1 = gen.Workload("one", B=1, H=1, L=w.L, n=16, x_dtype="f32", mode=w.mode, alpha=w.alpha, seed=0)
        x1 = np.ascontiguousarray(x.reshape(w.B, w.L, w.H, 256)[b:b + 1, :, h])
        dS1 = dS[b:b + 1, :, h:h + 1].astype(np.float64)
        dx_o, _ = oracle.backward(oracle_problem(w1), x1, dS1)
        e = _rel(dx[b, :, h], dx_o.reshape(w.L, 256), axis=-1)
        print("n16 Cayley workload backward:", b, h, e.max(), np.median(e))
        assert e.max() <= TOL_BWD, (b, h, e.max(), np.median(e))


def test_backward_readout_n64_tensor_cores_long_sequence():
    """The n = 64 readout backward in tf32 with the workload's construction
    and default chunking over one sequence of 4096 tokens (64 chunks): the
    tf32 rounding of the gradient chains accumulated over a quarter of the
    workload's length, against the oracle."""
    t = torch()
    B, H, L, n = 1, 1, 4096, 64
    w = gen.Workload("bro64l", B=B, H=H, L=L, n=n, x_dtype="f32", mode=gen.MODE_DETNORM, alpha=0.03 / 8,
                     math="tf32", seed=1007)
    x = gen.make_x(w)
    r = np.random.default_rng(78)
    u = r.standard_normal(n).astype(np.float32)
    d_o = r.standard_normal((B, L, H, n, 1)).astype(np.float32)
    d_snap = r.standard_normal((B, L // 256, H, n, n)).astype(np.float32)
    p = mru.problem_from_workload(w)
    dx, _, ws = mru.scan_backward_readout_t(p, to_device_x(x), t.from_numpy(u).cuda(), t.from_numpy(d_o).cuda(),
                                            snapshot_every=256, d_snaps=t.from_numpy(d_snap).cuda())
    assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK
    dx_o, _ = oracle.backward_readout(oracle_problem(w), x, u.astype(np.float64), d_o[..., 0],
                                      snapshot_every=256, d_snap=d_snap)
    e = _rel(dx.cpu().numpy().astype(np.float64).reshape(B, L, H, n * n), dx_o.reshape(B, L, H, n * n), axis=-1)
    print("n64 tensor-core readout backward, L = 4096: max", e.max(), "median", np.median(e))
    assert e.max() <= TOL_BWD_TF32, (e.max(), np.median(e))
