"""Pins of the oracle's backward (vector-Jacobian product), independent of
it: central finite differences of J = sum_t <dS_t, S_t> computed with the
oracle's forward scan (Richardson-extrapolated, on inputs exact in fp32), a
closed form for diagonal inputs, and bf16 inputs against the same values
given as fp32."""
from __future__ import annotations

import numpy as np
import pytest

import oracle

MODES = [  # (mode, n, add_identity, alpha)
    (oracle.MODE_RESHAPE, 3, 1, 0.3),
    (oracle.MODE_RESHAPE, 3, 0, 0.7),
    (oracle.MODE_DETNORM, 3, 1, 0.25),
    (oracle.MODE_DETNORM, 4, 0, 0.5),
    (oracle.MODE_LDU, 4, 1, 1.0),
    (oracle.MODE_CAYLEY, 4, 1, 0.6),
    (oracle.MODE_EXPM, 4, 1, 0.6),
    (oracle.MODE_EXPM, 3, 1, 2.5),      # scaling and squaring in the forward
]


def _dyadic(rng, shape, scale_bits=8, lim=2.0):
    """Values k / 2^scale_bits in [-lim, lim]: x +- 2^-11 stays exact in fp32."""
    k = rng.integers(-int(lim * 2 ** scale_bits), int(lim * 2 ** scale_bits) + 1, size=shape)
    return (k / 2.0 ** scale_bits).astype(np.float32)


def _J(p, x, S0, dS):
    return float(np.sum(oracle.scan(p, x, S0=S0, nthreads=1) * dS))


def _fd(f, h):
    """Richardson-extrapolated central difference (error O(h^4))."""
    d1 = (f(h) - f(-h)) / (2 * h)
    d2 = (f(h / 2) - f(-h / 2)) / h
    return (4 * d2 - d1) / 3


@pytest.mark.parametrize("mode,n,add_identity,alpha", MODES)
def test_backward_matches_finite_differences(mode, n, add_identity, alpha):
    rng = np.random.default_rng(40 + 7 * mode + n + add_identity)
    B, H, L = 1, 2, 5
    p = oracle.make_problem(B, H, L, n, mode=mode, alpha=alpha, add_identity=add_identity,
                            ldu_offdiag=0.3, ldu_diag=0.5)
    x = _dyadic(rng, (B, L, H * n * n), lim=1.0)
    S0 = np.eye(n)[None, None] + 0.3 * rng.standard_normal((B, H, n, n))
    dS = rng.standard_normal((B, L, H, n, n))
    dx, dS0 = oracle.backward(p, x, dS, S0=S0, nthreads=1)
    h = 2.0 ** -11
    worst = 0.0
    scale = np.abs(dx).max()
    for idx in np.ndindex(x.shape):
        def f(e, idx=idx):
            xe = x.copy()
            xe[idx] = np.float32(x[idx] + e)
            return _J(p, xe, S0, dS)
        worst = max(worst, abs(_fd(f, h) - dx[idx]) / scale)
    assert worst < 1e-7, worst
    worst = 0.0
    scale = np.abs(dS0).max()
    for idx in np.ndindex(S0.shape):
        def g(e, idx=idx):
            Se = S0.copy()
            Se[idx] += e
            return _J(p, x, Se, dS)
        worst = max(worst, abs(_fd(g, 1e-4) - dS0[idx]) / scale)
    assert worst < 1e-8, worst


def test_backward_diagonal_closed_form():
    """X_t = diag(d_t) (reshape, alpha 1, no identity), S0 = I:
    J = sum_t sum_i dS_t[i, i] prod_{s <= t} d_{s,i}, so
    dJ/dd_{s,i} = sum_{t >= s} dS_t[i, i] prod_{r <= t, r != s} d_{r,i}."""
    rng = np.random.default_rng(3)
    B, H, L, n = 1, 1, 6, 4
    p = oracle.make_problem(B, H, L, n, mode=oracle.MODE_RESHAPE, alpha=1.0, add_identity=0)
    d = rng.uniform(0.5, 1.5, size=(L, n)).astype(np.float32)
    X = np.zeros((B, L, H, n, n), np.float32)
    for t in range(L):
        X[0, t, 0][np.arange(n), np.arange(n)] = d[t]
    dS = rng.standard_normal((B, L, H, n, n))
    dx, _ = oracle.backward(p, X.reshape(B, L, H * n * n), dS, nthreads=1)
    dx = dx.reshape(B, L, H, n, n)
    dd = d.astype(np.float64)
    for s in range(L):
        for i in range(n):
            want = sum(dS[0, t, 0, i, i] * np.prod([dd[r, i] for r in range(t + 1) if r != s]) for t in range(s, L))
            assert dx[0, s, 0, i, i] == pytest.approx(want, rel=1e-12, abs=1e-12)


def test_backward_bf16_equals_widened_f32():
    rng = np.random.default_rng(11)
    B, H, L, n = 1, 2, 7, 4
    bits = (rng.standard_normal((B, L, H * n * n)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    widened = (bits.astype(np.uint32) << 16).view(np.float32)
    dS = rng.standard_normal((B, L, H, n, n))
    for mode in (oracle.MODE_LDU, oracle.MODE_DETNORM):
        pb = oracle.make_problem(B, H, L, n, x_dtype="bf16", mode=mode, alpha=0.2)
        pf = oracle.make_problem(B, H, L, n, x_dtype="f32", mode=mode, alpha=0.2)
        assert np.array_equal(oracle.backward(pb, bits, dS, nthreads=1)[0],
                              oracle.backward(pf, widened, dS, nthreads=1)[0])


def _J_readout(p, x, S0, u, d_o, every, d_snap):
    o, snaps = oracle.readout(p, x, u, snapshot_every=every, S0=S0, nthreads=1)
    j = float(np.sum(o * d_o))
    if every:
        j += float(np.sum(snaps * d_snap))
    return j


@pytest.mark.parametrize("mode,n,add_identity,alpha,ushape,every", [
    (oracle.MODE_RESHAPE, 3, 1, 0.3, "vector", 2),
    (oracle.MODE_DETNORM, 3, 1, 0.25, "shared", 3),
    (oracle.MODE_LDU, 3, 1, 1.0, "per_head", 2),
    (oracle.MODE_CAYLEY, 3, 1, 0.6, "shared", 0),
])
def test_backward_readout_matches_finite_differences(mode, n, add_identity, alpha, ushape, every):
    """The readout form's VJP (gradients of o_t = S_t U and of the snapshots
    given, no state stored) against central finite differences of
    J = sum_t <do_t, o_t> + sum_k <dP_k, P_k> computed with the oracle's
    readout forward, with respect to every embedding value and to S0."""
    rng = np.random.default_rng(70 + 5 * mode + n)
    B, H, L = 1, 2, 6
    p = oracle.make_problem(B, H, L, n, mode=mode, alpha=alpha, add_identity=add_identity,
                            ldu_offdiag=0.3, ldu_diag=0.5)
    x = _dyadic(rng, (B, L, H * n * n), lim=1.0)
    S0 = np.eye(n)[None, None] + 0.3 * rng.standard_normal((B, H, n, n))
    q = 2
    u = {"vector": rng.standard_normal(n), "shared": rng.standard_normal((n, q)),
         "per_head": rng.standard_normal((H, n, q))}[ushape]
    o, _ = oracle.readout(p, x, u, S0=S0, nthreads=1)
    d_o = rng.standard_normal(o.shape)
    d_snap = rng.standard_normal((B, L // every, H, n, n)) if every else None
    dx, dS0 = oracle.backward_readout(p, x, u, d_o, snapshot_every=every, d_snap=d_snap, S0=S0, nthreads=1)
    h = 2.0 ** -11
    worst, scale = 0.0, np.abs(dx).max()
    for idx in np.ndindex(x.shape):
        def f(e, idx=idx):
            xe = x.copy()
            xe[idx] = np.float32(x[idx] + e)
            return _J_readout(p, xe, S0, u, d_o, every, d_snap)
        worst = max(worst, abs(_fd(f, h) - dx[idx]) / scale)
    assert worst < 1e-7, worst
    worst, scale = 0.0, np.abs(dS0).max()
    for idx in np.ndindex(S0.shape):
        def g(e, idx=idx):
            Se = S0.copy()
            Se[idx] += e
            return _J_readout(p, x, Se, u, d_o, every, d_snap)
        worst = max(worst, abs(_fd(g, 1e-4) - dS0[idx]) / scale)
    assert worst < 1e-8, worst
