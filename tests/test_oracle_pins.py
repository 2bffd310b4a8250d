"""Pins for the fp64 oracle: checks against facts the pages and the mathematics
fix, not against the oracle itself.

What MRU computes ("MRU Update: An independent developer's alternative to
Attention is now running successfully", section "What MRU Actually Does"):
lift each token's embedding to a matrix X_t, multiply S_t = S_{t-1} X_t along
the sequence (the product is associative, which the parallel scan relies on),
reduce S_t to a vector.  Construction variants ("Improving Matrix Recurrent
Units as an Attention Alternative", "Key Points" and "Technical Deep Dive"):
determinant-correcting scalar and LDU factor filling, and the orthogonal
constructions (Cayley map, matrix exponential) that the pages report tried.

Every pin is written as a check that takes an oracle (``scan`` and ``lift``
callables).  The real C oracle must pass every pin; an independent numpy
restatement must pass them too; and each numpy variant with one planted
mistake (wrong multiplication side, transposed reshape, dropped identity,
wrong sign of the determinant exponent, swapped LDU triangles, ...) must fail
at least one pin, which shows the pins can see that kind of mistake.
"""
from __future__ import annotations

import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

from linear_rnn_scan_b200 import inputs as gen


# ---------------------------------------------------------------- oracles ---

def params(B, H, L, n, *, x_dtype="f32", mode=0, alpha=1.0, add_identity=1,
           ldu_offdiag=0.02, ldu_diag=0.1):
    return dict(B=B, H=H, L=L, n=n, x_dtype=x_dtype, mode=mode, alpha=np.float32(alpha),
                add_identity=add_identity, ldu_offdiag=np.float32(ldu_offdiag),
                ldu_diag=np.float32(ldu_diag))


class COracle:
    name = "c-oracle"

    def __init__(self, mod):
        self.m = mod

    def _p(self, P):
        return self.m.make_problem(P["B"], P["H"], P["L"], P["n"], x_dtype=P["x_dtype"], mode=P["mode"],
                                   alpha=float(P["alpha"]), add_identity=P["add_identity"],
                                   ldu_offdiag=float(P["ldu_offdiag"]), ldu_diag=float(P["ldu_diag"]))

    def scan(self, P, x, S0=None):
        return self.m.scan(self._p(P), x, S0)

    def lift(self, P, x, b, t, h):
        return self.m.lift(self._p(P), x, b, t, h)

    def readout(self, P, x, U, every=0):
        return self.m.readout(self._p(P), x, U, every)


class NumpyTwin:
    """Independent numpy restatement of the definition; ``mistake`` plants one
    error so that the pins can be shown to catch it."""

    def __init__(self, mistake=None):
        self.mistake = mistake
        self.name = f"numpy[{mistake}]"

    def lift(self, P, x, b, t, h):
        n = P["n"]
        xs = np.asarray(x)
        if P["x_dtype"] == "bf16":
            xs = gen.bf16_bits_to_f32(xs)
        xs = xs.astype(np.float64).reshape(P["B"], P["L"], P["H"], n * n)
        M = xs[b, t, h].reshape(n, n)
        if self.mistake == "column_major_reshape":
            M = M.T
        if P["mode"] in (3, 4):
            a = float(P["alpha"])
            A = 0.5 * a * (M - M.T)
            if self.mistake == "skew_sign":
                A = -A
            if self.mistake == "skew_no_half":
                A = 2.0 * A
            if self.mistake == "skew_from_upper":
                A = a * (np.triu(M, 1) - np.triu(M, 1).T)
            I = np.eye(n)
            if P["mode"] == 3:
                if self.mistake == "cayley_swapped":
                    return np.linalg.solve(I + A, I - A)
                return np.linalg.solve(I - A, I + A)
            if self.mistake == "expm_first_order":
                return I + A
            import scipy.linalg
            return scipy.linalg.expm(A)
        if P["mode"] in (0, 1):
            X = float(P["alpha"]) * M
            if P["add_identity"] and self.mistake != "drop_identity":
                X = X + np.eye(n)
            if P["mode"] == 1:
                sign, logdet = np.linalg.slogdet(X)
                if sign == 0:
                    raise FloatingPointError("singular")
                e = +1.0 if self.mistake == "det_exponent_sign" else -1.0
                if self.mistake == "det_power_not_root":
                    X = X * math.exp(e * logdet)
                else:
                    X = X * math.exp(e * logdet / n)
            return X
        a, d = float(P["ldu_offdiag"]), float(P["ldu_diag"])
        Lm = np.eye(n) + a * np.tril(M, -1)
        Um = np.eye(n) + a * np.triu(M, 1)
        if self.mistake == "ldu_swap_triangles":
            Lm, Um = np.eye(n) + a * np.tril(M.T, -1), np.eye(n) + a * np.triu(M.T, 1)
        Dm = np.diag(np.exp(d * np.tanh(np.diag(M))))
        if self.mistake == "ldu_diag_no_tanh":
            Dm = np.diag(np.exp(d * np.diag(M)))
        if self.mistake == "ldu_order_udl":
            return Um @ Dm @ Lm
        return Lm @ Dm @ Um

    def scan(self, P, x, S0=None):
        B, H, L, n = P["B"], P["H"], P["L"], P["n"]
        out = np.empty((B, L, H, n, n))
        for b in range(B):
            for h in range(H):
                S = np.eye(n) if S0 is None else np.asarray(S0, np.float64).reshape(B, H, n, n)[b, h]
                for t in range(L):
                    X = self.lift(P, x, b, t, h)
                    if self.mistake == "exclusive_output":     # emits S_{t-1} at position t
                        out[b, t, h] = S
                        S = S @ X
                        continue
                    S = X @ S if self.mistake == "left_multiply" else S @ X
                    out[b, t, h] = S
        return out

    def readout(self, P, x, U, every=0):
        """o_t = S_t U (U [n, q] shared or [H, n, q] per head) and the
        snapshots S_t at 1-based t = every, 2 every, ..."""
        S = self.scan(P, x)
        H, L = P["H"], P["L"]
        U = np.asarray(U, np.float64)
        Uh = [U] * H if U.ndim == 2 else [U[h] for h in range(H)]
        if self.mistake == "readout_head_shift":
            Uh = [Uh[(h + 1) % H] for h in range(H)]
        St = np.swapaxes(S, -1, -2) if self.mistake == "readout_transposed_state" else S
        o = np.stack([St[:, :, h] @ Uh[h] for h in range(H)], axis=2)
        snaps = None
        if every > 0:
            first = 0 if self.mistake == "snapshot_zero_based" else every - 1
            snaps = S[:, first::every][:, :L // every]
        return o, snaps


MISTAKES = ["left_multiply", "column_major_reshape", "drop_identity", "det_exponent_sign",
            "det_power_not_root", "ldu_swap_triangles", "ldu_diag_no_tanh", "ldu_order_udl",
            "exclusive_output", "skew_sign", "skew_no_half", "skew_from_upper", "cayley_swapped",
            "expm_first_order", "readout_transposed_state", "readout_head_shift", "snapshot_zero_based"]


# ------------------------------------------------------------------- pins ---
# Each pin returns None when the oracle satisfies it and raises AssertionError
# otherwise.

def _rng(seed):
    return np.random.default_rng(seed)


def pin_identity_inputs(o):
    """x = 0 with the identity added gives X_t = I, hence S_t = I exactly
    (reshape and determinant-corrected modes)."""
    for mode in (0, 1):
        P = params(2, 3, 5, 4, mode=mode, alpha=0.37)
        x = np.zeros((2, 5, 3 * 16), np.float32)
        S = o.scan(P, x)
        assert np.array_equal(S, np.broadcast_to(np.eye(4), S.shape)), f"mode {mode}"


def pin_diagonal_reshape(o):
    """Diagonal X_t: S_t is diagonal with the running product of the diagonal
    entries (closed form: numpy.cumprod)."""
    n, L = 5, 9
    r = _rng(1)
    d = r.uniform(0.5, 1.5, size=(L, n)).astype(np.float32)
    x = np.zeros((1, L, n * n), np.float32)
    for t in range(L):
        x[0, t, :].reshape(n, n)[np.arange(n), np.arange(n)] = d[t] - np.float32(1.0)
    P = params(1, 1, L, n, alpha=1.0, add_identity=1)
    S = o.scan(P, x)[0, :, 0]
    dd = (d.astype(np.float64) - 1.0) + 1.0
    ref = np.cumprod(dd, axis=0)
    for t in range(L):
        np.testing.assert_allclose(np.diag(S[t]), ref[t], rtol=1e-14, atol=0)
        assert np.count_nonzero(S[t] - np.diag(np.diag(S[t]))) == 0


def pin_diagonal_detnorm(o):
    """Diagonal X~ = diag(d): the corrected X = diag(d) / |prod d|^(1/n), so
    S_t = diag(prod_s d_s) / prod_s |prod_i d_{s,i}|^(1/n).  Negative entries
    keep their sign (|det X| = 1, sign of det kept)."""
    n, L = 4, 7
    r = _rng(2)
    d = r.uniform(0.6, 1.7, size=(L, n))
    d[2, 1] *= -1.0
    d[5, 3] *= -1.0
    d = d.astype(np.float32)
    x = np.zeros((1, L, n * n), np.float32)
    for t in range(L):
        x[0, t].reshape(n, n)[np.arange(n), np.arange(n)] = d[t]
    P = params(1, 1, L, n, mode=1, alpha=1.0, add_identity=0)
    S = o.scan(P, x)[0, :, 0]
    dd = d.astype(np.float64)
    scale = np.abs(np.prod(dd, axis=1)) ** (-1.0 / n)
    ref = np.cumprod(dd * scale[:, None], axis=0)
    for t in range(L):
        np.testing.assert_allclose(np.diag(S[t]), ref[t], rtol=1e-13, atol=0)


def _perm_matrix(p):
    n = len(p)
    M = np.zeros((n, n), np.float32)
    M[np.arange(n), p] = 1.0
    return M


def pin_permutations_exact(o):
    """Products of permutation matrices are permutation matrices; composing
    the permutations exactly in integers gives every S_t bit for bit."""
    n, L, H = 6, 8, 2
    r = _rng(3)
    perms = [[list(r.permutation(n)) for _ in range(L)] for _ in range(H)]
    x = np.zeros((1, L, H * n * n), np.float32)
    for h in range(H):
        for t in range(L):
            x[0, t, h * n * n:(h + 1) * n * n] = _perm_matrix(perms[h][t]).ravel()
    P = params(1, H, L, n, alpha=1.0, add_identity=0)
    S = o.scan(P, x)
    for h in range(H):
        cur = list(range(n))                 # S as a map: row i has its 1 in column cur[i]
        for t in range(L):
            p = perms[h][t]
            cur = [p[c] for c in cur]        # (S X)[i, :] = row cur[i] of X
            ref = np.zeros((n, n))
            ref[np.arange(n), cur] = 1.0
            assert np.array_equal(S[0, t, h], ref), (h, t)


def pin_integer_shears_exact(o):
    """Unipotent integer shears (upper and lower, mixed so that they do not
    commute): the product is an integer matrix computed exactly with Python
    ints; fp64 holds it exactly while entries stay below 2**53."""
    n, L = 4, 10
    r = _rng(4)
    mats = []
    for t in range(L):
        A = np.eye(n, dtype=np.int64)
        k = np.triu_indices(n, 1) if t % 2 == 0 else np.tril_indices(n, -1)
        A[k] = r.integers(-2, 3, size=len(k[0]))
        mats.append(A)
    x = np.stack([m.astype(np.float32).ravel() for m in mats])[None]
    P = params(1, 1, L, n, alpha=1.0, add_identity=0)
    S = o.scan(P, x)[0, :, 0]
    cur = [[int(i == j) for j in range(n)] for i in range(n)]
    for t in range(L):
        X = mats[t].tolist()
        cur = [[sum(cur[i][k] * X[k][j] for k in range(n)) for j in range(n)] for i in range(n)]
        assert max(abs(v) for row in cur for v in row) < 2 ** 53
        assert np.array_equal(S[t], np.array(cur, dtype=np.float64)), t


def _all_parenthesizations(ms):
    """Every full parenthesisation of the product ms[0] ... ms[-1], exactly."""
    if len(ms) == 1:
        return [ms[0]]
    out = []
    for k in range(1, len(ms)):
        for left in _all_parenthesizations(ms[:k]):
            for right in _all_parenthesizations(ms[k:]):
                out.append(_fmul(left, right))
    return out


def _fmul(A, Bm):
    n = len(A)
    return tuple(tuple(sum(A[i][k] * Bm[k][j] for k in range(n)) for j in range(n)) for i in range(n))


def pin_bruteforce_exact(o):
    """Tiny inputs: every parenthesisation of X_1 ... X_6 in exact rationals
    gives one product (associativity, on which the parallel scan rests: 42
    trees for 6 factors), and the oracle's S_t agree with the exact rational
    prefix products to fp64 rounding."""
    n, L = 3, 6
    x = gen.randn_f32((1, L, n * n), 5) * np.float32(0.5)
    P = params(1, 1, L, n, alpha=np.float32(0.75), add_identity=1)
    S = o.scan(P, x)[0, :, 0]
    a = Fraction(float(np.float32(0.75)))
    mats = []
    for t in range(L):
        M = x[0, t].reshape(n, n)
        mats.append(tuple(tuple(a * Fraction(float(M[i, j])) + (1 if i == j else 0) for j in range(n))
                          for i in range(n)))
    trees = _all_parenthesizations(mats)
    assert len(trees) == 42
    assert all(tr == trees[0] for tr in trees)
    pref = mats[0]
    for t in range(L):
        if t:
            pref = _fmul(pref, mats[t])
        exact = np.array([[float(v) for v in row] for row in pref])
        err = np.linalg.norm(S[t] - exact) / np.linalg.norm(exact)
        assert err < 1e-14, (t, err)
    assert pref == trees[0]


def pin_detnorm_unit_det(o):
    """Determinant correction: |det X_t| = 1 for every token (checked with
    numpy.linalg.det), the sign of det X~ is kept, and X_t is a positive
    multiple of X~; near identity and far from it (pivoting needed)."""
    for alpha, add_id, seed in ((0.0125, 1, 6), (0.9, 1, 7), (1.0, 0, 8)):
        n, L, H = 6, 5, 2
        x = gen.randn_f32((1, L, H * n * n), seed)
        P = params(1, H, L, n, mode=1, alpha=alpha, add_identity=add_id)
        for t in range(L):
            for h in range(H):
                X = o.lift(P, x, 0, t, h)
                Xr = float(np.float32(alpha)) * x[0, t, h * n * n:(h + 1) * n * n].astype(np.float64).reshape(n, n)
                if add_id:
                    Xr = Xr + np.eye(n)
                assert abs(abs(np.linalg.det(X)) - 1.0) < 1e-12
                assert np.sign(np.linalg.det(X)) == np.sign(np.linalg.det(Xr))
                c = X / Xr
                assert np.all(c > 0) and np.ptp(c) < 1e-12 * np.max(c)


def pin_detnorm_product_det(o):
    """det S_t = prod_s det X_s = prod_s sign(det X~_s) while S_t is well
    conditioned enough for det to be computed."""
    n, L = 4, 40
    x = gen.randn_f32((1, L, n * n), 9)
    P = params(1, 1, L, n, mode=1, alpha=0.6, add_identity=1)
    S = o.scan(P, x)[0, :, 0]
    sign = 1.0
    for t in range(L):
        Xr = np.eye(n) + float(np.float32(0.6)) * x[0, t].astype(np.float64).reshape(n, n)
        sign *= np.sign(np.linalg.det(Xr))
        if np.linalg.cond(S[t]) < 1e8:
            assert abs(np.linalg.det(S[t]) - sign) < 1e-8, t


def pin_ldu_factors(o):
    """LDU fill: det X = prod_i D_ii = exp(sum_i d*tanh(M_ii)) (closed form),
    and the textbook LU factorisation of X (scipy, which pivots only when a
    sub-diagonal entry outgrows the pivot; it does not here) returns the unit
    lower factor I + a*tril(M) and the upper factor D (I + a*triu(M))."""
    import scipy.linalg
    n, L = 8, 4
    xf = gen.randn_f32((1, L, n * n), 10)
    for dtype in ("f32", "bf16"):
        x = xf if dtype == "f32" else gen.f32_to_bf16_bits(xf)
        xm = xf if dtype == "f32" else gen.bf16_bits_to_f32(x)
        P = params(1, 1, L, n, x_dtype=dtype, mode=2, ldu_offdiag=0.02, ldu_diag=0.1)
        a, d = float(np.float32(0.02)), float(np.float32(0.1))
        for t in range(L):
            M = xm[0, t].astype(np.float64).reshape(n, n)
            X = o.lift(P, x, 0, t, 0)
            det_ref = math.exp(sum(d * math.tanh(M[i, i]) for i in range(n)))
            assert abs(np.linalg.det(X) - det_ref) < 1e-13 * det_ref
            Pm, Lf, Uf = scipy.linalg.lu(X)
            assert np.array_equal(Pm, np.eye(n))
            np.testing.assert_allclose(Lf, np.eye(n) + a * np.tril(M, -1), atol=1e-14)
            Dm = np.diag(np.exp(d * np.tanh(np.diag(M))))
            np.testing.assert_allclose(Uf, Dm @ (np.eye(n) + a * np.triu(M, 1)), atol=1e-14)


def pin_initial_state_and_resume(o):
    """S0 enters on the left: S_t(S0) = S0 S_t(I); and a run split at any
    point and resumed from the last state equals the whole run (associativity
    again; this is also the segmented / decode use of the scan)."""
    n, L, H = 4, 12, 2
    x = gen.randn_f32((1, L, H * n * n), 11)
    P = params(1, H, L, n, alpha=0.3, add_identity=1)
    S = o.scan(P, x)
    S0 = np.eye(n) + 0.2 * gen.randn_f32((1, H, n, n), 12).astype(np.float64)
    S_s0 = o.scan(P, x, S0)
    for t in range(L):
        for h in range(H):
            np.testing.assert_allclose(S_s0[0, t, h], S0[0, h] @ S[0, t, h], rtol=1e-13, atol=1e-14)
    cut = 5
    P1 = dict(P, L=cut)
    P2 = dict(P, L=L - cut)
    first = o.scan(P1, np.ascontiguousarray(x[:, :cut]))
    second = o.scan(P2, np.ascontiguousarray(x[:, cut:]), first[:, -1])
    whole = np.concatenate([first, second], axis=1)
    np.testing.assert_allclose(whole, S, rtol=1e-13, atol=1e-14)


def pin_orthogonal_2x2_closed_forms(o):
    """n = 2: the skew-symmetric part of alpha M is A = [[0, a], [-a, 0]] with
    a = alpha (M01 - M10) / 2.  Cayley map: X = [[1 - a^2, 2a], [-2a, 1 - a^2]]
    / (1 + a^2); matrix exponential: the rotation [[cos a, sin a],
    [-sin a, cos a]] (closed forms; the larger alpha needs the squaring)."""
    L = 8
    x = gen.randn_f32((1, L, 4), 31) * np.float32(2.0)
    for alpha in (0.3, 2.5):
        al = float(np.float32(alpha))
        for mode in (3, 4):
            P = params(1, 1, L, 2, mode=mode, alpha=alpha)
            for t in range(L):
                M = x[0, t].astype(np.float64).reshape(2, 2)
                a = 0.5 * al * (M[0, 1] - M[1, 0])
                if mode == 3:
                    ref = np.array([[1 - a * a, 2 * a], [-2 * a, 1 - a * a]]) / (1 + a * a)
                else:
                    ref = np.array([[math.cos(a), math.sin(a)], [-math.sin(a), math.cos(a)]])
                np.testing.assert_allclose(o.lift(P, x, 0, t, 0), ref, rtol=0, atol=1e-13)


def pin_orthogonal_modes(o):
    """Cayley map and matrix exponential: X_t is orthogonal with det +1, it
    depends only on the skew-symmetric part of M (adding a symmetric matrix
    to M changes nothing, bit for bit: the inputs are dyadic, so every sum is
    exact), it agrees with numpy.linalg.solve(I - A, I + A) and
    scipy.linalg.expm(A), and every S_t stays orthogonal along the sequence."""
    import scipy.linalg
    n, L = 8, 30
    r = _rng(32)
    M = (np.round(r.standard_normal((L, n, n)) * 256) / 256).astype(np.float32)
    Y = np.round(r.standard_normal((L, n, n)) * 64) / 64
    Msym = (M + (Y + np.swapaxes(Y, 1, 2))).astype(np.float32)
    x1, x2 = M.reshape(1, L, n * n), Msym.reshape(1, L, n * n)
    for alpha in (0.05, 0.7):
        al = float(np.float32(alpha))
        for mode in (3, 4):
            P = params(1, 1, L, n, mode=mode, alpha=alpha)
            for t in range(0, L, 7):
                X = o.lift(P, x1, 0, t, 0)
                assert np.array_equal(X, o.lift(P, x2, 0, t, 0)), (mode, t)
                assert np.abs(X.T @ X - np.eye(n)).max() < 1e-13
                assert abs(np.linalg.det(X) - 1.0) < 1e-12
                Mt = M[t].astype(np.float64)
                A = 0.5 * al * (Mt - Mt.T)
                ref = (np.linalg.solve(np.eye(n) - A, np.eye(n) + A) if mode == 3 else scipy.linalg.expm(A))
                np.testing.assert_allclose(X, ref, rtol=0, atol=1e-13)
            S = o.scan(P, x1)[0, :, 0]
            for t in range(L):
                assert np.abs(S[t].T @ S[t] - np.eye(n)).max() < 1e-12, (mode, t)


# ------------------------------------------------------------ readout pins ---
# The pages leave the reduction of S_t open; the reading taken is o_t = S_t U
# with q query columns (one U for every head, or one per head) and full
# snapshots of S_t at the 1-based steps t = every, 2 every, ...  These pins
# check an oracle's ``readout(P, x, U, every)`` against integer products
# computed exactly with Python ints.

def _shear_chains(H, L, n, seed):
    """Per-head chains of unipotent integer shears (upper and lower mixed)
    and their exact prefix products as nested Python-int lists."""
    r = _rng(seed)
    x = np.zeros((1, L, H * n * n), np.float32)
    prefix = []
    for h in range(H):
        cur = [[int(i == j) for j in range(n)] for i in range(n)]
        seq = []
        for t in range(L):
            A = np.eye(n, dtype=np.int64)
            k = np.triu_indices(n, 1) if (t + h) % 2 == 0 else np.tril_indices(n, -1)
            A[k] = r.integers(-2, 3, size=len(k[0]))
            x[0, t, h * n * n:(h + 1) * n * n] = A.astype(np.float32).ravel()
            X = A.tolist()
            cur = [[sum(cur[i][m] * X[m][j] for m in range(n)) for j in range(n)] for i in range(n)]
            seq.append(cur)
        prefix.append(seq)
    return x, prefix


def _int_matmul(A, Bm):
    return [[sum(A[i][m] * Bm[m][j] for m in range(len(Bm))) for j in range(len(Bm[0]))] for i in range(len(A))]


def pin_readout_exact_integer(o):
    """Integer shear chains read out through integer query columns: o_t = S_t U
    entry for entry, exactly, with one U for every head and with one U per
    head (each head reads its own)."""
    n, L, H, q = 4, 9, 3, 2
    x, prefix = _shear_chains(H, L, n, 31)
    P = params(1, H, L, n, alpha=1.0, add_identity=0)
    r = _rng(32)
    U_shared = r.integers(-3, 4, size=(n, q))
    U_head = r.integers(-3, 4, size=(H, n, q))
    for U, per_head in ((U_shared, False), (U_head, True)):
        out, _ = o.readout(P, x, U.astype(np.float64), 0)
        out = np.asarray(out).reshape(1, L, H, n, q)
        for h in range(H):
            Uh = (U_head[h] if per_head else U_shared).tolist()
            for t in range(L):
                ref = _int_matmul(prefix[h][t], Uh)
                assert max(abs(v) for row in ref for v in row) < 2 ** 53
                assert np.array_equal(out[0, t, h], np.array(ref, np.float64)), (per_head, h, t)


def pin_snapshots_one_based(o):
    """Snapshots are S_t at 1-based t = every, 2 every, ... (floor(L / every)
    of them), compared with the exact integer prefix products."""
    n, L, H, every = 4, 10, 2, 3
    x, prefix = _shear_chains(H, L, n, 33)
    P = params(1, H, L, n, alpha=1.0, add_identity=0)
    _, snaps = o.readout(P, x, np.eye(n)[:, :1], every)
    snaps = np.asarray(snaps).reshape(1, L // every, H, n, n)
    for k in range(L // every):
        for h in range(H):
            assert np.array_equal(snaps[0, k, h], np.array(prefix[h][(k + 1) * every - 1], np.float64)), (k, h)


PINS = [pin_identity_inputs, pin_diagonal_reshape, pin_diagonal_detnorm, pin_permutations_exact,
        pin_integer_shears_exact, pin_bruteforce_exact, pin_detnorm_unit_det,
        pin_detnorm_product_det, pin_ldu_factors, pin_initial_state_and_resume,
        pin_orthogonal_2x2_closed_forms, pin_orthogonal_modes, pin_readout_exact_integer,
        pin_snapshots_one_based]


# ------------------------------------------------------------------ tests ---

@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_c_oracle_passes_pin(pin, oracle_mod):
    pin(COracle(oracle_mod))


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_numpy_twin_passes_pin(pin):
    pin(NumpyTwin())


@pytest.mark.parametrize("mistake", MISTAKES)
def test_planted_mistake_fails_some_pin(mistake):
    o = NumpyTwin(mistake)
    failed = []
    for pin in PINS:
        try:
            pin(o)
        except (AssertionError, FloatingPointError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {mistake!r}"


def test_bf16_widening_is_exact(oracle_mod):
    for bits, val in ((0x3F80, 1.0), (0xC000, -2.0), (0x3F81, 1.0078125), (0x0000, 0.0),
                      (0x8000, -0.0), (0x7F7F, 3.3895313892515355e38), (0x0001, 9.183549615799121e-41)):
        assert oracle_mod.bf16_to_float(bits) == val


def test_singular_detnorm_is_reported(oracle_mod):
    p = oracle_mod.make_problem(1, 1, 3, 4, mode=1, alpha=1.0, add_identity=0)
    x = np.zeros((1, 3, 16), np.float32)
    with pytest.raises(FloatingPointError):
        oracle_mod.scan(p, x)


def test_second_oracle_numpy_on_small_workload(oracle_mod):
    """The small reshape workload (n = 4, L = 1024) with a numpy fp64 `@` loop
    as an independent second oracle."""
    w = gen.WORKLOADS["n4_reshape_l1024"]
    x = gen.make_x(w)
    p = oracle_mod.make_problem(w.B, w.H, w.L, w.n, mode=w.mode, alpha=w.alpha, add_identity=1)
    S = oracle_mod.scan(p, x)[0, :, 0]
    a = float(np.float32(w.alpha))
    cur = np.eye(4)
    for t in range(w.L):
        cur = cur @ (np.eye(4) + a * x[0, t].astype(np.float64).reshape(4, 4))
        assert np.linalg.norm(S[t] - cur) <= 1e-13 * np.linalg.norm(cur)


def test_readout_and_snapshots_match_scan(oracle_mod):
    """o_t = S_t u (the pages leave the reduction open; this build reads it as
    one shared readout vector) and snapshots are S_t at 1-based t = k*every."""
    B, H, L, n, every = 2, 3, 16, 8, 4
    x = gen.randn_f32((B, L, H * n * n), 13)
    p = oracle_mod.make_problem(B, H, L, n, mode=1, alpha=0.05, add_identity=1)
    u = gen.make_u(gen.Workload("t", B, H, L, n, "f32", 1, seed=14)).astype(np.float64)
    S = oracle_mod.scan(p, x)
    o, snaps = oracle_mod.readout(p, x, u, every)
    np.testing.assert_allclose(o, S @ u, rtol=1e-13, atol=1e-15)
    for k in range(L // every):
        np.testing.assert_array_equal(snaps[:, k], S[:, (k + 1) * every - 1])


def test_compare_reports_errors_where_planted(oracle_mod):
    B, H, L, n = 2, 2, 10, 4
    x = gen.randn_f32((B, L, H * n * n), 15)
    p = oracle_mod.make_problem(B, H, L, n, mode=1, alpha=0.1, add_identity=1)
    S = oracle_mod.scan(p, x)
    g = S.astype(np.float32)
    res = oracle_mod.compare(p, x, S_gpu=g)
    st = oracle_mod.error_stats(*res["S"])
    assert st["count"] == B * L * H and st["max"] < 1e-7
    g2 = g.copy()
    g2[1, 7, 0, 2, 3] += 1e-3
    st2 = oracle_mod.error_stats(*oracle_mod.compare(p, x, S_gpu=g2)["S"])
    assert st2["max"] > 1e-4
    assert np.unravel_index(st2["argmax"], (B, L, H)) == (1, 7, 0)
    g3 = np.swapaxes(g, -1, -2).copy()              # transposed output layout
    assert oracle_mod.error_stats(*oracle_mod.compare(p, x, S_gpu=g3)["S"])["max"] > 1e-3
    # a subset of sequences and a prefix of the time axis
    res = oracle_mod.compare(p, x, S_gpu=g, bh=[3], t_end=6)
    d2 = res["S"][0]
    assert np.isnan(d2[0]).all() and not np.isnan(d2[1, :6, 1]).any() and np.isnan(d2[1, 6:, 1]).all()


def test_readout_query_columns(oracle_mod):
    """Query columns U ([n, q] shared or [H, n, q] per head): o_t = S_t U.
    Identity columns return S_t itself and unit columns pick columns of S_t
    (both exact: every product has one non-zero term); general U agrees with
    numpy's product of the scanned states, head by head."""
    B, H, L, n, every = 2, 3, 12, 8, 3
    x = gen.randn_f32((B, L, H * n * n), 21)
    p = oracle_mod.make_problem(B, H, L, n, mode=1, alpha=0.05, add_identity=1)
    S = oracle_mod.scan(p, x)
    o, _ = oracle_mod.readout(p, x, np.eye(n))
    assert o.shape == (B, L, H, n, n)
    np.testing.assert_array_equal(o, S)
    cols = [5, 0, 5]
    o, _ = oracle_mod.readout(p, x, np.eye(n)[:, cols])
    np.testing.assert_array_equal(o, S[..., cols])
    rng = np.random.default_rng(22)
    U = rng.standard_normal((H, n, 3))
    o, snaps = oracle_mod.readout(p, x, U, every)
    for h in range(H):
        np.testing.assert_allclose(o[:, :, h], S[:, :, h] @ U[h], rtol=1e-12, atol=1e-14)
    assert np.abs(o[:, :, 0] - S[:, :, 0] @ U[1]).max() > 1e-2       # heads are not interchangeable
    o1, _ = oracle_mod.readout(p, x, U[0])
    np.testing.assert_allclose(o1, S @ U[0], rtol=1e-12, atol=1e-14)
    # the streaming comparison locates a planted error in one query column
    g = o.astype(np.float32)
    st = oracle_mod.error_stats(*oracle_mod.compare(p, x, u=U, o_gpu=g)["o"])
    assert st["count"] == B * L * H and st["max"] < 1e-6
    g[1, 4, 2, 6, 1] += 1e-2
    st = oracle_mod.error_stats(*oracle_mod.compare(p, x, u=U, o_gpu=g)["o"])
    assert st["max"] > 1e-3 and np.unravel_index(st["argmax"], (B, L, H)) == (1, 4, 2)
    with pytest.raises(ValueError):
        oracle_mod.readout(p, x, np.zeros((n, n + 1)))
