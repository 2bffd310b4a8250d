"""GPU parity of the exponential map on the n = 16 tensor-core passes
(X = exp(A), A = alpha (M - M^T) / 2; the reduce and apply passes form
F = X - I over each slice by scaling and squaring, the Taylor polynomial in
Horner form over B^2 on split-tf32 mma) against the fp64 oracle.

The cases span the degrees the norm selects (small alpha: low degree, no
squaring; alpha 0.3 to 4: higher degrees and up to about 7 squarings), odd
head counts, ragged stages and chunks, several chunks per sequence (the
carry scan between the passes) and single-chunk problems (the apply pass
alone, from S0), and the single-read kernel (opt-in)."""
from __future__ import annotations

import os

import numpy as np
import pytest

from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

from gpu_helpers import TOL_FP32, compare_S, run_fused, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    mru.load()


def wl(B, H, L, alpha, seed):
    return gen.Workload("expm16", B=B, H=H, L=L, n=16, x_dtype="f32", mode=gen.MODE_EXPM, alpha=float(alpha),
                        add_identity=1, seed=seed)


def orthogonality_gap(S):
    S = S.astype(np.float64)
    G = np.einsum("...ki,...kj->...ij", S, S)
    return float(np.abs(G - np.eye(16)).max())


CASES = [
    # B, H, L, chunk, alpha
    (2, 3, 8 * 13 + 5, 8, 0.0125),       # odd H, ragged last stage and chunk, 14 chunks
    (1, 2, 16 * 9, 16, 0.3),             # higher Taylor degree
    (2, 2, 77, 16, 1.0),                 # squarings
    (1, 3, 61, 8, 4.0),                  # many squarings, degree at its cap
    (3, 1, 517, 0, 0.0125),              # automatic chunk
]


@pytest.mark.parametrize("B,H,L,chunk,alpha", CASES)
@pytest.mark.parametrize("with_s0", [False, True])
def test_expm16_against_oracle(B, H, L, chunk, alpha, with_s0):
    w = wl(B, H, L, alpha, seed=B * 1000 + L)
    p = mru.problem_from_workload(w, chunk=chunk)
    assert mru.kernel_names(p)[0] in ("k16_reduce", "k16_apply")
    x = gen.make_x(w)
    S0 = None
    if with_s0:
        r = np.random.default_rng(L)
        q, _ = np.linalg.qr(r.standard_normal((B, H, 16, 16)))
        S0 = q.astype(np.float32)
    S, st = run_fused(w, x, S0=S0, chunk=chunk)
    assert st == mru.OK
    e = compare_S(w, x, S, S0=S0)
    assert e["count"] == B * H * L
    assert e["max"] <= TOL_FP32, e
    assert orthogonality_gap(S) < 1e-4


def test_expm16_single_chunk_from_s0():
    """L <= chunk: the apply pass alone, its carry read from S0."""
    w = wl(4, 3, 13, 0.5, seed=77)
    p = mru.problem_from_workload(w, chunk=16)
    assert mru.kernel_names(p) == ["k16_apply"]
    x = gen.make_x(w)
    r = np.random.default_rng(78)
    S0 = np.linalg.qr(r.standard_normal((4, 3, 16, 16)))[0].astype(np.float32)
    S, st = run_fused(w, x, S0=S0, chunk=16)
    assert st == mru.OK
    e = compare_S(w, x, S, S0=S0)
    assert e["max"] <= TOL_FP32, e


def test_expm16_zero_input_is_identity():
    """M = 0 gives A = 0 and X = I exactly: every state equals S0 bit for bit."""
    w = wl(1, 2, 40, 0.7, seed=5)
    x = np.zeros((1, 40, 2 * 256), np.float32)
    r = np.random.default_rng(6)
    S0 = r.standard_normal((1, 2, 16, 16)).astype(np.float32)
    S, st = run_fused(w, x, S0=S0, chunk=8)
    assert st == mru.OK
    assert np.array_equal(S, np.broadcast_to(S0[:, None], S.shape))


def test_expm16_single_read_kernel():
    old = os.environ.get("MRU_N16_FUSED")
    os.environ["MRU_N16_FUSED"] = "1"
    try:
        w = wl(1, 4, 8 * 16 * 3 + 8, 0.2, seed=91)
        p = mru.problem_from_workload(w, chunk=8)
        assert mru.kernel_names(p) == ["k16_fused"]
        x = gen.make_x(w)
        S, st = run_fused(w, x, chunk=8)
        assert st == mru.OK
        e = compare_S(w, x, S)
        assert e["max"] <= TOL_FP32, e
    finally:
        if old is None:
            os.environ.pop("MRU_N16_FUSED", None)
        else:
            os.environ["MRU_N16_FUSED"] = old
