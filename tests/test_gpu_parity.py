"""GPU parity: the CUDA path (through the C-ABI) against the fp64 oracle on
the same seeded inputs.  Bit-exact where the arithmetic is exact (integer
permutation and shear products check indexing, layout, chunking and carries),
within the relative Frobenius gate elsewhere (1e-4 fp32, 1e-2 tensor-core
paths), over several chunks and ragged tails, every n, every construction
mode, both input dtypes, with and without S0, and with the readout (one
vector or q query columns)."""
from __future__ import annotations

import numpy as np
import pytest

from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

from gpu_helpers import (TOL_FP32, compare_readout, compare_S, oracle_problem, run_fused, to_device_x,
                         tol_for_problem, torch)

import oracle

pytestmark = pytest.mark.gpu

NS = [4, 8, 16, 32, 64]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    mru.load()
    yield


def small(n, mode, *, B=1, H=1, L=37, x_dtype="f32", alpha=None, add_identity=1, seed=7):
    if alpha is None:
        alpha = 0.3 / np.sqrt(n)
    return gen.Workload(f"t{n}", B=B, H=H, L=L, n=n, x_dtype=x_dtype, mode=mode, alpha=float(alpha),
                        add_identity=add_identity, seed=seed)


# ---------------------------------------------------------------- exact ---

def _perm_inputs(B, H, L, n, seed):
    r = np.random.default_rng(seed)
    x = np.zeros((B, L, H, n, n), np.float32)
    for b in range(B):
        for t in range(L):
            for h in range(H):
                x[b, t, h, np.arange(n), r.permutation(n)] = 1.0
    return x.reshape(B, L, H * n * n)


def _shear_inputs(B, H, L, n, seed):
    r = np.random.default_rng(seed)
    x = np.zeros((B, L, H, n, n), np.float32)
    for b in range(B):
        for t in range(L):
            for h in range(H):
                x[b, t, h] = np.eye(n, dtype=np.float32)
                i, j = sorted(r.choice(n, 2, replace=False))
                if t % 2:
                    i, j = j, i
                x[b, t, h, i, j] = r.choice([-1.0, 1.0])
    return x.reshape(B, L, H * n * n)


@pytest.mark.parametrize("n", NS)
@pytest.mark.parametrize("kind", ["perm", "shear"])
@pytest.mark.parametrize("chunk", [1, 5, 16, 0])
def test_exact_integer_products(n, kind, chunk):
    B, H, L = 2, 3, 41
    w = small(n, gen.MODE_RESHAPE, B=B, H=H, L=L, alpha=1.0, add_identity=0)
    x = (_perm_inputs if kind == "perm" else _shear_inputs)(B, H, L, n, seed=n + chunk)
    S_ref = oracle.scan(oracle_problem(w), x)
    assert np.abs(S_ref).max() < 2 ** 22
    S, st = run_fused(w, x, chunk=chunk)
    assert st == mru.OK
    assert np.array_equal(S.astype(np.float64), S_ref), np.argwhere(S.astype(np.float64) != S_ref)[:5]


@pytest.mark.parametrize("n", [4, 16, 64])
def test_exact_with_initial_state(n):
    B, H, L = 1, 2, 23
    w = small(n, gen.MODE_RESHAPE, B=B, H=H, L=L, alpha=1.0, add_identity=0)
    x = _perm_inputs(B, H, L, n, seed=3)
    S0 = _perm_inputs(B, 1, H, n, seed=4).reshape(B, H, n, n) * 2.0 - np.eye(n, dtype=np.float32)
    S_ref = oracle.scan(oracle_problem(w), x, S0.astype(np.float64))
    S, st = run_fused(w, x, S0=S0, chunk=4)
    assert st == mru.OK and np.array_equal(S.astype(np.float64), S_ref)


# --------------------------------------------------------------- parity ---

MODES = [gen.MODE_RESHAPE, gen.MODE_DETNORM, gen.MODE_LDU, gen.MODE_CAYLEY, gen.MODE_EXPM]


@pytest.mark.parametrize("n", NS)
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("L,chunk", [(1, 0), (15, 16), (16, 16), (17, 16), (53, 16), (97, 0)])
def test_parity_small(n, mode, L, chunk):
    w = small(n, mode, B=2, H=3, L=L, seed=100 + n + L)
    x = gen.make_x(w)
    S, st = run_fused(w, x, chunk=chunk)
    assert st == mru.OK
    e = compare_S(w, x, S)
    assert e["count"] == w.B * w.L * w.H
    assert e["max"] <= TOL_FP32, e


@pytest.mark.parametrize("n", NS)
@pytest.mark.parametrize("mode", MODES)
def test_parity_bf16_and_initial_state(n, mode):
    w = small(n, mode, B=1, H=2, L=29, x_dtype="bf16", seed=300 + n)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=301 + n)
    S, st = run_fused(w, x, S0=S0, chunk=8)
    assert st == mru.OK
    e = compare_S(w, x, S, S0=S0)
    assert e["max"] <= tol_for_problem(w, chunk=8), e


@pytest.mark.parametrize("n", [4, 16, 64])
def test_parity_far_from_identity(n):
    """Reshape without the identity and determinant correction of a matrix
    that needs pivoting: the general (not near-identity) construction."""
    for mode, add_id, alpha in ((gen.MODE_RESHAPE, 0, 1.0 / np.sqrt(n)), (gen.MODE_DETNORM, 0, 1.0),
                                (gen.MODE_DETNORM, 1, 3.0)):
        w = small(n, mode, B=1, H=2, L=19, alpha=alpha, add_identity=add_id, seed=400 + n)
        x = gen.make_x(w)
        S, st = run_fused(w, x, chunk=4)
        assert st == mru.OK
        e = compare_S(w, x, S, t_end=19)
        assert e["max"] <= TOL_FP32, (mode, add_id, e)


@pytest.mark.parametrize("chunk", [1, 2, 3, 31, 64, 1024])
def test_chunk_sizes_agree(chunk):
    w = small(16, gen.MODE_DETNORM, B=2, H=2, L=200, alpha=0.05 / 4, seed=500)
    x = gen.make_x(w)
    S, st = run_fused(w, x, chunk=chunk)
    assert st == mru.OK
    assert compare_S(w, x, S)["max"] <= TOL_FP32


@pytest.mark.parametrize("n", NS)
@pytest.mark.parametrize("mode", [gen.MODE_CAYLEY, gen.MODE_EXPM])
def test_parity_orthogonal_large_alpha(n, mode):
    """Cayley map and exponential far from the identity (the exponential
    scales and squares, with Taylor degrees up to the cap): the states stay
    orthogonal, so the fp32 gate holds over the whole sequence."""
    for alpha in (1.0, 4.0):
        w = small(n, mode, B=1, H=2, L=40, alpha=alpha, seed=420 + n)
        x = gen.make_x(w)
        S, st = run_fused(w, x, chunk=16)
        assert st == mru.OK
        e = compare_S(w, x, S)
        assert e["max"] <= TOL_FP32, (alpha, e)
        G = np.einsum("...ki,...kj->...ij", S.astype(np.float64), S.astype(np.float64))
        assert np.abs(G - np.eye(n)).max() < 1e-4


@pytest.mark.parametrize("n", NS)
def test_readout_and_snapshots(n):
    w = small(n, gen.MODE_DETNORM, B=2, H=2, L=70, seed=600 + n).with_(readout=True, snapshot_every=8)
    x = gen.make_x(w)
    u = gen.make_u(w)
    S0 = gen.make_S0(w, seed=601)
    for s0 in (None, S0):
        (o, snaps), st = run_fused(w, x, S0=s0, u=u, every=8, chunk=16)
        assert st == mru.OK and snaps.shape == (2, 8, 2, n, n)
        e = compare_readout(w, x, o, snaps, u, 8, S0=s0)
        tol = tol_for_problem(w, chunk=16)
        assert e["o"]["max"] <= tol and e["snap"]["max"] <= tol, e
    (o, snaps), st = run_fused(w, x, u=u, every=0, chunk=16)
    assert snaps is None and compare_readout(w, x, o, None, u, 0)["o"]["max"] <= tol


@pytest.mark.parametrize("n", NS)
@pytest.mark.parametrize("q,per_head,chunk", [(1, False, 16), (3, True, 16), (0, False, 16), (0, True, 0)])
def test_readout_query_columns(n, q, per_head, chunk):
    """o_t = S_t U with q query columns (q = 0 here: q = n), one U for all
    heads or one per head, over chunk boundaries and a ragged tail."""
    q = q or n
    w = small(n, gen.MODE_DETNORM, B=2, H=3, L=53, seed=640 + n + q).with_(readout=True, snapshot_every=8)
    x = gen.make_x(w)
    rng = np.random.default_rng(641 + n + q)
    U = (rng.standard_normal((w.H, n, q) if per_head else (n, q)) / np.sqrt(n)).astype(np.float32)
    (o, snaps), st = run_fused(w, x, u=U, every=8, chunk=chunk)
    assert st == mru.OK and o.shape == (w.B, w.L, w.H, n, q)
    e = compare_readout(w, x, o, snaps, U, 8)
    tol = tol_for_problem(w, chunk=chunk)
    assert e["o"]["count"] == w.B * w.L * w.H
    assert e["o"]["max"] <= tol and e["snap"]["max"] <= tol, e


@pytest.mark.parametrize("n", NS)
def test_readout_unit_columns_exact(n):
    """Permutation products read out through unit query columns (a different
    column set per head) are picked columns of S_t, exactly."""
    B, H, L = 2, 2, 37
    w = small(n, gen.MODE_RESHAPE, B=B, H=H, L=L, alpha=1.0, add_identity=0).with_(readout=True)
    x = _perm_inputs(B, H, L, n, seed=650 + n)
    S_ref = oracle.scan(oracle_problem(w), x)
    cols = [[n - 1, 0, n // 2], [1, 1, n - 2]]
    U = np.stack([np.eye(n, dtype=np.float32)[:, c] for c in cols])
    (o, _), st = run_fused(w, x, u=U, chunk=16)
    assert st == mru.OK
    for h in range(H):
        assert np.array_equal(o[:, :, h].astype(np.float64), S_ref[:, :, h][..., cols[h]])


@pytest.mark.parametrize("chunk", [16, 32])
def test_n64_determinant_series_and_lu_tokens_mixed(chunk):
    """n = 64 readout in the determinant-corrected mode near the identity:
    most tokens take the scale from the trace series on the tensor cores;
    tokens t = 1 mod 3 (slice scaled by 6, |E|_F about 1.4) fail the series'
    certificate and are factorised instead, tokens t = 2 mod 5 (scaled by
    60, pivots far from 1) need the pivoted LU."""
    n = 64
    w = small(n, gen.MODE_DETNORM, B=1, H=2, L=90, alpha=0.03 / np.sqrt(n), seed=660).with_(readout=True,
                                                                                          snapshot_every=8)
    x = gen.make_x(w).reshape(w.B, w.L, w.H * n * n).copy()
    x[:, 1::3] *= 6.0
    x[:, 2::5] *= 60.0
    u = gen.make_u(w)
    (o, snaps), st = run_fused(w, x, u=u, every=8, chunk=chunk)
    assert st == mru.OK
    e = compare_readout(w, x, o, snaps, u, 8)
    tol = tol_for_problem(w, chunk=chunk)
    assert e["o"]["count"] == w.B * w.L * w.H
    assert e["o"]["max"] <= tol and e["snap"]["max"] <= tol, e


def _near_permutation_x(w, seed, with_identity):
    """Embeddings whose X~ = I + 0.03 N(0, 1), with the rows of every fifth
    token rotated by one (a zero-ish diagonal: the construction must pivot);
    with_identity=False stores X~ - I (for add_identity = 1).  Products stay
    within fp32 range over thousands of tokens, unlike Gaussian X~."""
    r = np.random.default_rng(seed)
    n = w.n
    X = np.eye(n) + 0.03 * r.standard_normal((w.B, w.L, w.H, n, n))
    rot = np.arange(w.L) % 5 == 3
    X[:, rot] = np.roll(X[:, rot], 1, axis=-2)
    if not with_identity:
        X -= np.eye(n)
    x = X.astype(np.float32).reshape(w.B, w.L, w.H * n * n)
    return gen.f32_to_bf16_bits(x) if w.x_dtype == "bf16" else x


# (mode, add_identity, alpha, embeddings): Gaussian near the identity, or the
# rotated near-permutations above for the pivoting constructions
SMALL_CASES = [(gen.MODE_RESHAPE, 1, 0.05, "gauss"), (gen.MODE_RESHAPE, 0, 1.0, "perm"),
               (gen.MODE_DETNORM, 1, 0.05, "gauss"), (gen.MODE_DETNORM, 0, 1.0, "perm"),
               (gen.MODE_DETNORM, 1, 1.0, "perm"), (gen.MODE_LDU, 1, 0.05, "gauss")]


@pytest.mark.parametrize("mode,add_id,alpha,emb", SMALL_CASES)
@pytest.mark.parametrize("L", [1, 255, 257, 1000, 4099])
@pytest.mark.parametrize("x_dtype,with_s0", [("f32", False), ("bf16", True)])
def test_small_problems_one_launch(mode, add_id, alpha, emb, L, x_dtype, with_s0):
    """n = 4 with the automatic chunk runs in one launch (each thread a
    segment of tokens, the segment products scanned across the CTA): every
    construction it takes (near-identity and pivoted determinant correction
    included), segments that are full, partial and empty, with and without
    S0, against the oracle over every token."""
    w = small(4, mode, B=2, H=3, L=L, x_dtype=x_dtype, alpha=alpha, add_identity=add_id, seed=900 + L)
    p = mru.problem_from_workload(w)
    assert mru.launch_count(p) == 1 and mru.kernel_names(p) == ["k_small_scan"]
    x = gen.make_x(w) if emb == "gauss" else _near_permutation_x(w, 902 + L, with_identity=not add_id)
    S0 = gen.make_S0(w, seed=901) if with_s0 else None
    S, st = run_fused(w, x, S0=S0)
    assert st == mru.OK
    e = compare_S(w, x, S, S0=S0)
    assert e["count"] == w.B * w.L * w.H
    assert e["max"] <= TOL_FP32, e


def test_small_problems_singular_and_lifted_input():
    """The one-launch path reports a singular determinant-corrected matrix
    (the other heads stay within tolerance), and scans lifted matrices X
    (mru_scan)."""
    t = torch()
    w = small(4, gen.MODE_DETNORM, B=1, H=2, L=300, alpha=1.0, add_identity=0, seed=950)
    x = _near_permutation_x(w, 950, with_identity=True)
    x[0, 123, 16:32] = 0.0                      # head 1, token 123: X~ = 0
    S, st = run_fused(w, x)
    assert st == mru.ERR_SINGULAR and np.isfinite(S).all()
    assert compare_S(w, x, S, bh=[0])["max"] <= TOL_FP32
    w = small(4, gen.MODE_LDU, B=2, H=2, L=700, seed=951)
    x = gen.make_x(w)
    for smi in (0, 1):
        p = mru.problem_from_workload(w, store_minus_identity=smi)
        assert mru.kernel_names(p) == ["k_small_scan"]
        S = mru.scan_t(p, mru.build_states_t(p, to_device_x(x))).cpu().numpy()
        assert compare_S(w, x, S)["max"] <= TOL_FP32


@pytest.mark.parametrize("n", [4, 16, 32])
@pytest.mark.parametrize("mode", MODES)
def test_unfused_build_then_scan(n, mode):
    t = torch()
    w = small(n, mode, B=1, H=3, L=45, seed=700 + n)
    x = gen.make_x(w)
    S_fused, _ = run_fused(w, x, chunk=8)
    for smi in (0, 1):
        p = mru.problem_from_workload(w, chunk=8, store_minus_identity=smi)
        X = mru.build_states_t(p, to_device_x(x))
        t.cuda.synchronize()
        # lifted matrices against the oracle's X_t
        Xh = X.cpu().numpy().astype(np.float64)
        for (tt, h) in ((0, 0), (17, 2), (44, 1)):
            ref = oracle.lift(oracle_problem(w), x, 0, tt, h)
            got = Xh[0, tt, h] + (np.eye(n) if smi else 0.0)
            assert np.abs(got - ref).max() <= 2e-6 * max(1.0, np.abs(ref).max())
        S = mru.scan_t(p, X).cpu().numpy()
        assert compare_S(w, x, S)["max"] <= TOL_FP32
        np.testing.assert_allclose(S, S_fused, rtol=0, atol=5e-5 * np.abs(S_fused).max())


def test_empty_and_degenerate_shapes():
    t = torch()
    for B, H, L in ((0, 2, 5), (2, 0, 5), (2, 2, 0)):
        p = mru.problem(B, H, L, 16, mode=gen.MODE_DETNORM, alpha=0.01)
        x = t.zeros((max(B, 1), max(L, 1), max(H, 1) * 256), device="cuda")
        out = t.empty((max(B, 1), max(L, 1), max(H, 1), 16, 16), device="cuda")
        ws = mru.workspace_t(p)
        assert mru.scan_fused(p, x.data_ptr(), None, None, out.data_ptr(), None, ws.data_ptr(), ws.numel(),
                              t.cuda.current_stream().cuda_stream) == mru.OK
        assert mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream) == mru.OK


def test_singular_matrix_reported():
    w = small(16, gen.MODE_DETNORM, B=1, H=2, L=9, alpha=1.0, add_identity=0)
    x = gen.make_x(w)
    x[0, 4, 256:512] = 0.0                      # head 1, token 4: X~ = 0
    S, st = run_fused(w, x, chunk=4)
    assert st == mru.ERR_SINGULAR
    assert np.isfinite(S).all()
    # the other head is unaffected
    e = compare_S(w, x, S, bh=[0])
    assert e["max"] <= TOL_FP32


def test_status_resets_between_calls():
    w = small(16, gen.MODE_DETNORM, B=1, H=1, L=5, alpha=1.0, add_identity=0)
    x = gen.make_x(w)
    x0 = x.copy()
    x0[0, 2] = 0.0
    _, st = run_fused(w, x0)
    assert st == mru.ERR_SINGULAR
    _, st = run_fused(w, x)
    assert st == mru.OK


@pytest.mark.parametrize("n,mode,dtype", [(32, gen.MODE_LDU, "bf16"), (16, gen.MODE_DETNORM, "f32"),
                                           (64, gen.MODE_DETNORM, "f32")])
def test_repeated_calls_are_deterministic(n, mode, dtype):
    w = small(n, mode, B=2, H=4, L=300, x_dtype=dtype, seed=800)
    x = gen.make_x(w)
    first, _ = run_fused(w, x)
    for _ in range(5):
        again, _ = run_fused(w, x)
        assert np.array_equal(first, again)


@pytest.mark.parametrize("L,chunk", [(1, 0), (7, 8), (8, 8), (9, 8), (100, 0), (300, 64), (129, 16)])
@pytest.mark.parametrize("add_s0", [False, True])
def test_parity_n32_ldu_tensor_path(L, chunk, add_s0):
    """The bf16 tensor-core LDU kernels at n = 32: ragged chunks, S0."""
    w = small(32, gen.MODE_LDU, B=2, H=3, L=L, x_dtype="bf16", seed=900 + L)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=901) if add_s0 else None
    p = mru.problem_from_workload(w, chunk=chunk)
    assert mru.effective_math(p) == "bf16x3"
    S, st = run_fused(w, x, S0=S0, chunk=chunk)
    assert st == mru.OK
    e = compare_S(w, x, S, S0=S0)
    assert e["count"] == w.B * w.L * w.H
    assert e["max"] <= tol_for_problem(w, chunk=chunk), e


@pytest.mark.parametrize("L,chunk", [(1, 0), (7, 8), (16, 8), (17, 8), (100, 0), (333, 32)])
def test_parity_n16_tensor_path(L, chunk):
    """The split-tf32 tensor-core kernels at n = 16 (fp32-accurate gate)."""
    w = small(16, gen.MODE_DETNORM, B=2, H=3, L=L, alpha=0.05 / 4, seed=950 + L)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=951)
    p = mru.problem_from_workload(w, chunk=chunk)
    assert mru.effective_math(p) == "tf32x3"
    S, st = run_fused(w, x, S0=S0, chunk=chunk)
    assert st == mru.OK
    e = compare_S(w, x, S, S0=S0)
    assert e["max"] <= TOL_FP32, e


@pytest.mark.parametrize("B,H,L,chunk,mode,add_identity", [
    (1, 2, 2059, 8, gen.MODE_DETNORM, 1),       # 258 chunk totals: two levels below the top
    (1, 1, 32800, 8, gen.MODE_DETNORM, 1),      # 4100 chunk totals: three levels
    (2, 3, 41, 8, gen.MODE_DETNORM, 0),         # per-token scales in the reduce pass (short: these
                                                # chains grow about e^0.4 a token)
    (2, 2, 530, 16, gen.MODE_RESHAPE, 1),
    (1, 3, 203, 8, gen.MODE_RESHAPE, 0),
])
def test_parity_n16_carry_levels(B, H, L, chunk, mode, add_identity):
    """n = 16 tensor-core path: the in-launch carry scan over one to three
    levels of groups, ragged last groups, both modes, with and without the
    identity."""
    # near identity with the identity added; alpha M of spectral radius about
    # 1 without it (the determinant-corrected mode is scale free)
    alpha = (0.05 / 4 if mode == gen.MODE_DETNORM else 0.01) if add_identity else 0.25
    w = small(16, mode, B=B, H=H, L=L, alpha=alpha, add_identity=add_identity, seed=970 + L)
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=971)
    assert mru.effective_math(mru.problem_from_workload(w, chunk=chunk)) == "tf32x3"
    S, st = run_fused(w, x, S0=S0, chunk=chunk)
    assert st == mru.OK
    e = compare_S(w, x, S, S0=S0)
    assert e["count"] == B * H * L
    assert e["max"] <= TOL_FP32, e


@pytest.mark.parametrize("mode,add_id,L,chunk", [(gen.MODE_DETNORM, 1, 130, 16), (gen.MODE_RESHAPE, 1, 53, 16),
                                                 (gen.MODE_DETNORM, 1, 257, 0)])
@pytest.mark.parametrize("with_s0", [False, True])
def test_n64_every_state_on_the_tensor_cores(mode, add_id, L, chunk, with_s0):
    """n = 64 without the readout, tf32 asked for: the readout path's chunk
    kernel records every Q_t as a snapshot and its fix-up writes
    S_t = C + C Q_t for every token.  Every state within the tf32 gate."""
    w = small(64, mode, B=2, H=3, L=L, add_identity=add_id, alpha=0.03 / 8, seed=770 + L).with_(math="tf32")
    p = mru.problem_from_workload(w, chunk=chunk)
    assert mru.kernel_names(p)[0] == "k64_chunk_readout"
    x = gen.make_x(w)
    S0 = gen.make_S0(w, seed=771) if with_s0 else None
    S, st = run_fused(w, x, S0=S0, chunk=chunk)
    assert st == mru.OK
    e = compare_S(w, x, S, S0=S0)
    assert e["count"] == w.B * w.L * w.H
    assert e["max"] <= tol_for_problem(w, chunk=chunk), e
