"""Host checks of the determinant scale the n = 64 chunk kernel computes on
the tensor cores (no GPU; numpy restatements of the kernel's arithmetic).

For X = I + E, E = alpha M, the kernel takes
    log det X = tr E - tr E^2 / 2 + tr E^3 / 3 - tr E^4 / 4 + R
with tr E^k = <E^(k-1), E^T> from bf16 products M2 = M M, M3 = M2 M, and
accepts it when the remainder bound
    |R| <= |E^3|_F |E^2|_F / (5 (1 - |E|_F))        (|E|_F < 1)
is at most 1e-6; otherwise it factorises (LU).  These tests pin the series
against numpy's slogdet, the bound against the true remainder, the
acceptance at the benchmark's alpha, the rejection far from the identity,
and the integer-operation tf32 rounding (round to nearest, ties away) the
kernels use for the chain's tensor-core operands.

The n = 64 backward (k64b_apply) forms the same series from P2 = (M^T)^2 and
P3 = P2 M^T, and from them the chain rule's inverse
    Xr^-T = I - E^T + (E^T)^2 - (E^T)^3 + R,  |R|_F <= |E^3|_F |E|_F / (1 - |E|_F),
taken when that bound is at most 1e-3: the last tests pin the transposed
traces, the inverse against numpy's, its bound, acceptance and rejection."""
import numpy as np

N = 64
TAU = 1e-6


def tf32_round(a):
    """The kernels' rounding: (bits + 0x1000) & 0xffffe000 on the fp32 bits."""
    b = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
    return (((b + 0x1000) & 0xFFFFE000).astype(np.uint32)).view(np.float32)


def tf32_reference(a):
    """Round to 11 significant bits, ties away from zero, from frexp."""
    a = np.asarray(a, np.float64)
    m, e = np.frexp(a)                      # a = m 2^e, 0.5 <= |m| < 1
    s = np.sign(m) * np.floor(np.abs(m) * 2.0 ** 11 + 0.5) / 2.0 ** 11
    return (s * 2.0 ** e).astype(np.float32)


def bf16_round(a):
    """Round to bf16, nearest even (cvt.rn.bf16x2.f32)."""
    b = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def series(M, alpha, rounded=True):
    r = bf16_round if rounded else (lambda a: a)
    M = M.astype(np.float64)
    M2 = r(M).astype(np.float64) @ r(M).astype(np.float64)
    M3 = r(M2).astype(np.float64) @ r(M).astype(np.float64)
    t = [np.trace(M), np.sum(M * M.T), np.sum(M2 * M.T), np.sum(M3 * M.T)]
    ld = alpha * t[0] - alpha ** 2 * t[1] / 2 + alpha ** 3 * t[2] / 3 - alpha ** 4 * t[3] / 4
    fe = alpha * np.linalg.norm(M)
    bound = (alpha ** 3 * np.linalg.norm(M3)) * (alpha ** 2 * np.linalg.norm(M2)) / (5 * (1 - fe)) \
        if fe < 1 else np.inf
    return ld, bound


def test_tf32_rounding_is_nearest_ties_away():
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        (rng.standard_normal(2000) * 1e-30).astype(np.float32),
                        (rng.standard_normal(2000) * 1e30).astype(np.float32),
                        # exact ties: 12 significant bits ending in 1
                        np.float32((2 ** 11 + 2 * np.arange(1, 200) + 1)) * np.float32(2.0 ** -7)])
    np.testing.assert_array_equal(tf32_round(v), tf32_reference(v))
    assert tf32_round(np.float32(1.0 + 2.0 ** -11)) == np.float32(1.0 + 2.0 ** -10)   # tie away
    assert tf32_round(np.float32(-(1.0 + 2.0 ** -11))) == np.float32(-(1.0 + 2.0 ** -10))


def test_series_matches_slogdet_within_the_bound_exact_products():
    """Exact products: the truncation error never exceeds the bound."""
    rng = np.random.default_rng(12)
    for alpha in (0.002, 0.00375, 0.0045):
        for _ in range(40):
            M = rng.standard_normal((N, N)).astype(np.float32)
            ld, bound = series(M, alpha, rounded=False)
            true = np.linalg.slogdet(np.eye(N) + alpha * M.astype(np.float64))[1]
            assert abs(ld - true) <= bound


def test_series_accepted_at_benchmark_alpha_and_accurate_with_bf16_products():
    rng = np.random.default_rng(13)
    alpha = 0.03 / np.sqrt(N)
    for _ in range(60):
        M = rng.standard_normal((N, N)).astype(np.float32)
        ld, bound = series(M, alpha)
        assert bound <= TAU
        true = np.linalg.slogdet(np.eye(N) + alpha * M.astype(np.float64))[1]
        assert abs(ld - true) <= 2e-7        # c = exp(-ld / 64) good to 3e-9


def test_series_rejected_far_from_identity():
    rng = np.random.default_rng(14)
    for alpha in (0.3 / np.sqrt(N), 0.02, 0.2):
        M = rng.standard_normal((N, N)).astype(np.float32)
        _, bound = series(M, alpha)
        assert not bound <= TAU


def test_series_sign_and_terms_are_all_needed():
    """Dropping any one trace term (or flipping its sign) moves log det far
    beyond the acceptance bound at the benchmark's alpha."""
    rng = np.random.default_rng(15)
    alpha = 0.03 / np.sqrt(N)
    M = rng.standard_normal((N, N)).astype(np.float64)
    M2, M3 = M @ M, M @ M @ M
    t = np.array([np.trace(M), np.sum(M * M.T), np.sum(M2 * M.T), np.sum(M3 * M.T)])
    w = np.array([alpha, -alpha ** 2 / 2, alpha ** 3 / 3, -alpha ** 4 / 4])
    true = np.linalg.slogdet(np.eye(N) + alpha * M)[1]
    assert abs(w @ t - true) < 1e-7
    for k in range(3):               # the fourth term is itself below the bound's scale
        ww = w.copy()
        ww[k] = -ww[k]
        assert abs(ww @ t - true) > 1e-6


# ---- the n = 64 backward (k64b_apply): the same series on transposed
# products, and the chain rule's inverse from them ----
INV_TAU = 1e-3


def transposed_products(M, rounded=True):
    """P2 = (M^T)^2 and P3 = P2 M^T as the backward kernels form them (bf16
    operands, wide accumulation)."""
    r = bf16_round if rounded else (lambda a: a)
    Mt = r(M.astype(np.float32).T).astype(np.float64)
    P2 = Mt @ Mt
    P3 = r(P2).astype(np.float64) @ Mt
    return P2, P3


def inverse_series(M, alpha, rounded=True):
    """Xr^-T ~ I - E^T + alpha^2 P2 - alpha^3 P3 and the bound on the dropped
    tail, |E^3|_F |E|_F / (1 - |E|_F)."""
    P2, P3 = transposed_products(M, rounded)
    Z = np.eye(N) - alpha * M.astype(np.float64).T + alpha ** 2 * P2 - alpha ** 3 * P3
    fe = alpha * np.linalg.norm(M.astype(np.float64))
    bound = (alpha ** 3 * np.linalg.norm(P3)) * fe / (1 - fe) if fe < 1 else np.inf
    return Z, bound


def test_transposed_products_give_the_same_traces_and_norms():
    """tr M^3 = <P2, M>, tr M^4 = <P3, M>, |M^2|_F = |P2|_F and |M^3|_F =
    |P3|_F for P2 = (M^T)^2, P3 = (M^T)^3: the backward's series equals the
    forward's."""
    rng = np.random.default_rng(21)
    M = rng.standard_normal((N, N)).astype(np.float32).astype(np.float64)     # exact in fp32, as the slices are
    P2, P3 = transposed_products(M, rounded=False)
    M2, M3 = M @ M, M @ M @ M
    np.testing.assert_allclose(np.sum(P2 * M), np.trace(M3), rtol=1e-10)
    np.testing.assert_allclose(np.sum(P3 * M), np.trace(M3 @ M), rtol=1e-10)
    np.testing.assert_allclose(np.linalg.norm(P2), np.linalg.norm(M2), rtol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(P3), np.linalg.norm(M3), rtol=1e-12)
    # and not the untransposed pairing: <M2, M> is tr(M^2 M^T), a different number
    assert abs(np.sum(M2 * M) - np.trace(M3)) > 1e-3 * abs(np.trace(M3)) + 1.0


def test_inverse_series_within_its_bound_exact_products():
    rng = np.random.default_rng(22)
    for alpha in (0.002, 0.00375, 0.006):
        for _ in range(20):
            M = rng.standard_normal((N, N)).astype(np.float32)
            Z, bound = inverse_series(M, alpha, rounded=False)
            true = np.linalg.inv(np.eye(N) + alpha * M.astype(np.float64)).T
            assert np.linalg.norm(Z - true) <= bound


def test_inverse_series_accepted_at_benchmark_alpha_and_accurate_with_bf16_products():
    rng = np.random.default_rng(23)
    alpha = 0.03 / np.sqrt(N)
    for _ in range(30):
        M = rng.standard_normal((N, N)).astype(np.float32)
        Z, bound = inverse_series(M, alpha)
        assert bound <= INV_TAU
        true = np.linalg.inv(np.eye(N) + alpha * M.astype(np.float64)).T
        assert np.linalg.norm(Z - true) / np.linalg.norm(true) <= 2e-5


def test_inverse_series_rejected_far_from_identity():
    rng = np.random.default_rng(24)
    for alpha in (0.3 / np.sqrt(N), 0.05, 0.2):
        M = rng.standard_normal((N, N)).astype(np.float32)
        _, bound = inverse_series(M, alpha)
        assert not bound <= INV_TAU


def test_inverse_series_each_term_needed():
    """Dropping or flipping any of the three terms beyond I moves the inverse
    by more than the bound at the benchmark's alpha."""
    rng = np.random.default_rng(25)
    alpha = 0.03 / np.sqrt(N)
    M = rng.standard_normal((N, N)).astype(np.float32)
    P2, P3 = transposed_products(M, rounded=False)
    Mt = M.astype(np.float64).T
    true = np.linalg.inv(np.eye(N) + alpha * M.astype(np.float64)).T
    terms = [-alpha * Mt, alpha ** 2 * P2, -alpha ** 3 * P3]
    _, bound = inverse_series(M, alpha, rounded=False)
    for k in range(3):
        Z = np.eye(N) + sum(-t if i == k else t for i, t in enumerate(terms))
        assert np.linalg.norm(Z - true) > bound
