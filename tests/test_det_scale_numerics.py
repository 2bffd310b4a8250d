"""Host emulation of the n = 16 apply pass's per-token determinant scale, in
fp32 as the kernel takes it: elimination of X~ = I + E on E alone without
pivoting (pivots 1 + delta_k), |det| as the fp32 product of the 16 pivots,
c - 1 = expm1(-log1p(u) / 16) with u = |det| - 1.  Against fp64 slogdet at the
default workload's alpha the scale is good to about 1e-8 (the error the
design relies on: unbiased, adding as a random walk along the sequence), and
the near-identity branch is the one taken (no pivot below 0.5)."""
from __future__ import annotations

import numpy as np

from linear_rnn_scan_b200 import inputs as gen


def _scale_minus_one_fp32(E):
    f32 = np.float32
    W = E.astype(f32).copy()
    n = W.shape[-1]
    for k in range(n):
        r = (f32(1) / (f32(1) + W[:, k, k])).astype(f32)
        lk = (W[:, k + 1:, k] * r[:, None]).astype(f32)
        W[:, k + 1:, k + 1:] = (W[:, k + 1:, k + 1:] - (lk[:, :, None] * W[:, k, None, k + 1:]).astype(f32)).astype(f32)
    piv = np.stack([W[:, k, k] for k in range(n)], 1)
    prod = np.ones(W.shape[0], f32)
    for k in range(n):
        prod = (prod * (f32(1) + piv[:, k])).astype(f32)
    u = (np.abs(prod) - f32(1)).astype(f32)
    cm1 = np.expm1((-np.log1p(u) / f32(n)).astype(f32)).astype(f32)
    return cm1, piv


def test_fp32_determinant_scale_is_good_to_1e_8():
    w = gen.WORKLOADS["n16_detnorm_b8h8l4096"]
    n = w.n
    M = gen.randn_f32((3000, n, n), 77)
    E = (np.float32(w.alpha) * M).astype(np.float32)
    cm1, piv = _scale_minus_one_fp32(E)
    assert (np.abs(1.0 + piv) >= 0.5).all()
    _, logdet = np.linalg.slogdet(np.eye(n) + E.astype(np.float64))
    err = np.abs(cm1.astype(np.float64) - np.expm1(-logdet / n))
    assert err.max() < 1e-7 and np.median(err) < 2e-8, (err.max(), np.median(err))
    # unbiased: the signed errors average out
    signed = cm1.astype(np.float64) - np.expm1(-logdet / n)
    assert abs(signed.mean()) < 5 * signed.std() / np.sqrt(signed.size)
