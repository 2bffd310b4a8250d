"""GPU parity of the single-read n = 16 kernel (one launch of mru_scan_fused
for n = 16, fp32 embeddings, reshape / determinant-corrected / Cayley modes,
more than one chunk per sequence; opt-in with MRU_N16_FUSED=1) against the
fp64 oracle, and its bounded waits.

The kernel hands out reduce and apply items from one ticket counter; group
scans and a decoupled look-back over groups of chunks give every chunk its
carry.  The cases here make the look-back long (many groups per sequence,
short chunks), leave ragged tails (last chunk and last group partial), start
from S0, use several batches and heads, and grow the group size past 16 (more
than 65,536 chunks in one sequence).  The timeout case withholds one group's
carry through the library's testing hook: every wait then gives up after its
limit, the status word says so, and the next call on the same context is
correct again."""
from __future__ import annotations

import os

import numpy as np
import pytest

from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

from gpu_helpers import TOL_FP32, compare_S, run_fused, torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    mru.load()
    old = os.environ.get("MRU_N16_FUSED")
    os.environ["MRU_N16_FUSED"] = "1"            # the kernel is opt-in; read by the library at each call
    yield
    if old is None:
        os.environ.pop("MRU_N16_FUSED", None)
    else:
        os.environ["MRU_N16_FUSED"] = old


def wl(B, H, L, mode, *, alpha=0.0125, add_identity=1, seed=11):
    return gen.Workload("fused16", B=B, H=H, L=L, n=16, x_dtype="f32", mode=mode, alpha=float(alpha),
                        add_identity=add_identity, seed=seed)


def check_single_launch(w, chunk):
    p = mru.problem_from_workload(w, chunk=chunk)
    assert mru.launch_count(p) == 1
    assert mru.kernel_names(p) == ["k16_fused"]


CASES = [
    # B, H, L, chunk, mode, add_identity, alpha
    (1, 1, 8 * 16 * 9 + 5, 8, gen.MODE_DETNORM, 1, 0.0125),     # 10 groups, ragged chunk and group
    (2, 3, 8 * 16 * 5, 8, gen.MODE_RESHAPE, 1, 0.05),          # whole groups, several heads and batches
    (3, 2, 161, 8, gen.MODE_DETNORM, 0, 0.3),                  # corrected without the identity (short:
                                                               # its products leave the fp32 range later)
    (1, 4, 8 * 16 * 3 + 8, 8, gen.MODE_CAYLEY, 1, 0.2),        # Cayley map, one-chunk last group
    (4, 8, 2049, 32, gen.MODE_DETNORM, 1, 0.0125),             # many sequences, short look-backs
    (1, 1, 16 * 8 * 40, 8, gen.MODE_DETNORM, 1, 0.005),        # 40 groups in one sequence
]


@pytest.mark.parametrize("B,H,L,chunk,mode,add_identity,alpha", CASES)
@pytest.mark.parametrize("with_s0", [False, True])
def test_fused_against_oracle(B, H, L, chunk, mode, add_identity, alpha, with_s0):
    w = wl(B, H, L, mode, alpha=alpha, add_identity=add_identity, seed=B * 100 + L)
    check_single_launch(w, chunk)
    x = gen.make_x(w)
    S0 = None
    if with_s0:
        r = np.random.default_rng(L)
        S0 = (np.eye(16) + 0.1 * r.standard_normal((B, H, 16, 16))).astype(np.float32)
    S, st = run_fused(w, x, S0=S0, chunk=chunk)
    assert st == mru.OK
    e = compare_S(w, x, S, S0=S0)
    assert e["count"] == B * H * L
    assert e["max"] <= TOL_FP32, e


def test_fused_exact_permutation_chain_many_groups():
    """Permutation matrices make every product exact: the fused kernel must
    return the oracle's states bit for bit over 20 groups of chunks (any
    mistake in the look-back order, the in-group prefixes or the carry shows
    as a wrong permutation)."""
    B, H, L, n = 1, 2, 8 * 16 * 20 + 3, 16
    w = gen.Workload("perm16", B=B, H=H, L=L, n=n, x_dtype="f32", mode=gen.MODE_RESHAPE, alpha=1.0,
                     add_identity=0, seed=3)
    r = np.random.default_rng(5)
    x = np.zeros((B, L, H, n, n), np.float32)
    for t in range(L):
        for h in range(H):
            x[0, t, h, np.arange(n), r.permutation(n)] = 1.0
    x = x.reshape(B, L, H * n * n)
    check_single_launch(w, 8)
    S, st = run_fused(w, x, chunk=8)
    assert st == mru.OK
    S_ref = oracle.scan(oracle.make_problem(B, H, L, n, mode=gen.MODE_RESHAPE, alpha=1.0, add_identity=0), x)
    assert np.array_equal(S.astype(np.float64), S_ref)


def test_fused_group_size_above_16():
    """More than 65,536 chunks in one sequence: the groups grow to 32 chunks
    (the look-back passes at most 4,096 groups).  Every state is compared
    with the oracle."""
    L = 8 * 65536 + 200
    w = wl(1, 1, L, gen.MODE_DETNORM, alpha=0.003, seed=19)    # the states stay within the fp32 range
    check_single_launch(w, 8)
    x = gen.make_x(w)
    S, st = run_fused(w, x, chunk=8)
    assert st == mru.OK
    e = compare_S(w, x, S)
    assert e["count"] == L
    assert e["max"] <= TOL_FP32, e


def test_fused_wait_timeout_reported_and_context_recovers():
    """The testing hook withholds the first group's carry: the apply items of
    that group can never start, every wait gives up after 50 ms, the launch
    ends early and the status word reads ERR_TIMEOUT.  The same context then
    runs the same problem correctly."""
    t = torch()
    w = wl(2, 2, 8 * 16 * 4 + 7, gen.MODE_DETNORM, seed=23)
    x = gen.make_x(w)
    p = mru.problem_from_workload(w, chunk=8)
    xd = t.from_numpy(x).cuda()
    ws = mru.workspace_t(p)
    stream = t.cuda.current_stream().cuda_stream
    mru.debug_stall_next_fused(50)
    S = mru.scan_fused_t(p, xd, ws=ws)
    assert mru.last_device_status(ws.data_ptr(), stream) == mru.ERR_TIMEOUT
    S = mru.scan_fused_t(p, xd, ws=ws)
    assert mru.last_device_status(ws.data_ptr(), stream) == mru.OK
    e = compare_S(w, x, S.cpu().numpy())
    assert e["max"] <= TOL_FP32, e
