"""Shared helpers of the GPU parity tests: run the CUDA path through the
C-ABI binding and compare with the fp64 oracle on the same input bytes."""
from __future__ import annotations

import numpy as np

import oracle
from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

# Relative Frobenius gates, per output matrix (max over every compared
# (b, t, h)): fp32 paths 1e-4, tf32 / bf16 tensor-core paths 1e-2.
TOL_FP32 = 1e-4
TOL_TENSOR = 1e-2


def tol_for(math: str) -> float:
    """Gate by the arithmetic the chosen kernels use: split-tf32 keeps fp32
    accuracy (1e-4); single tf32 and split-bf16 tensor paths get 1e-2."""
    return TOL_TENSOR if math in ("tf32", "bf16", "bf16x3") else TOL_FP32


def tol_for_problem(w, **over) -> float:
    p = mru.problem_from_workload(w, **over)
    return tol_for(mru.effective_math(p, w.readout))


def torch():
    import torch as t
    return t


def to_device_x(x_np: np.ndarray):
    t = torch()
    if x_np.dtype == np.uint16:
        return t.from_numpy(x_np.view(np.int16)).cuda().view(t.bfloat16)
    return t.from_numpy(np.ascontiguousarray(x_np)).cuda()


def oracle_problem(w: gen.Workload):
    return oracle.make_problem(w.B, w.H, w.L, w.n, x_dtype=w.x_dtype, mode=w.mode, alpha=w.alpha,
                               add_identity=w.add_identity, ldu_offdiag=w.ldu_offdiag, ldu_diag=w.ldu_diag)


def run_fused(w: gen.Workload, x_np, *, S0=None, chunk=0, u=None, every=0, math=None):
    """Returns S (numpy [B, L, H, n, n]) or (o, snapshots) and the device status."""
    t = torch()
    p = mru.problem_from_workload(w, chunk=chunk, **({} if math is None else {"math": math}))
    x = to_device_x(x_np)
    S0_t = None if S0 is None else t.from_numpy(np.ascontiguousarray(S0, np.float32)).cuda()
    ws = mru.workspace_t(p)
    if u is None:
        S = mru.scan_fused_t(p, x, S0=S0_t, ws=ws)
        status = mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream)
        return S.cpu().numpy(), status
    u_t = t.from_numpy(np.ascontiguousarray(u, np.float32)).cuda()
    o, snaps = mru.scan_fused_t(p, x, S0=S0_t, u=u_t, snapshot_every=every, ws=ws)
    status = mru.last_device_status(ws.data_ptr(), t.cuda.current_stream().cuda_stream)
    return (o.cpu().numpy(), None if snaps is None else snaps.cpu().numpy()), status


def compare_S(w, x_np, S_gpu, *, S0=None, bh=None, t_end=None):
    res = oracle.compare(oracle_problem(w), x_np, S0=None if S0 is None else S0.astype(np.float64),
                         bh=bh, t_end=t_end, S_gpu=S_gpu)
    return oracle.error_stats(*res["S"])


def compare_readout(w, x_np, o_gpu, snaps_gpu, u, every, *, S0=None, bh=None):
    res = oracle.compare(oracle_problem(w), x_np, S0=None if S0 is None else S0.astype(np.float64), bh=bh,
                         u=u.astype(np.float64), o_gpu=o_gpu, snapshot_every=every if snaps_gpu is not None else 0,
                         snap_gpu=snaps_gpu)
    out = {"o": oracle.error_stats(*res["o"])}
    if "snap" in res:
        out["snap"] = oracle.error_stats(*res["snap"])
    return out
