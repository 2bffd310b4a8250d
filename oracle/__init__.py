"""fp64 CPU oracle for the MRU prefix-product scan (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does, and this
package imports nothing from the product: it shares no code with the CUDA
library.  Callers hand it plain numpy arrays.

The arithmetic lives in ``mru_oracle.c`` (plain C, fp64, serial product);
this module compiles it with gcc on first use and wraps it with ctypes.

Pages followed (see ``mru_oracle.c`` for the readings adopted):
  * "MRU Update: An independent developer's alternative to Attention is now
    running successfully", section "What MRU Actually Does" -- lift, cumulative
    product S_t = S_{t-1} X_t, reduction;
  * "Improving Matrix Recurrent Units as an Attention Alternative", sections
    "Key Points" and "Technical Deep Dive" -- determinant-correcting scalar,
    LDU factor filling.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mru_oracle.c")
_LIB = os.path.join(_HERE, "libmru_oracle.so")
_lock = threading.Lock()
_lib = None

MODE_RESHAPE, MODE_DETNORM, MODE_LDU, MODE_CAYLEY, MODE_EXPM = 0, 1, 2, 3, 4
DTYPE_F32, DTYPE_BF16 = 0, 1
OK, ERR_ARG, ERR_SINGULAR = 0, 1, 5


class Problem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int64), ("H", ctypes.c_int64), ("L", ctypes.c_int64),
        ("n", ctypes.c_int32), ("x_dtype", ctypes.c_int32), ("mode", ctypes.c_int32),
        ("alpha", ctypes.c_float), ("add_identity", ctypes.c_int32),
        ("ldu_offdiag", ctypes.c_float), ("ldu_diag", ctypes.c_float),
    ]


def build(force: bool = False) -> str:
    """Compile mru_oracle.c into libmru_oracle.so (no optimisation that
    changes floating-point semantics: -O2 without fast-math or contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-shared", "-fPIC",
               "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER
            vp, dp, fp, i64p = ctypes.c_void_p, P(ctypes.c_double), P(ctypes.c_float), P(ctypes.c_int64)
            lib.mro_lift.argtypes = [P(Problem), vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, dp, dp]
            lib.mro_lift.restype = ctypes.c_int
            lib.mro_scan.argtypes = [P(Problem), vp, dp, dp, ctypes.c_int]
            lib.mro_scan.restype = ctypes.c_int
            ci = ctypes.c_int
            lib.mro_readout.argtypes = [P(Problem), vp, dp, dp, ci, ci, dp, ctypes.c_int64, dp, ci]
            lib.mro_readout.restype = ctypes.c_int
            lib.mro_compare.argtypes = [P(Problem), vp, dp, i64p, ctypes.c_int64, ctypes.c_int64,
                                        fp, dp, dp, dp, ci, ci, fp, dp, dp, ctypes.c_int64, fp, dp, dp,
                                        ci]
            lib.mro_compare.restype = ctypes.c_int
            lib.mro_backward.argtypes = [P(Problem), vp, dp, dp, dp, dp, ctypes.c_int]
            lib.mro_backward.restype = ctypes.c_int
            lib.mro_backward_readout.argtypes = [P(Problem), vp, dp, dp, ci, ci, dp, ctypes.c_int64, dp, dp, dp,
                                                 ci]
            lib.mro_backward_readout.restype = ctypes.c_int
            lib.mro_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.mro_bf16_to_double.restype = ctypes.c_double
            _lib = lib
    return _lib


def _ptr(a, ctype):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctype))


def make_problem(B, H, L, n, *, x_dtype="f32", mode=MODE_RESHAPE, alpha=1.0,
                 add_identity=1, ldu_offdiag=0.02, ldu_diag=0.1) -> Problem:
    """Parameters are stored as the same float32 numbers the GPU receives."""
    dt = {"f32": DTYPE_F32, "bf16": DTYPE_BF16}[x_dtype] if isinstance(x_dtype, str) else int(x_dtype)
    return Problem(int(B), int(H), int(L), int(n), dt, int(mode), float(alpha), int(add_identity),
                   float(ldu_offdiag), float(ldu_diag))


def _check_x(p: Problem, x: np.ndarray) -> np.ndarray:
    want = np.float32 if p.x_dtype == DTYPE_F32 else np.uint16
    x = np.ascontiguousarray(x)
    if x.dtype != want:
        raise TypeError(f"x must be {want.__name__} (bf16 inputs as raw uint16 patterns)")
    if x.size != p.B * p.L * p.H * p.n * p.n:
        raise ValueError("x has the wrong number of elements for the problem")
    return x


def _raise(rc, what):
    if rc == ERR_SINGULAR:
        raise FloatingPointError(f"{what}: singular input matrix (det = 0 or not finite)")
    if rc != OK:
        raise ValueError(f"{what}: oracle returned status {rc}")


def bf16_to_float(bits: int) -> float:
    return _load().mro_bf16_to_double(int(bits))


def lift(p: Problem, x: np.ndarray, b: int, t: int, h: int) -> np.ndarray:
    """X_t for one token-head, fp64 [n, n]."""
    x = _check_x(p, x)
    X = np.empty((p.n, p.n), np.float64)
    work = np.empty(3 * p.n * p.n, np.float64)
    rc = _load().mro_lift(ctypes.byref(p), x.ctypes.data, b, t, h, _ptr(X, ctypes.c_double),
                          _ptr(work, ctypes.c_double))
    _raise(rc, "lift")
    return X


def scan(p: Problem, x: np.ndarray, S0: np.ndarray | None = None, nthreads: int = 0) -> np.ndarray:
    """All states S_t, fp64 [B, L, H, n, n] (memory position t holds S_{t+1})."""
    x = _check_x(p, x)
    S0 = None if S0 is None else np.ascontiguousarray(S0, np.float64).reshape(p.B, p.H, p.n, p.n)
    S = np.empty((p.B, p.L, p.H, p.n, p.n), np.float64)
    rc = _load().mro_scan(ctypes.byref(p), x.ctypes.data, _ptr(S0, ctypes.c_double),
                          _ptr(S, ctypes.c_double), nthreads or os.cpu_count() or 1)
    _raise(rc, "scan")
    return S


def backward(p: Problem, x: np.ndarray, dS: np.ndarray, S0: np.ndarray | None = None,
             nthreads: int = 0):
    """Vector-Jacobian product of the scan: (dx [B, L, H*n*n], dS0 [B, H, n, n]
    or None) from upstream gradients dS [B, L, H, n, n] (fp64)."""
    x = _check_x(p, x)
    dS = np.ascontiguousarray(dS, np.float64).reshape(p.B, p.L, p.H, p.n, p.n)
    S0 = None if S0 is None else np.ascontiguousarray(S0, np.float64).reshape(p.B, p.H, p.n, p.n)
    dx = np.empty((p.B, p.L, p.H * p.n * p.n), np.float64)
    dS0 = None if S0 is None else np.empty((p.B, p.H, p.n, p.n), np.float64)
    rc = _load().mro_backward(ctypes.byref(p), x.ctypes.data, _ptr(S0, ctypes.c_double),
                              _ptr(dS, ctypes.c_double), _ptr(dx, ctypes.c_double), _ptr(dS0, ctypes.c_double),
                              nthreads or os.cpu_count() or 1)
    _raise(rc, "backward")
    return dx, dS0


def backward_readout(p: Problem, x: np.ndarray, u: np.ndarray, d_o: np.ndarray, snapshot_every: int = 0,
                     d_snap: np.ndarray | None = None, S0: np.ndarray | None = None, nthreads: int = 0):
    """Vector-Jacobian product of the readout form: (dx [B, L, H*n*n], dS0
    [B, H, n, n] or None) from the gradients of o_t = S_t U (d_o shaped like
    o: [B, L, H, n] for one vector u, [B, L, H, n, q] for query columns) and
    of the snapshots (d_snap [B, L//every, H, n, n] or None), fp64."""
    x = _check_x(p, x)
    U, q, per_head = query_columns(p, u)
    d_o = np.ascontiguousarray(d_o, np.float64).reshape(p.B, p.L, p.H, p.n, q)
    if d_snap is not None:
        d_snap = np.ascontiguousarray(d_snap, np.float64).reshape(p.B, p.L // snapshot_every, p.H, p.n, p.n)
    S0 = None if S0 is None else np.ascontiguousarray(S0, np.float64).reshape(p.B, p.H, p.n, p.n)
    dx = np.empty((p.B, p.L, p.H * p.n * p.n), np.float64)
    dS0 = None if S0 is None else np.empty((p.B, p.H, p.n, p.n), np.float64)
    rc = _load().mro_backward_readout(ctypes.byref(p), x.ctypes.data, _ptr(S0, ctypes.c_double),
                                      _ptr(U, ctypes.c_double), q, per_head, _ptr(d_o, ctypes.c_double),
                                      int(snapshot_every if d_snap is not None else 0),
                                      _ptr(d_snap, ctypes.c_double), _ptr(dx, ctypes.c_double),
                                      _ptr(dS0, ctypes.c_double), nthreads or os.cpu_count() or 1)
    _raise(rc, "backward_readout")
    return dx, dS0


def query_columns(p: Problem, u: np.ndarray):
    """The readout's query columns as (U fp64 contiguous, q, per_head):
    u of shape [n] is one vector (q = 1), [n, q] one U for every head,
    [H, n, q] one U per head."""
    u = np.asarray(u, np.float64)
    if u.ndim == 1:
        u, per_head = u.reshape(p.n, 1), 0
    elif u.ndim == 2:
        per_head = 0
    elif u.ndim == 3:
        if u.shape[0] != p.H:
            raise ValueError("per-head query columns must be [H, n, q]")
        per_head = 1
    else:
        raise ValueError("u must be [n], [n, q] or [H, n, q]")
    if u.shape[-2] != p.n or not 1 <= u.shape[-1] <= p.n:
        raise ValueError("query columns must be n x q with 1 <= q <= n")
    return np.ascontiguousarray(u), int(u.shape[-1]), per_head


def readout(p: Problem, x: np.ndarray, u: np.ndarray, snapshot_every: int = 0,
            S0: np.ndarray | None = None, nthreads: int = 0):
    """(o, snapshots [B, L//every, H, n, n] or None), fp64; o is
    [B, L, H, n] for a single vector u and [B, L, H, n, q] for query columns
    U ([n, q] or [H, n, q]): o_t = S_t U."""
    x = _check_x(p, x)
    U, q, per_head = query_columns(p, u)
    S0 = None if S0 is None else np.ascontiguousarray(S0, np.float64).reshape(p.B, p.H, p.n, p.n)
    o = np.empty((p.B, p.L, p.H, p.n, q), np.float64)
    snaps = None
    if snapshot_every > 0:
        snaps = np.empty((p.B, p.L // snapshot_every, p.H, p.n, p.n), np.float64)
    rc = _load().mro_readout(ctypes.byref(p), x.ctypes.data, _ptr(S0, ctypes.c_double),
                             _ptr(U, ctypes.c_double), q, per_head, _ptr(o, ctypes.c_double),
                             int(snapshot_every), _ptr(snaps, ctypes.c_double),
                             nthreads or os.cpu_count() or 1)
    _raise(rc, "readout")
    return (o[..., 0] if np.ndim(u) == 1 else o), snaps


def compare(p: Problem, x: np.ndarray, *, S0=None, bh=None, t_end=None, S_gpu=None,
            u=None, o_gpu=None, snapshot_every=0, snap_gpu=None, nthreads=0):
    """Streaming comparison of GPU results (float32, host arrays) with the oracle.

    Returns a dict with per-(b,t,h) squared norms of the difference and of the
    oracle value for each compared output ("S", "o", "snap"); entries of
    sequences that were not listed in ``bh`` stay NaN."""
    x = _check_x(p, x)
    if bh is None:
        bh = np.arange(p.B * p.H, dtype=np.int64)
    bh = np.ascontiguousarray(bh, np.int64)
    t_end = p.L if t_end is None else int(t_end)
    S0 = None if S0 is None else np.ascontiguousarray(S0, np.float64).reshape(p.B, p.H, p.n, p.n)
    out = {}

    def pair(shape):
        return np.full(shape, np.nan, np.float64), np.full(shape, np.nan, np.float64)

    dS = rS = dO = rO = dP = rP = None
    if S_gpu is not None:
        S_gpu = np.ascontiguousarray(S_gpu, np.float32).reshape(p.B, p.L, p.H, p.n, p.n)
        dS, rS = pair((p.B, p.L, p.H))
        out["S"] = (dS, rS)
    q = per_head = 0
    if u is not None:
        u, q, per_head = query_columns(p, u)
    if o_gpu is not None:
        if u is None:
            raise ValueError("o_gpu needs the query columns u")
        o_gpu = np.ascontiguousarray(o_gpu, np.float32).reshape(p.B, p.L, p.H, p.n, q)
        dO, rO = pair((p.B, p.L, p.H))
        out["o"] = (dO, rO)
    if snap_gpu is not None:
        ls = p.L // snapshot_every
        snap_gpu = np.ascontiguousarray(snap_gpu, np.float32).reshape(p.B, ls, p.H, p.n, p.n)
        dP, rP = pair((p.B, ls, p.H))
        out["snap"] = (dP, rP)
    f, d = ctypes.c_float, ctypes.c_double
    rc = _load().mro_compare(
        ctypes.byref(p), x.ctypes.data, _ptr(S0, d), _ptr(bh, ctypes.c_int64), len(bh), t_end,
        _ptr(S_gpu, f), _ptr(dS, d), _ptr(rS, d),
        _ptr(u, d), q, per_head, _ptr(o_gpu, f), _ptr(dO, d), _ptr(rO, d),
        int(snapshot_every), _ptr(snap_gpu, f), _ptr(dP, d), _ptr(rP, d),
        nthreads or os.cpu_count() or 1)
    _raise(rc, "compare")
    return out


def error_stats(d2: np.ndarray, r2: np.ndarray) -> dict:
    """Relative errors from squared norms: per-item max and median of
    ||gpu - ref|| / ||ref||, plus the whole-tensor ratio."""
    m = ~np.isnan(d2)
    d2, r2 = d2[m], r2[m]
    if d2.size == 0:
        return {"count": 0, "max": float("nan"), "median": float("nan"), "global": float("nan")}
    with np.errstate(divide="ignore", invalid="ignore"):
        rel = np.sqrt(np.where(r2 > 0, d2 / r2, np.where(d2 > 0, np.inf, 0.0)))
    return {
        "count": int(d2.size),
        "max": float(rel.max()),
        "argmax": int(np.flatnonzero(m)[int(rel.argmax())]),
        "median": float(np.median(rel)),
        "global": float(np.sqrt(d2.sum() / r2.sum())) if r2.sum() > 0 else float(np.sqrt(d2.sum())),
    }
