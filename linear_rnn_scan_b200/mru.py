"""ctypes binding of libmru.so (declared in include/mru.h).

Argument marshalling only: every step of the scan runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
CPU fallback: if libmru.so has not been built, the first call raises.

Low level (same names as the C-ABI; pointers are ints, streams are ints):
    workspace_size, build_states, scan, scan_fused, last_device_status,
    status_string, chosen_chunk, launch_count
Tensor level:
    problem(...)                 -> Problem
    scan_fused_t(p, x, ...)      -> S [B, L, H, n, n]  or  (o, snapshots)
    scan_t(p, X, ...)            -> S
    build_states_t(p, x, ...)    -> X (or F)
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmru.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_SINGULAR, ERR_TIMEOUT = range(7)
MODE_RESHAPE, MODE_DETNORM, MODE_LDU, MODE_CAYLEY, MODE_EXPM = 0, 1, 2, 3, 4
F32, BF16 = 0, 1
MATH = {"auto": 0, "fp32": 1, "tf32": 2, "tf32x3": 3, "bf16x3": 4}

# Every symbol include/mru.h declares.
EXPORTS = ["mru_workspace_size", "mru_build_states", "mru_scan", "mru_scan_fused",
           "mru_last_device_status", "mru_status_string", "mru_chosen_chunk", "mru_launch_count",
           "mru_set_profile_events", "mru_scan_fused_noalloc", "mru_kernel_name", "mru_effective_math",
           "mru_backward_workspace_size", "mru_scan_backward", "mru_scan_fused_host",
           "mru_debug_stall_next_fused", "mru_backward_readout_workspace_size", "mru_scan_backward_readout"]
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class Problem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int64), ("H", ctypes.c_int64), ("L", ctypes.c_int64),
        ("n", ctypes.c_int32), ("x_dtype", ctypes.c_int32), ("mode", ctypes.c_int32),
        ("math", ctypes.c_int32), ("alpha", ctypes.c_float), ("add_identity", ctypes.c_int32),
        ("ldu_offdiag", ctypes.c_float), ("ldu_diag", ctypes.c_float),
        ("store_minus_identity", ctypes.c_int32), ("chunk", ctypes.c_int32),
    ]


class Readout(ctypes.Structure):
    _fields_ = [("u", ctypes.c_void_p), ("snapshot_every", ctypes.c_int64), ("snapshots", ctypes.c_void_p),
                ("q", ctypes.c_int32), ("u_per_head", ctypes.c_int32)]


class MruError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lock = threading.Lock()
_lib = None


def load(path: str = LIB_PATH):
    """Load libmru.so (once).  Raises when it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise ImportError(f"{path} is missing: build it with `python -m linear_rnn_scan_b200.build`")
            lib = ctypes.CDLL(path)
            P = ctypes.POINTER(Problem)
            vp, sz = ctypes.c_void_p, ctypes.c_size_t
            lib.mru_workspace_size.argtypes = [P]
            lib.mru_workspace_size.restype = sz
            lib.mru_build_states.argtypes = [P, vp, vp, vp, sz, vp]
            lib.mru_build_states.restype = ctypes.c_int
            lib.mru_scan.argtypes = [P, vp, vp, vp, vp, sz, vp]
            lib.mru_scan.restype = ctypes.c_int
            lib.mru_scan_fused.argtypes = [P, vp, vp, ctypes.POINTER(Readout), vp, vp, vp, sz, vp]
            lib.mru_scan_fused.restype = ctypes.c_int
            lib.mru_last_device_status.argtypes = [vp, vp]
            lib.mru_last_device_status.restype = ctypes.c_int
            lib.mru_status_string.argtypes = [ctypes.c_int]
            lib.mru_status_string.restype = ctypes.c_char_p
            lib.mru_chosen_chunk.argtypes = [P, ctypes.c_int32]
            lib.mru_chosen_chunk.restype = ctypes.c_int32
            lib.mru_launch_count.argtypes = [P, ctypes.c_int32]
            lib.mru_launch_count.restype = ctypes.c_int32
            lib.mru_set_profile_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
            lib.mru_set_profile_events.restype = ctypes.c_int
            lib.mru_scan_fused_noalloc.argtypes = [P, vp, vp, ctypes.POINTER(Readout), vp, vp, vp, vp]
            lib.mru_scan_fused_noalloc.restype = ctypes.c_int
            lib.mru_kernel_name.argtypes = [P, ctypes.c_int32, ctypes.c_int32]
            lib.mru_kernel_name.restype = ctypes.c_char_p
            lib.mru_effective_math.argtypes = [P, ctypes.c_int32]
            lib.mru_effective_math.restype = ctypes.c_int32
            lib.mru_backward_workspace_size.argtypes = [P]
            lib.mru_backward_workspace_size.restype = sz
            lib.mru_scan_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            lib.mru_scan_backward.restype = ctypes.c_int
            lib.mru_scan_fused_host.argtypes = [P, vp, vp, ctypes.POINTER(Readout), vp, vp, vp, vp, vp, sz,
                                                ctypes.c_int32, vp, vp, vp]
            lib.mru_scan_fused_host.restype = ctypes.c_int
            lib.mru_backward_readout_workspace_size.argtypes = [P]
            lib.mru_backward_readout_workspace_size.restype = sz
            lib.mru_scan_backward_readout.argtypes = [P, vp, vp, ctypes.POINTER(Readout), vp, vp, vp, vp, vp, sz,
                                                      vp]
            lib.mru_scan_backward_readout.restype = ctypes.c_int
            lib.mru_debug_stall_next_fused.argtypes = [ctypes.c_int32]
            lib.mru_debug_stall_next_fused.restype = None
            _lib = lib
    return _lib


def problem(B, H, L, n, *, x_dtype="f32", mode=MODE_RESHAPE, math="auto", alpha=1.0, add_identity=1,
            ldu_offdiag=0.02, ldu_diag=0.1, store_minus_identity=0, chunk=0) -> Problem:
    dt = {"f32": F32, "bf16": BF16}[x_dtype] if isinstance(x_dtype, str) else int(x_dtype)
    mt = MATH[math] if isinstance(math, str) else int(math)
    return Problem(int(B), int(H), int(L), int(n), dt, int(mode), mt, float(alpha), int(add_identity),
                   float(ldu_offdiag), float(ldu_diag), int(store_minus_identity), int(chunk))


def problem_from_workload(w, **over) -> Problem:
    kw = dict(x_dtype=w.x_dtype, mode=w.mode, math=w.math, alpha=w.alpha, add_identity=w.add_identity,
              ldu_offdiag=w.ldu_offdiag, ldu_diag=w.ldu_diag)
    kw.update(over)
    return problem(w.B, w.H, w.L, w.n, **kw)


# ---------------------------------------------------------------- C-ABI ---

def workspace_size(p: Problem) -> int:
    return int(load().mru_workspace_size(ctypes.byref(p)))


def chosen_chunk(p: Problem, readout: bool = False) -> int:
    return int(load().mru_chosen_chunk(ctypes.byref(p), 1 if readout else 0))


def launch_count(p: Problem, readout: bool = False) -> int:
    return int(load().mru_launch_count(ctypes.byref(p), int(bool(readout))))


def kernel_names(p: Problem, readout: bool = False) -> list:
    n = launch_count(p, readout)
    return [load().mru_kernel_name(ctypes.byref(p), int(bool(readout)), i).decode() for i in range(n)]


MATH_NAMES = {v: k for k, v in MATH.items()}


def effective_math(p: Problem, readout: bool = False) -> str:
    """Name of the arithmetic the chosen kernels use: "fp32", "tf32x3", "bf16x3"."""
    return MATH_NAMES.get(int(load().mru_effective_math(ctypes.byref(p), int(bool(readout)))), "invalid")


def status_string(status: int) -> str:
    return load().mru_status_string(int(status)).decode()


def build_states(p: Problem, x: int, X_out: int, ws: int, ws_bytes: int, stream: int = 0) -> int:
    return load().mru_build_states(ctypes.byref(p), x, X_out, ws, ws_bytes, stream)


def scan(p: Problem, X: int, S0: int | None, S_out: int, ws: int, ws_bytes: int, stream: int = 0) -> int:
    return load().mru_scan(ctypes.byref(p), X, S0, S_out, ws, ws_bytes, stream)


def scan_fused(p: Problem, x: int, S0: int | None, readout: Readout | None, S_out: int | None,
               o_out: int | None, ws: int, ws_bytes: int, stream: int = 0) -> int:
    ro = ctypes.byref(readout) if readout is not None else None
    return load().mru_scan_fused(ctypes.byref(p), x, S0, ro, S_out, o_out, ws, ws_bytes, stream)


def scan_fused_noalloc(p: Problem, x: int, S0: int | None, readout: Readout | None, S_out: int | None,
                       o_out: int | None, status_out: int | None = None, stream: int = 0) -> int:
    """mru_scan_fused without a workspace: scratch is the library's fixed
    device array (for callers that may not allocate device memory)."""
    ro = ctypes.byref(readout) if readout is not None else None
    return load().mru_scan_fused_noalloc(ctypes.byref(p), x, S0, ro, S_out, o_out, status_out, stream)


def scan_fused_host(p: Problem, x_host: int, S0: int | None, readout: Readout | None, out_host: int,
                    snaps_host: int | None, x_dev: int, out_dev: int, ws: int, ws_bytes: int, pieces: int = 0,
                    compute_stream: int = 0, h2d_stream: int = 0, d2h_stream: int = 0) -> int:
    """mru_scan_fused from and to host buffers, upload / scan / download
    pipelined over `pieces` parts on the three streams."""
    ro = ctypes.byref(readout) if readout is not None else None
    return load().mru_scan_fused_host(ctypes.byref(p), x_host, S0, ro, out_host, snaps_host, x_dev, out_dev, ws,
                                      ws_bytes, int(pieces), compute_stream, h2d_stream, d2h_stream)


def backward_workspace_size(p: Problem) -> int:
    return load().mru_backward_workspace_size(ctypes.byref(p))


def scan_backward(p: Problem, x: int, S0: int | None, S_fwd: int, dS: int, dx: int, dS0: int | None, ws: int,
                  ws_bytes: int, stream: int = 0) -> int:
    return load().mru_scan_backward(ctypes.byref(p), x, S0, S_fwd, dS, dx, dS0, ws, ws_bytes, stream)


def backward_readout_workspace_size(p: Problem) -> int:
    return load().mru_backward_readout_workspace_size(ctypes.byref(p))


def scan_backward_readout(p: Problem, x: int, S0: int | None, readout: Readout, d_o: int, d_snaps: int | None,
                          dx: int, dS0: int | None, ws: int, ws_bytes: int, stream: int = 0) -> int:
    return load().mru_scan_backward_readout(ctypes.byref(p), x, S0, ctypes.byref(readout), d_o, d_snaps, dx, dS0,
                                            ws, ws_bytes, stream)


def last_device_status(ws: int, stream: int = 0) -> int:
    return load().mru_last_device_status(ws, stream)


def debug_stall_next_fused(ms: int) -> None:
    """Testing hook: the next single-read n = 16 launch withholds its first
    group's carry and bounds its waits by `ms` milliseconds, so that it ends
    with ERR_TIMEOUT in the status word."""
    load().mru_debug_stall_next_fused(int(ms))


def set_profile_events(handles) -> int:
    """handles: list of cudaEvent_t values (ints), or None/[] to switch off."""
    if not handles:
        return load().mru_set_profile_events(None, 0)
    arr = (ctypes.c_void_p * len(handles))(*handles)
    return load().mru_set_profile_events(arr, len(handles))


# --------------------------------------------------------- tensor level ---

def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev_ptr(t, name):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _check(rc, what):
    if rc != OK:
        raise MruError(rc, what)


def workspace_t(p: Problem, device="cuda"):
    torch = _torch()
    nbytes = workspace_size(p)
    if nbytes == 0:
        raise MruError(ERR_INVALID_ARG, "workspace_size")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def check_device_status(ws, stream=None):
    _check(last_device_status(ws.data_ptr(), _stream(stream)), "device status")


def scan_fused_t(p: Problem, x, *, S0=None, u=None, snapshot_every: int = 0, out=None, o_out=None,
                 snapshots=None, ws=None, stream=None):
    """x: CUDA tensor [B, L, H*n*n] (float32, or bfloat16 when x_dtype is bf16).
    Without u: returns S [B, L, H, n, n].  With u: returns (o, snapshots),
    o = S_t U per token and head: u of shape [n] gives o [B, L, H, n];
    query columns [n, q] (one U for every head) or [H, n, q] (one per head)
    give o [B, L, H, n, q]."""
    torch = _torch()
    dev = x.device
    if ws is None:
        ws = workspace_t(p, dev)
    B, L, H, n = p.B, p.L, p.H, p.n
    s = _stream(stream)
    if u is None:
        if out is None:
            out = torch.empty((B, L, H, n, n), dtype=torch.float32, device=dev)
        rc = scan_fused(p, _dev_ptr(x, "x"), _dev_ptr(S0, "S0"), None, _dev_ptr(out, "out"), None,
                        ws.data_ptr(), ws.numel(), s)
        _check(rc, "mru_scan_fused")
        return out
    if u.dim() == 1:
        q, per_head, oshape = 1, 0, (B, L, H, n)
    elif u.dim() in (2, 3):
        q, per_head, oshape = int(u.shape[-1]), int(u.dim() == 3), (B, L, H, n, int(u.shape[-1]))
        if u.shape[-2] != n or (per_head and u.shape[0] != H):
            raise ValueError("query columns must be [n, q] or [H, n, q]")
    else:
        raise ValueError("u must be [n], [n, q] or [H, n, q]")
    if u.dtype != torch.float32 or not u.is_contiguous():
        raise ValueError("u must be a contiguous float32 tensor")
    if o_out is None:
        o_out = torch.empty(oshape, dtype=torch.float32, device=dev)
    if snapshot_every > 0 and snapshots is None:
        snapshots = torch.empty((B, L // snapshot_every, H, n, n), dtype=torch.float32, device=dev)
    ro = Readout(_dev_ptr(u, "u"), int(snapshot_every), _dev_ptr(snapshots, "snapshots") if snapshot_every > 0 else None,
                 q, per_head)
    rc = scan_fused(p, _dev_ptr(x, "x"), _dev_ptr(S0, "S0"), ro, None, _dev_ptr(o_out, "o_out"),
                    ws.data_ptr(), ws.numel(), s)
    _check(rc, "mru_scan_fused")
    return o_out, snapshots


def scan_fused_host_t(p: Problem, x_host, *, S0=None, out_host=None, x_dev=None, out_dev=None, ws=None,
                      pieces: int = 0, streams=None, device="cuda"):
    """Full-state scan from and to host memory: x_host is a CPU tensor
    [B, L, H*n*n] (pinned for full speed); returns the CPU tensor S
    [B, L, H, n, n] (out_host, pinned when allocated here) after the copies
    completed.  The device staging buffers and the workspace are allocated
    here when not given; streams = (compute, h2d, d2h) torch streams."""
    torch = _torch()
    B, L, H, n = p.B, p.L, p.H, p.n
    if x_host.device.type != "cpu" or not x_host.is_contiguous():
        raise ValueError("x_host must be a contiguous CPU tensor")
    if out_host is None:
        out_host = torch.empty((B, L, H, n, n), dtype=torch.float32, pin_memory=True)
    if x_dev is None:
        x_dev = torch.empty(x_host.shape, dtype=x_host.dtype, device=device)
    if out_dev is None:
        out_dev = torch.empty((B, L, H, n, n), dtype=torch.float32, device=device)
    if ws is None:
        ws = workspace_t(p, device)
    if streams is None:
        streams = (torch.cuda.current_stream(), torch.cuda.Stream(), torch.cuda.Stream())
    sc, si, so = (st.cuda_stream for st in streams)
    rc = scan_fused_host(p, x_host.data_ptr(), _dev_ptr(S0, "S0"), None, out_host.data_ptr(), None,
                         x_dev.data_ptr(), out_dev.data_ptr(), ws.data_ptr(), ws.numel(), pieces, sc, si, so)
    _check(rc, "mru_scan_fused_host")
    streams[0].synchronize()
    return out_host


def scan_backward_t(p: Problem, x, S_fwd, dS, *, S0=None, dx=None, dS0=None, ws=None, stream=None):
    """Gradients of sum <dS, S> with respect to the embeddings (dx [B, L, H*n*n]
    fp32) and, with S0, to S0 (dS0 [B, H, n, n]); S_fwd is the forward's S."""
    torch = _torch()
    dev = x.device
    if ws is None:
        nbytes = backward_workspace_size(p)
        if nbytes == 0:
            raise MruError(ERR_INVALID_ARG, "backward_workspace_size")
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if dx is None:
        dx = torch.empty((p.B, p.L, p.H * p.n * p.n), dtype=torch.float32, device=dev)
    if S0 is not None and dS0 is None:
        dS0 = torch.empty((p.B, p.H, p.n, p.n), dtype=torch.float32, device=dev)
    rc = scan_backward(p, _dev_ptr(x, "x"), _dev_ptr(S0, "S0"), _dev_ptr(S_fwd, "S_fwd"), _dev_ptr(dS, "dS"),
                       _dev_ptr(dx, "dx"), _dev_ptr(dS0, "dS0"), ws.data_ptr(), ws.numel(), _stream(stream))
    _check(rc, "mru_scan_backward")
    return dx, dS0, ws


def scan_backward_readout_t(p: Problem, x, u, d_o, *, snapshot_every: int = 0, d_snaps=None, S0=None,
                            q: int = 0, u_per_head: int = 0, dx=None, dS0=None, ws=None, stream=None):
    """Gradients of a loss of the readout's outputs (d_o [B, L, H, n, q],
    and d_snaps [B, L//every, H, n, n] or None) with respect to the
    embeddings (dx) and, with S0, to S0 (dS0); no forward state is needed."""
    torch = _torch()
    dev = x.device
    if ws is None:
        nbytes = backward_readout_workspace_size(p)
        if nbytes == 0:
            raise MruError(ERR_INVALID_ARG, "backward_readout_workspace_size")
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if dx is None:
        dx = torch.empty((p.B, p.L, p.H * p.n * p.n), dtype=torch.float32, device=dev)
    if S0 is not None and dS0 is None:
        dS0 = torch.empty((p.B, p.H, p.n, p.n), dtype=torch.float32, device=dev)
    ro = Readout(_dev_ptr(u, "u"), int(snapshot_every), None, int(q), int(u_per_head))
    rc = scan_backward_readout(p, _dev_ptr(x, "x"), _dev_ptr(S0, "S0"), ro, _dev_ptr(d_o, "d_o"),
                               _dev_ptr(d_snaps, "d_snaps"), _dev_ptr(dx, "dx"), _dev_ptr(dS0, "dS0"),
                               ws.data_ptr(), ws.numel(), _stream(stream))
    _check(rc, "mru_scan_backward_readout")
    return dx, dS0, ws


def scan_t(p: Problem, X, *, S0=None, out=None, ws=None, stream=None):
    torch = _torch()
    if ws is None:
        ws = workspace_t(p, X.device)
    if out is None:
        out = torch.empty((p.B, p.L, p.H, p.n, p.n), dtype=torch.float32, device=X.device)
    rc = scan(p, _dev_ptr(X, "X"), _dev_ptr(S0, "S0"), _dev_ptr(out, "out"), ws.data_ptr(), ws.numel(),
              _stream(stream))
    _check(rc, "mru_scan")
    return out


def build_states_t(p: Problem, x, *, out=None, ws=None, stream=None):
    torch = _torch()
    if ws is None:
        ws = workspace_t(p, x.device)
    if out is None:
        out = torch.empty((p.B, p.L, p.H, p.n, p.n), dtype=torch.float32, device=x.device)
    rc = build_states(p, _dev_ptr(x, "x"), _dev_ptr(out, "out"), ws.data_ptr(), ws.numel(), _stream(stream))
    _check(rc, "mru_build_states")
    return out
