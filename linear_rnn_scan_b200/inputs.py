"""Seeded synthetic inputs for the MRU scan workloads.

This module only draws random numbers and describes workload shapes.  It
holds none of the method's arithmetic, imports neither the CUDA binding nor
the oracle, and is shared by the tests, the smoke check and the benchmark so
that both sides of every comparison read identical bytes.

Recipe: embeddings are i.i.d. N(0, 1) float32 drawn on the host from a torch
CPU generator seeded with the workload's seed, laid out [B, L, H*n*n]
(token-major, heads contiguous inside a token).  bf16 workloads round those
float32 draws to bf16 (round-to-nearest-even) and hand the raw 16-bit patterns
around as uint16.  The readout vector u is g/||g||_2 with g ~ N(0, 1)[n] from
a second generator seeded with seed + 7919; a workload with q query columns
per head draws g ~ N(0, 1)[H, n, q] from that generator instead and scales
every column to unit length.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

MODE_RESHAPE, MODE_DETNORM, MODE_LDU, MODE_CAYLEY, MODE_EXPM = 0, 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    n: int
    x_dtype: str          # "f32" or "bf16"
    mode: int             # MODE_*
    alpha: float = 1.0    # X~ = add_identity*I + alpha*reshape(x)
    add_identity: int = 1
    ldu_offdiag: float = 0.02
    ldu_diag: float = 0.1
    readout: bool = False
    snapshot_every: int = 0
    queries: int = 0      # readout: 0 = one vector u [n]; q >= 1 = query columns U [H, n, q]
    math: str = "auto"    # "auto", "fp32", "tf32", "tf32x3", "bf16x3"
    seed: int = 0

    @property
    def D(self) -> int:
        return self.H * self.n * self.n

    @property
    def token_heads(self) -> int:
        return self.B * self.L * self.H

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _alpha(c: float, n: int) -> float:
    return c / math.sqrt(n)


# The five workloads the method is measured on, named by what they are.
WORKLOADS = {
    "n4_reshape_l1024": Workload(
        "n4_reshape_l1024", B=1, H=1, L=1024, n=4, x_dtype="f32", mode=MODE_RESHAPE,
        alpha=_alpha(0.1, 4), seed=1001),
    "n16_detnorm_b8h8l4096": Workload(
        "n16_detnorm_b8h8l4096", B=8, H=8, L=4096, n=16, x_dtype="f32", mode=MODE_DETNORM,
        alpha=_alpha(0.05, 16), seed=1002),
    "n32_ldu_bf16_b4h16l8192": Workload(
        "n32_ldu_bf16_b4h16l8192", B=4, H=16, L=8192, n=32, x_dtype="bf16", mode=MODE_LDU,
        ldu_offdiag=0.02, ldu_diag=0.1, seed=1003),
    "n16_detnorm_b1h8l262144": Workload(
        "n16_detnorm_b1h8l262144", B=1, H=8, L=262144, n=16, x_dtype="f32", mode=MODE_DETNORM,
        alpha=_alpha(0.02, 16), seed=1004),
    "n64_detnorm_readout_b2h4l16384": Workload(
        "n64_detnorm_readout_b2h4l16384", B=2, H=4, L=16384, n=64, x_dtype="f32",
        mode=MODE_DETNORM, alpha=_alpha(0.03, 64), readout=True, snapshot_every=256,
        math="tf32", seed=1005),
    # the orthogonal constructions on the default workload's shapes and scale
    "n16_cayley_b8h8l4096": Workload(
        "n16_cayley_b8h8l4096", B=8, H=8, L=4096, n=16, x_dtype="f32", mode=MODE_CAYLEY,
        alpha=_alpha(0.05, 16), seed=1006),
    "n16_expm_b8h8l4096": Workload(
        "n16_expm_b8h8l4096", B=8, H=8, L=4096, n=16, x_dtype="f32", mode=MODE_EXPM,
        alpha=_alpha(0.05, 16), seed=1007),
    # the readout generalised to several query columns per head (o_t = S_t U,
    # U [H, 64, 8]) on the same sequences
    "n64_detnorm_readout_q8_b2h4l16384": Workload(
        "n64_detnorm_readout_q8_b2h4l16384", B=2, H=4, L=16384, n=64, x_dtype="f32",
        mode=MODE_DETNORM, alpha=_alpha(0.03, 64), readout=True, snapshot_every=256,
        queries=8, math="tf32", seed=1005),
}

# Workload order as listed by the method's measurement plan (small case first).
WORKLOAD_ORDER = list(WORKLOADS)


def randn_f32(shape, seed: int) -> np.ndarray:
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32).numpy()


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even, by torch) and return raw uint16 patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_x(w: Workload, seed: int | None = None) -> np.ndarray:
    """Embeddings [B, L, H*n*n]: float32, or uint16 bf16 patterns."""
    x = randn_f32((w.B, w.L, w.D), w.seed if seed is None else seed)
    if w.x_dtype == "bf16":
        return f32_to_bf16_bits(x)
    return x


def make_u(w: Workload, seed: int | None = None) -> np.ndarray:
    """Readout vector u = g / ||g||_2 (float32 [n]), or with w.queries = q
    per-head query columns of unit length (float32 [H, n, q])."""
    s = (w.seed if seed is None else seed) + 7919
    if w.queries:
        g = randn_f32((w.H, w.n, w.queries), s).astype(np.float64)
        return (g / np.linalg.norm(g, axis=1, keepdims=True)).astype(np.float32)
    g = randn_f32((w.n,), s).astype(np.float64)
    return (g / np.linalg.norm(g)).astype(np.float32)


def make_S0(w: Workload, seed: int, scale: float = 0.3) -> np.ndarray:
    """A seeded initial state [B, H, n, n]: I + scale * N(0, 1) / sqrt(n)."""
    r = randn_f32((w.B, w.H, w.n, w.n), seed).astype(np.float64) * (scale / math.sqrt(w.n))
    r += np.eye(w.n)
    return r.astype(np.float32)
