"""The oracle and the CUDA path share no code: the package never imports or
reads anything under oracle/, the CUDA sources include nothing from it, and
the oracle's C source includes nothing from the library's headers or
sources.  The only module both sides use is the seeded input generator.
Also: the oracle's multi-threaded runs (sequences split across threads)
give the same bits as one thread."""
from __future__ import annotations

import os
import re

import numpy as np

from linear_rnn_scan_b200 import inputs as gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "linear_rnn_scan_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for d, _, names in os.walk(top):
        if "__pycache__" in d:
            continue
        for nm in names:
            if nm.endswith(exts):
                yield os.path.join(d, nm)


def test_package_never_touches_the_oracle():
    pat = re.compile(r"^\s*(import\s+oracle\b|from\s+oracle\b)|[\"']oracle[/\"']|mru_oracle", re.M)
    for f in _files(PKG, (".py", ".cu", ".cuh", ".h", ".cpp")):
        with open(f, encoding="utf-8") as fh:
            text = fh.read()
        assert not pat.search(text), f"{os.path.relpath(f, ROOT)} refers to the oracle"


def test_cuda_sources_include_only_their_own_headers():
    inc = re.compile(r'^\s*#\s*include\s*"([^"]+)"', re.M)
    own = {os.path.basename(f) for f in _files(PKG, (".cuh", ".h"))} | {"mru.h"}
    for f in _files(PKG, (".cu", ".cuh")):
        with open(f, encoding="utf-8") as fh:
            for name in inc.findall(fh.read()):
                assert os.path.basename(name) in own and "oracle" not in name, (f, name)


def test_oracle_sources_include_nothing_of_the_library():
    inc = re.compile(r'^\s*#\s*include\s*[<"]([^">]+)[">]', re.M)
    lib = {os.path.basename(f) for f in _files(PKG, (".cu", ".cuh", ".h"))} | {"mru.h"}
    for f in _files(ORACLE, (".c", ".h")):
        with open(f, encoding="utf-8") as fh:
            for name in inc.findall(fh.read()):
                assert os.path.basename(name) not in lib, (f, name)
    for f in _files(ORACLE, (".py",)):
        with open(f, encoding="utf-8") as fh:
            text = fh.read()
        assert "libmru.so" not in text and "linear_rnn_scan_b200.mru" not in text, f


def test_input_generator_holds_no_method_arithmetic():
    """inputs.py draws numbers and names workloads (and scales the readout
    vectors to unit length); it builds no state matrix, determinant or
    product."""
    with open(os.path.join(PKG, "inputs.py"), encoding="utf-8") as fh:
        text = fh.read()
    pat = re.compile(r"np\.linalg\.(?!norm\b)|scipy|cumprod|matmul|einsum|\bexpm|\btanh\(|\bexp\(|\blog\(|\w \@ \w")
    assert not pat.search(text), pat.search(text).group(0)


def test_oracle_threads_give_identical_bits(oracle_mod):
    w = gen.Workload("t", B=2, H=3, L=37, n=8, x_dtype="f32", mode=gen.MODE_DETNORM, alpha=0.1, seed=71)
    x = gen.make_x(w)
    p = oracle_mod.make_problem(w.B, w.H, w.L, w.n, mode=w.mode, alpha=w.alpha, add_identity=1)
    one = oracle_mod.scan(p, x, nthreads=1)
    for k in (2, 5, 16):
        assert np.array_equal(one, oracle_mod.scan(p, x, nthreads=k)), k
    dS = np.random.default_rng(72).standard_normal(one.shape)
    b1 = oracle_mod.backward(p, x, dS, nthreads=1)
    b4 = oracle_mod.backward(p, x, dS, nthreads=4)
    assert np.array_equal(b1[0], b4[0]) and np.array_equal(b1[1], b4[1])
