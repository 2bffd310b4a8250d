"""Host-side checks of the C-ABI library (no GPU needed, no kernel launched):
libmru.so loads, exports every entry point include/mru.h declares, sizes its
workspace, and rejects bad arguments synchronously before touching CUDA."""
import ctypes
import os
import re

import pytest

from linear_rnn_scan_b200 import inputs as gen
from linear_rnn_scan_b200 import mru

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from linear_rnn_scan_b200 import build
    build.build()
    return mru.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mru.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mru_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 8
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(mru.EXPORTS) == names


def test_problem_struct_matches_header():
    # field order and widths of mru_problem as declared in include/mru.h
    text = open(os.path.join(ROOT, "include", "mru.h")).read()
    body = re.search(r"typedef struct \{(.*?)\} mru_problem;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if not decl:
            continue
        typ, names = decl.split(None, 1)
        for nm in names.split(","):
            fields.append((nm.strip(), typ))
    widths = {"int64_t": 8, "int32_t": 4, "float": 4}
    assert [f for f, _ in fields] == [f for f, _ in mru.Problem._fields_]
    for (f, typ), (f2, ct) in zip(fields, mru.Problem._fields_):
        assert widths[typ] == ctypes.sizeof(ct), f


def test_workspace_size(lib):
    w = gen.WORKLOADS["n16_detnorm_b8h8l4096"]
    p = mru.problem_from_workload(w)
    ws = mru.workspace_size(p)
    assert ws >= 256 and ws % 256 == 0
    C = mru.chosen_chunk(p)
    assert C >= 1 and (C & (C - 1)) == 0
    K = -(-w.L // C)
    assert ws >= 256 + w.B * w.H * K * 256 * 4          # at least the fp32 chunk totals
    for n in (4, 8, 16, 32, 64):
        assert mru.workspace_size(mru.problem(1, 1, 7, n)) >= 256
    assert mru.workspace_size(mru.problem(1, 1, 7, 12)) == 0          # unsupported n
    assert mru.workspace_size(mru.problem(-1, 1, 7, 16)) == 0         # negative size
    assert mru.workspace_size(mru.problem(0, 0, 0, 16)) >= 256        # empty is valid


def test_chunk_override(lib):
    p = mru.problem(2, 3, 100, 16, chunk=7)
    assert mru.chosen_chunk(p) == 7 and mru.chosen_chunk(p, readout=True) == 7
    # the n = 64 tensor-core path (the readout, and every state when tf32 is
    # asked for, as this workload does) takes longer chunks than the generic
    # state-writing one (fp32)
    p64 = mru.problem_from_workload(gen.WORKLOADS["n64_detnorm_readout_b2h4l16384"])
    assert mru.chosen_chunk(p64, readout=True) == 128 and mru.chosen_chunk(p64) == 128
    p64f = mru.problem_from_workload(gen.WORKLOADS["n64_detnorm_readout_b2h4l16384"], math="auto")
    assert mru.chosen_chunk(p64f, readout=True) == 128 and mru.chosen_chunk(p64f) == 32
    assert mru.launch_count(p) >= 1
    assert mru.launch_count(mru.problem(0, 3, 100, 16)) == 0


def test_status_strings(lib):
    for s in range(7):
        assert isinstance(mru.status_string(s), str) and mru.status_string(s)
    assert "unknown" in mru.status_string(99)


def test_invalid_arguments_rejected_before_any_launch(lib):
    p = mru.problem(1, 1, 8, 16)
    nb = mru.workspace_size(p)
    fake = 1 << 20  # never dereferenced: every call below fails its checks first
    assert mru.scan_fused(p, 0, None, None, fake, None, fake, nb) == mru.ERR_INVALID_ARG       # x null
    assert mru.scan_fused(p, fake, None, None, 0, None, fake, nb) == mru.ERR_INVALID_ARG       # S_out null
    assert mru.scan_fused(p, fake + 4, None, None, fake, None, fake, nb) == mru.ERR_INVALID_ARG  # misaligned
    assert mru.scan_fused(p, fake, None, None, fake, None, fake, nb) == mru.ERR_INVALID_ARG    # alias
    # (the size is the largest any call of this problem needs; this call needs less, but more than 255 bytes)
    assert mru.scan_fused(p, fake, None, None, 2 * fake, None, 3 * fake, 255) == mru.ERR_WORKSPACE
    bad = mru.problem(1, 1, 8, 12)
    assert mru.scan_fused(bad, fake, None, None, 2 * fake, None, 3 * fake, nb) == mru.ERR_UNSUPPORTED
    bad = mru.problem(1, 1, 8, 16, mode=7)
    assert mru.scan_fused(bad, fake, None, None, 2 * fake, None, 3 * fake, nb) == mru.ERR_INVALID_ARG
    ro = mru.Readout(None, 0, None)
    assert mru.scan_fused(p, fake, None, ro, None, 2 * fake, 3 * fake, nb) == mru.ERR_INVALID_ARG  # u null
    ro = mru.Readout(4 * fake, 4, None)
    assert mru.scan_fused(p, fake, None, ro, None, 2 * fake, 3 * fake, nb) == mru.ERR_INVALID_ARG  # snaps null
    for q, per_head in ((17, 0), (-1, 0), (2, 2)):                 # q outside [0, n], bad per-head flag
        ro = mru.Readout(4 * fake, 0, None, q, per_head)
        assert mru.scan_fused(p, fake, None, ro, None, 2 * fake, 3 * fake, nb) == mru.ERR_INVALID_ARG
    assert mru.scan(p, fake, None, fake, 3 * fake, nb) == mru.ERR_INVALID_ARG                  # X aliases S
    assert mru.build_states(p, 0, fake, 3 * fake, nb) == mru.ERR_INVALID_ARG
    assert mru.last_device_status(0) == mru.ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path):
    missing = str(tmp_path / "libmru.so")
    saved = mru._lib
    try:
        mru._lib = None
        with pytest.raises(ImportError):
            mru.load(missing)
    finally:
        mru._lib = saved


def test_single_chunk_problems_take_one_launch(lib):
    """A problem of one chunk per sequence (L <= chunk: decode steps, short
    segments) runs one kernel from S0; longer ones run the full pass order
    (for n = 16 the three passes, or the single-read kernel when asked for)."""
    cases = [(mru.problem(8, 8, 1, 16, mode=mru.MODE_DETNORM, alpha=0.0125), ["k16_apply"]),
             (mru.problem(4, 16, 1, 32, x_dtype="bf16", mode=mru.MODE_LDU), ["k32_apply"]),
             (mru.problem(2, 3, 5, 8, mode=mru.MODE_CAYLEY, alpha=0.1), ["k_chunk_prefix"]),
             (mru.problem(2, 4, 16, 64, mode=mru.MODE_DETNORM, alpha=0.01, chunk=16), ["k_chunk_prefix"])]
    for p, names in cases:
        assert mru.launch_count(p) == 1 and mru.kernel_names(p) == names
    p = mru.problem(8, 8, 4096, 16, mode=mru.MODE_DETNORM, alpha=0.0125)
    assert mru.kernel_names(p) == ["k16_reduce", "k16_carry", "k16_apply"]
    for mode in (mru.MODE_CAYLEY, mru.MODE_EXPM):           # orthogonal maps on the same passes
        q = mru.problem(8, 8, 4096, 16, mode=mode, alpha=0.0125)
        assert mru.kernel_names(q) == ["k16_reduce", "k16_carry", "k16_apply"]
        assert mru.effective_math(q) == "tf32x3"
    os.environ["MRU_N16_FUSED"] = "1"
    try:
        assert mru.kernel_names(p) == ["k16_fused"] and mru.launch_count(p) == 1
    finally:
        os.environ.pop("MRU_N16_FUSED", None)
    p = mru.problem(2, 4, 16, 64, mode=mru.MODE_DETNORM, alpha=0.01, chunk=16)
    assert mru.kernel_names(p, True) == ["k_chunk_prefix"]
    p = mru.problem(2, 4, 4096, 64, mode=mru.MODE_DETNORM, alpha=0.01, math="tf32")
    assert mru.kernel_names(p, True)[0] == "k64_chunk_readout" and mru.launch_count(p, True) == 5
    os.environ["MRU_N64_TCGEN05"] = "1"
    try:
        assert mru.kernel_names(p, True)[0] == "k64_chunk_readout_tc" and mru.launch_count(p, True) == 5
    finally:
        os.environ.pop("MRU_N64_TCGEN05", None)
    # every state at n = 64: the tensor-core path when tf32 is asked for, fp32 generic otherwise
    p = mru.problem(2, 4, 4096, 64, mode=mru.MODE_DETNORM, alpha=0.01, math="tf32")
    assert mru.kernel_names(p) == ["k64_chunk_readout", "k_carry_local", "k_carry_groups", "k_carry_final",
                                   "k64_fixup"]
    assert mru.effective_math(p) == "tf32"
    p = mru.problem(2, 4, 4096, 64, mode=mru.MODE_DETNORM, alpha=0.01)
    assert mru.kernel_names(p)[0] == "k_chunk_prefix" and mru.effective_math(p) == "fp32"


def test_small_problems_choose_one_launch(lib):
    """n = 4 without a readout, automatic chunk, sequences of up to 16384
    tokens and either up to 2^20 tokens or at least 148 sequences: the whole
    sequence is one chunk on the one-launch kernel; otherwise the passes."""
    for p in (mru.problem(1, 1, 1024, 4), mru.problem(2, 3, 16384, 4, mode=mru.MODE_DETNORM, alpha=0.1),
              mru.problem(64, 16, 1024, 4, x_dtype="bf16", mode=mru.MODE_LDU), mru.problem(128, 16, 1024, 4),
              mru.problem(148, 1, 16384, 4)):
        assert mru.kernel_names(p) == ["k_small_scan"] and mru.chosen_chunk(p) == p.L
    assert mru.kernel_names(mru.problem(1, 1, 1024, 4), True) == ["k_chunk_prefix", "k_carry_local",
                                                                  "k_carry_groups", "k_carry_final", "k_fixup"]
    for p in (mru.problem(1, 1, 16385, 4), mru.problem(147, 1, 16384, 4), mru.problem(1, 1, 1024, 8),
              mru.problem(1, 1, 1024, 4, mode=mru.MODE_CAYLEY, alpha=0.1), mru.problem(1, 1, 1024, 4, chunk=16)):
        assert "k_small_scan" not in mru.kernel_names(p)


def test_host_entry_rejects_bad_arguments(lib):
    p = mru.problem(2, 2, 8, 16)
    nb = mru.workspace_size(p)
    fake = 1 << 20
    ok = dict(x_host=fake, out_host=2 * fake, x_dev=3 * fake, out_dev=4 * fake, ws=5 * fake)

    def call(**kw):
        a = dict(ok, **kw)
        return mru.scan_fused_host(p, a["x_host"], None, None, a["out_host"], None, a["x_dev"], a["out_dev"],
                                   a["ws"], nb, kw.get("pieces", 0))
    assert call(x_host=0) == mru.ERR_INVALID_ARG
    assert call(out_host=0) == mru.ERR_INVALID_ARG
    assert call(x_dev=3 * fake + 8) == mru.ERR_INVALID_ARG          # misaligned staging
    assert call(out_dev=3 * fake) == mru.ERR_INVALID_ARG            # staging buffers alias
    assert call(pieces=-1) == mru.ERR_INVALID_ARG
    ro = mru.Readout(6 * fake, 4, None)                              # snapshots without a staging buffer
    assert mru.scan_fused_host(p, fake, None, ro, 2 * fake, None, 3 * fake, 4 * fake, 5 * fake, nb) == \
        mru.ERR_INVALID_ARG
    assert mru.scan_fused_host(p, fake, None, None, 2 * fake, None, 3 * fake, 4 * fake, 5 * fake, 255) == \
        mru.ERR_WORKSPACE


def test_plain_c_program_uses_the_library(lib, tmp_path):
    """A C99 program that includes only include/mru.h and links libmru.so
    sizes a workspace, picks the chunk and reads status strings, agreeing
    with the Python binding: the boundary needs no C++ and no torch."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    src = tmp_path / "use_mru.c"
    src.write_text(r'''
#include "mru.h"
#include <stdio.h>
int main(void) {
    mru_problem p = {0};
    p.B = 8; p.H = 8; p.L = 4096; p.n = 16;
    p.x_dtype = MRU_F32; p.mode = MRU_MODE_DETNORM; p.math = MRU_MATH_AUTO;
    p.alpha = 0.0125f; p.add_identity = 1;
    printf("%zu %d %s\n", mru_workspace_size(&p), (int)mru_chosen_chunk(&p, 0),
           mru_status_string(MRU_ERR_WORKSPACE));
    p.n = 12;
    printf("%zu\n", mru_workspace_size(&p));
    return 0;
}
''')
    libdir = os.path.dirname(mru.LIB_PATH)
    exe = tmp_path / "use_mru"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(mru.LIB_PATH),
                        "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    first, second = out.stdout.strip().splitlines()
    ws, chunk, msg = first.split(" ", 2)
    p = mru.problem(8, 8, 4096, 16, mode=mru.MODE_DETNORM, alpha=0.0125)
    assert int(ws) == mru.workspace_size(p) and int(chunk) == mru.chosen_chunk(p)
    assert msg == mru.status_string(mru.ERR_WORKSPACE)
    assert second == "0"
