"""The bench's multi-process logic on CPU: two gloo ranks take the barrier
and the max over ranks of their timings exactly as the NCCL ranks of
`torchrun ... bench.py --gpus N` do; only rank 0 prints; the whole-job rate
counts every rank's units over the slowest rank's time; the reference arm
exits at once on ranks other than 0."""
from __future__ import annotations

import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir, per_rank_ms):
    import torch
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    r = bench.Ranks("gloo", torch.device("cpu"), timeout_s=60)
    r.barrier()
    ms = r.max(per_rank_ms[rank])
    r.barrier()
    out = {"rank": r.rank, "world": r.world, "printer": r.printer, "ms": ms,
           "rate": bench.aggregate_rate(r.world, 1000, ms)}
    r.close()
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
        json.dump(out, f)


def test_two_gloo_ranks_barrier_and_max(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    per_rank_ms = [1.25, 2.5]
    mp.spawn(_rank_main, args=(world, port, str(tmp_path), per_rank_ms), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [x["rank"] for x in res] == [0, 1]
    assert all(x["world"] == 2 for x in res)
    assert [x["printer"] for x in res] == [True, False]
    assert all(x["ms"] == 2.5 for x in res)                    # slowest rank's time on every rank
    assert all(x["rate"] == pytest.approx(2 * 1000 / 2.5e-3) for x in res)


def test_single_process_needs_no_process_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    r = bench.Ranks("gloo")
    assert (r.rank, r.world, r.printer) == (0, 1, True)
    assert r.max(3.5) == 3.5
    r.barrier()
    r.close()


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = bench.argparse.Namespace(gpus=2, steps=1, warmup=3, impl="reference")
    assert bench.run_reference(args, bench.gen.WORKLOADS[bench.DEFAULT_WORKLOAD]) == 0
    assert capsys.readouterr().out == ""


def test_every_forward_kernel_has_own_bytes():
    """Each kernel the library names for a workload's forward step has a
    byte count of its own design (the roofline's per-kernel figure), at the
    workloads' sizes and at small sizes that take other paths."""
    from linear_rnn_scan_b200 import inputs as gen
    from linear_rnn_scan_b200 import mru
    mru.load()
    ws = list(gen.WORKLOADS.values())
    ws += [w.with_(L=1) for w in ws] + [w.with_(n=8) for w in ws if w.n == 4]
    for w in ws:
        for ro in ((False, True) if w.readout else (False,)):
            p = mru.problem_from_workload(w)
            chunk = mru.chosen_chunk(p, readout=ro)
            names = mru.kernel_names(p, ro)
            assert names, w.name
            for k in names:
                assert bench.kernel_bytes(k, w, chunk) > 0, (w.name, k)


def test_algorithmic_bytes_per_unit():
    """The roofline's per-unit bytes (embeddings in, results out): n16 fp32
    2,048 B; n32 bf16 in 6,144 B; n64 readout 16,384 + 256 B plus the
    snapshots; n4 128 B."""
    from linear_rnn_scan_b200 import inputs as gen
    W = gen.WORKLOADS
    per_unit = lambda w: bench.step_bytes(w)["total"] / w.token_heads
    assert per_unit(W["n16_detnorm_b8h8l4096"]) == 2048
    assert per_unit(W["n16_detnorm_b1h8l262144"]) == 2048
    assert per_unit(W["n32_ldu_bf16_b4h16l8192"]) == 6144
    assert per_unit(W["n4_reshape_l1024"]) == 128
    w = W["n64_detnorm_readout_b2h4l16384"]
    snaps = w.B * (w.L // 256) * w.H * 64 * 64 * 4
    assert bench.step_bytes(w)["total"] == w.token_heads * (16384 + 256) + snaps
    assert snaps == 8388608


def test_clock_sampler_with_a_fake_nvml(monkeypatch):
    """The clock record of the timed region, read through a fake NVML (no
    GPU setting is read or changed): median SM clock, the visible-device
    index mapped to the physical one, reason bits named (idle left out)."""
    import types
    import time as _time
    calls = {"index": None}
    clocks = iter([1965, 1965, 1900, 1965, 1500] + [1965] * 10000)
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: calls.__setitem__("index", i) or "h",
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: next(clocks),
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x1 | 0x4 | 0x8,
    )
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "5,3")
    with bench.ClockSampler(1, period_s=0.001) as cs:
        _time.sleep(0.05)
    s = cs.summary()
    assert calls["index"] == 3
    assert s["sm_max_mhz"] == 1965 and s["samples"] >= 5 and s["sm_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap", "hw_slowdown"] and s["sm_mhz_min"] == 1500


def test_clock_sampler_without_nvml(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", None)      # import fails
    with bench.ClockSampler(0) as cs:
        pass
    s = cs.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and s["note"]


def test_oracle_rate_is_a_bounded_sample():
    """The CPU baseline times the oracle on a bounded sample: the first
    t_end tokens of a spread subset of sequences, repeated to about the
    target time; the rate is the units it ran over the seconds they took."""
    import time as _time
    import oracle
    from linear_rnn_scan_b200 import inputs as gen
    oracle.build()
    w = gen.WORKLOADS["n16_detnorm_b8h8l4096"]
    x = gen.make_x(w)
    t0 = _time.perf_counter()
    rate, units, secs, sample = bench.oracle_rate(w, x, 0.3, 2)
    wall = _time.perf_counter() - t0
    assert wall < 10.0 and secs >= 0.15 and rate == units / secs
    assert "of 4096 tokens of 8 of 64 (b,h) sequences" in sample and "2 threads" in sample
    t_end = int(sample.split()[1])
    reps = int(sample.split(" x")[1].split(",")[0])
    assert units == 8 * t_end * reps and 16 <= t_end <= 4096


def test_reference_arm_line_on_rank_0(monkeypatch, capsys):
    """Rank 0 of the reference arm prints one JSON line with the contract's
    keys: the oracle's rate as value, cpu_baseline describing the run, e2e
    with no host-device bytes, at least three warm-up steps."""
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    monkeypatch.setenv("MRU_REF_STEP_SECONDS", "0.2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0", "--workload",
                       "n4_reshape_l1024"]) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["warmup"] == 3 and d["steps"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True and d["config"]["workload"] == "n4_reshape_l1024"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_roofline_sides_of_the_quoted_workloads():
    """Both sides of the step roofline for the five workloads the metric is
    quoted on: bytes at the HBM peak and 2 n^3 scan FLOPs per token-head at
    the peak of the pipe the products use (tf32 for n = 16 and 64, bf16 for
    the n = 32 LDU path); HBM binds every one of them."""
    from linear_rnn_scan_b200 import inputs as gen
    peaks = {"hbm_gbs": 6549.4, "bf16_tflops": 1657.1, "bf16_tflops_sustained": 1394.4, "source": "measured"}
    assert len(bench.BASELINE_WORKLOADS) == 5
    assert bench.DEFAULT_WORKLOAD in bench.BASELINE_WORKLOADS
    for name in bench.BASELINE_WORKLOADS:
        w = gen.WORKLOADS[name]
        r = bench.roofline_min_ms(w, peaks)
        assert r["flop"]["flops_per_step"] == 2 * w.n ** 3 * w.token_heads
        assert r["bound"] == "hbm", (name, r)
        assert abs(r["hbm_min_ms"] - bench.step_bytes(w)["total"] / 6549.4e9 * 1e3) < 1e-12
    w2 = gen.WORKLOADS["n16_detnorm_b8h8l4096"]
    assert abs(bench.roofline_min_ms(w2, peaks)["min_ms"] - 536870912 / 6549.4e9 * 1e3) < 1e-9
    w5 = gen.WORKLOADS["n64_detnorm_readout_b2h4l16384"]
    f5 = bench.flop_side(w5, peaks)
    assert f5["pipe"].startswith("tf32") and abs(f5["peak_tflops"] - 1657.1 * 1.1 / 2.25) < 1e-6
    assert bench.flop_side(gen.WORKLOADS["n32_ldu_bf16_b4h16l8192"], peaks)["pipe"].startswith("bf16")
