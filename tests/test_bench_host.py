"""bench.py's multi-rank host logic on CPU: two gloo ranks, as torchrun would launch them.

The timing all-reduce returns the maximum over the ranks on every rank, and the whole-job time per
chunk counts the chunks of all ranks (replicas, weak scaling).
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(10.0 + rank, world)
        bench.barrier(world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_timing_is_the_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 11.0, 1: 11.0}


def test_whole_job_time_per_chunk_counts_every_rank():
    # 2 ranks x 50 calls x 32 chunks in 1000 ms -> 1e6 us / 3200 chunks
    assert bench.job_us_per_chunk(1000.0, 2, 50, 32) == pytest.approx(312.5)
    assert bench.job_us_per_chunk(9.0, 1, 1, 1) == pytest.approx(9000.0)


def test_prefix_cpu_baseline_samples_one_layer():
    import synthetic
    import bench
    cfg = synthetic.PrefixConfig("tiny_prefix", L=4, D=64, Hq=2, Hkv=1, dh=32, F=96, B=2, P=20, dtype="bf16")
    inp = synthetic.make_prefix_pass_inputs(cfg, 0)
    us, threads, sample = bench.cpu_prefix_time(cfg, inp)
    assert us > 0 and threads >= 1 and "layer 0" in sample
    # algorithmic FLOPs: (L-1) full layers and the last layer's QKV per token
    D, F, dq, nkv, P = cfg.D, cfg.F, cfg.Hq * cfg.dh, cfg.Hkv * cfg.dh, cfg.P
    full = 2 * ((dq + 2 * nkv) * D + D * dq + 2 * F * D + D * F) + 4 * P * cfg.dh * cfg.Hq
    want = cfg.B * P * ((cfg.L - 1) * full + 2 * (dq + 2 * nkv) * D)
    assert bench.prefix_flops(cfg) == want


def test_reference_arm_prints_the_contract_line(capsys, monkeypatch):
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON line with the keys the
    native arm prints, on the same metric and workload."""
    import json
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is False and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert "pi05_bf16_b1" in line["config"]["workload"]


def test_reference_arm_is_silent_on_other_ranks(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out.strip() == ""


def test_options_warmup_floor_and_persistent_headline_only():
    """At least three warm-up calls; `--exec persistent` times the batch-1 headline workload only (the
    persistent kernel serves batch-1-sized calls), with no other workloads in the line."""
    a = bench.parse_args(["--warmup", "1"])
    assert a.warmup == 3 and a.exec_mode == "auto" and not a.no_extra
    a = bench.parse_args(["--exec", "persistent"])
    assert a.exec_mode == "persistent" and a.no_extra
    a = bench.parse_args(["--exec", "graph", "--workload", "pi05_bf16_b32"])
    assert a.exec_mode == "graph" and not a.no_extra and a.workload == "pi05_bf16_b32"
    with pytest.raises(SystemExit):
        bench.parse_args(["--exec", "eager"])


def test_peaks_come_from_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks() == (6650.0, 1590.0, 1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        '{"hbm_gbs": 7012.5, "bf16_tflops": 1702.0, "bf16_tflops_sustained": 1455.5, "sm_mhz": 1965}')
    assert bench.load_peaks() == (7012.5, 1702.0, 1455.5, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 7012.5}')   # incomplete: not used
    assert bench.load_peaks()[3] == "fallback"


def test_clock_samples_summarise_median_max_and_active_reasons():
    s = bench.ClockSampler(0)
    # index, sm, max sm, power, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    s.lines = ["0, 1965, 1965, 702.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
               "0, 1800, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
               "0, 1950, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
               "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",   # unparsable: skipped
               "garbled"]
    got = s.summary()
    assert got == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    s.lines = ["0, 1200, 1965, 500.0, 0x0000000000000040, Active, Not Active, Active, Not Active"]
    assert s.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    s.lines = []
    assert s.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
