"""Benchmark of the batch-1 π0.5-shaped 10-step action chunk on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

One step = one fr_denoise call: a whole 10-step Euler chunk (all 18 layers,
every phase) on one batch of synthetic inputs resident in HBM.  The metric is
microseconds per action chunk (lower is better) and the achieved HBM GB/s of
the algorithmic bytes.  With N > 1 (launched by torchrun) every rank runs an
independent replica: the batch-1 loop does not shard, so the whole-job value
is the time of K steps (max over ranks) divided by the N*K chunks processed.

--impl reference times the CPU oracle (float64 numpy) on the host cores: each
step is one Euler step of the same workload, scaled to a 10-step chunk.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "µs per 10-step action chunk (batch 1); achieved HBM GB/s vs 8 TB/s"
UNIT = "us/chunk"


# DRAM bytes (read + written) of one whole chunk from an ncu capture, keyed by workload and by the
# digest of the kernel sources it was taken on (kernel_digest()): a figure is reported as the
# roofline traffic only while those sources are unchanged, otherwise traffic is null.
MEASURED_TRAFFIC = {}

# Workloads measured besides the headline one in a default single-GPU run (their results go into
# the line's "workloads" object); each is timed for EXTRA_STEPS calls after EXTRA_WARMUP.
EXTRA_WORKLOADS = ("tiny_f32", "pi05_fp8_b1", "pi05_bf16_b32", "stress_bf16_b4", "pi05_w4a16_b1")
EXTRA_STEPS, EXTRA_WARMUP = 20, 3


def kernel_digest() -> str:
    """First 16 hex digits of the SHA-256 of the library's kernel sources (csrc/*.cu, *.h)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "flow_matching_action_loop_b200", "csrc", "*"))):
        if f.endswith((".cu", ".h", ".cpp")):
            with open(f, "rb") as fh:
                h.update(os.path.basename(f).encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def workload_bytes(cfg) -> dict:
    """Algorithmic bytes of one chunk: weights streamed once per Euler step plus the KV read per step."""
    D, F, dq, nkv = cfg.D, cfg.F, cfg.Hq * cfg.dh, cfg.Hkv * cfg.dh
    layer_w = (dq + 2 * nkv) * D + D * dq + 2 * F * D + D * F
    if cfg.dtype == "w4a16":   # half a byte per weight plus a bf16 scale per 128 inputs of each row
        rows_k = [((dq + 2 * nkv), D), (D, dq), (2 * F, D), (D, F)]
        layer_bytes = layer_w // 2 + sum(r * -(-k // 128) * 2 for r, k in rows_k)
    else:
        layer_bytes = layer_w * {"f32": 4, "bf16": 2, "fp8": 1}[cfg.dtype]
    small = 2 * (cfg.D * cfg.A * 2 + 3 * cfg.D * 4) + cfg.A * 4   # in/out-proj (bf16) + gains/biases
    w_step = cfg.L * (layer_bytes + 2 * D * 4) + small
    if getattr(cfg, "adarms", False):   # per-step gates and folded shifts (W b) read by the epilogues
        w_step += cfg.L * (2 * D * 4 + ((dq + 2 * nkv) + 2 * F) * 4)
    kv_step = cfg.L * cfg.B * cfg.Hkv * (cfg.P + cfg.H) * cfg.dh * 2 * (4 if cfg.dtype == "f32" else 2)
    return {"weights_per_step": w_step, "kv_per_step": kv_step, "per_chunk": cfg.K * (w_step + kv_step),
            "weights_per_chunk": cfg.K * w_step}


def workload_flops(cfg) -> float:
    """Algorithmic FLOPs of one call (B chunks of K steps): every projection of every token and layer,
    attention of every query row over its P + H keys, the in/out projections; unpadded."""
    D, F, dq, nkv = cfg.D, cfg.F, cfg.Hq * cfg.dh, cfg.Hkv * cfg.dh
    proj = (dq + 2 * nkv) * D + D * dq + 2 * F * D + D * F
    attn = 2 * (cfg.P + cfg.H) * cfg.dh * cfg.Hq * 2          # QK^T and PV per query token
    per_tok = cfg.L * (2 * proj + attn) + 2 * 2 * cfg.A * D
    return float(per_tok) * cfg.B * cfg.H * cfg.K


def workload_desc(cfg) -> str:
    return (f"{cfg.name}: L={cfg.L} D={cfg.D} Hq/Hkv={cfg.Hq}/{cfg.Hkv} dh={cfg.dh} F={cfg.F} "
            f"H={cfg.H} A={cfg.A} B={cfg.B} P={cfg.P} K={cfg.K} {cfg.dtype}")


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    """The largest v over the ranks (an all-reduce of the timing only; no data-path collective)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_us_per_chunk(ms_max: float, world: int, steps: int, batch: int) -> float:
    """Whole-job time per chunk: every rank ran `steps` calls of `batch` chunks within ms_max."""
    return ms_max * 1e3 / (world * steps * batch)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_oracle_time(cfg, inp, n_steps: int):
    """Oracle wall time for n_steps Euler steps (model preparation outside); returns (us per chunk, threads)."""
    from oracle import oracle as O
    model = O.PreparedModel(cfg, inp["weights"])
    # fp8: fixed activation scales for the timing sample (the arithmetic does not depend on them)
    scales = {(l, n): 0.01 for l in range(cfg.L) for n in O.PROJ_INPUTS} if cfg.dtype == "fp8" else None
    t0 = time.perf_counter()
    O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"], samples=[0], K=n_steps, model=model,
              scales=scales)
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    return dt / n_steps * cfg.K * 1e6, threads


def run_reference(args, cfg):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synthetic
    from oracle import oracle as O
    inp = synthetic.make_inputs(cfg, 0)
    model = O.PreparedModel(cfg, inp["weights"])
    ts, dt = O.time_grid(cfg.K)
    kv_k, kv_v = O._sample_kv(model, inp["prefix_k"], inp["prefix_v"], 0)
    x = np.asarray(inp["x0"][0], np.float64)
    for i in range(args.warmup):
        O.velocity(model, x, i % cfg.K, ts[i % cfg.K], kv_k, kv_v)
    times = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        x = x + dt * O.velocity(model, x, i % cfg.K, ts[i % cfg.K], kv_k, kv_v)
        times.append(time.perf_counter() - t0)
    us_chunk = sum(times) / len(times) * cfg.K * 1e6
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    sample = f"one Euler step of {cfg.name} per bench step (1/{cfg.K} chunk), scaled x{cfg.K}"
    line = {"impl": "reference", "metric": METRIC, "value": round(us_chunk, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sum(times) / len(times) * 1e3, 3),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(cfg), "parallelism": "host cores"},
            "cpu_baseline": {"value": round(us_chunk, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(us_chunk, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def prefix_flops(cfg) -> float:
    """Algorithmic FLOPs of one prefix pass: every projection of layers 0..L-2, attention among the P
    tokens, and the last layer's QKV projection (its K and V are the output), unpadded."""
    D, F, dq, nkv, P = cfg.D, cfg.F, cfg.Hq * cfg.dh, cfg.Hkv * cfg.dh, cfg.P
    proj = (dq + 2 * nkv) * D + D * dq + 2 * F * D + D * F
    attn = 2 * P * cfg.dh * cfg.Hq * 2   # QK^T and PV per query token
    per_tok = (cfg.L - 1) * (2 * proj + attn) + 2 * (dq + 2 * nkv) * D
    return float(per_tok) * cfg.B * P


class _DeviceView:
    """A device address seen by torch through the CUDA array interface (no copy)."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
                                         "version": 3}


def cpu_prefix_time(cfg, inp):
    """Oracle wall time of the prefix pass, sampled as its first layer over every token and scaled by the
    layer count; returns (us per pass, threads, sample description)."""
    from oracle import oracle as O
    one = cfg.replace(L=1)
    w = {"layers": inp["weights"]["layers"][:1]}
    model = O.PrefixModel(one, w)
    t0 = time.perf_counter()
    O.prefill(one, w, inp["emb"], model=model, samples=[0])
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    sample = (f"layer 0 of {cfg.name} over all {cfg.P} tokens of sample 0 (float64 numpy), "
              f"scaled x{cfg.L} layers x{cfg.B} samples")
    return dt * cfg.L * cfg.B * 1e6, threads, sample


def run_prefix(args, cfg):
    """The prefix pass (the step before the loop): us per pass over B x P embedded tokens."""
    import synthetic
    import torch
    from flow_matching_action_loop_b200 import PrefixPass
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = synthetic.make_prefix_pass_inputs(cfg, 0)
    pp = PrefixPass(cfg, device=local)
    pp.load_weights(inp["weights"])
    emb = torch.from_numpy(inp["emb"]).to(dev).to(torch.bfloat16).contiguous()
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        pp.run(emb)
    torch.cuda.synchronize(dev)
    assert pp.sync_status() == 0, "device status after warm-up"
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            pp.run(emb)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    us_pass = ms * 1e3 / (world * args.steps)
    # end to end: embeddings from pinned host memory in, the last layer's K and V of sample 0 out
    kptr, _ = pp.buffer("kv_k")
    vptr, _ = pp.buffer("kv_v")
    layer_bytes = pp.buffer("kv_k")[1] // cfg.L
    S_max = 1 + cfg.P
    last_k = torch.as_tensor(_DeviceView(kptr + (cfg.L - 1) * layer_bytes, (cfg.Hkv, S_max, cfg.dh), "<i2"), device=dev)
    last_v = torch.as_tensor(_DeviceView(vptr + (cfg.L - 1) * layer_bytes, (cfg.Hkv, S_max, cfg.dh), "<i2"), device=dev)
    hemb = emb.cpu().pin_memory()
    hk = torch.empty((cfg.Hkv, cfg.P, cfg.dh), dtype=torch.int16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    demb = torch.empty_like(emb)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        demb.copy_(hemb, non_blocking=True)
        pp.run(demb)
        hk.copy_(last_k[:, :cfg.P], non_blocking=True)
        hv.copy_(last_v[:, :cfg.P], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_us = max_over_ranks(e0.elapsed_time(e1), world) * 1e3 / (world * args.steps)
    hbm, tf, tf_sus, peak_kind = load_peaks()
    flops = prefix_flops(cfg)
    achieved = flops / (us_pass * 1e-6) / 1e12
    line = {
        "metric": "us per prefix pass (backbone over the observation's tokens)", "value": round(us_pass, 1),
        "unit": "us/pass", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(us_pass / 1e3, 4), "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": cfg.dtype, "data": "synthetic (seeded, random-init)",
        "config": {"workload": f"{cfg.name}: L={cfg.L} D={cfg.D} Hq/Hkv={cfg.Hq}/{cfg.Hkv} dh={cfg.dh} F={cfg.F} "
                               f"B={cfg.B} P={cfg.P} {cfg.dtype}", "parallelism": f"replicas x{world}",
                   "l2": "weights 3.9 GB per pass > 126 MB L2; no flush needed"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": tf_sus, "unit": "TFLOP/s",
                     "frac": round(achieved / tf_sus, 4), "traffic": None,
                     "peak_kind": f"{peak_kind} cuBLAS bf16, sustained", "kernel": "prefix pass, whole graph",
                     "flops_per_launch": flops},
        "e2e": {"value": round(e2e_us, 1), "unit": "us/pass", "h2d_bytes_per_step": int(hemb.numel() * 2),
                "d2h_bytes_per_step": int(2 * hk.numel() * 2)},
        "gpu_launches": pp.launches_per_call() * args.steps,
        "device_status": pp.sync_status(),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        us_cpu, threads, sample = cpu_prefix_time(cfg, inp)
        line["cpu_baseline"] = {"value": round(us_cpu, 1), "unit": "us/pass", "cores": threads, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    pp.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def parse_args(argv=None):
    """Command-line options; --exec persistent times the headline batch-1 workload only."""
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="pi05_bf16_b1", help="a workload name, or 'all' (one line each)")
    ap.add_argument("--no-extra", action="store_true", help="headline workload only (no 'workloads' object)")
    ap.add_argument("--path", type=int, default=0, help="FR_PATH_* (0 auto, 1 stepwise, 2 tensor)")
    ap.add_argument("--exec", dest="exec_mode", default="auto", choices=["auto", "graph", "persistent"],
                    help="execution of fr_denoise (FR_EXEC_*): the library's choice, the CUDA graph, or the "
                         "persistent kernel (batch-1-sized calls)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-steps", type=int, default=10, help="oracle Euler steps timed for cpu_baseline")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    if args.exec_mode == "persistent":   # the persistent kernel serves batch-1-sized calls only
        args.no_extra = True
    return args


def main(argv=None):
    args = parse_args(argv)

    import synthetic
    if args.workload in synthetic.PREFIX_CONFIGS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the prefix-pass workload has no oracle timing arm"}))
            return 0
        return run_prefix(args, synthetic.PREFIX_CONFIGS[args.workload])
    cfg = synthetic.CONFIGS["pi05_bf16_b1" if args.workload == "all" else args.workload]
    if args.impl == "reference":
        return run_reference(args, cfg)

    world, rank, local = dist_setup(args.gpus)
    if args.workload == "all":
        names = ("pi05_bf16_b1",) + EXTRA_WORKLOADS
        for name in names:
            line = run_loop(synthetic.CONFIGS[name], args, world, rank, local, args.steps, args.warmup,
                            cpu_steps=1 if name != "pi05_bf16_b1" else args.cpu_steps)
            if rank == 0:
                print(json.dumps(line), flush=True)
    else:
        line = run_loop(cfg, args, world, rank, local, args.steps, args.warmup, cpu_steps=args.cpu_steps)
        if world == 1 and not args.no_extra and args.workload == "pi05_bf16_b1":
            line["workloads"] = {}
            for name in EXTRA_WORKLOADS:
                sub = run_loop(synthetic.CONFIGS[name], args, world, rank, local, EXTRA_STEPS, EXTRA_WARMUP,
                               cpu_steps=1)
                line["workloads"][name] = {k: sub[k] for k in (
                    "value", "unit", "ms_per_step", "chunks_per_s", "dtype", "config", "roofline", "e2e",
                    "gpu_launches", "device_status", "clocks", "cpu_baseline", "steps", "warmup") if k in sub}
        if rank == 0:
            print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_loop(cfg, args, world, rank, local, steps, warmup, cpu_steps):
    """Time fr_denoise on one workload; returns the bench line (without printing it)."""
    import synthetic
    import torch
    from flow_matching_action_loop_b200 import ActionExpertLoop, fr_launches_per_call
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    inp = synthetic.make_inputs(cfg, 0)
    loop = ActionExpertLoop(cfg, device=local, path=args.path)
    if args.path == 0 and cfg.dtype != "f32" and loop.path != "tensor":
        raise SystemExit(f"{cfg.name}: the automatic kernel set is {loop.path!r}, expected the tensor path")
    if args.exec_mode != "auto":
        from flow_matching_action_loop_b200 import FR_EXEC_GRAPH, FR_EXEC_PERSISTENT
        loop.set_exec_mode(FR_EXEC_GRAPH if args.exec_mode == "graph" else FR_EXEC_PERSISTENT)
    loop.load_weights(inp["weights"])
    if cfg.dtype == "fp8":
        obs = synthetic.make_observation(cfg, 1)
        cx0 = torch.from_numpy(obs["x0"]).to(dev)
        cpk = torch.from_numpy(obs["prefix_k"]).to(dev).to(torch.bfloat16)
        cpv = torch.from_numpy(obs["prefix_v"]).to(dev).to(torch.bfloat16)
        loop.calibrate(cx0, cpk, cpv)
        del cx0, cpk, cpv
    kv_dtype = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    pk = torch.from_numpy(inp["prefix_k"]).to(dev).to(kv_dtype)
    pv = torch.from_numpy(inp["prefix_v"]).to(dev).to(kv_dtype)
    loop.set_prefix_kv(pk, pv)
    del pk, pv
    x0 = torch.from_numpy(inp["x0"]).to(dev)
    out = torch.empty_like(x0)
    stream = torch.cuda.current_stream(dev)
    wb = workload_bytes(cfg)
    l2_note = (f"weights stream {wb['weights_per_step'] / 1e6:.0f} MB/step > 126 MB L2; no flush needed"
               if wb["weights_per_step"] > 126e6 else
               f"weights {wb['weights_per_step'] / 1e6:.1f} MB/step fit L2: timed L2-warm, latency-bound parity case")

    # ---- device-resident timing
    for _ in range(warmup):
        loop.denoise(x0, out)
    torch.cuda.synchronize(dev)
    assert loop.sync_status() == 0, "device status after warm-up"
    barrier(world)
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for i in range(steps):
            loop.denoise(x0, out)
            marks[i].record(stream)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    per_call = sorted([ev0.elapsed_time(marks[0])] + [marks[i - 1].elapsed_time(marks[i]) for i in range(1, steps)])
    barrier(world)
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world)
    status = loop.sync_status()
    ms_per_step = ms / steps
    chunks = world * steps * cfg.B
    us_per_chunk = job_us_per_chunk(ms, world, steps, cfg.B)

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region
    hx0 = torch.from_numpy(inp["x0"]).pin_memory()
    hout = torch.empty_like(hx0).pin_memory()
    dx = torch.empty_like(x0)
    for _ in range(warmup):
        dx.copy_(hx0, non_blocking=True)
        loop.denoise(dx, dx)
        hout.copy_(dx, non_blocking=True)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        dx.copy_(hx0, non_blocking=True)
        loop.denoise(dx, dx)
        hout.copy_(dx, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_us = ms_e2e * 1e3 / chunks
    xbytes = cfg.B * cfg.H * cfg.A * 4

    hbm, tf, tf_sus, peak_kind = load_peaks()
    flops = workload_flops(cfg)
    launches = fr_launches_per_call(loop.h, cfg.B)
    # dominant kernel: the path's kernel set of one call; its algorithmic work over its device time.
    # Bound by arithmetic intensity against the ridge of the measured peaks (sustained bf16: the call
    # is a long step); fp8 contractions take the bf16 peak x 2 (nominal ratio).
    tf_dtype = tf_sus * (2.0 if cfg.dtype == "fp8" else 1.0)
    # (the tensor roofline only when it binds clearly: its time at least 1.1x the HBM roofline's)
    tensor_bound = flops / (tf_dtype * 1e12) > 1.1 * wb["per_chunk"] / (hbm * 1e9) and cfg.dtype != "f32"
    digest = kernel_digest()
    traffic = MEASURED_TRAFFIC.get((cfg.name, digest))
    if tensor_bound:
        achieved = flops / (ms_per_step * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(tf_dtype, 1), "unit": "TFLOP/s",
                    "frac": round(achieved / tf_dtype, 4), "traffic": traffic,
                    "peak_kind": f"{peak_kind} cuBLAS bf16, sustained" + (" x2 (fp8 nominal ratio)" if cfg.dtype == "fp8" else ""),
                    "kernel": f"{loop.path} path, whole call", "flops_per_launch": flops,
                    "frac_of_burst": round(achieved / (tf * (2.0 if cfg.dtype == "fp8" else 1.0)), 4)}
    else:
        achieved_gbs = wb["per_chunk"] / (ms_per_step * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved_gbs / hbm, 4), "traffic": traffic,
                    "peak_kind": f"{peak_kind} HBM copy", "kernel": f"{loop.path} path, whole call",
                    "bytes_per_launch": wb["per_chunk"]}
    line = {
        "metric": METRIC, "value": round(us_per_chunk, 2), "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(ms_per_step, 4),
        "ms_per_step_p50": round(per_call[len(per_call) // 2], 4),
        "ms_per_step_p99": round(per_call[min(len(per_call) - 1, (len(per_call) * 99) // 100)], 4),
        "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded, random-init)",
        "config": {"workload": workload_desc(cfg), "global_batch": cfg.B * world, "parallelism": f"replicas x{world}",
                   "l2": l2_note, "path": loop.path, "exec": args.exec_mode, "kernel_digest": digest},
        "per_replica_us_per_chunk": round(ms_local * 1e3 / (steps * cfg.B), 2),
        "chunks_per_s": round(chunks / (ms * 1e-3), 1),
        "achieved_hbm_gbs": round(wb["per_chunk"] / (ms_per_step * 1e-3) / 1e9, 1),
        "frac_of_8tbs_weights_only": round(wb["weights_per_chunk"] / (ms_per_step * 1e-3) / 8e12, 4),
        "roofline": roofline,
        "e2e": {"value": round(e2e_us, 2), "unit": UNIT, "h2d_bytes_per_step": xbytes, "d2h_bytes_per_step": xbytes},
        "gpu_launches": launches * steps,
        "device_status": status,
    }
    line["clocks"] = clk.summary()
    loop.close()
    del x0, out, dx, hx0, hout
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        us_cpu, threads = cpu_oracle_time(cfg, inp, cpu_steps)
        line["cpu_baseline"] = {"value": round(us_cpu, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"{cpu_steps} Euler step(s) of sample 0 of {cfg.name} "
                                          f"(float64 numpy), scaled to {cfg.B} chunk(s) of {cfg.K} steps"}
    return line


if __name__ == "__main__":
    sys.exit(main())
