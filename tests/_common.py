"""Helpers shared by the GPU tests: run the library and the oracle on one seeded workload."""
from __future__ import annotations

import functools

import numpy as np

import synthetic
from oracle import oracle as O

# Tolerances per chunk (x at t=0 against the oracle on the same inputs)
TOL_F32_REL_L2 = 1e-4
TOL_BF16_REL_L2 = 2e-2
TOL_BF16_COS = 0.999
TOL_FP8_COS = 0.995
TOL_CALIB_REL = 2.0 ** -7

# Small workloads that the oracle finishes in seconds but that span several
# 128-wide tiles with ragged tails in every dimension.
RAGGED = {
    "ragged_bf16": synthetic.ActionExpertConfig("ragged_bf16", L=2, D=320, Hq=4, Hkv=2, dh=64, F=704, H=37,
                                                A=7, B=3, P=75, K=3, dtype="bf16"),
    "ragged_fp8": synthetic.ActionExpertConfig("ragged_fp8", L=2, D=320, Hq=4, Hkv=2, dh=64, F=704, H=37,
                                               A=7, B=3, P=75, K=3, dtype="fp8"),
    "ragged_w4a16": synthetic.ActionExpertConfig("ragged_w4a16", L=2, D=320, Hq=4, Hkv=2, dh=64, F=704, H=37,
                                                 A=7, B=3, P=75, K=3, dtype="w4a16"),
    "ragged_f32": synthetic.ActionExpertConfig("ragged_f32", L=2, D=192, Hq=6, Hkv=3, dh=32, F=200, H=21,
                                               A=5, B=2, P=33, K=2, dtype="f32"),
    "mha_bf16": synthetic.ActionExpertConfig("mha_bf16", L=1, D=256, Hq=2, Hkv=2, dh=128, F=512, H=50,
                                             A=32, B=1, P=16, K=2, dtype="bf16"),
    "minimal_bf16": synthetic.ActionExpertConfig("minimal_bf16", L=1, D=128, Hq=1, Hkv=1, dh=128, F=128, H=1,
                                                 A=1, B=1, P=1, K=1, dtype="bf16"),
    # batch-1-sized calls (B*H <= 64 tokens): the persistent kernel's shapes, ragged in every dimension
    "b1_ragged_bf16": synthetic.ActionExpertConfig("b1_ragged_bf16", L=2, D=320, Hq=4, Hkv=2, dh=64, F=704, H=37,
                                                   A=7, B=1, P=75, K=3, dtype="bf16"),
    "b2_ragged_bf16": synthetic.ActionExpertConfig("b2_ragged_bf16", L=3, D=384, Hq=6, Hkv=2, dh=64, F=448, H=23,
                                                   A=5, B=2, P=130, K=2, dtype="bf16"),
    "b1_dh128_bf16": synthetic.ActionExpertConfig("b1_dh128_bf16", L=2, D=256, Hq=4, Hkv=1, dh=128, F=512, H=64,
                                                  A=9, B=1, P=100, K=2, dtype="bf16"),
    "b4_dh256_bf16": synthetic.ActionExpertConfig("b4_dh256_bf16", L=1, D=256, Hq=2, Hkv=1, dh=256, F=256, H=16,
                                                  A=4, B=4, P=900, K=2, dtype="bf16"),
}
# the same ragged shapes with adaptive-RMSNorm time conditioning
for _n in ("bf16", "fp8", "w4a16", "f32"):
    _c = RAGGED["ragged_" + _n]
    RAGGED["ragged_adarms_" + _n] = _c.replace(name="ragged_adarms_" + _n, adarms=True)


def get_config(name):
    return synthetic.CONFIGS[name] if name in synthetic.CONFIGS else RAGGED[name]


@functools.lru_cache(maxsize=2)
def inputs(name: str, seed: int = 0):
    return synthetic.make_inputs(get_config(name), seed)


def chunk_metrics(got, want):
    """Per-chunk relative L2 and cosine of x_K (R14)."""
    got = np.asarray(got, np.float64).reshape(len(got), -1)
    want = np.asarray(want, np.float64).reshape(len(want), -1)
    rel = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
    cos = np.sum(got * want, axis=1) / (np.linalg.norm(got, axis=1) * np.linalg.norm(want, axis=1))
    return rel, cos


def to_device(inp, cfg, torch, device="cuda"):
    kv_dtype = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    pk = torch.from_numpy(inp["prefix_k"]).to(device).to(kv_dtype).contiguous()
    pv = torch.from_numpy(inp["prefix_v"]).to(device).to(kv_dtype).contiguous()
    x0 = torch.from_numpy(inp["x0"]).to(device).contiguous()
    return pk, pv, x0


def oracle_scales(cfg, inp_weights, model=None):
    """The oracle's own calibration on the seed-1 observation (R11)."""
    obs = synthetic.make_observation(cfg, seed=1)
    return O.calibrate(cfg, inp_weights, obs["prefix_k"], obs["prefix_v"], obs["x0"], model=model)


def run_library(cfg, inp, path=0, scales=None, calibrate=False, B_max=None, P_max=None, exec_mode=None):
    """Run fr_denoise once on inp; returns (x_K as numpy, loop).  exec_mode: FR_EXEC_* (tensor path)."""
    import torch
    from flow_matching_action_loop_b200 import ActionExpertLoop
    loop = ActionExpertLoop(cfg, B_max=B_max, P_max=P_max, path=path)
    if exec_mode is not None:
        loop.set_exec_mode(exec_mode)
    loop.load_weights(inp["weights"])
    if cfg.dtype == "fp8":
        if calibrate:
            obs = synthetic.make_observation(cfg, seed=1)
            cpk, cpv, cx0 = to_device(obs, cfg, torch)
            loop.calibrate(cx0, cpk, cpv)
        if scales is not None:
            loop.set_scales(scales)
    pk, pv, x0 = to_device(inp, cfg, torch)
    loop.set_prefix_kv(pk, pv)
    out = loop.denoise(x0)
    assert loop.sync_status() == 0
    torch.cuda.synchronize()
    return out.cpu().numpy(), loop
