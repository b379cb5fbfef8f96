"""Seeded synthetic workloads for the flow-matching action-expert denoising loop.

This module is shared by the CPU oracle and by the GPU library's tests and bench.
It holds only sizes and random draws: no step of the method's arithmetic lives
here (no rounding, no normalisation, no time grid).  Every random number the
method consumes is drawn here and passed in as an input.

Workload shapes follow the π0.5-shaped action-expert description (PhyAI page,
"ten-step Euler iteration" of the π0.5 action expert; FlashRT walkthrough,
component 5, the "Pi0.5 decoder" attention site) plus the five sized cases
below.  The prefix length 816 = 3 camera views x 256 image tokens + 48 prompt
tokens stands in for the multi-view LIBERO-style observation that the pages
benchmark on (APXInf page, two-view π0.5 on Thor; FlashRT-PAI summary,
LIBERO-10); no benchmark item is used.

Draw order (numpy PCG64 ``default_rng(seed)``, standard normal in float64,
scaled, then stored as float32):
  1. for each layer: W_q, W_k, W_v, W_o, W_gate, W_up, W_down, each / sqrt(fan_in)
  2. W_in, W_out, W_t1, W_t2, each / sqrt(fan_in)
  3. prefix K then prefix V, shape [L][B][P][Hkv][dh], N(0, 1)
  4. noise x0, shape [B][H][A], N(0, 1)
  5. adaRMS workloads only: for each layer W_mod1 then W_mod2 [3D][D], then W_modf [2D][D],
     each / sqrt(D) (drawn last, so the other tensors equal those of the plain workload)
RMSNorm gains are ones and biases are zeros (explicit arrays, not drawn).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import numpy as np

__all__ = ["ActionExpertConfig", "CONFIGS", "PREFIX_CONFIGS", "PrefixConfig", "make_inputs", "make_modulation",
           "make_noise", "make_prefix", "make_prefix_pass_inputs"]


@dataclasses.dataclass(frozen=True)
class ActionExpertConfig:
    """Sizes of one action-expert workload.

    dtype is the arithmetic format of the layer projections: "f32", "bf16",
    "fp8" (e4m3 weights and projection inputs) or "w4a16" (4-bit weights with a
    scale per group of input features, bf16 projection inputs).
    """

    name: str
    L: int          # transformer layers
    D: int          # width
    Hq: int         # query heads
    Hkv: int        # key/value heads
    dh: int         # head dim
    F: int          # MLP hidden width (gate and up each)
    H: int          # action tokens per chunk (horizon)
    A: int          # action dim
    B: int          # batch (independent chunks)
    P: int          # prefix KV length per layer
    K: int          # Euler steps
    dtype: str
    rope_theta: float = 10000.0
    eps: float = 1e-6
    time_dim: int = 256
    time_base: float = 10000.0
    adarms: bool = False   # time conditioning by adaptive RMSNorm instead of an added embedding

    @property
    def T(self) -> int:
        return self.B * self.H

    @property
    def n_qkv(self) -> int:
        return (self.Hq + 2 * self.Hkv) * self.dh

    def replace(self, **kw) -> "ActionExpertConfig":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, ActionExpertConfig] = {
    # tiny action expert, fp32 end to end
    "tiny_f32": ActionExpertConfig("tiny_f32", L=2, D=256, Hq=4, Hkv=1, dh=64, F=1024,
                                   H=16, A=8, B=1, P=64, K=2, dtype="f32"),
    # π0.5-shaped action expert, batch 1, bf16 weights and activations
    "pi05_bf16_b1": ActionExpertConfig("pi05_bf16_b1", L=18, D=1024, Hq=8, Hkv=1, dh=256,
                                       F=4096, H=50, A=32, B=1, P=816, K=10, dtype="bf16"),
    # same with e4m3 weights and projection inputs, per-tensor scales
    "pi05_fp8_b1": ActionExpertConfig("pi05_fp8_b1", L=18, D=1024, Hq=8, Hkv=1, dh=256,
                                      F=4096, H=50, A=32, B=1, P=816, K=10, dtype="fp8"),
    # throughput regime: 32 independent chunks
    "pi05_bf16_b32": ActionExpertConfig("pi05_bf16_b32", L=18, D=1024, Hq=8, Hkv=1, dh=256,
                                        F=4096, H=50, A=32, B=32, P=816, K=10, dtype="bf16"),
    # same with 4-bit weights (group scales) and bf16 projection inputs
    "pi05_w4a16_b1": ActionExpertConfig("pi05_w4a16_b1", L=18, D=1024, Hq=8, Hkv=1, dh=256,
                                        F=4096, H=50, A=32, B=1, P=816, K=10, dtype="w4a16"),
    # π0.5-style adaptive-RMSNorm time conditioning, batch 1, bf16
    "pi05_adarms_bf16_b1": ActionExpertConfig("pi05_adarms_bf16_b1", L=18, D=1024, Hq=8, Hkv=1, dh=256,
                                              F=4096, H=50, A=32, B=1, P=816, K=10, dtype="bf16",
                                              adarms=True),
    # larger stress variant
    "stress_bf16_b4": ActionExpertConfig("stress_bf16_b4", L=18, D=2048, Hq=16, Hkv=2, dh=128,
                                         F=8192, H=100, A=32, B=4, P=2048, K=10, dtype="bf16"),
}


def _scaled_normal(rng: np.random.Generator, shape, fan_in: int) -> np.ndarray:
    w = rng.standard_normal(size=shape, dtype=np.float64)
    w /= np.sqrt(float(fan_in))
    return w.astype(np.float32)


def make_weights(cfg: ActionExpertConfig, rng: np.random.Generator) -> dict:
    """Draw all weights in the documented order.  Layout is [out][in] (row-major)."""
    D, F, dh = cfg.D, cfg.F, cfg.dh
    layers: List[dict] = []
    for _ in range(cfg.L):
        lw = {
            "wq": _scaled_normal(rng, (cfg.Hq * dh, D), D),
            "wk": _scaled_normal(rng, (cfg.Hkv * dh, D), D),
            "wv": _scaled_normal(rng, (cfg.Hkv * dh, D), D),
            "wo": _scaled_normal(rng, (D, cfg.Hq * dh), cfg.Hq * dh),
            "wg": _scaled_normal(rng, (F, D), D),
            "wu": _scaled_normal(rng, (F, D), D),
            "wd": _scaled_normal(rng, (D, F), F),
            "g1": np.ones(D, np.float32),
            "g2": np.ones(D, np.float32),
        }
        layers.append(lw)
    w = {
        "layers": layers,
        "w_in": _scaled_normal(rng, (D, cfg.A), cfg.A),
        "w_out": _scaled_normal(rng, (cfg.A, D), D),
        "w_t1": _scaled_normal(rng, (D, cfg.time_dim), cfg.time_dim),
        "w_t2": _scaled_normal(rng, (D, D), D),
        "b_in": np.zeros(D, np.float32),
        "b_out": np.zeros(cfg.A, np.float32),
        "b_t1": np.zeros(D, np.float32),
        "b_t2": np.zeros(D, np.float32),
        "g_f": np.ones(D, np.float32),
    }
    return w


def make_prefix(cfg: ActionExpertConfig, rng: np.random.Generator):
    shape = (cfg.L, cfg.B, cfg.P, cfg.Hkv, cfg.dh)
    pk = rng.standard_normal(size=shape, dtype=np.float64).astype(np.float32)
    pv = rng.standard_normal(size=shape, dtype=np.float64).astype(np.float32)
    return pk, pv


def make_noise(cfg: ActionExpertConfig, rng: np.random.Generator) -> np.ndarray:
    return rng.standard_normal(size=(cfg.B, cfg.H, cfg.A), dtype=np.float64).astype(np.float32)


def make_modulation(cfg: ActionExpertConfig, rng: np.random.Generator, w: dict) -> None:
    """adaRMS modulation weights (draw step 5) into w: per layer w_mod1/b_mod1 (pre-attention norm)
    and w_mod2/b_mod2 (pre-MLP norm) [3D][D], [3D] as (scale | shift | gate) rows; w_modf/b_modf
    [2D][D], [2D] as (scale | shift) rows for the final norm.  Biases are zeros."""
    D = cfg.D
    for lw in w["layers"]:
        lw["w_mod1"] = _scaled_normal(rng, (3 * D, D), D)
        lw["w_mod2"] = _scaled_normal(rng, (3 * D, D), D)
        lw["b_mod1"] = np.zeros(3 * D, np.float32)
        lw["b_mod2"] = np.zeros(3 * D, np.float32)
    w["w_modf"] = _scaled_normal(rng, (2 * D, D), D)
    w["b_modf"] = np.zeros(2 * D, np.float32)


def make_inputs(cfg: ActionExpertConfig, seed: int = 0) -> dict:
    """All inputs of one workload from one seed, in the documented draw order."""
    rng = np.random.default_rng(seed)
    w = make_weights(cfg, rng)
    pk, pv = make_prefix(cfg, rng)
    x0 = make_noise(cfg, rng)
    if cfg.adarms:
        make_modulation(cfg, rng, w)
    return {"weights": w, "prefix_k": pk, "prefix_v": pv, "x0": x0}


def make_observation(cfg: ActionExpertConfig, seed: int) -> dict:
    """A prefix and noise draw without weights (e.g. the calibration input, seed 1)."""
    rng = np.random.default_rng(seed)
    pk, pv = make_prefix(cfg, rng)
    x0 = make_noise(cfg, rng)
    return {"prefix_k": pk, "prefix_v": pv, "x0": x0}


def zero_weights(cfg: ActionExpertConfig) -> dict:
    """A weight set with every matrix and bias zero and gains one (closed-form pins)."""
    w = make_weights(cfg, np.random.default_rng(0))
    for lw in w["layers"]:
        for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd"):
            lw[k][...] = 0.0
    for k in ("w_in", "w_out", "w_t1", "w_t2", "b_in", "b_out", "b_t1", "b_t2"):
        w[k][...] = 0.0
    return w


# --------------------------------------------------------------------------------------
# The prefix pass: the vision-language backbone run once over the observation's tokens to
# produce the per-layer keys and values the action expert attends to.
# --------------------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class PrefixConfig:
    """Sizes of one prefix-pass workload: an L-layer transformer of the action expert's block
    (RMSNorm, fused QKV with RoPE, grouped-query attention, gated-GeLU MLP) over P prefix tokens
    per sample with full attention among them; its KV shape (L, Hkv, dh) matches the expert's."""

    name: str
    L: int
    D: int
    Hq: int
    Hkv: int
    dh: int
    F: int
    B: int
    P: int          # prefix tokens per sample
    dtype: str
    rope_theta: float = 10000.0
    eps: float = 1e-6

    @property
    def n_qkv(self) -> int:
        return (self.Hq + 2 * self.Hkv) * self.dh

    def replace(self, **kw) -> "PrefixConfig":
        return dataclasses.replace(self, **kw)


PREFIX_CONFIGS: Dict[str, PrefixConfig] = {
    # the 2B-parameter backbone of a pi0.5-style policy (width 2048, 18 layers, 8 query heads
    # sharing one 256-wide KV head, MLP 16384) over the 816-token three-view observation
    "vlm_bf16_p816": PrefixConfig("vlm_bf16_p816", L=18, D=2048, Hq=8, Hkv=1, dh=256, F=16384, B=1, P=816,
                                  dtype="bf16"),
}


def make_prefix_pass_inputs(cfg: PrefixConfig, seed: int = 0) -> dict:
    """Weights and token embeddings of one prefix-pass workload.

    Draw order (PCG64 ``default_rng(seed)``, standard normal drawn in float32 to keep the
    2B-parameter case affordable, scaled by 1/sqrt(fan_in) in float32): for each layer W_q, W_k,
    W_v, W_o, W_gate, W_up, W_down; then the embedded prefix tokens [B][P][D] ~ N(0, 1) (the
    vision encoder's and the text embedding's outputs, synthetic).  Gains are ones."""
    rng = np.random.default_rng(seed)
    D, F, dh = cfg.D, cfg.F, cfg.dh

    def w(shape, fan_in):
        a = rng.standard_normal(size=shape, dtype=np.float32)
        a *= np.float32(1.0 / np.sqrt(float(fan_in)))
        return a

    layers = []
    for _ in range(cfg.L):
        layers.append({
            "wq": w((cfg.Hq * dh, D), D), "wk": w((cfg.Hkv * dh, D), D), "wv": w((cfg.Hkv * dh, D), D),
            "wo": w((D, cfg.Hq * dh), cfg.Hq * dh), "wg": w((F, D), D), "wu": w((F, D), D), "wd": w((D, F), F),
            "g1": np.ones(D, np.float32), "g2": np.ones(D, np.float32),
        })
    emb = rng.standard_normal(size=(cfg.B, cfg.P, D), dtype=np.float32)
    return {"weights": {"layers": layers}, "emb": emb}
