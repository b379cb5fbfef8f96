"""CPU oracle for the flow-matching action-expert denoising loop.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the bench's
CPU-baseline leg may import this module.  The GPU library never calls it and
shares no code with it; both sides consume the seeded inputs of ``synthetic``.

Plain, slow, float64.  Every step is written the way the method defines it, in
the order the method takes it; library primitives used as steps are numpy's
matmul, exp, tanh, sqrt and Python's math.sin/math.cos.

What the method computes (sources: the web pages on the subject, plus the
sized workload descriptions for everything architectural):
  * PhyAI page ("PhyAI: Real-Time Physical AI at the Edge, Scalable Rollouts in
    the Cloud", optimisation paragraph): the π0.5 action expert runs a ten-step
    Euler iteration; Q/K/V are one fused projection and the MLP gate and up are
    one fused projection; offline quantisation W8A8 is among the schemes.
  * FlashRT walkthrough (m.lqnn.cn), component 8 (kernel library): norm,
    activation, residual+norm+quant fusion, QKV split + RoPE are the
    memory-bound ops; component 6 (calibration): a measure pass records the
    amax of every FP8 GEMM input, then alpha = act_scale x weight_scale;
    component 5: the "Pi0.5 decoder" attention site; section comparing with
    TensorRT/vLLM/SGLang: the KV cache is a static per-layer device buffer.
  * Workload descriptions: width, heads, gated-GeLU(tanh) MLP, RMSNorm eps
    1e-6, RoPE theta 1e4 at positions P..P+H-1 (actions) and 0..P-1 (prefix),
    sinusoidal time embedding (dim 256, base 1e4) -> Linear-SiLU-Linear added
    to the action-token embeddings, in-proj Linear(A->D), out-proj Linear(D->A),
    actions attend to every prefix and action token, dt = -1/K from t=1 to 0.

Readings where the pages are silent (each listed in the design notes):
  R1  t_k = 1 - k/K, dt = -1/K; v is evaluated at the start of each step.
  R2  sinusoidal embedding: sin half first, w_i = base^(-i/half), t unscaled.
  R3  time MLP Linear(256->D)-SiLU-Linear(D->D) with (zero) biases; in/out-proj
      have biases; transformer projections have none.
  R4  the time embedding is added to every action token after the in-proj only.
  R5  RMSNorm y = x / sqrt(mean x^2 + eps) * gamma; a final RMSNorm precedes the
      out-proj.
  R6  RoPE rotate-half pairing (j, j+dh/2), w_j = theta^(-2j/dh); cos/sin are
      computed in float64 and rounded once to float32.
  R7  attention scale 1/sqrt(dh), no mask; query head j uses KV head
      floor(j*Hkv/Hq).
  R8  the caller's prefix K is pre-RoPE; it is rotated once at 0..P-1.
  R9  gate is the first F rows of the fused gate|up; GeLU applies to gate.
  R10 bf16 workloads: every tensor that feeds a projection or attention is
      rounded to bf16 (RNE); accumulation, softmax, residual and x are wide.
      Weights and prefix K/V are bf16-rounded copies of the float32 draws.
  R11 fp8 workload: the four layer projections use e4m3 weights (one scale per
      fused projection, s_w = max|w|/448) and e4m3 inputs (s_a per projection
      input per layer, from a calibration amax over all steps and tokens,
      s_a = amax/448); y = (s_a*s_w) * sum(a_q*w_q).  Everything else is as bf16.
  R12 f32 workloads round nothing.
  R16 w4a16 workload (PhyAI page, optimisation paragraph: W4A16 among the
      offline quantisation schemes; the pages give no group size): each of the
      four layer projections is stored per output row in groups of 128
      consecutive input features as 4-bit integers q in [-7, 7] with one bf16
      scale per group, s = bf16(max|w| / 7), q = clamp(round-half-even(w / s));
      the tensor-core operand is the dequantised weight bf16(q * s).
      Projection inputs are bf16 as in R10; everything else is as bf16.
  R17 adaRMS workloads (pi0.5-style time conditioning; the pages describe the
      pi0.5 action expert but not its conditioning, so the variant follows the
      "Pi0.5-style" workload description): the time embedding is not added to
      the tokens (R4 does not apply); it is the condition c = temb(t), rounded
      like any projection input, of every RMSNorm.  Each of the two norms of a
      layer has (s, b, g) = W_mod c + b_mod (three D-vectors: scale, shift,
      gate); the final norm has (s, b).  The normalised tensor is
      RMS(h) * (1 + s) + b, and each residual update is scaled by the gate:
      h <- h + g * update.  Where the normalised tensor feeds a projection W,
      the projection input (rounded or quantised as in R10/R11/R16) is
      RMS(h) * (1 + s) and W b is added to the projection's output in full
      precision: W (a + b) = W a + W b, with the rounding point placed before
      the shift, as R10 places it before the rstd factor.
  R18 prefix pass (the step before the loop; FlashRT walkthrough, component 5:
      the Pi0.5 attention sites; the KV cache the loop reads is the backbone's
      per-layer keys and values): the backbone is the action expert's layer
      block at its own sizes, run once over the P embedded prefix tokens of a
      sample (inputs: the vision encoder's and text embedding's outputs, bf16)
      with full attention among them (no mask inside the prefix), RoPE at
      positions 0..P-1, no time input; layer l's rotated K and its V are the
      action expert's prefix K/V of layer l.  The last layer stops after its
      QKV projection.
"""
from __future__ import annotations

import math
from typing import Callable, Dict, List, Optional

import numpy as np

E4M3_MAX = 448.0
W4_GROUP = 128     # input features per 4-bit scale group (R16)
W4_QMAX = 7        # symmetric 4-bit range [-7, 7] (R16)
PROJ_INPUTS = ("qkv", "o", "gu", "down")   # the four FP8 projection inputs per layer


# --------------------------------------------------------------------------------------
# Number formats (R10, R11).  bf16: 8 significant bits, float32 exponent range.
# e4m3 ("fn" variant of the OCP 8-bit floating point format): 4 significant bits,
# exponent bias 7, subnormal quantum 2^-9, largest finite 448, no infinity.
# --------------------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    """Round to the nearest bf16 value, ties to even; returned as float64.

    The significand is scaled to an 8-bit integer and rounded with np.rint
    (round-half-even).  Values are assumed to lie in the bf16 normal range.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def round_e4m3(x) -> np.ndarray:
    """Saturate to +-448, then round to the nearest e4m3 value, ties to even."""
    x = np.clip(np.asarray(x, dtype=np.float64), -E4M3_MAX, E4M3_MAX)
    ax = np.abs(x)
    _, e = np.frexp(ax)                      # ax in [2^(e-1), 2^e)
    lead = np.maximum(e - 1, -6)             # exponent of the leading bit, subnormals at -6
    quantum = np.ldexp(1.0, lead - 3)        # 3 fraction bits
    return np.sign(x) * np.rint(ax / quantum) * quantum


def quantize_w4(w, group: int = W4_GROUP):
    """4-bit group quantisation of a [rows][cols] weight (R16).

    Per row and per group of `group` consecutive columns: s = bf16(max|w| / 7) and
    q = clamp(round-half-even(w / s), -7, 7); an all-zero group has s = 0, q = 0.
    Returns q (int8 [rows][cols]) and s (float64 [rows][ceil(cols / group)]).
    """
    w = np.asarray(w, dtype=np.float64)
    rows, cols = w.shape
    ng = -(-cols // group)
    q = np.zeros((rows, cols), dtype=np.int8)
    s = np.zeros((rows, ng), dtype=np.float64)
    for g in range(ng):
        blk = w[:, g * group:(g + 1) * group]
        sg = round_bf16(np.max(np.abs(blk), axis=1) / W4_QMAX)
        s[:, g] = sg
        safe = np.where(sg > 0, sg, 1.0)[:, None]
        r = np.where(sg[:, None] > 0, blk / safe, 0.0)
        q[:, g * group:(g + 1) * group] = np.clip(np.rint(r), -W4_QMAX, W4_QMAX).astype(np.int8)
    return q, s


def dequantize_w4(q, s, group: int = W4_GROUP):
    """The tensor-core operand of a 4-bit weight: bf16(q * s) per element (R16)."""
    q = np.asarray(q, dtype=np.float64)
    rep = np.repeat(np.asarray(s, dtype=np.float64), group, axis=1)[:, :q.shape[1]]
    return round_bf16(q * rep)


def decode_e4m3(code: int) -> float:
    """Value of an e4m3 byte from its bit fields (sign, 4-bit exponent, 3-bit fraction)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    f = code & 0x7
    if e == 0xF and f == 0x7:
        return float("nan")
    if e == 0:
        return s * f * 2.0 ** -9
    return s * (1.0 + f / 8.0) * 2.0 ** (e - 7)


def decode_bf16(bits: int) -> float:
    """Value of a bf16 bit pattern (the high half of a float32)."""
    s = -1.0 if bits & 0x8000 else 1.0
    e = (bits >> 7) & 0xFF
    f = bits & 0x7F
    if e == 0xFF:
        return s * math.inf if f == 0 else float("nan")
    if e == 0:
        return s * f * 2.0 ** -133
    return s * (1.0 + f / 128.0) * 2.0 ** (e - 127)


# --------------------------------------------------------------------------------------
# Elementwise pieces
# --------------------------------------------------------------------------------------

def silu(z):
    """SiLU z * sigmoid(z) (time MLP, workload description)."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def gelu_tanh(z):
    """GeLU, tanh form: 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))) (gated-GeLU(tanh) MLP)."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


def rms_norm(h, gamma, eps):
    """RMSNorm over the last axis (R5; FlashRT walkthrough, component 8: norm ops)."""
    h = np.asarray(h, dtype=np.float64)
    ms = np.mean(h * h, axis=-1, keepdims=True)
    return h / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)


def softmax(s, axis=-1):
    s = np.asarray(s, dtype=np.float64)
    s = s - np.max(s, axis=axis, keepdims=True)
    p = np.exp(s)
    return p / np.sum(p, axis=axis, keepdims=True)


# --------------------------------------------------------------------------------------
# Time: the Euler grid (R1) and the sinusoidal embedding (R2)
# --------------------------------------------------------------------------------------

def time_grid(K: int):
    """t_k = 1 - k/K for k < K and the step dt = -1/K (PhyAI page: ten-step Euler iteration)."""
    return [1.0 - k / K for k in range(K)], -1.0 / K


def euler(v_fn: Callable[[np.ndarray, float, int], np.ndarray], x0, K: int) -> np.ndarray:
    """Explicit Euler from t=1 to t=0: x <- x + dt * v(x, t_k), v taken at the step start."""
    ts, dt = time_grid(K)
    x = np.asarray(x0, dtype=np.float64).copy()
    for k, t in enumerate(ts):
        x = x + dt * v_fn(x, t, k)
    return x


def sinusoidal_embedding(t: float, dim: int, base: float) -> np.ndarray:
    """[sin(t w_i)]_{i<half} ++ [cos(t w_i)]_{i<half}, w_i = base^(-i/half) (R2)."""
    half = dim // 2
    w = np.array([base ** (-i / half) for i in range(half)], dtype=np.float64)
    return np.concatenate([np.sin(t * w), np.cos(t * w)])


# --------------------------------------------------------------------------------------
# RoPE (R6, R8; FlashRT walkthrough, component 8: qkv split + RoPE)
# --------------------------------------------------------------------------------------

def rope_tables(n_pos: int, dh: int, theta: float):
    """cos/sin of pos * theta^(-2j/dh), pos < n_pos, j < dh/2; float64 math, rounded once to float32."""
    half = dh // 2
    cos_t = np.empty((n_pos, half), dtype=np.float32)
    sin_t = np.empty((n_pos, half), dtype=np.float32)
    for j in range(half):
        inv = math.pow(theta, -2.0 * j / dh)
        for p in range(n_pos):
            a = p * inv
            cos_t[p, j] = math.cos(a)
            sin_t[p, j] = math.sin(a)
    return cos_t, sin_t


def rope_rotate(z, cos_rows, sin_rows):
    """Rotate-half: (z_j, z_{j+h}) -> (z_j c - z_{j+h} s, z_j s + z_{j+h} c), h = dh/2.

    z has shape [..., n, dh]; cos_rows/sin_rows have shape [n, dh/2] (one row per position).
    """
    z = np.asarray(z, dtype=np.float64)
    h = z.shape[-1] // 2
    c = np.asarray(cos_rows, dtype=np.float64)
    s = np.asarray(sin_rows, dtype=np.float64)
    lo, hi = z[..., :h], z[..., h:]
    return np.concatenate([lo * c - hi * s, lo * s + hi * c], axis=-1)


# --------------------------------------------------------------------------------------
# Attention (R7; FlashRT walkthrough, component 5: the Pi0.5 decoder site)
# --------------------------------------------------------------------------------------

def attention(q, k, v):
    """softmax(q k^T / sqrt(dh)) v for every query head, grouped query heads share KV heads.

    q: [Hq][n][dh]; k, v: [Hkv][S][dh]; returns [Hq][n][dh].  Query head j reads KV
    head floor(j * Hkv / Hq).  No mask: every query sees every key.
    """
    q = np.asarray(q, dtype=np.float64)
    Hq, dh = q.shape[0], q.shape[-1]
    Hkv = k.shape[0]
    out = np.empty_like(q)
    for j in range(Hq):
        g = (j * Hkv) // Hq
        kg = np.asarray(k[g], dtype=np.float64)
        vg = np.asarray(v[g], dtype=np.float64)
        p = softmax(q[j] @ kg.T / math.sqrt(dh), axis=-1)
        out[j] = p @ vg
    return out


# --------------------------------------------------------------------------------------
# Model preparation: the stored (rounded / quantised) weights the method computes with
# --------------------------------------------------------------------------------------

def _prepare_layer(dtype: str, lw: dict, rnd) -> dict:
    """One layer's weights as the method stores them (R10, R11, R16)."""
    d = {"g1": np.asarray(lw["g1"], np.float64), "g2": np.asarray(lw["g2"], np.float64)}
    if dtype == "fp8":
        for name, parts in (("qkv", ("wq", "wk", "wv")), ("o", ("wo",)),
                            ("gu", ("wg", "wu")), ("down", ("wd",))):
            amax = max(float(np.max(np.abs(np.asarray(lw[p], np.float64)))) for p in parts)
            s_w = amax / E4M3_MAX
            d["sw_" + name] = s_w
            for p in parts:
                d[p] = round_e4m3(np.asarray(lw[p], np.float64) / s_w)   # codes' values
    elif dtype == "w4a16":
        for p in ("wq", "wk", "wv", "wo", "wg", "wu", "wd"):
            d[p] = dequantize_w4(*quantize_w4(lw[p]))
    else:
        for p in ("wq", "wk", "wv", "wo", "wg", "wu", "wd"):
            d[p] = rnd(lw[p])
    return d


class PreparedModel:
    """Weights as the method stores them for one workload (R10, R11, R12).

    For bf16 and fp8 the float32 draws are rounded to bf16 (R10).  For fp8 the
    four layer projections are additionally held as e4m3 values w_q on the grid
    of w / s_w with one s_w per fused projection (PhyAI page: fused QKV, merged
    gate/up; FlashRT walkthrough, component 4: FP8 quantisation with scales).
    For w4a16 they are held as their dequantised 4-bit values bf16(q * s) (R16).
    """

    def __init__(self, cfg, weights: dict):
        self.cfg = cfg
        self.dtype = cfg.dtype
        rnd = (lambda a: np.asarray(a, np.float64)) if cfg.dtype == "f32" else round_bf16
        self.rnd = rnd
        self.w_in = rnd(weights["w_in"])
        self.w_out = rnd(weights["w_out"])
        self.w_t1 = rnd(weights["w_t1"])
        self.w_t2 = rnd(weights["w_t2"])
        self.b_in = np.asarray(weights["b_in"], np.float64)
        self.b_out = np.asarray(weights["b_out"], np.float64)
        self.b_t1 = np.asarray(weights["b_t1"], np.float64)
        self.b_t2 = np.asarray(weights["b_t2"], np.float64)
        self.g_f = np.asarray(weights["g_f"], np.float64)
        self.layers: List[dict] = [_prepare_layer(cfg.dtype, lw, rnd) for lw in weights["layers"]]
        self.adarms = bool(getattr(cfg, "adarms", False))
        if self.adarms:   # R17: modulation projections of the condition, stored like the time MLP
            for d, lw in zip(self.layers, weights["layers"]):
                for n in ("1", "2"):
                    d["w_mod" + n] = rnd(lw["w_mod" + n])
                    d["b_mod" + n] = np.asarray(lw["b_mod" + n], np.float64)
            self.w_modf = rnd(weights["w_modf"])
            self.b_modf = np.asarray(weights["b_modf"], np.float64)
        self.cos, self.sin = rope_tables(cfg.P + cfg.H, cfg.dh, cfg.rope_theta)

    def temb(self, t: float) -> np.ndarray:
        """Time MLP: W_t2 silu(W_t1 e(t) + b_t1) + b_t2 (R2, R3; inputs rounded per R10)."""
        cfg = self.cfg
        e = self.rnd(sinusoidal_embedding(t, cfg.time_dim, cfg.time_base))
        z = self.rnd(silu(self.w_t1 @ e + self.b_t1))
        return self.w_t2 @ z + self.b_t2

    def rotate_prefix_k(self, pk_b):
        """Prefix K of one sample [L][P][Hkv][dh] -> rotated at 0..P-1, [L][Hkv][P][dh] (R8)."""
        cfg = self.cfg
        k = self.rnd(pk_b).transpose(0, 2, 1, 3)          # [L][Hkv][P][dh]
        return self.rnd(rope_rotate(k, self.cos[:cfg.P], self.sin[:cfg.P]))


# --------------------------------------------------------------------------------------
# One velocity evaluation and the full loop
# --------------------------------------------------------------------------------------

def _project(model: PreparedModel, l: int, which: str, a, ws, scales, record):
    """Apply one of the four layer projections to input a ([n][in]); ws are the weight blocks.

    f32/bf16: y = a_r @ W^T with a_r = a (f32) or bf16(a).
    fp8: a_q = e4m3(a / s_a), y = (s_a * s_w) * a_q @ W_q^T (FlashRT walkthrough,
    component 6: alpha = act_scale x weight_scale).
    record (calibration measure pass): remember max|a| and use the unquantised a
    with the dequantised e4m3 weights.
    """
    lay = model.layers[l]
    if model.dtype == "fp8":
        s_w = lay["sw_" + which]
        if record is not None:
            key = (l, which)
            record[key] = max(record.get(key, 0.0), float(np.max(np.abs(a))))
            return [a @ (w * s_w).T for w in ws]
        s_a = scales[(l, which)]
        aq = round_e4m3(a / s_a)
        return [(s_a * s_w) * (aq @ w.T) for w in ws]
    ar = model.rnd(a)
    return [ar @ w.T for w in ws]


def _dequantised(model: PreparedModel, l: int, which: str, w):
    """The weight values a projection multiplies by (s_w * codes for fp8)."""
    return w * model.layers[l]["sw_" + which] if model.dtype == "fp8" else w


def _modulation(model: PreparedModel, c, l: int, n: str):
    """R17: (scale, shift, gate) of norm n ("1" pre-attention, "2" pre-MLP) of layer l."""
    lay = model.layers[l]
    m = lay["w_mod" + n] @ c + lay["b_mod" + n]
    D = model.cfg.D
    return m[:D], m[D:2 * D], m[2 * D:]


def velocity(model: PreparedModel, x, k_step: int, t: float, kv_k, kv_v,
             scales: Optional[Dict] = None, record: Optional[Dict] = None) -> np.ndarray:
    """v(x, t) for one chunk x [H][A] (the action expert; configs' architecture).

    kv_k, kv_v: [L][Hkv][P][dh] prefix keys (already rotated) and values of this sample.
    """
    cfg = model.cfg
    rnd = model.rnd
    P, H, dh, Hq, Hkv = cfg.P, cfg.H, cfg.dh, cfg.Hq, cfg.Hkv
    ones = np.ones(cfg.D)
    if model.adarms:
        # R17: in-proj only; the time embedding conditions the norms
        h = rnd(x) @ model.w_in.T + model.b_in
        cond = rnd(model.temb(t))
    else:
        # in-proj + time (R3, R4)
        h = rnd(x) @ model.w_in.T + model.b_in + model.temb(t)
    cos_a, sin_a = model.cos[P:P + H], model.sin[P:P + H]
    for l, lay in enumerate(model.layers):
        if model.adarms:
            s1, b1, g1 = _modulation(model, cond, l, "1")
            s2, b2, g2 = _modulation(model, cond, l, "2")
            gain1, gain2 = 1.0 + s1, 1.0 + s2
        else:
            gain1, gain2, g1, g2 = lay["g1"], lay["g2"], ones, ones
        # pre-attention RMSNorm, fused QKV projection (PhyAI page: Q/K/V in one GEMM)
        a = rms_norm(h, gain1, cfg.eps)
        q, k, v = _project(model, l, "qkv", a, (lay["wq"], lay["wk"], lay["wv"]), scales, record)
        if model.adarms:   # R17: the shift enters as W b
            q, k, v = (y + _dequantised(model, l, "qkv", w) @ b1
                       for y, w in ((q, lay["wq"]), (k, lay["wk"]), (v, lay["wv"])))
        q = q.reshape(H, Hq, dh).transpose(1, 0, 2)           # [Hq][H][dh]
        k = k.reshape(H, Hkv, dh).transpose(1, 0, 2)          # [Hkv][H][dh]
        v = v.reshape(H, Hkv, dh).transpose(1, 0, 2)
        # QKV split + RoPE at positions P..P+H-1 (FlashRT walkthrough, component 8)
        q = rnd(rope_rotate(q, cos_a, sin_a))
        k = rnd(rope_rotate(k, cos_a, sin_a))
        v = rnd(v)
        keys = np.concatenate([kv_k[l], k], axis=1)            # [Hkv][P+H][dh]
        vals = np.concatenate([kv_v[l], v], axis=1)
        o = attention(q, keys, vals)                           # [Hq][H][dh]
        o = o.transpose(1, 0, 2).reshape(H, Hq * dh)
        (dh_o,) = _project(model, l, "o", o, (lay["wo"],), scales, record)
        h = h + g1 * dh_o
        # pre-MLP RMSNorm, merged gate|up projection, GeLU(gate) * up, down (R9)
        a = rms_norm(h, gain2, cfg.eps)
        g, u = _project(model, l, "gu", a, (lay["wg"], lay["wu"]), scales, record)
        if model.adarms:
            g = g + _dequantised(model, l, "gu", lay["wg"]) @ b2
            u = u + _dequantised(model, l, "gu", lay["wu"]) @ b2
        m = gelu_tanh(g) * u
        (dh_d,) = _project(model, l, "down", m, (lay["wd"],), scales, record)
        h = h + g2 * dh_d
    # final RMSNorm + out-proj (R5; R17 modulates it)
    if model.adarms:
        mf = model.w_modf @ cond + model.b_modf
        s_f, b_f = mf[:cfg.D], mf[cfg.D:]
        return rnd(rms_norm(h, 1.0 + s_f, cfg.eps)) @ model.w_out.T + model.w_out @ b_f + model.b_out
    return rnd(rms_norm(h, model.g_f, cfg.eps)) @ model.w_out.T + model.b_out


def _sample_kv(model: PreparedModel, prefix_k, prefix_v, b: int, k_rotated: bool = False):
    if k_rotated:   # already carries RoPE at 0..P-1 (the prefix pass's output)
        kv_k = model.rnd(np.asarray(prefix_k)[:, b]).transpose(0, 2, 1, 3)
    else:
        kv_k = model.rotate_prefix_k(np.asarray(prefix_k)[:, b])          # [L][Hkv][P][dh]
    kv_v = model.rnd(np.asarray(prefix_v)[:, b]).transpose(0, 2, 1, 3)
    return kv_k, kv_v


def denoise(cfg, weights: dict, prefix_k, prefix_v, x0, scales: Optional[Dict] = None,
            samples: Optional[List[int]] = None, K: Optional[int] = None,
            model: Optional[PreparedModel] = None, prefix_k_rotated: bool = False) -> np.ndarray:
    """Run the K-step Euler loop for the chosen samples of the batch; returns [len(samples)][H][A].

    Samples are independent (each has its own prefix and noise), so a subset of
    the batch can be checked without the rest.  K defaults to cfg.K; a smaller K
    runs only the first K steps of the same grid (a bounded sample of the work).
    prefix_k_rotated: the prefix K already carries RoPE (R8 does not rotate it again).
    """
    model = model or PreparedModel(cfg, weights)
    samples = list(range(cfg.B)) if samples is None else list(samples)
    if cfg.dtype == "fp8" and scales is None:
        raise ValueError("fp8 workload needs activation scales (see calibrate)")
    Kfull = cfg.K
    ts, dt = time_grid(Kfull)
    nsteps = Kfull if K is None else K
    out = []
    for b in samples:
        kv_k, kv_v = _sample_kv(model, prefix_k, prefix_v, b, prefix_k_rotated)
        x = np.asarray(x0[b], dtype=np.float64).copy()
        for k in range(nsteps):
            x = x + dt * velocity(model, x, k, ts[k], kv_k, kv_v, scales=scales)
        out.append(x)
    return np.stack(out)


def calibrate(cfg, weights: dict, prefix_k, prefix_v, x0,
              model: Optional[PreparedModel] = None) -> Dict:
    """FP8 measure pass (FlashRT walkthrough, component 6, stage (a)).

    Runs the loop over every sample and all K steps with e4m3 weights
    dequantised and projection inputs unquantised, records max|a| of every
    projection input, and returns s_a = amax / 448 per (layer, input) (R11).
    """
    assert cfg.dtype == "fp8"
    model = model or PreparedModel(cfg, weights)
    record: Dict = {}
    ts, dt = time_grid(cfg.K)
    for b in range(cfg.B):
        kv_k, kv_v = _sample_kv(model, prefix_k, prefix_v, b)
        x = np.asarray(x0[b], dtype=np.float64).copy()
        for k in range(cfg.K):
            x = x + dt * velocity(model, x, k, ts[k], kv_k, kv_v, record=record)
    return {key: amax / E4M3_MAX for key, amax in record.items()}


def scales_to_array(cfg, scales: Dict) -> np.ndarray:
    """Flatten {(layer, input): s_a} to [L][4] in PROJ_INPUTS order."""
    arr = np.zeros((cfg.L, len(PROJ_INPUTS)), np.float64)
    for (l, which), s in scales.items():
        arr[l, PROJ_INPUTS.index(which)] = s
    return arr


def array_to_scales(arr) -> Dict:
    arr = np.asarray(arr, np.float64)
    return {(l, w): float(arr[l, i]) for l in range(arr.shape[0]) for i, w in enumerate(PROJ_INPUTS)}


def weight_scales(model: PreparedModel) -> np.ndarray:
    """[L][4] e4m3 weight scales s_w of the fused projections (fp8 workloads)."""
    return np.array([[lay["sw_" + w] for w in PROJ_INPUTS] for lay in model.layers], np.float64)


# --------------------------------------------------------------------------------------
# The prefix pass (R18): the backbone over the observation's tokens, producing the KV cache
# --------------------------------------------------------------------------------------

class PrefixModel:
    """Backbone weights of the prefix pass as the method stores them (R10, R16): the same layer
    block as the action expert (pi0.5's action expert attends to the backbone's per-layer keys and
    values; FlashRT walkthrough, component 5, attention sites of the Pi0.5 model)."""

    def __init__(self, cfg, weights: dict):
        self.cfg = cfg
        self.dtype = cfg.dtype
        self.rnd = round_bf16
        self.layers: List[dict] = [_prepare_layer(cfg.dtype, lw, self.rnd) for lw in weights["layers"]]
        self.cos, self.sin = rope_tables(cfg.P, cfg.dh, cfg.rope_theta)


def prefill(cfg, weights: dict, emb, model: Optional[PrefixModel] = None, samples: Optional[List[int]] = None):
    """Keys and values of every layer for the P prefix tokens of each sample (R18).

    emb [B][P][D]: the embedded tokens.  Per layer: a = RMS(h) gamma1, fused QKV, RoPE at
    positions 0..P-1, K and V stored (bf16, K rotated); then, except after the last layer (whose
    keys and values are all the action expert needs), full attention among the P tokens, the
    O projection and residual, RMS(h) gamma2, gated-GeLU MLP and residual.
    Returns (K, V), each [L][len(samples)][P][Hkv][dh]: the rotated prefix K and V.
    """
    model = model or PrefixModel(cfg, weights)
    rnd = model.rnd
    samples = list(range(cfg.B)) if samples is None else list(samples)
    P, dh, Hq, Hkv = cfg.P, cfg.dh, cfg.Hq, cfg.Hkv
    K_out = np.zeros((cfg.L, len(samples), P, Hkv, dh))
    V_out = np.zeros_like(K_out)
    for si, b in enumerate(samples):
        h = rnd(np.asarray(emb[b], np.float64))         # the caller hands bf16 embeddings
        for l, lay in enumerate(model.layers):
            a = rms_norm(h, lay["g1"], cfg.eps)
            q, k, v = _project(model, l, "qkv", a, (lay["wq"], lay["wk"], lay["wv"]), None, None)
            q = rnd(rope_rotate(q.reshape(P, Hq, dh).transpose(1, 0, 2), model.cos, model.sin))
            k = rnd(rope_rotate(k.reshape(P, Hkv, dh).transpose(1, 0, 2), model.cos, model.sin))
            v = rnd(v.reshape(P, Hkv, dh).transpose(1, 0, 2))
            K_out[l, si] = k.transpose(1, 0, 2)
            V_out[l, si] = v.transpose(1, 0, 2)
            if l == cfg.L - 1:
                break
            o = attention(q, k, v).transpose(1, 0, 2).reshape(P, Hq * dh)
            (dh_o,) = _project(model, l, "o", o, (lay["wo"],), None, None)
            h = h + dh_o
            a = rms_norm(h, lay["g2"], cfg.eps)
            g, u = _project(model, l, "gu", a, (lay["wg"], lay["wu"]), None, None)
            (dh_d,) = _project(model, l, "down", gelu_tanh(g) * u, (lay["wd"],), None, None)
            h = h + dh_d
    return K_out, V_out
