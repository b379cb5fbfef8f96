"""Pins for the oracle's number formats and elementwise pieces (CPU only).

Each test ties an oracle function to something other than itself: a library
routine (torch's dtype conversions, math.erf, scipy's expit), a public format
specification (tests/golden), exhaustive enumeration, or a closed form.
"""
import math
import os

import numpy as np
import torch

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- bf16

def test_bf16_rounding_matches_torch_rne():
    rng = np.random.default_rng(123)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(5000) * 1e-20).astype(np.float32),
        (rng.standard_normal(5000) * 1e20).astype(np.float32),
    ])
    # exact ties: bf16 value + half an ulp (bit 15 set, lower bits clear)
    ties = (rng.integers(0x3F000000, 0x41000000, 4000, dtype=np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = np.concatenate([x, ties.view(np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_every_normal_pattern_round_trips():
    bits = np.arange(0, 0x10000, dtype=np.int64)
    exps = (bits >> 7) & 0xFF
    bits = bits[(exps > 0) & (exps < 0xFF)]
    vals = np.array([O.decode_bf16(int(b)) for b in bits])
    assert np.array_equal(O.round_bf16(vals), vals)
    # the decoder agrees with reinterpreting the pattern as the top half of a float32
    f32 = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(vals, f32)


# ---------------------------------------------------------------- e4m3

def _golden_e4m3():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_ocp_encodings.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                rows.append((int(c, 16), float(v)))
    return rows


def test_e4m3_decoder_matches_ocp_table():
    rows = _golden_e4m3()
    assert len(rows) >= 8
    for code, value in rows:
        assert O.decode_e4m3(code) == value, hex(code)
    assert math.isnan(O.decode_e4m3(0x7F)) and math.isnan(O.decode_e4m3(0xFF))


def test_e4m3_all_finite_codes_round_trip():
    n = 0
    for code in range(256):
        v = O.decode_e4m3(code)
        if math.isnan(v):
            continue
        n += 1
        assert O.round_e4m3(v) == v, hex(code)
    assert n == 254
    assert O.E4M3_MAX == O.decode_e4m3(0x7E)


def test_e4m3_matches_torch_in_range_and_saturates():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.uniform(-448, 448, 100000),
                        rng.standard_normal(100000) * 0.01,
                        rng.standard_normal(20000) * 1e-3])
    x = x.astype(np.float32).astype(np.float64)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(O.round_e4m3(x), want)
    # values beyond the largest finite code saturate instead of overflowing
    assert O.round_e4m3(1e6) == 448.0 and O.round_e4m3(-463.9) == -448.0
    # ties go to even: 2^-10 lies between 0 and 2^-9
    assert O.round_e4m3(2.0 ** -10) == 0.0 and O.round_e4m3(3 * 2.0 ** -10) == 2 * 2.0 ** -9


def test_e4m3_exact_on_scaled_grid():
    """Quantise -> dequantise is exact for representable multiples of the scale."""
    s = 0.0123
    codes = np.array([O.decode_e4m3(c) for c in range(256) if not math.isnan(O.decode_e4m3(c))])
    w = codes * s
    assert np.array_equal(O.round_e4m3(w / s) * s, w)


# ---------------------------------------------------------------- elementwise

def test_gelu_tanh_against_erf_gelu_and_symmetry():
    z = np.linspace(-6, 6, 2401)
    exact = np.array([0.5 * t * (1 + math.erf(t / math.sqrt(2))) for t in z])
    g = O.gelu_tanh(z)
    assert np.max(np.abs(g - exact)) < 5e-4      # tanh form tracks erf GeLU closely
    assert O.gelu_tanh(0.0) == 0.0
    assert np.allclose(O.gelu_tanh(z) - O.gelu_tanh(-z), z, atol=1e-12)
    # dropping the cubic term would miss by more than the bound
    no_cubic = 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * z))
    assert np.max(np.abs(no_cubic - exact)) > 5e-3


def test_silu_against_scipy():
    from scipy.special import expit
    z = np.linspace(-30, 30, 1001)
    assert np.allclose(O.silu(z), z * expit(z), rtol=1e-14, atol=1e-300)


def test_rms_norm_unit_rms_and_hand_example():
    rng = np.random.default_rng(0)
    h = rng.standard_normal((7, 64)) * 5
    y = O.rms_norm(h, np.ones(64), 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-12)
    assert np.allclose(O.rms_norm(3.5 * h, np.ones(64), 0.0), y, atol=1e-12)
    assert np.allclose(O.rms_norm(np.array([3.0, 4.0]), np.array([1.0, 2.0]), 0.0),
                       [3 / math.sqrt(12.5), 8 / math.sqrt(12.5)])
    # eps enters under the square root
    assert np.allclose(O.rms_norm(np.array([0.0, 0.0]), np.ones(2), 1e-6), 0.0)
    assert np.allclose(O.rms_norm(np.array([1e-3, 1e-3]), np.ones(2), 1e-6),
                       1e-3 / math.sqrt(1e-6 + 1e-6))


# ---------------------------------------------------------------- time

def _golden_grid():
    rows = []
    with open(os.path.join(GOLDEN, "euler_grid_k10.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals = [float(v) for v in line.split()]
                K = int(vals[0])
                rows.append((K, vals[1:1 + K], vals[1 + K]))
    return rows


def test_time_grid_and_euler_direction():
    for K, ts_want, total in _golden_grid():
        ts, dt = O.time_grid(K)
        assert np.allclose(ts, ts_want, atol=1e-15) and dt == -1.0 / K
        x = O.euler(lambda x, t, k: np.full_like(x, t), np.zeros(3), K)
        assert np.allclose(x, total, atol=1e-14)


def test_euler_linear_field_closed_form():
    x0 = np.array([1.0, -2.0, 0.5])
    for K in (1, 2, 10):
        for lam in (-1.3, 0.7):
            x = O.euler(lambda x, t, k: lam * x, x0, K)
            assert np.allclose(x, (1 - lam / K) ** K * x0, rtol=1e-13)


def test_sinusoidal_embedding_layout():
    e0 = O.sinusoidal_embedding(0.0, 256, 1e4)
    assert np.array_equal(e0, np.concatenate([np.zeros(128), np.ones(128)]))   # sin half first
    t = 1e-7
    e = O.sinusoidal_embedding(t, 256, 1e4)
    assert math.isclose(e[0], math.sin(t), rel_tol=1e-12)                       # w_0 = 1
    # w_i = base^(-i/half): the last frequency is 1e4^(-127/128), not 1e4^(-1)
    assert math.isclose(e[127] / t, 1e4 ** (-127 / 128), rel_tol=1e-9)
    assert np.allclose(e[:128] ** 2 + e[128:] ** 2, 1.0, atol=1e-15)


# ---------------------------------------------------------------- RoPE

def test_rope_hand_example_rotate_half_pairing():
    c, s = O.rope_tables(2, 4, 1e4)       # frequencies 1 and 1e4^(-1/2) = 0.01
    z = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0]])
    out = O.rope_rotate(z, np.repeat(c[1:2], 2, 0), np.repeat(s[1:2], 2, 0))
    c1, s1 = float(np.float32(math.cos(1.0))), float(np.float32(math.sin(1.0)))
    c2, s2 = float(np.float32(math.cos(0.01))), float(np.float32(math.sin(0.01)))
    assert np.allclose(out[0], [c1, 0.0, s1, 0.0], atol=1e-15)
    assert np.allclose(out[1], [0.0, c2, 0.0, s2], atol=1e-15)


def test_rope_invariants():
    rng = np.random.default_rng(1)
    dh = 64
    c, s = O.rope_tables(200, dh, 1e4)
    assert np.array_equal(c[0], np.ones(dh // 2, np.float32)) and np.array_equal(s[0], np.zeros(dh // 2, np.float32))
    q = rng.standard_normal(dh)
    k = rng.standard_normal(dh)

    def R(z, p):
        return O.rope_rotate(z[None], c[p:p + 1], s[p:p + 1])[0]
    # position 0 is the identity; norms are preserved up to the float32 table rounding
    assert np.allclose(R(q, 0), q, atol=0)
    for p in (1, 17, 199):
        assert abs(np.linalg.norm(R(q, p)) - np.linalg.norm(q)) < 1e-6 * np.linalg.norm(q)
    # the score depends only on the relative position m - n
    d1 = R(q, 50) @ R(k, 30)
    d2 = R(q, 120) @ R(k, 100)
    d3 = R(q, 20) @ R(k, 0)
    assert abs(d1 - d2) < 1e-5 and abs(d1 - d3) < 1e-5
    assert abs(d1 - R(q, 31) @ R(k, 30)) > 1e-3


def test_rope_tables_float32_rounding_once():
    c, s = O.rope_tables(866, 256, 1e4)
    assert c.dtype == np.float32 and s.dtype == np.float32
    # cos^2 + sin^2 = 1 up to one float32 rounding of each entry
    r = c.astype(np.float64) ** 2 + s.astype(np.float64) ** 2
    assert np.max(np.abs(r - 1)) < 2.5e-7
    # a position with a large angle still matches float64 math rounded once
    inv = 1e4 ** (-2 * 3 / 256)
    assert c[865, 3] == np.float32(math.cos(865 * inv))


# ---------------------------------------------------------------- 4-bit group weights (R16)

def test_w4_quantiser_closed_forms():
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((6, 300)) / 17.0).astype(np.float32)   # ragged last group: 300 = 2 x 128 + 44
    q, s = O.quantize_w4(w)
    assert q.dtype == np.int8 and s.shape == (6, 3)
    assert q.min() >= -7 and q.max() <= 7
    for r in range(6):
        for g in range(3):
            blk = w[r, g * 128:(g + 1) * 128].astype(np.float64)
            amax = np.max(np.abs(blk))
            # the scale is amax / 7 rounded to bf16 (torch's RNE conversion, an independent rounding)
            assert s[r, g] == torch.tensor(amax / 7.0, dtype=torch.float64).to(torch.bfloat16).double().item()
            qb = q[r, g * 128:(g + 1) * 128].astype(np.float64)
            # every code is the nearest integer to w / s (ties to even), clamped: |w/s - q| <= 1/2 inside the range
            ratio = blk / s[r, g]
            inside = np.abs(ratio) <= 7.0
            assert np.all(np.abs(ratio[inside] - qb[inside]) <= 0.5)
            assert np.all(np.abs(qb[~inside]) == 7)
            # the largest magnitude lands at +-7: amax / s = 7 / (1 +- 2^-9) rounds to 7
            k = int(np.argmax(np.abs(blk)))
            assert abs(int(q[r, g * 128 + k])) == 7


def test_w4_quantiser_special_cases():
    # an all-zero group: zero scale, zero codes, zero operand
    w = np.zeros((2, 256), np.float32)
    w[1, 128:] = 1.0
    q, s = O.quantize_w4(w)
    assert s[0, 0] == 0 and s[0, 1] == 0 and s[1, 0] == 0 and not q[0].any() and not q[1, :128].any()
    # a group of one repeated value v: s = bf16(v / 7); the codes all equal round(v / s) = 7
    assert s[1, 1] == torch.tensor(1.0 / 7.0, dtype=torch.float64).to(torch.bfloat16).double().item()
    assert np.all(q[1, 128:] == 7)
    # exact grid: w = k * s0 with a power-of-two s0 and integer k in [-7, 7] comes back exactly
    s0 = 2.0 ** -5
    ks = np.tile(np.arange(-7, 8), 10)[:128]
    ks[0] = 7                                   # make max|w| = 7 s0 so that s = s0 exactly
    w = (ks * s0).astype(np.float32)[None, :]
    q, s = O.quantize_w4(w)
    assert s[0, 0] == s0 and np.array_equal(q[0], ks)
    assert np.array_equal(O.dequantize_w4(q, s)[0], ks * s0)


def test_w4_dequantised_operand_is_bf16_of_the_exact_product():
    rng = np.random.default_rng(8)
    w = (rng.standard_normal((4, 256)) * 0.05).astype(np.float32)
    q, s = O.quantize_w4(w)
    deq = O.dequantize_w4(q, s)
    # q * s (3 magnitude bits times an 8-bit bf16 significand) is exact in float32, so torch's
    # float32 -> bf16 conversion of the float32 product is the same single rounding
    prod32 = torch.from_numpy(q.astype(np.float32)) * torch.from_numpy(np.repeat(s, 128, axis=1).astype(np.float32))
    assert np.array_equal(deq, prod32.to(torch.bfloat16).double().numpy())
    # and the operand stays within half a code step plus one bf16 rounding of w
    step = np.repeat(s, 128, axis=1)
    assert np.all(np.abs(deq - w) <= 0.5 * step + np.abs(deq) * 2.0 ** -8 + 1e-30)
