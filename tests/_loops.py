"""Scalar helpers of the loop-by-loop second formulations the oracle is pinned against (CPU only).

They share nothing with the oracle: bf16 rounding is written on the IEEE-754 bit pattern (the
oracle uses frexp/rint), and products are explicit Python sums (the oracle uses numpy matmul)."""
import math
import struct


def bf16(v: float) -> float:
    """Round a float64 to 8 significant bits, ties to even, on its IEEE-754 bit pattern."""
    if v == 0.0 or not math.isfinite(v):
        return v
    b = struct.unpack("<Q", struct.pack("<d", v))[0]
    drop = 45                                     # 52 fraction bits -> 7
    rem = b & ((1 << drop) - 1)
    half = 1 << (drop - 1)
    b >>= drop
    if rem > half or (rem == half and (b & 1)):
        b += 1                                    # a carry into the exponent is the right result
    return struct.unpack("<d", struct.pack("<Q", b << drop))[0]


def matvec(W, x):
    return [sum(W[n][c] * x[c] for c in range(len(x))) for n in range(len(W))]


def gelu(z: float) -> float:
    return 0.5 * z * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


def rope_entry(pos: int, j: int, dh: int, theta: float):
    """(cos, sin) of pos * theta^(-2j/dh) in float64, each rounded once to float32 (reading R6)."""
    import numpy as np
    ang = pos * math.pow(theta, -2.0 * j / dh)
    return float(np.float32(math.cos(ang))), float(np.float32(math.sin(ang)))


def rotate_half(vec, pos: int, theta: float):
    dh = len(vec)
    half = dh // 2
    out = list(vec)
    for j in range(half):
        c, s = rope_entry(pos, j, dh, theta)
        out[j] = vec[j] * c - vec[j + half] * s
        out[j + half] = vec[j] * s + vec[j + half] * c
    return out


def rms(vec, g, eps):
    ms = sum(a * a for a in vec) / len(vec)
    return [a / math.sqrt(ms + eps) * gg for a, gg in zip(vec, g)]
