"""Pins for the oracle's prefix pass (reading R18; CPU only).

Structural facts the pass must have whatever its weights: layer 0's keys and values of a
token come from that token alone; attention inside the prefix is unmasked, so a later
token reaches an earlier one from layer 1 on; identical tokens give identical values and
keys that differ only by their RoPE position; and the pass's output, handed to the action
expert as an already-rotated prefix, is what the loop consumes.
"""
import numpy as np

import synthetic
from oracle import oracle as O

MICRO = synthetic.PrefixConfig("micro_prefix", L=3, D=32, Hq=4, Hkv=2, dh=8, F=48, B=2, P=7, dtype="bf16")


def _inputs(cfg=MICRO, seed=0):
    return synthetic.make_prefix_pass_inputs(cfg, seed)


def test_layer0_kv_of_a_token_depend_on_that_token_only():
    inp = _inputs()
    K, V = O.prefill(MICRO, inp["weights"], inp["emb"])
    emb = inp["emb"].copy()
    emb[:, 3] += 1.0                       # change token 3 only
    K2, V2 = O.prefill(MICRO, inp["weights"], emb)
    others = [p for p in range(MICRO.P) if p != 3]
    assert np.array_equal(K[0][:, others], K2[0][:, others])
    assert np.array_equal(V[0][:, others], V2[0][:, others])
    assert not np.array_equal(K[0][:, 3], K2[0][:, 3])
    # from layer 1 on every token has seen token 3
    assert not np.allclose(V[1][:, 0], V2[1][:, 0])


def test_attention_in_the_prefix_is_unmasked():
    """The first token sees the last one (no causal mask inside the prefix)."""
    inp = _inputs(seed=1)
    K, V = O.prefill(MICRO, inp["weights"], inp["emb"])
    emb = inp["emb"].copy()
    emb[:, -1] *= -2.0
    K2, V2 = O.prefill(MICRO, inp["weights"], emb)
    assert not np.allclose(K[1][:, 0], K2[1][:, 0])
    assert not np.allclose(V[2][:, 0], V2[2][:, 0])


def test_identical_tokens_differ_only_by_position():
    """All tokens equal: every layer's values are equal across tokens, and each key is the
    position-0 key rotated to its own position (up to one bf16 rounding)."""
    cfg = MICRO
    inp = _inputs(seed=2)
    emb = np.repeat(inp["emb"][:, :1], cfg.P, axis=1)
    K, V = O.prefill(cfg, inp["weights"], emb)
    cos, sin = O.rope_tables(cfg.P, cfg.dh, cfg.rope_theta)
    for l in range(cfg.L):
        assert np.array_equal(V[l], np.repeat(V[l][:, :1], cfg.P, axis=1))
        k0 = K[l][:, 0].transpose(1, 0, 2)                        # [Hkv][B][dh] at position 0
        for p in range(cfg.P):
            want = O.rope_rotate(k0, cos[p:p + 1].repeat(cfg.B, 0), sin[p:p + 1].repeat(cfg.B, 0))
            got = K[l][:, p].transpose(1, 0, 2)
            assert np.allclose(got, want, rtol=2.0 ** -7, atol=2.0 ** -7 * np.abs(k0).max())


def test_samples_are_independent_and_selectable():
    inp = _inputs(seed=3)
    K, V = O.prefill(MICRO, inp["weights"], inp["emb"])
    K1, V1 = O.prefill(MICRO, inp["weights"], inp["emb"], samples=[1])
    assert np.array_equal(K[:, 1:2], K1) and np.array_equal(V[:, 1:2], V1)


def test_the_loop_consumes_the_rotated_prefix():
    """Prefix pass -> action loop: passing the pass's rotated K as rotated equals passing its
    un-rotated K and letting R8 rotate it, up to the rounding of the round trip."""
    pcfg = MICRO
    ecfg = synthetic.ActionExpertConfig("micro_expert", L=pcfg.L, D=16, Hq=4, Hkv=pcfg.Hkv, dh=pcfg.dh, F=24,
                                        H=3, A=2, B=pcfg.B, P=pcfg.P, K=2, dtype="bf16", time_dim=8)
    pin = _inputs(seed=4)
    K, V = O.prefill(pcfg, pin["weights"], pin["emb"])
    ein = synthetic.make_inputs(ecfg, 5)
    rot = O.denoise(ecfg, ein["weights"], K, V, ein["x0"], prefix_k_rotated=True)
    cos, sin = O.rope_tables(pcfg.P, pcfg.dh, pcfg.rope_theta)
    # rotating by -p undoes position p
    unrot = O.rope_rotate(K.transpose(0, 1, 3, 2, 4), cos, -sin).transpose(0, 1, 3, 2, 4)
    again = O.denoise(ecfg, ein["weights"], unrot, V, ein["x0"])
    rel = np.linalg.norm(rot - again) / np.linalg.norm(rot)
    assert rel < 2e-2
    # and the prefix matters
    other = O.denoise(ecfg, ein["weights"], K[:, ::-1].copy(), V[:, ::-1].copy(), ein["x0"], prefix_k_rotated=True)
    assert np.linalg.norm(other - rot) / np.linalg.norm(rot) > 1e-3
