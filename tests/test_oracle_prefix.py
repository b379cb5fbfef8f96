"""Pins for the oracle's prefix pass (reading R18; CPU only).

Structural facts the pass must have whatever its weights: layer 0's keys and values of a
token come from that token alone; attention inside the prefix is unmasked, so a later
token reaches an earlier one from layer 1 on; identical tokens give identical values and
keys that differ only by their RoPE position; and the pass's output, handed to the action
expert as an already-rotated prefix, is what the loop consumes.  On top of these, the whole
pass is compared with a second, loop-by-loop formulation that has its own bf16 rounding
(written on the IEEE bit pattern), on a micro backbone with non-unit gains.
"""
import math

import numpy as np

import synthetic
from oracle import oracle as O
from tests._loops import bf16 as _bf16, gelu, matvec as _matvec, rms as _rms, rotate_half

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


# ---------------------------------------------------------------- second formulation (loops)

def _prefill_loops(cfg, w, emb_b):
    """K and V of every layer for one sample, as explicit scalar loops (reading R18, bf16 rounding
    points as R10): h = emb; per layer a = bf16(RMS(h) g1), q/k/v = W a, RoPE at the token's
    position then bf16; after the last layer's QKV nothing more is needed; otherwise softmax
    attention over all P tokens, h += W_o bf16(o), a = bf16(RMS(h) g2), h += W_d bf16(gelu(W_g a) W_u a)."""
    L, Hq, Hkv, dh, P = cfg.L, cfg.Hq, cfg.Hkv, cfg.dh, cfg.P

    def rms(vec, g):
        return _rms(vec, g, cfg.eps)

    def rot(vec, pos):
        return rotate_half(vec, pos, cfg.rope_theta)

    Kl = np.zeros((L, P, Hkv, dh))
    Vl = np.zeros((L, P, Hkv, dh))
    hs = [[_bf16(float(x)) for x in emb_b[p]] for p in range(P)]
    for l, lw in enumerate(w["layers"]):
        W = {n: [[_bf16(float(x)) for x in row] for row in lw[n]] for n in ("wq", "wk", "wv", "wo", "wg", "wu", "wd")}
        g1 = [float(x) for x in lw["g1"]]
        g2 = [float(x) for x in lw["g2"]]
        qs, ks, vs = [], [], []
        for p in range(P):
            a = [_bf16(x) for x in rms(hs[p], g1)]
            q, k, v = _matvec(W["wq"], a), _matvec(W["wk"], a), _matvec(W["wv"], a)
            qs.append([[_bf16(x) for x in rot(q[j * dh:(j + 1) * dh], p)] for j in range(Hq)])
            ks.append([[_bf16(x) for x in rot(k[g * dh:(g + 1) * dh], p)] for g in range(Hkv)])
            vs.append([[_bf16(x) for x in v[g * dh:(g + 1) * dh]] for g in range(Hkv)])
            Kl[l, p] = ks[p]
            Vl[l, p] = vs[p]
        if l == L - 1:
            break
        for p in range(P):
            o = []
            for j in range(Hq):
                g = j * Hkv // Hq
                sc = [sum(qs[p][j][d] * ks[s][g][d] for d in range(dh)) / math.sqrt(dh) for s in range(P)]
                mx = max(sc)
                ex = [math.exp(x - mx) for x in sc]
                tot = sum(ex)
                o += [sum(ex[s] * vs[s][g][d] for s in range(P)) / tot for d in range(dh)]
            hs[p] = [hh + dd for hh, dd in zip(hs[p], _matvec(W["wo"], [_bf16(x) for x in o]))]
            a2 = [_bf16(x) for x in rms(hs[p], g2)]
            gate, up = _matvec(W["wg"], a2), _matvec(W["wu"], a2)
            m = [_bf16(gelu(gg) * uu) for gg, uu in zip(gate, up)]
            hs[p] = [hh + dd for hh, dd in zip(hs[p], _matvec(W["wd"], m))]
    return Kl, Vl


LOOPS = synthetic.PrefixConfig("loops_prefix", L=3, D=16, Hq=4, Hkv=2, dh=4, F=24, B=2, P=5, dtype="bf16")


def _loops_inputs(seed=21):
    """Micro prefix-pass inputs with non-unit gains, so that g1 and g2 are told apart."""
    inp = synthetic.make_prefix_pass_inputs(LOOPS, seed)
    rng = np.random.default_rng(seed + 1)
    for lw in inp["weights"]["layers"]:
        lw["g1"] = (1 + 0.3 * rng.standard_normal(LOOPS.D)).astype(np.float32)
        lw["g2"] = (1 + 0.3 * rng.standard_normal(LOOPS.D)).astype(np.float32)
    return inp


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _worst_layer_rel(K, V, want):
    return max(max(_rel(K[l, si], want[si][0][l]), _rel(V[l, si], want[si][1][l]))
               for si in range(K.shape[1]) for l in range(K.shape[0]))


def test_prefill_matches_loop_formulation():
    """Every layer's K and V of every sample equal the loop formulation's: residuals after the
    O projection and after the MLP, g1 before QKV and g2 before the MLP in every layer, gate
    through GeLU times up, and the last layer's QKV.  The two sides round at the same points;
    only their float64 summation orders differ."""
    inp = _loops_inputs()
    K, V = O.prefill(LOOPS, inp["weights"], inp["emb"])
    want = [_prefill_loops(LOOPS, inp["weights"], inp["emb"][b]) for b in range(LOOPS.B)]
    assert _worst_layer_rel(K, V, want) < 1e-12


def test_prefill_loop_pin_catches_planted_mistakes(monkeypatch):
    """Mistakes planted in the oracle (CPU only) make the loop comparison fail: the pin above is
    not blind to them."""
    inp = _loops_inputs()
    want = [_prefill_loops(LOOPS, inp["weights"], inp["emb"][b]) for b in range(LOOPS.B)]
    # g1 applied where g2 belongs
    w_bad = {"layers": [dict(lw, g2=lw["g1"]) for lw in inp["weights"]["layers"]]}
    K, V = O.prefill(LOOPS, w_bad, inp["emb"])
    assert _worst_layer_rel(K, V, want) > 1e-2
    # gate and up swapped
    real_project = O._project

    def swapped(model, l, which, a, ws, scales, record):
        out = real_project(model, l, which, a, ws, scales, record)
        return out[::-1] if which == "gu" else out

    monkeypatch.setattr(O, "_project", swapped)
    K, V = O.prefill(LOOPS, inp["weights"], inp["emb"])
    assert _worst_layer_rel(K, V, want) > 1e-2
    monkeypatch.setattr(O, "_project", real_project)
    # the MLP's residual update dropped
    monkeypatch.setattr(O, "gelu_tanh", lambda z: np.zeros_like(np.asarray(z, np.float64)))
    K, V = O.prefill(LOOPS, inp["weights"], inp["emb"])
    assert _worst_layer_rel(K, V, want) > 1e-2
