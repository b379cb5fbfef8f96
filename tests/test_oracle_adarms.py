"""Pins for the oracle's adaptive-RMSNorm time conditioning (reading R17; CPU only).

The variant is checked against the plain model it must reduce to, against a
second route to the same degenerate network, and against the exact linear
effect of the final norm's shift.
"""
import numpy as np
import pytest

import synthetic
from oracle import oracle as O

MICRO = synthetic.ActionExpertConfig("micro_adarms", L=2, D=8, Hq=4, Hkv=2, dh=4, F=6, H=3, A=2, B=2,
                                     P=2, K=3, dtype="f32", time_dim=8, adarms=True)


def _inputs(cfg, seed=0):
    return synthetic.make_inputs(cfg, seed)


def _run(cfg, inp, w=None, scales=None, K=None):
    w = inp["weights"] if w is None else w
    return O.denoise(cfg, w, inp["prefix_k"], inp["prefix_v"], inp["x0"], scales=scales, K=K)


def _copy(w):
    out = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in w.items() if k != "layers"}
    out["layers"] = [{k: v.copy() for k, v in lw.items()} for lw in w["layers"]]
    return out


@pytest.mark.parametrize("dtype", ["f32", "bf16", "w4a16", "fp8"])
def test_constant_modulation_reduces_to_the_plain_model(dtype):
    """W_mod = 0 and biases (gamma - 1 | 0 | 1) give RMS(h)*gamma, no shift and ungated residuals:
    exactly the plain model with gains gamma and a zero time embedding (R4 off)."""
    cfg = MICRO.replace(dtype=dtype)
    inp = _inputs(cfg)
    rng = np.random.default_rng(7)
    ada = _copy(inp["weights"])
    plain = _copy(inp["weights"])
    D = cfg.D
    for la, lp in zip(ada["layers"], plain["layers"]):
        for n, g in (("1", "g1"), ("2", "g2")):
            gamma = rng.uniform(0.6, 1.8, D).astype(np.float32)
            lp[g] = gamma
            la["w_mod" + n][...] = 0.0
            la["b_mod" + n] = np.concatenate([gamma - np.float32(1.0), np.zeros(D, np.float32),
                                              np.ones(D, np.float32)])
    gf = rng.uniform(0.6, 1.8, D).astype(np.float32)
    plain["g_f"] = gf
    ada["w_modf"][...] = 0.0
    ada["b_modf"] = np.concatenate([gf - np.float32(1.0), np.zeros(D, np.float32)])
    plain["w_t2"][...] = 0.0   # temb = 0: the plain model's added embedding vanishes
    pcfg = cfg.replace(adarms=False)
    scales = None
    if dtype == "fp8":
        scales = O.calibrate(pcfg, plain, inp["prefix_k"], inp["prefix_v"], inp["x0"])
        assert O.calibrate(cfg, ada, inp["prefix_k"], inp["prefix_v"], inp["x0"]) == scales
    got = _run(cfg, inp, ada, scales)
    want = O.denoise(pcfg, plain, inp["prefix_k"], inp["prefix_v"], inp["x0"], scales=scales)
    assert np.array_equal(got, want)


def test_zero_gates_equal_zero_layer_weights():
    """Gates of zero and layer projections of zero are two routes to layers that change nothing."""
    cfg = MICRO
    inp = _inputs(cfg, 3)
    D = cfg.D
    rng = np.random.default_rng(11)
    gated = _copy(inp["weights"])
    zeroed = _copy(inp["weights"])
    for lg, lz in zip(gated["layers"], zeroed["layers"]):
        for n in ("1", "2"):
            s = rng.standard_normal(D).astype(np.float32)
            b = rng.standard_normal(D).astype(np.float32)
            lg["w_mod" + n][...] = 0.0
            lz["w_mod" + n][...] = 0.0
            lg["b_mod" + n] = np.concatenate([s, b, np.zeros(D, np.float32)])
            lz["b_mod" + n] = np.concatenate([s, b, np.ones(D, np.float32)])
        for p in ("wq", "wk", "wv", "wo", "wg", "wu", "wd"):
            lz[p][...] = 0.0
    a = _run(cfg, inp, gated)
    b = _run(cfg, inp, zeroed)
    assert np.array_equal(a, b)
    # and the layers really matter once the gates open
    opened = _copy(gated)
    for lw in opened["layers"]:
        lw["b_mod1"][2 * D:] = 1.0
    assert not np.allclose(_run(cfg, inp, opened), a)


def test_final_shift_moves_one_step_by_dt_w_out_b():
    """One Euler step: a shift b on the final norm adds exactly dt * W_out b to x (R17)."""
    cfg = MICRO.replace(K=1)
    inp = _inputs(cfg, 5)
    D = cfg.D
    base = _copy(inp["weights"])
    base["w_modf"][D:] = 0.0                  # the shift comes from the bias alone
    shifted = _copy(base)
    b = np.random.default_rng(2).standard_normal(D).astype(np.float32)
    shifted["b_modf"][D:] = b
    diff = _run(cfg, inp, shifted) - _run(cfg, inp, base)
    _, dt = O.time_grid(cfg.K)
    want = dt * (np.asarray(inp["weights"]["w_out"], np.float64) @ b.astype(np.float64))
    assert np.allclose(diff, np.broadcast_to(want, diff.shape), rtol=1e-12, atol=1e-14)


def test_condition_is_the_time_embedding_of_each_step():
    """The modulation follows t: with the time MLP zeroed, every step sees the same (zero)
    condition, so the loop equals one with the modulation weights zeroed as well."""
    cfg = MICRO
    inp = _inputs(cfg, 9)
    a = _copy(inp["weights"])
    for k in ("w_t1", "w_t2", "b_t1", "b_t2"):
        a[k][...] = 0.0
    b = _copy(a)
    for lw in b["layers"]:
        lw["w_mod1"][...] = 0.0
        lw["w_mod2"][...] = 0.0
    b["w_modf"][...] = 0.0
    assert np.array_equal(_run(cfg, inp, a), _run(cfg, inp, b))
    # with the time MLP on, the condition and the result change
    assert not np.allclose(_run(cfg, inp), _run(cfg, inp, a))


def test_plain_tensors_do_not_depend_on_the_variant():
    """The adaRMS draws come last: every other tensor equals the plain workload's."""
    cfg = MICRO
    a = _inputs(cfg, 4)
    p = _inputs(cfg.replace(adarms=False), 4)
    for key in ("prefix_k", "prefix_v", "x0"):
        assert np.array_equal(a[key], p[key])
    for k in ("w_in", "w_out", "w_t1", "w_t2"):
        assert np.array_equal(a["weights"][k], p["weights"][k])
    for la, lp in zip(a["weights"]["layers"], p["weights"]["layers"]):
        for k in lp:
            assert np.array_equal(la[k], lp[k])


def _velocity_unfolded(model, x, t, kv_k, kv_v):
    """R17 written with the shift inside the normalised tensor, RMS(h) * (1 + s) + b, before every
    projection (float32 workload: no rounding, so folding W b out must not change the result)."""
    cfg = model.cfg
    P, H, dh, Hq, Hkv, D = cfg.P, cfg.H, cfg.dh, cfg.Hq, cfg.Hkv, cfg.D
    h = x @ model.w_in.T + model.b_in
    c = model.temb(t)
    cos_a, sin_a = model.cos[P:P + H], model.sin[P:P + H]
    for l, lay in enumerate(model.layers):
        m1 = lay["w_mod1"] @ c + lay["b_mod1"]
        a = O.rms_norm(h, 1.0 + m1[:D], cfg.eps) + m1[D:2 * D]
        q = (a @ lay["wq"].T).reshape(H, Hq, dh).transpose(1, 0, 2)
        k = (a @ lay["wk"].T).reshape(H, Hkv, dh).transpose(1, 0, 2)
        v = (a @ lay["wv"].T).reshape(H, Hkv, dh).transpose(1, 0, 2)
        q, k = O.rope_rotate(q, cos_a, sin_a), O.rope_rotate(k, cos_a, sin_a)
        o = O.attention(q, np.concatenate([kv_k[l], k], 1), np.concatenate([kv_v[l], v], 1))
        h = h + m1[2 * D:] * (o.transpose(1, 0, 2).reshape(H, Hq * dh) @ lay["wo"].T)
        m2 = lay["w_mod2"] @ c + lay["b_mod2"]
        a = O.rms_norm(h, 1.0 + m2[:D], cfg.eps) + m2[D:2 * D]
        u = O.gelu_tanh(a @ lay["wg"].T) * (a @ lay["wu"].T)
        h = h + m2[2 * D:] * (u @ lay["wd"].T)
    mf = model.w_modf @ c + model.b_modf
    return (O.rms_norm(h, 1.0 + mf[:D], cfg.eps) + mf[D:]) @ model.w_out.T + model.b_out


def test_folded_shift_equals_the_shift_inside_the_norm():
    cfg = MICRO
    inp = _inputs(cfg, 6)
    w = _copy(inp["weights"])
    rng = np.random.default_rng(1)
    for lw in w["layers"]:   # nonzero biases so that every shift and gate term is exercised
        for n in ("1", "2"):
            lw["b_mod" + n] = rng.standard_normal(3 * cfg.D).astype(np.float32)
    w["b_modf"] = rng.standard_normal(2 * cfg.D).astype(np.float32)
    model = O.PreparedModel(cfg, w)
    ts, _ = O.time_grid(cfg.K)
    for b in range(cfg.B):
        kv_k, kv_v = O._sample_kv(model, inp["prefix_k"], inp["prefix_v"], b)
        x = np.asarray(inp["x0"][b], np.float64)
        for k in range(cfg.K):
            got = O.velocity(model, x, k, ts[k], kv_k, kv_v)
            want = _velocity_unfolded(model, x, ts[k], kv_k, kv_v)
            assert np.allclose(got, want, rtol=1e-11, atol=1e-12)
