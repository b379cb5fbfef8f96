"""GPU parity: fr_denoise through the C ABI against the CPU oracle on the same seeded inputs.

Tolerances per action chunk (x at t=0): f32 rel-L2 <= 1e-4; bf16 rel-L2 <= 2e-2
and cosine >= 0.999; fp8 cosine >= 0.995 (against the FP8-emulating oracle);
RoPE tables and KV index math bit-exact.
"""
import numpy as np
import pytest

import synthetic
from oracle import oracle as O
from tests import _common as C

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from flow_matching_action_loop_b200 import (  # noqa: E402
    FR_ERR_SHAPE, FR_ERR_STATE, FR_PATH_AUTO, FR_PATH_STEPWISE, FR_PATH_TENSOR, ActionExpertLoop, FrError,
)


def _assert_close(cfg, got, want, label=""):
    rel, cos = C.chunk_metrics(got, want)
    if cfg.dtype == "f32":
        assert np.all(rel <= C.TOL_F32_REL_L2), (label, rel)
    elif cfg.dtype in ("bf16", "w4a16"):   # w4a16: both sides use the same dequantised bf16 operands
        assert np.all(rel <= C.TOL_BF16_REL_L2) and np.all(cos >= C.TOL_BF16_COS), (label, rel, cos)
    else:
        assert np.all(cos >= C.TOL_FP8_COS), (label, rel, cos)
    return rel, cos


def _paths(cfg):
    # bf16/fp8 handles run both kernel sets; the tensor path is requested explicitly so that a
    # configuration it does not support fails instead of silently running the stepwise kernels
    return [FR_PATH_STEPWISE] if cfg.dtype == "f32" else [FR_PATH_STEPWISE, FR_PATH_TENSOR]


SMALL = ["tiny_f32", "ragged_f32", "ragged_bf16", "mha_bf16", "minimal_bf16", "ragged_w4a16"]


@pytest.mark.parametrize("name", SMALL)
def test_parity_small_workloads(name):
    cfg = C.get_config(name)
    inp = C.inputs(name)
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        _assert_close(cfg, got, want, f"{name} path={loop.path}")
        loop.close()


def test_parity_ragged_fp8_with_oracle_scales_and_own_calibration():
    cfg = C.get_config("ragged_fp8")
    inp = C.inputs("ragged_fp8")
    model = O.PreparedModel(cfg, inp["weights"])
    sc = C.oracle_scales(cfg, inp["weights"], model)
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"], scales=sc, model=model)
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path, calibrate=True)
        sa, sw = loop.get_scales()
        # the GPU measure pass agrees with the oracle's within 2^-7 relative
        assert np.allclose(sa, O.scales_to_array(cfg, sc), rtol=C.TOL_CALIB_REL, atol=0)
        assert np.allclose(sw, O.weight_scales(model), rtol=1e-7, atol=0)
        _assert_close(cfg, got, want, "own calibration")
        loop.set_scales(O.scales_to_array(cfg, sc))
        import torch as T
        pk, pv, x0 = C.to_device(inp, cfg, T)
        loop.set_prefix_kv(pk, pv)
        got2 = loop.denoise(x0).cpu().numpy()
        _assert_close(cfg, got2, want, "oracle scales")
        loop.close()


@pytest.mark.slow
def test_parity_pi05_bf16_batch1():
    cfg = synthetic.CONFIGS["pi05_bf16_b1"]
    inp = C.inputs("pi05_bf16_b1")
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        rel, cos = _assert_close(cfg, got, want, f"path={loop.path}")
        print(f"pi05_bf16_b1 {loop.path}: rel-L2 {rel.max():.3e} cos {cos.min():.6f}")
        loop.close()


@pytest.mark.slow
def test_parity_pi05_fp8_batch1():
    cfg = synthetic.CONFIGS["pi05_fp8_b1"]
    inp = C.inputs("pi05_fp8_b1")
    model = O.PreparedModel(cfg, inp["weights"])
    sc = C.oracle_scales(cfg, inp["weights"], model)
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"], scales=sc, model=model)
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path, calibrate=True)
        sa, _ = loop.get_scales()
        assert np.allclose(sa, O.scales_to_array(cfg, sc), rtol=C.TOL_CALIB_REL, atol=0)
        rel, cos = _assert_close(cfg, got, want, f"own calibration, path={loop.path}")
        print(f"pi05_fp8_b1 {loop.path}: rel-L2 {rel.max():.3e} cos {cos.min():.6f}")
        loop.close()


@pytest.mark.slow
def test_parity_pi05_w4a16_batch1():
    cfg = synthetic.CONFIGS["pi05_w4a16_b1"]
    inp = C.inputs("pi05_w4a16_b1")
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        rel, cos = _assert_close(cfg, got, want, f"path={loop.path}")
        print(f"pi05_w4a16_b1 {loop.path}: rel-L2 {rel.max():.3e} cos {cos.min():.6f}")
        loop.close()


@pytest.mark.slow
def test_parity_pi05_bf16_batch32_sampled():
    """Full B=32 launch; the oracle checks three of the independent samples."""
    cfg = synthetic.CONFIGS["pi05_bf16_b32"]
    inp = synthetic.make_inputs(cfg, 0)
    samples = [0, 13, 31]
    model = O.PreparedModel(cfg, inp["weights"])
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"], samples=samples, model=model)
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        _assert_close(cfg, got[samples], want, f"path={loop.path}")
        assert np.all(np.isfinite(got))
        # batch independence: sample 13 alone through a B=1 call of the same handle
        one = {k: v for k, v in inp.items()}
        one["prefix_k"] = inp["prefix_k"][:, 13:14]
        one["prefix_v"] = inp["prefix_v"][:, 13:14]
        one["x0"] = inp["x0"][13:14]
        pk, pv, x0 = C.to_device(one, cfg, torch)
        loop.set_prefix_kv(pk, pv)
        alone = loop.denoise(x0).cpu().numpy()
        _assert_close(cfg, alone, want[1:2], "B=1 rerun")
        loop.close()


@pytest.mark.slow
def test_parity_stress_bf16_batch4_sampled():
    cfg = synthetic.CONFIGS["stress_bf16_b4"]
    inp = synthetic.make_inputs(cfg, 0)
    samples = [2]
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"], samples=samples)
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        _assert_close(cfg, got[samples], want, f"path={loop.path}")
        assert np.all(np.isfinite(got))
        loop.close()


# ------------------------------------------------------------------ closed forms on the GPU

@pytest.mark.parametrize("name", ["tiny_f32", "ragged_bf16", "ragged_fp8"])
def test_zero_network_is_identity_bitwise(name):
    cfg = C.get_config(name)
    inp = dict(C.inputs(name))
    inp["weights"] = synthetic.zero_weights(cfg)
    for path in _paths(cfg):
        sc = np.ones((cfg.L, 4)) if cfg.dtype == "fp8" else None
        got, loop = C.run_library(cfg, inp, path=path, scales=sc)
        assert np.array_equal(got, inp["x0"]), loop.path
        loop.close()


@pytest.mark.parametrize("name", ["tiny_f32", "ragged_bf16"])
def test_constant_field(name):
    cfg = C.get_config(name)
    inp = dict(C.inputs(name))
    w = synthetic.zero_weights(cfg)
    c = np.linspace(-1.0, 1.0, cfg.A).astype(np.float32)
    w["b_out"] = c
    inp["weights"] = w
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        assert np.allclose(got, inp["x0"] - c, atol=2e-6), loop.path
        loop.close()


def test_rope_tables_and_prefix_ingest_bit_exact():
    cfg = C.get_config("ragged_bf16")
    inp = C.inputs("ragged_bf16")
    _, loop = C.run_library(cfg, inp)
    c, s = loop.rope_tables(cfg.P + cfg.H)
    oc, os_ = O.rope_tables(cfg.P + cfg.H, cfg.dh, cfg.rope_theta)
    assert c.tobytes() == oc.tobytes() and s.tobytes() == os_.tobytes()
    model = O.PreparedModel(cfg, inp["weights"])
    for layer, b in ((0, 0), (1, 2)):
        k, v = loop.read_kv(layer, b, cfg.P + cfg.H)
        kf = (k.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        vf = (v.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        # V prefix: a copy into slots 0..P-1 of [Hkv][slots][dh]
        want_v = O.round_bf16(inp["prefix_v"][layer, b]).transpose(1, 0, 2)
        assert np.array_equal(vf[:, :cfg.P], want_v)
        # K prefix: rotated at 0..P-1 in float32 then rounded; within one bf16 ulp of the oracle
        want_k = model.rotate_prefix_k(inp["prefix_k"][:, b])[layer]
        ulp = np.maximum(np.abs(want_k), 1e-30) * 2.0 ** -7
        assert np.all(np.abs(kf[:, :cfg.P] - want_k) <= ulp)
    loop.close()


def test_determinism_and_aliasing():
    cfg = C.get_config("ragged_bf16")
    inp = C.inputs("ragged_bf16")
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        _, _, x0 = C.to_device(inp, cfg, torch)
        again = loop.denoise(x0).cpu().numpy()
        assert np.array_equal(got, again), loop.path           # bitwise reproducible
        loop.denoise(x0, out=x0)                                # in place
        assert np.array_equal(x0.cpu().numpy(), got)
        loop.close()


def test_smaller_batch_and_prefix_than_the_handle_maximum():
    cfg = C.get_config("ragged_bf16")
    small = cfg.replace(B=1, P=40)
    inp = synthetic.make_inputs(small, 5)
    want = O.denoise(small, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
    for path in _paths(cfg):
        got, loop = C.run_library(small, inp, path=path, B_max=cfg.B, P_max=cfg.P)
        _assert_close(small, got, want, f"path={loop.path}")
        loop.close()


def test_automatic_path_is_the_tensor_path_for_bf16_and_fp8():
    for name in ("pi05_bf16_b1", "pi05_fp8_b1", "pi05_w4a16_b1", "pi05_bf16_b32", "stress_bf16_b4", "ragged_bf16",
                 "mha_bf16", "ragged_w4a16"):
        loop = ActionExpertLoop(C.get_config(name), path=FR_PATH_AUTO)
        assert loop.path == "tensor", (name, loop.path)
        loop.close()


def test_misuse_error_codes():
    cfg = C.get_config("ragged_fp8")
    inp = C.inputs("ragged_fp8")
    loop = ActionExpertLoop(cfg)
    pk, pv, x0 = C.to_device(inp, cfg, torch)
    with pytest.raises(FrError) as e:
        loop.denoise(x0)
    assert e.value.code == FR_ERR_STATE                      # no weights
    loop.load_weights(inp["weights"])
    with pytest.raises(FrError) as e:
        loop.denoise(x0)
    assert e.value.code == FR_ERR_STATE                      # no prefix
    loop.set_prefix_kv(pk, pv)
    with pytest.raises(FrError) as e:
        loop.denoise(x0)
    assert e.value.code == FR_ERR_STATE                      # fp8 without scales
    with pytest.raises(FrError) as e:
        loop.set_prefix_kv(torch.zeros((cfg.L, cfg.B, cfg.P + 1, cfg.Hkv, cfg.dh), dtype=torch.bfloat16, device="cuda"),
                           torch.zeros((cfg.L, cfg.B, cfg.P + 1, cfg.Hkv, cfg.dh), dtype=torch.bfloat16, device="cuda"))
    assert e.value.code == FR_ERR_SHAPE                      # P > P_max
    big = torch.zeros((cfg.B + 1, cfg.H, cfg.A), device="cuda")
    loop.set_scales(np.ones((cfg.L, 4)))
    with pytest.raises(FrError) as e:
        loop.denoise(big)
    assert e.value.code == FR_ERR_SHAPE                      # B > B_max
    one = {"prefix_k": inp["prefix_k"][:, :1], "prefix_v": inp["prefix_v"][:, :1], "x0": inp["x0"][:1]}
    pk1, pv1, _ = C.to_device(one, cfg, torch)
    loop.set_prefix_kv(pk1, pv1)
    with pytest.raises(FrError) as e:
        loop.denoise(x0)                                     # prefix for 1 sample, 3 asked
    assert e.value.code == FR_ERR_STATE
    with pytest.raises(FrError):
        loop.set_scales(np.zeros((cfg.L, 4)))
    assert loop.sync_status() == 0
    loop.close()
