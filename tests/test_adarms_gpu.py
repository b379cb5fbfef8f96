"""GPU parity of the adaptive-RMSNorm time conditioning (reading R17) through the C ABI.

Both kernel sets run the variant: the tensor path applies the per-step gains 1 + s in its
norm staging, adds the folded shifts W b in the QKV and gate|up epilogues and scales the
residual updates by the gates; the stepwise kernels do the same with their GEMM's bias and
gate terms.  Tolerances are those of the plain workloads.
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
    FR_ERR_ARG, FR_PATH_STEPWISE, FR_PATH_TENSOR, ActionExpertLoop, FrError,
)


def _paths(cfg):
    return [FR_PATH_STEPWISE] if cfg.dtype == "f32" else [FR_PATH_STEPWISE, FR_PATH_TENSOR]


def _assert_close(cfg, got, want, label):
    rel, cos = C.chunk_metrics(got, want)
    if cfg.dtype == "f32":
        assert np.all(rel <= C.TOL_F32_REL_L2), (label, rel)
    elif cfg.dtype == "fp8":
        assert np.all(cos >= C.TOL_FP8_COS), (label, rel, cos)
    else:
        assert np.all(rel <= C.TOL_BF16_REL_L2) and np.all(cos >= C.TOL_BF16_COS), (label, rel, cos)
    return rel, cos


@pytest.mark.parametrize("name", ["ragged_adarms_f32", "ragged_adarms_bf16", "ragged_adarms_w4a16"])
def test_adarms_parity_small(name):
    cfg = C.get_config(name)
    inp = C.inputs(name)
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
    plain = O.denoise(cfg.replace(adarms=False), inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
    assert C.chunk_metrics(plain, want)[0].min() > 0.05   # the variant changes the result
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        _assert_close(cfg, got, want, f"{name} path={loop.path}")
        loop.close()


def test_adarms_fp8_own_calibration():
    name = "ragged_adarms_fp8"
    cfg = C.get_config(name)
    inp = C.inputs(name)
    model = O.PreparedModel(cfg, inp["weights"])
    sc = C.oracle_scales(cfg, inp["weights"], model)
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"], scales=sc, model=model)
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path, calibrate=True)
        sa, _ = loop.get_scales()
        assert np.allclose(sa, O.scales_to_array(cfg, sc), rtol=C.TOL_CALIB_REL, atol=0)
        _assert_close(cfg, got, want, f"path={loop.path}")
        loop.close()


@pytest.mark.parametrize("name", ["ragged_adarms_bf16", "ragged_adarms_f32"])
def test_adarms_zero_network_is_identity_bitwise(name):
    """Every weight and modulation zero: gates are zero, the final norm's input is zero, v = 0."""
    cfg = C.get_config(name)
    inp = dict(C.inputs(name))
    w = synthetic.zero_weights(cfg)
    synthetic.make_modulation(cfg, np.random.default_rng(0), w)
    for lw in w["layers"]:
        lw["w_mod1"][...] = 0.0
        lw["w_mod2"][...] = 0.0
    w["w_modf"][...] = 0.0
    inp["weights"] = w
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        assert np.array_equal(got, inp["x0"]), loop.path
        loop.close()


def test_adarms_handle_needs_the_modulation_weights():
    cfg = C.get_config("ragged_adarms_bf16")
    inp = C.inputs("ragged_bf16")   # the plain workload's weights: no modulation tensors
    loop = ActionExpertLoop(cfg, path=FR_PATH_TENSOR)
    with pytest.raises(FrError) as ei:
        loop.load_weights(inp["weights"])
    assert ei.value.code == FR_ERR_ARG
    loop.close()


@pytest.mark.slow
def test_parity_pi05_adarms_bf16_batch1():
    cfg = synthetic.CONFIGS["pi05_adarms_bf16_b1"]
    inp = C.inputs("pi05_adarms_bf16_b1")
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
    for path in _paths(cfg):
        got, loop = C.run_library(cfg, inp, path=path)
        rel, cos = _assert_close(cfg, got, want, f"path={loop.path}")
        print(f"pi05_adarms_bf16_b1 {loop.path}: rel-L2 {rel.max():.3e} cos {cos.min():.6f}")
        loop.close()
