"""The tensor-core path's launch plans, computed on the host (fr_debug_plan, no GPU needed).

Every launch of a call is sized by host logic: the token tiling, per projection the split-K cluster,
the ring depth, the epilogue staging pass, the kernel (persistent or not), the k-chunks per ring slot
and the shared memory; then the attention kernel and key split.  These tests check the invariants
the kernels rely on for every workload shape and batch size, on a device described by its SM count
and shared-memory limits (B200: 148 SMs, 227 KB per CTA, 228 KB per SM), and pin the plans the
measured workloads run.
"""
import math

import pytest

import synthetic
from flow_matching_action_loop_b200 import _abi
from tests import _common as C

NSM = 148
STATIC = 2048                          # static shared memory of the GEMM kernels (barriers, rstd)
MAX_DYN = 232448 - STATIC              # one CTA per SM
MAX_DYN2 = 233472 // 2 - 1024 - STATIC  # two CTAs per SM (1 KB reserved per CTA)


def _plan(cfg, B, P, prefix=False):
    c = _abi.make_prefix_config(cfg) if prefix else _abi.make_config(cfg, path=_abi.FR_PATH_TENSOR)
    return _abi.fr_debug_plan(c, B, P, NSM, MAX_DYN, MAX_DYN2)


def _check_invariants(cfg, plan, T, prefix=False):
    NT, Nt = plan["NT"], plan["Nt"]
    assert NT * Nt >= T and Nt % 16 == 0 and 16 <= Nt <= 256
    nt0 = math.ceil(T / 256)
    assert nt0 <= NT <= 2 * nt0
    if T <= 64:
        assert NT == 1
    fp8 = cfg.dtype == "fp8"
    w4 = cfg.dtype == "w4a16"
    for name in _abi.PLAN_GEMMS:
        g = plan[name]
        S, stages, kpu, smem, tiles, NKC = g["S"], g["stages"], g["kpu"], g["smem"], g["tiles"], g["NKC"]
        assert 1 <= S <= min(16, NKC) and stages >= 1 and kpu in (1, 2)
        assert 0 < smem <= MAX_DYN, (name, smem)
        norm = fp8 and name in ("qkv", "gate_up")   # the e4m3 operand is made inside the GEMM
        if kpu == 2:
            # one copy per operand and slot: every split rank holds whole two-chunk slots of bulk-copied operands
            assert not norm and not w4 and NKC % (2 * S) == 0, (name, g)
            units = NKC // S // 2
            assert stages >= 2 or stages == units, (name, g)   # double-buffered, or the whole k-range at once
        if g["persist"]:
            assert name == "gate_up" and cfg.dtype == "bf16" and S == 1 and tiles >= 2 * NSM, g
        elif Nt <= 64:
            assert smem <= MAX_DYN2, (name, g)   # the next kernel's CTA fits beside it
        elif S == 1 and tiles > NSM and not prefix:
            assert smem <= MAX_DYN2, (name, g)   # two CTAs per SM
        assert g["red_tok"] % 16 == 0 and 16 <= g["red_tok"] <= Nt
    assert plan["attn_C"] >= 1 and plan["attn_KC"] % 64 == 0


@pytest.mark.parametrize("name", [n for n, c in synthetic.CONFIGS.items() if c.dtype != "f32"])
def test_workload_plans_keep_the_kernel_invariants(name):
    cfg = synthetic.CONFIGS[name]
    for B in sorted({1, cfg.B}):
        for P in sorted({1, cfg.P // 2, cfg.P}):
            if P < 1:
                continue
            _check_invariants(cfg, _plan(cfg, B, P), B * cfg.H)


@pytest.mark.parametrize("name", [n for n, c in C.RAGGED.items() if c.dtype != "f32"])
def test_ragged_plans_keep_the_kernel_invariants(name):
    cfg = C.get_config(name)
    for B in range(1, cfg.B + 1):
        _check_invariants(cfg, _plan(cfg, B, cfg.P), B * cfg.H)


def test_prefix_pass_plans_keep_the_kernel_invariants():
    cfg = synthetic.PREFIX_CONFIGS["vlm_bf16_p816"]
    for P in (75, 300, 816):
        _check_invariants(cfg, _plan(cfg, 1, P, prefix=True), P, prefix=True)


def test_measured_workloads_run_the_pinned_plans():
    b1 = _plan(synthetic.CONFIGS["pi05_bf16_b1"], 1, 816)
    assert (b1["NT"], b1["Nt"]) == (1, 64) and b1["attn_umma"] == 0 and b1["attn_C"] == 14
    assert [b1[n]["S"] for n in _abi.PLAN_GEMMS] == [6, 16, 2, 16]
    b32 = _plan(synthetic.CONFIGS["pi05_bf16_b32"], 32, 816)
    assert (b32["NT"], b32["Nt"]) == (9, 192) and b32["attn_umma"] == 1
    assert b32["gate_up"]["persist"] == 1 and b32["qkv"]["red_tok"] < 192   # QKV: two CTAs per SM
    assert b32["o"]["kpu"] == 2 and b32["down"]["kpu"] == 2
    stress = _plan(synthetic.CONFIGS["stress_bf16_b4"], 4, 2048)
    assert (stress["NT"], stress["Nt"]) == (2, 208) and stress["gate_up"]["persist"] == 0


def test_plan_errors_before_any_device_work():
    cfg = synthetic.CONFIGS["pi05_bf16_b1"]
    c = _abi.make_config(cfg, path=_abi.FR_PATH_TENSOR)
    for args, code in (((0, 816, NSM, MAX_DYN, MAX_DYN2), _abi.FR_ERR_SHAPE),
                       ((2, 816, NSM, MAX_DYN, MAX_DYN2), _abi.FR_ERR_SHAPE),
                       ((1, 817, NSM, MAX_DYN, MAX_DYN2), _abi.FR_ERR_SHAPE),
                       ((1, 816, 0, MAX_DYN, MAX_DYN2), _abi.FR_ERR_ARG)):
        with pytest.raises(_abi.FrError) as e:
            _abi.fr_debug_plan(c, *args)
        assert e.value.code == code
    f32 = _abi.make_config(synthetic.CONFIGS["tiny_f32"], path=_abi.FR_PATH_TENSOR)
    with pytest.raises(_abi.FrError) as e:
        _abi.fr_debug_plan(f32, 1, 64, NSM, MAX_DYN, MAX_DYN2)
    assert e.value.code == _abi.FR_ERR_UNSUPPORTED
