"""GPU: the execution contract across chunks through the C ABI.

Selective prefix refresh, execution-state capsules (snapshot, restore, fork, going back to
an earlier state), named buffers and the graph-variant table (FlashRT-PAI overview,
mechanisms 2 and 3; FlashRT walkthrough, "exec/" and "serving/").  A capsule or a refresh
only moves state, so the loop run on the moved state must be what the oracle computes on
the same inputs gathered with numpy, and untouched samples must not change by one bit
(the loop is deterministic and samples are independent).
"""
import numpy as np
import pytest

from oracle import oracle as O
from tests import _common as C

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from flow_matching_action_loop_b200 import (  # noqa: E402
    FR_ERR_ARG, FR_ERR_SHAPE, FR_ERR_STATE, FR_EXEC_GRAPH, FR_PATH_STEPWISE, FR_PATH_TENSOR, ActionExpertLoop, FrError,
)

NAME = "ragged_bf16"   # B=3, P=75, Hq/Hkv=4/2, dh=64, H=37, A=7: 4-byte x rows, 16-byte KV rows


def _setup(path=FR_PATH_TENSOR, name=NAME):
    cfg = C.get_config(name)
    inp = C.inputs(name, 0)
    other = C.inputs(name, 5)   # a second observation (only its prefix is used)
    loop = ActionExpertLoop(cfg, path=path)
    loop.load_weights(inp["weights"])
    pk, pv, x0 = C.to_device(inp, cfg, torch)
    qk, qv, _ = C.to_device(other, cfg, torch)
    return cfg, inp, other, loop, (pk, pv, x0), (qk, qv)


def _oracle(cfg, inp, pk, pv, x0):
    return O.denoise(cfg, inp["weights"], pk, pv, x0)


def _close(cfg, got, want, label):
    rel, cos = C.chunk_metrics(got, want)
    if cfg.dtype == "f32":
        assert np.all(rel <= C.TOL_F32_REL_L2), (label, rel)
    else:
        assert np.all(rel <= C.TOL_BF16_REL_L2) and np.all(cos >= C.TOL_BF16_COS), (label, rel, cos)


@pytest.mark.parametrize("path", [FR_PATH_TENSOR, FR_PATH_STEPWISE])
def test_capsule_round_trip_brings_back_the_saved_state(path):
    cfg, inp, other, loop, (pk, pv, x0), (qk, qv) = _setup(path)
    loop.set_prefix_kv(pk, pv)
    y0 = loop.denoise(x0).clone()
    cap = loop.save_capsule(cfg.B, x=x0)
    assert cap[1].B == cfg.B and cap[1].P == cfg.P and cap[1].has_x == 1
    loop.set_prefix_kv(qk, qv)                  # another observation replaces the state
    y1 = loop.denoise(x0).clone()
    assert not torch.equal(y1, y0)
    xr = torch.zeros_like(x0)
    loop.restore_capsule(cap, x_out=xr)         # back to the saved state
    y2 = loop.denoise(xr)
    assert loop.sync_status() == 0
    assert torch.equal(xr, x0)
    assert torch.equal(y2, y0)
    _close(cfg, y2.cpu().numpy(), _oracle(cfg, inp, inp["prefix_k"], inp["prefix_v"], inp["x0"]), "restored")
    _close(cfg, y1.cpu().numpy(), _oracle(cfg, inp, other["prefix_k"], other["prefix_v"], inp["x0"]), "replaced")
    loop.close()


def test_capsule_fork_repeats_and_reorders_samples():
    cfg, inp, _, loop, (pk, pv, x0), _ = _setup()
    loop.set_prefix_kv(pk, pv)
    cap = loop.save_capsule(cfg.B, x=x0)
    smap = [2, 2, 0]
    xf = torch.zeros_like(x0)
    loop.restore_capsule(cap, sample_map=smap, x_out=xf)
    assert torch.equal(xf, x0[smap])
    y = loop.denoise(xf)
    assert loop.sync_status() == 0
    assert torch.equal(y[0], y[1])              # one observation and one noise forked twice
    want = _oracle(cfg, inp, inp["prefix_k"][:, smap], inp["prefix_v"][:, smap], inp["x0"][smap])
    _close(cfg, y.cpu().numpy(), want, "fork")
    # a fork to fewer samples, and the KV rows of a forked slot equal the source slot's
    loop.restore_capsule(cap, sample_map=[1])
    k1, _ = loop.read_kv(0, 0, cfg.P)
    loop.restore_capsule(cap)
    k_ref, _ = loop.read_kv(0, 1, cfg.P)
    assert np.array_equal(k1, k_ref)
    loop.close()


def test_selective_refresh_changes_only_the_given_slots():
    cfg, inp, other, loop, (pk, pv, x0), (qk, qv) = _setup()
    loop.set_prefix_kv(pk, pv)
    y = loop.denoise(x0).clone()
    loop.refresh_prefix_kv(qk[:, [1]].contiguous(), qv[:, [1]].contiguous(), slots=[1])
    y1 = loop.denoise(x0).clone()
    assert torch.equal(y1[0], y[0]) and torch.equal(y1[2], y[2])
    assert not torch.equal(y1[1], y[1])
    mk, mv = inp["prefix_k"].copy(), inp["prefix_v"].copy()
    mk[:, 1], mv[:, 1] = other["prefix_k"][:, 1], other["prefix_v"][:, 1]
    _close(cfg, y1.cpu().numpy(), _oracle(cfg, inp, mk, mv, inp["x0"]), "refresh slot 1")
    # two slots in the order given: source sample 0 -> slot 2, source sample 1 -> slot 0
    loop.refresh_prefix_kv(qk[:, [0, 2]].contiguous(), qv[:, [0, 2]].contiguous(), slots=[2, 0])
    y2 = loop.denoise(x0)
    assert loop.sync_status() == 0
    assert torch.equal(y2[1], y1[1])
    mk[:, 2], mv[:, 2] = other["prefix_k"][:, 0], other["prefix_v"][:, 0]
    mk[:, 0], mv[:, 0] = other["prefix_k"][:, 2], other["prefix_v"][:, 2]
    _close(cfg, y2.cpu().numpy(), _oracle(cfg, inp, mk, mv, inp["x0"]), "refresh slots 2, 0")
    loop.close()


def test_contract_misuse_error_codes():
    cfg, _, _, loop, (pk, pv, x0), _ = _setup()
    with pytest.raises(FrError) as ei:
        loop.refresh_prefix_kv(pk[:, [0]].contiguous(), pv[:, [0]].contiguous(), slots=[0])
    assert ei.value.code == FR_ERR_STATE                       # nothing cached yet
    from flow_matching_action_loop_b200 import fr_capsule_save
    scratch = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(FrError) as ei:
        fr_capsule_save(loop.h, scratch.data_ptr(), scratch.numel(), 1)
    assert ei.value.code == FR_ERR_STATE
    loop.set_prefix_kv(pk, pv)
    with pytest.raises(FrError) as ei:
        loop.refresh_prefix_kv(pk[:, :2, :10].contiguous(), pv[:, :2, :10].contiguous(), slots=[0, 1])
    assert ei.value.code == FR_ERR_SHAPE                       # another prefix length
    with pytest.raises(FrError) as ei:
        loop.refresh_prefix_kv(pk[:, :2].contiguous(), pv[:, :2].contiguous(), slots=[1, 1])
    assert ei.value.code == FR_ERR_ARG                         # a slot twice
    with pytest.raises(FrError) as ei:
        loop.refresh_prefix_kv(pk[:, :1].contiguous(), pv[:, :1].contiguous(), slots=[3])
    assert ei.value.code == FR_ERR_SHAPE                       # beyond the cached batch
    buf, desc = loop.save_capsule(2)                           # without x
    with pytest.raises(FrError) as ei:
        loop.restore_capsule((buf, desc), x_out=torch.zeros_like(x0[:2]))
    assert ei.value.code == FR_ERR_STATE
    with pytest.raises(FrError) as ei:
        loop.restore_capsule((buf, desc), sample_map=[0, 2])
    assert ei.value.code == FR_ERR_ARG                         # the capsule holds 2 samples
    with pytest.raises(FrError) as ei:
        loop.restore_capsule((buf, desc), B=3)
    assert ei.value.code == FR_ERR_SHAPE
    bad = type(desc).from_buffer_copy(desc)
    bad.dh = cfg.dh * 2
    with pytest.raises(FrError) as ei:
        loop.restore_capsule((buf, bad))
    assert ei.value.code == FR_ERR_SHAPE                       # another handle shape
    bad = type(desc).from_buffer_copy(desc)
    bad.magic = 0
    with pytest.raises(FrError) as ei:
        loop.restore_capsule((buf, bad))
    assert ei.value.code == FR_ERR_ARG
    with pytest.raises(FrError) as ei:
        fr_capsule_save(loop.h, buf.data_ptr(), desc.bytes - 1, 2)
    assert ei.value.code == FR_ERR_SHAPE                       # buffer too small
    with pytest.raises(FrError) as ei:
        fr_capsule_save(loop.h, buf.data_ptr(), desc.bytes, cfg.B + 1)
    assert ei.value.code == FR_ERR_SHAPE
    with pytest.raises(FrError) as ei:
        loop.buffer("weights")
    assert ei.value.code == FR_ERR_ARG
    loop.close()


class _DeviceView:
    """A device address seen by torch through the CUDA array interface (no copy)."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
                                         "version": 3}


def test_named_buffers_are_the_state_the_loop_reads():
    cfg, _, _, loop, (pk, pv, x0), _ = _setup()
    loop.set_prefix_kv(pk, pv)
    loop.denoise(x0)
    torch.cuda.synchronize()
    half = cfg.dh // 2
    S = cfg.P + cfg.H
    ptr, n = loop.buffer("rope_cos")
    assert n == S * half * 4
    cos = torch.as_tensor(_DeviceView(ptr, (S, half), "<f4"), device="cuda").cpu().numpy()
    c_ref, _ = loop.rope_tables(S)
    assert np.array_equal(cos, c_ref)
    ptr, n = loop.buffer("kv_k")
    layer_bytes = -(-(cfg.B * cfg.Hkv * S * cfg.dh * 2) // 256) * 256
    assert n == cfg.L * layer_bytes
    kv = torch.as_tensor(_DeviceView(ptr + layer_bytes, (cfg.B, cfg.Hkv, S, cfg.dh), "<i2"), device="cuda")
    k_ref, _ = loop.read_kv(1, 2, S)                           # layer 1, sample 2, prefix + action slots
    assert np.array_equal(kv[2].cpu().numpy(), k_ref.view(np.int16))
    for name, size in (("temb", cfg.K * cfg.D * 4), ("s_act", cfg.L * 16), ("status", 4), ("kv_v", cfg.L * layer_bytes)):
        p, b = loop.buffer(name)
        assert p != 0 and b == size, name
    loop.close()


def test_graph_variant_table_keeps_the_most_recent():
    cfg, _, _, loop, (pk, pv, x0), _ = _setup()
    loop.set_exec_mode(FR_EXEC_GRAPH)   # every batch size through the graph table (B=1 would run the persistent kernel)
    loop.set_prefix_kv(pk, pv)
    y3 = loop.denoise(x0).clone()
    assert loop.graph_count() == 1
    loop.set_graph_capacity(1)
    y2 = loop.denoise(x0[:2].contiguous()).clone()   # another (B, P): the B=3 graph is evicted
    assert loop.graph_count() == 1
    # another batch size may split K differently: equal within the bf16 tolerance, not bitwise
    _close(cfg, y2.cpu().numpy(), y3[:2].cpu().numpy(), "B=2 against B=3")
    assert torch.equal(loop.denoise(x0), y3)         # rebuilt, same result
    loop.set_graph_capacity(2)
    loop.denoise(x0[:1].contiguous())
    assert loop.graph_count() == 2
    loop.set_graph_capacity(1)
    assert loop.graph_count() == 1
    with pytest.raises(FrError) as ei:
        loop.set_graph_capacity(0)
    assert ei.value.code == FR_ERR_ARG
    assert loop.sync_status() == 0
    loop.close()
