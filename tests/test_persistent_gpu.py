"""GPU: the persistent kernel, one cooperative launch per fr_denoise (batch-1-sized calls).

Against the CPU oracle on the same seeded inputs, with the tolerances of every bf16 workload
(rel-L2 <= 2e-2, cosine >= 0.999 per chunk), on shapes ragged in every dimension (tokens not a
multiple of 16, widths not a multiple of 128, several KV heads, 1 to 15 key chunks, head dims 64,
128 and 256) and at the pi0.5 batch-1 size.  The same calls on the CUDA-graph execution agree
within the same tolerance (their split-K factors differ, so not bitwise).  Also: the kernel is
one launch; two calls are bitwise equal; a zero network leaves x
unchanged bit for bit; calls of other batch sizes and prefix lengths follow one another (the
kernel clears its counters for the next call); and a device wait that gives up (a wait bound the
test makes too short) surfaces as FR_ERR_TIMEOUT with the context intact.
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
    FR_ERR_TIMEOUT, FR_ERR_UNSUPPORTED, FR_EXEC_GRAPH, FR_EXEC_PERSISTENT, FR_PATH_TENSOR, ActionExpertLoop, FrError,
)

SHAPES = ["b1_ragged_bf16", "b2_ragged_bf16", "b1_dh128_bf16", "b4_dh256_bf16", "mha_bf16", "minimal_bf16"]


def _close(cfg, got, want, label):
    rel, cos = C.chunk_metrics(got, want)
    assert np.all(rel <= C.TOL_BF16_REL_L2) and np.all(cos >= C.TOL_BF16_COS), (label, rel, cos)
    return rel, cos


@pytest.mark.parametrize("name", SHAPES)
def test_persistent_parity_small(name):
    cfg = C.get_config(name)
    inp = C.inputs(name)
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
    got_p, loop = C.run_library(cfg, inp, path=FR_PATH_TENSOR, exec_mode=FR_EXEC_PERSISTENT)
    assert loop.exec_mode() == FR_EXEC_PERSISTENT and loop.launches_per_call() == 1
    loop.close()
    _close(cfg, got_p, want, f"{name} persistent")
    got_g, loop = C.run_library(cfg, inp, path=FR_PATH_TENSOR, exec_mode=FR_EXEC_GRAPH)
    assert loop.exec_mode() == FR_EXEC_GRAPH
    loop.close()
    _close(cfg, got_g, want, f"{name} graph")
    _close(cfg, got_p, got_g, f"{name} persistent against graph")


def test_persistent_parity_pi05_bf16_batch1():
    cfg = C.get_config("pi05_bf16_b1")
    inp = C.inputs("pi05_bf16_b1")
    want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
    got, loop = C.run_library(cfg, inp, path=FR_PATH_TENSOR, exec_mode=FR_EXEC_PERSISTENT)
    assert loop.exec_mode() == FR_EXEC_PERSISTENT and loop.launches_per_call() == 1
    loop.close()
    rel, cos = _close(cfg, got, want, "persistent")
    print(f"pi05_bf16_b1 persistent: rel-L2 {rel.max():.3e} cos {cos.min():.6f}")


def test_persistent_determinism_aliasing_and_zero_network():
    cfg = C.get_config("b1_ragged_bf16")
    inp = C.inputs("b1_ragged_bf16")
    got, loop = C.run_library(cfg, inp, path=FR_PATH_TENSOR, exec_mode=FR_EXEC_PERSISTENT)
    pk, pv, x0 = C.to_device(inp, cfg, torch)
    again = loop.denoise(x0)
    assert np.array_equal(again.cpu().numpy(), got)                 # fixed-order reductions: bitwise
    inplace = x0.clone()
    loop.denoise(inplace, inplace)                                  # x in and out may alias
    assert np.array_equal(inplace.cpu().numpy(), got)
    assert loop.sync_status() == 0
    loop.close()
    zw = synthetic.zero_weights(cfg)
    zinp = dict(inp, weights=zw)
    out, loop = C.run_library(cfg, zinp, path=FR_PATH_TENSOR, exec_mode=FR_EXEC_PERSISTENT)
    assert np.array_equal(out, inp["x0"])
    loop.close()


def test_persistent_calls_of_other_batch_and_prefix_follow_one_another():
    """One handle (B_max 2, P_max 130): calls of B = 2, 1, 2 at two prefix lengths, each against the
    oracle on its own inputs; the counters the kernel leaves cleared carry no state between calls."""
    cfg = C.get_config("b2_ragged_bf16")
    inp = C.inputs("b2_ragged_bf16")
    loop = ActionExpertLoop(cfg, path=FR_PATH_TENSOR)
    loop.set_exec_mode(FR_EXEC_PERSISTENT)
    loop.load_weights(inp["weights"])
    pk, pv, x0 = C.to_device(inp, cfg, torch)
    for P in (cfg.P, 41):
        small = cfg.replace(P=P)
        loop.set_prefix_kv(pk[:, :, :P].contiguous(), pv[:, :, :P].contiguous())
        want = O.denoise(small, inp["weights"], inp["prefix_k"][:, :, :P], inp["prefix_v"][:, :, :P], inp["x0"])
        for B in (2, 1, 2):
            got = loop.denoise(x0[:B].contiguous()).cpu().numpy()
            _close(small, got, want[:B], f"P={P} B={B}")
    assert loop.sync_status() == 0
    loop.close()


def test_persistent_wait_gives_up_and_the_context_survives():
    """A wait bound of 1 ns makes the kernel's first wait on another CTA give up: the call latches
    FR_ERR_TIMEOUT (read once, then cleared), every CTA returns, and with the default bound the next
    call gives the earlier result bit for bit."""
    cfg = C.get_config("b1_ragged_bf16")
    inp = C.inputs("b1_ragged_bf16")
    got, loop = C.run_library(cfg, inp, path=FR_PATH_TENSOR, exec_mode=FR_EXEC_PERSISTENT)
    pk, pv, x0 = C.to_device(inp, cfg, torch)
    loop.set_wait_limit(1)
    loop.denoise(x0)
    with pytest.raises(FrError) as ei:
        loop.sync_status()
    assert ei.value.code == FR_ERR_TIMEOUT
    assert loop.sync_status() == 0
    loop.set_wait_limit(0)
    again = loop.denoise(x0).cpu().numpy()
    assert loop.sync_status() == 0
    assert np.array_equal(again, got)
    loop.close()


def test_persistent_mode_rejects_calls_it_does_not_serve():
    cfg = C.get_config("ragged_bf16")            # B*H = 111 tokens: more than one 64-token tile
    inp = C.inputs("ragged_bf16")
    loop = ActionExpertLoop(cfg, path=FR_PATH_TENSOR)
    loop.load_weights(inp["weights"])
    pk, pv, x0 = C.to_device(inp, cfg, torch)
    loop.set_prefix_kv(pk, pv)
    assert loop.exec_mode() == FR_EXEC_GRAPH
    loop.set_exec_mode(FR_EXEC_PERSISTENT)
    with pytest.raises(FrError) as ei:
        loop.denoise(x0)
    assert ei.value.code == FR_ERR_UNSUPPORTED
    assert loop.exec_mode(1) == FR_EXEC_PERSISTENT   # one sample of 37 tokens is served
    loop.close()
