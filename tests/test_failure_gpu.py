"""GPU: failure detection without a GPU fault.

A device wait that nothing completes gives up after its limit, latches the timeout bit and a
where-code in the handle's status word and lets the kernel return; fr_sync_status reports
FR_ERR_TIMEOUT once and clears the word; the context stays usable and the loop still gives
the same result bit for bit.
"""
import numpy as np
import pytest

from tests import _common as C

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from flow_matching_action_loop_b200 import (  # noqa: E402
    FR_ERR_ARG, FR_ERR_TIMEOUT, FR_PATH_TENSOR, FrError, fr_selftest_wait,
)


def test_bounded_wait_gives_up_and_the_context_survives():
    cfg = C.get_config("ragged_bf16")
    inp = C.inputs("ragged_bf16")
    got, loop = C.run_library(cfg, inp, path=FR_PATH_TENSOR)
    fr_selftest_wait(loop.h, 2_000_000, loop._stream())        # a 2 ms wait that nothing completes
    with pytest.raises(FrError) as ei:
        loop.sync_status()
    assert ei.value.code == FR_ERR_TIMEOUT
    assert "000007f0" in str(ei.value)                          # the self-test's where-code
    assert loop.sync_status() == 0                              # read and cleared
    pk, pv, x0 = C.to_device(inp, cfg, torch)
    loop.set_prefix_kv(pk, pv)
    again = loop.denoise(x0).cpu().numpy()
    assert loop.sync_status() == 0
    assert np.array_equal(again, got)
    for bad in (10, 10 ** 9):
        with pytest.raises(FrError) as ei:
            fr_selftest_wait(loop.h, bad, loop._stream())
        assert ei.value.code == FR_ERR_ARG
    loop.close()
