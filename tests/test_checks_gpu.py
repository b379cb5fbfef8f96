"""GPU: device bounds checks of the checked build (libflowloop_checked.so, -DFR_DEVICE_CHECKS).

In a child process that loads the checked build: the loop runs with no check firing and matches the
oracle; then a buffer is declared smaller than it is (fr_debug_limit_extent), so that the stores
past the declared extent are refused without any access leaving the real allocation.  The call
reports FR_ERR_DEVICE with the store site's where-code, and with the real extents restored the next
call gives the first result bit for bit.  Both executions are covered: the CUDA graph (GEMM residual
epilogue, 0x9001; attention output, 0x9010) and the persistent kernel (in-proj, 0xa021; attention
output, 0xa010).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED = os.path.join(ROOT, "flow_matching_action_loop_b200", "libflowloop_checked.so")

CHILD = r'''
import numpy as np, torch
from flow_matching_action_loop_b200 import (FR_ERR_DEVICE, FR_EXEC_GRAPH, FR_EXEC_PERSISTENT, FR_PATH_TENSOR,
                                            FrError, fr_device_checks)
from oracle import oracle as O
from tests import _common as C
assert fr_device_checks()
cfg = C.get_config("b1_ragged_bf16")
inp = C.inputs("b1_ragged_bf16")
want = O.denoise(cfg, inp["weights"], inp["prefix_k"], inp["prefix_v"], inp["x0"])
for mode, cases in ((FR_EXEC_GRAPH, (("h", 64, "00009001"), ("obuf", 256, "00009010"))),
                    (FR_EXEC_PERSISTENT, (("h", 64, "0000a021"), ("obuf", 256, "0000a010")))):
    got, loop = C.run_library(cfg, inp, path=FR_PATH_TENSOR, exec_mode=mode)
    rel, cos = C.chunk_metrics(got, want)
    assert np.all(rel <= C.TOL_BF16_REL_L2) and np.all(cos >= C.TOL_BF16_COS), (mode, rel, cos)
    pk, pv, x0 = C.to_device(inp, cfg, torch)
    for buf, limit, where in cases:
        loop.limit_extent(buf, limit)
        loop.denoise(x0)
        try:
            loop.sync_status()
            raise AssertionError(f"{buf}: no bounds check fired")
        except FrError as e:
            assert e.code == FR_ERR_DEVICE, (buf, e)
            assert where in str(e), (buf, where, str(e))
        assert loop.sync_status() == 0            # read and cleared
        loop.limit_extent(buf, 0)
        again = loop.denoise(x0).cpu().numpy()
        assert loop.sync_status() == 0
        assert np.array_equal(again, got), buf
    loop.close()
print("CHECKS_OK")
'''


def _checked_library():
    if not os.path.exists(CHECKED):
        r = subprocess.run([sys.executable, os.path.join(ROOT, "flow_matching_action_loop_b200", "build.py"), "--checked"],
                           capture_output=True, text=True, timeout=1200)
        assert r.returncode == 0, r.stdout + r.stderr
    return CHECKED


def test_bounds_checks_fire_on_declared_extents_and_clear():
    env = dict(os.environ, FR_LIBRARY=_checked_library(), PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "CHECKS_OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
