"""fr_attention_noalloc: the attention op with its merge scratch in the library's own fixed
device array, against fr_attention given a caller-owned scratch buffer.

Two calls in a row on the same stream, with different inputs, each compared with
fr_attention's output on the same inputs: relative L2 <= 1e-2 and cosine >= 0.9999 per
(sample, query head), the attention kernel test's tolerance.  The second call would
show a stale-scratch problem of the first.  This file sorts last so that it also runs
after every other GPU test in one process; it passes alone too.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from flow_matching_action_loop_b200 import (  # noqa: E402
    FR_ATTENTION_NOALLOC_SCRATCH_BYTES, FR_ERR_UNSUPPORTED, FrError, fr_attention, fr_attention_noalloc,
    fr_attention_scratch_bytes, fr_ops_sync_status,
)

CASES = [
    # B, Hq, Hkv, H, S_keys, dh
    (1, 8, 1, 50, 866, 256),    # the π0.5 layer shape: 14 key chunks, 5.8 MB of scratch
    (2, 4, 2, 37, 112, 64),     # ragged: 2 chunks
    (1, 1, 1, 1, 2, 128),       # one chunk: no scratch used
    (4, 8, 1, 128, 320, 64),    # enough query tiles for the tcgen05 kernel: its merge reads the array, 5.6 MB
]


def _inputs(B, Hq, Hkv, H, S, dh, seed):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, Hq, H, dh, generator=g) * 1.5).to(torch.bfloat16).cuda()
    k = torch.randn(B, Hkv, S, dh, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, S, dh, generator=g).to(torch.bfloat16).cuda()
    return q, k, v


def _close(got, want, B, H, Hq, dh):
    g = got.float().cpu().numpy().reshape(B, H, Hq, dh).astype(np.float64)
    w = want.float().cpu().numpy().reshape(B, H, Hq, dh).astype(np.float64)
    for b in range(B):
        for j in range(Hq):
            gj, wj = g[b, :, j, :], w[b, :, j, :]
            rel = np.linalg.norm(gj - wj) / np.linalg.norm(wj)
            cos = np.sum(gj * wj) / (np.linalg.norm(gj) * np.linalg.norm(wj))
            assert rel <= 1e-2 and cos >= 0.9999, (b, j, rel, cos)


@pytest.mark.parametrize("B,Hq,Hkv,H,S,dh", CASES)
def test_noalloc_matches_caller_scratch_on_two_calls(B, Hq, Hkv, H, S, dh):
    assert fr_attention_scratch_bytes(B, Hq, H, S, dh) <= FR_ATTENTION_NOALLOC_SCRATCH_BYTES
    stream = torch.cuda.current_stream().cuda_stream
    runs = []
    for seed in (11, 12):
        q, k, v = _inputs(B, Hq, Hkv, H, S, dh, seed + H + S)
        o = torch.empty(B, H, Hq * dh, dtype=torch.bfloat16, device="cuda")
        fr_attention_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), B, Hq, Hkv, H, S, dh, stream)
        runs.append((q, k, v, o))
    for q, k, v, o in runs:
        nbytes = fr_attention_scratch_bytes(B, Hq, H, S, dh)
        scratch = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(o)
        fr_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), ref.data_ptr(), B, Hq, Hkv, H, S, dh,
                     scratch.data_ptr(), nbytes, stream)
        torch.cuda.synchronize()
        _close(o, ref, B, H, Hq, dh)
    assert fr_ops_sync_status(stream) == 0          # no device wait gave up


def test_noalloc_rejects_sizes_beyond_its_array():
    B, Hq, Hkv, H, S, dh = 2, 8, 1, 50, 866, 256          # 11.6 MB of scratch > 8 MiB
    assert fr_attention_scratch_bytes(B, Hq, H, S, dh) > FR_ATTENTION_NOALLOC_SCRATCH_BYTES
    t = torch.zeros(B * Hq * S * dh, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(FrError) as e:
        fr_attention_noalloc(t.data_ptr(), t.data_ptr(), t.data_ptr(), t.data_ptr(), B, Hq, Hkv, H, S, dh, 0)
    assert e.value.code == FR_ERR_UNSUPPORTED
    assert "scratch" in str(e.value)
