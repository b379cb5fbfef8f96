"""The split-KV attention kernels on their own (fr_attention) against the oracle's attention.

Tolerance per (sample, query head): relative L2 <= 1e-2 and cosine >= 0.9999 -- the output is
rounded to bf16 and P is rounded to bf16 inside the kernel (flash-attention practice).
"""
import numpy as np
import pytest

from oracle import oracle as O

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from flow_matching_action_loop_b200 import FR_ERR_SHAPE, FrError, fr_attention, fr_attention_scratch_bytes  # noqa: E402

CASES = [
    # B, Hq, Hkv, H, S_keys, dh
    (1, 8, 1, 50, 866, 256),    # the π0.5 layer: 14 key chunks
    (2, 4, 2, 37, 112, 64),     # ragged: 2 chunks, owner rows > 16
    (1, 2, 2, 50, 66, 128),     # MHA
    (3, 16, 2, 100, 2148, 128), # stress shapes: 12 chunks of 192
    (1, 1, 1, 1, 2, 128),       # one query row, one chunk (no cluster)
    (1, 4, 1, 128, 900, 64),    # largest query count
    # batched shapes run the tcgen05 kernel (query tiles x key chunks fill the SMs)
    (40, 2, 2, 50, 66, 128),    # one chunk of two sub-chunks, the second of 2 keys
    (12, 8, 1, 50, 866, 256),   # 3 chunks of 5 sub-chunks: online softmax, O rescale, merge
]


@pytest.mark.parametrize("B,Hq,Hkv,H,S,dh", CASES)
def test_attention_kernel_matches_oracle(B, Hq, Hkv, H, S, dh):
    g = torch.Generator().manual_seed(1000 + H + S)
    q = (torch.randn(B, Hq, H, dh, generator=g) * 1.5).to(torch.bfloat16)
    k = torch.randn(B, Hkv, S, dh, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, S, dh, generator=g).to(torch.bfloat16)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty(B, H, Hq * dh, dtype=torch.bfloat16, device="cuda")
    nbytes = fr_attention_scratch_bytes(B, Hq, H, S, dh)
    scratch = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    fr_attention(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), o.data_ptr(), B, Hq, Hkv, H, S, dh,
                 scratch.data_ptr(), nbytes, stream)
    torch.cuda.synchronize()
    got = o.float().cpu().numpy().reshape(B, H, Hq, dh)
    qf, kf, vf = q.double().numpy(), k.double().numpy(), v.double().numpy()
    for b in range(B):
        want = O.attention(qf[b], kf[b], vf[b])           # [Hq][H][dh]
        for j in range(Hq):
            gj, wj = got[b, :, j, :].astype(np.float64), want[j]
            rel = np.linalg.norm(gj - wj) / np.linalg.norm(wj)
            cos = np.sum(gj * wj) / (np.linalg.norm(gj) * np.linalg.norm(wj))
            assert rel <= 1e-2 and cos >= 0.9999, (b, j, rel, cos)


def test_attention_kernel_rejects_small_scratch():
    B, Hq, Hkv, H, S, dh = 1, 8, 1, 50, 866, 256
    need = fr_attention_scratch_bytes(B, Hq, H, S, dh)
    assert need > 0
    t = torch.zeros(B * max(Hq, Hkv) * S * dh, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(FrError) as e:
        fr_attention(t.data_ptr(), t.data_ptr(), t.data_ptr(), t.data_ptr(), B, Hq, Hkv, H, S, dh,
                     t.data_ptr(), need - 16, 0)
    assert e.value.code == FR_ERR_SHAPE
