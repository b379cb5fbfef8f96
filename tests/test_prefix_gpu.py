"""GPU parity of the prefix pass (reading R18) through the C ABI.

fr_prefill runs the backbone over the embedded prefix tokens on the tensor-core kernels and
leaves every layer's rotated K and its V in the KV cache; the oracle computes the same from
the same seeded inputs.  Per layer the keys and values must agree within the bf16 tolerance,
and the action loop fed by the pass must match the oracle's loop fed by the oracle's pass.
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
    FR_ERR_SHAPE, FR_ERR_STATE, FR_PATH_TENSOR, ActionExpertLoop, FrError, PrefixPass,
)

# 75 tokens: the warp-MMA attention kernel; 300 tokens: tcgen05 attention and RoPE staged per token
SMALL = {
    "prefix_p75": synthetic.PrefixConfig("prefix_p75", L=3, D=320, Hq=4, Hkv=2, dh=64, F=704, B=2, P=75, dtype="bf16"),
    "prefix_p300": synthetic.PrefixConfig("prefix_p300", L=2, D=256, Hq=4, Hkv=2, dh=64, F=512, B=1, P=300,
                                          dtype="bf16"),
    "prefix_w4_p150": synthetic.PrefixConfig("prefix_w4_p150", L=2, D=256, Hq=2, Hkv=2, dh=64, F=256, B=2, P=150,
                                             dtype="w4a16"),
}


def _kv_metrics(got, want):
    got = np.asarray(got, np.float64).ravel()
    want = np.asarray(want, np.float64).ravel()
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    cos = float(got @ want / (np.linalg.norm(got) * np.linalg.norm(want)))
    return rel, cos


def _bf16_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _run_pass(cfg, inp, expert=None):
    pp = PrefixPass(cfg)
    pp.load_weights(inp["weights"])
    emb = torch.from_numpy(inp["emb"]).to("cuda").to(torch.bfloat16).contiguous()
    pp.run(emb, expert)
    assert pp.sync_status() == 0
    torch.cuda.synchronize()
    return pp


def _pass_kv(pp, cfg):
    """[L][B][P][Hkv][dh] K and V from the pass handle's cache."""
    K = np.zeros((cfg.L, cfg.B, cfg.P, cfg.Hkv, cfg.dh))
    V = np.zeros_like(K)
    for l in range(cfg.L):
        for b in range(cfg.B):
            k, v = pp.read_kv(l, b, cfg.P)                     # [Hkv][P][dh] bf16 bits
            K[l, b] = _bf16_to_f64(k).transpose(1, 0, 2)
            V[l, b] = _bf16_to_f64(v).transpose(1, 0, 2)
    return K, V


@pytest.mark.parametrize("name", sorted(SMALL))
def test_prefix_pass_kv_parity(name):
    cfg = SMALL[name]
    inp = synthetic.make_prefix_pass_inputs(cfg, 0)
    Kw, Vw = O.prefill(cfg, inp["weights"], inp["emb"])
    pp = _run_pass(cfg, inp)
    K, V = _pass_kv(pp, cfg)
    for l in range(cfg.L):
        for what, got, want in (("K", K[l], Kw[l]), ("V", V[l], Vw[l])):
            rel, cos = _kv_metrics(got, want)
            assert rel <= C.TOL_BF16_REL_L2 and cos >= C.TOL_BF16_COS, (name, l, what, rel, cos)
    assert pp.launches_per_call() == 1 + 5 * (cfg.L - 1) + 1
    pp.close()


def test_prefix_pass_feeds_the_loop():
    pcfg = SMALL["prefix_p75"]
    ecfg = C.RAGGED["ragged_bf16"].replace(name="ragged_from_prefix", L=pcfg.L, Hkv=pcfg.Hkv, dh=pcfg.dh)
    pin = synthetic.make_prefix_pass_inputs(pcfg, 1)
    ein = synthetic.make_inputs(ecfg, 2)
    Kw, Vw = O.prefill(pcfg, pin["weights"], pin["emb"])
    want = O.denoise(ecfg, ein["weights"], Kw, Vw, ein["x0"][:pcfg.B], samples=range(pcfg.B), prefix_k_rotated=True)
    loop = ActionExpertLoop(ecfg, path=FR_PATH_TENSOR)
    loop.load_weights(ein["weights"])
    pp = _run_pass(pcfg, pin, expert=loop)
    x0 = torch.from_numpy(ein["x0"][:pcfg.B]).to("cuda").contiguous()
    got = loop.denoise(x0).cpu().numpy()
    assert loop.sync_status() == 0
    rel, cos = C.chunk_metrics(got, want)
    assert np.all(rel <= C.TOL_BF16_REL_L2) and np.all(cos >= C.TOL_BF16_COS), (rel, cos)
    # the expert's prefix slots hold the pass's rows bit for bit
    k_pass, v_pass = pp.read_kv(1, 1, pcfg.P)
    k_exp, v_exp = loop.read_kv(1, 1, pcfg.P)
    assert np.array_equal(k_pass, k_exp) and np.array_equal(v_pass, v_exp)
    pp.close()
    loop.close()


def test_prefix_pass_misuse():
    pcfg = SMALL["prefix_p75"]
    pin = synthetic.make_prefix_pass_inputs(pcfg, 0)
    pp = PrefixPass(pcfg)
    emb = torch.from_numpy(pin["emb"]).to("cuda").to(torch.bfloat16).contiguous()
    with pytest.raises(FrError) as ei:
        pp.run(emb)
    assert ei.value.code == FR_ERR_STATE                        # no weights yet
    pp.load_weights(pin["weights"])
    big = torch.zeros((1, pcfg.P + 1, pcfg.D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(FrError) as ei:
        pp.run(big)
    assert ei.value.code == FR_ERR_SHAPE                        # more tokens than the handle holds
    wrong = ActionExpertLoop(C.RAGGED["ragged_bf16"], path=FR_PATH_TENSOR)   # L, Hkv, dh differ
    with pytest.raises(FrError) as ei:
        pp.run(emb, wrong)
    assert ei.value.code == FR_ERR_SHAPE
    from flow_matching_action_loop_b200 import fr_denoise, fr_prefill
    with pytest.raises(FrError) as ei:
        fr_denoise(pp.h, emb.data_ptr(), emb.data_ptr(), 1)
    assert ei.value.code == FR_ERR_STATE                        # the pass handle runs no loop
    with pytest.raises(FrError) as ei:
        fr_prefill(wrong.h, emb.data_ptr(), 1, 10)
    assert ei.value.code == FR_ERR_STATE                        # an expert handle runs no pass
    wrong.close()
    pp.close()


@pytest.mark.slow
def test_prefix_pass_full_size_sampled():
    """The 2B-parameter backbone over 816 tokens: layer 0's K and V of every token (they depend on
    the token alone) against the oracle's single-layer pass; every layer finite and of unit scale."""
    cfg = synthetic.PREFIX_CONFIGS["vlm_bf16_p816"]
    inp = synthetic.make_prefix_pass_inputs(cfg, 0)
    pp = _run_pass(cfg, inp)
    one = cfg.replace(L=1)
    Kw, Vw = O.prefill(one, {"layers": inp["weights"]["layers"][:1]}, inp["emb"])
    k, v = pp.read_kv(0, 0, cfg.P)
    for what, got, want in (("K", _bf16_to_f64(k).transpose(1, 0, 2), Kw[0, 0]),
                            ("V", _bf16_to_f64(v).transpose(1, 0, 2), Vw[0, 0])):
        rel, cos = _kv_metrics(got, want)
        assert rel <= C.TOL_BF16_REL_L2 and cos >= C.TOL_BF16_COS, (what, rel, cos)
    for l in range(cfg.L):
        k, v = pp.read_kv(l, 0, cfg.P)
        kf, vf = _bf16_to_f64(k), _bf16_to_f64(v)
        assert np.all(np.isfinite(kf)) and np.all(np.isfinite(vf)), l
        assert 0.05 < np.sqrt(np.mean(vf ** 2)) < 20.0, l
    pp.close()
