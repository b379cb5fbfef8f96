"""C-ABI library on the host (no GPU): it loads, exports every declared symbol,
and its packer's number formats agree bit for bit with the oracle's own.
"""
import ctypes
import subprocess

import numpy as np
import pytest

from oracle import oracle as O


@pytest.fixture(scope="module")
def abi():
    from flow_matching_action_loop_b200 import _abi
    _abi.load_library()
    return _abi


def test_every_header_function_is_exported(abi):
    names = abi.header_functions()
    assert len(names) >= 17
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(abi.LIB_PATH)
    for n in names:
        assert getattr(lib, n) is not None
    # the binding declares every call's signature: no pointer or size goes through ctypes' default int
    bound = abi.load_library()
    assert [n for n in names if getattr(bound, n).argtypes is None] == []


def test_rope_tables_byte_identical_to_oracle(abi):
    for n_pos, dh, theta in ((866, 256, 1e4), (2148, 128, 1e4), (80, 64, 1e4), (7, 2, 500.0)):
        c, s = abi.fr_rope_tables(n_pos, dh, theta)
        oc, os_ = O.rope_tables(n_pos, dh, theta)
        assert c.tobytes() == oc.tobytes() and s.tobytes() == os_.tobytes()


def test_packer_bf16_matches_oracle_rounding(abi):
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(300000) / 32).astype(np.float32)
    bits = abi.fr_round_bf16(x)
    vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(vals, O.round_bf16(x.astype(np.float64)))


def test_packer_e4m3_matches_oracle_quantiser(abi):
    rng = np.random.default_rng(1)
    w = (rng.standard_normal(200000) / 32).astype(np.float32)
    s_w = float(np.max(np.abs(w.astype(np.float64)))) / 448.0
    codes = abi.fr_quantize_e4m3(w, s_w)
    decoded = np.array([O.decode_e4m3(int(c)) for c in range(256)])[codes]
    assert np.array_equal(decoded, O.round_e4m3(w.astype(np.float64) / s_w))
    # saturation, zero, and the NaN code
    special = np.array([1e9, -1e9, 0.0, -0.0, np.nan], np.float32)
    assert list(abi.fr_quantize_e4m3(special, 1.0)) == [0x7E, 0xFE, 0x00, 0x80, 0x7F]


def test_invalid_configs_rejected_before_any_device_work(abi):
    import synthetic
    base = synthetic.CONFIGS["tiny_f32"]
    bad = [
        (abi.make_config(base.replace(dh=63)), abi.FR_ERR_UNSUPPORTED),
        (abi.make_config(base.replace(Hq=3, Hkv=2)), abi.FR_ERR_UNSUPPORTED),
        (abi.make_config(base.replace(L=0)), abi.FR_ERR_ARG),
        (abi.make_config(base, path=7), abi.FR_ERR_ARG),
        (abi.make_config(base, path=abi.FR_PATH_TENSOR), abi.FR_ERR_UNSUPPORTED),   # f32 has no tensor path
    ]
    # empty inputs: no Euler step, no action row or feature, an empty prefix or batch, no width
    bad += [(abi.make_config(base.replace(**{f: 0})), abi.FR_ERR_ARG)
            for f in ("K", "H", "A", "P", "B", "D", "F", "Hq", "Hkv", "time_dim")]
    # constants that would give NaN tables: a negative eps, a non-positive or non-finite base
    bad += [(abi.make_config(base.replace(**{f: v})), abi.FR_ERR_ARG)
            for f, v in (("eps", -1e-6), ("eps", float("nan")), ("rope_theta", 0.0), ("rope_theta", float("inf")),
                         ("time_base", -10000.0))]
    for cfg, code in bad:
        with pytest.raises(abi.FrError) as ei:
            abi.fr_create(cfg, 0)
        assert ei.value.code == code, abi.fr_last_error()
    lib = abi.load_library()
    h = ctypes.c_void_p()
    assert lib.fr_create(None, 0, ctypes.byref(h)) == abi.FR_ERR_ARG
    assert lib.fr_denoise(None, None, None, 1, None) == abi.FR_ERR_ARG
    assert lib.fr_last_error() != b""
    lib.fr_destroy(None)   # no-op


def test_attention_op_sizes_and_validation(abi):
    # one key chunk needs no scratch; more chunks need [B][Hq][C][H][dh+4] floats
    assert abi.fr_attention_scratch_bytes(1, 2, 1, 60, 128) == 0
    assert abi.fr_attention_scratch_bytes(1, 8, 50, 866, 256) == 8 * 14 * 50 * (256 + 4) * 4
    assert abi.fr_attention_scratch_bytes(3, 16, 100, 2148, 128) == 3 * 16 * 12 * 100 * (128 + 4) * 4
    p = 1  # any non-NULL value: validation fails before any device access
    bad = [((None, p, p, p, 1, 8, 1, 50, 866, 256), abi.FR_ERR_ARG),
           ((p, p, p, p, 1, 8, 3, 50, 866, 256), abi.FR_ERR_UNSUPPORTED),   # Hq % Hkv
           ((p, p, p, p, 1, 8, 1, 50, 866, 96), abi.FR_ERR_UNSUPPORTED),    # dh
           ((p, p, p, p, 1, 8, 1, 129, 866, 256), abi.FR_ERR_UNSUPPORTED),  # H > 128
           ((p, p, p, p, 1, 8, 1, 50, 40, 256), abi.FR_ERR_UNSUPPORTED),    # H > S_keys
           ((p, p, p, p, 0, 8, 1, 50, 866, 256), abi.FR_ERR_ARG),
           ((p, p, p, p, 1, 8, 1, 50, 866, 256), abi.FR_ERR_SHAPE)]         # no scratch given
    lib = abi.load_library()
    for args, code in bad:
        assert lib.fr_attention(*args, None, 0, None) == code, (args, abi.fr_last_error())


def test_noalloc_attention_rejects_before_device_work(abi):
    lib = abi.load_library()
    p = 1
    # the π0.5 layer fits the built-in 8 MiB array; two samples of it do not
    assert abi.fr_attention_scratch_bytes(1, 8, 50, 866, 256) <= abi.FR_ATTENTION_NOALLOC_SCRATCH_BYTES
    assert lib.fr_attention_noalloc(p, p, p, p, 2, 8, 1, 50, 866, 256, None) == abi.FR_ERR_UNSUPPORTED
    assert b"scratch" in lib.fr_last_error()
    assert lib.fr_attention_noalloc(None, p, p, p, 1, 8, 1, 50, 866, 256, None) == abi.FR_ERR_ARG


def test_packer_w4_matches_oracle_quantiser(abi):
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((37, 300)) / 19).astype(np.float32)   # ragged last group (300 = 2 x 128 + 44)
    w[3, :128] = 0.0                                                 # an all-zero group
    w[4, 128:256] = 0.25                                             # a constant group
    q, sb = abi.fr_quantize_w4(w)
    oq, os_ = O.quantize_w4(w)
    assert np.array_equal(q, oq)
    sv = (sb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(sv, os_)
    assert abi.load_library().fr_quantize_w4(None, 1, 1, None, None) == abi.FR_ERR_ARG


def test_capsule_sizes_and_contract_calls_reject_before_device_work(abi):
    import synthetic
    cfg = synthetic.CONFIGS["pi05_bf16_b1"]
    fc = abi.make_config(cfg, B_max=4, P_max=cfg.P)
    # K then V [L][B][Hkv][P][dh] bf16, then x [B][H][A] float32, each part on a 256-byte boundary
    kv = cfg.L * 2 * cfg.Hkv * cfg.P * cfg.dh * 2
    up = lambda n: -(-n // 256) * 256   # noqa: E731
    assert abi.fr_capsule_bytes(fc, 2, cfg.P, False) == 2 * up(kv)
    assert abi.fr_capsule_bytes(fc, 2, cfg.P, True) == 2 * up(kv) + up(2 * cfg.H * cfg.A * 4)
    f32 = abi.make_config(synthetic.CONFIGS["tiny_f32"], B_max=3)
    t = synthetic.CONFIGS["tiny_f32"]
    assert abi.fr_capsule_bytes(f32, 3, t.P, False) == 2 * up(t.L * 3 * t.Hkv * t.P * t.dh * 4)
    for B, P in ((0, cfg.P), (5, cfg.P), (1, 0), (1, cfg.P + 1)):
        assert abi.fr_capsule_bytes(fc, B, P, True) == 0
    assert abi.fr_capsule_bytes(abi.make_config(cfg.replace(L=0)), 1, 1, False) == 0
    lib = abi.load_library()
    assert lib.fr_capsule_bytes(None, 1, 1, 0) == 0
    p = ctypes.c_void_p(1)
    sl = (ctypes.c_int * 1)(0)
    assert lib.fr_refresh_prefix_kv(None, p, p, sl, 1, 1, 0, None) == abi.FR_ERR_ARG
    out, n = ctypes.c_void_p(), ctypes.c_size_t()
    assert lib.fr_get_buffer(None, b"kv_k", ctypes.byref(out), ctypes.byref(n)) == abi.FR_ERR_ARG
    d = abi.FrCapsule()
    assert lib.fr_capsule_save(None, p, 1, 1, None, ctypes.byref(d), None) == abi.FR_ERR_ARG
    assert lib.fr_capsule_restore(None, p, ctypes.byref(d), None, 1, None, None) == abi.FR_ERR_ARG
    assert lib.fr_set_graph_capacity(None, 1) == abi.FR_ERR_ARG
    assert lib.fr_graph_count(None) == abi.FR_ERR_ARG
    assert lib.fr_selftest_wait(None, 1000000, None) == abi.FR_ERR_ARG
    assert lib.fr_prefill(None, p, 1, 1, None, None) == abi.FR_ERR_ARG


def test_plain_c_client_of_the_header(abi, tmp_path):
    """A C program built against include/fr.h alone links the library and uses its host calls."""
    import os
    src = os.path.join(os.path.dirname(__file__), "c", "abi_host.c")
    exe = str(tmp_path / "abi_host")
    lib_dir = os.path.dirname(abi.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.dirname(abi.HEADER), src, "-o", exe,
                    "-L", lib_dir, "-lflowloop", "-lm", f"-Wl,-rpath,{lib_dir}"], check=True)
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stderr
