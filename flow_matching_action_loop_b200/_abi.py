"""ctypes binding of include/fr.h: argument marshalling only.

Every function here has the name of the C entry point it calls and raises
FrError when the call returns a negative code.  Nothing of the method runs in
Python: the loop, its kernels and the weight packer live in libflowloop.so.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
# FR_LIBRARY selects another build of the library (e.g. the checked build, libflowloop_checked.so)
LIB_PATH = os.environ.get("FR_LIBRARY") or os.path.join(PKG, "libflowloop.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "fr.h")

FR_OK = 0
FR_ERR_ARG, FR_ERR_SHAPE, FR_ERR_STATE, FR_ERR_CUDA, FR_ERR_TIMEOUT, FR_ERR_DEVICE, FR_ERR_UNSUPPORTED = range(-1, -8, -1)
FR_DTYPE_F32, FR_DTYPE_BF16, FR_DTYPE_FP8, FR_DTYPE_W4A16 = 0, 1, 2, 3
FR_W4_GROUP = 128
FR_PATH_AUTO, FR_PATH_STEPWISE, FR_PATH_TENSOR = 0, 1, 2
FR_EXEC_AUTO, FR_EXEC_GRAPH, FR_EXEC_PERSISTENT = 0, 1, 2
FR_PREFIX_K_ROTATED = 1
FR_ROLE_EXPERT, FR_ROLE_PREFIX = 0, 1
DTYPES = {"f32": FR_DTYPE_F32, "bf16": FR_DTYPE_BF16, "fp8": FR_DTYPE_FP8, "w4a16": FR_DTYPE_W4A16}
ERR_NAMES = {FR_ERR_ARG: "FR_ERR_ARG", FR_ERR_SHAPE: "FR_ERR_SHAPE", FR_ERR_STATE: "FR_ERR_STATE",
             FR_ERR_CUDA: "FR_ERR_CUDA", FR_ERR_TIMEOUT: "FR_ERR_TIMEOUT", FR_ERR_DEVICE: "FR_ERR_DEVICE",
             FR_ERR_UNSUPPORTED: "FR_ERR_UNSUPPORTED"}


class FrError(RuntimeError):
    def __init__(self, code: int, func: str, msg: str):
        super().__init__(f"{func} -> {ERR_NAMES.get(code, code)}: {msg}")
        self.code = code


class FrConfig(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int), ("D", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("dh", ctypes.c_int), ("F", ctypes.c_int), ("H", ctypes.c_int), ("A", ctypes.c_int),
                ("B_max", ctypes.c_int), ("P_max", ctypes.c_int), ("K", ctypes.c_int),
                ("dtype", ctypes.c_int), ("path", ctypes.c_int), ("rope_theta", ctypes.c_float),
                ("eps", ctypes.c_float), ("time_dim", ctypes.c_int), ("time_base", ctypes.c_float),
                ("adarms", ctypes.c_int), ("role", ctypes.c_int)]


_FP = ctypes.POINTER(ctypes.c_float)


LAYER_TENSORS = ("wq", "wk", "wv", "wo", "wg", "wu", "wd", "g1", "g2", "w_mod1", "b_mod1", "w_mod2", "b_mod2")
MODEL_TENSORS = ("w_in", "b_in", "w_out", "b_out", "w_t1", "b_t1", "w_t2", "b_t2", "g_f", "w_modf", "b_modf")


class FrLayerWeights(ctypes.Structure):
    _fields_ = [(n, _FP) for n in LAYER_TENSORS]


class FrWeights(ctypes.Structure):
    _fields_ = [("layers", ctypes.POINTER(FrLayerWeights))] + [(n, _FP) for n in MODEL_TENSORS]


FR_CAPSULE_MAGIC = 0x46524350


class FrCapsule(ctypes.Structure):
    _fields_ = [("magic", ctypes.c_uint32), ("L", ctypes.c_int), ("Hkv", ctypes.c_int), ("dh", ctypes.c_int),
                ("kv_bytes_per_elem", ctypes.c_int), ("H", ctypes.c_int), ("A", ctypes.c_int),
                ("B", ctypes.c_int), ("P", ctypes.c_int), ("has_x", ctypes.c_int), ("bytes", ctypes.c_size_t)]


_lib: Optional[ctypes.CDLL] = None


def header_functions():
    """Names of the functions include/fr.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fr_[a-z0-9_]+)\s*\(", text)))


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libflowloop.so; raise if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python flow_matching_action_loop_b200/build.py`")
    lib = ctypes.CDLL(path)
    c_int, c_void_p, c_uint, c_char_p = ctypes.c_int, ctypes.c_void_p, ctypes.c_uint, ctypes.c_char_p
    H = c_void_p
    sig = {
        "fr_create": (c_int, [ctypes.POINTER(FrConfig), c_int, ctypes.POINTER(c_void_p)]),
        "fr_load_weights": (c_int, [H, ctypes.POINTER(FrWeights), c_void_p]),
        "fr_set_prefix_kv": (c_int, [H, c_void_p, c_void_p, c_int, c_int, c_uint, c_void_p]),
        "fr_calibrate": (c_int, [H, c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p]),
        "fr_denoise": (c_int, [H, c_void_p, c_void_p, c_int, c_void_p]),
        "fr_get_scales": (c_int, [H, _FP, _FP, c_int]),
        "fr_set_scales": (c_int, [H, _FP, c_int]),
        "fr_sync_status": (c_int, [H, c_void_p]),
        "fr_selftest_wait": (c_int, [H, ctypes.c_uint64, c_void_p]),
        "fr_last_error": (c_char_p, []),
        "fr_destroy": (None, [H]),
        "fr_read_kv": (c_int, [H, c_int, c_int, c_void_p, c_void_p, c_int]),
        "fr_get_rope_tables": (c_int, [H, _FP, _FP, c_int]),
        "fr_path_name": (c_char_p, [H]),
        "fr_launches_per_call": (c_int, [H, c_int]),
        "fr_set_exec_mode": (c_int, [H, c_int]),
        "fr_exec_mode": (c_int, [H, c_int]),
        "fr_set_wait_limit": (c_int, [H, ctypes.c_uint64]),
        "fr_device_checks": (c_int, []),
        "fr_debug_limit_extent": (c_int, [H, c_char_p, ctypes.c_uint64]),
        "fr_debug_plan": (c_int, [ctypes.POINTER(FrConfig), c_int, c_int, c_int, c_int, c_int, ctypes.POINTER(c_int), c_int]),
        "fr_rope_tables": (c_int, [c_int, c_int, ctypes.c_double, _FP, _FP]),
        "fr_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                 c_void_p, ctypes.c_size_t, c_void_p]),
        "fr_attention_scratch_bytes": (ctypes.c_size_t, [c_int, c_int, c_int, c_int, c_int]),
        "fr_ops_sync_status": (c_int, [c_void_p]),
        "fr_attention_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                         c_int, c_void_p]),
        "fr_prefill": (c_int, [H, c_void_p, c_int, c_int, H, c_void_p]),
        "fr_refresh_prefix_kv": (c_int, [H, c_void_p, c_void_p, ctypes.POINTER(c_int), c_int, c_int, c_uint,
                                         c_void_p]),
        "fr_get_buffer": (c_int, [H, c_char_p, ctypes.POINTER(c_void_p), ctypes.POINTER(ctypes.c_size_t)]),
        "fr_capsule_bytes": (ctypes.c_size_t, [ctypes.POINTER(FrConfig), c_int, c_int, c_int]),
        "fr_capsule_save": (c_int, [H, c_void_p, ctypes.c_size_t, c_int, c_void_p, ctypes.POINTER(FrCapsule),
                                    c_void_p]),
        "fr_capsule_restore": (c_int, [H, c_void_p, ctypes.POINTER(FrCapsule), ctypes.POINTER(c_int), c_int,
                                       c_void_p, c_void_p]),
        "fr_set_graph_capacity": (c_int, [H, c_int]),
        "fr_graph_count": (c_int, [H]),
        "fr_round_bf16": (None, [_FP, ctypes.POINTER(ctypes.c_uint16), ctypes.c_size_t]),
        "fr_quantize_e4m3": (None, [_FP, ctypes.POINTER(ctypes.c_uint8), ctypes.c_size_t, ctypes.c_double]),
        "fr_quantize_w4": (c_int, [_FP, c_int, c_int, ctypes.POINTER(ctypes.c_int8), ctypes.POINTER(ctypes.c_uint16)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(rc: int, func: str) -> int:
    if rc < 0:
        raise FrError(rc, func, load_library().fr_last_error().decode())
    return rc


def _fptr(a: np.ndarray):
    return a.ctypes.data_as(_FP)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def make_config(cfg, B_max: Optional[int] = None, P_max: Optional[int] = None, path: int = FR_PATH_AUTO) -> FrConfig:
    """fr_config from any object with the action-expert size attributes."""
    dtype = cfg.dtype if isinstance(cfg.dtype, int) else DTYPES[cfg.dtype]
    return FrConfig(L=cfg.L, D=cfg.D, Hq=cfg.Hq, Hkv=cfg.Hkv, dh=cfg.dh, F=cfg.F, H=cfg.H, A=cfg.A,
                    B_max=B_max or cfg.B, P_max=P_max or cfg.P, K=cfg.K, dtype=dtype, path=path,
                    rope_theta=cfg.rope_theta, eps=cfg.eps, time_dim=cfg.time_dim, time_base=cfg.time_base,
                    adarms=1 if getattr(cfg, "adarms", False) else 0)


def make_prefix_config(cfg, B_max: Optional[int] = None, P_max: Optional[int] = None) -> FrConfig:
    """fr_config of a prefix-pass (backbone) handle from a PrefixConfig-like object: H is the
    largest number of prefix tokens per sample; the loop-only fields get neutral values."""
    dtype = cfg.dtype if isinstance(cfg.dtype, int) else DTYPES[cfg.dtype]
    return FrConfig(L=cfg.L, D=cfg.D, Hq=cfg.Hq, Hkv=cfg.Hkv, dh=cfg.dh, F=cfg.F, H=P_max or cfg.P, A=1,
                    B_max=B_max or cfg.B, P_max=1, K=1, dtype=dtype, path=FR_PATH_TENSOR,
                    rope_theta=cfg.rope_theta, eps=cfg.eps, time_dim=2, time_base=10000.0, adarms=0,
                    role=FR_ROLE_PREFIX)


# ------------------------------------------------------------------ same-name wrappers

def fr_create(cfg: FrConfig, device: int = 0) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(load_library().fr_create(ctypes.byref(cfg), device, ctypes.byref(h)), "fr_create")
    return h


def fr_load_weights(h, weights: dict, stream: int = 0) -> None:
    """weights: the dict layout of host float32 arrays ({'layers': [...], 'w_in': ..., ...}); a tensor
    the dict does not hold (the adaRMS ones of a plain model) is passed as NULL."""
    keep = []

    def p(a):
        if a is None:
            return _FP()
        a = _f32(a)
        keep.append(a)
        return _fptr(a)

    layers = (FrLayerWeights * len(weights["layers"]))()
    for i, lw in enumerate(weights["layers"]):
        for n in LAYER_TENSORS:
            setattr(layers[i], n, p(lw.get(n)))
    w = FrWeights(layers=layers, **{n: p(weights.get(n)) for n in MODEL_TENSORS})
    _check(load_library().fr_load_weights(h, ctypes.byref(w), stream), "fr_load_weights")


def fr_set_prefix_kv(h, k_dev: int, v_dev: int, B: int, P: int, flags: int = 0, stream: int = 0) -> None:
    _check(load_library().fr_set_prefix_kv(h, k_dev, v_dev, B, P, flags, stream), "fr_set_prefix_kv")


def fr_calibrate(h, x0_dev: int, pk_dev: int, pv_dev: int, B: int, P: int, stream: int = 0) -> None:
    _check(load_library().fr_calibrate(h, x0_dev, pk_dev, pv_dev, B, P, stream), "fr_calibrate")


def fr_denoise(h, x0_dev: int, x_out_dev: int, B: int, stream: int = 0) -> None:
    _check(load_library().fr_denoise(h, x0_dev, x_out_dev, B, stream), "fr_denoise")


def fr_get_scales(h, n: int):
    sa = np.zeros(n, np.float32)
    sw = np.zeros(n, np.float32)
    _check(load_library().fr_get_scales(h, _fptr(sa), _fptr(sw), n), "fr_get_scales")
    return sa, sw


def fr_set_scales(h, s_act) -> None:
    s = _f32(s_act).ravel()
    _check(load_library().fr_set_scales(h, _fptr(s), s.size), "fr_set_scales")


def fr_sync_status(h, stream: int = 0) -> int:
    return _check(load_library().fr_sync_status(h, stream), "fr_sync_status")


def fr_selftest_wait(h, limit_ns: int, stream: int = 0) -> None:
    _check(load_library().fr_selftest_wait(h, limit_ns, stream), "fr_selftest_wait")


def fr_last_error() -> str:
    return load_library().fr_last_error().decode()


def fr_destroy(h) -> None:
    if h:
        load_library().fr_destroy(h)


def fr_read_kv(h, layer: int, b: int, n_slots: int, Hkv: int, dh: int, bf16: bool):
    dt = np.uint16 if bf16 else np.float32
    k = np.zeros((Hkv, n_slots, dh), dt)
    v = np.zeros((Hkv, n_slots, dh), dt)
    _check(load_library().fr_read_kv(h, layer, b, k.ctypes.data, v.ctypes.data, n_slots), "fr_read_kv")
    return k, v


def fr_get_rope_tables(h, n_pos: int, dh: int):
    c = np.zeros((n_pos, dh // 2), np.float32)
    s = np.zeros((n_pos, dh // 2), np.float32)
    _check(load_library().fr_get_rope_tables(h, _fptr(c), _fptr(s), n_pos), "fr_get_rope_tables")
    return c, s


def fr_path_name(h) -> str:
    return load_library().fr_path_name(h).decode()


def fr_launches_per_call(h, B: int) -> int:
    return load_library().fr_launches_per_call(h, B)


def _ints(values):
    a = (ctypes.c_int * len(values))(*[int(v) for v in values])
    return a


def fr_prefill(h, emb_dev: int, B: int, P: int, expert=None, stream: int = 0) -> None:
    _check(load_library().fr_prefill(h, emb_dev, B, P, expert, stream), "fr_prefill")


def fr_refresh_prefix_kv(h, k_dev: int, v_dev: int, slots, P: int, flags: int = 0, stream: int = 0) -> None:
    sl = _ints(slots)
    _check(load_library().fr_refresh_prefix_kv(h, k_dev, v_dev, sl, len(sl), P, flags, stream),
           "fr_refresh_prefix_kv")


def fr_get_buffer(h, name: str):
    """(device address, bytes) of a named buffer of the handle."""
    p = ctypes.c_void_p()
    n = ctypes.c_size_t()
    _check(load_library().fr_get_buffer(h, name.encode(), ctypes.byref(p), ctypes.byref(n)), "fr_get_buffer")
    return p.value or 0, n.value


def fr_capsule_bytes(cfg: FrConfig, B: int, P: int, with_x: bool) -> int:
    return load_library().fr_capsule_bytes(ctypes.byref(cfg), B, P, 1 if with_x else 0)


def fr_capsule_save(h, cap_dev: int, cap_bytes: int, B: int, x_dev: int = 0, stream: int = 0) -> FrCapsule:
    d = FrCapsule()
    _check(load_library().fr_capsule_save(h, cap_dev, cap_bytes, B, x_dev or None, ctypes.byref(d), stream),
           "fr_capsule_save")
    return d


def fr_capsule_restore(h, cap_dev: int, desc: FrCapsule, B: int, sample_map=None, x_dev: int = 0,
                       stream: int = 0) -> None:
    m = _ints(sample_map) if sample_map is not None else None
    _check(load_library().fr_capsule_restore(h, cap_dev, ctypes.byref(desc), m, B, x_dev or None, stream),
           "fr_capsule_restore")


def fr_set_exec_mode(h, mode: int) -> None:
    _check(load_library().fr_set_exec_mode(h, mode), "fr_set_exec_mode")


def fr_exec_mode(h, B: int) -> int:
    return _check(load_library().fr_exec_mode(h, B), "fr_exec_mode")


def fr_device_checks() -> bool:
    return load_library().fr_device_checks() == 1


PLAN_GEMMS = ("qkv", "o", "gate_up", "down")
PLAN_GEMM_FIELDS = ("S", "stages", "red_tok", "persist", "kpu", "smem", "tiles", "NKC")


def fr_debug_plan(cfg, B: int, P: int, nsm: int, max_dyn: int, max_dyn2: int) -> dict:
    """The tensor-core path's launch plan of one call, computed on the host (no device)."""
    out = (ctypes.c_int * 64)()
    n = _check(load_library().fr_debug_plan(ctypes.byref(cfg), B, P, nsm, max_dyn, max_dyn2, out, 64), "fr_debug_plan")
    v = list(out[:n])
    plan = {"NT": v[0], "Nt": v[1]}
    for i, name in enumerate(PLAN_GEMMS):
        plan[name] = dict(zip(PLAN_GEMM_FIELDS, v[2 + 8 * i: 10 + 8 * i]))
    plan["attn_umma"], plan["attn_C"], plan["attn_KC"] = v[34:37]
    return plan


def fr_debug_limit_extent(h, buffer: str, elems: int) -> None:
    _check(load_library().fr_debug_limit_extent(h, buffer.encode(), elems), "fr_debug_limit_extent")


def fr_set_wait_limit(h, limit_ns: int) -> None:
    _check(load_library().fr_set_wait_limit(h, limit_ns), "fr_set_wait_limit")


def fr_set_graph_capacity(h, capacity: int) -> None:
    _check(load_library().fr_set_graph_capacity(h, capacity), "fr_set_graph_capacity")


def fr_graph_count(h) -> int:
    return _check(load_library().fr_graph_count(h), "fr_graph_count")


def fr_attention(q: int, k: int, v: int, o: int, B: int, Hq: int, Hkv: int, H: int, S_keys: int, dh: int,
                 scratch: int = 0, scratch_bytes: int = 0, stream: int = 0) -> None:
    _check(load_library().fr_attention(q, k, v, o, B, Hq, Hkv, H, S_keys, dh, scratch, scratch_bytes, stream),
           "fr_attention")


def fr_ops_sync_status(stream: int = 0) -> int:
    return _check(load_library().fr_ops_sync_status(stream), "fr_ops_sync_status")


def fr_attention_scratch_bytes(B: int, Hq: int, H: int, S_keys: int, dh: int) -> int:
    return load_library().fr_attention_scratch_bytes(B, Hq, H, S_keys, dh)


FR_ATTENTION_NOALLOC_SCRATCH_BYTES = 8 << 20


def fr_attention_noalloc(q: int, k: int, v: int, o: int, B: int, Hq: int, Hkv: int, H: int, S_keys: int, dh: int,
                         stream: int = 0) -> None:
    _check(load_library().fr_attention_noalloc(q, k, v, o, B, Hq, Hkv, H, S_keys, dh, stream),
           "fr_attention_noalloc")


def fr_rope_tables(n_pos: int, dh: int, theta: float):
    c = np.zeros((n_pos, dh // 2), np.float32)
    s = np.zeros((n_pos, dh // 2), np.float32)
    _check(load_library().fr_rope_tables(n_pos, dh, theta, _fptr(c), _fptr(s)), "fr_rope_tables")
    return c, s


def fr_round_bf16(x) -> np.ndarray:
    x = _f32(x)
    out = np.zeros(x.shape, np.uint16)
    load_library().fr_round_bf16(_fptr(x), out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)), x.size)
    return out


def fr_quantize_e4m3(x, scale: float) -> np.ndarray:
    x = _f32(x)
    out = np.zeros(x.shape, np.uint8)
    load_library().fr_quantize_e4m3(_fptr(x), out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), x.size, scale)
    return out


def fr_quantize_w4(w):
    """4-bit codes [rows][cols] (int8) and bf16 scale bits [rows][groups] (uint16) of a 2-D weight."""
    w = np.ascontiguousarray(np.asarray(w, np.float32))
    rows, cols = w.shape
    q = np.zeros((rows, cols), np.int8)
    sb = np.zeros((rows, -(-cols // FR_W4_GROUP)), np.uint16)
    _check(load_library().fr_quantize_w4(_fptr(w), rows, cols, q.ctypes.data_as(ctypes.POINTER(ctypes.c_int8)),
                                          sb.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16))), "fr_quantize_w4")
    return q, sb
