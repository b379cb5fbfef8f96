"""B200 flow-matching action-expert denoising loop.

The compute path is libflowloop.so (CUDA kernels for sm_100a behind the C ABI
in include/fr.h).  This package only marshals arguments: PyTorch supplies
device memory and the current CUDA stream.  Importing it loads the library and
fails loudly if it has not been built; there is no CPU fallback.

    loop = ActionExpertLoop(cfg)            # fr_create
    loop.load_weights(weights)              # fr_load_weights (host float32 arrays)
    loop.set_prefix_kv(k, v)                # fr_set_prefix_kv (device tensors)
    x_t0 = loop.denoise(x_t1)               # fr_denoise
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from ._abi import (  # noqa: F401
    DTYPES, FR_DTYPE_BF16, FR_DTYPE_F32, FR_DTYPE_FP8, FR_DTYPE_W4A16, FR_ERR_ARG, FR_ERR_CUDA, FR_ERR_DEVICE, FR_ERR_SHAPE,
    FR_ERR_STATE, FR_ERR_TIMEOUT, FR_ERR_UNSUPPORTED, FR_OK, FR_PATH_AUTO, FR_PATH_STEPWISE, FR_PATH_TENSOR,
    FR_EXEC_AUTO, FR_EXEC_GRAPH, FR_EXEC_PERSISTENT, fr_set_exec_mode, fr_exec_mode, fr_set_wait_limit,
    fr_device_checks, fr_debug_limit_extent,
    FR_ATTENTION_NOALLOC_SCRATCH_BYTES, FR_CAPSULE_MAGIC, FR_PREFIX_K_ROTATED, FrCapsule, FrConfig, FrError,
    fr_attention, fr_attention_noalloc, fr_attention_scratch_bytes, fr_ops_sync_status, fr_calibrate, fr_capsule_bytes,
    fr_capsule_restore, fr_capsule_save, fr_create, fr_denoise, fr_destroy, fr_get_buffer, fr_get_rope_tables,
    fr_get_scales, fr_graph_count, fr_last_error, fr_launches_per_call, fr_load_weights, fr_path_name,
    fr_quantize_e4m3, fr_quantize_w4, fr_read_kv, fr_refresh_prefix_kv, fr_rope_tables, fr_round_bf16,
    fr_set_graph_capacity, fr_set_prefix_kv, fr_set_scales, fr_sync_status, header_functions, load_library,
    make_config, make_prefix_config, fr_prefill, fr_selftest_wait, FR_ROLE_EXPERT, FR_ROLE_PREFIX,
)

load_library()

__all__ = ["ActionExpertLoop", "FrError", "PrefixPass", "load_library", "make_config"]


class ActionExpertLoop:
    """One fr_handle on one GPU.  Device tensors are torch tensors; host weights are numpy arrays."""

    def __init__(self, cfg, device: int = 0, B_max: Optional[int] = None, P_max: Optional[int] = None,
                 path: int = FR_PATH_AUTO):
        import torch
        self._torch = torch
        self.cfg = cfg
        self.device = device
        self.B_max = B_max or cfg.B
        self.P_max = P_max or cfg.P
        self.kv_dtype = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
        self.h = fr_create(make_config(cfg, self.B_max, self.P_max, path), device)

    # -- plumbing
    def _stream(self) -> int:
        return self._torch.cuda.current_stream(self.device).cuda_stream

    def _dev(self, t, dtype, shape, name):
        torch = self._torch
        if not isinstance(t, torch.Tensor) or t.device.type != "cuda" or t.dtype != dtype or not t.is_contiguous():
            raise FrError(FR_ERR_ARG, name, f"expected a contiguous {dtype} CUDA tensor")
        if t.device.index != self.device:   # the kernels run on the handle's device
            raise FrError(FR_ERR_ARG, name, f"expected a tensor on cuda:{self.device}, got {t.device}")
        if tuple(t.shape) != tuple(shape):
            raise FrError(FR_ERR_SHAPE, name, f"expected shape {tuple(shape)}, got {tuple(t.shape)}")
        return t.data_ptr()

    # -- the C ABI
    @property
    def path(self) -> str:
        return fr_path_name(self.h)

    def launches_per_call(self, B: Optional[int] = None) -> int:
        return fr_launches_per_call(self.h, B or self.B_max)

    def load_weights(self, weights: dict) -> None:
        fr_load_weights(self.h, weights, self._stream())

    def set_prefix_kv(self, k, v, rotated: bool = False) -> None:
        c = self.cfg
        L, B, P = k.shape[0], k.shape[1], k.shape[2]
        shape = (L, B, P, c.Hkv, c.dh)
        pk = self._dev(k, self.kv_dtype, shape, "fr_set_prefix_kv")
        pv = self._dev(v, self.kv_dtype, shape, "fr_set_prefix_kv")
        fr_set_prefix_kv(self.h, pk, pv, B, P, FR_PREFIX_K_ROTATED if rotated else 0, self._stream())
        self._P = P

    def calibrate(self, x0, k, v) -> None:
        c = self.cfg
        L, B, P = k.shape[0], k.shape[1], k.shape[2]
        shape = (L, B, P, c.Hkv, c.dh)
        fr_calibrate(self.h, self._dev(x0, self._torch.float32, (B, c.H, c.A), "fr_calibrate"),
                     self._dev(k, self.kv_dtype, shape, "fr_calibrate"),
                     self._dev(v, self.kv_dtype, shape, "fr_calibrate"), B, P, self._stream())
        self._P = P   # the calibration prefix is now the cached one

    def denoise(self, x0, out=None):
        c = self.cfg
        B = x0.shape[0]
        px = self._dev(x0, self._torch.float32, (B, c.H, c.A), "fr_denoise")
        if out is None:
            out = self._torch.empty_like(x0)
        po = self._dev(out, self._torch.float32, (B, c.H, c.A), "fr_denoise")
        fr_denoise(self.h, px, po, B, self._stream())
        return out

    # -- execution contract across chunks
    def refresh_prefix_kv(self, k, v, slots, rotated: bool = False) -> None:
        """Replace the prefix of batch slots `slots` (k, v: [L][len(slots)][P][Hkv][dh])."""
        c = self.cfg
        L, n, P = k.shape[0], k.shape[1], k.shape[2]
        shape = (L, n, P, c.Hkv, c.dh)
        fr_refresh_prefix_kv(self.h, self._dev(k, self.kv_dtype, shape, "fr_refresh_prefix_kv"),
                             self._dev(v, self.kv_dtype, shape, "fr_refresh_prefix_kv"), list(slots), P,
                             FR_PREFIX_K_ROTATED if rotated else 0, self._stream())

    def buffer(self, name: str):
        """(device address, bytes) of the handle's named buffer `name`."""
        return fr_get_buffer(self.h, name)

    def save_capsule(self, B: int, x=None):
        """Snapshot slots 0..B-1 (and x [B][H][A] if given) into a new device buffer: (buffer, description)."""
        torch = self._torch
        c = self.cfg
        n = fr_capsule_bytes(make_config(c, self.B_max, self.P_max), B, self._prefix_P(), x is not None)
        if n == 0:
            raise FrError(FR_ERR_SHAPE, "fr_capsule_bytes", f"no capsule size for B={B}")
        buf = torch.empty(n, dtype=torch.uint8, device=f"cuda:{self.device}")
        px = self._dev(x, torch.float32, (B, c.H, c.A), "fr_capsule_save") if x is not None else 0
        desc = fr_capsule_save(self.h, buf.data_ptr(), n, B, px, self._stream())
        return buf, desc

    def restore_capsule(self, capsule, B: Optional[int] = None, sample_map=None, x_out=None) -> None:
        """Make (buffer, description) the prefix state; sample_map forks or reorders its samples."""
        buf, desc = capsule
        c = self.cfg
        B = B or (len(sample_map) if sample_map is not None else desc.B)
        px = self._dev(x_out, self._torch.float32, (B, c.H, c.A), "fr_capsule_restore") if x_out is not None else 0
        fr_capsule_restore(self.h, buf.data_ptr(), desc, B, sample_map, px, self._stream())
        self._P = desc.P

    def set_graph_capacity(self, capacity: int) -> None:
        fr_set_graph_capacity(self.h, capacity)

    def set_exec_mode(self, mode: int) -> None:
        """FR_EXEC_AUTO, FR_EXEC_GRAPH or FR_EXEC_PERSISTENT (tensor-path expert handles)."""
        fr_set_exec_mode(self.h, mode)

    def exec_mode(self, B: Optional[int] = None) -> int:
        """FR_EXEC_PERSISTENT or FR_EXEC_GRAPH: what a call of batch B runs."""
        return fr_exec_mode(self.h, B or self.B_max)

    def limit_extent(self, buffer: str, elems: int) -> None:
        """Checked builds: declare a smaller extent for one of the handle's buffers (0: the real one)."""
        fr_debug_limit_extent(self.h, buffer, elems)

    def set_wait_limit(self, limit_ns: int) -> None:
        """Bound of the persistent kernel's waits on other CTAs (0: the default)."""
        fr_set_wait_limit(self.h, limit_ns)

    def graph_count(self) -> int:
        return fr_graph_count(self.h)

    def _prefix_P(self) -> int:
        P = getattr(self, "_P", None)
        if P is None:
            raise FrError(FR_ERR_STATE, "fr_capsule_save", "no prefix set")
        return P

    def get_scales(self):
        sa, sw = fr_get_scales(self.h, self.cfg.L * 4)
        return sa.reshape(self.cfg.L, 4), sw.reshape(self.cfg.L, 4)

    def set_scales(self, s_act) -> None:
        fr_set_scales(self.h, np.asarray(s_act, np.float32).reshape(-1))

    def sync_status(self) -> int:
        return fr_sync_status(self.h, self._stream())

    def read_kv(self, layer: int, b: int, n_slots: int):
        return fr_read_kv(self.h, layer, b, n_slots, self.cfg.Hkv, self.cfg.dh, self.cfg.dtype != "f32")

    def rope_tables(self, n_pos: int):
        return fr_get_rope_tables(self.h, n_pos, self.cfg.dh)

    def close(self) -> None:
        if self.h:
            fr_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class PrefixPass:
    """One prefix-pass (backbone) handle: the step before the loop, producing the expert's prefix KV."""

    def __init__(self, cfg, device: int = 0, B_max: Optional[int] = None, P_max: Optional[int] = None):
        import torch
        self._torch = torch
        self.cfg = cfg
        self.device = device
        self.h = fr_create(make_prefix_config(cfg, B_max, P_max), device)

    def _stream(self) -> int:
        return self._torch.cuda.current_stream(self.device).cuda_stream

    def load_weights(self, weights: dict) -> None:
        """weights: {'layers': [...]} with the layer tensors of the backbone (host float32)."""
        fr_load_weights(self.h, weights, self._stream())

    def run(self, emb, expert: Optional["ActionExpertLoop"] = None) -> None:
        """emb: bf16 CUDA tensor [B][P][D].  Fills this handle's KV cache and, if given, the expert's prefix."""
        torch = self._torch
        if not isinstance(emb, torch.Tensor) or emb.device.type != "cuda" or emb.dtype != torch.bfloat16 \
                or not emb.is_contiguous() or emb.dim() != 3 or emb.shape[2] != self.cfg.D:
            raise FrError(FR_ERR_ARG, "fr_prefill", "expected a contiguous bf16 CUDA tensor [B][P][D]")
        if emb.device.index != self.device:
            raise FrError(FR_ERR_ARG, "fr_prefill", f"expected a tensor on cuda:{self.device}, got {emb.device}")
        B, P = emb.shape[0], emb.shape[1]
        fr_prefill(self.h, emb.data_ptr(), B, P, expert.h if expert is not None else None, self._stream())
        if expert is not None:
            expert._P = P

    def buffer(self, name: str):
        return fr_get_buffer(self.h, name)

    def read_kv(self, layer: int, b: int, n_slots: int):
        return fr_read_kv(self.h, layer, b, n_slots, self.cfg.Hkv, self.cfg.dh, True)

    def sync_status(self) -> int:
        return fr_sync_status(self.h, self._stream())

    def launches_per_call(self) -> int:
        return fr_launches_per_call(self.h, 1)

    def close(self) -> None:
        if self.h:
            fr_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
