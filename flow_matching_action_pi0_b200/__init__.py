"""Python binding of libpae.so, the C ABI in include/pae.h.

Argument marshalling only: every step of the denoise loop runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory and streams.  If the
library has not been built this module raises on first use; there is no
fallback path.

Functions keep the C names (pae_create, pae_set_prefix, pae_set_prefix_hidden,
pae_precompute_tables,
pae_denoise, pae_denoise_host, pae_denoise_steps, pae_sync, ...).  The
ActionExpert class wraps a context for convenience.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpae.so")

PAE_OK, PAE_ERR_ARG, PAE_ERR_STATE, PAE_ERR_CUDA, PAE_ERR_OOM, PAE_ERR_TIMEOUT, PAE_ERR_UNSUPPORTED = range(7)
PAE_FP32, PAE_BF16, PAE_W4A16 = 0, 1, 2
PAE_OPT_USE_GRAPH, PAE_OPT_WAIT_LIMIT_US, PAE_OPT_PROFILE, PAE_OPT_PDL, PAE_OPT_MAX_SPLITK = 1, 2, 3, 4, 5
PAE_OPT_PERSISTENT = 6
PAE_OPT_FUSED_NORM = 7
PAE_OPT_DATAFLOW, PAE_OPT_DATAFLOW_CLUSTER = 8, 9
PAE_OPT_FACTORED_NORM = 10
(PAE_K_TRANSITION, PAE_K_QKV, PAE_K_ATTENTION, PAE_K_OPROJ, PAE_K_NORM, PAE_K_GATEUP,
 PAE_K_DOWN, PAE_K_PERSISTENT, PAE_K_DATAFLOW) = range(9)
KERNEL_CLASSES = ("transition", "qkv", "attention", "o_proj", "norm", "gate_up", "down", "persistent", "dataflow")
PAE_Q_GRAPH_KERNELS, PAE_Q_SPLITS, PAE_Q_TOKEN_TILE, PAE_Q_ATTN_SPLITS, PAE_Q_PERSISTENT, PAE_Q_FUSED_NORM = 1, 2, 3, 4, 5, 6
PAE_Q_DATAFLOW = 7
PAE_Q_ATTN_CHUNK = 8
STATUS_NAMES = {0: "PAE_OK", 1: "PAE_ERR_ARG", 2: "PAE_ERR_STATE", 3: "PAE_ERR_CUDA", 4: "PAE_ERR_OOM",
                5: "PAE_ERR_TIMEOUT", 6: "PAE_ERR_UNSUPPORTED"}

# Every symbol include/pae.h declares.
EXPORTS = ("pae_create", "pae_set_prefix", "pae_set_prefix_hidden", "pae_precompute_tables", "pae_denoise", "pae_denoise_host",
           "pae_denoise_steps", "pae_set_option", "pae_profile_read", "pae_query", "pae_plan_query", "pae_sync",
           "pae_clear_error", "pae_last_error", "pae_debug_copy", "pae_precompute_tables_static",
           "pae_destroy")


class PaeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class pae_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "layers", "width", "n_q_heads", "n_kv_heads", "head_dim", "mlp_dim", "action_dim", "chunk",
        "max_batch", "max_prefix", "group_size", "dtype")] + [("rms_eps", ctypes.c_float),
                                                              ("rope_base", ctypes.c_float),
                                                              ("prefix_width", ctypes.c_int)]


_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)


class pae_weights(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("w_in", "b_in", "w_out", "b_out", "w_t1", "b_t1", "w_t2", "b_t2",
                                  "w_mod", "b_mod", "w_modf", "b_modf")] + \
               [(n, _PP) for n in ("w_qkv", "w_o", "w_gate", "w_up", "w_down",
                                   "s_qkv", "s_o", "s_gate", "s_up", "s_down", "w_prefix_kv")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libpae.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run `python -m flow_matching_action_pi0_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    i, v, vp, st = ctypes.c_int, ctypes.c_void_p, _PP, ctypes.c_void_p
    sig = {
        "pae_create": (i, [ctypes.POINTER(pae_config), ctypes.POINTER(pae_weights), ctypes.POINTER(v)]),
        "pae_set_prefix": (i, [v, i, vp, vp, i, st]),
        "pae_set_prefix_hidden": (i, [v, i, vp, i, st]),
        "pae_precompute_tables": (i, [v, ctypes.POINTER(ctypes.c_double), i, st]),
        "pae_denoise": (i, [v, v, v, i, st]),
        "pae_denoise_host": (i, [v, v, v, i, st]),
        "pae_denoise_steps": (i, [v, v, v, i, i, i, st]),
        "pae_set_option": (i, [v, i, ctypes.c_longlong]),
        "pae_profile_read": (i, [v, i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]),
        "pae_query": (i, [v, i, i, ctypes.POINTER(ctypes.c_longlong)]),
        "pae_plan_query": (i, [ctypes.POINTER(pae_config), i, i, ctypes.POINTER(ctypes.c_longlong)]),
        "pae_sync": (i, [v, st]),
        "pae_clear_error": (None, [v]),
        "pae_last_error": (ctypes.c_char_p, [v]),
        "pae_debug_copy": (i, [v, ctypes.c_char_p, v, ctypes.POINTER(ctypes.c_size_t)]),
        "pae_destroy": (None, [v]),
        "pae_precompute_tables_static": (i, [i, i, i, ctypes.POINTER(pae_weights), ctypes.POINTER(ctypes.c_double),
                                             i, v, v, st]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _check(status: int, ctx=None):
    if status != PAE_OK:
        msg = lib().pae_last_error(ctx)
        raise PaeError(status, msg.decode() if msg else "")


def _ptr_array(ptrs: Sequence[int]):
    arr = (ctypes.c_void_p * len(ptrs))(*ptrs)
    return ctypes.cast(arr, _PP), arr


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ---------------------------------------------------------------- C names
def pae_create(cfg: pae_config, weights: pae_weights) -> int:
    out = ctypes.c_void_p()
    _check(lib().pae_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(out)))
    return out.value


def pae_set_prefix(ctx: int, row: int, k_ptrs: Sequence[int], v_ptrs: Sequence[int], length: int, stream=None):
    kp, _ka = _ptr_array(k_ptrs)
    vp, _va = _ptr_array(v_ptrs)
    _check(lib().pae_set_prefix(ctx, row, kp, vp, length, _stream(stream)), ctx)


def pae_set_prefix_hidden(ctx: int, row: int, h_ptrs: Sequence[int], length: int, stream=None):
    hp, _ha = _ptr_array(h_ptrs)
    _check(lib().pae_set_prefix_hidden(ctx, row, hp, length, _stream(stream)), ctx)


def pae_precompute_tables(ctx: int, t: Sequence[float], K: int, stream=None):
    arr = (ctypes.c_double * (K + 1))(*[float(v) for v in t[:K + 1]])
    _check(lib().pae_precompute_tables(ctx, arr, K, _stream(stream)), ctx)


def pae_denoise(ctx: int, noise_ptr: int, out_ptr: int, batch: int, stream=None):
    _check(lib().pae_denoise(ctx, noise_ptr, out_ptr, batch, _stream(stream)), ctx)


def pae_denoise_host(ctx: int, noise_host_ptr: int, out_host_ptr: int, batch: int, stream=None):
    _check(lib().pae_denoise_host(ctx, noise_host_ptr, out_host_ptr, batch, _stream(stream)), ctx)


def pae_denoise_steps(ctx: int, x_in_ptr: int, x_out_ptr: int, batch: int, k_begin: int, k_end: int, stream=None):
    _check(lib().pae_denoise_steps(ctx, x_in_ptr, x_out_ptr, batch, k_begin, k_end, _stream(stream)), ctx)


def pae_set_option(ctx: int, option: int, value: int):
    _check(lib().pae_set_option(ctx, option, value), ctx)


def pae_profile_read(ctx: int, kernel_class: int):
    """(total device ms, launches) of one kernel class over the last run."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int(0)
    _check(lib().pae_profile_read(ctx, kernel_class, ctypes.byref(ms), ctypes.byref(n)), ctx)
    return ms.value, n.value


def pae_query(ctx: int, what: int, batch: int) -> int:
    v = ctypes.c_longlong(0)
    _check(lib().pae_query(ctx, what, batch, ctypes.byref(v)), ctx)
    return v.value


def pae_plan_query(cfg: pae_config, what: int, batch: int) -> int:
    v = ctypes.c_longlong(0)
    _check(lib().pae_plan_query(ctypes.byref(cfg), what, batch, ctypes.byref(v)))
    return v.value


def pae_sync(ctx: int, stream=None):
    _check(lib().pae_sync(ctx, _stream(stream)), ctx)


def pae_clear_error(ctx: int):
    lib().pae_clear_error(ctx)


def pae_debug_copy(ctx: int, name: str):
    import numpy as np
    n = ctypes.c_size_t(0)
    _check(lib().pae_debug_copy(ctx, name.encode(), None, ctypes.byref(n)), ctx)
    buf = np.empty(n.value, dtype=np.uint8)
    _check(lib().pae_debug_copy(ctx, name.encode(), buf.ctypes.data, ctypes.byref(n)), ctx)
    return buf


def pae_precompute_tables_static(layers: int, width: int, dtype: int, weights: pae_weights, t: Sequence[float],
                                 tables_ptr: int, dt_ptr: int, stream=None):
    """Context-free, allocation-free table build into caller-owned buffers."""
    K = len(t) - 1
    arr = (ctypes.c_double * (K + 1))(*[float(x) for x in t])
    _check(lib().pae_precompute_tables_static(layers, width, dtype, ctypes.byref(weights), arr, K, tables_ptr,
                                              dt_ptr, _stream(stream)))


def pae_destroy(ctx: int):
    if ctx:
        lib().pae_destroy(ctx)


# ---------------------------------------------------------------- wrapper
DTYPE_CODES = {"fp32": PAE_FP32, "bf16": PAE_BF16, "w4a16": PAE_W4A16}


def make_config(layers, width, n_q_heads, n_kv_heads, head_dim, mlp_dim, action_dim, chunk,
                max_batch, max_prefix, dtype, group_size=128, rms_eps=1e-6, rope_base=0.0,
                prefix_width=0) -> pae_config:
    c = pae_config()
    for k, v in dict(layers=layers, width=width, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads, head_dim=head_dim,
                     mlp_dim=mlp_dim, action_dim=action_dim, chunk=chunk, max_batch=max_batch,
                     max_prefix=max_prefix, group_size=group_size, prefix_width=prefix_width).items():
        setattr(c, k, int(v))
    c.dtype = DTYPE_CODES[dtype] if isinstance(dtype, str) else int(dtype)
    c.rms_eps = float(rms_eps)
    c.rope_base = float(rope_base)
    return c


class ActionExpert:
    """One pae context.  `weights` maps the pae_weights field names to CUDA
    tensors (per-layer fields are lists); they may be freed after __init__."""

    def __init__(self, cfg: pae_config, weights: Dict[str, object]):
        self.cfg = cfg
        keep = []
        w = pae_weights()
        for name, _ in pae_weights._fields_:
            val = weights.get(name)
            if val is None:
                continue
            if isinstance(val, (list, tuple)):
                arr, a = _ptr_array([t.data_ptr() for t in val])
                keep.append(a)
                setattr(w, name, arr)
            else:
                setattr(w, name, val.data_ptr())
        self.ctx = pae_create(cfg, w)
        del keep

    def close(self):
        if getattr(self, "ctx", None):
            pae_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_prefix(self, row: int, ks: List, vs: List, length: Optional[int] = None, stream=None):
        n = int(ks[0].shape[0]) if length is None else length
        pae_set_prefix(self.ctx, row, [t.data_ptr() for t in ks], [t.data_ptr() for t in vs], n, stream)

    def set_prefix_hidden(self, row: int, hs: List, length: Optional[int] = None, stream=None):
        n = int(hs[0].shape[0]) if length is None else length
        pae_set_prefix_hidden(self.ctx, row, [t.data_ptr() for t in hs], n, stream)

    def precompute_tables(self, t: Sequence[float], stream=None):
        pae_precompute_tables(self.ctx, list(t), len(t) - 1, stream)

    def denoise(self, noise, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(noise)
        assert noise.dtype == torch.float32 and noise.is_cuda and noise.is_contiguous()
        pae_denoise(self.ctx, noise.data_ptr(), out.data_ptr(), int(noise.shape[0]), stream)
        return out

    def denoise_host(self, noise_host, out_host, stream=None):
        pae_denoise_host(self.ctx, noise_host.data_ptr(), out_host.data_ptr(), int(noise_host.shape[0]), stream)
        return out_host

    def denoise_steps(self, x_in, x_out, k_begin: int, k_end: int, stream=None):
        pae_denoise_steps(self.ctx, x_in.data_ptr(), x_out.data_ptr(), int(x_in.shape[0]), k_begin, k_end, stream)
        return x_out

    def set_option(self, option: int, value: int):
        pae_set_option(self.ctx, option, value)

    def sync(self, stream=None):
        pae_sync(self.ctx, stream)

    def profile_read(self, kernel_class: int):
        return pae_profile_read(self.ctx, kernel_class)

    def query(self, what: int, batch: int) -> int:
        return pae_query(self.ctx, what, batch)

    def debug_copy(self, name: str):
        return pae_debug_copy(self.ctx, name)
