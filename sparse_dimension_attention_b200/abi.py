"""Thin ctypes binding of libaqua_b200.so (the C ABI declared in include/aqua.h).

Argument marshalling only: every step of the attention path runs in the CUDA
kernels behind these calls.  Functions carry the C names and raise AquaError
on a negative status.  There is no fallback: if the shared library is missing
or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libaqua_b200.so")

AQUA_OK = 0
AQUA_ERR_ARG = -1
AQUA_ERR_UNSUPPORTED = -2
AQUA_ERR_WORKSPACE = -3
AQUA_ERR_CUDA = -4
AQUA_ERR_TIMEOUT = -5
AQUA_F32 = 0
AQUA_BF16 = 1
AQUA_CTRL_WORDS = 16

EXPORTED = (
    "aqua_last_error", "aqua_version", "aqua_status",
    "aqua_calibrate_workspace_size", "aqua_calibrate",
    "aqua_project_keys",
    "aqua_decode_workspace_size", "aqua_decode_attn", "aqua_decode_select", "aqua_decode_attend",
    "aqua_decode_attn_static",
    "aqua_prefill_workspace_size", "aqua_prefill_attn",
    "aqua_h2o_update",
    "aqua_selftest_wait_timeout",
)


class AquaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"AQUA status {code}: {msg}")
        self.code = code


class aqua_cache(ctypes.Structure):
    """Mirror of struct aqua_cache in include/aqua.h."""
    _fields_ = [
        ("k_proj", c_void_p), ("v", c_void_p), ("len", c_void_p), ("n_abs", c_void_p),
        ("pos", c_void_p), ("score", c_void_p), ("ctrl", c_void_p),
        ("B", c_int), ("Hkv", c_int), ("d", c_int), ("d_store", c_int), ("Tcap", c_int),
        ("max_len", c_int), ("dtype", c_int), ("dv_store", c_int),
    ]


_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libaqua_b200.so once and declare the signatures; raises if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"AQUA CUDA library not built: {path} is missing "
                           "(run python -m sparse_dimension_attention_b200.build)")
    lib = ctypes.CDLL(path)
    P = c_void_p
    C = POINTER(aqua_cache)
    sig = {
        "aqua_last_error": (ctypes.c_char_p, []),
        "aqua_version": (c_int, []),
        "aqua_status": (c_int, [C, POINTER(c_int), P]),
        "aqua_calibrate_workspace_size": (c_size_t, [c_int, c_int]),
        "aqua_calibrate": (c_int, [P, c_int, c_int, P, P, P, c_size_t, P]),
        "aqua_project_keys": (c_int, [C, P, P, P, c_int, P]),
        "aqua_decode_workspace_size": (c_size_t, [C, c_int]),
        "aqua_decode_attn": (c_int, [C, P, P, P, P, c_int, c_int, c_float, P, c_int, P, P, P, P, P, c_size_t, P]),
        "aqua_decode_select": (c_int, [C, P, P, P, P, c_int, c_int, c_float, P, P, P, c_size_t, P]),
        "aqua_decode_attend": (c_int, [C, P, c_int, c_int, P, c_int, P, P, P, c_size_t, P]),
        "aqua_decode_attn_static": (c_int, [C, P, P, P, P, c_int, c_int, c_float, P, c_int, P, P, P, P, P]),
        "aqua_selftest_wait_timeout": (c_int, [C, ctypes.c_ulonglong, P]),
        "aqua_prefill_workspace_size": (c_size_t, [C, c_int, c_int]),
        "aqua_prefill_attn": (c_int, [C, P, c_int, c_int, P, c_int, c_int, c_float, P, c_int, P, P, P, c_size_t, P]),
        "aqua_h2o_update": (c_int, [C, P, P, c_int, c_int, c_int, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(t) -> int | None:
    """Device (or host) address of a tensor, None for None."""
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(rc: int) -> int:
    if rc != AQUA_OK:
        raise AquaError(rc, load_library().aqua_last_error().decode())
    return rc


# ------------------------------------------------------------------ entry points

def aqua_version() -> int:
    return load_library().aqua_version()


def aqua_last_error() -> str:
    return load_library().aqua_last_error().decode()


def aqua_selftest_wait_timeout(cache: aqua_cache, limit_ns: int, stream=None) -> None:
    """One CTA waits on a barrier nothing completes for limit_ns; the device
    records AQUA_ERR_TIMEOUT in the cache's status word (see aqua_status)."""
    _check(load_library().aqua_selftest_wait_timeout(ctypes.byref(cache), limit_ns, _stream(stream)))


def aqua_status(cache: aqua_cache, stream=None) -> int:
    out = c_int(0)
    _check(load_library().aqua_status(ctypes.byref(cache), ctypes.byref(out), _stream(stream)))
    return out.value


def aqua_calibrate_workspace_size(n: int, d: int) -> int:
    return load_library().aqua_calibrate_workspace_size(n, d)


def aqua_calibrate(X, P_out, sigma_out, workspace, stream=None) -> None:
    n, d = X.shape
    _check(load_library().aqua_calibrate(_ptr(X), n, d, _ptr(P_out), _ptr(sigma_out), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)))


def aqua_project_keys(cache: aqua_cache, k_new, v_new, P, L: int, stream=None) -> None:
    _check(load_library().aqua_project_keys(ctypes.byref(cache), _ptr(k_new), _ptr(v_new), _ptr(P), L,
                                            _stream(stream)))


def aqua_decode_workspace_size(cache: aqua_cache, Hq: int) -> int:
    return load_library().aqua_decode_workspace_size(ctypes.byref(cache), Hq)


def aqua_decode_attn(cache: aqua_cache, q, P, Hq: int, k: int, out, workspace, scale: float = 0.0,
                     k_new=None, v_new=None, sel_out=None, qproj_out=None, scores_out=None, lse_out=None,
                     stream=None) -> None:
    """One decode step; with k_new/v_new ([B, Hkv, d]) the step's token is appended first."""
    out_dtype = AQUA_BF16 if str(out.dtype) == "torch.bfloat16" else AQUA_F32
    _check(load_library().aqua_decode_attn(
        ctypes.byref(cache), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(P), Hq, k, scale, _ptr(out), out_dtype,
        _ptr(sel_out), _ptr(qproj_out), _ptr(scores_out), _ptr(lse_out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def aqua_decode_select(cache: aqua_cache, q, P, Hq: int, k: int, workspace, scale: float = 0.0, k_new=None,
                       v_new=None, sel_out=None, qproj_out=None, stream=None) -> None:
    """First half of a decode step: projection, top-k, group union (and the append)."""
    _check(load_library().aqua_decode_select(
        ctypes.byref(cache), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(P), Hq, k, scale, _ptr(sel_out),
        _ptr(qproj_out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def aqua_decode_attend(cache: aqua_cache, Hq: int, out, workspace, appended: bool = False, P=None,
                       scores_out=None, lse_out=None, stream=None) -> None:
    """Second half of a decode step: attention over the selection aqua_decode_select left in the
    workspace (P is needed only with projected values)."""
    out_dtype = AQUA_BF16 if str(out.dtype) == "torch.bfloat16" else AQUA_F32
    _check(load_library().aqua_decode_attend(
        ctypes.byref(cache), _ptr(P), Hq, int(bool(appended)), _ptr(out), out_dtype, _ptr(scores_out),
        _ptr(lse_out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def aqua_decode_attn_static(cache: aqua_cache, q, P, Hq: int, k: int, out, scale: float = 0.0, k_new=None,
                            v_new=None, sel_out=None, qproj_out=None, scores_out=None, lse_out=None,
                            stream=None) -> None:
    """The decode step without a workspace argument, for callers that cannot allocate
    device scratch: the library's built-in 8 MiB scratch array is used instead."""
    out_dtype = AQUA_BF16 if str(out.dtype) == "torch.bfloat16" else AQUA_F32
    _check(load_library().aqua_decode_attn_static(
        ctypes.byref(cache), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(P), Hq, k, scale, _ptr(out), out_dtype,
        _ptr(sel_out), _ptr(qproj_out), _ptr(scores_out), _ptr(lse_out), _stream(stream)))


def aqua_prefill_workspace_size(cache: aqua_cache, Hq: int, L: int) -> int:
    return load_library().aqua_prefill_workspace_size(ctypes.byref(cache), Hq, L)


def aqua_prefill_attn(cache: aqua_cache, q, pos0: int, L: int, P, Hq: int, k: int, out, workspace,
                      scale: float = 0.0, sel_out=None, qproj_out=None, stream=None) -> None:
    out_dtype = AQUA_BF16 if str(out.dtype) == "torch.bfloat16" else AQUA_F32
    _check(load_library().aqua_prefill_attn(
        ctypes.byref(cache), _ptr(q), pos0, L, _ptr(P), Hq, k, scale, _ptr(out), out_dtype, _ptr(sel_out),
        _ptr(qproj_out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def aqua_h2o_update(cache: aqua_cache, scores, lse, Hq: int, budget: int, recent: int, evicted_out=None,
                    stream=None) -> None:
    _check(load_library().aqua_h2o_update(ctypes.byref(cache), _ptr(scores), _ptr(lse), Hq, budget, recent,
                                          _ptr(evicted_out), _stream(stream)))
