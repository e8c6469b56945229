"""ctypes binding of liblamp.so (declared in include/lamp.h).

Argument marshalling only: every computation runs in the library's CUDA
kernels. Pointers are taken from torch tensors (``data_ptr()``) or plain
integers; streams from ``torch.cuda.Stream`` objects, raw handles or None.
The library must have been built (``python -m mixed_precision_attention_ps_b200.build``);
loading fails loudly otherwise, and there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblamp.so")

LAMP_STRICT, LAMP_RELAXED, LAMP_GIVEN_MASK = 0, 1, 2
LAMP_OK = 0
LAMP_ERR_ARG = -1
LAMP_ERR_UNSUPPORTED = -2
LAMP_ERR_WORKSPACE = -3
LAMP_ERR_CUDA = -4
LAMP_ERR_TIMEOUT = -5
LAMP_ERR_CHECK = -6
LAMP_MAX_SCORE_SLAB_BYTES = 64 << 30
LAMP_NOALLOC_SCRATCH_BYTES = 4 << 20
LAMP_DEBUG_STALL_PRODUCERS = 1

STATUS_NAMES = {
    LAMP_OK: "LAMP_OK", LAMP_ERR_ARG: "LAMP_ERR_ARG", LAMP_ERR_UNSUPPORTED: "LAMP_ERR_UNSUPPORTED",
    LAMP_ERR_WORKSPACE: "LAMP_ERR_WORKSPACE", LAMP_ERR_CUDA: "LAMP_ERR_CUDA",
    LAMP_ERR_TIMEOUT: "LAMP_ERR_TIMEOUT", LAMP_ERR_CHECK: "LAMP_ERR_CHECK",
}


class LampError(RuntimeError):
    """A non-zero lamp_status, with the library's message."""

    def __init__(self, code: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {message}")
        self.code = code


class lamp_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("n_q", ctypes.c_int),
                ("n_k", ctypes.c_int), ("d", ctypes.c_int)]


_P = ctypes.c_void_p


class lamp_args(ctypes.Structure):
    _fields_ = [
        ("dims", lamp_dims),
        ("Q", _P), ("K", _P), ("V", _P),
        ("out", _P),
        ("mask_out", _P),
        ("mu", ctypes.c_int),
        ("tau", ctypes.c_float),
        ("variant", ctypes.c_int),
        ("causal", ctypes.c_int),
        ("stream", _P),
        ("scale", ctypes.c_float),
        ("mask_in", _P),
        ("out_f32", _P),
        ("ps_scores_out", _P),
        ("mixed_scores_out", _P),
        ("lse_out", _P),
        ("n_selected_out", _P),
        ("workspace", _P),
        ("workspace_bytes", ctypes.c_size_t),
        ("status_out", _P),
        ("debug_stall", ctypes.c_int),
    ]


class lamp_gelu_args(ctypes.Structure):
    _fields_ = [
        ("M", ctypes.c_int), ("N", ctypes.c_int), ("K", ctypes.c_int),
        ("x", _P), ("W", _P),
        ("out", _P),
        ("mask_out", _P),
        ("mu", ctypes.c_int),
        ("tau", ctypes.c_float),
        ("variant", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("mask_in", _P),
        ("out_f32", _P),
        ("ps_out", _P),
        ("mixed_out", _P),
        ("n_selected_out", _P),
        ("stream", _P),
    ]


class lamp_ln_args(ctypes.Structure):
    _fields_ = [
        ("M", ctypes.c_int), ("N", ctypes.c_int), ("K", ctypes.c_int),
        ("x", _P), ("W", _P),
        ("out", _P),
        ("mask_out", _P),
        ("mu", ctypes.c_int),
        ("tau", ctypes.c_float),
        ("variant", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("mask_in", _P),
        ("out_f32", _P),
        ("ps_out", _P),
        ("mixed_out", _P),
        ("n_selected_out", _P),
        ("workspace", _P),
        ("workspace_bytes", ctypes.c_size_t),
        ("stream", _P),
    ]


_lock = threading.Lock()
_lib = None

# Every symbol include/lamp.h declares, with its ctypes signature.
SIGNATURES = {
    "lamp_attention": (ctypes.c_int, [ctypes.POINTER(lamp_dims), _P, _P, _P, _P, _P, ctypes.c_int,
                                      ctypes.c_float, ctypes.c_int, ctypes.c_int, _P]),
    "lamp_attention_ex": (ctypes.c_int, [ctypes.POINTER(lamp_args)]),
    "lamp_attention_noalloc": (ctypes.c_int, [ctypes.POINTER(lamp_args)]),
    "lamp_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(lamp_dims), ctypes.c_int]),
    "lamp_last_error": (ctypes.c_char_p, []),
    "lamp_ps_round": (ctypes.c_int, [_P, _P, ctypes.c_size_t, ctypes.c_int, ctypes.c_int, _P]),
    "lamp_version": (ctypes.c_char_p, []),
    "lamp_args_size": (ctypes.c_size_t, []),
    "lamp_linear_gelu": (ctypes.c_int, [ctypes.POINTER(lamp_gelu_args)]),
    "lamp_gelu_args_size": (ctypes.c_size_t, []),
    "lamp_linear_layernorm": (ctypes.c_int, [ctypes.POINTER(lamp_ln_args)]),
    "lamp_ln_workspace_size": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int]),
    "lamp_ln_args_size": (ctypes.c_size_t, []),
}


def load(path: str = LIB_PATH):
    """Load liblamp.so (once). Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise ImportError(
                    f"{path} is missing: build it with `python -m mixed_precision_attention_ps_b200.build` "
                    "(the LAMP kernels have no fallback)")
            L = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            if L.lamp_args_size() != ctypes.sizeof(lamp_args):
                raise ImportError("lamp_args layout of the binding does not match liblamp.so")
            if L.lamp_gelu_args_size() != ctypes.sizeof(lamp_gelu_args):
                raise ImportError("lamp_gelu_args layout of the binding does not match liblamp.so")
            if L.lamp_ln_args_size() != ctypes.sizeof(lamp_ln_args):
                raise ImportError("lamp_ln_args layout of the binding does not match liblamp.so")
            _lib = L
    return _lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x or None
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s or None
    return s.cuda_stream or None


def _check(rc: int) -> int:
    if rc != LAMP_OK:
        raise LampError(rc, load().lamp_last_error().decode())
    return rc


def lamp_last_error() -> str:
    return load().lamp_last_error().decode()


def lamp_version() -> str:
    return load().lamp_version().decode()


def lamp_args_size() -> int:
    return int(load().lamp_args_size())


def lamp_workspace_size(dims, variant: int) -> int:
    return int(load().lamp_workspace_size(ctypes.byref(lamp_dims(*dims)), int(variant)))


def lamp_attention(dims, Q, K, V, out, mask_out, mu: int, tau: float, variant: int, causal: int,
                   stream=None, check: bool = True) -> int:
    """Basic entry point. dims = (B, H, n_q, n_k, d). Returns the status (raises
    LampError on a non-zero status when check is true)."""
    rc = load().lamp_attention(ctypes.byref(lamp_dims(*dims)), _ptr(Q), _ptr(K), _ptr(V), _ptr(out),
                               _ptr(mask_out), int(mu), float(tau), int(variant), int(causal),
                               _stream(stream))
    return _check(rc) if check else rc


def make_args(dims, Q, K, V, out, *, mask_out=None, mu=4, tau=0.0, variant=LAMP_STRICT, causal=1,
              stream=None, scale=0.0, mask_in=None, out_f32=None, ps_scores_out=None,
              mixed_scores_out=None, lse_out=None, n_selected_out=None, workspace=None,
              workspace_bytes=0, status_out=None, debug_stall=0) -> lamp_args:
    return lamp_args(lamp_dims(*dims), _ptr(Q), _ptr(K), _ptr(V), _ptr(out), _ptr(mask_out), int(mu),
                     float(tau), int(variant), int(causal), _stream(stream), float(scale), _ptr(mask_in),
                     _ptr(out_f32), _ptr(ps_scores_out), _ptr(mixed_scores_out), _ptr(lse_out),
                     _ptr(n_selected_out), _ptr(workspace), int(workspace_bytes), _ptr(status_out),
                     int(debug_stall))


def lamp_attention_ex(args: lamp_args | None = None, check: bool = True, **kw) -> int:
    """Extended entry point: pass a lamp_args, or make_args' keyword arguments."""
    if args is None:
        args = make_args(**kw)
    rc = load().lamp_attention_ex(ctypes.byref(args))
    return _check(rc) if check else rc


def lamp_attention_noalloc(args: lamp_args | None = None, check: bool = True, **kw) -> int:
    """Entry point without device allocation: scratch comes from the library's fixed
    per-device array (workspace must stay unset)."""
    if args is None:
        args = make_args(**kw)
    rc = load().lamp_attention_noalloc(ctypes.byref(args))
    return _check(rc) if check else rc


def lamp_ps_round(x, y, n: int, mu: int, path: int = 0, stream=None, check: bool = True) -> int:
    rc = load().lamp_ps_round(_ptr(x), _ptr(y), int(n), int(mu), int(path), _stream(stream))
    return _check(rc) if check else rc


def lamp_gelu_args_size() -> int:
    return int(load().lamp_gelu_args_size())


def make_gelu_args(M, N, K, x, W, out, *, mask_out=None, mu=4, tau=0.0, variant=LAMP_STRICT, scale=0.0,
                   mask_in=None, out_f32=None, ps_out=None, mixed_out=None, n_selected_out=None,
                   stream=None) -> lamp_gelu_args:
    return lamp_gelu_args(int(M), int(N), int(K), _ptr(x), _ptr(W), _ptr(out), _ptr(mask_out), int(mu),
                          float(tau), int(variant), float(scale), _ptr(mask_in), _ptr(out_f32), _ptr(ps_out),
                          _ptr(mixed_out), _ptr(n_selected_out), _stream(stream))


def lamp_linear_gelu(args: lamp_gelu_args | None = None, check: bool = True, **kw) -> int:
    """LAMP GELU(scale * x W^T): pass a lamp_gelu_args, or make_gelu_args' keyword arguments."""
    if args is None:
        args = make_gelu_args(**kw)
    rc = load().lamp_linear_gelu(ctypes.byref(args))
    return _check(rc) if check else rc


def lamp_ln_args_size() -> int:
    return int(load().lamp_ln_args_size())


def lamp_ln_workspace_size(M: int, N: int) -> int:
    return int(load().lamp_ln_workspace_size(int(M), int(N)))


def make_ln_args(M, N, K, x, W, out, *, mask_out=None, mu=4, tau=0.0, variant=LAMP_STRICT, scale=0.0, eps=0.0,
                 mask_in=None, out_f32=None, ps_out=None, mixed_out=None, n_selected_out=None, workspace=None,
                 workspace_bytes=0, stream=None) -> lamp_ln_args:
    return lamp_ln_args(int(M), int(N), int(K), _ptr(x), _ptr(W), _ptr(out), _ptr(mask_out), int(mu), float(tau),
                        int(variant), float(scale), float(eps), _ptr(mask_in), _ptr(out_f32), _ptr(ps_out),
                        _ptr(mixed_out), _ptr(n_selected_out), _ptr(workspace), int(workspace_bytes),
                        _stream(stream))


def lamp_linear_layernorm(args: lamp_ln_args | None = None, check: bool = True, **kw) -> int:
    """LAMP LayerNorm(scale * x W^T): pass a lamp_ln_args, or make_ln_args' keyword arguments."""
    if args is None:
        args = make_ln_args(**kw)
    rc = load().lamp_linear_layernorm(ctypes.byref(args))
    return _check(rc) if check else rc
