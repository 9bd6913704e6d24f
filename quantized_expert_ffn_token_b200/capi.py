"""Thin ctypes binding of the C ABI in include/moe.h.

Argument marshalling only: every step of the layer runs in the CUDA library
``libqeffn.so`` (built in-tree by ``build.py``).  Functions keep the C names;
device buffers are passed as torch CUDA tensors (or raw integer addresses),
streams as torch streams (or raw handles).  A non-zero status raises
``MoeError``.  There is no fallback: if the library is missing, importing
this module fails.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqeffn.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_OOM = -2
MOE_ERR_CUDA = -3
MOE_ERR_NOT_LOADED = -4
MOE_ERR_TOO_MANY_TOKENS = -5
MOE_ERR_DEVICE_TIMEOUT = -6
MOE_ERR_UNSUPPORTED = -7
MOE_Q4B32 = 1
MOE_Q3B32 = 2
MOE_Q2B32 = 3
MOE_FLAG_NO_DECODE_KERNEL = 1
MOE_FLAG_NO_TENSOR_PREFILL = 2
MOE_FLAG_NO_MULTI_DECODE = 8
MOE_FLAG_SPLIT_DECODE = 16
MOE_FLAG_TEST_WITHHOLD = 256
MOE_FLAG_TRACE = 4
MOE_L2_STREAM = 0
MOE_L2_KEEP_SHARED = 1
MOE_ROUTE_STATIC_MAX_LOGITS = 65536
FORMATS = {"q4": MOE_Q4B32, "q3": MOE_Q3B32, "q2": MOE_Q2B32}

EXPORTED = [
    "moe_create", "moe_load_layer", "moe_forward", "moe_forward_stack",
    "moe_forward_stack_host", "moe_destroy", "moe_get_device_error",
    "moe_status_string", "moe_last_error", "moe_timing_enable", "moe_timing_read",
    "moe_trace_read", "moe_route_static", "moe_set_l2_policy",
]


class moe_config(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("n_experts", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("top_k", ctypes.c_int), ("n_shared", ctypes.c_int), ("d_ff_shared", ctypes.c_int),
                ("n_layers", ctypes.c_int), ("max_tokens", ctypes.c_int), ("fmt", ctypes.c_int),
                ("device_mem_limit", ctypes.c_longlong), ("flags", ctypes.c_int)]


class moe_layer_weights(ctypes.Structure):
    _fields_ = [("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("codes", ctypes.c_void_p * 3), ("scales", ctypes.c_void_p * 3),
                ("sh_codes", ctypes.c_void_p * 3), ("sh_scales", ctypes.c_void_p * 3),
                ("on_device", ctypes.c_int)]


class moe_stack_record(ctypes.Structure):
    _fields_ = [("x_bf16", ctypes.c_void_p), ("y_bf16", ctypes.c_void_p), ("y_f32", ctypes.c_void_p),
                ("ids", ctypes.c_void_p), ("w", ctypes.c_void_p), ("rows", ctypes.c_void_p),
                ("n_rows", ctypes.c_int)]


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status}) {last_error()}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python quantized_expert_ffn_token_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i = ctypes.c_void_p, ctypes.c_int
    L.moe_create.argtypes = [ctypes.POINTER(moe_config), i, ctypes.POINTER(vp)]
    L.moe_load_layer.argtypes = [vp, i, ctypes.POINTER(moe_layer_weights), vp]
    L.moe_forward.argtypes = [vp, i, vp, i, vp, vp, vp, vp, vp]
    L.moe_forward_stack.argtypes = [vp, i, i, vp, i, vp, ctypes.POINTER(moe_stack_record), vp]
    L.moe_forward_stack_host.argtypes = [vp, i, i, vp, i, vp, vp]
    L.moe_destroy.argtypes = [vp]
    L.moe_get_device_error.argtypes = [vp, ctypes.POINTER(i)]
    L.moe_timing_enable.argtypes = [vp, i]
    L.moe_set_l2_policy.argtypes = [vp, i]
    L.moe_timing_read.argtypes = [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong),
                                  ctypes.POINTER(ctypes.c_longlong), ctypes.c_char_p, i]
    L.moe_trace_read.argtypes = [vp, ctypes.POINTER(ctypes.c_ulonglong), i, ctypes.POINTER(i)]
    L.moe_route_static.argtypes = [vp, i, i, vp, vp, i, i, vp, vp, vp]
    L.moe_status_string.argtypes = [i]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_last_error.argtypes = []
    L.moe_last_error.restype = ctypes.c_char_p
    for n in ("moe_create", "moe_load_layer", "moe_forward", "moe_forward_stack",
              "moe_forward_stack_host", "moe_destroy", "moe_get_device_error",
              "moe_timing_enable", "moe_timing_read", "moe_trace_read", "moe_route_static",
              "moe_set_l2_policy"):
        getattr(L, n).restype = i
    return L


lib = _load()


def _ptr(t) -> int | None:
    """Address of a tensor's data (None for None); ints pass through."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, what: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, what)


def status_string(status: int) -> str:
    return lib.moe_status_string(status).decode()


def last_error() -> str:
    return lib.moe_last_error().decode()


def moe_create(cfg: moe_config, device: int = 0) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib.moe_create(ctypes.byref(cfg), device, ctypes.byref(h)), "moe_create")
    return h


def moe_load_layer(ctx, layer: int, w: moe_layer_weights, stream=None) -> None:
    _check(lib.moe_load_layer(ctx, layer, ctypes.byref(w), _stream(stream)), "moe_load_layer")


def moe_forward(ctx, layer: int, x, T: int, y, y_f32=None, ids=None, w=None, stream=None) -> None:
    _check(lib.moe_forward(ctx, layer, _ptr(x), T, _ptr(y), _ptr(y_f32), _ptr(ids), _ptr(w),
                           _stream(stream)), "moe_forward")


def moe_forward_stack(ctx, layer0: int, n_layers: int, x, T: int, resid_out, rec=None,
                      stream=None) -> None:
    _check(lib.moe_forward_stack(ctx, layer0, n_layers, _ptr(x), T, _ptr(resid_out),
                                 ctypes.byref(rec) if rec is not None else None, _stream(stream)),
           "moe_forward_stack")


def moe_forward_stack_host(ctx, layer0: int, n_layers: int, x_host, T: int, resid_host,
                           stream=None) -> None:
    _check(lib.moe_forward_stack_host(ctx, layer0, n_layers, _ptr(x_host), T, _ptr(resid_host),
                                      _stream(stream)), "moe_forward_stack_host")


def moe_destroy(ctx) -> None:
    _check(lib.moe_destroy(ctx), "moe_destroy")


def moe_set_l2_policy(ctx, mode: int) -> None:
    """L2 eviction priorities of the decode kernels' weight copies (see include/moe.h)."""
    _check(lib.moe_set_l2_policy(ctx, mode), "moe_set_l2_policy")


def moe_get_device_error(ctx) -> int:
    code = ctypes.c_int(0)
    _check(lib.moe_get_device_error(ctx, ctypes.byref(code)), "moe_get_device_error")
    return code.value


def moe_timing_enable(ctx, on: bool = True) -> None:
    _check(lib.moe_timing_enable(ctx, 1 if on else 0), "moe_timing_enable")


def moe_timing_read(ctx) -> dict:
    ms = ctypes.c_double()
    timed = ctypes.c_longlong()
    allk = ctypes.c_longlong()
    name = ctypes.create_string_buffer(128)
    _check(lib.moe_timing_read(ctx, ctypes.byref(ms), ctypes.byref(timed), ctypes.byref(allk), name, 128),
           "moe_timing_read")
    return {"ms": ms.value, "timed_launches": timed.value, "all_launches": allk.value,
            "kernel": name.value.decode()}


def moe_trace_read(ctx, n_max: int = 1 << 16):
    """Phase trace records as a list of 24-tuples (see include/moe.h)."""
    buf = (ctypes.c_ulonglong * (24 * n_max))()
    n = ctypes.c_int(0)
    _check(lib.moe_trace_read(ctx, buf, n_max, ctypes.byref(n)), "moe_trace_read")
    return [tuple(buf[24 * i:24 * i + 24]) for i in range(n.value)]


def moe_route_static(x, T: int, d_model: int, router_w, router_bias, n_experts: int, top_k: int,
                     ids, w, stream=None) -> None:
    """Allocation-free routing (see include/moe.h): device buffers in, ids/w out."""
    _check(lib.moe_route_static(_ptr(x), T, d_model, _ptr(router_w), _ptr(router_bias), n_experts,
                                top_k, _ptr(ids), _ptr(w), _stream(stream)), "moe_route_static")


def make_record(x=None, y=None, y_f32=None, ids=None, w=None, rows=None) -> moe_stack_record:
    r = moe_stack_record()
    r.x_bf16, r.y_bf16, r.y_f32 = _ptr(x), _ptr(y), _ptr(y_f32)
    r.ids, r.w = _ptr(ids), _ptr(w)
    r.rows = _ptr(rows)
    r.n_rows = 0 if rows is None else int(rows.numel())
    return r
