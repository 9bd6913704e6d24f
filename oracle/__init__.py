"""ORACLE - test infrastructure, not product code.

Plain fp64 CPU restatement of the quantized sparse-MoE feed-forward layer
(C in ``moe_oracle.c``, orchestration here in numpy).  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs
use it.  It imports nothing from the CUDA library package, and the library
never imports it.

Every function cites the passage it follows; the C file's header lists the
pages.  Parity of each function is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

Q4B32, Q3B32, Q2B32 = 1, 2, 3
FMT = {"q4": Q4B32, "q3": Q3B32, "q2": Q2B32}
ZERO = {Q4B32: 8, Q3B32: 4, Q2B32: 2}
BLOCK_BYTES = {Q4B32: 16, Q3B32: 12, Q2B32: 8}

_dp = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_fp = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_u8 = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_u16 = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_i32 = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, OpenMP over tokens) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            L.oracle_half_to_double.restype = ctypes.c_double
            L.oracle_half_to_double.argtypes = [ctypes.c_uint16]
            L.oracle_bf16_to_double.restype = ctypes.c_double
            L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            L.oracle_code.restype = ctypes.c_int
            L.oracle_code.argtypes = [ctypes.c_int, _u8, ctypes.c_int]
            L.oracle_weight.restype = ctypes.c_double
            L.oracle_weight.argtypes = [ctypes.c_int, _u8, ctypes.c_uint16, ctypes.c_int]
            L.oracle_silu.restype = ctypes.c_double
            L.oracle_silu.argtypes = [ctypes.c_double]
            L.oracle_dequant.restype = None
            L.oracle_dequant.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _u8, _u16, _dp]
            L.oracle_qmatvec.restype = None
            L.oracle_qmatvec.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _u8, _u16, _dp, _dp]
            L.oracle_expert.restype = None
            L.oracle_expert.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        _u8, _u16, _u8, _u16, _u8, _u16, _dp, _dp, ctypes.c_void_p]
            L.oracle_router_logits.restype = None
            L.oracle_router_logits.argtypes = [ctypes.c_int, ctypes.c_int, _dp, _fp, ctypes.c_void_p, _dp]
            L.oracle_route.restype = None
            L.oracle_route.argtypes = [ctypes.c_int, ctypes.c_int, _dp, _i32, _dp, _dp]
            L.oracle_moe_layer.restype = None
            L.oracle_moe_layer.argtypes = [ctypes.c_int] * 8 + [
                _u16, _fp, ctypes.c_void_p,
                _u8, _u16, _u8, _u16, _u8, _u16,
                _u8, _u16, _u8, _u16, _u8, _u16,
                _dp, _i32, _dp, _dp]
            L.oracle_rmsnorm.restype = None
            L.oracle_rmsnorm.argtypes = [ctypes.c_int, _dp, ctypes.c_double, _dp]
            L.oracle_round_bf16.restype = ctypes.c_uint16
            L.oracle_round_bf16.argtypes = [ctypes.c_double]
            L.oracle_round_bf16_array.restype = None
            L.oracle_round_bf16_array.argtypes = [ctypes.c_size_t, _dp, _u16]
            L.oracle_bf16_to_double_array.restype = None
            L.oracle_bf16_to_double_array.argtypes = [ctypes.c_size_t, _u16, _dp]
            L.oracle_half_to_double_array.restype = None
            L.oracle_half_to_double_array.argtypes = [ctypes.c_size_t, _u16, _dp]
            _lib = L
    return _lib


def _fmt(fmt) -> int:
    return FMT[fmt] if isinstance(fmt, str) else int(fmt)


def _u16a(a) -> np.ndarray:
    a = np.asarray(a)
    return np.ascontiguousarray(a.view(np.uint16) if a.dtype == np.int16 else a.astype(np.uint16, copy=False))


def _u8a(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=np.uint8)


def _np(t) -> np.ndarray:
    """Accept numpy arrays or CPU torch tensors (the generator returns torch)."""
    if hasattr(t, "detach"):
        t = t.detach().cpu().numpy()
    return np.asarray(t)


# --- formats -----------------------------------------------------------------

def half_to_f64(bits) -> np.ndarray:
    """IEEE binary16 bit patterns -> fp64 (from the format's definition)."""
    b = _u16a(_np(bits)).ravel()
    out = np.empty(b.size, dtype=np.float64)
    lib().oracle_half_to_double_array(b.size, b, out)
    return out.reshape(np.shape(bits))


def bf16_to_f64(bits) -> np.ndarray:
    b = _u16a(_np(bits)).ravel()
    out = np.empty(b.size, dtype=np.float64)
    lib().oracle_bf16_to_double_array(b.size, b, out)
    return out.reshape(np.shape(bits))


def round_bf16(v) -> np.ndarray:
    """fp64 -> bf16 bits, one round-to-nearest-even step."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.size, dtype=np.uint16)
    lib().oracle_round_bf16_array(v.size, v.ravel(), out)
    return out.reshape(v.shape)


def block_codes(fmt, blk) -> np.ndarray:
    """The 32 codes of one packed block (Q4B32: nibbles, low first; Q3B32 / Q2B32:
    3-bit / 2-bit fields of a little-endian 96-bit / 64-bit integer)."""
    f = _fmt(fmt)
    blk = _u8a(blk)
    return np.array([lib().oracle_code(f, blk, j) for j in range(32)], dtype=np.int64)


def block_weights(fmt, blk, scale_bits) -> np.ndarray:
    """w_j = s * (q_j - 8) (Q4B32), s * (q_j - 4) (Q3B32) or s * (q_j - 2) (Q2B32)."""
    f = _fmt(fmt)
    blk = _u8a(blk)
    return np.array([lib().oracle_weight(f, blk, int(scale_bits) & 0xFFFF, j) for j in range(32)])


def dequant(fmt, codes, scales) -> np.ndarray:
    """Dense fp64 [rows, K] of a packed matrix (codes [rows, K/32, B], scales
    [rows, K/32]): w = s * (q - zero) element by element, in C."""
    codes = _u8a(_np(codes))
    scales = _u16a(_np(scales))
    rows, nb = codes.shape[0], codes.shape[1]
    out = np.empty((rows, nb * 32))
    lib().oracle_dequant(_fmt(fmt), rows, nb * 32, codes, scales, out)
    return out


# --- layer steps ---------------------------------------------------------------

def qmatvec(fmt, codes, scales, x) -> np.ndarray:
    """y = W x, W packed [rows][K/32] blocks along K."""
    codes = _u8a(_np(codes))
    scales = _u16a(_np(scales))
    rows, nb = codes.shape[0], codes.shape[1]
    x = np.ascontiguousarray(x, dtype=np.float64)
    assert x.size == nb * 32
    y = np.empty(rows)
    lib().oracle_qmatvec(_fmt(fmt), rows, nb * 32, codes, scales, x, y)
    return y


def expert(fmt, gate, up, down, x, want_h: bool = False):
    """SwiGLU expert on one token.  gate/up/down are (codes, scales) pairs of one
    expert: gate/up codes [I, d/32, B], down codes [d, I/32, B]."""
    gc, gs = _u8a(_np(gate[0])), _u16a(_np(gate[1]))
    uc, us = _u8a(_np(up[0])), _u16a(_np(up[1]))
    dc, ds = _u8a(_np(down[0])), _u16a(_np(down[1]))
    I, d = gc.shape[0], gc.shape[1] * 32
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty(d)
    h = np.empty(I) if want_h else None
    lib().oracle_expert(_fmt(fmt), d, I, gc, gs, uc, us, dc, ds, x, y,
                        h.ctypes.data if want_h else None)
    return (y, h) if want_h else y


def silu(z: float) -> float:
    return lib().oracle_silu(float(z))


def router_logits(x, Wr, bias=None) -> np.ndarray:
    """logit_e = x . W_r[e] (+ b_e), fp64 accumulation; x fp64 [d]."""
    Wr = np.ascontiguousarray(Wr, dtype=np.float32)
    E, d = Wr.shape
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(E)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    lib().oracle_router_logits(d, E, x, Wr, None if b is None else b.ctypes.data, out)
    return out


def route(logits, k: int):
    """Softmax over all E, top-k by probability (ties -> lower id), renormalise.
    Returns (ids int32 [k], w fp64 [k], gap = k-th minus (k+1)-th logit)."""
    lg = np.ascontiguousarray(logits, dtype=np.float64)
    ids = np.empty(k, dtype=np.int32)
    w = np.empty(k)
    gap = np.empty(1)
    lib().oracle_route(lg.size, k, lg, ids, w, gap)
    return ids, w, float(gap[0])


def rmsnorm(r, eps: float = 1e-6) -> np.ndarray:
    r = np.ascontiguousarray(r, dtype=np.float64)
    out = np.empty_like(r)
    lib().oracle_rmsnorm(r.size, r, eps, out)
    return out


def moe_layer(fmt, k, x_bf16, W: dict):
    """The whole layer over T tokens (each token independently) in C.

    W is ``synth.layer_weights`` output (all E experts present).  Returns
    (y fp64 [T, d], ids int32 [T, k], w fp64 [T, k], gap fp64 [T])."""
    f = _fmt(fmt)
    x = _u16a(_np(x_bf16))
    T, d = x.shape
    Wr = np.ascontiguousarray(W["router_w"], dtype=np.float32)
    E = Wr.shape[0]
    b = W.get("router_b")
    b = None if b is None else np.ascontiguousarray(b, dtype=np.float32)
    c = [_u8a(_np(t)) for t in W["codes"]]
    s = [_u16a(_np(t)) for t in W["scales"]]
    sc = [_u8a(_np(t)) for t in W["sh_codes"]]
    ss = [_u16a(_np(t)) for t in W["sh_scales"]]
    I = c[0].shape[1]
    n_sh = sc[0].shape[0]
    I_s = sc[0].shape[1] if n_sh else 32
    if n_sh == 0:   # placeholders, never read
        sc = [np.zeros(1, np.uint8)] * 3
        ss = [np.zeros(1, np.uint16)] * 3
    y = np.empty((T, d))
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k))
    gap = np.empty(T)
    lib().oracle_moe_layer(f, d, E, I, k, n_sh, I_s, T, x, Wr,
                           None if b is None else b.ctypes.data,
                           c[0], s[0], c[1], s[1], c[2], s[2],
                           sc[0], ss[0], sc[1], ss[1], sc[2], ss[2],
                           y, ids, w, gap)
    return y, ids, w, gap


def moe_token(fmt, k, x_bf16_row, router_w, router_b, get_expert, get_shared, n_shared=1):
    """One token through one layer, fetching only the experts it needs.

    get_expert(e) / get_shared(s) return ((gc, gs), (uc, us), (dc, ds)) of one
    expert.  Same steps as ``moe_layer``; used where the full layer does not fit
    on the host.  Returns (y fp64 [d], ids, w, gap)."""
    x = bf16_to_f64(np.asarray(x_bf16_row))
    lg = router_logits(x, router_w, router_b)
    ids, w, gap = route(lg, k)
    y = np.zeros(x.size)
    for j in range(k):
        g, u, dn = get_expert(int(ids[j]))
        y += w[j] * expert(fmt, g, u, dn, x)
    for s in range(n_shared):
        g, u, dn = get_shared(s)
        y += expert(fmt, g, u, dn, x)
    return y, ids, w, gap


def moe_token_with_ids(fmt, x_bf16_row, ids, router_w, router_b, get_expert, get_shared, n_shared=1):
    """As ``moe_token`` but with the expert set given (used for a token whose
    10th/11th logits are within the near-tie margin: the oracle then evaluates
    the GPU's choice).  The weights are still the oracle's softmax of its own
    logits, renormalised over the given ids."""
    x = bf16_to_f64(np.asarray(x_bf16_row))
    lg = router_logits(x, router_w, router_b)
    p = np.exp(lg - lg.max())
    p /= p.sum()
    ids = np.asarray(ids, dtype=np.int64)
    w = p[ids] / p[ids].sum()
    y = np.zeros(x.size)
    for j, e in enumerate(ids):
        g, u, dn = get_expert(int(e))
        y += w[j] * expert(fmt, g, u, dn, x)
    for s in range(n_shared):
        g, u, dn = get_shared(s)
        y += expert(fmt, g, u, dn, x)
    return y, w


def moe_rows_dense(fmt, k, x_bf16, router_w, router_b, get_expert, get_shared, n_shared=1,
                   ids_for=None, threads: int | None = None):
    """The layer for many tokens, each on its own, with the experts' matrix
    products done per expert over all of its tokens at once.

    Same steps and the same fp64 arithmetic as ``moe_token`` (router logits,
    softmax top-k, SwiGLU per chosen expert, weighted sum + shared), with two
    library primitives in place of the per-token loops: the router logits are
    one fp64 matrix product, and every expert is dequantised once (``dequant``)
    and applied to the stacked rows of its tokens with fp64 matrix products.
    Only the order of the fp64 sums differs from ``moe_token``.

    x_bf16: bf16 bits [n, d].  ids_for: optional {row: ids} for rows whose
    experts are given (the GPU's choice at a near tie); their weights are the
    softmax of the oracle's logits renormalised over the given ids, as in
    ``moe_token_with_ids``.  Returns (y fp64 [n, d], ids [n, k], w [n, k],
    gap [n])."""
    from concurrent.futures import ThreadPoolExecutor

    x = bf16_to_f64(np.asarray(x_bf16))
    n, d = x.shape
    lg = x @ np.asarray(router_w, dtype=np.float64).T
    if router_b is not None:
        lg = lg + np.asarray(router_b, dtype=np.float64)
    ids = np.empty((n, k), dtype=np.int32)
    w = np.empty((n, k))
    gap = np.empty(n)
    for t in range(n):
        ids[t], w[t], gap[t] = route(lg[t], k)
    for t, g_ids in (ids_for or {}).items():
        p = np.exp(lg[t] - lg[t].max())
        p /= p.sum()
        g_ids = np.asarray(g_ids, dtype=np.int64)
        ids[t] = g_ids
        w[t] = p[g_ids] / p[g_ids].sum()
    y = np.zeros((n, d))
    experts = sorted(set(int(e) for e in ids.ravel()))

    def apply(mats, xs):
        (gc, gs), (uc, us), (dc, ds) = mats
        g = xs @ dequant(fmt, gc, gs).T
        u = xs @ dequant(fmt, uc, us).T
        h = g / (1.0 + np.exp(-g)) * u
        return h @ dequant(fmt, dc, ds).T

    def routed(e):
        rows, slots = np.nonzero(ids == e)
        return e, rows, slots, apply(get_expert(e), x[rows])

    try:   # one BLAS thread per worker: the workers already use every core
        from threadpoolctl import threadpool_limits
        blas = threadpool_limits(1)
    except ImportError:
        import contextlib
        blas = contextlib.nullcontext()
    with blas, ThreadPoolExecutor(max_workers=threads or min(32, os.cpu_count() or 1)) as ex:
        res = list(ex.map(routed, experts))
        shared = list(ex.map(lambda s: apply(get_shared(s), x), range(n_shared)))
    contrib = [[] for _ in range(n)]   # (slot j, y_e row) per token
    for e, rows, slots, ye in res:
        for i, (t, j) in enumerate(zip(rows, slots)):
            contrib[t].append((int(j), ye[i]))
    for t in range(n):
        for j, ye in sorted(contrib[t], key=lambda c: c[0]):   # j = 0..k-1, as moe_token
            y[t] += w[t, j] * ye
    for ys in shared:
        y += ys
    return y, ids, w, gap
