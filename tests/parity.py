"""Shared helpers of the GPU parity tests: run the CUDA library through the C ABI
and the oracle on the same seeded inputs, and compare.

The bar:
* expert ids identical, except for a token whose oracle 10th and 11th logits
  (fp64) differ by less than 1e-5; such a token is re-evaluated by the oracle
  with the GPU's ids before its outputs are compared;
* routing weights within 1e-5 absolute;
* relative L2 of the fp32 layer output (the value the library rounds to bf16)
  against the oracle's fp64 output <= 1e-3 (fp32 accumulation);
* the bf16 output is the round-to-nearest-even of that fp32 value, bit for bit;
* relative L2 of the bf16 output against the oracle's bf16-rounded output
  <= BF16_TOL (see its note).
"""
from __future__ import annotations

import functools
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
import synth

NEAR_TIE = 1e-5
W_TOL = 1e-5
F32_TOL = 1e-3
# Comparing two bf16 roundings: where the fp32 value and the exact value fall
# on different sides of a rounding boundary the two differ by one bf16 ulp
# (2^-8..2^-7 relative).  With a pre-rounding relative error e that happens for
# a fraction ~e/ulp of elements, so the relative L2 of the difference is about
# sqrt(e * ulp); e <= 1e-4 gives <= 8e-4.
BF16_TOL = 1e-3
# The tensor-core path (T >= 64) rounds the dequantised weights and the
# SwiGLU outputs to fp16 (the MMA takes one operand type): about 4e-4
# relative L2 before the bf16 rounding (inside F32_TOL), hence about
# sqrt(4e-4 * 2^-7.5) = 1.5e-3 between the two bf16 roundings.
TC_BF16_TOL = 2e-3
TC_MIN_TOKENS = 9   # the library's first token count on the tensor-core path


def bf16_tol(T: int) -> float:
    return TC_BF16_TOL if T >= TC_MIN_TOKENS else BF16_TOL


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    n = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (n if n > 0 else 1.0))


def bits_to_f64(bits) -> np.ndarray:
    return oracle.bf16_to_f64(np.asarray(bits).view(np.uint16))


class HostLayer:
    """One whole layer of the seeded generator in host memory, generated on the
    device (fast) and copied over once; the same interface as ExpertSource."""

    def __init__(self, cfg: synth.LayerConfig, layer: int, device="cuda"):
        self.cfg, self.layer = cfg, layer
        W = synth.layer_weights(cfg, layer, device=device)
        self.router_w = np.asarray(W["router_w"], dtype=np.float32)
        self.router_b = W["router_b"]
        self.codes = [to_np(t) for t in W["codes"]]
        self.scales = [to_np(t).view(np.uint16) for t in W["scales"]]
        self.sh_codes = [to_np(t) for t in W["sh_codes"]]
        self.sh_scales = [to_np(t).view(np.uint16) for t in W["sh_scales"]]
        del W

    def expert(self, e: int):
        return tuple((self.codes[t][e], self.scales[t][e]) for t in range(3))

    def shared(self, s: int):
        return tuple((self.sh_codes[t][s], self.sh_scales[t][s]) for t in range(3))


def oracle_rows_dense(cfg, src, x_bits: np.ndarray, rows):
    """Oracle outputs of many token rows at once (experts applied per expert
    with fp64 matrix products): (y [n, d], ids, w, gap)."""
    rows = list(rows)
    return oracle.moe_rows_dense(cfg.fmt, cfg.k, x_bits[rows], src.router_w, src.router_b,
                                 src.expert, src.shared, cfg.n_shared)


def oracle_routing(cfg, src, x_bits: np.ndarray):
    """Oracle routing of every row (router logits as one fp64 matrix product,
    then the oracle's softmax top-k per token): ids [n, k], w [n, k], gap [n]."""
    x = oracle.bf16_to_f64(np.asarray(x_bits).view(np.uint16))
    lg = x @ np.asarray(src.router_w, dtype=np.float64).T
    if src.router_b is not None:
        lg = lg + np.asarray(src.router_b, dtype=np.float64)
    n = lg.shape[0]
    ids = np.empty((n, cfg.k), dtype=np.int32)
    w = np.empty((n, cfg.k))
    gap = np.empty(n)
    for t in range(n):
        ids[t], w[t], gap[t] = oracle.route(lg[t], cfg.k)
    return ids, w, gap, lg


def ids_agree(g_ids, o_ids, o_gap: float, logits) -> str:
    """How the GPU's ids of one token relate to the oracle's.

    'same': identical, in order.  'order': the same experts, and wherever the
    order differs the oracle's logits of the two experts at that position are
    within NEAR_TIE of each other (a near tie inside the chosen set).  'tie':
    a different set, allowed because the oracle's k-th and (k+1)-th logits are
    within NEAR_TIE.  Anything else fails the assertion."""
    g_ids, o_ids = np.asarray(g_ids), np.asarray(o_ids)
    if np.array_equal(g_ids, o_ids):
        return "same"
    if sorted(g_ids.tolist()) == sorted(o_ids.tolist()):
        lg = logits()
        diff = np.nonzero(g_ids != o_ids)[0]
        worst = max(abs(lg[g_ids[j]] - lg[o_ids[j]]) for j in diff)
        assert worst < NEAR_TIE, f"ids {g_ids.tolist()} != oracle {o_ids.tolist()} (order, gap {worst:.3g})"
        return "order"
    assert o_gap < NEAR_TIE, (f"ids {g_ids.tolist()} != oracle {o_ids.tolist()} "
                              f"(k-th to (k+1)-th gap {o_gap:.3g})")
    return "tie"


class ExpertSource:
    """Generates (on the host) exactly the experts the oracle asks for."""

    def __init__(self, cfg: synth.LayerConfig, layer: int):
        self.cfg, self.layer = cfg, layer
        self.router_w = synth.router_weights(cfg, layer)
        self.router_b = synth.router_bias(cfg, layer)

    @functools.lru_cache(maxsize=64)
    def expert(self, e: int):
        c, l = self.cfg, self.layer
        return tuple((synth.expert_codes(c, l, t, e, e + 1)[0].numpy(),
                      synth.expert_scales(c, l, t, e, e + 1)[0].numpy()) for t in range(3))

    @functools.lru_cache(maxsize=4)
    def shared(self, s: int):
        c, l = self.cfg, self.layer
        return tuple((synth.expert_codes(c, l, t, s, s + 1, shared=True)[0].numpy(),
                      synth.expert_scales(c, l, t, s, s + 1, shared=True)[0].numpy())
                     for t in range(3))


def oracle_rows(cfg, src: ExpertSource, x_bits: np.ndarray, rows):
    """Oracle outputs for the given token rows: (y [n, d], ids, w, gap).

    Tokens run on a thread pool: the C oracle releases the GIL inside ctypes
    calls, and each token is independent."""
    def one(t):
        return oracle.moe_token(cfg.fmt, cfg.k, x_bits[t], src.router_w, src.router_b,
                                src.expert, src.shared, cfg.n_shared)
    rows = list(rows)
    with ThreadPoolExecutor(max_workers=max(1, min(len(rows), os.cpu_count() or 1, 32))) as ex:
        res = list(ex.map(one, rows))
    return (np.array([r[0] for r in res]), np.array([r[1] for r in res]),
            np.array([r[2] for r in res]), np.array([r[3] for r in res]))


def check_rows(cfg, src, x_bits, rows, g_y_bits, g_yf, g_ids, g_w, o=None, report=None, tol16=BF16_TOL):
    """Compare GPU outputs of `rows` (arrays indexed like rows) with the oracle.

    Ids follow the near-tie rule (ids_agree); a token whose set differs at a
    near tie is re-evaluated by the oracle with the GPU's ids; a token whose
    chosen experts come in another order at a near tie is compared weight by
    weight in the GPU's order."""
    oy, oids, ow, ogap = o if o is not None else oracle_rows(cfg, src, x_bits, rows)
    oy = oy.copy()
    ow = ow.copy()
    flips = reorders = 0
    for i, t in enumerate(rows):
        xf = lambda: oracle.router_logits(oracle.bf16_to_f64(x_bits[t]), src.router_w, src.router_b)
        kind = ids_agree(g_ids[i], oids[i], ogap[i], xf)
        if kind == "tie":
            flips += 1
            oy[i], ow[i] = oracle.moe_token_with_ids(cfg.fmt, x_bits[t], g_ids[i], src.router_w,
                                                     src.router_b, src.expert, src.shared,
                                                     cfg.n_shared)
        elif kind == "order":
            reorders += 1
            pos = {int(e): j for j, e in enumerate(oids[i])}
            ow[i] = ow[i][[pos[int(e)] for e in g_ids[i]]]
    assert np.max(np.abs(g_w - ow)) <= W_TOL, np.max(np.abs(g_w - ow))
    e32 = rel_l2(g_yf, oy)
    assert e32 <= F32_TOL, e32
    own_round = oracle.round_bf16(np.asarray(g_yf, dtype=np.float64))
    assert np.array_equal(np.asarray(g_y_bits).view(np.uint16), own_round)
    e16 = rel_l2(bits_to_f64(g_y_bits), bits_to_f64(oracle.round_bf16(oy)))
    assert e16 <= tol16, e16
    if report is not None:
        report.update(rel_l2_f32=e32, rel_l2_bf16=e16, near_tie_flips=flips, near_tie_reorders=reorders)
    return e32, e16, flips


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
