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
    """Compare GPU outputs of `rows` (arrays indexed like rows) with the oracle."""
    oy, oids, ow, ogap = o if o is not None else oracle_rows(cfg, src, x_bits, rows)
    oy = oy.copy()
    ow = ow.copy()
    flips = 0
    for i, t in enumerate(rows):
        if not np.array_equal(g_ids[i], oids[i]):
            assert ogap[i] < NEAR_TIE, (
                f"token {t}: ids {g_ids[i].tolist()} != oracle {oids[i].tolist()} "
                f"(10th-11th gap {ogap[i]:.3g})")
            flips += 1
            oy[i], ow[i] = oracle.moe_token_with_ids(cfg.fmt, x_bits[t], g_ids[i], src.router_w,
                                                     src.router_b, src.expert, src.shared,
                                                     cfg.n_shared)
    assert np.max(np.abs(g_w - ow)) <= W_TOL, np.max(np.abs(g_w - ow))
    e32 = rel_l2(g_yf, oy)
    assert e32 <= F32_TOL, e32
    own_round = oracle.round_bf16(np.asarray(g_yf, dtype=np.float64))
    assert np.array_equal(np.asarray(g_y_bits).view(np.uint16), own_round)
    e16 = rel_l2(bits_to_f64(g_y_bits), bits_to_f64(oracle.round_bf16(oy)))
    assert e16 <= tol16, e16
    if report is not None:
        report.update(rel_l2_f32=e32, rel_l2_bf16=e16, near_tie_flips=flips)
    return e32, e16, flips


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
