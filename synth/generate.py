"""Seeded, counter-based generators for every input of the MoE FFN layer.

Workloads (sizes as the pages' model has them: 48 layers x 512 experts, top-10
routing plus one always-on shared expert, hidden size 2560; see "Qwen3.8-Flash-
Next at 45 Tokens/sec on a 12GB GPU?", 1:37-2:16, and "Running Qwen3.8-Flash-Next
on a 4090 24GB", section "The engine rejects Unsloth's embedding format" for the
2560 hidden size).  The expert intermediate size, the block formats and the
value distributions are fixed by this library's specification because the
pages do not give them.

Recipe (all reproducible from ``seed``):

* packed codes: uniform random bytes.  A byte holds two uniform 4-bit codes
  (Q4B32) and 12 uniform bytes hold 32 uniform 3-bit codes (Q3B32), so codes are
  uniform on 0..15 / 0..7.  Bytes come from a 32-bit counter hash so that any
  expert of any layer can be regenerated on its own, on the host or on the GPU,
  with identical bits.
* scales: fp16(lo + (hi - lo) * u), u a 24-bit uniform in [0, 1), computed in
  fp32 and rounded to fp16 with round-to-nearest-even.
* router weights: N(0, 0.02) (0.02 is the standard deviation), fp64 normal
  rounded to fp32.
* router bias (Zipf workloads): a seeded permutation gives each expert a rank
  r in 1..E and b = ln(r^-s / sum_j j^-s), s = 1.1, rounded to fp32.
* tokens: N(0, 1), fp64 -> fp32 -> bf16 (both round-to-nearest-even).

The counter hash is the "lowbias32" integer mixer (two xor-shift-multiply
rounds, constants 0x21f0aaad and 0x735a2d97) published by C. Wellons ("Hash
Prospector").  Both constants are below 2**31, so every product of a 32-bit
value and a constant fits a signed 64-bit integer and torch int64 arithmetic
reproduces it exactly on any device.
"""
from __future__ import annotations

import dataclasses
import zlib

import numpy as np
import torch

M32 = 0xFFFFFFFF
_C1 = 0x21F0AAAD
_C2 = 0x735A2D97

# tensor ids inside a layer
T_GATE, T_UP, T_DOWN = 0, 1, 2
_T_CODES, _T_SCALES = 0, 1


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    d: int              # hidden size
    E: int              # routed experts per layer
    I: int              # routed expert intermediate size
    k: int              # experts chosen per token
    n_shared: int       # always-on shared experts (0 or 1)
    I_s: int            # shared expert intermediate size
    L: int              # layers in the stack
    T: int              # tokens per call
    fmt: str            # "q4" (Q4B32), "q3" (Q3B32) or "q2" (Q2B32)
    scale_lo: float
    scale_hi: float
    zipf_s: float | None  # Zipf exponent of the router bias, None = no bias
    seed: int = 0

    @property
    def block_bytes(self) -> int:
        return block_bytes(self.fmt)


def block_bytes(fmt: str) -> int:
    """Bytes of packed codes in one 32-weight block."""
    return {"q4": 16, "q3": 12, "q2": 8}[fmt]


CONFIGS = {
    c.name: c
    for c in [
        LayerConfig("tiny_d256_e16_q4_t8", 256, 16, 128, 2, 1, 128, 1, 8, "q4", 0.005, 0.02, None),
        LayerConfig("decode_48l_q4_t1", 2560, 512, 512, 10, 1, 512, 48, 1, "q4", 0.005, 0.02, None),
        LayerConfig("verify_48l_q3_t4_zipf", 2560, 512, 512, 10, 1, 512, 48, 4, "q3", 0.01, 0.04, 1.1),
        LayerConfig("prefill_1l_q4_t4096_zipf", 2560, 512, 512, 10, 1, 512, 1, 4096, "q4", 0.005, 0.02, 1.1),
        LayerConfig("prefill_48l_q3_t32768", 2560, 512, 512, 10, 1, 512, 48, 32768, "q3", 0.01, 0.04, None),
        # the decode shape in the 2-bit format (the pages' fastest size, Q2_0)
        LayerConfig("decode_48l_q2_t1", 2560, 512, 512, 10, 1, 512, 48, 1, "q2", 0.02, 0.08, None),
    ]
}


def mix32(x: torch.Tensor) -> torch.Tensor:
    """lowbias32 mixer on an int64 tensor holding unsigned 32-bit values."""
    x = x ^ (x >> 16)
    x = (x * _C1) & M32
    x = x ^ (x >> 15)
    x = (x * _C2) & M32
    x = x ^ (x >> 15)
    return x


def _mix_int(v: int) -> int:
    v &= M32
    v ^= v >> 16
    v = (v * _C1) & M32
    v ^= v >> 15
    v = (v * _C2) & M32
    v ^= v >> 15
    return v


def _key(cfg: LayerConfig, *parts: int) -> tuple[int, int]:
    h = _mix_int(cfg.seed ^ 0x9E3779B9)
    h = _mix_int(h ^ zlib.crc32(cfg.name.encode()))
    for p in parts:
        h = _mix_int(h ^ (p & M32))
    return h, _mix_int(h ^ 0x85EBCA6B)


def _rows(cfg: LayerConfig, tensor: int, shared: bool) -> tuple[int, int]:
    """(rows, K) of one expert's gate/up/down matrix."""
    inner = cfg.I_s if shared else cfg.I
    if tensor in (T_GATE, T_UP):
        return inner, cfg.d
    return cfg.d, inner


def _expert_keys(cfg: LayerConfig, layer: int, tensor: int, kind: int, e0: int, e1: int,
                 shared: bool, device) -> tuple[torch.Tensor, torch.Tensor]:
    ks = [_key(cfg, layer, tensor, kind, (1 << 20) + e if shared else e) for e in range(e0, e1)]
    k1 = torch.tensor([a for a, _ in ks], dtype=torch.int64, device=device)
    k2 = torch.tensor([b for _, b in ks], dtype=torch.int64, device=device)
    return k1, k2


def _expert_words(cfg, layer, tensor, kind, e0, e1, n_words, shared, device, chunk_words=1 << 25):
    """Yield (first expert, int64 [n, n_words] words) in bounded-size chunks."""
    k1, k2 = _expert_keys(cfg, layer, tensor, kind, e0, e1, shared, device)
    per = max(1, chunk_words // max(1, n_words))
    i = torch.arange(n_words, dtype=torch.int64, device=device)
    for a in range(0, e1 - e0, per):
        b = min(e1 - e0, a + per)
        w = mix32((mix32(i[None, :] ^ k1[a:b, None]) + k2[a:b, None]) & M32)
        yield a, w


def expert_codes(cfg: LayerConfig, layer: int, tensor: int, e0: int, e1: int,
                 device="cpu", shared: bool = False) -> torch.Tensor:
    """Packed codes of experts [e0, e1) as uint8 [e1-e0, rows, K/32, block_bytes].

    ``shared=True`` addresses the shared expert(s) (index 0..n_shared-1).
    """
    rows, K = _rows(cfg, tensor, shared)
    nb = K // 32
    B = cfg.block_bytes
    n_words = rows * nb * B // 4
    out = torch.empty((e1 - e0, rows * nb * B), dtype=torch.uint8, device=device)
    for a, w in _expert_words(cfg, layer, tensor, _T_CODES, e0, e1, n_words, shared, device):
        n = w.shape[0]
        dst = out[a:a + n].view(n, n_words, 4)
        for j, sh in enumerate((0, 8, 16, 24)):
            dst[:, :, j] = ((w >> sh) & 0xFF).to(torch.uint8)
    return out.view(e1 - e0, rows, nb, B)


def expert_scales(cfg: LayerConfig, layer: int, tensor: int, e0: int, e1: int,
                  device="cpu", shared: bool = False) -> torch.Tensor:
    """fp16 block scales of experts [e0, e1) as int16 bit patterns [e1-e0, rows, K/32]."""
    rows, K = _rows(cfg, tensor, shared)
    nb = K // 32
    out = torch.empty((e1 - e0, rows * nb), dtype=torch.int16, device=device)
    lo = torch.tensor(cfg.scale_lo, dtype=torch.float32, device=device)
    span = torch.tensor(cfg.scale_hi, dtype=torch.float32, device=device) - lo
    for a, w in _expert_words(cfg, layer, tensor, _T_SCALES, e0, e1, rows * nb, shared, device):
        u = (w >> 8).to(torch.float32) * (1.0 / (1 << 24))   # exact: 24-bit integer times 2^-24
        s = (u * span) + lo
        out[a:a + w.shape[0]] = s.to(torch.float16).view(torch.int16)
    return out.view(e1 - e0, rows, nb)


def _np_rng(cfg: LayerConfig, *parts: int) -> np.random.Generator:
    k1, k2 = _key(cfg, *parts)
    return np.random.default_rng([k1, k2])


def router_weights(cfg: LayerConfig, layer: int) -> np.ndarray:
    """fp32 [E, d] router matrix, N(0, 0.02)."""
    rng = _np_rng(cfg, layer, 100)
    return (rng.standard_normal((cfg.E, cfg.d)) * 0.02).astype(np.float32)


def router_bias(cfg: LayerConfig, layer: int) -> np.ndarray | None:
    """fp32 [E] Zipf(s) log-prior over a seeded expert ranking, or None."""
    if cfg.zipf_s is None:
        return None
    rng = _np_rng(cfg, layer, 101)
    ranks = rng.permutation(cfg.E) + 1
    r = np.arange(1, cfg.E + 1, dtype=np.float64)
    norm = np.sum(r ** -cfg.zipf_s)
    return np.log(ranks.astype(np.float64) ** -cfg.zipf_s / norm).astype(np.float32)


def _f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def tokens_bf16(cfg: LayerConfig, T: int | None = None, stream: int = 0) -> np.ndarray:
    """bf16 bit patterns [T, d] of N(0, 1) tokens."""
    T = cfg.T if T is None else T
    rng = _np_rng(cfg, 200, stream)
    return _f32_to_bf16_bits(rng.standard_normal((T, cfg.d)).astype(np.float32))


def layer_weights(cfg: LayerConfig, layer: int, device="cpu") -> dict:
    """Every tensor of one layer in the canonical packed layout.

    Keys: router_w [E,d] f32, router_b [E] f32 or None, codes/scales lists
    (gate, up, down) for routed experts, sh_codes/sh_scales for the shared one.
    Codes are uint8 [E, rows, K/32, B]; scales int16 fp16 bits [E, rows, K/32].
    """
    out = {
        "router_w": router_weights(cfg, layer),
        "router_b": router_bias(cfg, layer),
        "codes": [expert_codes(cfg, layer, t, 0, cfg.E, device) for t in (T_GATE, T_UP, T_DOWN)],
        "scales": [expert_scales(cfg, layer, t, 0, cfg.E, device) for t in (T_GATE, T_UP, T_DOWN)],
        "sh_codes": [expert_codes(cfg, layer, t, 0, cfg.n_shared, device, shared=True) for t in (T_GATE, T_UP, T_DOWN)],
        "sh_scales": [expert_scales(cfg, layer, t, 0, cfg.n_shared, device, shared=True) for t in (T_GATE, T_UP, T_DOWN)],
    }
    return out
