"""The seeded input generator: deterministic, per-expert addressable, and with
the distributions its recipe states."""
import numpy as np
import torch

import synth
from synth.generate import _mix_int


def test_mix32_vector_matches_scalar():
    v = torch.tensor([0, 1, 2, 0xFFFFFFFF, 0x12345678, 0x80000000], dtype=torch.int64)
    got = synth.mix32(v).tolist()
    assert got == [_mix_int(int(a)) for a in v]


def test_codes_deterministic_and_per_expert():
    c = synth.CONFIGS["tiny_d256_e16_q4_t8"]
    a = synth.expert_codes(c, 0, 0, 0, 4)
    b = synth.expert_codes(c, 0, 0, 2, 3)
    assert torch.equal(a[2], b[0])
    assert torch.equal(a, synth.expert_codes(c, 0, 0, 0, 4))
    assert not torch.equal(a[0], a[1])
    assert not torch.equal(a, synth.expert_codes(c, 1, 0, 0, 4))


def test_code_and_scale_distributions():
    c = synth.CONFIGS["verify_48l_q3_t4_zipf"]
    s = synth.expert_scales(c, 0, 2, 0, 8).view(torch.float16).float()
    lo, hi = float(np.float16(0.01)), float(np.float16(0.04))   # bounds as fp16 values
    assert s.min() >= lo and s.max() <= hi
    assert abs(s.mean().item() - 0.025) < 1e-3
    codes = synth.expert_codes(c, 0, 1, 0, 2).flatten().numpy()
    bits = np.unpackbits(codes, bitorder="little").reshape(-1, 96)
    q = bits[:, 0::3] | (bits[:, 1::3] << 1) | (bits[:, 2::3] << 2)
    counts = np.bincount(q.ravel(), minlength=8) / q.size
    assert np.allclose(counts, 1 / 8, atol=2e-3)


def test_router_and_tokens():
    c = synth.CONFIGS["tiny_d256_e16_q4_t8"]
    W = synth.router_weights(c, 0)
    assert W.dtype == np.float32 and W.shape == (16, 256)
    assert abs(W.std() - 0.02) < 1e-3
    x = synth.tokens_bf16(c)
    assert x.shape == (8, 256) and x.dtype == np.uint16
    assert np.array_equal(x, synth.tokens_bf16(c))
    assert synth.router_bias(c, 0) is None


def test_zipf_bias_is_log_prior():
    c = synth.CONFIGS["prefill_1l_q4_t4096_zipf"]
    b = synth.router_bias(c, 0).astype(np.float64)
    assert abs(np.exp(b).sum() - 1.0) < 1e-5
    ranks = np.argsort(-b) + 0
    p = np.sort(np.exp(b))[::-1]
    r = np.arange(1, 513, dtype=np.float64)
    assert np.allclose(p, r ** -1.1 / np.sum(r ** -1.1), rtol=1e-5)
    assert len(set(ranks.tolist())) == 512
