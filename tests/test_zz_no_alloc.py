"""The allocation-free routing entry point (moe_route_static).

It is meant for callers that cannot allocate device memory; it keeps its
logits in a fixed device array.  Checked here through the C ABI against the
routing that moe_forward reports on the same tokens and router weights, on
two calls in a row (the fixed array keeps the previous call's contents), and
for its size limit.  This file is collected last so that a failure here does
not hide the rest of the suite.
"""
import numpy as np
import pytest
import torch

import synth
from tests.parity import W_TOL

pytestmark = pytest.mark.gpu


def _libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_expert_ffn_token_b200 import capi, session
    return capi, session


@pytest.mark.parametrize("name,T", [("tiny_d256_e16_q4_t8", 8), ("verify_48l_q3_t4_zipf", 4),
                                    ("prefill_1l_q4_t4096_zipf", 64)])
def test_route_static_matches_forward_twice(name, T):
    capi, session = _libs()
    cfg = synth.CONFIGS[name]
    sess = session.Session(cfg, max_tokens=T, n_layers=1)
    sess.load_synthetic(layers=[0])
    x = torch.from_numpy(synth.tokens_bf16(cfg, T, stream=3).view(np.int16)).cuda()
    _, _, ids_ref, w_ref = sess.forward(0, x)
    torch.cuda.synchronize()
    sess.close()
    rw = torch.from_numpy(synth.router_weights(cfg, 0)).cuda()
    b = synth.router_bias(cfg, 0)
    rb = None if b is None else torch.from_numpy(b).cuda()
    for _ in range(2):
        ids = torch.full((T, cfg.k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, cfg.k), -1.0, dtype=torch.float32, device="cuda")
        capi.moe_route_static(x, T, cfg.d, rw, rb, cfg.E, cfg.k, ids, w)
        torch.cuda.synchronize()
        assert torch.equal(ids, ids_ref)
        assert float((w - w_ref).abs().max()) <= W_TOL


def test_route_static_rejects_oversize():
    capi, _ = _libs()
    E, d, k = 512, 256, 10
    T = capi.MOE_ROUTE_STATIC_MAX_LOGITS // E + 1
    x = torch.zeros((T, d), dtype=torch.int16, device="cuda")
    rw = torch.zeros((E, d), dtype=torch.float32, device="cuda")
    ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    with pytest.raises(capi.MoeError) as e:
        capi.moe_route_static(x, T, d, rw, None, E, k, ids, w)
    assert e.value.status == capi.MOE_ERR_TOO_MANY_TOKENS
    assert "MOE_ROUTE_STATIC_MAX_LOGITS" in capi.last_error()
