"""The allocation-free routing entry point (moe_route_static).

It serves callers that cannot allocate device memory (code inside another
runtime's memory pool, services that fix their device memory at start-up,
plain C hosts that only receive device pointers); it keeps its logits in a
fixed device array.  Checked here through the C ABI, on two calls in a row
(the fixed array keeps the previous call's contents):

* against the oracle's routing, under the near-tie rule of every other
  routing check, and against the routing that moe_forward reports on the same
  tokens and router weights (ids wherever both agree with the oracle, weights
  within the same 1e-5);
* that the calls leave the device's free memory unchanged;
* its argument checks (size limit, misaligned router rows, hidden size), which
  all return before any work reaches the GPU.

This file is collected last so that a failure here does not hide the rest of
the suite.
"""
import numpy as np
import pytest
import torch

import synth
from tests.parity import W_TOL, ExpertSource, ids_agree, oracle_routing

pytestmark = pytest.mark.gpu


def _libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_expert_ffn_token_b200 import capi, session
    return capi, session


@pytest.mark.parametrize("name,T", [("tiny_d256_e16_q4_t8", 8), ("verify_48l_q3_t4_zipf", 4),
                                    ("prefill_1l_q4_t4096_zipf", 64)])
def test_route_static_matches_oracle_and_forward_twice(name, T):
    capi, session = _libs()
    cfg = synth.CONFIGS[name]
    sess = session.Session(cfg, max_tokens=T, n_layers=1)
    sess.load_synthetic(layers=[0])
    x_bits = synth.tokens_bf16(cfg, T, stream=3)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    _, _, ids_fwd, w_fwd = sess.forward(0, x)
    torch.cuda.synchronize()
    sess.close()
    ids_fwd, w_fwd = ids_fwd.cpu().numpy(), w_fwd.cpu().numpy()
    src = ExpertSource(cfg, 0)
    oids, ow, ogap, olg = oracle_routing(cfg, src, x_bits)
    rw = torch.from_numpy(synth.router_weights(cfg, 0)).cuda()
    b = synth.router_bias(cfg, 0)
    rb = None if b is None else torch.from_numpy(b).cuda()
    for _ in range(2):
        ids = torch.full((T, cfg.k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, cfg.k), -1.0, dtype=torch.float32, device="cuda")
        capi.moe_route_static(x, T, cfg.d, rw, rb, cfg.E, cfg.k, ids, w)
        torch.cuda.synchronize()
        ids, w = ids.cpu().numpy(), w.cpu().numpy()
        for t in range(T):
            kind = ids_agree(ids[t], oids[t], ogap[t], lambda: olg[t])
            if kind == "same":
                assert np.max(np.abs(w[t] - ow[t])) <= W_TOL
                if np.array_equal(ids_fwd[t], oids[t]):   # moe_forward agrees with the oracle too
                    assert np.max(np.abs(w[t] - w_fwd[t])) <= W_TOL


def test_route_static_allocates_nothing():
    """After a first call (which loads the library's code and looks up the fixed
    array), further calls leave the device's free memory as it was."""
    capi, _ = _libs()
    cfg = synth.CONFIGS["verify_48l_q3_t4_zipf"]
    T = 16
    x = torch.from_numpy(synth.tokens_bf16(cfg, T, stream=5).view(np.int16)).cuda()
    rw = torch.from_numpy(synth.router_weights(cfg, 0)).cuda()
    rb = torch.from_numpy(synth.router_bias(cfg, 0)).cuda()
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    capi.moe_route_static(x, T, cfg.d, rw, rb, cfg.E, cfg.k, ids, w)
    capi.moe_route_static(x, T, cfg.d, rw, None, cfg.E, cfg.k, ids, w)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        capi.moe_route_static(x, T, cfg.d, rw, rb, cfg.E, cfg.k, ids, w)
        capi.moe_route_static(x, T, cfg.d, rw, None, cfg.E, cfg.k, ids, w)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_route_static_rejects_bad_arguments():
    capi, _ = _libs()
    E, d, k = 512, 256, 10
    T = capi.MOE_ROUTE_STATIC_MAX_LOGITS // E + 1
    x = torch.zeros((T, d), dtype=torch.int16, device="cuda")
    rw = torch.zeros((E * d + 4,), dtype=torch.float32, device="cuda")
    ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    with pytest.raises(capi.MoeError) as e:
        capi.moe_route_static(x, T, d, rw, None, E, k, ids, w)
    assert e.value.status == capi.MOE_ERR_TOO_MANY_TOKENS
    assert "MOE_ROUTE_STATIC_MAX_LOGITS" in capi.last_error()
    # router rows one float past a 16-byte boundary
    with pytest.raises(capi.MoeError) as e:
        capi.moe_route_static(x, 4, d, rw.data_ptr() + 4, None, E, k, ids, w)
    assert e.value.status == capi.MOE_ERR_INVALID_ARG
    for dd in (16384 + 4, 258):   # above the largest hidden size; not a multiple of 4
        with pytest.raises(capi.MoeError) as e:
            capi.moe_route_static(x, 1, dd, rw, None, E, k, ids, w)
        assert e.value.status == capi.MOE_ERR_INVALID_ARG
