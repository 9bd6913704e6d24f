"""GPU parity of the 48-layer stacks, teacher-forced: every layer's recorded
bf16 input (the GPU's own) is fed to the oracle, whose output, ids and
weights are compared with the GPU's record of that layer; the residual chain
between layers is checked separately."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import (W_TOL, ExpertSource, HostLayer, bf16_tol, bits_to_f64, check_rows, ids_agree,
                          oracle_routing, oracle_rows_dense, to_np)

pytestmark = pytest.mark.gpu


def _stack(name, rows=None, check_layers=None, dense=False, layer0_all=False, flags=0):
    """The whole stack through the C ABI with per-layer records of `rows` (all
    when None), checked layer by layer against the oracle (teacher-forced).
    dense: the oracle evaluates each layer's rows with per-expert fp64 matrix
    products over a host copy of that layer.  layer0_all: also route every
    token of layer 0 (its recorded input) and check every token's ids and
    weights against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_expert_ffn_token_b200 import capi, session
    cfg = synth.CONFIGS[name] if isinstance(name, str) else name
    L, T, d, k = cfg.L, cfg.T, cfg.d, cfg.k
    sess = session.Session(cfg, max_tokens=T, flags=flags)
    sess.load_synthetic()
    x_bits = synth.tokens_bf16(cfg)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    n_rec = T if rows is None else len(rows)
    dev = "cuda"
    xr = torch.empty((L, n_rec, d), dtype=torch.int16, device=dev)
    yr = torch.empty((L, n_rec, d), dtype=torch.int16, device=dev)
    yfr = torch.empty((L, n_rec, d), dtype=torch.float32, device=dev)
    idr = torch.empty((L, n_rec, k), dtype=torch.int32, device=dev)
    wr = torch.empty((L, n_rec, k), dtype=torch.float32, device=dev)
    rows_t = None if rows is None else torch.tensor(rows, dtype=torch.int32, device=dev)
    rec = capi.make_record(xr, yr, yfr, idr, wr, rows_t)
    r_out = torch.empty((T, d), dtype=torch.float32, device=dev)
    capi.moe_forward_stack(sess.ctx, 0, L, x, T, r_out, rec)
    torch.cuda.synchronize()
    assert capi.moe_get_device_error(sess.ctx) == 0
    all0 = None
    if layer0_all:
        x0 = torch.empty((1, T, d), dtype=torch.int16, device=dev)
        id0 = torch.empty((1, T, k), dtype=torch.int32, device=dev)
        w0 = torch.empty((1, T, k), dtype=torch.float32, device=dev)
        r1 = torch.empty((T, d), dtype=torch.float32, device=dev)
        capi.moe_forward_stack(sess.ctx, 0, 1, x, T, r1, capi.make_record(x=x0, ids=id0, w=w0))
        torch.cuda.synchronize()
        all0 = (to_np(x0[0]), to_np(id0[0]), to_np(w0[0]))
        del x0, id0, w0, r1
    sess.close()
    xr, yr, yfr, idr, wr, r_out = map(to_np, (xr, yr, yfr, idr, wr, r_out))
    rows = list(range(T)) if rows is None else list(rows)

    # residual chain: r_0 = x, x_l = bf16(rmsnorm(r_l)), r_{l+1} = r_l + y_l
    r = bits_to_f64(x_bits[rows])
    for l in range(L):
        want = np.array([oracle.rmsnorm(ri, 1e-6) for ri in r])
        got = bits_to_f64(xr[l])
        ulp = np.abs(bits_to_f64(oracle.round_bf16(want))) * 2.0 ** -7 + 1e-30
        assert np.all(np.abs(got - want) <= ulp), f"layer {l}: stack input off by more than 1 ulp"
        r = r + bits_to_f64(yr[l])
    assert np.allclose(r_out[rows], r, rtol=1e-5, atol=1e-5 * np.abs(r).max())

    worst = {}
    for l in (range(L) if check_layers is None else check_layers):
        src = HostLayer(cfg, l) if dense else ExpertSource(cfg, l)
        rep = {}
        idx = list(range(len(rows)))
        o = oracle_rows_dense(cfg, src, xr[l], idx) if dense else None
        check_rows(cfg, src, xr[l], idx, yr[l], yfr[l], idr[l], wr[l], o=o, report=rep, tol16=bf16_tol(T))
        worst[l] = rep
        if l == 0 and all0 is not None:
            # every token of layer 0: the recorded input of a sampled row is the same row of the
            # all-token record, and every token's routing matches the oracle
            xa, ida, wa = all0
            assert np.array_equal(xa[rows], xr[0])
            oids, ow, ogap, olg = oracle_routing(cfg, src, xa)
            flips = 0
            for t in range(T):
                kind = ids_agree(ida[t], oids[t], ogap[t], lambda: olg[t])
                if kind == "same":
                    assert np.max(np.abs(wa[t] - ow[t])) <= W_TOL
                flips += kind != "same"
            worst["layer0_all_tokens_not_identical"] = flips
        del src
    return worst


def test_decode_stack_48_layers():
    _stack("decode_48l_q4_t1")


def test_verify_stack_48_layers():
    _stack("verify_48l_q3_t4_zipf")


def test_split_kernel_stack_48_layers():
    """The 48-layer Q4 decode stack through the split single-token kernel (MOE_FLAG_SPLIT_DECODE)."""
    from quantized_expert_ffn_token_b200 import capi
    _stack("decode_48l_q4_t1", flags=capi.MOE_FLAG_SPLIT_DECODE)


def test_few_token_stack_48_layers_13_tokens():
    """Thirteen tokens through the 48-layer Q4 stack: two launches of the
    few-token kernel (7 + 6 tokens), every token's record of every layer
    against the oracle."""
    import dataclasses
    _stack(dataclasses.replace(synth.CONFIGS["decode_48l_q4_t1"], T=13))


@pytest.mark.slow
def test_long_prefill_stack_48_layers_sampled():
    """The long-prefill stack (32768 tokens, 48 layers, Q3B32): a seeded sample
    of 256 tokens checked in every one of the 48 layers, plus the routing of
    every token in layer 0."""
    T = synth.CONFIGS["prefill_48l_q3_t32768"].T
    rows = sorted(np.random.default_rng(2026).choice(T, size=256, replace=False).tolist())
    _stack("prefill_48l_q3_t32768", rows=rows, dense=True, layer0_all=True)
