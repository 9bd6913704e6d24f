"""GPU parity of one MoE layer through the C ABI against the oracle, plus the
edge cases and error codes of the boundary."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import (ExpertSource, HostLayer, W_TOL, bf16_tol, check_rows, ids_agree, oracle_routing,
                          oracle_rows_dense, rel_l2, to_np)

pytestmark = pytest.mark.gpu

TINY = synth.CONFIGS["tiny_d256_e16_q4_t8"]
TINY_Q3 = dataclasses.replace(TINY, name="tiny_d256_e16_q3_t8", fmt="q3")
TINY_Q2 = dataclasses.replace(TINY, name="tiny_d256_e16_q2_t8", fmt="q2", scale_lo=0.02, scale_hi=0.08)
DECODE_Q2 = synth.CONFIGS["decode_48l_q2_t1"]


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_expert_ffn_token_b200 import capi, session
    return capi, session


def _tokens(cfg, T, stream=0):
    return synth.tokens_bf16(cfg, T, stream)


def _run(sess, layer, x_bits):
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    y, yf, ids, w = sess.forward(layer, x)
    torch.cuda.synchronize()
    return to_np(y), to_np(yf), to_np(ids), to_np(w)


def test_generator_bits_identical_on_device():
    _cuda()
    c = synth.CONFIGS["verify_48l_q3_t4_zipf"]
    for t in range(3):
        a = synth.expert_codes(c, 3, t, 100, 102, device="cuda").cpu()
        b = synth.expert_codes(c, 3, t, 100, 102)
        assert torch.equal(a, b)
        a = synth.expert_scales(c, 3, t, 7, 8, device="cuda").cpu()
        assert torch.equal(a, synth.expert_scales(c, 3, t, 7, 8))


@pytest.mark.parametrize("fmt", ["q4", "q3", "q2"])
def test_tiny_layer_all_tokens(fmt):
    capi, session = _cuda()
    import dataclasses
    cfg = {"q4": TINY, "q3": dataclasses.replace(TINY, fmt=fmt, name=TINY.name + fmt), "q2": TINY_Q2}[fmt]
    sess = session.Session(cfg, max_tokens=256)
    sess.load_synthetic()
    x = _tokens(cfg, cfg.T)
    gy, gyf, gids, gw = _run(sess, 0, x)
    W = synth.layer_weights(cfg, 0)
    oy, oids, ow, ogap = oracle.moe_layer(cfg.fmt, cfg.k, x, W)
    src = ExpertSource(cfg, 0)
    check_rows(cfg, src, x, list(range(cfg.T)), gy, gyf, gids, gw, o=(oy, oids, ow, ogap))
    sess.close()


@pytest.mark.parametrize("T", list(range(1, 18)) + [63, 64, 127, 128, 129])
def test_tiny_ragged_token_counts(T):
    capi, session = _cuda()
    sess = session.Session(TINY, max_tokens=256)
    sess.load_synthetic()
    x = _tokens(TINY, T, stream=T)
    gy, gyf, gids, gw = _run(sess, 0, x)
    W = synth.layer_weights(TINY, 0)
    o = oracle.moe_layer(TINY.fmt, TINY.k, x, W)
    check_rows(TINY, ExpertSource(TINY, 0), x, list(range(T)), gy, gyf, gids, gw, o=o, tol16=bf16_tol(T))
    sess.close()


@pytest.mark.parametrize("fmt,T", [("q3", 2), ("q3", 7), ("q3", 12), ("q2", 3), ("q2", 8), ("q2", 16)])
def test_few_token_kernel_other_formats(fmt, T):
    """The few-token kernel (2..16 tokens, up to eight per launch) on Q3B32 and
    Q2B32 against the oracle, every token."""
    capi, session = _cuda()
    cfg = TINY_Q3 if fmt == "q3" else TINY_Q2
    sess = session.Session(cfg, max_tokens=16)
    sess.load_synthetic()
    x = _tokens(cfg, T, stream=100 + T)
    gy, gyf, gids, gw = _run(sess, 0, x)
    o = oracle.moe_layer(cfg.fmt, cfg.k, x, synth.layer_weights(cfg, 0))
    check_rows(cfg, ExpertSource(cfg, 0), x, list(range(T)), gy, gyf, gids, gw, o=o)
    sess.close()


@pytest.mark.parametrize("name,T", [("tiny_d256_e16_q4_t8", 6), ("verify_48l_q3_t4_zipf", 4),
                                    ("decode_48l_q4_t1", 8), ("decode_q2", 5)])
def test_few_token_kernel_matches_single_token_kernel(name, T):
    """A batch through the few-token kernel against the same tokens one at a
    time through the single-token kernel (both exact-operand paths whose
    per-block offset removal leaves about 2^-16 relative per partial): same
    ids, weights within 1e-6, fp32 outputs within 1e-4 relative L2."""
    capi, session = _cuda()
    cfg = {"decode_q2": DECODE_Q2}.get(name) or synth.CONFIGS[name]
    a = session.Session(cfg, max_tokens=16, n_layers=1)
    b = session.Session(cfg, max_tokens=16, n_layers=1, flags=capi.MOE_FLAG_NO_MULTI_DECODE)
    W = synth.layer_weights(cfg, 0, device="cuda")
    a.load(0, W)
    b.load(0, W)
    del W
    x = _tokens(cfg, T, stream=55)
    ya, yfa, ida, wa = _run(a, 0, x)
    yb, yfb, idb, wb = _run(b, 0, x)
    assert capi.moe_get_device_error(a.ctx) == 0
    assert np.array_equal(ida, idb)
    assert np.max(np.abs(wa - wb)) <= 1e-6
    assert rel_l2(yfa, yfb) <= 1e-4
    a.close()
    b.close()


@pytest.mark.parametrize("name,T", [("decode_48l_q4_t1", 8), ("decode_48l_q4_t1", 13), ("verify_48l_q3_t4_zipf", 16)])
def test_few_token_full_size(name, T):
    """Full-size layers through the few-token kernel (one launch of eight, two
    launches for 13 and 16 tokens), every token against the oracle."""
    capi, session = _cuda()
    cfg = synth.CONFIGS[name]
    sess = session.Session(cfg, max_tokens=T, n_layers=1)
    sess.load_synthetic(layers=[0])
    x = _tokens(cfg, T, stream=900 + T)
    gy, gyf, gids, gw = _run(sess, 0, x)
    assert capi.moe_get_device_error(sess.ctx) == 0
    sess.close()
    src = HostLayer(cfg, 0)
    rows = list(range(T))
    check_rows(cfg, src, x, rows, gy, gyf, gids, gw, o=oracle_rows_dense(cfg, src, x, rows))


def test_few_token_wait_times_out_and_context_recovers():
    """The bounded waits of the few-token kernel: with the test hook its CTA 0
    withholds its logits in the context's first call, every wait gives up,
    MOE_ERR_DEVICE_TIMEOUT is reported, and the next calls are correct."""
    capi, session = _cuda()
    s = session.Session(TINY, max_tokens=8, n_layers=1, flags=capi.MOE_FLAG_TEST_WITHHOLD)
    s.load_synthetic()
    x = _tokens(TINY, 5, stream=78)
    _run(s, 0, x)
    assert capi.moe_get_device_error(s.ctx) == capi.MOE_ERR_DEVICE_TIMEOUT
    o = oracle.moe_layer(TINY.fmt, TINY.k, x, synth.layer_weights(TINY, 0))
    for rep in range(2):
        gy, gyf, gids, gw = _run(s, 0, x)
        assert capi.moe_get_device_error(s.ctx) == 0
        check_rows(TINY, ExpertSource(TINY, 0), x, list(range(5)), gy, gyf, gids, gw, o=o)
    s.close()


@pytest.mark.parametrize("fmt", ["q4", "q3", "q2"])
def test_split_kernel_tiny_against_oracle(fmt):
    """The split single-token kernel (one-token contexts with MOE_FLAG_SPLIT_DECODE: gate/up and the
    matching slice of the down projection per 16-row unit, the shared expert during the logits
    exchange): several single tokens against the oracle."""
    capi, session = _cuda()
    cfg = {"q4": TINY, "q3": TINY_Q3, "q2": TINY_Q2}[fmt]
    sess = session.Session(cfg, max_tokens=1, flags=capi.MOE_FLAG_SPLIT_DECODE)
    sess.load_synthetic()
    W = synth.layer_weights(cfg, 0)
    for s in range(6):
        x = _tokens(cfg, 1, stream=300 + s)
        gy, gyf, gids, gw = _run(sess, 0, x)
        assert capi.moe_get_device_error(sess.ctx) == 0
        o = oracle.moe_layer(cfg.fmt, cfg.k, x, W)
        check_rows(cfg, ExpertSource(cfg, 0), x, [0], gy, gyf, gids, gw, o=o)
    sess.close()


@pytest.mark.parametrize("name", ["decode_48l_q4_t1", "verify_48l_q3_t4_zipf", "decode_q2"])
def test_split_kernel_matches_single_token_kernel(name):
    """The split kernel against the default single-token kernel (two one-token contexts): same ids,
    weights within 1e-6, fp32 outputs within 5e-5 (1e-4 for Q2B32) relative L2 (both remove the code
    offset per block in fp32)."""
    capi, session = _cuda()
    cfg = {"decode_q2": DECODE_Q2}.get(name) or synth.CONFIGS[name]
    a = session.Session(cfg, max_tokens=1, n_layers=1, flags=capi.MOE_FLAG_SPLIT_DECODE)
    b = session.Session(cfg, max_tokens=1, n_layers=1)
    W = synth.layer_weights(cfg, 0, device="cuda")
    a.load(0, W)
    b.load(0, W)
    del W
    for s in range(4):
        x = _tokens(cfg, 1, stream=600 + s)
        ya, yfa, ida, wa = _run(a, 0, x)
        yb, yfb, idb, wb = _run(b, 0, x)
        assert capi.moe_get_device_error(a.ctx) == 0
        assert np.array_equal(ida, idb)
        assert np.max(np.abs(wa - wb)) <= 1e-6
        assert rel_l2(yfa, yfb) <= (1e-4 if cfg.fmt == "q2" else 5e-5)
    a.close()
    b.close()


def test_split_wait_times_out_and_context_recovers():
    """The split kernel's bounded waits: CTA 0 withholds its logits in the context's first call,
    the waits give up, MOE_ERR_DEVICE_TIMEOUT is reported, and later calls are correct."""
    capi, session = _cuda()
    s = session.Session(TINY, max_tokens=1, n_layers=1,
                        flags=capi.MOE_FLAG_TEST_WITHHOLD | capi.MOE_FLAG_SPLIT_DECODE)
    s.load_synthetic()
    x = _tokens(TINY, 1, stream=79)
    _run(s, 0, x)
    assert capi.moe_get_device_error(s.ctx) == capi.MOE_ERR_DEVICE_TIMEOUT
    o = oracle.moe_layer(TINY.fmt, TINY.k, x, synth.layer_weights(TINY, 0))
    for rep in range(2):
        gy, gyf, gids, gw = _run(s, 0, x)
        assert capi.moe_get_device_error(s.ctx) == 0
        check_rows(TINY, ExpertSource(TINY, 0), x, [0], gy, gyf, gids, gw, o=o)
    s.close()


def test_batch_equals_single_tokens():
    """Token independence of the CUDA-core grouped path: a token's output does not
    depend on which other tokens share the call (bit for bit).  Pinned to that
    path: small calls would otherwise run the single-token kernel and larger ones
    the tensor cores, whose fp32 atomics sum in no fixed order."""
    capi, session = _cuda()
    sess = session.Session(TINY, max_tokens=64,
                           flags=capi.MOE_FLAG_NO_DECODE_KERNEL | capi.MOE_FLAG_NO_TENSOR_PREFILL)
    sess.load_synthetic()
    x = _tokens(TINY, 37, stream=5)
    gy, gyf, gids, gw = _run(sess, 0, x)
    for t in range(37):
        pair = x[[t, (t + 11) % 37]]
        y2, yf2, ids2, w2 = _run(sess, 0, pair)
        assert np.array_equal(ids2[0], gids[t])
        assert np.array_equal(y2[0], gy[t])
        assert np.array_equal(yf2[0], gyf[t])
    sess.close()


@pytest.mark.parametrize("name", ["tiny_d256_e16_q4_t8", "tiny_q3", "tiny_q2", "decode_48l_q4_t1",
                                  "verify_48l_q3_t4_zipf", "decode_q2"])
def test_decode_kernel_matches_general_path(name):
    """Single-token calls: the persistent decode kernel against the general
    grouped path on the same inputs (same ids; fp32 outputs within 5e-5, 1e-4
    for Q2B32).

    The decode kernel reads Q4 codes as fp16 1024 + q and removes 1032 x the
    block sum of the input from each fp32 block partial afterwards; that
    cancellation leaves about 2^-16 of relative error per partial (the offset
    term is ~2^8 times the useful one), so the two paths agree to a few 1e-5,
    not to fp32 rounding.  Q2B32 reads a quarter of its codes as 1024 + q with
    |q - 2| <= 2, one bit more cancellation (~2^-14 per partial on those, much
    less on the 4q, 16q and 64q places): about 3e-5 over the output, so the
    bound is doubled."""
    capi, session = _cuda()
    cfg = {"tiny_q3": TINY_Q3, "tiny_q2": TINY_Q2, "decode_q2": DECODE_Q2}.get(name) or synth.CONFIGS[name]
    a = session.Session(cfg, max_tokens=4, n_layers=1)
    b = session.Session(cfg, max_tokens=4, n_layers=1, flags=capi.MOE_FLAG_NO_DECODE_KERNEL)
    W = synth.layer_weights(cfg, 0, device="cuda")
    a.load(0, W)
    b.load(0, W)
    del W
    for s in range(4):
        x = _tokens(cfg, 1, stream=40 + s)
        ya, yfa, ida, wa = _run(a, 0, x)
        yb, yfb, idb, wb = _run(b, 0, x)
        assert np.array_equal(ida, idb)
        assert np.max(np.abs(wa - wb)) <= 1e-6
        assert rel_l2(yfa, yfb) <= (1e-4 if cfg.fmt == "q2" else 5e-5)
    a.close()
    b.close()


def test_decode_wait_times_out_and_context_recovers():
    """A bounded device wait that runs out, and recovery: with the test hook,
    CTA 0 of the single-token kernel withholds its router logits in the
    context's first call, every CTA's wait on them gives up after about a
    second, moe_get_device_error reports MOE_ERR_DEVICE_TIMEOUT (and resets the
    kernel's arrival counters), and the next call on the same context matches
    the general path again."""
    capi, session = _cuda()
    s = session.Session(TINY, max_tokens=4, n_layers=1, flags=capi.MOE_FLAG_TEST_WITHHOLD)
    ref = session.Session(TINY, max_tokens=4, n_layers=1, flags=capi.MOE_FLAG_NO_DECODE_KERNEL)
    W = synth.layer_weights(TINY, 0, device="cuda")
    s.load(0, W)
    ref.load(0, W)
    del W
    x = _tokens(TINY, 1, stream=77)
    _run(s, 0, x)
    assert capi.moe_get_device_error(s.ctx) == capi.MOE_ERR_DEVICE_TIMEOUT
    for rep in range(3):
        y, yf, ids, w = _run(s, 0, x)
        assert capi.moe_get_device_error(s.ctx) == 0
        yb, yfb, idb, wb = _run(ref, 0, x)
        assert np.array_equal(ids, idb)
        assert rel_l2(yf, yfb) <= 5e-5
    s.close()
    ref.close()


def test_tensor_core_wait_times_out_and_context_recovers():
    """The tensor-core path's bounded waits: with the test hook, CTA 0 of the
    context's first gate/up GEMM never signals its first accumulator as full,
    its epilogue's wait gives up after about two seconds, the call reports
    MOE_ERR_DEVICE_TIMEOUT (the MMAs in flight are drained before the CTA frees
    its tensor memory), and the next calls on the same context match a context
    without the hook."""
    capi, session = _cuda()
    T = 64
    s = session.Session(TINY, max_tokens=T, n_layers=1, flags=capi.MOE_FLAG_TEST_WITHHOLD)
    ref = session.Session(TINY, max_tokens=T, n_layers=1)
    W = synth.layer_weights(TINY, 0, device="cuda")
    s.load(0, W)
    ref.load(0, W)
    del W
    x = _tokens(TINY, T, stream=78)
    _run(s, 0, x)
    assert capi.moe_get_device_error(s.ctx) == capi.MOE_ERR_DEVICE_TIMEOUT
    yb, yfb, idb, wb = _run(ref, 0, x)
    for rep in range(3):
        y, yf, ids, w = _run(s, 0, x)
        assert capi.moe_get_device_error(s.ctx) == 0
        assert np.array_equal(ids, idb)
        assert rel_l2(yf, yfb) <= 1e-5
    s.close()
    ref.close()


@pytest.mark.parametrize("T", [1, 4])
def test_l2_policy_leaves_results_unchanged(T):
    """The decode kernels' L2 eviction priorities change where the weights are
    cached, never what is computed: a two-layer stack gives the same residual
    stream under both modes (bit for bit for one token, whose kernel sums in a
    fixed order; for several tokens the few-token kernel's fp32 atomics sum in
    no fixed order, so two runs in the same mode differ too, and the bound is
    the one its tests use against the single-token kernel)."""
    capi, session = _cuda()
    cfg = synth.CONFIGS["verify_48l_q3_t4_zipf"]
    s = session.Session(cfg, max_tokens=max(T, 2), n_layers=2)
    s.load_synthetic()
    x = torch.from_numpy(_tokens(cfg, T, stream=91).view(np.int16)).cuda()
    outs = []
    for mode in (capi.MOE_L2_STREAM, capi.MOE_L2_KEEP_SHARED, capi.MOE_L2_KEEP_SHARED):
        capi.moe_set_l2_policy(s.ctx, mode)
        r = torch.empty((T, cfg.d), dtype=torch.float32, device="cuda")
        capi.moe_forward_stack(s.ctx, 0, 2, x, T, r)
        torch.cuda.synchronize()
        assert capi.moe_get_device_error(s.ctx) == 0
        outs.append(to_np(r))
    for o in outs[1:]:
        if T == 1:
            assert np.array_equal(o, outs[0])
        else:
            assert rel_l2(o, outs[0]) <= 1e-4
    with pytest.raises(capi.MoeError):
        capi.moe_set_l2_policy(s.ctx, 7)
    s.close()


def _tiny_weights_with(mutate):
    W = synth.layer_weights(TINY, 0, device="cuda")
    mutate(W)
    return W


def test_skew_every_token_to_the_same_experts():
    capi, session = _cuda()
    sess = session.Session(TINY, max_tokens=256)
    bias = np.full(TINY.E, -30.0, dtype=np.float32)
    bias[5], bias[11] = 30.0, 29.0

    def mut(W):
        W["router_b"] = bias
    W = _tiny_weights_with(mut)
    sess.load(0, W)
    x = _tokens(TINY, 200, stream=9)
    gy, gyf, gids, gw = _run(sess, 0, x)
    assert all(set(r.tolist()) == {5, 11} for r in gids)
    Wh = synth.layer_weights(TINY, 0)
    Wh["router_b"] = bias
    o = oracle.moe_layer(TINY.fmt, TINY.k, x, Wh)
    src = ExpertSource(TINY, 0)
    src.router_b = bias
    check_rows(TINY, src, x, list(range(200)), gy, gyf, gids, gw, o=o, tol16=bf16_tol(200))
    sess.close()


def test_zero_scale_routed_experts_leave_only_shared():
    """With every routed expert's scales zeroed the layer is the shared expert
    alone.  A routed expert that still contributed would move the output by
    O(1) relative; the bound 5e-5 covers the single-token kernel's arithmetic
    (the per-block offset removal leaves ~2^-16 relative per block partial)."""
    capi, session = _cuda()
    sess = session.Session(TINY, max_tokens=16)

    def mut(W):
        for t in range(3):
            W["scales"][t].zero_()
    sess.load(0, _tiny_weights_with(mut))
    x = _tokens(TINY, 8)
    gy, gyf, gids, gw = _run(sess, 0, x)
    Wh = synth.layer_weights(TINY, 0)
    xf = oracle.bf16_to_f64(x)
    sh = tuple((Wh["sh_codes"][t][0].numpy(), Wh["sh_scales"][t][0].numpy()) for t in range(3))
    want = np.array([oracle.expert("q4", *sh, xf[t]) for t in range(8)])
    assert rel_l2(gyf, want) <= 5e-5
    sess.close()


def test_boundary_errors_and_noop():
    capi, session = _cuda()
    sess = session.Session(TINY, max_tokens=16, n_layers=2)
    sess.load_synthetic(layers=[0])
    x = torch.zeros((17, TINY.d), dtype=torch.int16, device="cuda")
    y = torch.zeros((17, TINY.d), dtype=torch.int16, device="cuda")
    with pytest.raises(capi.MoeError) as e:
        capi.moe_forward(sess.ctx, 0, x, 17, y)
    assert e.value.status == capi.MOE_ERR_TOO_MANY_TOKENS
    with pytest.raises(capi.MoeError) as e:
        capi.moe_forward(sess.ctx, 1, x, 4, y)
    assert e.value.status == capi.MOE_ERR_NOT_LOADED
    with pytest.raises(capi.MoeError) as e:
        capi.moe_forward(sess.ctx, 2, x, 4, y)
    assert e.value.status == capi.MOE_ERR_INVALID_ARG
    with pytest.raises(capi.MoeError) as e:
        capi.moe_forward(sess.ctx, 0, None, 4, y)
    assert e.value.status == capi.MOE_ERR_INVALID_ARG
    y.fill_(7)
    capi.moe_forward(sess.ctx, 0, x, 0, y)          # T == 0: nothing written
    torch.cuda.synchronize()
    assert int(y.min()) == 7 and int(y.max()) == 7
    assert capi.moe_get_device_error(sess.ctx) == 0
    sess.close()


def test_memory_limit_gives_oom():
    capi, session = _cuda()
    with pytest.raises(capi.MoeError) as e:
        session.Session(TINY, max_tokens=16, mem_limit=4096)
    assert e.value.status == capi.MOE_ERR_OOM
    sess = session.Session(TINY, max_tokens=16, mem_limit=700_000)   # workspace fits, weights not
    with pytest.raises(capi.MoeError) as e:
        sess.load_synthetic(layers=[0])
    assert e.value.status == capi.MOE_ERR_OOM
    sess.close()


def _full_layer(name, T, rows=None, dense=False):
    """One full-size layer on T tokens through the C ABI; the listed rows (all
    when None) against the oracle.  dense: the oracle evaluates the rows with
    per-expert fp64 matrix products over a host copy of the whole layer."""
    capi, session = _cuda()
    cfg = synth.CONFIGS[name]
    sess = session.Session(cfg, max_tokens=T, n_layers=1)
    sess.load_synthetic(layers=[0])
    x = _tokens(cfg, T)
    gy, gyf, gids, gw = _run(sess, 0, x)
    assert capi.moe_get_device_error(sess.ctx) == 0
    sess.close()
    rows = list(range(T)) if rows is None else list(rows)
    src = HostLayer(cfg, 0) if dense else ExpertSource(cfg, 0)
    o = oracle_rows_dense(cfg, src, x, rows) if dense else None
    rep = {}
    check_rows(cfg, src, x, rows, gy[rows], gyf[rows], gids[rows], gw[rows], o=o, report=rep,
               tol16=bf16_tol(T))
    return cfg, x, gids, gw, src, rep


def test_decode_layer_full_size():
    _full_layer("decode_48l_q4_t1", 1, [0])


def test_verify_layer_full_size():
    _full_layer("verify_48l_q3_t4_zipf", 4, range(4))


def test_prefill_layer_full_size_all_tokens():
    """All 4096 tokens of the single-layer prefill workload (Zipf-skewed routing,
    tensor-core path, decoded-weight cache): every token's ids and weights and
    the whole [4096, 2560] output against the oracle."""
    cfg, x, gids, gw, src, rep = _full_layer("prefill_1l_q4_t4096_zipf", 4096, dense=True)
    assert rep["near_tie_flips"] <= 4


@pytest.mark.parametrize("name,T", [("tiny_d256_e16_q4_t8", 300), ("prefill_1l_q4_t4096_zipf", 512),
                                    ("verify_48l_q3_t4_zipf", 256)])
def test_tensor_core_path_matches_oracle_and_cuda_core_path(name, T):
    """Many-token calls on the tcgen05 grouped-GEMM path: every token against
    the oracle.  Then, as a supplementary check between two GPU paths, the
    CUDA-core path (exact fp32 weights) on the same inputs: same ids and
    weights wherever the two agree on the expert set (their routers sum in
    different orders, so a near tie may go either way), fp32 outputs of those
    tokens within the fp16 weight rounding (relative L2 <= 1e-3)."""
    capi, session = _cuda()
    cfg = synth.CONFIGS[name]
    a = session.Session(cfg, max_tokens=T, n_layers=1)
    b = session.Session(cfg, max_tokens=T, n_layers=1, flags=capi.MOE_FLAG_NO_TENSOR_PREFILL)
    W = synth.layer_weights(cfg, 0, device="cuda")
    a.load(0, W)
    b.load(0, W)
    del W
    x = _tokens(cfg, T, stream=77)
    ya, yfa, ida, wa = _run(a, 0, x)
    yb, yfb, idb, wb = _run(b, 0, x)
    assert capi.moe_get_device_error(a.ctx) == 0
    a.close()
    b.close()
    src = HostLayer(cfg, 0)
    rows = list(range(T))
    check_rows(cfg, src, x, rows, ya, yfa, ida, wa, o=oracle_rows_dense(cfg, src, x, rows), tol16=bf16_tol(T))
    same = np.all(ida == idb, axis=1)
    assert same.mean() >= 0.995
    assert np.max(np.abs(wa[same] - wb[same])) <= 1e-5
    assert rel_l2(yfa[same], yfb[same]) <= 1e-3


@pytest.mark.parametrize("T,flags", [(4, 0), (64, 0), (16, 1 | 2)])
def test_nan_and_inf_logits_keep_ids_in_range(T, flags):
    """A router bias with NaN and +inf entries (so NaN and +inf logits) on every
    path: each token still gets k distinct ids below E, chosen by the stated
    rule (a NaN logit ranks as -inf, ties by lower id), checked against the
    oracle's logits with that rule applied."""
    capi, session = _cuda()
    cfg = TINY
    bias = np.zeros(cfg.E, dtype=np.float32)
    bias[[1, 6, 12]] = np.nan
    bias[9] = np.inf
    sess = session.Session(cfg, max_tokens=max(T, 8), n_layers=1, flags=flags)

    def mut(W):
        W["router_b"] = bias
    sess.load(0, _tiny_weights_with(mut))
    x = _tokens(cfg, T, stream=31)
    _, _, gids, _ = _run(sess, 0, x)
    sess.close()
    src = ExpertSource(cfg, 0)
    src.router_b = bias
    xf = oracle.bf16_to_f64(x)
    for t in range(T):
        lg = oracle.router_logits(xf[t], src.router_w, bias)
        lg = np.where(np.isnan(lg), -np.inf, lg)
        want = np.lexsort((np.arange(cfg.E), -lg))[:cfg.k]
        assert np.all((gids[t] >= 0) & (gids[t] < cfg.E)) and len(set(gids[t].tolist())) == cfg.k
        assert gids[t][0] == 9                 # the +inf logit
        assert not set(gids[t].tolist()) & {1, 6, 12}
        fin = np.sort(lg[np.isfinite(lg)])[::-1]
        if fin.size > cfg.k and fin[cfg.k - 2] - fin[cfg.k - 1] >= 1e-5:
            assert np.array_equal(gids[t], want)
