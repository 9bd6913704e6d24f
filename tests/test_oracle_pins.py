"""Pins for the CPU oracle: it is checked against things other than itself.

* golden blocks worked out by hand from the format definitions (tests/golden);
* library routines (numpy float16, torch bfloat16, scipy softmax / expit);
* closed forms (constant-code matrices, silu identities, rmsnorm of constants);
* brute force on tiny inputs (dense SwiGLU over every expert, exhaustive
  top-k subset search);
* the invariants the layer's specification states (weights sum to 1,
  identical experts -> one dense SwiGLU + shared, zero-scale expert -> no
  contribution) and a few more (token independence, expert-id permutation
  equivariance, k = E -> full softmax mixture).
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from tests.packing import dense, pack, random_matrix

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "blocks.txt")


# --- number formats -----------------------------------------------------------

def test_half_decode_matches_numpy_for_every_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.half_to_f64(bits)
    lib = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])


def test_bf16_decode_matches_torch():
    bits = np.arange(0, 1 << 16, 7, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(bits)
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    nan = np.isnan(lib)
    assert np.array_equal(ours[~nan], lib[~nan])


def test_round_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [0.0, -0.0, 1.0, -3.0, 1e-40, -1e-39, 3e38]]).astype(np.float32)
    ours = oracle.round_bf16(v.astype(np.float64))
    lib = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)


def test_round_bf16_ties_and_single_rounding():
    # spacing of bf16 at 1.0 is 2^-7
    assert oracle.round_bf16(np.array([1 + 2.0 ** -8]))[0] == 0x3F80          # tie -> even (1.0)
    assert oracle.round_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 0x3F82      # tie -> even (1 + 2^-6)
    # just above the tie, below fp32 resolution: one rounding step goes up;
    # rounding through fp32 first would have lost the 2^-40 and gone down
    assert oracle.round_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == 0x3F81


# --- block formats -------------------------------------------------------------

def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            p = line.split()
            rows.append((p[0], bytes.fromhex(p[1]), int(p[2], 16), np.array([float(v) for v in p[3:]])))
    return rows


@pytest.mark.parametrize("case", range(len(_golden())))
def test_golden_blocks(case):
    fmt, blk, sbits, want = _golden()[case]
    got = oracle.block_weights(fmt, np.frombuffer(blk, np.uint8), sbits)
    assert got.shape == (32,)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("case", range(len(_golden())))
def test_golden_blocks_dense(case):
    fmt, blk, sbits, want = _golden()[case]
    got = oracle.dequant(fmt, np.frombuffer(blk, np.uint8).reshape(1, 1, -1), np.array([[sbits]], np.uint16))
    assert np.array_equal(got[0], want)


@pytest.mark.parametrize("fmt", ["q4", "q3", "q2"])
def test_dequant_matches_independent_packer_dense(fmt):
    rng = np.random.default_rng(21)
    q, s, packed, W = random_matrix(rng, fmt, 24, 160)
    assert np.array_equal(oracle.dequant(fmt, packed, s), W)


@pytest.mark.parametrize("fmt", ["q4", "q3", "q2"])
def test_block_codes_roundtrip_through_independent_packer(fmt):
    rng = np.random.default_rng(2)
    q = rng.integers(0, {"q4": 16, "q3": 8, "q2": 4}[fmt], size=(50, 32))
    packed = pack(fmt, q)
    for r in range(50):
        assert np.array_equal(oracle.block_codes(fmt, packed[r, 0]), q[r])


@pytest.mark.parametrize("fmt", ["q4", "q3", "q2"])
def test_qmatvec_matches_dense_definition(fmt):
    rng = np.random.default_rng(3)
    q, s, packed, W = random_matrix(rng, fmt, 40, 96)
    x = rng.standard_normal(96)
    assert np.allclose(oracle.qmatvec(fmt, packed, s, x), W @ x, rtol=1e-13, atol=1e-15)


def test_qmatvec_constant_codes_closed_form():
    # every code c: W[r, k] = s[r, b] (c - 8), so y_r = (c - 8) sum_b s_rb * sum_{k in b} x_k
    rng = np.random.default_rng(4)
    for c in (0, 3, 8, 15):
        q = np.full((6, 128), c)
        s = rng.uniform(0.01, 0.04, size=(6, 4)).astype(np.float16)
        x = rng.standard_normal(128)
        xb = x.reshape(4, 32).sum(axis=1)
        want = (c - 8) * (s.astype(np.float64) @ xb)
        got = oracle.qmatvec("q4", pack("q4", q), s.view(np.uint16), x)
        assert np.allclose(got, want, rtol=1e-13, atol=1e-15)


def test_qmatvec_q2_constant_codes_closed_form():
    # Q2B32, every code c: W[r, k] = s[r, b] (c - 2); code 2 gives an all-zero matrix
    rng = np.random.default_rng(5)
    for c in range(4):
        q = np.full((5, 96), c)
        s = rng.uniform(0.01, 0.04, size=(5, 3)).astype(np.float16)
        x = rng.standard_normal(96)
        want = (c - 2) * (s.astype(np.float64) @ x.reshape(3, 32).sum(axis=1))
        got = oracle.qmatvec("q2", pack("q2", q), s.view(np.uint16), x)
        assert np.allclose(got, want, rtol=1e-13, atol=1e-15)
        if c == 2:
            assert np.all(got == 0.0)


# --- activation -----------------------------------------------------------------

def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert math.isclose(oracle.silu(math.log(3.0)), 0.75 * math.log(3.0), rel_tol=1e-15)
    for z in (-7.5, -1.0, 0.3, 2.0, 30.0):
        # silu(z) - silu(-z) = z, and silu(z) = z * expit(z) (library logistic)
        assert math.isclose(oracle.silu(z) - oracle.silu(-z), z, rel_tol=1e-14, abs_tol=1e-15)
        assert math.isclose(oracle.silu(z), z * scipy.special.expit(z), rel_tol=1e-14)


# --- routing ---------------------------------------------------------------------

def test_route_brute_force_subsets():
    rng = np.random.default_rng(5)
    for trial in range(50):
        E, k = int(rng.integers(2, 9)), 0
        k = int(rng.integers(1, E + 1))
        lg = rng.standard_normal(E) * 2.0
        ids, w, gap = oracle.route(lg, k)
        best = max(itertools.combinations(range(E), k), key=lambda c: sum(lg[list(c)]))
        assert set(ids.tolist()) == set(best)
        assert all(lg[ids[j]] >= lg[ids[j + 1]] for j in range(k - 1))
        p = scipy.special.softmax(lg)
        assert np.allclose(w, p[ids] / p[ids].sum(), rtol=1e-14)
        assert math.isclose(w.sum(), 1.0, rel_tol=1e-14)
        # renormalised softmax over E equals softmax over the chosen logits
        assert np.allclose(w, scipy.special.softmax(lg[ids]), rtol=1e-13)
        srt = np.sort(lg)[::-1]
        assert gap == (srt[k - 1] - srt[k] if k < E else math.inf)


def test_route_ties_prefer_lower_id():
    ids, w, gap = oracle.route(np.array([0.5, 1.0, 1.0, 0.2, 1.0]), 2)
    assert ids.tolist() == [1, 2]
    assert np.allclose(w, [0.5, 0.5])
    assert gap == 0.0


def test_route_k_equals_e_is_full_softmax():
    lg = np.array([0.3, -1.2, 2.0, 0.0])
    ids, w, _ = oracle.route(lg, 4)
    assert ids.tolist() == [2, 0, 3, 1]
    assert np.allclose(w, scipy.special.softmax(lg)[ids], rtol=1e-14)


def test_router_logits_matches_numpy():
    rng = np.random.default_rng(6)
    Wr = (rng.standard_normal((7, 64)) * 0.02).astype(np.float32)
    b = rng.standard_normal(7).astype(np.float32)
    x = rng.standard_normal(64)
    assert np.allclose(oracle.router_logits(x, Wr), Wr.astype(np.float64) @ x, rtol=1e-13)
    assert np.allclose(oracle.router_logits(x, Wr, b), Wr.astype(np.float64) @ x + b, rtol=1e-13)


# --- expert and layer --------------------------------------------------------------

def _expert(rng, fmt, d, I, lo=0.005, hi=0.02, zero_scale=False):
    g = random_matrix(rng, fmt, I, d, lo, hi)
    u = random_matrix(rng, fmt, I, d, lo, hi)
    dn = random_matrix(rng, fmt, d, I, lo, hi)
    mats = [g, u, dn]
    if zero_scale:
        mats = [(q, np.zeros_like(s), p, np.zeros_like(W)) for (q, s, p, W) in mats]
    return mats


def _dense_swiglu(Wg, Wu, Wd, x):
    g, u = Wg @ x, Wu @ x
    return Wd @ (g * scipy.special.expit(g) * u)


@pytest.mark.parametrize("fmt", ["q4", "q3", "q2"])
def test_expert_matches_dense_swiglu(fmt):
    rng = np.random.default_rng(7)
    d, I = 128, 64
    (g, u, dn) = _expert(rng, fmt, d, I)
    x = rng.standard_normal(d)
    y, h = oracle.expert(fmt, (g[2], g[1]), (u[2], u[1]), (dn[2], dn[1]), x, want_h=True)
    gg, uu = g[3] @ x, u[3] @ x
    assert np.allclose(h, gg * scipy.special.expit(gg) * uu, rtol=1e-12)
    assert np.allclose(y, _dense_swiglu(g[3], u[3], dn[3], x), rtol=1e-11, atol=1e-13)


def _layer(rng, fmt, d, E, I, n_sh, I_s, bias=False, identical=False, zero_routed=False):
    ex = [_expert(rng, fmt, d, I, zero_scale=zero_routed) for _ in range(1 if identical else E)]
    if identical:
        ex = ex * E
    sh = [_expert(rng, fmt, d, I_s) for _ in range(n_sh)]
    W = {
        "router_w": (rng.standard_normal((E, d)) * 0.3).astype(np.float32),
        "router_b": rng.standard_normal(E).astype(np.float32) if bias else None,
        "codes": [np.stack([e[t][2] for e in ex]) for t in range(3)],
        "scales": [np.stack([e[t][1] for e in ex]) for t in range(3)],
        "sh_codes": [np.stack([e[t][2] for e in sh]) if sh else np.zeros((0,), np.uint8) for t in range(3)],
        "sh_scales": [np.stack([e[t][1] for e in sh]) if sh else np.zeros((0,), np.uint16) for t in range(3)],
        "_dense": [[e[t][3] for t in range(3)] for e in ex],
        "_dense_sh": [[e[t][3] for t in range(3)] for e in sh],
    }
    if not sh:
        W["sh_codes"] = [np.zeros((0, 1, 1, 1), np.uint8)] * 3
        W["sh_scales"] = [np.zeros((0, 1, 1), np.uint16)] * 3
    return W


def _tokens(rng, T, d):
    return oracle.round_bf16(rng.standard_normal((T, d)))


def _rows_dense(fmt, k, x, W, ids_for=None):
    ge = lambda e: tuple((W["codes"][t][e], W["scales"][t][e]) for t in range(3))
    gs = lambda s: tuple((W["sh_codes"][t][s], W["sh_scales"][t][s]) for t in range(3))
    return oracle.moe_rows_dense(fmt, k, x, W["router_w"], W["router_b"], ge, gs,
                                 n_shared=W["sh_codes"][0].shape[0], ids_for=ids_for)


@pytest.mark.parametrize("fmt,bias,batched", [("q4", False, False), ("q3", True, False), ("q2", True, False),
                                              ("q4", True, True), ("q3", False, True), ("q2", True, True)])
def test_layer_brute_force(fmt, bias, batched):
    rng = np.random.default_rng(8)
    d, E, I, k, T = 64, 6, 32, 2, 5
    W = _layer(rng, fmt, d, E, I, 1, 32, bias=bias)
    x = _tokens(rng, T, d)
    y, ids, w, gap = (_rows_dense if batched else oracle.moe_layer)(fmt, k, x, W)
    xf = x.view(np.uint16).astype(np.uint32) << 16
    xf = xf.view(np.float32).astype(np.float64)
    for t in range(T):
        lg = W["router_w"].astype(np.float64) @ xf[t]
        if bias:
            lg = lg + W["router_b"]
        best = max(itertools.combinations(range(E), k), key=lambda c: sum(lg[list(c)]))
        assert set(ids[t].tolist()) == set(best)
        p = scipy.special.softmax(lg)
        wt = p[ids[t]] / p[ids[t]].sum()
        assert np.allclose(w[t], wt, rtol=1e-13)
        ys = [_dense_swiglu(*W["_dense"][e], xf[t]) for e in range(E)]
        want = sum(wt[j] * ys[ids[t][j]] for j in range(k)) + _dense_swiglu(*W["_dense_sh"][0], xf[t])
        assert np.allclose(y[t], want, rtol=1e-11, atol=1e-12)


def test_layer_identical_experts_is_one_dense_swiglu_plus_shared():
    rng = np.random.default_rng(9)
    d, E, I, k, T = 64, 8, 32, 3, 4
    W = _layer(rng, "q4", d, E, I, 1, 32, identical=True)
    x = _tokens(rng, T, d)
    y, ids, w, _ = oracle.moe_layer("q4", k, x, W)
    xf = oracle.bf16_to_f64(x)
    for t in range(T):
        want = _dense_swiglu(*W["_dense"][0], xf[t]) + _dense_swiglu(*W["_dense_sh"][0], xf[t])
        assert np.allclose(y[t], want, rtol=1e-11, atol=1e-12)
        assert math.isclose(w[t].sum(), 1.0, rel_tol=1e-14)


def test_layer_zero_scale_experts_contribute_nothing():
    rng = np.random.default_rng(10)
    d, E, I, k, T = 64, 6, 32, 2, 3
    W = _layer(rng, "q3", d, E, I, 1, 32, zero_routed=True)
    x = _tokens(rng, T, d)
    y, _, _, _ = oracle.moe_layer("q3", k, x, W)
    xf = oracle.bf16_to_f64(x)
    for t in range(T):
        assert np.allclose(y[t], _dense_swiglu(*W["_dense_sh"][0], xf[t]), rtol=1e-12, atol=1e-14)


def test_layer_single_expert_no_shared_is_dense_swiglu():
    rng = np.random.default_rng(11)
    W = _layer(rng, "q4", 64, 1, 32, 0, 32)
    x = _tokens(rng, 3, 64)
    y, ids, w, gap = oracle.moe_layer("q4", 1, x, W)
    xf = oracle.bf16_to_f64(x)
    assert np.all(ids == 0) and np.all(w == 1.0) and np.all(np.isinf(gap))
    for t in range(3):
        assert np.allclose(y[t], _dense_swiglu(*W["_dense"][0], xf[t]), rtol=1e-11)


def test_layer_k_equals_e_is_softmax_mixture():
    rng = np.random.default_rng(12)
    d, E = 64, 4
    W = _layer(rng, "q4", d, E, 32, 0, 32)
    x = _tokens(rng, 2, d)
    y, ids, w, _ = oracle.moe_layer("q4", E, x, W)
    xf = oracle.bf16_to_f64(x)
    for t in range(2):
        p = scipy.special.softmax(W["router_w"].astype(np.float64) @ xf[t])
        want = sum(p[e] * _dense_swiglu(*W["_dense"][e], xf[t]) for e in range(E))
        assert np.allclose(y[t], want, rtol=1e-11)


def test_layer_token_independence_and_permutation_equivariance():
    rng = np.random.default_rng(13)
    d, E, I, k, T = 64, 6, 32, 2, 6
    W = _layer(rng, "q4", d, E, I, 1, 32, bias=True)
    x = _tokens(rng, T, d)
    y, ids, w, gap = oracle.moe_layer("q4", k, x, W)
    for t in range(T):
        y1, ids1, w1, _ = oracle.moe_layer("q4", k, x[t:t + 1], W)
        assert np.array_equal(y1[0], y[t]) and np.array_equal(ids1[0], ids[t])
    perm = rng.permutation(E)       # new expert e' = perm position: expert perm[e'] moves to e'
    Wp = dict(W)
    Wp["router_w"] = W["router_w"][perm]
    Wp["router_b"] = W["router_b"][perm]
    Wp["codes"] = [c[perm] for c in W["codes"]]
    Wp["scales"] = [s[perm] for s in W["scales"]]
    yp, idsp, wp, _ = oracle.moe_layer("q4", k, x, Wp)
    assert np.allclose(yp, y, rtol=1e-13, atol=1e-14)
    assert np.array_equal(perm[idsp], ids)
    assert np.allclose(wp, w, rtol=1e-14)


def test_moe_token_matches_moe_layer():
    rng = np.random.default_rng(14)
    d, E, I, k = 64, 6, 32, 2
    W = _layer(rng, "q3", d, E, I, 1, 32, bias=True)
    x = _tokens(rng, 3, d)
    y, ids, w, gap = oracle.moe_layer("q3", k, x, W)
    ge = lambda e: tuple((W["codes"][t][e], W["scales"][t][e]) for t in range(3))
    gs = lambda s: tuple((W["sh_codes"][t][s], W["sh_scales"][t][s]) for t in range(3))
    for t in range(3):
        yt, idt, wt, gt = oracle.moe_token("q3", k, x[t], W["router_w"], W["router_b"], ge, gs)
        assert np.allclose(yt, y[t], rtol=1e-13) and np.array_equal(idt, ids[t])
        yf, wf = oracle.moe_token_with_ids("q3", x[t], ids[t], W["router_w"], W["router_b"], ge, gs)
        assert np.allclose(yf, y[t], rtol=1e-13) and np.allclose(wf, w[t], rtol=1e-13)


# --- stack normalisation -------------------------------------------------------------

def test_rmsnorm_closed_forms():
    c = np.full(256, -3.0)
    assert np.allclose(oracle.rmsnorm(c, 0.0), -1.0, rtol=1e-15)
    assert np.allclose(oracle.rmsnorm(c, 1e-6), -3.0 / math.sqrt(9.0 + 1e-6), rtol=1e-15)
    rng = np.random.default_rng(15)
    r = rng.standard_normal(2560) * 7.0
    out = oracle.rmsnorm(r, 0.0)
    assert math.isclose(np.mean(out ** 2), 1.0, rel_tol=1e-13)
    assert np.allclose(oracle.rmsnorm(r * 1024.0, 0.0), out, rtol=1e-14)


@pytest.mark.parametrize("fmt", ["q4", "q3", "q2"])
def test_rows_dense_matches_moe_layer_and_given_ids(fmt):
    """The batched evaluation is the per-token layer with its fp64 sums reordered;
    with ids given it matches moe_token_with_ids."""
    rng = np.random.default_rng(22)
    d, E, I, k, T = 96, 8, 64, 3, 17
    W = _layer(rng, fmt, d, E, I, 1, 64, bias=True)
    x = _tokens(rng, T, d)
    y, ids, w, gap = oracle.moe_layer(fmt, k, x, W)
    yd, idd, wd, gd = _rows_dense(fmt, k, x, W)
    assert np.array_equal(ids, idd)
    assert np.allclose(wd, w, rtol=1e-13)
    assert np.allclose(gd, gap, rtol=1e-9, atol=1e-12)
    assert np.allclose(yd, y, rtol=1e-12, atol=1e-13)
    alt = {4: ids[4][::-1].copy(), 9: np.array([0, 1, 2], np.int32)}
    ya, ida, wa, _ = _rows_dense(fmt, k, x, W, ids_for=alt)
    ge = lambda e: tuple((W["codes"][t][e], W["scales"][t][e]) for t in range(3))
    gs = lambda s: tuple((W["sh_codes"][t][s], W["sh_scales"][t][s]) for t in range(3))
    for t, g_ids in alt.items():
        yw, ww = oracle.moe_token_with_ids(fmt, x[t], g_ids, W["router_w"], W["router_b"], ge, gs)
        assert np.array_equal(ida[t], g_ids)
        assert np.allclose(wa[t], ww, rtol=1e-13)
        assert np.allclose(ya[t], yw, rtol=1e-12, atol=1e-13)
