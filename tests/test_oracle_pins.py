"""Pins for the CPU oracle: facts fixed by the pages and by mathematics, not by the oracle itself.

Each test names the passage or the mathematical fact it checks. None of these
touches the CUDA path.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
import synth as S

GOLD = os.path.join(os.path.dirname(__file__), "golden")
U32 = 2.0 ** -24


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- exp & co.
def test_cexp_within_2ulp_of_libm():
    """Own fp32 exp vs the correctly rounded fp64 exp, over the whole clamp range."""
    a = np.concatenate([np.linspace(-87, 88, 1_000_001, dtype=np.float32),
                        rng(0).uniform(-87, 88, 200_000).astype(np.float32),
                        np.array([0.0, -0.0, 1e-30, -1e-30, 0.5, -0.5], np.float32)])
    got = O.cexp(a).astype(np.float64)
    ref = np.exp(a.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(got - ref) / ulp) <= 2.0
    assert O.cexp(np.float32(0.0)) == 1.0


def test_cexp_saturates_outside_range():
    a = np.array([100.0, 88.0, -87.0, -200.0], np.float32)
    got = O.cexp(a)
    assert got[0] == got[1] and got[2] == got[3]
    assert np.isfinite(got).all() and got[3] > 0


def test_sigmoid_and_swiglu_close_to_fp64():
    """SwiGLU h = silu(g) * u (mtlm-7m-base card, architecture list) and the sigmoid score."""
    g = rng(1).normal(0, 3, 100_000).astype(np.float32)
    u = rng(2).normal(0, 3, 100_000).astype(np.float32)
    g64, u64 = g.astype(np.float64), u.astype(np.float64)
    s = O.sigmoid(g).astype(np.float64)
    assert np.max(np.abs(s - 1 / (1 + np.exp(-g64)))) <= 4 * U32
    h = O.swiglu(g, u).astype(np.float64)
    h64 = g64 / (1 + np.exp(-g64)) * u64
    assert np.all(np.abs(h - h64) <= 8 * U32 * np.abs(h64) + 1e-37)


# -------------------------------------------------------------- quantization
def test_q8_0_golden_group():
    g = gold("q8_0_group_example.json")
    x = (np.array(g["m"], np.float64) * 2.0 ** -7).astype(np.float32)[None, :]
    q, s = O.quantize_act(x, g32=True)
    assert s[0, 0] == np.float32(g["scale"])
    assert q[0].tolist() == g["q"]


def test_int4_golden_group_and_packing():
    g = gold("int4_group_example.json")
    w = (np.array(g["m"], np.float64) * 2.0 ** -4).astype(np.float32)[None, :]
    q, s = O.quantize_rows(w, 7, g32=True)
    assert s[0, 0] == np.float32(g["scale"])
    assert q[0].tolist() == g["q"]
    assert O.pack_int4(q)[0].tolist() == g["packed"]


def test_int2_golden_group_and_packing():
    g = gold("int2_group_example.json")
    w = (np.array(g["m"], np.float64) * 2.0 ** -3).astype(np.float32)[None, :]
    q, s = O.quantize_rows(w, O.QMAX[2], g32=True)
    assert s[0, 0] == np.float32(g["scale"])
    assert q[0].tolist() == g["q"]
    assert O.pack_int2(q)[0].tolist() == g["packed"]


@pytest.mark.parametrize("qmax,g32", [(127, True), (127, False), (7, True), (7, False), (1, True), (1, False)])
def test_quantization_roundtrip_bound(qmax, g32):
    """|w - q*d| <= d/2 for every element, |q| <= Q, and each group's largest |w| maps to +-Q."""
    w = rng(qmax + g32).normal(0, 0.02, (64, 256)).astype(np.float32)
    w[3, :32] = 0.0                                   # an all-zero group -> scale 0, codes 0
    q, s = O.quantize_rows(w, qmax, g32)
    d = np.repeat(s, 32, axis=1) if g32 else s[:, None]
    err = np.abs(w.astype(np.float64) - q.astype(np.float64) * d)
    assert np.all(err <= d / 2 * (1 + 1e-6) + 1e-45)
    assert np.abs(q).max() <= qmax
    if g32:
        assert np.all(np.float16(s).astype(np.float32) == s)      # stored scales are fp16 values
        grp = np.abs(q.reshape(64, -1, 32)).max(axis=2)
        nz = s > 0
        assert np.all(grp[nz] == qmax) and np.all(grp[~nz] == 0)
    else:
        assert np.all(np.abs(q).max(axis=1) == qmax)


def test_int4_packing_bit_identical_to_int8_container():
    """'Packing validated bit-identical to the int8 container' (GLM page, Quantization kernels)."""
    w = rng(5).normal(0, 0.02, (32, 512)).astype(np.float32)
    q, _ = O.quantize_rows(w, 7, True)
    p = O.pack_int4(q).astype(np.int16)
    lo = ((p & 0xF) ^ 8) - 8
    hi = (((p >> 4) & 0xF) ^ 8) - 8
    un = np.stack([lo, hi], axis=-1).reshape(q.shape)
    assert np.array_equal(un.astype(np.int8), q)
    a = rng(6).integers(-127, 128, 512).astype(np.int64)
    assert np.array_equal(un.astype(np.int64) @ a, q.astype(np.int64) @ a)


def _unpack_int2(p):
    p = p.astype(np.int16)
    return np.stack([(((p >> (2 * i)) & 3) ^ 2) - 2 for i in range(4)], -1).reshape(p.shape[0], -1)


def test_int2_packing_bit_identical_to_int8_container():
    w = rng(7).normal(0, 0.02, (32, 512)).astype(np.float32)
    q, _ = O.quantize_rows(w, O.QMAX[2], True)
    assert set(np.unique(q).tolist()) == {-1, 0, 1}
    un = _unpack_int2(O.pack_int2(q))
    assert np.array_equal(un.astype(np.int8), q)
    a = rng(8).integers(-127, 128, 512).astype(np.int64)
    assert np.array_equal(un.astype(np.int64) @ a, q.astype(np.int64) @ a)


@pytest.mark.parametrize("wbits,g32", [(8, True), (8, False), (4, True), (4, False), (2, True), (2, False)])
def test_blob_decodes_to_codes_and_scales(wbits, g32):
    """The oracle's blob decodes (by reshapes) back to the logical codes and scales."""
    E, H, I = 2, 256, 128
    r = rng(wbits * 2 + g32)
    gu = r.normal(0, 0.02, (E, 2 * I, H)).astype(np.float32)
    dn = r.normal(0, 0.02, (E, H, I)).astype(np.float32)
    ex = O.QExperts.quantize(gu, dn, wbits, g32)
    blob = ex.pack_blob()
    off = O.blob_layout(E, H, I, wbits, g32)
    assert all(o % 256 == 0 for o in off) and blob.size == off[4]

    def codes(region, rows, block, kb, K):
        a = region.reshape(rows // block, kb // 16, block, 16).transpose(0, 2, 1, 3).reshape(rows, kb)
        if wbits == 8:
            return a.view(np.int8).reshape(rows, K)
        if wbits == 2:
            return _unpack_int2(a).reshape(rows, K).astype(np.int8)
        b = a.astype(np.int16)
        return np.stack([((b & 15) ^ 8) - 8, (((b >> 4) & 15) ^ 8) - 8], -1).reshape(rows, K).astype(np.int8)

    kb_gu, kb_dn = H * wbits // 8, I * wbits // 8
    got_gu = codes(blob[off[0]:off[0] + E * 2 * I * kb_gu], E * 2 * I, 128, kb_gu, H)
    # row order inside each 128-row block: 64 gate rows then the matching 64 up rows
    order = np.concatenate([np.concatenate([np.arange(64 * s, 64 * s + 64),
                                            I + np.arange(64 * s, 64 * s + 64)])
                            for s in range(I // 64)])
    want_gu = ex.q_gu[:, order, :].reshape(E * 2 * I, H)
    assert np.array_equal(got_gu, want_gu)
    # down: slabs of 64 columns, each [128-row block][piece][row][16 bytes]
    U, HB, sb = I // 64, H // 128, kb_dn // (I // 64)
    dn = blob[off[1]:off[1] + E * H * kb_dn].reshape(E, U, HB, sb // 16, 128, 16)
    dn = dn.transpose(0, 2, 4, 1, 3, 5).reshape(E * H, kb_dn)
    if wbits == 8:
        got_dn = dn.view(np.int8).reshape(E * H, I)
    elif wbits == 2:
        got_dn = _unpack_int2(dn).reshape(E * H, I)
    else:
        b16 = dn.astype(np.int16)
        got_dn = np.stack([((b16 & 15) ^ 8) - 8, (((b16 >> 4) & 15) ^ 8) - 8], -1).reshape(E * H, I)
    assert np.array_equal(got_dn, ex.q_dn.reshape(E * H, I))
    if g32:
        sg = blob[off[2]:off[2] + E * 2 * I * (H // 32) * 2].view(np.float16).astype(np.float32)
        sg = sg.reshape(E * 2 * I // 128, H // 32, 128).transpose(0, 2, 1).reshape(E, 2 * I, H // 32)
        assert np.array_equal(sg, ex.s_gu[:, order, :])
        sd = blob[off[3]:off[3] + E * H * (I // 32) * 2].view(np.float16).astype(np.float32)
        sd = sd.reshape(E, U, HB, 2, 128).transpose(0, 2, 4, 1, 3).reshape(E, H, I // 32)
        assert np.array_equal(sd, ex.s_dn)
    else:
        sg = blob[off[2]:off[2] + E * 2 * I * 4].view(np.float32).reshape(E, 2 * I)
        assert np.array_equal(sg, ex.s_gu[:, order])
        sd = blob[off[3]:off[3] + E * H * 4].view(np.float32).reshape(E, H)
        assert np.array_equal(sd, ex.s_dn)


# ------------------------------------------------------------------- routing
def test_router_chunk_order_golden():
    g = gold("routing_examples.json")["router_chunks"]
    x = np.zeros((1, g["H"]), np.float32)
    for k, v in g["x_nonzero"].items():
        x[0, int(k)] = v
    Wr = np.ones((3, g["H"]), np.float32)
    L = O.router_logits(x, Wr)
    assert np.all(L == np.float32(g["logit"]))


def test_router_logits_within_fp32_bound_of_fp64():
    """L = x . W_r^T: recursive-summation error bound (H+1) u sum|x w|; a transposed or shifted
    operand fails it."""
    r = rng(7)
    x = r.normal(0, 1, (5, 512)).astype(np.float32)
    Wr = r.normal(0, 0.05, (16, 512)).astype(np.float32)
    L = O.router_logits(x, Wr).astype(np.float64)
    ref = x.astype(np.float64) @ Wr.astype(np.float64).T
    bound = (512 + 1) * U32 * (np.abs(x).astype(np.float64) @ np.abs(Wr).astype(np.float64).T)
    assert np.all(np.abs(L - ref) <= bound)


def test_topk_golden_ties():
    g = gold("routing_examples.json")["topk_ties"]
    L = np.array([g["logits"]], np.float32)
    idx, w = O.route(L, None, "softmax", g["k"], True, 1.0)
    assert idx[0].tolist() == g["idx"]
    e1 = math.exp(-1.0)
    assert np.allclose(w[0], [1 / (1 + 3 * e1)] + [e1 / (1 + 3 * e1)] * 3, rtol=0, atol=1e-15)


def test_sigmoid_bias_golden():
    g = gold("routing_examples.json")["sigmoid_bias"]
    L = np.array([g["logits"]], np.float32)
    idx, w = O.route(L, np.array(g["bias"], np.float32), "sigmoid", g["k"], True, g["rsf"])
    assert idx[0].tolist() == g["idx"]
    assert np.allclose(w[0], g["w"], rtol=1e-6)


@pytest.mark.parametrize("E,k", [(8, 2), (64, 8), (512, 10), (17, 17)])
def test_topk_equals_brute_force_sort(E, k):
    r = rng(E + k)
    L = r.normal(0, 1, (40, E)).astype(np.float32)
    L[:, ::5] = np.round(L[:, ::5])                     # many exact ties
    idx, _ = O.route(L, None, "softmax", k, True, 1.0)
    for t in range(L.shape[0]):
        want = sorted(range(E), key=lambda e: (-float(L[t, e]), e))[:k]
        assert idx[t].tolist() == want


def test_softmax_weights_closed_form():
    """Renormalised: exp(L_j) / sum_sel exp; plain: exp(L_j) / sum_all exp (fp64, math.fsum)."""
    r = rng(11)
    L = r.normal(0, 1, (6, 64)).astype(np.float32)
    for renorm in (True, False):
        idx, w = O.route(L, None, "softmax", 8, renorm, 1.0)
        for t in range(6):
            ex = [math.exp(float(v)) for v in L[t]]
            den = math.fsum(ex[e] for e in idx[t]) if renorm else math.fsum(ex)
            assert np.allclose(w[t], [ex[e] / den for e in idx[t]], rtol=1e-13, atol=0)
            assert np.all(np.diff(w[t]) <= 0)
        if renorm:
            assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)


def test_noaux_tc_bias_selects_but_does_not_weight():
    r = rng(12)
    L = r.normal(0, 1, (8, 32)).astype(np.float32)
    b = r.normal(0, 0.05, 32).astype(np.float32)
    b[31] = 10.0                                       # expert 31 always selected via the bias
    idx, w = O.route(L, b, "sigmoid", 4, True, 2.5)
    assert np.all(idx[:, 0] == 31)
    sig = 1 / (1 + np.exp(-L.astype(np.float64)))
    for t in range(8):
        s = sig[t, idx[t]]
        assert np.allclose(w[t], s / s.sum() * 2.5, rtol=1e-12)
        assert abs(w[t].sum() - 2.5) < 1e-12
    idx0, w0 = O.route(L, None, "sigmoid", 4, False, 1.0)
    assert np.array_equal(idx0, np.argsort(-L, axis=1, kind="stable")[:, :4])  # monotone in L
    assert np.allclose(w0, np.take_along_axis(sig, idx0, 1), rtol=1e-12)


def test_zero_input_routes_to_first_k_uniformly():
    x = np.zeros((3, 128), np.float32)
    Wr = rng(13).normal(0, 1, (16, 128)).astype(np.float32)
    L = O.router_logits(x, Wr)
    assert np.all(L == 0)
    idx, w = O.route(L, None, "softmax", 4, True, 1.0)
    assert np.all(idx == np.arange(4)) and np.allclose(w, 0.25, atol=1e-15)
    idx, w = O.route(L, None, "softmax", 4, False, 1.0)
    assert np.allclose(w, 1 / 16, atol=1e-15)


def test_permute_stable_counting_sort():
    """Batch-union grouping (GLM page, 'Batch-union MoE'): pairs sorted by (expert, token)."""
    r = rng(14)
    T, k, E = 300, 6, 40
    idx = np.stack([r.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    offsets, perm = O.permute(idx, E)
    flat = idx.reshape(-1)
    want = sorted(range(T * k), key=lambda p: (int(flat[p]), p))
    assert perm.tolist() == want
    assert np.array_equal(np.diff(offsets), np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k


# ------------------------------------------------------------ expert stages
MODES = [(True, True), (False, True), (True, False), (False, False)]


@pytest.mark.parametrize("wg32,ag32", MODES)
def test_stage_within_bound_of_exact_dequantized_dot(wg32, ag32):
    """Canonical fp32 stage vs the exact dequantize-then-dot: |v - v64| <= (G+2) u sum|terms|."""
    r = rng(20 + 2 * wg32 + ag32)
    K = 1024
    for wbits in (8, 4):
        w = r.normal(0, 0.02, (16, K)).astype(np.float32)
        a = r.normal(0, 1, (1, K)).astype(np.float32)
        qw, sw = O.quantize_rows(w, 127 if wbits == 8 else 7, wg32)
        qa, sa = O.quantize_act(a, ag32)
        for n in range(16):
            v, dots = O.stage(qw[n], sw[n], wg32, qa[0], sa[0], ag32)
            dw = qw[n].astype(np.float64) * (np.repeat(sw[n], 32) if wg32 else sw[n])
            da = qa[0].astype(np.float64) * (np.repeat(sa[0], 32) if ag32 else sa[0])
            exact = float(np.dot(dw, da))
            G = K // 32 if (wg32 or ag32) else 1
            assert abs(float(v) - exact) <= (G + 2) * U32 * float(np.sum(np.abs(dw * da))) + 1e-30
            assert abs(O.stage_f64(qw[n], sw[n], wg32, qa[0], sa[0], ag32) - exact) <= 1e-12 * abs(exact) + 1e-30
            prods = qw[n].astype(np.int64) * qa[0].astype(np.int64)
            want = prods.reshape(-1, 32).sum(1) if (wg32 or ag32) else np.array([prods.sum()])
            assert np.array_equal(dots.astype(np.int64), want)


def test_activation_power_of_two_scaling_invariance():
    """x -> 2^m x leaves codes and integer dots unchanged and scales s_x (and g, u) by 2^m."""
    cfg = S.CONFIGS["olmoe_int8"].with_(H=256, I=128, E=4)
    case = S.Case.make(cfg, 2)
    x = case.x()
    ex = O.QExperts.quantize(np.stack([case.gate_up(e) for e in range(4)]),
                             np.stack([case.down(e) for e in range(4)]), 8, True)
    q1, s1 = O.quantize_act(x, True)
    q2, s2 = O.quantize_act(x * np.float32(8.0), True)
    assert np.array_equal(q1, q2) and np.array_equal(s2, s1 * 8)
    a = O.expert_ffn(ex, 1, q1[0], s1[0], True)
    b = O.expert_ffn(ex, 1, q2[0], s2[0], True)
    assert np.array_equal(b["gate"], a["gate"] * 8) and np.array_equal(b["up"], a["up"] * 8)


# ------------------------------------------------------ whole-layer pins
def _numpy_dense_ffn(ex, e, qx, sx, ag32, I):
    """Independent fp64 SwiGLU FFN on the dequantized operands (numpy matmuls)."""
    wg = ex.q_gu[e].astype(np.float64) * (np.repeat(ex.s_gu[e], 32, axis=1) if ex.wg32 else ex.s_gu[e][:, None])
    wd = ex.q_dn[e].astype(np.float64) * (np.repeat(ex.s_dn[e], 32, axis=1) if ex.wg32 else ex.s_dn[e][:, None])
    xd = qx.astype(np.float64) * (np.repeat(sx, 32) if ag32 else sx)
    gu = wg @ xd
    g, u = gu[:I], gu[I:]
    h = g / (1 + np.exp(-g)) * u
    return wd, h, g, u


def _check_ffn_against_numpy(ex, e, qx, sx, ag32, got):
    """Every stage within its error bound; the h-quantization bound closes the loop on y."""
    I, H = ex.I, ex.H
    wd, h64, g64, u64 = _numpy_dense_ffn(ex, e, qx, sx, ag32, I)
    wg = ex.q_gu[e].astype(np.float64) * (np.repeat(ex.s_gu[e], 32, axis=1) if ex.wg32 else ex.s_gu[e][:, None])
    xd = qx.astype(np.float64) * (np.repeat(sx, 32) if ag32 else sx)
    G = H // 32 if (ex.wg32 or ag32) else 1
    bound_gu = (G + 2) * U32 * (np.abs(wg) @ np.abs(xd)) + 1e-38
    assert np.all(np.abs(got["gate"] - g64) <= bound_gu[:I])
    assert np.all(np.abs(got["up"] - u64) <= bound_gu[I:])
    sh = np.repeat(got["sh"], 32) if ag32 else np.full(I, got["sh"][0])
    hq = got["qh"].astype(np.float64) * sh
    h32 = O.swiglu(got["gate"], got["up"]).astype(np.float64)
    assert np.all(np.abs(hq - h32) <= sh / 2 * (1 + 1e-6) + 1e-45)       # quantization bound on h
    assert np.allclose(h32, h64, rtol=1e-4, atol=1e-6 * np.abs(h64).max())
    y_dense = wd @ h64
    bound = np.abs(wd) @ (sh / 2 + np.abs(h32 - h64) + 1e-7 * np.abs(h64)) + 1e-12 * np.abs(y_dense).max()
    assert np.all(np.abs(got["ye"] - y_dense) <= bound)
    assert np.allclose(got["ye"], wd @ hq, rtol=1e-12, atol=1e-18)


@pytest.mark.parametrize("wbits,wg32,ag32", [(8, False, False), (8, True, True), (4, True, True), (4, False, True),
                                             (2, True, True), (2, False, True)])
def test_single_expert_reproduces_dense_swiglu_ffn(wbits, wg32, ag32):
    """E = 1, k = 1, weight 1: the layer is one dense SwiGLU FFN on the quantized operands."""
    cfg = S.CONFIGS["olmoe_int8"].with_(H=256, I=128, E=1, top_k=1)
    case = S.Case.make(cfg, 3)
    x = case.x()
    ex = O.QExperts.quantize(case.gate_up(0)[None], case.down(0)[None], wbits, wg32)
    Wr = case.router_w()
    o = O.layer_forward(x, Wr, None, ex, None, "softmax", 1, True, 1.0, ag32)
    assert np.all(o["idx"] == 0) and np.all(o["w"] == 1.0)
    for t in range(3):
        got = dict(gate=o["gate"][t], up=o["up"][t], qh=o["qh"][t], sh=np.atleast_1d(o["sh"][t]),
                   ye=o["ye"][t])
        _check_ffn_against_numpy(ex, 0, o["qx"][t], o["sx"][t], ag32, got)
        assert np.array_equal(o["y"][t], o["ye"][t])


def test_full_topk_softmax_equals_dense_soft_mixture():
    """k = E with renormalised softmax: y = sum_e softmax_e(L) FFN_e (the MoE analogue of 'keep
    every key reproduces dense attention', GLM page, DSA sparse attention)."""
    cfg = S.CONFIGS["olmoe_int8"].with_(H=128, I=128, E=6, top_k=6)
    case = S.Case.make(cfg, 2)
    x, Wr = case.x(), case.router_w()
    ex = O.QExperts.quantize(np.stack([case.gate_up(e) for e in range(6)]),
                             np.stack([case.down(e) for e in range(6)]), 8, True)
    o = O.layer_forward(x, Wr, None, ex, None, "softmax", 6, True, 1.0, True)
    L = x.astype(np.float64) @ Wr.astype(np.float64).T
    for t in range(2):
        p = np.exp(L[t] - L[t].max())
        p /= p.sum()
        y = sum(p[e] * O.expert_ffn(ex, e, o["qx"][t], o["sx"][t], True)["ye"] for e in range(6))
        assert np.allclose(o["y"][t], y, rtol=1e-5, atol=1e-7 * np.abs(y).max())


@pytest.mark.parametrize("name", ["tiny", "e512_int4"])
def test_batch_union_equals_per_token_bitwise(name):
    """'each unique expert of the batch is read once and applied to every position that routes
    to it' (GLM page, Batch-union MoE) must not change the result."""
    cfg = S.CONFIGS[name]
    if name == "e512_int4":
        cfg = cfg.with_(H=256, I=128, E=32, shared_I=128)
    case = S.Case.make(cfg, 9)
    x, Wr = case.x(), case.router_w()
    ex = O.QExperts.quantize(np.stack([case.gate_up(e) for e in range(cfg.E)]),
                             np.stack([case.down(e) for e in range(cfg.E)]),
                             8 if cfg.wtype == "int8" else 4, cfg.wscale == "g32_f16")
    sh = None
    if cfg.shared_I:
        sh = O.QExperts.quantize(case.shared_gate_up()[None], case.shared_down()[None],
                                 8 if cfg.wtype == "int8" else 4, cfg.wscale == "g32_f16")
    args = (x, Wr, case.bias(), ex, sh, cfg.score, cfg.top_k, cfg.renormalize, cfg.rsf,
            cfg.act == "g32_f16")
    a = O.layer_forward(*args)
    b = O.layer_forward(*args, union=True)
    for key in ("y", "ye", "qh", "gate", "up", "idx"):
        assert np.array_equal(a[key], b[key]), key
    assert b["offsets"][-1] == 9 * cfg.top_k


def test_tiny_brute_force_layer():
    """H = 64, E = 4, T = 3, top-2: routing, weights and y re-derived in numpy fp64."""
    r = rng(30)
    H, I, E, T, k = 64, 32, 4, 3, 2
    x = r.normal(0, 1, (T, H)).astype(np.float32)
    Wr = r.normal(0, 0.3, (E, H)).astype(np.float32)
    gu = r.normal(0, 0.05, (E, 2 * I, H)).astype(np.float32)
    dn = r.normal(0, 0.05, (E, H, I)).astype(np.float32)
    ex = O.QExperts.quantize(gu, dn, 8, True)
    o = O.layer_forward(x, Wr, None, ex, None, "softmax", k, True, 1.0, True)
    L = x.astype(np.float64) @ Wr.astype(np.float64).T
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-L[t, e], e))
        srt = sorted(L[t], reverse=True)
        if srt[k - 1] - srt[k] > 1e-5:
            assert o["idx"][t].tolist() == order[:k]
        sel = o["idx"][t]
        p = np.exp(L[t, sel] - L[t, sel].max())
        p /= p.sum()
        assert np.allclose(o["w"][t], p, rtol=1e-5)
        y = np.zeros(H)
        for j, e in enumerate(sel):
            got = dict(gate=o["gate"][t * k + j], up=o["up"][t * k + j], qh=o["qh"][t * k + j],
                       sh=o["sh"][t * k + j], ye=o["ye"][t * k + j])
            _check_ffn_against_numpy(ex, e, o["qx"][t], o["sx"][t], True, got)
            y += o["w"][t, j] * o["ye"][t * k + j]
        assert np.allclose(o["y"][t], y, rtol=1e-12, atol=1e-15)


def test_shared_expert_adds_with_weight_one():
    """Shared expert (GLM page, 'shared expert'): y = routed combine + FFN_shared, ungated."""
    cfg = S.CONFIGS["glm_int4"].with_(H=256, I=128, E=8, shared_I=128)
    case = S.Case.make(cfg, 2)
    x, Wr = case.x(), case.router_w()
    ex = O.QExperts.quantize(np.stack([case.gate_up(e) for e in range(8)]),
                             np.stack([case.down(e) for e in range(8)]), 4, False)
    sh = O.QExperts.quantize(case.shared_gate_up()[None], case.shared_down()[None], 4, False)
    with_sh = O.layer_forward(x, Wr, case.bias(), ex, sh, "sigmoid", 8, True, 2.5, True)
    no_sh = O.layer_forward(x, Wr, case.bias(), ex, None, "sigmoid", 8, True, 2.5, True)
    for t in range(2):
        ys = O.expert_ffn(sh, 0, with_sh["qx"][t], with_sh["sx"][t], True)["ye"]
        assert np.allclose(with_sh["y"][t], no_sh["y"][t] + ys, rtol=1e-14, atol=1e-18)
        assert np.allclose(with_sh["w"][t].sum(), 2.5)


# ------------------------------------------------------- adaptive expert top-p
# The GLM page's "--topp" knob ("adaptive expert top-p"): per token, keep the shortest prefix
# of the sorted top-k list whose share of the list's mass reaches p.
def _topp_masses(L_t, sel, score):
    """fp64 masses of a token's top-k list (slot order), computed here from the logits."""
    Lt = L_t.astype(np.float64)
    return np.exp(Lt[sel] - Lt[sel[0]]) if score == "softmax" else 1.0 / (1.0 + np.exp(-Lt[sel]))


@pytest.mark.parametrize("score,renorm", [("softmax", True), ("softmax", False), ("sigmoid", True),
                                          ("sigmoid", False)])
@pytest.mark.parametrize("p", [0.3, 0.5, 0.7, 0.9])
def test_topp_keeps_shortest_prefix_reaching_p(score, renorm, p):
    r = rng(40 + int(100 * p))
    T, E, k = 300, 64, 8
    rsf = 2.5 if score == "sigmoid" else 1.0
    L = r.normal(0, 1, (T, E)).astype(np.float32)
    b = r.normal(0, 0.05, E).astype(np.float32) if score == "sigmoid" else None
    idx0, w0 = O.route(L, b, score, k, renorm, rsf)
    idx, w = O.route(L, b, score, k, renorm, rsf, top_p=p)
    decided = 0
    for t in range(T):
        m = int((idx[t] >= 0).sum())
        assert 1 <= m <= k
        assert np.array_equal(idx[t, :m], idx0[t, :m]) and np.all(idx[t, m:] == -1)
        assert np.all(w[t, m:] == 0.0)
        v = _topp_masses(L[t], idx0[t], score)
        share = np.cumsum(v) / v.sum()
        want = int(np.argmax(share >= p)) + 1
        # the cut is taken on fp32 sums: only a share within rounding of p may land either side
        if all(abs(share[j] - p) > 1e-5 for j in range(k)):
            assert m == want, (t, m, want)
            decided += 1
        if renorm:
            assert np.allclose(w[t, :m], v[:m] / v[:m].sum() * rsf, rtol=1e-12, atol=0)
            assert abs(w[t, :m].sum() - rsf) < 1e-12
        else:
            assert np.array_equal(w[t, :m], w0[t, :m])
    assert decided > 0.9 * T


@pytest.mark.parametrize("p", [0.0, 1.0, 1.5, -0.0])
def test_topp_off_values_give_plain_topk(p):
    r = rng(50)
    L = r.normal(0, 1, (20, 32)).astype(np.float32)
    for score in ("softmax", "sigmoid"):
        a = O.route(L, None, score, 6, True, 1.0)
        b = O.route(L, None, score, 6, True, 1.0, top_p=p)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
def test_topp_equal_logits_keep_ceil_pk(score):
    """All logits equal: every slot has the same mass (exactly 1, or 1/2 for the sigmoid), so
    the kept count is ceil(p k) -- p k computed as the fp32 product, exact for k = 8."""
    L = np.zeros((1, 16), np.float32)
    for p in (0.05, 0.125, 0.2, 0.3, 0.5, 0.51, 0.75, 0.99):
        idx, w = O.route(L, None, score, 8, True, 1.0, top_p=p)
        m = math.ceil(float(np.float32(p)) * 8)
        assert idx[0].tolist() == list(range(m)) + [-1] * (8 - m), p
        assert np.allclose(w[0, :m], 1.0 / m, rtol=1e-15)


def test_topp_kept_count_grows_with_p():
    r = rng(51)
    L = r.normal(0, 1, (100, 64)).astype(np.float32)
    prev = np.zeros(100, np.int64)
    for p in np.linspace(0.05, 0.95, 19):
        idx, _ = O.route(L, None, "softmax", 8, True, 1.0, top_p=float(p))
        m = (idx >= 0).sum(1)
        assert np.all(m >= prev)
        prev = m
    assert prev.min() >= 1 and prev.max() <= 8


def test_topp_permute_leaves_out_dropped_slots():
    idx = np.array([[3, 1, -1], [1, -1, -1], [0, 3, 2]], np.int32)
    offsets, perm = O.permute(idx, 4)
    assert offsets.tolist() == [0, 1, 3, 4, 6]
    assert perm.tolist() == [6, 1, 3, 8, 0, 7]
    with pytest.raises(ValueError):
        O.permute(np.array([[0, -2]], np.int32), 4)


@pytest.mark.parametrize("name,p", [("olmoe_int8", 0.6), ("glm_int4", 0.7), ("e512_int4", 0.5)])
def test_topp_layer_equals_kept_expert_composition(name, p):
    """The layer with top-p equals a composition built here from single-expert FFN calls: each
    token's kept experts weighted by the renormalised (or plain) routing weights, plus the
    shared expert; the batch-union path gives the same bits."""
    cfg = S.CONFIGS[name].with_(H=256, I=128, E=16, top_k=4)
    if cfg.shared_I:
        cfg = cfg.with_(shared_I=128)
    case = S.Case.make(cfg, 7)
    x, Wr = case.x(), case.router_w()
    wb, g32 = (8 if cfg.wtype == "int8" else 4), cfg.wscale == "g32_f16"
    ex = O.QExperts.quantize(np.stack([case.gate_up(e) for e in range(cfg.E)]),
                             np.stack([case.down(e) for e in range(cfg.E)]), wb, g32)
    sh = None
    if cfg.shared_I:
        sh = O.QExperts.quantize(case.shared_gate_up()[None], case.shared_down()[None], wb, g32)
    ag32 = cfg.act == "g32_f16"
    args = (x, Wr, case.bias(), ex, sh, cfg.score, cfg.top_k, cfg.renormalize, cfg.rsf, ag32)
    a = O.layer_forward(*args, top_p=p)
    u = O.layer_forward(*args, union=True, top_p=p)
    assert np.array_equal(a["y"], u["y"]) and np.array_equal(a["idx"], u["idx"])
    assert u["offsets"][-1] == int((a["idx"] >= 0).sum()) < 7 * cfg.top_k
    L = O.router_logits(x, Wr)
    idx, w = O.route(L, case.bias(), cfg.score, cfg.top_k, cfg.renormalize, cfg.rsf, top_p=p)
    assert np.array_equal(idx, a["idx"])
    qx, sx = O.quantize_act(x, ag32)
    for t in range(7):
        want = np.zeros(cfg.H)
        for j in range(cfg.top_k):
            if idx[t, j] >= 0:
                want += w[t, j] * O.expert_ffn(ex, int(idx[t, j]), qx[t], sx[t], ag32)["ye"]
        if sh is not None:
            want += O.expert_ffn(sh, 0, qx[t], sx[t], ag32)["ye"]
        assert np.allclose(a["y"][t], want, rtol=1e-12, atol=1e-15)


# ----------------------------------------------------- FP8 checkpoint conversion
# The GLM page's FP8 -> int4 converter: FP8 (E4M3) weights with one inverse scale per
# 128 x 128 block are dequantized, then quantized like any fp32 weight.
def test_fp8_e4m3_decode_matches_library_for_all_codes():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    got = O.fp8_e4m3_decode(codes)
    nan = np.isnan(want)
    assert nan.sum() == 2 and np.array_equal(np.isnan(got), nan)      # 0x7f, 0xff
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))   # -0 included


def test_fp8_e4m3_closed_forms():
    """Values fixed by the E4M3 definition (bias 7, 3 mantissa bits, no infinities)."""
    cases = {0x38: 1.0, 0x30: 0.5, 0xC0: -2.0, 0x7E: 448.0, 0x08: 2.0 ** -6, 0x01: 2.0 ** -9,
             0x07: 7 * 2.0 ** -9, 0x3F: 1.875, 0x00: 0.0}
    got = O.fp8_e4m3_decode(np.array(list(cases), np.uint8))
    assert got.tolist() == list(cases.values())


def test_fp8_block_scales_cover_ragged_blocks():
    torch = pytest.importorskip("torch")
    r = rng(60)
    E, N, K = 2, 300, 200                                  # ragged last blocks in both dims
    w8 = r.integers(0, 256, (E, N, K), dtype=np.uint8)
    w8[(w8 & 0x7F) == 0x7F] = 0x38                         # no NaN codes
    s = (2.0 ** r.integers(-12, -2, (E, 3, 2))).astype(np.float32) * r.uniform(1, 2, (E, 3, 2)).astype(np.float32)
    got = O.dequant_fp8(w8, s)
    dec = torch.from_numpy(w8.reshape(-1).copy()).view(torch.float8_e4m3fn).float().numpy().reshape(E, N, K)
    full = np.repeat(np.repeat(s, 128, axis=1), 128, axis=2)[:, :N, :K]
    assert np.array_equal(got, (dec * full).astype(np.float32))
    assert got[1, 299, 199] == dec[1, 299, 199] * s[1, 2, 1]
