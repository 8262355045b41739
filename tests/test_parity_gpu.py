"""GPU parity: every step of the CUDA path through the C ABI against the CPU oracle, on the
same seeded inputs. Integer results (codes, indices, permutations, int32 dots) and every
fp32 value that decides one (logits, gate/up stage values) must match bit for bit; routing
weights to fp32 rounding; the layer output to rel-L2 <= 1e-5 and max-abs <= 1e-4 * max|y|."""
import numpy as np
import pytest

import oracle as O
import synth as S
from helpers import (ag32, assert_close_y, expected_down_dots, gpu_layer, oracle_layer, route_cfg, wbits,
                     wg32)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def M():
    import quantized_expert_ffn_logits_b200 as m
    return m


# Reduced versions of the five workloads (same formats and routing; sizes the oracle
# finishes in seconds, still several blocks per expert and ragged token counts), plus
# format combinations the five do not use.
BASE = S.CONFIGS
REDUCED = {
    "tiny": BASE["tiny"],
    "olmoe_int8": BASE["olmoe_int8"].with_(name="olmoe_int8_r", H=512, E=16, I=256, top_k=4),
    "olmoe_int4": BASE["olmoe_int4"].with_(name="olmoe_int4_r", H=512, E=16, I=256, top_k=4),
    "glm_int4": BASE["glm_int4"].with_(name="glm_int4_r", H=768, E=32, I=256, top_k=4, shared_I=128),
    "e512_int4": BASE["e512_int4"].with_(name="e512_int4_r", H=512, E=64, I=128, top_k=6, shared_I=128),
    "int8_g32_tok": BASE["olmoe_int8"].with_(name="int8_g32_tok", H=384, E=8, I=128, top_k=3,
                                             act="token_f32"),
    "int4_g32_tok": BASE["olmoe_int4"].with_(name="int4_g32_tok", H=256, E=8, I=256, top_k=2,
                                             act="token_f32", shared_I=128),
    "int8_row_g32": BASE["tiny"].with_(name="int8_row_g32", H=384, act="g32_f16", x_sigma=1.0,
                                       renormalize=True),
    "int4_row_tok": BASE["glm_int4"].with_(name="int4_row_tok", H=256, E=16, I=128, top_k=4,
                                           act="token_f32", shared_I=256),
    # packed int2 experts (the GLM page's third container): group-32 scales and activations,
    # and per-row scales with per-token activations and a shared expert
    "int2_g32": BASE["olmoe_int2"].with_(name="int2_g32", H=512, E=16, I=256, top_k=4),
    "int2_row_tok": BASE["olmoe_int2"].with_(name="int2_row_tok", H=384, E=8, I=128, top_k=3,
                                             wscale="row_f32", act="token_f32", shared_I=128),
}
CASES = [("tiny", 1), ("tiny", 4), ("tiny", 37),
         ("olmoe_int8", 1), ("olmoe_int8", 8), ("olmoe_int8", 33), ("olmoe_int8", 70),
         ("olmoe_int4", 1), ("olmoe_int4", 40), ("olmoe_int4", 130),
         ("glm_int4", 1), ("glm_int4", 4), ("glm_int4", 50),
         ("e512_int4", 1), ("e512_int4", 64), ("e512_int4", 100),
         ("int8_g32_tok", 5), ("int4_g32_tok", 9), ("int8_row_g32", 6), ("int4_row_tok", 3),
         ("int2_g32", 1), ("int2_g32", 8), ("int2_g32", 37), ("int2_row_tok", 1), ("int2_row_tok", 5)]


def _np(t):
    return t.detach().cpu().numpy()


def _run_layer(case, flags, top_p=0.0):
    m = M()
    c = case.cfg
    g = gpu_layer(case)
    cfg = route_cfg(c, flags=flags, top_p=top_p)
    y, ws = m.moe_layer_forward(g["x"], g["wr"], g["bias"], g["blob"], g["shared"], cfg)
    torch.cuda.synchronize()
    views = m.moe_layer_debug_views(case.T, g["blob"], g["shared"], cfg)
    return g, cfg, y, ws, views


@pytest.mark.parametrize("name,T", CASES)
def test_layer_forward_matches_oracle(name, T):
    _check_layer(name, T, M().MOE_FLAG_DEBUG)


# The tensor-core path (experts with >= 16 pairs at T > 32; every expert with the force flag):
# the same bit-exact gate/up values, h codes and scales as the streaming path and the oracle.
MMA_CASES = [("olmoe_int4", 300, False), ("olmoe_int4", 40, True), ("olmoe_int8", 70, True),
             ("e512_int4", 100, True), ("glm_int4", 50, True), ("int2_g32", 300, False), ("int2_g32", 40, True)]


@pytest.mark.parametrize("name,T,force", MMA_CASES)
def test_tensor_core_path_matches_oracle(name, T, force):
    m = M()
    _check_layer(name, T, m.MOE_FLAG_DEBUG | (m.MOE_FLAG_FORCE_MMA if force else 0))


# Adaptive expert top-p (the GLM page's "--topp"): every routing path -- the single-launch
# decode kernel (T = 1, group-32 activations), the fused routing kernel (rank-based and warp
# top-k, and its one-token grouping with per-token scales), the four-launch routing with the
# tensor-core GEMMs -- drops the same slots as the oracle, bit for bit, and the layer output
# leaves their experts out.
TOPP_CASES = [("olmoe_int8", 1, 0.5), ("glm_int4", 1, 0.7), ("e512_int4", 1, 0.6),
              ("tiny", 1, 0.3), ("tiny", 4, 0.3), ("glm_int4", 4, 0.7), ("olmoe_int8", 8, 0.5),
              ("e512_int4", 30, 0.4), ("olmoe_int4", 130, 0.6), ("e512_int4", 100, 0.5)]


@pytest.mark.parametrize("name,T,p", TOPP_CASES)
def test_adaptive_top_p_matches_oracle(name, T, p):
    _check_layer(name, T, M().MOE_FLAG_DEBUG, top_p=p)


@pytest.mark.parametrize("score,renorm,E,k", [("softmax", True, 64, 8), ("softmax", False, 512, 10),
                                              ("sigmoid", True, 256, 8)])
def test_route_topk_adaptive_top_p(score, renorm, E, k):
    m = M()
    r = np.random.default_rng(E + k)
    T = 200
    L = r.normal(0, 1, (T, E)).astype(np.float32)
    b = r.normal(0, 0.05, E).astype(np.float32) if score == "sigmoid" else None
    rsf = 2.5 if score == "sigmoid" else 1.0
    for p in (0.3, 0.6, 0.9):
        want_idx, want_w = O.route(L, b, score, k, renorm, rsf, top_p=p)
        cfg = m.RouteCfg(score=score, top_k=k, renormalize=renorm, routed_scaling_factor=rsf, top_p=p)
        idx, w = m.moe_route_topk(torch.from_numpy(L).cuda(), torch.from_numpy(b).cuda() if b is not None else None,
                                  cfg)
        torch.cuda.synchronize()
        assert np.array_equal(_np(idx), want_idx)
        assert np.allclose(_np(w), want_w, rtol=2e-6, atol=1e-7)
        if p < 0.8:          # (sigmoid masses of a top-8 are near equal: 0.9 keeps all 8)
            assert (want_idx < 0).any()


def _check_layer(name, T, flags, top_p=0.0):
    m = M()
    c = REDUCED[name]
    case = S.Case.make(c, T)
    g, cfg, y, ws, v = _run_layer(case, flags, top_p)
    assert m.moe_read_device_status(ws) == m.MOE_OK
    ref = oracle_layer(case, union=True, top_p=top_p)
    k, E, H, I = c.top_k, c.E, c.H, c.I
    if top_p:
        assert (ref["idx"] < 0).any(), "no slot dropped: the case does not exercise top-p"
    P = int((ref["idx"] >= 0).sum())             # kept (token, slot) pairs
    view = lambda off, dt, shape: _np(m.workspace_view(ws, off, dt, shape))
    # routing: bit-exact logits and indices, weights to fp32 rounding
    assert np.array_equal(view(v["logits"], torch.float32, (T, E)), ref["logits"])
    idx = view(v["idx"], torch.int32, (T, k))
    assert np.array_equal(idx, ref["idx"])
    w = view(v["w"], torch.float32, (T, k))
    assert np.allclose(w, ref["w"], rtol=2e-6, atol=1e-7)
    # quantized activations
    assert np.array_equal(view(v["q_x"], torch.int8, (T, H)), ref["qx"])
    sx = view(v["s_x"], torch.float16 if ag32(c) else torch.float32, (T, H // 32) if ag32(c) else (T,))
    assert np.array_equal(sx.astype(np.float32), ref["sx"])
    # batch-union grouping
    assert np.array_equal(view(v["offsets"], torch.int32, (E + 1,)), ref["offsets"])
    perm = view(v["perm"], torch.int32, (P,))
    assert np.array_equal(perm, ref["perm"])
    n_active = int(view(v["n_active"], torch.int32, (1,))[0])
    assert n_active == len(set(ref["idx"].reshape(-1).tolist()) - {-1})
    # per-pair stage values (grouped row r holds pair perm[r]) and quantized h
    gate = view(v["gate"], torch.float32, (P, I))
    up = view(v["up"], torch.float32, (P, I))
    assert np.array_equal(gate, ref["gate"][perm]), "gate stage values"
    assert np.array_equal(up, ref["up"][perm]), "up stage values"
    qh = view(v["q_h"], torch.int8, (P, I))
    assert np.array_equal(qh, ref["qh"][perm])
    if ag32(c):
        sh = view(v["s_h"], torch.float16, (P, I // 32)).astype(np.float32)
    else:
        sh = view(v["s_h"], torch.float32, (P,))
    assert np.array_equal(sh, ref["sh"][perm])
    ye = view(v["y_pair"], torch.float32, (P, H))
    assert_close_y(ye, ref["ye"][perm], "per-pair expert outputs")
    _check_down_dots(m, ws, v, case, ref, perm)
    assert_close_y(_np(y), ref["y"])


def _check_down_dots(m, ws, v, case, ref, perm):
    """The down projection's int32 group dots, as the expert kernels formed them (streaming
    and tensor-core paths alike), equal the exact integer dots of the oracle's h codes with the
    oracle's down codes, for every kept pair and every shared-expert row; dropped slots stay 0.
    Two entries are also checked against the oracle's own stage routine."""
    c = case.cfg
    T, k, H, I, Is = case.T, c.top_k, c.H, c.I, c.shared_I
    P = len(perm)
    got = _np(m.workspace_view(ws, v["dn_dots"], torch.int32, (T * k, H, I // 32)))
    want, want_sh = expected_down_dots(ref, case, perm)
    bad = np.argwhere(got[:P] != want)
    assert bad.size == 0, f"{len(bad)} down group dots differ, first (row, n, g) {bad[:4].tolist()}"
    assert not got[P:].any(), "dropped slots' dots must stay 0"
    ex, sh = ref["experts"]
    for r in (0, P - 1):
        pair = int(perm[r])
        e = int(ref["idx"].reshape(-1)[pair])
        n = (7 * r + 3) % H
        _, dots = O.stage(ex.q_dn[e, n], ex.s_dn[e, n], wg32(c), ref["qh"][pair], ref["sh"][pair], ag32(c))
        # (per-row weights with per-token activations: the stage routine's one whole-row dot)
        mine = got[r, n] if dots.size > 1 else got[r, n].sum(keepdims=True)
        assert np.array_equal(mine, dots), (r, n)
    if Is:
        off = v["dn_dots"] + T * k * H * (I // 32) * 4
        got_sh = _np(m.workspace_view(ws, off, torch.int32, (T, H, Is // 32)))
        assert np.array_equal(got_sh, want_sh), "shared-expert down group dots"


@pytest.mark.parametrize("name,T", [("olmoe_int8", 8), ("glm_int4", 4), ("e512_int4", 64)])
def test_down_stage_values_close(name, T):
    """Per-pair down values: fp32 sums of the per-slab shares (any order) against the
    oracle's fp64 down projection of the same quantized h (the int32 dots themselves are
    pinned bit-exact through moe_expert_group_dots)."""
    m = M()
    case = S.Case.make(REDUCED[name], T)
    g, cfg, y, ws, v = _run_layer(case, m.MOE_FLAG_DEBUG)
    ref = oracle_layer(case, union=True)
    P, H = T * case.cfg.top_k, case.cfg.H
    perm = _np(m.workspace_view(ws, v["perm"], torch.int32, (P,)))
    ye = _np(m.workspace_view(ws, v["y_pair"], torch.float32, (P, H)))
    assert_close_y(ye, ref["ye"][perm], "per-pair down values")


@pytest.mark.parametrize("name,T", [("olmoe_int8", 33), ("glm_int4", 4), ("e512_int4", 100)])
def test_forward_without_debug_equals_debug(name, T):
    m = M()
    case = S.Case.make(REDUCED[name], T)
    g = gpu_layer(case)
    c = case.cfg
    y0, ws0 = m.moe_layer_forward(g["x"], g["wr"], g["bias"], g["blob"], g["shared"], route_cfg(c))
    y1, ws1 = m.moe_layer_forward(g["x"], g["wr"], g["bias"], g["blob"], g["shared"],
                                  route_cfg(c, m.MOE_FLAG_DEBUG))
    torch.cuda.synchronize()
    assert_close_y(_np(y0), _np(y1).astype(np.float64))
    ref = oracle_layer(case)
    assert_close_y(_np(y0), ref["y"])


@pytest.mark.parametrize("name,T", [("olmoe_int8", 1), ("e512_int4", 64)])
def test_forward_debug_entry_point(name, T):
    """moe_layer_forward_debug: the forward with the debug intermediates kept, and their offsets
    returned in the same call (routing indices and h codes equal to the oracle's; y within the
    layer tolerance); moe_get_device_status reads the clean status word."""
    m = M()
    case = S.Case.make(REDUCED[name], T)
    g = gpu_layer(case)
    c = case.cfg
    y, ws, v = m.moe_layer_forward_debug(g["x"], g["wr"], g["bias"], g["blob"], g["shared"], route_cfg(c))
    torch.cuda.synchronize()
    assert m.moe_get_device_status(ws) == m.MOE_OK
    assert v == m.moe_layer_debug_views(T, g["blob"], g["shared"], route_cfg(c, m.MOE_FLAG_DEBUG))
    assert v["gate"] >= 0 and v["y_pair"] >= 0
    ref = oracle_layer(case)
    idx = _np(m.workspace_view(ws, v["idx"], torch.int32, (T, c.top_k)))
    assert np.array_equal(idx, ref["idx"])
    assert_close_y(_np(y), ref["y"])


@pytest.mark.parametrize("name,T", [("olmoe_int8", 1), ("glm_int4", 3), ("olmoe_int4", 40)])
def test_forward_host_buffers_equal_device_path(name, T):
    """moe_layer_forward_host (pinned host x in, y out, one C call per step) on four different
    inputs enqueued back to back with no synchronization between them, each into its own host
    output: every call's y matches the oracle on its own x (to the layer tolerance). The calls
    share the device staging buffer of x, which the next call's input copy overwrites while the
    previous call's kernels may still be running; a copy that overtook a reader of x would
    show up here as a wrong y. The first call's y also matches moe_layer_forward on device
    buffers."""
    m = M()
    case = S.Case.make(REDUCED[name], T)
    g = gpu_layer(case)
    c = case.cfg
    lay = m.Layer(T, g["blob"], g["shared"], route_cfg(c), g["wr"], g["bias"])
    xs = [case.x()] + [S.normal_cpu(T * c.H, 4242 + i, 0, c.x_sigma).reshape(T, c.H) for i in range(3)]
    xh = [torch.from_numpy(x).pin_memory() for x in xs]
    yh = [torch.full((T, c.H), float("nan"), dtype=torch.float32).pin_memory() for _ in xs]
    yd = torch.empty((T, c.H), dtype=torch.float32, device="cuda")
    lay(g["x"], yd)
    for a, b in zip(xh, yh):
        lay.forward_host(a, b)
    torch.cuda.synchronize()
    assert m.moe_read_device_status(lay.workspace) == m.MOE_OK
    assert_close_y(yh[0].numpy(), _np(yd).astype(np.float64))
    for i, x in enumerate(xs):
        assert_close_y(yh[i].numpy(), oracle_layer(case, x=x)["y"], f"call {i}")


def test_synth_device_generator_matches_host():
    t = torch.empty(1_000_003, dtype=torch.float32, device="cuda")
    S.normal_gpu_(t, 12345, 777, 0.02)
    assert np.array_equal(_np(t), S.normal_cpu(1_000_003, 12345, 777, 0.02))


@pytest.mark.parametrize("wtype,wscale", [("int8", "row_f32"), ("int8", "g32_f16"),
                                          ("int4", "row_f32"), ("int4", "g32_f16"),
                                          ("int2", "row_f32"), ("int2", "g32_f16")])
@pytest.mark.parametrize("E,H,I", [(3, 256, 128), (2, 384, 256)])
def test_quantize_experts_blob_bytes_identical(wtype, wscale, E, H, I):
    m = M()
    c = S.CONFIGS["olmoe_int8"].with_(E=E, H=H, I=I, wtype=wtype, wscale=wscale)
    case = S.Case.make(c, 1)
    gu = torch.empty((E, 2 * I, H), dtype=torch.float32, device="cuda")
    dn = torch.empty((E, H, I), dtype=torch.float32, device="cuda")
    case.gate_up_gpu(gu)
    case.down_gpu(dn)
    gu[0, 5, :32] = 0.0                       # an all-zero group
    blob = m.ExpertBlob.quantize(gu, dn, wtype, wscale)
    ex = O.QExperts.quantize(_np(gu), _np(dn), wbits(c), wg32(c))
    got = _np(blob.data)
    want = ex.pack_blob()
    assert got.size == want.size
    diff = np.nonzero(got != want)[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at {diff[:8]}"


@pytest.mark.parametrize("wtype,wscale", [("int8", "row_f32"), ("int8", "g32_f16"),
                                          ("int4", "row_f32"), ("int4", "g32_f16")])
@pytest.mark.parametrize("E,H,I", [(3, 256, 128), (2, 384, 256)])
def test_quantize_experts_fp8_blob_bytes_identical(wtype, wscale, E, H, I):
    """The FP8 checkpoint converter (GLM page): E4M3 codes with 128 x 128 block scales give the
    oracle's blob byte for byte (every code but the two NaNs, scales varying per block)."""
    m = M()
    r = np.random.default_rng(E * H + I)
    cdiv = lambda a: (a + 127) // 128
    gu8 = r.integers(0, 256, (E, 2 * I, H), dtype=np.uint8)
    dn8 = r.integers(0, 256, (E, H, I), dtype=np.uint8)
    for a in (gu8, dn8):
        a[(a & 0x7F) == 0x7F] = 0x3A                      # no NaN codes
    gu8[0, 5, :32] = 0                                     # an all-zero group
    sgu = (r.uniform(0.5, 2.0, (E, cdiv(2 * I), cdiv(H))) * 2.0 ** -8).astype(np.float32)
    sdn = (r.uniform(0.5, 2.0, (E, cdiv(H), cdiv(I))) * 2.0 ** -8).astype(np.float32)
    blob = m.ExpertBlob.quantize_fp8(torch.from_numpy(gu8).cuda(), torch.from_numpy(sgu).cuda(),
                                     torch.from_numpy(dn8).cuda(), torch.from_numpy(sdn).cuda(), wtype, wscale)
    ex = O.QExperts.quantize(O.dequant_fp8(gu8, sgu), O.dequant_fp8(dn8, sdn), 8 if wtype == "int8" else 4,
                             wscale == "g32_f16")
    got = _np(blob.data)
    want = ex.pack_blob()
    assert got.size == want.size
    diff = np.nonzero(got != want)[0]
    assert diff.size == 0, f"{diff.size} bytes differ, first at {diff[:8]}"


@pytest.mark.parametrize("act", ["g32_f16", "token_f32"])
# (H = 32, 96, 160: fewer groups than a CTA has warps, and groups that do not divide among them)
@pytest.mark.parametrize("T,H,sigma", [(1, 2048, 1.0), (7, 256, 0.02), (65, 6144, 3.0), (3, 32, 1.0),
                                       (9, 96, 1.0), (17, 160, 0.5)])
def test_quantize_activations_bit_exact(act, T, H, sigma):
    m = M()
    x = S.normal_cpu(T * H, 99 + T, 0, sigma).reshape(T, H)
    x[0, :32] = 0.0
    q, s = m.moe_quantize_activations(torch.from_numpy(x).cuda(), act)
    rq, rs = O.quantize_act(x, act == "g32_f16")
    assert np.array_equal(_np(q), rq)
    assert np.array_equal(_np(s).astype(np.float32), rs)


@pytest.mark.parametrize("T,E,H", [(1, 64, 2048), (5, 256, 6144), (32, 512, 2048), (33, 64, 2048),
                                   (200, 100, 96), (4096 + 7, 512, 256), (3, 8, 32)])
def test_router_logits_bit_exact(T, E, H):
    m = M()
    x = S.normal_cpu(T * H, 5, 0, 1.0).reshape(T, H)
    wr = S.normal_cpu(E * H, 6, 0, 1.0 / np.sqrt(H)).reshape(E, H)
    got = _np(m.moe_router_logits(torch.from_numpy(x).cuda(), torch.from_numpy(wr).cuda()))
    assert np.array_equal(got, O.router_logits(x, wr))


@pytest.mark.parametrize("score,renorm,rsf,E,k", [("softmax", True, 1.0, 64, 8), ("softmax", False, 1.0, 512, 10),
                                                   ("sigmoid", True, 2.5, 256, 8), ("sigmoid", False, 1.5, 40, 5),
                                                   ("softmax", True, 1.0, 7, 7), ("softmax", True, 1.0, 1024, 32)])
def test_route_topk_matches_oracle(score, renorm, rsf, E, k):
    m = M()
    T = 300
    L = S.normal_cpu(T * E, 7, 0, 1.0).reshape(T, E)
    L[:, ::3] = np.round(L[:, ::3])           # exact ties
    L[7] = 0.0
    bias = S.normal_cpu(E, 8, 0, 0.05) if score == "sigmoid" else None
    cfg = m.RouteCfg(score=score, top_k=k, renormalize=renorm, routed_scaling_factor=rsf)
    idx, w = m.moe_route_topk(torch.from_numpy(L).cuda(),
                              torch.from_numpy(bias).cuda() if bias is not None else None, cfg)
    ridx, rw = O.route(L, bias, score, k, renorm, rsf)
    assert np.array_equal(_np(idx), ridx)
    assert np.allclose(_np(w), rw, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T,k,E", [(1, 8, 64), (2, 2, 8), (31, 4, 16), (32, 8, 64), (33, 8, 64),
                                   (1000, 10, 512), (4096, 8, 64), (77, 1, 1024)])
def test_permute_matches_oracle(T, k, E):
    m = M()
    r = np.random.default_rng(T * 31 + k)
    idx = np.stack([r.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    offsets, perm, ws = m.moe_permute(torch.from_numpy(idx).cuda(), E)
    ro, rp = O.permute(idx, E)
    assert m.moe_read_device_status(ws) == m.MOE_OK
    assert np.array_equal(_np(offsets), ro)
    assert np.array_equal(_np(perm), rp)


def test_permute_flags_out_of_range_expert():
    """An expert id outside [0, E) is caught by the kernel's own bounds check: the pair is
    dropped and the device status word reports MOE_ERR_DEVICE_CHECK."""
    m = M()
    idx = np.array([[0, 1], [2, 9]], np.int32)
    offsets, perm, ws = m.moe_permute(torch.from_numpy(idx).cuda(), 4)
    assert m.moe_read_device_status(ws) == m.MOE_ERR_DEVICE_CHECK
    assert _np(offsets)[-1] == 3
    assert m.moe_read_device_status(ws) == m.MOE_OK


@pytest.mark.parametrize("wtype,wscale", [("int8", "g32_f16"), ("int4", "g32_f16"), ("int4", "row_f32"),
                                          ("int2", "g32_f16"), ("int2", "row_f32")])
def test_expert_group_dots_bit_exact(wtype, wscale):
    m = M()
    c = S.CONFIGS["olmoe_int8"].with_(E=4, H=512, I=256, wtype=wtype, wscale=wscale)
    case = S.Case.make(c, 1)
    gu = torch.empty((4, 512, 512), dtype=torch.float32, device="cuda")
    dn = torch.empty((4, 512, 256), dtype=torch.float32, device="cuda")
    case.gate_up_gpu(gu)
    case.down_gpu(dn)
    blob = m.ExpertBlob.quantize(gu, dn, wtype, wscale)
    ex = O.QExperts.quantize(_np(gu), _np(dn), wbits(c), wg32(c))
    r = np.random.default_rng(3)
    for which, K, nrows in ((0, 512, 512), (1, 256, 512)):
        n = 40
        e = r.integers(0, 4, n).astype(np.int32)
        row = r.integers(0, nrows, n).astype(np.int32)
        act = r.integers(-127, 128, (n, K)).astype(np.int8)
        dots = _np(m.moe_expert_group_dots(blob, which, torch.from_numpy(e).cuda(),
                                           torch.from_numpy(row).cuda(), torch.from_numpy(act).cuda()))
        for s in range(n):
            qw = ex.q_gu[e[s], row[s]] if which == 0 else ex.q_dn[e[s], row[s]]
            want = (qw.astype(np.int64) * act[s].astype(np.int64)).reshape(-1, 32).sum(1)
            assert np.array_equal(dots[s], want)


def test_zero_tokens_is_a_noop():
    m = M()
    case = S.Case.make(REDUCED["tiny"], 4)
    g = gpu_layer(case)
    y = torch.full((0, case.cfg.H), 7.0, device="cuda")
    x = torch.empty((0, case.cfg.H), device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    m.moe_layer_forward(x, g["wr"], None, g["blob"], None, route_cfg(case.cfg), y=y, workspace=ws)


def test_zero_input_gives_zero_output_and_first_experts():
    m = M()
    case = S.Case.make(REDUCED["olmoe_int8"], 3)
    g = gpu_layer(case)
    x = torch.zeros((3, case.cfg.H), device="cuda")
    cfg = route_cfg(case.cfg, m.MOE_FLAG_DEBUG)
    y, ws = m.moe_layer_forward(x, g["wr"], None, g["blob"], None, cfg)
    v = m.moe_layer_debug_views(3, g["blob"], None, cfg)
    idx = _np(m.workspace_view(ws, v["idx"], torch.int32, (3, case.cfg.top_k)))
    assert np.all(idx == np.arange(case.cfg.top_k))
    assert np.all(_np(y) == 0)


@pytest.mark.parametrize("k", [1, 16])
def test_extreme_top_k(k):
    """k = 1 and k = E (every expert; renormalised softmax = dense soft mixture)."""
    c = REDUCED["olmoe_int8"].with_(top_k=k)
    case = S.Case.make(c, 5)
    m = M()
    g = gpu_layer(case)
    y, ws = m.moe_layer_forward(g["x"], g["wr"], None, g["blob"], None, route_cfg(c))
    assert_close_y(_np(y), oracle_layer(case)["y"])


@pytest.mark.parametrize("wtype", ["int8", "int4"])
def test_tensor_core_dots_exact_at_extreme_codes(wtype):
    """The tensor-core path forms each group's dot with fp16 operands and an fp32
    accumulator; that is exact only because every partial sum is an integer below 2^24. Pin it
    where the sums are largest: x and every weight are +-1, so every activation code is +-127
    and every weight code +-127 (int8) or +-7 (int4), and half of the weight rows copy the sign
    pattern of token 0 (group dots up to 32 * 127 * 127). Gate/up stage values must equal the
    oracle's bit for bit."""
    m = M()
    rng = np.random.default_rng(77)
    E, H, I, T, k = 2, 256, 128, 40, 2
    x = np.where(rng.random((T, H)) < 0.5, -1.0, 1.0).astype(np.float32)
    gu = np.where(rng.random((E, 2 * I, H)) < 0.5, -1.0, 1.0).astype(np.float32)
    gu[:, ::2, :] = x[0]                       # rows whose dots with token 0 are maximal
    dn = np.where(rng.random((E, H, I)) < 0.5, -1.0, 1.0).astype(np.float32)
    wr = rng.normal(0.0, 1.0 / np.sqrt(H), (E, H)).astype(np.float32)
    wb = 8 if wtype == "int8" else 4
    ex = O.QExperts.quantize(gu, dn, wb, True)
    ref = O.layer_forward(x, wr, None, ex, None, "softmax", k, True, 1.0, True, union=True)
    blob = m.ExpertBlob.quantize(torch.from_numpy(gu).cuda(), torch.from_numpy(dn).cuda(), wtype, "g32_f16")
    cfg = m.RouteCfg(score="softmax", top_k=k, renormalize=True, routed_scaling_factor=1.0, act="g32_f16",
                     flags=m.MOE_FLAG_DEBUG | m.MOE_FLAG_FORCE_MMA)
    y, ws = m.moe_layer_forward(torch.from_numpy(x).cuda(), torch.from_numpy(wr).cuda(), None, blob, None, cfg)
    torch.cuda.synchronize()
    assert m.moe_read_device_status(ws) == m.MOE_OK
    v = m.moe_layer_debug_views(T, blob, None, cfg)
    view = lambda off, dt, shape: _np(m.workspace_view(ws, off, dt, shape))
    P = T * k
    perm = view(v["perm"], torch.int32, (P,))
    assert np.array_equal(perm, ref["perm"])
    gate = view(v["gate"], torch.float32, (P, I))
    up = view(v["up"], torch.float32, (P, I))
    assert np.abs(gate).max() > 0
    assert np.array_equal(gate, ref["gate"][perm]), "gate stage values"
    assert np.array_equal(up, ref["up"][perm]), "up stage values"
    assert np.array_equal(view(v["q_h"], torch.int8, (P, I)), ref["qh"][perm])
    ref["experts"] = (ex, None)
    _check_down_dots(m, ws, v, S.Case(S.CONFIGS["olmoe_int8"].with_(E=E, H=H, I=I, top_k=k, shared_I=0), T, 0),
                     ref, perm)
    assert_close_y(_np(y), ref["y"])


@pytest.mark.parametrize("wtype", ["int8", "int4", "int2"])
@pytest.mark.parametrize("path", ["mma", "stream"])
def test_down_dots_exact_at_extreme_codes(wtype, path):
    """The down projection at its largest group dots, on both expert paths: every gate and up
    row is the same +-1 pattern and every token agrees with it in most signs, so for each token
    all of its h values are equal and positive and every h code is +127; half of the down rows
    are all +1 (codes +127 / +7), the rest random
    signs, so group dots reach 32 * 127 * 127 (int8), 32 * 127 * 7 (int4) or 32 * 127 (int2) --
    partial sums far above fp16's integer range, exact only in the fp32 accumulator. The down
    group dots must
    equal the exact integer dots bit for bit, and y must meet the layer tolerance."""
    m = M()
    rng = np.random.default_rng(91)
    E, H, I, T, k = 2, 256, 128, 40, 2
    pat = np.where(rng.random(H) < 0.5, -1.0, 1.0).astype(np.float32)
    x = pat * np.where(rng.random((T, H)) < 0.3, -1.0, 1.0).astype(np.float32)   # gate values > 0
    x[0] = pat
    gu = np.broadcast_to(pat, (E, 2 * I, H)).copy()
    dn = np.where(rng.random((E, H, I)) < 0.5, -1.0, 1.0).astype(np.float32)
    dn[:, ::2, :] = 1.0
    wr = rng.normal(0.0, 1.0 / np.sqrt(H), (E, H)).astype(np.float32)
    wb = {"int8": 8, "int4": 4, "int2": 2}[wtype]
    ex = O.QExperts.quantize(gu, dn, wb, True)
    ref = O.layer_forward(x, wr, None, ex, None, "softmax", k, True, 1.0, True, union=True)
    ref["experts"] = (ex, None)
    assert (ref["qh"] == 127).all()
    blob = m.ExpertBlob.quantize(torch.from_numpy(gu).cuda(), torch.from_numpy(dn).cuda(), wtype, "g32_f16")
    force = m.MOE_FLAG_FORCE_MMA if path == "mma" else m.MOE_FLAG_FORCE_GEMV
    cfg = m.RouteCfg(score="softmax", top_k=k, renormalize=True, routed_scaling_factor=1.0, act="g32_f16",
                     flags=m.MOE_FLAG_DEBUG | force)
    y, ws = m.moe_layer_forward(torch.from_numpy(x).cuda(), torch.from_numpy(wr).cuda(), None, blob, None, cfg)
    torch.cuda.synchronize()
    assert m.moe_read_device_status(ws) == m.MOE_OK
    v = m.moe_layer_debug_views(T, blob, None, cfg)
    perm = _np(m.workspace_view(ws, v["perm"], torch.int32, (T * k,)))
    assert np.array_equal(perm, ref["perm"])
    assert np.array_equal(_np(m.workspace_view(ws, v["q_h"], torch.int8, (T * k, I))), ref["qh"][perm])
    case = S.Case(S.CONFIGS["olmoe_int8"].with_(E=E, H=H, I=I, top_k=k, shared_I=0), T, 0)
    _check_down_dots(m, ws, v, case, ref, perm)
    got = _np(m.workspace_view(ws, v["dn_dots"], torch.int32, (T * k, H, I // 32)))
    assert np.abs(got).max() == 32 * 127 * O.QMAX[wb]
    assert_close_y(_np(y), ref["y"])


def test_single_token_selection_ties_go_to_lower_experts():
    """x = 0 makes every router logit 0: the in-kernel selection of the single-token path
    (here 256 experts: four 64-expert chunks, then the candidates ranked against each other)
    must return experts 0 .. k-1 in that order, with equal softmax weights."""
    m = M()
    E, H, I, k = 256, 1024, 128, 8
    rng = np.random.default_rng(5)
    gu = rng.normal(0.0, 0.02, (E, 2 * I, H)).astype(np.float32)
    dn = rng.normal(0.0, 0.02, (E, H, I)).astype(np.float32)
    wr = rng.normal(0.0, 1.0 / np.sqrt(H), (E, H)).astype(np.float32)
    blob = m.ExpertBlob.quantize(torch.from_numpy(gu).cuda(), torch.from_numpy(dn).cuda(), "int8", "g32_f16")
    cfg = m.RouteCfg(score="softmax", top_k=k, renormalize=True, routed_scaling_factor=1.0, act="g32_f16",
                     flags=m.MOE_FLAG_DEBUG)
    assert m.moe_layer_kernel_count(1, blob, None, cfg) == 1          # the single-token kernel
    x = torch.zeros((1, H), dtype=torch.float32, device="cuda")
    y, ws = m.moe_layer_forward(x, torch.from_numpy(wr).cuda(), None, blob, None, cfg)
    torch.cuda.synchronize()
    assert m.moe_read_device_status(ws) == m.MOE_OK
    v = m.moe_layer_debug_views(1, blob, None, cfg)
    idx = _np(m.workspace_view(ws, v["idx"], torch.int32, (1, k)))
    w = _np(m.workspace_view(ws, v["w"], torch.float32, (1, k)))
    assert idx.tolist() == [list(range(k))]
    assert np.allclose(w, 1.0 / k, rtol=1e-6)
    assert np.array_equal(_np(y), np.zeros((1, H), np.float32))


@pytest.mark.parametrize("act", ["g32_f16", "token_f32"])
def test_quantize_activations_at_rounding_ties(act):
    """Codes decided at half-integers: every group's maximum is 127 * 2^-7 (so the scale is
    exactly 2^-7) and the other values are (j + 0.5) * 2^-7 -- exact ties, rounded half away
    from zero -- or one ulp either side of them. The kernel's reciprocal fast path must hand
    all of these to the exact division and match the oracle bit for bit."""
    m = M()
    H = 256
    rows = []
    for sign in (1.0, -1.0):
        for shift in (0, 1, -1):
            r = np.empty(H, np.float32)
            for g in range(H // 32):
                vals = np.array([(j % 126 + 0.5) * 2.0 ** -7 for j in range(g, g + 31)], np.float32) * sign
                if shift:
                    vals = np.nextafter(vals, np.float32(np.inf * shift)).astype(np.float32)
                r[32 * g] = 127 * 2.0 ** -7
                r[32 * g + 1:32 * g + 32] = vals
            rows.append(r)
    x = np.stack(rows)
    q, s = m.moe_quantize_activations(torch.from_numpy(x).cuda(), act)
    rq, rs = O.quantize_act(x, act == "g32_f16")
    assert np.array_equal(_np(q), rq)
    assert np.array_equal(_np(s).astype(np.float32), rs)
    if act == "g32_f16":
        assert (np.abs(rq[:2]) % 1 == 0).all() and np.any(np.abs(rq[0]) == 127)
