"""Expert parallelism through the CUDA layer, on one GPU: the experts split into disjoint
ranges, one layer call per range (moe_route_cfg.n_experts_total / expert_begin, the shared
expert with the first range only), as the ranks of an expert-parallel layer would run them.
Every call must route every token over all experts -- the same global idx as the oracle's --
and group only the pairs of its own range; the sum of the calls' outputs must meet the layer
tolerance against the oracle's whole layer. Paths: the single-token kernel, the fused routing
kernel, the four-launch routing with the tensor-core GEMMs, per-token activation scales."""
import numpy as np
import pytest

import oracle as O
import synth as S
from helpers import assert_close_y, oracle_layer, route_cfg, wbits, wg32

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

BASE = S.CONFIGS
CASES = [
    (BASE["olmoe_int8"].with_(name="ep_olmoe_r", H=512, E=16, I=256, top_k=4), 1, [(0, 8), (8, 8)], 0),
    (BASE["olmoe_int8"].with_(name="ep_olmoe_r", H=512, E=16, I=256, top_k=4), 8, [(0, 5), (5, 6), (11, 5)], 0),
    (BASE["olmoe_int4"].with_(name="ep_olmoe4_r", H=512, E=16, I=256, top_k=4), 70, [(0, 7), (7, 9)], 4),
    (BASE["glm_int4"].with_(name="ep_glm_r", H=768, E=32, I=256, top_k=4, shared_I=128), 1, [(0, 16), (16, 16)], 0),
    (BASE["glm_int4"].with_(name="ep_glm_r", H=768, E=32, I=256, top_k=4, shared_I=128), 4, [(0, 10), (10, 22)], 0),
    (BASE["e512_int4"].with_(name="ep_e512_r", H=512, E=64, I=128, top_k=6, shared_I=128), 40, [(0, 32), (32, 32)], 0),
    (BASE["tiny"], 4, [(0, 3), (3, 5)], 0),
]


@pytest.mark.parametrize("cfg,T,ranges,force", CASES)
def test_expert_ranges_sum_to_the_layer(cfg, T, ranges, force):
    import quantized_expert_ffn_logits_b200 as M
    case = S.Case.make(cfg, T)
    c = cfg
    gu = torch.empty((c.E, 2 * c.I, c.H), dtype=torch.float32, device="cuda")
    dn = torch.empty((c.E, c.H, c.I), dtype=torch.float32, device="cuda")
    case.gate_up_gpu(gu)
    case.down_gpu(dn)
    shared = None
    if c.shared_I:
        sgu = torch.empty((1, 2 * c.shared_I, c.H), dtype=torch.float32, device="cuda")
        sdn = torch.empty((1, c.H, c.shared_I), dtype=torch.float32, device="cuda")
        case.shared_gate_up_gpu(sgu)
        case.shared_down_gpu(sdn)
        shared = M.ExpertBlob.quantize(sgu, sdn, c.wtype, c.wscale)
    wr = torch.from_numpy(case.router_w()).cuda()
    b = case.bias()
    bias = torch.from_numpy(b).cuda() if b is not None else None
    x = torch.from_numpy(case.x()).cuda()
    ref = oracle_layer(case, union=True)
    y_sum = np.zeros((T, c.H))
    flags = M.MOE_FLAG_DEBUG | (M.MOE_FLAG_FORCE_MMA if force else 0)
    for i, (e0, n) in enumerate(ranges):
        blob = M.ExpertBlob.quantize(gu[e0:e0 + n].contiguous(), dn[e0:e0 + n].contiguous(), c.wtype, c.wscale)
        cfg_r = route_cfg(c, flags=flags)
        cfg_r.n_experts_total, cfg_r.expert_begin = c.E, e0
        y, ws = M.moe_layer_forward(x, wr, bias, blob, shared if i == 0 else None, cfg_r)
        torch.cuda.synchronize()
        assert M.moe_read_device_status(ws) == M.MOE_OK
        v = M.moe_layer_debug_views(T, blob, shared if i == 0 else None, cfg_r)
        view = lambda off, dt, shape: M.workspace_view(ws, off, dt, shape).cpu().numpy()
        assert np.array_equal(view(v["idx"], torch.int32, (T, c.top_k)), ref["idx"]), "global selection"
        assert np.array_equal(view(v["logits"], torch.float32, (T, c.E)), ref["logits"])
        # the grouping of this range: its pairs, by local id, in (expert, token) order
        mine = [(e - e0, t * c.top_k + j) for t in range(T) for j in range(c.top_k)
                for e in [int(ref["idx"][t, j])] if e0 <= e < e0 + n]
        mine.sort()
        offsets = view(v["offsets"], torch.int32, (n + 1,))
        assert offsets[-1] == len(mine)
        assert np.array_equal(view(v["perm"], torch.int32, (len(mine),)), [p for _, p in mine])
        y_sum += y.cpu().numpy().astype(np.float64)
    assert_close_y(y_sum, ref["y"])


# (config, tokens on each rank, each rank's expert range)
A2A_CASES = [
    (BASE["olmoe_int4"].with_(name="ep_olmoe4_r", H=512, E=16, I=256, top_k=4), [40, 7, 33],
     [(0, 6), (6, 5), (11, 5)]),
    (BASE["glm_int4"].with_(name="ep_glm_r", H=768, E=32, I=256, top_k=4, shared_I=128), [5, 1, 12],
     [(0, 10), (10, 12), (22, 10)]),
]


@pytest.mark.parametrize("cfg,t_local,ranges", A2A_CASES)
def test_all_to_all_dispatch_and_combine(cfg, t_local, ranges):
    """All-to-all expert parallelism emulated on one GPU (the exchange done by indexing): W ranks,
    each with its own tokens and expert range. EPLayerA2A.home runs the rank's layer on its own
    tokens with the shared expert, which also routes them; a2a_plan sends every token once to
    each other rank holding one of its selected experts; EPLayerA2A.partial runs that rank's
    layer (experts only) on what it received, which routes the rows again; a2a_combine adds the
    returned rows on the token's rank. Every rank's home routing equals the oracle's, and every
    rank's rows meet the layer tolerance against the oracle's whole layer on all tokens. Token
    counts on either side of the 32-token routing switch and a single-token rank."""
    import quantized_expert_ffn_logits_b200 as M
    from quantized_expert_ffn_logits_b200 import ep
    c = cfg
    W, T = len(ranges), sum(t_local)
    case = S.Case.make(c, T)
    gu = torch.empty((c.E, 2 * c.I, c.H), dtype=torch.float32, device="cuda")
    dn = torch.empty((c.E, c.H, c.I), dtype=torch.float32, device="cuda")
    case.gate_up_gpu(gu)
    case.down_gpu(dn)
    shared = None
    if c.shared_I:
        sgu = torch.empty((1, 2 * c.shared_I, c.H), dtype=torch.float32, device="cuda")
        sdn = torch.empty((1, c.H, c.shared_I), dtype=torch.float32, device="cuda")
        case.shared_gate_up_gpu(sgu)
        case.shared_down_gpu(sdn)
        shared = M.ExpertBlob.quantize(sgu, sdn, c.wtype, c.wscale)
    wr = torch.from_numpy(case.router_w()).cuda()
    b = case.bias()
    bias = torch.from_numpy(b).cuda() if b is not None else None
    x = torch.from_numpy(case.x()).cuda()
    ref = oracle_layer(case)
    st = np.cumsum([0] + t_local)
    layers = []
    for r, (e0, n) in enumerate(ranges):
        blob = M.ExpertBlob.quantize(gu[e0:e0 + n].contiguous(), dn[e0:e0 + n].contiguous(), c.wtype, c.wscale)
        layers.append(ep.EPLayerA2A(blob, shared, route_cfg(c), wr, bias, ranges, r, t_local[r], T))
    homes = [layers[r].home(x[st[r]:st[r + 1]]) for r in range(W)]
    plans = [ep.a2a_plan(homes[r][1], ranges, r) for r in range(W)]
    for r in range(W):
        assert plans[r][1][r] == 0
        assert np.array_equal(homes[r][1].cpu().numpy(), ref["idx"][st[r]:st[r + 1]]), f"rank {r} routing"
    # rank d receives, from every source s in rank order, the rows s planned for d
    y_recv = []
    for d in range(W):
        rows = [x[st[s]:st[s + 1]][plans[s][0][sum(plans[s][1][:d]):sum(plans[s][1][:d + 1])]] for s in range(W)]
        y_recv.append(layers[d].partial(torch.cat(rows)))
    torch.cuda.synchronize()
    for r in range(W):
        assert M.moe_read_device_status(layers[r]._ws_home) == M.MOE_OK
        assert M.moe_read_device_status(layers[r]._ws_recv) == M.MOE_OK
    for s in range(W):
        back = []
        for d in range(W):
            off = sum(plans[q][1][d] for q in range(s))
            back.append(y_recv[d][off:off + plans[s][1][d]])
        y = ep.a2a_combine(homes[s][0].clone(), plans[s][0], plans[s][1], torch.cat(back))
        assert_close_y(y.cpu().numpy(), ref["y"][st[s]:st[s + 1]], f"rank {s}")
