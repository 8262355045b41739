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

