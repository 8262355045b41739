"""GPU parity at the five workloads' full sizes, in the launch configuration bench.py times
(one moe_layer_forward call over the whole batch, no debug copies): every output row of the
decode batches; for the larger batches a seeded sample of tokens, which the oracle computes
one by one, regenerating only the experts those tokens use. Routing indices of the compared
tokens are bit-exact; their output rows meet the layer tolerance (rel-L2 1e-5, max-abs
1e-4 * max|y|)."""
import numpy as np
import pytest

import synth as S
from helpers import assert_close_y, gpu_layer, oracle_tokens, route_cfg

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

# (workload, T, tokens compared: None = all)
FULL = [
    ("tiny", 4, None),
    ("olmoe_int8", 1, None),
    ("olmoe_int8", 8, None),
    ("glm_int4", 1, None),
    ("glm_int4", 4, 2),
    ("e512_int4", 1, None),
    ("e512_int4", 64, 8),
    ("olmoe_int4", 512, 6),        # tensor-core path (experts with >= 16 pairs)
    ("olmoe_int4", 4096, 4),
    ("e512_int4", 4096, 4),        # Zipf-skewed: tensor cores for hot experts, streaming for the rest
]


@pytest.mark.parametrize("name,T,sample", FULL)
def test_full_size_layer(name, T, sample):
    import quantized_expert_ffn_logits_b200 as M
    c = S.CONFIGS[name]
    case = S.Case.make(c, T)
    g = gpu_layer(case)
    cfg = route_cfg(c)
    y, ws = M.moe_layer_forward(g["x"], g["wr"], g["bias"], g["blob"], g["shared"], cfg)
    torch.cuda.synchronize()
    assert M.moe_read_device_status(ws) == M.MOE_OK
    yg = y.cpu().numpy()
    assert np.isfinite(yg).all()
    rng = np.random.default_rng(1234 + T)
    toks = list(range(T)) if sample is None else sorted(rng.choice(T, size=sample, replace=False).tolist())
    ref = oracle_tokens(case, toks)
    v = M.moe_layer_debug_views(T, g["blob"], g["shared"], cfg)
    idx = M.workspace_view(ws, v["idx"], torch.int32, (T, c.top_k)).cpu().numpy()
    assert np.array_equal(idx[toks], ref["idx"])
    assert_close_y(yg[toks], ref["y"])
    del g, y, ws
    torch.cuda.empty_cache()
