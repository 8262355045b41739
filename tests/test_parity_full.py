"""GPU parity at the five workloads' full sizes, in the launch configuration bench.py times
(one moe_layer_forward call over the whole batch, no debug copies): every output row of the
decode batches; for the larger batches a seeded sample of tokens, which the oracle computes
one by one, regenerating only the experts those tokens use. Where some experts of the batch
run on the tensor cores (at least 16 pairs) and others are streamed, half of the sample is
drawn from the tokens routed to a streamed expert, so both paths are compared at their
full-size tile counts. Routing indices of the compared tokens are bit-exact; their output
rows meet the layer tolerance (rel-L2 1e-5, max-abs 1e-4 * max|y|)."""
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
    ("e512_int4", 64, None),       # Zipf-skewed: the hottest experts on the tensor cores
    ("olmoe_int4", 512, 32),       # tensor-core path (experts with >= 16 pairs)
    ("olmoe_int4", 4096, 64),
    ("e512_int4", 4096, 64),       # Zipf-skewed: tensor cores for hot experts, streaming for the rest
    ("olmoe_int2", 1, None),       # packed int2 experts: the single-token kernel
    ("olmoe_int2", 8, None),
]
MMA_MIN_PAIRS = 16                 # pairs an expert needs in a call for the tensor-core path


def _sample(idx, T, n, seed):
    """n tokens: half (when there are any) routed to an expert with fewer than MMA_MIN_PAIRS
    pairs in the batch (the streaming path), the rest at random."""
    rng = np.random.default_rng(seed)
    counts = np.bincount(idx[idx >= 0].reshape(-1), minlength=int(idx.max()) + 1)
    cold = np.nonzero(np.isin(idx, np.nonzero(counts < MMA_MIN_PAIRS)[0]).any(axis=1))[0]
    pick = set(rng.choice(cold, size=min(n // 2, len(cold)), replace=False).tolist()) if len(cold) else set()
    rest = [t for t in rng.permutation(T).tolist() if t not in pick]
    pick.update(rest[: n - len(pick)])
    return sorted(pick), len(cold), int((counts >= MMA_MIN_PAIRS).sum())


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
    v = M.moe_layer_debug_views(T, g["blob"], g["shared"], cfg)
    idx = M.workspace_view(ws, v["idx"], torch.int32, (T, c.top_k)).cpu().numpy()
    if sample is None:
        toks = list(range(T))
    else:
        toks, n_cold, n_hot = _sample(idx, T, sample, 1234 + T)
        if name == "e512_int4" and T == 4096:       # the mixed case must reach both paths
            assert n_cold > 0 and n_hot > 0
            assert any(np.isin(idx[t], np.nonzero(np.bincount(idx.reshape(-1)) < MMA_MIN_PAIRS)[0]).any()
                       for t in toks)
    ref = oracle_tokens(case, toks)
    assert np.array_equal(idx[toks], ref["idx"])
    assert_close_y(yg[toks], ref["y"])
    del g, y, ws
    torch.cuda.empty_cache()


def test_full_size_host_buffers_single_token():
    """moe_layer_forward_host at the full OLMoE int8 size with one token (the single-token
    kernel with the grid barrier between the input and output copy kernels): four different
    tokens enqueued back to back, each into its own page-locked output, against the oracle on
    its own x."""
    import quantized_expert_ffn_logits_b200 as M
    c = S.CONFIGS["olmoe_int8"]
    case = S.Case.make(c, 1)
    g = gpu_layer(case)
    lay = M.Layer(1, g["blob"], g["shared"], route_cfg(c), g["wr"], g["bias"])
    xs = [case.x()] + [S.normal_cpu(c.H, 5151 + i, 0, c.x_sigma).reshape(1, c.H) for i in range(3)]
    xh = [torch.from_numpy(x).pin_memory() for x in xs]
    yh = [torch.full((1, c.H), float("nan"), dtype=torch.float32).pin_memory() for _ in xs]
    for a, b in zip(xh, yh):
        lay.forward_host(a, b)
    torch.cuda.synchronize()
    assert M.moe_read_device_status(lay.workspace) == M.MOE_OK
    for i, x in enumerate(xs):
        assert_close_y(yh[i].numpy(), oracle_tokens(case, [0], x=x)["y"], f"call {i}")
    del g, lay
    torch.cuda.empty_cache()
