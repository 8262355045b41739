"""Expert parallelism, host side (CPU, no GPU): the expert placement and the exchange of one
step, run as two gloo ranks. Each rank holds half of the experts; its partial layer -- here the
oracle restricted to the rank's experts, standing in for the CUDA layer the rank would run --
adds only the pairs whose expert it holds (the shared expert on rank 0). After the all-gather of
x and the reduce-scatter of y, every rank's rows must equal the oracle's whole layer, and the
(token, slot) pairs the ranks computed must cover every routed pair exactly once."""
import datetime
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

import synth as S

CFG = S.CONFIGS["olmoe_int8"].with_(name="ep_small", H=256, E=8, I=128, top_k=3, shared_I=128)
T_LOCAL = 3


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_parts(x_all):
    """Per-pair expert outputs, routing and the shared expert of the whole layer (oracle)."""
    import oracle as O
    case = S.Case.make(CFG, 2 * T_LOCAL)
    ex = O.QExperts.quantize(np.stack([case.gate_up(e) for e in range(CFG.E)]),
                             np.stack([case.down(e) for e in range(CFG.E)]), 8, True)
    sh = O.QExperts.quantize(case.shared_gate_up()[None], case.shared_down()[None], 8, True)
    return O.layer_forward(x_all, case.router_w(), case.bias(), ex, sh, CFG.score, CFG.top_k,
                           CFG.renormalize, CFG.rsf, True)


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from quantized_expert_ffn_logits_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        begin, count = ep.expert_ranges(CFG.E, world)[rank]
        x_local = torch.from_numpy(S.normal_cpu(T_LOCAL * CFG.H, 500 + rank, 0, 1.0).reshape(T_LOCAL, CFG.H))
        computed = []

        def partial(x_all):
            o = _oracle_parts(x_all.numpy())
            T, k = o["idx"].shape
            y = np.zeros((T, CFG.H))
            for t in range(T):
                for j in range(k):
                    e = int(o["idx"][t, j])
                    if begin <= e < begin + count:
                        y[t] += o["w"][t, j] * o["ye"][t * k + j]
                        computed.append((t, j))
                if rank == 0:
                    y[t] += o["ysh"][t]
            return torch.from_numpy(y)

        y = ep.ep_step(x_local.double(), partial)
        pairs = [None] * world
        dist.all_gather_object(pairs, computed)
        xs = [torch.empty_like(x_local) for _ in range(world)]
        dist.all_gather(xs, x_local)
    finally:
        dist.destroy_process_group()
    q.put((rank, y.numpy(), pairs, torch.cat(xs).numpy()))


def test_two_rank_expert_parallel_step_equals_the_whole_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    x_all = res[0][3]
    ref = _oracle_parts(x_all)
    for rank, y, pairs, _ in res:
        want = ref["y"][rank * T_LOCAL:(rank + 1) * T_LOCAL]
        assert np.allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    a, b = set(res[0][2][0]), set(res[0][2][1])
    assert not a & b, "a pair computed on both ranks"
    assert a | b == {(t, j) for t in range(2 * T_LOCAL) for j in range(CFG.top_k)}


def test_expert_ranges_cover_the_experts():
    from quantized_expert_ffn_logits_b200 import ep
    for E, world in ((8, 2), (64, 8), (10, 3), (512, 7)):
        r = ep.expert_ranges(E, world)
        assert r[0][0] == 0 and sum(c for _, c in r) == E
        assert all(r[i][0] + r[i][1] == r[i + 1][0] for i in range(world - 1))
        assert max(c for _, c in r) - min(c for _, c in r) <= 1
    with pytest.raises(ValueError):
        ep.expert_ranges(2, 3)


def test_least_loaded_placement():
    """Greedy whole-expert placement: experts by decreasing load onto the least-loaded rank
    with room; each rank gets at most ceil(E / world); the result is a renumbering that lists
    rank 0's experts first. Pinned on a hand-worked case and on the greedy bound."""
    from quantized_expert_ffn_logits_b200 import ep
    order, ranges = ep.place_experts([5, 1, 4, 2, 3, 3], 2)
    # e0 (5) -> r0 [5]; e2 (4) -> r1 [4]; e4 (3) -> r1 [7]; e5 (3) -> r0 [10]; e3 (2) -> r1 [9],
    # which is then full (cap 3); e1 (1) -> r0 [11]
    assert ranges == [(0, 3), (3, 3)]
    assert sorted(order.tolist()) == list(range(6))
    assert set(order[:3].tolist()) == {0, 5, 1} and set(order[3:].tolist()) == {2, 4, 3}
    rng = np.random.default_rng(3)
    for E, world in ((64, 8), (256, 4), (30, 7)):
        load = rng.zipf(1.5, E).astype(float)
        order, ranges = ep.place_experts(load, world)
        assert sorted(order.tolist()) == list(range(E))
        per = [load[order[b:b + c]].sum() for b, c in ranges]
        assert max(c for _, c in ranges) <= -(-E // world)
        assert abs(sum(per) - load.sum()) < 1e-9
    import torch
    idx = torch.tensor([[0, 2, -1], [5, 1, 3]], dtype=torch.int32)
    order = np.array([3, 0, 5, 1, 4, 2])
    got = ep.original_ids(idx, order)
    assert got.tolist() == [[3, 5, -1], [2, 0, 1]]
    rw = np.arange(12, dtype=np.float32).reshape(6, 2)
    rw2, _ = ep.renumber(order, rw)
    assert np.array_equal(rw2[1], rw[0]) and np.array_equal(rw2[0], rw[3])


# all-to-all exchange: ranks with different token counts (one with a single token, one with none)
A2A_SPLITS = [[4, 1, 6], [3, 0, 5, 2]]


def _oracle_x(x):
    """The oracle's whole layer on rows x with the weights of one fixed case."""
    import oracle as O
    case = S.Case.make(CFG, 1)
    ex = O.QExperts.quantize(np.stack([case.gate_up(e) for e in range(CFG.E)]),
                             np.stack([case.down(e) for e in range(CFG.E)]), 8, True)
    sh = O.QExperts.quantize(case.shared_gate_up()[None], case.shared_down()[None], 8, True)
    return O.layer_forward(x, case.router_w(), case.bias(), ex, sh, CFG.score, CFG.top_k,
                           CFG.renormalize, CFG.rsf, True)


def _worker_a2a(rank, world, port, q, t_a2a):
    import torch
    import torch.distributed as dist
    from quantized_expert_ffn_logits_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ranges = ep.expert_ranges(CFG.E, world)
        begin, count = ranges[rank]
        n = t_a2a[rank]
        x_local = torch.from_numpy(S.normal_cpu(max(n, 1) * CFG.H, 700 + rank, 0, 1.0).reshape(max(n, 1), CFG.H)[:n])
        npairs = [0, 0]

        def local_sum(x, with_shared):
            if x.shape[0] == 0:
                return x.new_zeros((0, CFG.H)), torch.zeros((0, CFG.top_k), dtype=torch.int64)
            o = _oracle_x(x.numpy())
            T, k = o["idx"].shape
            y = np.zeros((T, CFG.H))
            for t in range(T):
                for j in range(k):
                    e = int(o["idx"][t, j])
                    if begin <= e < begin + count:
                        y[t] += o["w"][t, j] * o["ye"][t * k + j]
                        npairs[0] += 1
                if with_shared:
                    y[t] += o["ysh"][t]
                    npairs[1] += 1
            return torch.from_numpy(y), torch.from_numpy(o["idx"].astype(np.int64))

        def partial(x):
            if x.shape[0] == 0:
                return x.new_zeros((0, CFG.H))
            return local_sum(x, False)[0]

        y = ep.ep_step_a2a(x_local.double(), ranges, lambda x: local_sum(x, True), partial)
        xs = [None] * world
        dist.all_gather_object(xs, x_local.numpy())
        counts = [None] * world
        dist.all_gather_object(counts, npairs)
    finally:
        dist.destroy_process_group()
    q.put((rank, y.numpy(), counts, np.concatenate(xs)))


@pytest.mark.parametrize("t_a2a", A2A_SPLITS)
def test_all_to_all_step_equals_the_whole_layer(t_a2a):
    """ep_step_a2a on gloo ranks holding 4, 1 and 6 tokens, or 3, 0, 5 and 2 (uneven splits,
    empty ones, a rank with no tokens at all): every rank's rows equal the oracle's whole layer
    on all tokens, every routed pair is computed exactly once over all ranks (on the rank holding
    its expert), and the shared expert once per token (on the token's rank)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = len(t_a2a)
    procs = [ctx.Process(target=_worker_a2a, args=(r, world, port, q, t_a2a)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    x_all = res[0][3]
    ref = _oracle_x(x_all)
    st = np.cumsum([0] + t_a2a)
    for rank, y, _, _ in res:
        want = ref["y"][st[rank]:st[rank + 1]]
        assert y.shape == want.shape
        if want.size:
            assert np.allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    counts = res[0][2]
    assert sum(c[0] for c in counts) == sum(t_a2a) * CFG.top_k
    assert [c[1] for c in counts] == t_a2a


def test_dispatch_plan_and_combine():
    """a2a_plan on a hand-made routing: a token goes once to each other rank holding one of its
    experts (dropped slots -1 go nowhere), grouped by rank in ascending token order;
    a2a_combine adds the returned rows in that order."""
    import torch
    from quantized_expert_ffn_logits_b200 import ep
    ranges = [(0, 3), (3, 3), (6, 2)]
    idx = torch.tensor([[0, 4], [6, -1], [1, 2], [3, 7], [-1, -1]])
    send, counts = ep.a2a_plan(idx, ranges, 0)
    assert counts == [0, 2, 2] and send.tolist() == [0, 3, 1, 3]
    send1, counts1 = ep.a2a_plan(idx, ranges, 1)
    assert counts1 == [2, 0, 2] and send1.tolist() == [0, 2, 1, 3]
    y = torch.zeros(5, 2, dtype=torch.float64)
    back = torch.arange(8, dtype=torch.float64).reshape(4, 2)
    ep.a2a_combine(y, send, counts, back)
    assert y.tolist() == [[0, 1], [4, 5], [0, 0], [8, 10], [0, 0]]
