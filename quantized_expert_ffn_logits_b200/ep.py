"""Expert parallelism: the layer's experts spread over several GPUs (one process per GPU).

The GLM-5.2 colibri page ("Experimental resident CUDA backend") places whole experts on
devices, each on the least-loaded one. Here each rank holds a contiguous range of the (possibly
renumbered) experts in its own blob, and one step of the layer is

  1. all-gather x: every rank gets the tokens of all ranks;
  2. the local layer (moe_layer_forward with moe_route_cfg.n_experts_total / expert_begin):
     every token is routed over all experts -- the same selection on every rank -- and only
     the pairs whose expert is held here are computed and added into this rank's y (the shared
     expert on rank 0 only);
  3. reduce-scatter y: the partial outputs summed over ranks, each rank keeping its own
     tokens' rows.

This is the exchange for small token counts (decode, MTP verification), where the routed
copies an all-to-all dispatch would send are about as many as the tokens themselves. Every
rank must pass the same number of tokens.

For large token counts (prefill) the exchange is an all-to-all dispatch and combine
(ep_step_a2a, EPLayerA2A): each rank runs the layer on its own tokens (its experts and the
shared expert), which also routes them; every token then goes, once, to each other rank that
holds one of its selected experts; that rank runs the layer on what it received (its experts
only; the routing it recomputes is the same, bit for bit) and the partial rows travel back to be
added on the token's rank. Ranks may pass different numbers of tokens.

Routing and expert compute run in the CUDA kernels; this module only places experts, plans the
exchange and moves tensors with torch.distributed.
"""
from __future__ import annotations

import dataclasses

import numpy as np


def expert_ranges(n_experts: int, world: int):
    """Contiguous, balanced ranges: rank r holds experts begin_r .. begin_r + count_r - 1."""
    if world < 1 or n_experts < world:
        raise ValueError("need 1 <= world <= n_experts")
    base, extra = divmod(n_experts, world)
    out, b = [], 0
    for r in range(world):
        c = base + (1 if r < extra else 0)
        out.append((b, c))
        b += c
    return out


def place_experts(load, world: int):
    """Whole-expert placement on the least-loaded rank (the GLM page's rule), experts taken in
    decreasing load, ties to the lower expert id and then the lower rank, with at most
    ceil(E / world) experts per rank. Returns (order, ranges): order[i] is the original id of
    renumbered expert i (rank 0's experts first, each rank's in ascending original id), ranges
    as expert_ranges gives them for the renumbered experts. Renumbering experts (router rows,
    bias entries and blob slices permuted by `order`) changes which expert wins an exact tie
    of selection keys, nothing else."""
    load = np.asarray(load, dtype=np.float64)
    E = load.size
    if world < 1 or E < world:
        raise ValueError("need 1 <= world <= n_experts")
    cap = -(-E // world)
    rank_load = np.zeros(world)
    members = [[] for _ in range(world)]
    for e in sorted(range(E), key=lambda i: (-load[i], i)):
        open_ranks = [r for r in range(world) if len(members[r]) < cap]
        r = min(open_ranks, key=lambda q: (rank_load[q], q))
        members[r].append(e)
        rank_load[r] += load[e]
    order = np.array([e for r in range(world) for e in sorted(members[r])], dtype=np.int64)
    ranges, b = [], 0
    for r in range(world):
        ranges.append((b, len(members[r])))
        b += len(members[r])
    return order, ranges


def renumber(order, router_w, router_bias=None):
    """Router rows (and bias entries) in the renumbered expert order (tensors or arrays)."""
    rw = router_w[order]
    rb = None if router_bias is None else router_bias[order]
    return rw, rb


def original_ids(idx, order):
    """Selected experts of the renumbered layer as original ids (-1 stays -1)."""
    import torch
    o = torch.as_tensor(order, device=idx.device, dtype=torch.int64)
    out = torch.where(idx >= 0, o[idx.clamp(min=0).long()], torch.full_like(idx.long(), -1))
    return out.to(idx.dtype)


def ep_route_cfg(cfg, n_experts_total: int, expert_begin: int):
    """A RouteCfg restricted to one rank's expert range."""
    return dataclasses.replace(cfg, n_experts_total=int(n_experts_total), expert_begin=int(expert_begin))


def ep_step(x_local, partial, group=None):
    """One expert-parallel step around `partial` (x_all [world * T][H] -> this rank's partial y,
    same shape): all-gather x, partial, reduce-scatter y. Returns this rank's y [T][H]."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T = x_local.shape[0]
    xs = [torch.empty_like(x_local) for _ in range(world)]
    dist.all_gather(xs, x_local.contiguous(), group=group)
    y_part = partial(torch.cat(xs)).contiguous()
    if dist.get_backend(group) == "nccl":
        y = torch.empty_like(x_local)
        dist.reduce_scatter_tensor(y, y_part, group=group)
        return y
    dist.all_reduce(y_part, group=group)          # (the CPU backend has no reduce-scatter)
    return y_part[rank * T:(rank + 1) * T].clone()


class EPLayer:
    """One rank's share of an expert-parallel layer: its experts' blob (global ids
    expert_begin ..), the whole router, the shared expert on rank 0 only."""

    def __init__(self, T_local: int, world: int, experts, shared, cfg, router_w, router_bias=None,
                 expert_begin: int = 0):
        from . import Layer
        self.world = world
        E_total = router_w.shape[0]
        self.cfg = ep_route_cfg(cfg, E_total, expert_begin)
        self.layer = Layer(T_local * world, experts, shared, self.cfg, router_w, router_bias)
        self._y = None

    def __call__(self, x_local, group=None, stream=None):
        import torch

        def partial(x_all):
            if self._y is None or self._y.shape != x_all.shape:
                self._y = torch.empty_like(x_all)
            return self.layer(x_all, self._y, stream)
        return ep_step(x_local, partial, group)


def a2a_plan(idx, ranges, rank):
    """Dispatch plan of this rank's tokens: token t goes to every other rank r holding one of
    its selected experts (idx [T][k] global ids, -1 = a dropped slot; ranges as expert_ranges
    gives them). Returns (send_idx, counts): the token indices grouped by destination rank in
    rank order, ascending within a rank, and how many go to each rank (none to this rank, whose
    own layer call covers its experts)."""
    import torch
    idx = torch.as_tensor(idx)
    parts, counts = [], []
    for r, (b, c) in enumerate(ranges):
        if r == rank or c == 0:
            counts.append(0)
            continue
        t = torch.nonzero(((idx >= b) & (idx < b + c)).any(dim=1)).flatten()
        parts.append(t)
        counts.append(int(t.numel()))
    send_idx = torch.cat(parts) if parts else torch.empty(0, dtype=torch.long, device=idx.device)
    return send_idx.to(torch.long), counts


def a2a_combine(y, send_idx, counts, y_back):
    """Adds the partial rows that came back (y_back, in the order of send_idx) into this rank's
    y [T][H], one destination rank at a time in rank order (a token appears at most once per
    rank, so each add is free of collisions and the sum order is fixed)."""
    off = 0
    for n in counts:
        if n:
            y.index_add_(0, send_idx[off:off + n], y_back[off:off + n])
        off += n
    return y


def ep_step_a2a(x_local, ranges, home, partial, group=None):
    """One expert-parallel step with all-to-all dispatch and combine. home(x_local) -> (y, idx):
    this rank's layer on its own tokens (its experts and the shared expert) and the routing it
    made (idx [T][k] global ids); partial(x_recv) -> y_recv: this rank's experts on the tokens it
    received. Returns this rank's y [T][H]."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    y, idx = home(x_local)
    send_idx, counts = a2a_plan(idx, ranges, rank)
    cnt = torch.tensor(counts, dtype=torch.int64, device=x_local.device)
    rcnt = torch.empty_like(cnt)
    dist.all_to_all_single(rcnt, cnt, group=group)
    rcounts = [int(v) for v in rcnt.tolist()]
    H = x_local.shape[1]
    x_send = x_local.index_select(0, send_idx.to(x_local.device)).contiguous()
    x_recv = x_local.new_empty((sum(rcounts), H))
    dist.all_to_all_single(x_recv, x_send, rcounts, counts, group=group)
    y_recv = partial(x_recv).contiguous()
    y_back = y.new_empty((sum(counts), H))
    dist.all_to_all_single(y_back, y_recv, counts, rcounts, group=group)
    assert len(counts) == world
    return a2a_combine(y, send_idx.to(y.device), counts, y_back)


class EPLayerA2A:
    """One rank's share of an expert-parallel layer with all-to-all dispatch and combine: its
    experts' blob (global ids expert_begin ..), the whole router, the shared expert (every rank
    runs it for its own tokens). Workspaces are sized for t_local own tokens and t_recv
    received ones (at most t_local of every other rank)."""

    def __init__(self, experts, shared, cfg, router_w, router_bias, ranges, rank, t_local, t_recv):
        import torch
        from . import moe_layer_workspace_bytes
        self.ranges, self.rank = ranges, rank
        self.experts, self.shared = experts, shared
        self.router_w, self.router_bias = router_w, router_bias
        self.cfg = ep_route_cfg(cfg, router_w.shape[0], ranges[rank][0])
        dev = router_w.device
        nh = moe_layer_workspace_bytes(max(t_local, 1), experts, shared, self.cfg)
        nr = moe_layer_workspace_bytes(max(t_recv, 1), experts, None, self.cfg)
        self._ws_home = torch.zeros(nh, dtype=torch.uint8, device=dev)     # control blocks zeroed
        self._ws_recv = torch.zeros(nr, dtype=torch.uint8, device=dev)

    def home(self, x_local):
        import torch
        from . import moe_layer_forward, moe_layer_debug_views, workspace_view
        T = x_local.shape[0]
        y, ws = moe_layer_forward(x_local, self.router_w, self.router_bias, self.experts, self.shared,
                                  self.cfg, workspace=self._ws_home)
        v = moe_layer_debug_views(T, self.experts, self.shared, self.cfg)
        idx = workspace_view(ws, v["idx"], torch.int32, (T, self.cfg.top_k))
        return y, idx

    def partial(self, x_recv):
        from . import moe_layer_forward
        if x_recv.shape[0] == 0:
            return x_recv.new_zeros((0, x_recv.shape[1]))
        y, _ = moe_layer_forward(x_recv.contiguous(), self.router_w, self.router_bias, self.experts, None,
                                 self.cfg, workspace=self._ws_recv)
        return y

    def __call__(self, x_local, group=None):
        return ep_step_a2a(x_local, self.ranges, self.home, self.partial, group)
