"""Shared helpers of the tests: build one workload on the GPU (through the C ABI) and on
the CPU oracle from the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np

import oracle as O
import synth as S

REL_L2 = 1e-5      # layer output: relative L2 error bound
MAX_ABS = 1e-4     # layer output: max |error| relative to max |y_ref|


def wbits(cfg):
    return {"int8": 8, "int4": 4, "int2": 2}[cfg.wtype]


def wg32(cfg):
    return cfg.wscale == "g32_f16"


def ag32(cfg):
    return cfg.act == "g32_f16"


def route_cfg(cfg, flags=0, top_p=0.0):
    import quantized_expert_ffn_logits_b200 as M
    return M.RouteCfg(score=cfg.score, top_k=cfg.top_k, renormalize=cfg.renormalize,
                      routed_scaling_factor=cfg.rsf, act=cfg.act, flags=flags, top_p=top_p)


def gpu_layer(case: S.Case, device="cuda"):
    """Expert blobs, router weight, bias and x of a case, on the device."""
    import torch
    import quantized_expert_ffn_logits_b200 as M
    c = case.cfg
    gu = torch.empty((c.E, 2 * c.I, c.H), dtype=torch.float32, device=device)
    dn = torch.empty((c.E, c.H, c.I), dtype=torch.float32, device=device)
    case.gate_up_gpu(gu)
    case.down_gpu(dn)
    blob = M.ExpertBlob.quantize(gu, dn, c.wtype, c.wscale)
    del gu, dn
    shared = None
    if c.shared_I:
        sgu = torch.empty((1, 2 * c.shared_I, c.H), dtype=torch.float32, device=device)
        sdn = torch.empty((1, c.H, c.shared_I), dtype=torch.float32, device=device)
        case.shared_gate_up_gpu(sgu)
        case.shared_down_gpu(sdn)
        shared = M.ExpertBlob.quantize(sgu, sdn, c.wtype, c.wscale)
        del sgu, sdn
    wr = torch.from_numpy(case.router_w()).to(device)
    b = case.bias()
    bias = torch.from_numpy(b).to(device) if b is not None else None
    x = torch.from_numpy(case.x()).to(device)
    return dict(blob=blob, shared=shared, wr=wr, bias=bias, x=x)


def oracle_experts(case: S.Case, experts=None):
    """Oracle-quantized routed experts (all, or the listed ones in that order) and shared."""
    c = case.cfg
    ids = range(c.E) if experts is None else experts
    ex = O.QExperts.quantize(np.stack([case.gate_up(e) for e in ids]),
                             np.stack([case.down(e) for e in ids]), wbits(c), wg32(c))
    sh = None
    if c.shared_I:
        sh = O.QExperts.quantize(case.shared_gate_up()[None], case.shared_down()[None], wbits(c), wg32(c))
    return ex, sh


def oracle_layer(case: S.Case, union=False, top_p=0.0, x=None):
    """The oracle's layer on the case's inputs (or on another x with the case's weights);
    the result also carries the oracle-quantized experts under "experts" (routed, shared)."""
    c = case.cfg
    ex, sh = oracle_experts(case)
    o = O.layer_forward(case.x() if x is None else x, case.router_w(), case.bias(), ex, sh, c.score,
                        c.top_k, c.renormalize, c.rsf, ag32(c), union=union, top_p=top_p)
    o["experts"] = (ex, sh)
    return o


def group_dots(qw, qa):
    """Exact per-group integer dots: qw [N][K] int8 codes, qa [n][K] int8 -> int64 [n][N][K/32]
    (products and sums of integers below 2^53 are exact in fp64)."""
    qw = np.asarray(qw)
    N, K = qw.shape
    G = K // 32
    w = qw.astype(np.float64).reshape(N, G, 32)
    a = np.asarray(qa).astype(np.float64).reshape(-1, G, 32)
    return np.einsum("ngi,hgi->nhg", a, w).astype(np.int64)


def expected_down_dots(ref, case: S.Case, perm):
    """The down projection's exact group dots of every kept pair (grouped row r = pair
    perm[r]) and, with a shared expert, of every token against it: from the oracle's q_h and
    down codes. Returns (routed [P][H][I/32], shared [T][H][I_s/32] or None)."""
    c = case.cfg
    ex, sh = ref["experts"]
    k = c.top_k
    perm = np.asarray(perm)
    e_of = ref["idx"].reshape(-1)[perm]
    out = np.zeros((len(perm), c.H, c.I // 32), np.int64)
    for e in np.unique(e_of):
        rows = np.nonzero(e_of == e)[0]
        out[rows] = group_dots(ex.q_dn[e], ref["qh"][perm[rows]])
    shd = None
    if sh is not None:
        qh_sh = np.stack([O.expert_ffn(sh, 0, ref["qx"][t], ref["sx"][t], ag32(c))["qh"]
                          for t in range(case.T)])
        shd = group_dots(sh.q_dn[0], qh_sh)
    return out, shd


def oracle_tokens(case: S.Case, tokens, x=None):
    """Per-token oracle for selected tokens only (of the case's x, or of another x [T][H]),
    regenerating just the experts they use.
    Returns dict(y [n][H], idx, w, ye {(t, j): fp64 [H]}, qh/sh/gate/up per pair)."""
    c = case.cfg
    x = case.x() if x is None else np.asarray(x)
    L = O.router_logits(x[tokens], case.router_w())
    idx, w = O.route(L, case.bias(), c.score, c.top_k, c.renormalize, c.rsf)
    qx, sx = O.quantize_act(x[tokens], ag32(c))
    need = sorted(set(int(e) for e in idx.reshape(-1)))
    y = np.zeros((len(tokens), c.H))
    pairs = {}
    for e in need:
        ex = O.QExperts.quantize(case.gate_up(e)[None], case.down(e)[None], wbits(c), wg32(c))
        for n, t in enumerate(tokens):
            for j in range(c.top_k):
                if idx[n, j] == e:
                    r = O.expert_ffn(ex, 0, qx[n], sx[n], ag32(c))
                    pairs[(n, j)] = r
                    y[n] += w[n, j] * r["ye"]
        del ex
    if c.shared_I:
        sh = O.QExperts.quantize(case.shared_gate_up()[None], case.shared_down()[None], wbits(c), wg32(c))
        for n in range(len(tokens)):
            y[n] += O.expert_ffn(sh, 0, qx[n], sx[n], ag32(c))["ye"]
    return dict(y=y, idx=idx, w=w, logits=L, qx=qx, sx=sx, pairs=pairs)


def assert_close_y(got, ref, what="y"):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    den = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / den if den > 0 else np.linalg.norm(got)
    mabs = np.max(np.abs(got - ref)) if got.size else 0.0
    scale = np.max(np.abs(ref)) if ref.size else 1.0
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    assert mabs <= MAX_ABS * scale, f"{what}: max-abs {mabs:.3e} > {MAX_ABS} * {scale:.3e}"
    return rel, mabs
