"""The single-token kernel's bounded grid-barrier wait, made to run out (the GLM-5.2 colibri
page, "Experimental resident CUDA backend": a failure is reported, never a silent fallback).

The workspace's control block holds the grid-barrier counter (bytes 16-23; a multiple of 1024
between calls). Preset to base + 1023, the first CTA to arrive completes the old round and
every later one waits for a round that the grid can no longer fill. With MOE_FLAG_SHORT_WAITS
those waits give up after about 2 ms: the call must report MOE_ERR_TIMEOUT with the wait
record of the grid barrier, the status read must reset the control block, and the next call
must be correct again. Nothing here faults or hangs the GPU: every wait is bounded and the
kernel returns."""
import time

import numpy as np
import pytest

import synth as S
from helpers import assert_close_y, gpu_layer, oracle_tokens, route_cfg

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

WAIT_GRID_BARRIER = 6          # wait id of the single-token kernel's grid barrier
WAIT_Y_ZERO = 8                # ... and of its cluster variant's y-zero barrier
KERNEL_GATE_UP = 1

# The OLMoE-shaped decode layer runs the grid barrier (its 128 CTAs exceed the co-resident
# clusters); the reduced layer's 16 CTAs fit one cluster, which exchanges the logits in
# distributed shared memory and then waits on the same counter for y to be zeroed.
CASES = [(S.CONFIGS["olmoe_int8"], (WAIT_GRID_BARRIER,)),
         (S.CONFIGS["olmoe_int8"].with_(name="olmoe_int8_r", H=512, E=16, I=256, top_k=4),
          (WAIT_GRID_BARRIER, WAIT_Y_ZERO))]


@pytest.mark.parametrize("cfg_, waits", CASES, ids=["olmoe_int8", "olmoe_int8_reduced"])
def test_grid_barrier_timeout_is_reported_and_recovers(cfg_, waits):
    import quantized_expert_ffn_logits_b200 as M
    CFG = cfg_
    case = S.Case.make(CFG, 1)
    g = gpu_layer(case)
    cfg = route_cfg(CFG, flags=M.MOE_FLAG_SHORT_WAITS)
    lay = M.Layer(1, g["blob"], None, cfg, g["wr"], None)
    assert lay.kernels == 1                       # the single-token kernel
    y = torch.empty((1, CFG.H), dtype=torch.float32, device="cuda")
    lay(g["x"], y)
    torch.cuda.synchronize()
    assert M.moe_read_device_status(lay.workspace) == M.MOE_OK
    ref = oracle_tokens(case, [0])["y"]
    assert_close_y(y.cpu().numpy(), ref)

    ctr = lay.workspace[16:24].view(torch.int64)
    base = int(ctr.item())
    assert base % 1024 == 0 and base > 0         # the finished call moved it to the next round
    ctr.fill_(base + 1023)
    t0 = time.perf_counter()
    lay(g["x"], y)
    torch.cuda.synchronize()
    took = time.perf_counter() - t0
    words = lay.workspace[:16].view(torch.int32).cpu().numpy()
    assert M.moe_read_device_status(lay.workspace) == M.MOE_ERR_TIMEOUT
    assert words[2] in [KERNEL_GATE_UP | (w << 4) for w in waits], hex(int(words[2]))
    assert took < 1.0, f"the short wait bound took {took:.3f} s"
    # the status read reset the status word and the barrier counter (the wait record stays)
    assert int(ctr.item()) == 0
    assert M.moe_read_device_status(lay.workspace) == M.MOE_OK

    y2 = torch.full((1, CFG.H), float("nan"), dtype=torch.float32, device="cuda")
    lay(g["x"], y2)
    torch.cuda.synchronize()
    assert M.moe_read_device_status(lay.workspace) == M.MOE_OK
    assert_close_y(y2.cpu().numpy(), ref)
    assert np.isfinite(y2.cpu().numpy()).all()
