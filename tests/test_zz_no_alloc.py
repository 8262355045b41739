"""moe_permute_no_alloc: batch-union grouping for callers that cannot allocate device memory
(for example while a CUDA graph is being captured, or inside a host framework whose allocator
owns all device memory and that gives an operator no scratch buffer). The entry point uses a
fixed array compiled into the library instead of a workspace. Its results must equal those of
moe_permute, the workspace-taking entry point, on consecutive calls that reuse the array.

This file is collected last on purpose: it runs after every other test, and also alone."""
import ctypes as C

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _route(T, k, E, seed):
    r = np.random.default_rng(seed)
    return np.stack([r.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


def _no_alloc(M, idx_d, E):
    T, k = idx_d.shape
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    rc = M._lib.moe_permute_no_alloc(C.c_void_p(idx_d.data_ptr()), T, k, E,
                                     C.c_void_p(offsets.data_ptr()), C.c_void_p(perm.data_ptr()),
                                     C.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, offsets, perm


def test_no_alloc_permute_matches_workspace_permute_on_consecutive_calls():
    import quantized_expert_ffn_logits_b200 as M
    # the larger call first, so the second call runs on an array holding stale contents
    for T, k, E, seed in ((4096, 8, 512, 1), (37, 6, 64, 2), (1, 8, 64, 3)):
        idx = torch.from_numpy(_route(T, k, E, seed)).cuda()
        rc, offsets, perm = _no_alloc(M, idx, E)
        assert rc == M.MOE_OK, M.moe_status_string(rc)
        ref_offsets, ref_perm, _ = M.moe_permute(idx, E)
        torch.cuda.synchronize()
        assert torch.equal(offsets, ref_offsets), (T, k, E)
        assert torch.equal(perm, ref_perm), (T, k, E)


def test_no_alloc_permute_rejects_groupings_beyond_its_scratch():
    import quantized_expert_ffn_logits_b200 as M
    need = M._lib.moe_permute_workspace_bytes(8192, 8, 1024)
    assert need > (1 << 20)
    idx = torch.zeros((8192, 8), dtype=torch.int32, device="cuda")
    rc, _, _ = _no_alloc(M, idx, 1024)
    assert rc == M.MOE_ERR_WORKSPACE
