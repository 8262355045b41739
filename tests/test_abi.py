"""Host-side checks of the C ABI: the library loads, exports every declared entry point,
sizes agree with the documented layouts, and argument errors return before any CUDA call."""
import ctypes as C
import glob
import os
import re

import pytest

import oracle as O
import quantized_expert_ffn_logits_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 14
    lib = C.CDLL(M.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(M.EXPORTS)


def test_version_and_status_strings():
    assert M.moe_abi_version() == 4
    for s in range(7):
        assert M.moe_status_string(s).startswith("MOE_")
    assert M.moe_status_string(99) == "MOE_ERR_UNKNOWN"


@pytest.mark.parametrize("wtype,wscale", [(0, 0), (0, 1), (1, 0), (1, 1), (2, 0), (2, 1)])
@pytest.mark.parametrize("E,H,I", [(8, 256, 128), (64, 2048, 1024), (256, 6144, 2048), (1, 2048, 512)])
def test_blob_bytes_match_documented_layout(wtype, wscale, E, H, I):
    got = M.moe_expert_blob_bytes(wtype, wscale, E, H, I)
    assert got == O.blob_layout(E, H, I, {0: 8, 1: 4, 2: 2}[wtype], wscale == 1)[4]


@pytest.mark.parametrize("args", [(0, 0, 8, 96, 128), (0, 0, 8, 256, 100), (3, 0, 8, 256, 128),
                                  (0, 3, 8, 256, 128), (0, 0, 0, 256, 128), (0, 0, 2000, 256, 128)])
def test_blob_bytes_reject_unsupported(args):
    assert M.moe_expert_blob_bytes(*args) == 0


def _blob(E=8, H=256, I=128, wtype=0, wscale=1, data=256, nbytes=None):
    b = M.moe_expert_blob(wtype, wscale, E, H, I, 0, data, 0)
    b.bytes = nbytes if nbytes is not None else M.moe_expert_blob_bytes(wtype, wscale, E, H, I)
    return b


def _cfg(k=2, score=0, act=1, flags=0, top_p=0.0):
    return M.moe_route_cfg(score, k, 1, 1.0, act, flags, top_p)


def test_workspace_bytes_grow_with_tokens():
    b, c = _blob(), _cfg()
    sizes = [M._lib.moe_layer_workspace_bytes(T, C.byref(b), None, C.byref(c)) for T in (1, 8, 64, 512)]
    assert all(s > 0 and s % 256 == 0 for s in sizes)
    assert sizes == sorted(sizes)
    dbg = M._lib.moe_layer_workspace_bytes(8, C.byref(b), None, C.byref(_cfg(flags=1)))
    assert dbg > sizes[1]


def test_forward_argument_errors_return_before_launch():
    f = M._lib.moe_layer_forward
    b, c = _blob(), _cfg()
    ws_need = M._lib.moe_layer_workspace_bytes(4, C.byref(b), None, C.byref(c))
    fake = 1 << 20    # never dereferenced: every call below fails its host-side checks
    assert f(None, 4, fake, None, C.byref(b), None, C.byref(c), fake, fake, ws_need, None) == M.MOE_ERR_INVALID_ARG
    assert f(fake, 4, fake, None, C.byref(b), None, C.byref(c), fake, fake, ws_need - 256, None) == M.MOE_ERR_WORKSPACE
    assert f(fake, 4, fake, None, C.byref(b), None, C.byref(_cfg(k=9)), fake, fake, ws_need, None) == M.MOE_ERR_UNSUPPORTED
    assert f(fake, 4, fake, None, C.byref(b), None, C.byref(_cfg(k=0)), fake, fake, ws_need, None) == M.MOE_ERR_UNSUPPORTED
    assert f(fake, 4, fake, None, C.byref(b), None, C.byref(_cfg(score=7)), fake, fake, ws_need, None) == M.MOE_ERR_INVALID_ARG
    for bad_p in (float("nan"), -0.25, float("inf")):     # adaptive top-p: finite and >= 0
        assert f(fake, 4, fake, None, C.byref(b), None, C.byref(_cfg(top_p=bad_p)), fake, fake, ws_need, None) == M.MOE_ERR_INVALID_ARG
        assert M._lib.moe_route_topk(fake, None, 4, 8, C.byref(_cfg(top_p=bad_p)), fake, fake, None) == M.MOE_ERR_INVALID_ARG
    assert f(fake, -1, fake, None, C.byref(b), None, C.byref(c), fake, fake, ws_need, None) == M.MOE_ERR_INVALID_ARG
    assert f(fake + 4, 4, fake, None, C.byref(b), None, C.byref(c), fake, fake, ws_need, None) == M.MOE_ERR_INVALID_ARG
    small = _blob(nbytes=1024)
    assert f(fake, 4, fake, None, C.byref(small), None, C.byref(c), fake, fake, ws_need, None) == M.MOE_ERR_WORKSPACE
    odd = _blob(data=fake + 16)
    assert f(fake, 4, fake, None, C.byref(odd), None, C.byref(c), fake, fake, ws_need, None) == M.MOE_ERR_INVALID_ARG
    bad_shared = _blob(E=2)
    assert f(fake, 4, fake, None, C.byref(b), C.byref(bad_shared), C.byref(c), fake, fake, ws_need, None) == M.MOE_ERR_UNSUPPORTED
    other_fmt = _blob(E=1, wtype=1)
    assert f(fake, 4, fake, None, C.byref(b), C.byref(other_fmt), C.byref(c), fake, fake, ws_need, None) == M.MOE_ERR_UNSUPPORTED
    # T = 0 is a no-op that needs no buffers at all
    assert f(None, 0, None, None, C.byref(b), None, C.byref(c), None, None, 0, None) == M.MOE_OK


def test_other_entry_points_reject_bad_arguments():
    L = M._lib
    fake = 1 << 20
    b = _blob()
    assert L.moe_quantize_experts(None, fake, C.byref(b), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_experts(fake, fake, C.byref(_blob(nbytes=10)), None) == M.MOE_ERR_WORKSPACE
    assert L.moe_quantize_experts_fp8(fake, None, fake, fake, C.byref(b), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_experts_fp8(fake, fake, fake, fake, C.byref(_blob(nbytes=10)), None) == M.MOE_ERR_WORKSPACE
    assert L.moe_quantize_activations(fake, 4, 100, 1, fake, fake, None) == M.MOE_ERR_UNSUPPORTED
    assert L.moe_quantize_activations(fake, 4, 128, 5, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_activations(fake + 4, 4, 128, 1, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_activations(fake, 4, 128, 1, fake + 2, fake, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_router_logits(fake + 8, fake, 4, 8, 128, fake, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_router_logits(fake, fake, 4, 8, 100, fake, None) == M.MOE_ERR_UNSUPPORTED
    assert L.moe_route_topk(fake, None, 4, 8, C.byref(_cfg(k=9)), fake, fake, None) == M.MOE_ERR_UNSUPPORTED
    assert L.moe_route_topk(fake, None, 4, 2000, C.byref(_cfg()), fake, fake, None) == M.MOE_ERR_UNSUPPORTED
    need = L.moe_permute_workspace_bytes(100, 4, 16)
    assert need > 0
    assert L.moe_permute(fake, 100, 4, 16, fake, fake, fake, need - 1, None) == M.MOE_ERR_WORKSPACE
    assert L.moe_permute(fake, 100, 40, 16, fake, fake, fake, need, None) == M.MOE_ERR_UNSUPPORTED
    assert L.moe_expert_group_dots(C.byref(b), 2, 1, fake, fake, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    v = M.moe_debug_views()
    assert L.moe_layer_debug_views(4, C.byref(b), None, C.byref(_cfg(flags=1)), C.byref(v)) == M.MOE_OK
    assert v.gate > 0 and v.up > 0 and v.y_pair > 0 and v.total == L.moe_layer_workspace_bytes(4, C.byref(b), None, C.byref(_cfg(flags=1)))
    # the down projection's group dots: int32 [T*k][H][I/32], the last region of the debug layout
    assert v.dn_dots > v.y_pair and v.dn_dots + 4 * 2 * 256 * (128 // 32) * 4 <= v.total
    assert L.moe_layer_debug_views(4, C.byref(b), None, C.byref(_cfg()), C.byref(v)) == M.MOE_OK
    assert v.gate == -1 and v.dn_dots == -1
    assert L.moe_get_device_status(None, None) == M.MOE_ERR_INVALID_ARG
    # the debug forward sizes its workspace for the debug layout and leaves views alone on errors
    f = L.moe_layer_forward_debug
    plain = L.moe_layer_workspace_bytes(4, C.byref(b), None, C.byref(_cfg()))
    v.gate = 12345
    assert f(fake, 4, fake, None, C.byref(b), None, None, fake, fake, plain, None, C.byref(v)) == M.MOE_ERR_INVALID_ARG
    assert f(fake, 4, fake, None, C.byref(b), None, C.byref(_cfg()), fake, fake, plain, None, None) == M.MOE_ERR_INVALID_ARG
    assert f(fake, 4, fake, None, C.byref(b), None, C.byref(_cfg()), fake, fake, plain, None, C.byref(v)) == M.MOE_ERR_WORKSPACE
    assert v.gate == 12345


def test_build_entry_point_builds_and_checks_the_library():
    """__graft_entry__.build(): compiles what is stale (nothing, normally) and checks the
    library it loads (ABI version, exports)."""
    import importlib
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    g = importlib.import_module("__graft_entry__")
    g.build()


def test_fp8_binding_checks_shapes_and_devices():
    """ExpertBlob.quantize_fp8's argument checks run on the host, before any launch."""
    torch = pytest.importorskip("torch")

    class _Blob:                                     # shape fields only: nothing is launched
        n_experts, inter, hidden = 2, 128, 256
    gu = torch.zeros((2, 256, 256), dtype=torch.uint8)
    dn = torch.zeros((2, 256, 128), dtype=torch.uint8)
    sgu = torch.ones((2, 2, 2))
    sdn = torch.ones((2, 2, 1))
    with pytest.raises(ValueError, match="w_gate_up"):
        M.moe_quantize_experts_fp8(gu[:, :128], sgu, dn, sdn, _Blob())
    with pytest.raises(ValueError, match="w_down"):
        M.moe_quantize_experts_fp8(gu, sgu, dn.float(), sdn, _Blob())
    with pytest.raises(ValueError, match="block scales"):
        M.moe_quantize_experts_fp8(gu, sgu[:, :1], dn, sdn, _Blob())
    with pytest.raises(ValueError, match="CUDA"):  # right shapes, but host tensors
        M.moe_quantize_experts_fp8(gu, sgu, dn, sdn, _Blob())


def test_expert_range_arguments_are_checked():
    """Expert parallelism's range (moe_route_cfg.n_experts_total, expert_begin) is checked on
    the host: the size query returns 0 for a range the router cannot hold."""
    b = M.moe_expert_blob(0, 1, 8, 256, 128, 0, 256, M.moe_expert_blob_bytes(0, 1, 8, 256, 128))
    ok = M.moe_route_cfg(0, 2, 1, 1.0, 1, 0, 0.0, 16, 8)
    bad = [M.moe_route_cfg(0, 2, 1, 1.0, 1, 0, 0.0, 16, 9),       # range past the router's experts
           M.moe_route_cfg(0, 2, 1, 1.0, 1, 0, 0.0, 4, 0),        # fewer router experts than held
           M.moe_route_cfg(0, 2, 1, 1.0, 1, 0, 0.0, 2000, 0),     # > 1024
           M.moe_route_cfg(0, 2, 1, 1.0, 1, 0, 0.0, 16, -1)]
    assert M._lib.moe_layer_workspace_bytes(4, C.byref(b), None, C.byref(ok)) > 0
    for c in bad:
        assert M._lib.moe_layer_workspace_bytes(4, C.byref(b), None, C.byref(c)) == 0
