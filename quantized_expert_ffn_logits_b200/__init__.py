"""Python binding of the B200 quantized MoE FFN layer (include/moe_b200.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``_lib/libmoe_b200.so``; torch supplies device memory and the current stream.
The entry points keep the C names. Importing this package fails loudly when the
shared library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
import dataclasses
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"CUDA library not built: {LIB_PATH} (run quantized_expert_ffn_logits_b200/build.py)")

_lib = C.CDLL(LIB_PATH)

# ---------------------------------------------------------------- constants
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_DEVICE_CHECK, MOE_ERR_TIMEOUT = 4, 5, 6
MOE_W_INT8, MOE_W_INT4, MOE_W_INT2 = 0, 1, 2
MOE_SCALE_ROW_F32, MOE_SCALE_G32_F16 = 0, 1
MOE_ACT_TOKEN_F32, MOE_ACT_G32_F16 = 0, 1
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID_NOAUX_TC = 0, 1
MOE_FLAG_DEBUG, MOE_FLAG_FORCE_GEMV, MOE_FLAG_FORCE_MMA, MOE_FLAG_SHORT_WAITS = 1, 2, 4, 8

WTYPES = {"int8": MOE_W_INT8, "int4": MOE_W_INT4, "int2": MOE_W_INT2}
WSCALES = {"row_f32": MOE_SCALE_ROW_F32, "g32_f16": MOE_SCALE_G32_F16}
ACTS = {"token_f32": MOE_ACT_TOKEN_F32, "g32_f16": MOE_ACT_G32_F16}
SCORES = {"softmax": MOE_SCORE_SOFTMAX, "sigmoid": MOE_SCORE_SIGMOID_NOAUX_TC}


class moe_expert_blob(C.Structure):
    _fields_ = [("wtype", C.c_int32), ("wscale", C.c_int32), ("n_experts", C.c_int32),
                ("hidden", C.c_int32), ("inter", C.c_int32), ("reserved", C.c_int32),
                ("data", C.c_void_p), ("bytes", C.c_size_t)]


class moe_route_cfg(C.Structure):
    _fields_ = [("score", C.c_int32), ("top_k", C.c_int32), ("renormalize", C.c_int32),
                ("routed_scaling_factor", C.c_float), ("act", C.c_int32), ("flags", C.c_uint32),
                ("top_p", C.c_float), ("n_experts_total", C.c_int32), ("expert_begin", C.c_int32)]


class moe_debug_views(C.Structure):
    _fields_ = [(n, C.c_int64) for n in ("status", "q_x", "s_x", "logits", "idx", "w", "offsets",
                                          "perm", "n_active", "act_expert", "q_h", "s_h", "gate",
                                          "up", "y_pair", "dn_dots", "total")]


MOE_STAGES = ("quant_x", "router", "topk", "group", "gate_up", "quant_h", "down")


class moe_stage_events(C.Structure):
    _fields_ = [("begin", C.c_void_p * len(MOE_STAGES)), ("end", C.c_void_p * len(MOE_STAGES))]


_vp, _i32, _sz = C.c_void_p, C.c_int32, C.c_size_t
_PB, _PC = C.POINTER(moe_expert_blob), C.POINTER(moe_route_cfg)
_SIGS = {
    "moe_abi_version": (_i32, []),
    "moe_status_string": (C.c_char_p, [_i32]),
    "moe_last_error": (C.c_char_p, []),
    "moe_expert_blob_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "moe_quantize_experts": (_i32, [_vp, _vp, _PB, _vp]),
    "moe_quantize_experts_fp8": (_i32, [_vp, _vp, _vp, _vp, _PB, _vp]),
    "moe_quantize_activations": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_router_logits": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp]),
    "moe_route_topk": (_i32, [_vp, _vp, _i32, _i32, _PC, _vp, _vp, _vp]),
    "moe_permute_workspace_bytes": (_sz, [_i32, _i32, _i32]),
    "moe_permute": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_no_alloc": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_layer_workspace_bytes": (_sz, [_i32, _PB, _PB, _PC]),
    "moe_layer_forward": (_i32, [_vp, _i32, _vp, _vp, _PB, _PB, _PC, _vp, _vp, _sz, _vp]),
    "moe_layer_forward_host": (_i32, [_vp, _i32, _vp, _vp, _PB, _PB, _PC, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_layer_forward_timed": (_i32, [_vp, _i32, _vp, _vp, _PB, _PB, _PC, _vp, _vp, _sz, _vp,
                                       C.POINTER(moe_stage_events)]),
    "moe_layer_kernel_count": (_i32, [_i32, _PB, _PB, _PC]),
    "moe_layer_debug_views": (_i32, [_i32, _PB, _PB, _PC, C.POINTER(moe_debug_views)]),
    "moe_expert_group_dots": (_i32, [_PB, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "moe_read_device_status": (_i32, [_vp, _sz, _vp]),
    "moe_get_device_status": (_i32, [_vp, _vp]),
    "moe_layer_forward_debug": (_i32, [_vp, _i32, _vp, _vp, _PB, _PB, _PC, _vp, _vp, _sz, _vp,
                                       C.POINTER(moe_debug_views)]),
}
EXPORTS = tuple(_SIGS)
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args
ABI_VERSION = 4          # the struct layouts above (moe_route_cfg with top_p and the expert range,
                         # moe_debug_views with dn_dots)
if _lib.moe_abi_version() != ABI_VERSION:
    raise ImportError(f"{LIB_PATH}: ABI version {_lib.moe_abi_version()}, this binding needs "
                      f"{ABI_VERSION}: rebuild the library")


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == MOE_ERR_CUDA:
            detail = " [" + _lib.moe_last_error().decode() + "]"
        super().__init__(f"{where}: {moe_status_string(status)}{detail}")


def _check(rc: int, where: str) -> None:
    if rc != MOE_OK:
        raise MoeError(rc, where)


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _dev(t, dtype, name):
    import torch
    if t is None:
        return None
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got "
                         f"{t.dtype} on {t.device} (contiguous={t.is_contiguous()})")
    return t


# ---------------------------------------------------------------- config objects
@dataclass
class RouteCfg:
    score: str = "softmax"
    top_k: int = 8
    renormalize: bool = True
    routed_scaling_factor: float = 1.0
    act: str = "g32_f16"
    flags: int = 0
    top_p: float = 0.0      # adaptive expert top-p; 0 (or >= 1) = off
    n_experts_total: int = 0   # expert parallelism: the router's experts (0 = the blob's)
    expert_begin: int = 0      # ... and the first global expert id the blob holds

    def struct(self) -> moe_route_cfg:
        return moe_route_cfg(SCORES[self.score], self.top_k, int(self.renormalize),
                             float(self.routed_scaling_factor), ACTS[self.act], self.flags,
                             float(self.top_p), int(self.n_experts_total), int(self.expert_begin))


class ExpertBlob:
    """A quantized expert set in one device byte buffer (layout: include/moe_b200.h)."""

    def __init__(self, wtype: str, wscale: str, n_experts: int, hidden: int, inter: int,
                 data=None, device=None):
        import torch
        self.wtype, self.wscale = wtype, wscale
        self.n_experts, self.hidden, self.inter = n_experts, hidden, inter
        nbytes = moe_expert_blob_bytes(WTYPES[wtype], WSCALES[wscale], n_experts, hidden, inter)
        if nbytes == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "moe_expert_blob_bytes")
        if data is None:
            data = torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")
        if data.numel() < nbytes:
            raise ValueError("blob buffer too small")
        self.data = _dev(data, torch.uint8, "blob")
        self.nbytes = nbytes

    def struct(self) -> moe_expert_blob:
        return moe_expert_blob(WTYPES[self.wtype], WSCALES[self.wscale], self.n_experts,
                               self.hidden, self.inter, 0, self.data.data_ptr(), self.data.numel())

    @classmethod
    def quantize(cls, w_gate_up, w_down, wtype: str, wscale: str, stream=None) -> "ExpertBlob":
        """w_gate_up [E][2I][H], w_down [E][H][I] fp32 CUDA tensors -> blob."""
        E, twoI, H = w_gate_up.shape
        b = cls(wtype, wscale, E, H, twoI // 2, device=w_gate_up.device)
        moe_quantize_experts(w_gate_up, w_down, b, stream)
        return b

    @classmethod
    def quantize_fp8(cls, w_gate_up, s_gate_up, w_down, s_down, wtype: str, wscale: str,
                     stream=None) -> "ExpertBlob":
        """FP8 checkpoint weights -> blob: w_gate_up [E][2I][H] and w_down [E][H][I] E4M3 codes
        (torch.uint8 or torch.float8_e4m3fn CUDA tensors), s_gate_up / s_down fp32 inverse
        scales per 128 x 128 block ([E][ceil(2I/128)][ceil(H/128)], [E][ceil(H/128)][ceil(I/128)])."""
        E, twoI, H = w_gate_up.shape
        b = cls(wtype, wscale, E, H, twoI // 2, device=w_gate_up.device)
        moe_quantize_experts_fp8(w_gate_up, s_gate_up, w_down, s_down, b, stream)
        return b


# ---------------------------------------------------------------- entry points
def moe_abi_version() -> int:
    return int(_lib.moe_abi_version())


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(int(status)).decode()


def moe_expert_blob_bytes(wtype: int, wscale: int, n_experts: int, hidden: int, inter: int) -> int:
    return int(_lib.moe_expert_blob_bytes(wtype, wscale, n_experts, hidden, inter))


def moe_quantize_experts_fp8(w_gate_up, s_gate_up, w_down, s_down, blob: ExpertBlob, stream=None) -> None:
    import torch
    E, I, H = blob.n_experts, blob.inter, blob.hidden
    cdiv = lambda a: (a + 127) // 128
    codes = ((w_gate_up, "w_gate_up", (E, 2 * I, H)), (w_down, "w_down", (E, H, I)))
    for t, name, shape in codes:
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or tuple(t.shape) != shape:
            raise ValueError(f"{name}: want uint8/float8_e4m3fn {shape}, got {t.dtype} {tuple(t.shape)}")
    if tuple(s_gate_up.shape) != (E, cdiv(2 * I), cdiv(H)) or tuple(s_down.shape) != (E, cdiv(H), cdiv(I)):
        raise ValueError("block scales: want [E][ceil(2I/128)][ceil(H/128)] and [E][ceil(H/128)][ceil(I/128)]")
    for t, name, _ in codes:
        _dev(t, t.dtype, name)
    _dev(s_gate_up, torch.float32, "s_gate_up")
    _dev(s_down, torch.float32, "s_down")
    st = blob.struct()
    _check(_lib.moe_quantize_experts_fp8(_ptr(w_gate_up), _ptr(s_gate_up), _ptr(w_down), _ptr(s_down),
                                         C.byref(st), _stream(stream)), "moe_quantize_experts_fp8")


def moe_quantize_experts(w_gate_up, w_down, blob: ExpertBlob, stream=None) -> None:
    import torch
    _dev(w_gate_up, torch.float32, "w_gate_up")
    _dev(w_down, torch.float32, "w_down")
    st = blob.struct()
    _check(_lib.moe_quantize_experts(_ptr(w_gate_up), _ptr(w_down), C.byref(st), _stream(stream)),
           "moe_quantize_experts")


def moe_quantize_activations(x, act: str = "g32_f16", stream=None):
    import torch
    _dev(x, torch.float32, "x")
    T, H = x.shape
    q = torch.empty((T, H), dtype=torch.int8, device=x.device)
    if ACTS[act] == MOE_ACT_G32_F16:
        s = torch.empty((T, H // 32), dtype=torch.float16, device=x.device)
    else:
        s = torch.empty((T,), dtype=torch.float32, device=x.device)
    _check(_lib.moe_quantize_activations(_ptr(x), T, H, ACTS[act], _ptr(q), _ptr(s), _stream(stream)),
           "moe_quantize_activations")
    return q, s


def moe_router_logits(x, router_w, stream=None):
    import torch
    _dev(x, torch.float32, "x")
    _dev(router_w, torch.float32, "router_w")
    T, H = x.shape
    E = router_w.shape[0]
    out = torch.empty((T, E), dtype=torch.float32, device=x.device)
    _check(_lib.moe_router_logits(_ptr(x), _ptr(router_w), T, E, H, _ptr(out), _stream(stream)),
           "moe_router_logits")
    return out


def moe_route_topk(logits, bias, cfg: RouteCfg, stream=None):
    import torch
    _dev(logits, torch.float32, "logits")
    _dev(bias, torch.float32, "bias")
    T, E = logits.shape
    idx = torch.empty((T, cfg.top_k), dtype=torch.int32, device=logits.device)
    w = torch.empty((T, cfg.top_k), dtype=torch.float32, device=logits.device)
    st = cfg.struct()
    _check(_lib.moe_route_topk(_ptr(logits), _ptr(bias), T, E, C.byref(st), _ptr(idx), _ptr(w),
                               _stream(stream)), "moe_route_topk")
    return idx, w


def moe_permute(idx, n_experts: int, stream=None):
    import torch
    _dev(idx, torch.int32, "idx")
    T, k = idx.shape
    nb = int(_lib.moe_permute_workspace_bytes(T, k, n_experts))
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=idx.device)
    offsets = torch.empty(n_experts + 1, dtype=torch.int32, device=idx.device)
    perm = torch.empty(T * k, dtype=torch.int32, device=idx.device)
    _check(_lib.moe_permute(_ptr(idx), T, k, n_experts, _ptr(offsets), _ptr(perm), _ptr(ws),
                            ws.numel(), _stream(stream)), "moe_permute")
    return offsets, perm, ws


def moe_permute_no_alloc(idx, n_experts: int, stream=None):
    """moe_permute with the library's fixed 1 MiB device scratch (no workspace, no allocation
    inside the library; see include/moe_b200.h for the limits)."""
    import torch
    _dev(idx, torch.int32, "idx")
    T, k = idx.shape
    offsets = torch.empty(n_experts + 1, dtype=torch.int32, device=idx.device)
    perm = torch.empty(T * k, dtype=torch.int32, device=idx.device)
    _check(_lib.moe_permute_no_alloc(_ptr(idx), T, k, n_experts, _ptr(offsets), _ptr(perm),
                                     _stream(stream)), "moe_permute_no_alloc")
    return offsets, perm


def moe_layer_workspace_bytes(T: int, experts: ExpertBlob, shared: ExpertBlob | None,
                              cfg: RouteCfg) -> int:
    e = experts.struct()
    s = shared.struct() if shared is not None else None
    c = cfg.struct()
    return int(_lib.moe_layer_workspace_bytes(T, C.byref(e), C.byref(s) if s else None, C.byref(c)))


def moe_layer_forward(x, router_w, router_bias, experts: ExpertBlob, shared: ExpertBlob | None,
                      cfg: RouteCfg, y=None, workspace=None, stream=None):
    """y [T][H] = MoE FFN layer(x [T][H]). Returns (y, workspace)."""
    import torch
    _dev(x, torch.float32, "x")
    _dev(router_w, torch.float32, "router_w")
    _dev(router_bias, torch.float32, "router_bias")
    T, H = x.shape
    if y is None:
        y = torch.empty((T, H), dtype=torch.float32, device=x.device)
    _dev(y, torch.float32, "y")
    nb = moe_layer_workspace_bytes(T, experts, shared, cfg)
    if nb == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_layer_workspace_bytes")
    if workspace is None:
        workspace = torch.zeros(nb, dtype=torch.uint8, device=x.device)   # control block zeroed
    _dev(workspace, torch.uint8, "workspace")
    e = experts.struct()
    s = shared.struct() if shared is not None else None
    c = cfg.struct()
    _check(_lib.moe_layer_forward(_ptr(x), T, _ptr(router_w), _ptr(router_bias), C.byref(e),
                                  C.byref(s) if s else None, C.byref(c), _ptr(y), _ptr(workspace),
                                  workspace.numel(), _stream(stream)), "moe_layer_forward")
    return y, workspace


def moe_layer_kernel_count(T: int, experts: ExpertBlob, shared: ExpertBlob | None,
                           cfg: RouteCfg) -> int:
    e = experts.struct()
    s = shared.struct() if shared is not None else None
    c = cfg.struct()
    return int(_lib.moe_layer_kernel_count(T, C.byref(e), C.byref(s) if s else None, C.byref(c)))


class Layer:
    """A prepared layer call: the C structs and the workspace are built once, so each call
    is one ctypes call into moe_layer_forward (or moe_layer_forward_timed with events)."""

    def __init__(self, T: int, experts: ExpertBlob, shared: ExpertBlob | None, cfg: RouteCfg,
                 router_w, router_bias=None, workspace=None):
        import torch
        self.T, self.experts, self.shared, self.cfg = T, experts, shared, cfg
        self.router_w = _dev(router_w, torch.float32, "router_w")
        self.router_bias = _dev(router_bias, torch.float32, "router_bias")
        self._e = experts.struct()
        self._s = shared.struct() if shared is not None else None
        self._c = cfg.struct()
        nb = moe_layer_workspace_bytes(T, experts, shared, cfg)
        if nb == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "moe_layer_workspace_bytes")
        self.workspace = workspace if workspace is not None else torch.zeros(
            nb, dtype=torch.uint8, device=router_w.device)   # control block zeroed
        self._args = (self.router_w.data_ptr(), _ptr(self.router_bias), C.byref(self._e),
                      C.byref(self._s) if self._s is not None else None, C.byref(self._c))
        self.kernels = moe_layer_kernel_count(T, experts, shared, cfg)

    def __call__(self, x, y, stream=None, events: moe_stage_events | None = None):
        rw, rb, e, s, c = self._args
        st = _stream(stream)
        if events is None:
            rc = _lib.moe_layer_forward(x.data_ptr(), self.T, rw, rb, e, s, c, y.data_ptr(),
                                        self.workspace.data_ptr(), self.workspace.numel(), st)
        else:
            rc = _lib.moe_layer_forward_timed(x.data_ptr(), self.T, rw, rb, e, s, c, y.data_ptr(),
                                              self.workspace.data_ptr(), self.workspace.numel(), st,
                                              C.byref(events))
        _check(rc, "moe_layer_forward")
        return y

    def forward_host(self, x_host, y_host, stream=None):
        """The layer on host buffers (page-locked CPU tensors [T][H] fp32): one call into
        moe_layer_forward_host, which enqueues the copy in, the layer and the copy out on
        `stream` (synchronize it before reading y_host). Device staging buffers are the
        layer's own."""
        import torch
        if getattr(self, "_xd", None) is None:
            H = self.experts.hidden
            self._xd = torch.empty((self.T, H), dtype=torch.float32, device=self.router_w.device)
            self._yd = torch.empty((self.T, H), dtype=torch.float32, device=self.router_w.device)
        rw, rb, e, s, c = self._args
        rc = _lib.moe_layer_forward_host(x_host.data_ptr(), self.T, rw, rb, e, s, c, self._xd.data_ptr(),
                                         self._yd.data_ptr(), y_host.data_ptr(), self.workspace.data_ptr(),
                                         self.workspace.numel(), _stream(stream))
        _check(rc, "moe_layer_forward_host")
        return y_host


def moe_layer_debug_views(T: int, experts: ExpertBlob, shared: ExpertBlob | None,
                          cfg: RouteCfg) -> dict:
    e = experts.struct()
    s = shared.struct() if shared is not None else None
    c = cfg.struct()
    v = moe_debug_views()
    _check(_lib.moe_layer_debug_views(T, C.byref(e), C.byref(s) if s else None, C.byref(c),
                                      C.byref(v)), "moe_layer_debug_views")
    return {n: getattr(v, n) for n, _ in moe_debug_views._fields_}


def moe_expert_group_dots(blob: ExpertBlob, which: int, expert, row, act, stream=None):
    import torch
    _dev(expert, torch.int32, "expert")
    _dev(row, torch.int32, "row")
    _dev(act, torch.int8, "act")
    n, K = act.shape
    dots = torch.empty((n, K // 32), dtype=torch.int32, device=act.device)
    b = blob.struct()
    _check(_lib.moe_expert_group_dots(C.byref(b), which, n, _ptr(expert), _ptr(row), _ptr(act),
                                      _ptr(dots), _stream(stream)), "moe_expert_group_dots")
    return dots


def moe_read_device_status(workspace, stream=None) -> int:
    return int(_lib.moe_read_device_status(_ptr(workspace), workspace.numel(), _stream(stream)))


def moe_get_device_status(workspace, stream=None) -> int:
    return int(_lib.moe_get_device_status(_ptr(workspace), _stream(stream)))


def moe_layer_forward_debug(x, router_w, router_bias, experts: ExpertBlob,
                            shared: ExpertBlob | None, cfg: RouteCfg, y=None, workspace=None,
                            stream=None):
    """moe_layer_forward with the debug intermediates kept: returns (y, workspace, views), views
    being the byte offsets of moe_layer_debug_views (read them with workspace_view)."""
    import torch
    T, H = x.shape
    dbg = dataclasses.replace(cfg, flags=cfg.flags | MOE_FLAG_DEBUG)
    _dev(x, torch.float32, "x")
    _dev(router_w, torch.float32, "router_w")
    _dev(router_bias, torch.float32, "router_bias")
    if y is None:
        y = torch.empty((T, H), dtype=torch.float32, device=x.device)
    _dev(y, torch.float32, "y")
    nb = moe_layer_workspace_bytes(T, experts, shared, dbg)
    if nb == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_layer_workspace_bytes")
    if workspace is None:
        workspace = torch.zeros(nb, dtype=torch.uint8, device=x.device)   # control block zeroed
    _dev(workspace, torch.uint8, "workspace")
    e = experts.struct()
    s = shared.struct() if shared is not None else None
    c = cfg.struct()
    v = moe_debug_views()
    _check(_lib.moe_layer_forward_debug(_ptr(x), T, _ptr(router_w), _ptr(router_bias), C.byref(e),
                                        C.byref(s) if s else None, C.byref(c), _ptr(y), _ptr(workspace),
                                        workspace.numel(), _stream(stream), C.byref(v)),
           "moe_layer_forward_debug")
    return y, workspace, {n: getattr(v, n) for n, _ in moe_debug_views._fields_}


def workspace_view(workspace, offset: int, dtype, shape):
    """A typed tensor view of a region of a layer workspace (for inspecting intermediates)."""
    import torch
    n = 1
    for d in shape:
        n *= d
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    return workspace[offset:offset + nbytes].view(dtype).view(*shape)
