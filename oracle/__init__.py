"""Plain CPU oracle of the quantized MoE FFN layer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. It wraps ``moe_oracle.c`` (plain C, fp64 where no
integer is decided, the canonical fp32 sequences where one is) with ctypes and
numpy marshalling; it shares nothing with the CUDA path.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


class Experts(C.Structure):
    _fields_ = [("E", C.c_int32), ("H", C.c_int32), ("I", C.c_int32), ("wbits", C.c_int32),
                ("wg32", C.c_int32), ("q_gu", C.c_void_p), ("s_gu", C.c_void_p),
                ("q_dn", C.c_void_p), ("s_dn", C.c_void_p)]


class LayerIn(C.Structure):
    _fields_ = [("T", C.c_int32), ("score", C.c_int32), ("top_k", C.c_int32),
                ("renorm", C.c_int32), ("act_g32", C.c_int32), ("rsf", C.c_float),
                ("x", C.c_void_p), ("Wr", C.c_void_p), ("bias", C.c_void_p),
                ("ex", C.POINTER(Experts)), ("sh", C.POINTER(Experts)), ("top_p", C.c_float)]


class LayerOut(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("y", "logits", "idx", "w", "qx", "sx", "gate", "up", "qh",
                                          "sh", "ye", "ye32", "ysh", "offsets", "perm")]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        vp, i32, i64, f32 = C.c_void_p, C.c_int, C.c_int64, C.c_float
        sig = {
            "orc_cexp": (C.c_float, [f32]),
            "orc_sigmoid": (C.c_float, [f32]),
            "orc_swiglu": (C.c_float, [f32, f32]),
            "orc_cexp_n": (None, [vp, i64, vp]),
            "orc_sigmoid_n": (None, [vp, i64, vp]),
            "orc_swiglu_n": (None, [vp, vp, i64, vp]),
            "orc_quantize_rows": (i32, [vp, i64, i32, i32, i32, vp, vp]),
            "orc_pack_int4": (i32, [vp, i64, i32, vp]),
            "orc_pack_int2": (i32, [vp, i64, i32, vp]),
            "orc_blob_layout": (i32, [i32, i32, i32, i32, i32, vp]),
            "orc_pack_blob": (i32, [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]),
            "orc_router_logits": (None, [vp, vp, i32, i32, i32, vp]),
            "orc_fp8_e4m3_to_f32": (C.c_float, [C.c_uint8]),
            "orc_dequant_fp8": (None, [vp, vp, C.c_int64, C.c_int64, vp]),
            "orc_route": (i32, [vp, vp, i32, i32, i32, i32, i32, f32, f32, vp, vp]),
            "orc_permute": (i32, [vp, i32, i32, i32, vp, vp]),
            "orc_stage": (C.c_float, [vp, vp, i32, i32, vp, vp, i32, vp]),
            "orc_stage_f64": (C.c_double, [vp, vp, i32, i32, vp, vp, i32]),
            "orc_expert_ffn": (i32, [C.POINTER(Experts), i32, vp, vp, i32, vp, vp, vp, vp, vp, vp]),
            "orc_layer_forward": (i32, [C.POINTER(LayerIn), C.POINTER(LayerOut), i32]),
            "orc_layer_forward_union": (i32, [C.POINTER(LayerIn), C.POINTER(LayerOut)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ scalars
def cexp(a):
    a = _c(a, np.float32)
    out = np.empty_like(a)
    lib().orc_cexp_n(_p(a), a.size, _p(out))
    return out


def sigmoid(a):
    a = _c(a, np.float32)
    out = np.empty_like(a)
    lib().orc_sigmoid_n(_p(a), a.size, _p(out))
    return out


def swiglu(g, u):
    g = _c(g, np.float32)
    u = _c(u, np.float32)
    out = np.empty_like(g)
    lib().orc_swiglu_n(_p(g), _p(u), g.size, _p(out))
    return out


# ------------------------------------------------------------- quantization
def quantize_rows(w, qmax: int, g32: bool):
    """Rows of w -> (codes int8 [N][K], scales float32 [N][K/32] or [N])."""
    w = _c(w, np.float32)
    N, K = w.shape
    q = np.empty((N, K), np.int8)
    s = np.empty((N, K // 32) if g32 else (N,), np.float32)
    rc = lib().orc_quantize_rows(_p(w), N, K, qmax, int(g32), _p(q), _p(s))
    if rc:
        raise ValueError("orc_quantize_rows: bad shape")
    return q, s


def quantize_act(x, g32: bool):
    return quantize_rows(x, 127, g32)


def pack_int4(q):
    q = _c(q, np.int8)
    N, K = q.shape
    out = np.empty((N, K // 2), np.uint8)
    if lib().orc_pack_int4(_p(q), N, K, _p(out)):
        raise ValueError("odd K")
    return out


def pack_int2(q):
    q = _c(q, np.int8)
    N, K = q.shape
    out = np.empty((N, K // 4), np.uint8)
    if lib().orc_pack_int2(_p(q), N, K, _p(out)):
        raise ValueError("K not a multiple of 4")
    return out


QMAX = {8: 127, 4: 7, 2: 1}      # symmetric codes: 2^(bits-1) - 1


def blob_layout(E, H, I, wbits, g32):
    off = np.zeros(5, np.uint64)
    if lib().orc_blob_layout(E, H, I, wbits, int(g32), _p(off)):
        raise ValueError("unsupported blob shape")
    return [int(v) for v in off]


class QExperts:
    """Logical quantized experts (codes + scale values), as the oracle consumes them."""

    def __init__(self, q_gu, s_gu, q_dn, s_dn, wbits: int, wg32: bool):
        self.q_gu, self.s_gu, self.q_dn, self.s_dn = (_c(q_gu, np.int8), _c(s_gu, np.float32),
                                                      _c(q_dn, np.int8), _c(s_dn, np.float32))
        self.E, twoI, self.H = self.q_gu.shape
        self.I = twoI // 2
        self.wbits, self.wg32 = wbits, bool(wg32)

    @classmethod
    def quantize(cls, gate_up, down, wbits: int, wg32: bool):
        """gate_up [E][2I][H], down [E][H][I] float32 -> quantized experts."""
        gate_up = np.asarray(gate_up, np.float32)
        down = np.asarray(down, np.float32)
        E, twoI, H = gate_up.shape
        I = twoI // 2
        qmax = QMAX[wbits]
        qg, sg = quantize_rows(gate_up.reshape(E * twoI, H), qmax, wg32)
        qd, sd = quantize_rows(down.reshape(E * H, I), qmax, wg32)
        return cls(qg.reshape(E, twoI, H), sg.reshape((E, twoI, H // 32) if wg32 else (E, twoI)),
                   qd.reshape(E, H, I), sd.reshape((E, H, I // 32) if wg32 else (E, H)), wbits, wg32)

    def struct(self) -> Experts:
        return Experts(self.E, self.H, self.I, self.wbits, int(self.wg32), _p(self.q_gu),
                       _p(self.s_gu), _p(self.q_dn), _p(self.s_dn))

    def pack_blob(self) -> np.ndarray:
        off = blob_layout(self.E, self.H, self.I, self.wbits, self.wg32)
        blob = np.zeros(off[4], np.uint8)
        rc = lib().orc_pack_blob(self.E, self.H, self.I, self.wbits, int(self.wg32), _p(self.q_gu),
                                 _p(self.s_gu), _p(self.q_dn), _p(self.s_dn), _p(blob))
        if rc:
            raise ValueError("orc_pack_blob failed")
        return blob

    def select(self, e: int) -> "QExperts":
        """Single-expert view (E = 1) of expert e."""
        return QExperts(self.q_gu[e:e + 1], self.s_gu[e:e + 1], self.q_dn[e:e + 1],
                        self.s_dn[e:e + 1], self.wbits, self.wg32)


# ------------------------------------------------------------------ routing
SCORES = {"softmax": 0, "sigmoid": 1}


def fp8_e4m3_decode(codes):
    """float8 E4M3 codes (uint8) as fp32, from the format's definition."""
    codes = np.asarray(codes, np.uint8)
    f = lib().orc_fp8_e4m3_to_f32
    return np.array([f(int(c)) for c in codes.reshape(-1)], np.float32).reshape(codes.shape)


def dequant_fp8(w8, s_inv):
    """FP8 weights [..., N, K] (uint8 E4M3 codes) with fp32 inverse scales per 128 x 128 block
    [..., ceil(N/128), ceil(K/128)] -> fp32 [..., N, K] (decode, then one fp32 product)."""
    w8 = _c(w8, np.uint8)
    s_inv = _c(s_inv, np.float32)
    N, K = w8.shape[-2:]
    lead = w8.shape[:-2]
    out = np.empty(w8.shape, np.float32)
    w2 = w8.reshape(-1, N, K)
    s2 = s_inv.reshape(-1, (N + 127) // 128, (K + 127) // 128)
    o2 = out.reshape(-1, N, K)
    for i in range(w2.shape[0]):
        wi, si, oi = w2[i], np.ascontiguousarray(s2[i]), o2[i]
        lib().orc_dequant_fp8(_p(wi), _p(si), N, K, _p(oi))
    return out.reshape(*lead, N, K)


def router_logits(x, Wr):
    x = _c(x, np.float32)
    Wr = _c(Wr, np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    L = np.empty((T, E), np.float32)
    lib().orc_router_logits(_p(x), _p(Wr), T, E, H, _p(L))
    return L


def route(L, bias, score: str, k: int, renorm: bool, rsf: float, top_p: float = 0.0):
    L = _c(L, np.float32)
    T, E = L.shape
    b = None if bias is None else _c(bias, np.float32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    if lib().orc_route(_p(L), _p(b), T, E, SCORES[score], k, int(renorm), float(rsf), float(top_p),
                       _p(idx), _p(w)):
        raise ValueError("orc_route: bad k")
    return idx, w


def permute(idx, E: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    if lib().orc_permute(_p(idx), T, k, E, _p(offsets), _p(perm)):
        raise ValueError("expert index out of range")
    return offsets, perm[: offsets[E]]       # slots with expert -1 (dropped) are left out


# ---------------------------------------------------------------- expert math
def stage(qw, sw, wg32: bool, qa, sa, ag32: bool):
    """Canonical fp32 stage value of one row and its per-group int32 dots."""
    qw, qa = _c(qw, np.int8), _c(qa, np.int8)
    sw, sa = _c(np.atleast_1d(sw), np.float32), _c(np.atleast_1d(sa), np.float32)
    K = qw.size
    dots = np.zeros(max(K // 32, 1), np.int32)
    v = lib().orc_stage(_p(qw), _p(sw), K, int(wg32), _p(qa), _p(sa), int(ag32), _p(dots))
    return np.float32(v), (dots if (wg32 or ag32) else dots[:1])


def stage_f64(qw, sw, wg32: bool, qa, sa, ag32: bool) -> float:
    qw, qa = _c(qw, np.int8), _c(qa, np.int8)
    sw, sa = _c(np.atleast_1d(sw), np.float32), _c(np.atleast_1d(sa), np.float32)
    return float(lib().orc_stage_f64(_p(qw), _p(sw), qw.size, int(wg32), _p(qa), _p(sa), int(ag32)))


def expert_ffn(ex: QExperts, e: int, qx, sx, ag32: bool):
    """One expert on one quantized token: dict(ye f64 [H], gate, up [I], qh [I], sh, ye32 [H])."""
    qx = _c(qx, np.int8)
    sx = _c(np.atleast_1d(sx), np.float32)
    H, I = ex.H, ex.I
    out = dict(ye=np.empty(H, np.float64), gate=np.empty(I, np.float32), up=np.empty(I, np.float32),
               qh=np.empty(I, np.int8), sh=np.empty(I // 32 if ag32 else 1, np.float32),
               ye32=np.empty(H, np.float32))
    st = ex.struct()
    rc = lib().orc_expert_ffn(C.byref(st), e, _p(qx), _p(sx), int(ag32), _p(out["ye"]),
                              _p(out["gate"]), _p(out["up"]), _p(out["qh"]), _p(out["sh"]),
                              _p(out["ye32"]))
    if rc:
        raise ValueError("orc_expert_ffn failed")
    return out


def layer_forward(x, Wr, bias, ex: QExperts, sh: QExperts | None, score: str, k: int,
                  renorm: bool, rsf: float, act_g32: bool, union: bool = False,
                  nthreads: int = 1, debug: bool = True, top_p: float = 0.0):
    """Whole layer. Returns dict with y (fp64 [T][H]) and, if debug, every intermediate."""
    x = _c(x, np.float32)
    Wr = _c(Wr, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    T, H = x.shape
    E, I = ex.E, ex.I
    o = dict(y=np.zeros((T, H), np.float64))
    if debug:
        o.update(logits=np.empty((T, E), np.float32), idx=np.empty((T, k), np.int32),
                 w=np.empty((T, k), np.float64), qx=np.empty((T, H), np.int8),
                 sx=np.empty((T, H // 32) if act_g32 else (T,), np.float32),
                 gate=np.empty((T * k, I), np.float32), up=np.empty((T * k, I), np.float32),
                 qh=np.empty((T * k, I), np.int8),
                 sh=np.empty((T * k, I // 32) if act_g32 else (T * k,), np.float32),
                 ye=np.empty((T * k, H), np.float64), ye32=np.empty((T * k, H), np.float32),
                 ysh=np.zeros((T, H), np.float64))
        if union:
            o.update(offsets=np.empty(E + 1, np.int32), perm=np.empty(T * k, np.int32))
    st = ex.struct()
    sst = sh.struct() if sh is not None else None
    lin = LayerIn(T, SCORES[score], k, int(renorm), int(act_g32), float(rsf), _p(x), _p(Wr), _p(b),
                  C.pointer(st), C.pointer(sst) if sst is not None else None, float(top_p))
    lout = LayerOut(*[_p(o.get(n)) for n, _ in LayerOut._fields_])
    if union:
        rc = lib().orc_layer_forward_union(C.byref(lin), C.byref(lout))
    else:
        rc = lib().orc_layer_forward(C.byref(lin), C.byref(lout), int(nthreads))
    if rc:
        raise ValueError("oracle layer forward failed")
    if "perm" in o:
        o["perm"] = o["perm"][: o["offsets"][E]]   # slots dropped by adaptive top-p are left out
    return o
