"""Seeded synthetic inputs for the quantized MoE FFN layer.

This module is the ONE piece shared by the CUDA path's tests/benchmark and by
the oracle. It holds none of the layer's arithmetic (no quantization, routing
or matmul): it only defines the workloads (shapes, formats, routing modes) and
turns seeds into float tensors with a counter-based generator, implemented once
for the host (synth_cpu.c) and once for the device (synth_gpu.cu) from the
published SplitMix64 definition. Any slice of any tensor can be regenerated on
either side, so the oracle can rebuild just the experts a token routes to.

Workloads are shaped like the models the pages discuss: OLMoE-1B-7B (64
experts, top-8, from "I ran a 7B Mixture-of-Experts LLM in a language I
built"), GLM-5.2 (256 routed experts + shared expert, sigmoid noaux_tc router,
from the colibri "Show HN: getting GLM-5.2 running" page) and a 512-expert
model (from "FLE: Fast Local Experts"). There are no trained weights here:
everything is N(0, sigma) noise of the right shape.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIBDIR = os.path.join(_HERE, "_lib")
_cpu = None
_gpu = None

MASK64 = (1 << 64) - 1


def _load_cpu():
    global _cpu
    if _cpu is None:
        path = os.path.join(_LIBDIR, "libsynth_cpu.so")
        if not os.path.exists(path):
            from . import build as _b
            _b.build()
        lib = ctypes.CDLL(path)
        lib.synth_hash.restype = ctypes.c_uint64
        lib.synth_hash.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_normal_f32.restype = None
        lib.synth_normal_f32.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                         ctypes.c_uint64, ctypes.c_float, ctypes.c_int]
        _cpu = lib
    return _cpu


def _load_gpu():
    global _gpu
    if _gpu is None:
        path = os.path.join(_LIBDIR, "libsynth_gpu.so")
        if not os.path.exists(path):
            raise RuntimeError(f"device input generator not built: {path}")
        lib = ctypes.CDLL(path)
        lib.synth_normal_f32_device.restype = ctypes.c_int
        lib.synth_normal_f32_device.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                                ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p]
        _gpu = lib
    return _gpu


def hash64(seed: int, ctr: int) -> int:
    return int(_load_cpu().synth_hash(seed & MASK64, ctr & MASK64))


def normal_cpu(n: int, seed: int, offset: int = 0, sigma: float = 1.0, threads: int = 0) -> np.ndarray:
    """n float32 deviates: element i is normal(seed, offset + i) * sigma."""
    out = np.empty(int(n), dtype=np.float32)
    if n:
        th = threads or min(8, os.cpu_count() or 1)
        _load_cpu().synth_normal_f32(out.ctypes.data, int(n), seed & MASK64, int(offset),
                                     float(sigma), th)
    return out


def normal_gpu_(t, seed: int, offset: int = 0, sigma: float = 1.0) -> None:
    """Fill a contiguous float32 CUDA tensor in place; bit-identical to normal_cpu."""
    import torch
    assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    rc = _load_gpu().synth_normal_f32_device(t.data_ptr(), t.numel(), seed & MASK64, int(offset),
                                             float(sigma), torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError(f"synth_normal_f32_device failed ({rc})")


# Tensor tags: each tensor of a case draws from its own seed hash(case_seed, tag).
TAG_X, TAG_WR, TAG_BIAS, TAG_ZIPF = 1, 2, 3, 4
TAG_GU, TAG_DN, TAG_SH_GU, TAG_SH_DN = 10, 11, 20, 21


@dataclass(frozen=True)
class LayerConfig:
    """Shape and formats of one MoE FFN layer workload."""
    name: str
    H: int                      # hidden size
    E: int                      # routed experts
    I: int                      # expert intermediate size
    top_k: int
    score: str                  # "softmax" | "sigmoid"
    renormalize: bool
    rsf: float                  # routed_scaling_factor (1.0 for softmax models)
    wtype: str                  # "int8" | "int4" | "int2"
    wscale: str                 # "row_f32" | "g32_f16"
    act: str                    # "token_f32" | "g32_f16"
    shared_I: int = 0           # 0 = no shared expert
    tokens: tuple = ()          # the T values this workload is quoted at
    x_sigma: float = 1.0
    w_sigma: float = 0.02
    wr_sigma: float = 0.0       # 0 => 1/sqrt(H) so logits ~ N(0, x_sigma^2)
    bias_sigma: float = 0.0     # sigmoid noaux_tc selection bias
    zipf: float = 0.0           # >0: skew router logits by a Zipf law over experts

    def with_(self, **kw) -> "LayerConfig":
        d = {k: getattr(self, k) for k in self.__dataclass_fields__}
        d.update(kw)
        return LayerConfig(**d)

    @property
    def router_sigma(self) -> float:
        return self.wr_sigma if self.wr_sigma > 0 else 1.0 / math.sqrt(self.H)


CONFIGS = {
    # tiny correctness layer
    "tiny": LayerConfig("tiny", H=256, E=8, I=128, top_k=2, score="softmax", renormalize=False,
                        rsf=1.0, wtype="int8", wscale="row_f32", act="token_f32", tokens=(4,),
                        x_sigma=0.02, w_sigma=0.02, wr_sigma=0.02),
    # OLMoE-1B-7B-shaped decode layer, int8 experts with group-32 fp16 scales
    "olmoe_int8": LayerConfig("olmoe_int8", H=2048, E=64, I=1024, top_k=8, score="softmax",
                              renormalize=True, rsf=1.0, wtype="int8", wscale="g32_f16",
                              act="g32_f16", tokens=(1, 8)),
    # same layer with packed int4 experts, prefill
    "olmoe_int4": LayerConfig("olmoe_int4", H=2048, E=64, I=1024, top_k=8, score="softmax",
                              renormalize=True, rsf=1.0, wtype="int4", wscale="g32_f16",
                              act="g32_f16", tokens=(512, 4096)),
    # GLM-5.2-style: 256 routed + 1 shared, sigmoid noaux_tc, rsf 2.5, per-row int4
    "glm_int4": LayerConfig("glm_int4", H=6144, E=256, I=2048, top_k=8, score="sigmoid",
                            renormalize=True, rsf=2.5, wtype="int4", wscale="row_f32",
                            act="g32_f16", shared_I=2048, tokens=(1, 4), bias_sigma=0.05),
    # 512-expert layer with a shared expert and Zipf-skewed routing
    "e512_int4": LayerConfig("e512_int4", H=2048, E=512, I=512, top_k=10, score="softmax",
                             renormalize=False, rsf=1.0, wtype="int4", wscale="g32_f16",
                             act="g32_f16", shared_I=512, tokens=(1, 64, 4096), zipf=1.1),
    # the OLMoE-shaped decode layer with packed int2 experts (group-32 scales): the third code
    # container of the GLM page's quantization kernels
    "olmoe_int2": LayerConfig("olmoe_int2", H=2048, E=64, I=1024, top_k=8, score="softmax",
                              renormalize=True, rsf=1.0, wtype="int2", wscale="g32_f16",
                              act="g32_f16", tokens=(1, 8)),
}
CONFIG_ORDER = ["tiny", "olmoe_int8", "olmoe_int4", "glm_int4", "e512_int4", "olmoe_int2"]


def case_seed(cfg: LayerConfig, T: int, replica: int = 0) -> int:
    """Seed of one (workload, T, layer replica): 1000*config_index + T (+ 10^6 per replica)."""
    idx = CONFIG_ORDER.index(cfg.name) + 1 if cfg.name in CONFIG_ORDER else 99
    return 1000 * idx + T + 1_000_000 * replica


@dataclass
class Case:
    """All inputs of one layer invocation, generated on demand from one seed."""
    cfg: LayerConfig
    T: int
    seed: int
    _cache: dict = field(default_factory=dict, repr=False)

    @classmethod
    def make(cls, cfg: LayerConfig, T: int, replica: int = 0, seed: int | None = None) -> "Case":
        return cls(cfg, T, case_seed(cfg, T, replica) if seed is None else seed)

    def tseed(self, tag: int) -> int:
        return hash64(self.seed, tag)

    # ---- small tensors (host) -------------------------------------------------
    def x(self) -> np.ndarray:
        """Token activations [T][H] float32."""
        if "x" not in self._cache:
            c = self.cfg
            x = normal_cpu(self.T * c.H, self.tseed(TAG_X), 0, c.x_sigma).reshape(self.T, c.H)
            if c.zipf > 0:
                x[:, 0] = 1.0
            self._cache["x"] = x
        return self._cache["x"]

    def router_w(self) -> np.ndarray:
        """Router weight [E][H] float32 (Zipf workloads put ln p(rank_e) in column 0)."""
        if "wr" not in self._cache:
            c = self.cfg
            w = normal_cpu(c.E * c.H, self.tseed(TAG_WR), 0, c.router_sigma).reshape(c.E, c.H)
            if c.zipf > 0:
                w[:, 0] = zipf_log_prior(c.E, c.zipf, self.tseed(TAG_ZIPF))
            self._cache["wr"] = w
        return self._cache["wr"]

    def bias(self) -> np.ndarray | None:
        """Per-expert selection bias [E] (sigmoid noaux_tc only)."""
        c = self.cfg
        if c.score != "sigmoid":
            return None
        if "bias" not in self._cache:
            self._cache["bias"] = normal_cpu(c.E, self.tseed(TAG_BIAS), 0, c.bias_sigma or 0.05)
        return self._cache["bias"]

    # ---- expert weights, one expert at a time (host) --------------------------
    def gate_up(self, e: int) -> np.ndarray:
        """Expert e's fused gate||up weight [2I][H] (rows 0..I-1 gate, I..2I-1 up)."""
        c = self.cfg
        n = 2 * c.I * c.H
        return normal_cpu(n, self.tseed(TAG_GU), e * n, c.w_sigma).reshape(2 * c.I, c.H)

    def down(self, e: int) -> np.ndarray:
        """Expert e's down weight [H][I]."""
        c = self.cfg
        n = c.H * c.I
        return normal_cpu(n, self.tseed(TAG_DN), e * n, c.w_sigma).reshape(c.H, c.I)

    def shared_gate_up(self) -> np.ndarray:
        c = self.cfg
        return normal_cpu(2 * c.shared_I * c.H, self.tseed(TAG_SH_GU), 0, c.w_sigma).reshape(2 * c.shared_I, c.H)

    def shared_down(self) -> np.ndarray:
        c = self.cfg
        return normal_cpu(c.H * c.shared_I, self.tseed(TAG_SH_DN), 0, c.w_sigma).reshape(c.H, c.shared_I)

    # ---- whole expert tensors on the device ------------------------------------
    def gate_up_gpu(self, out) -> None:
        normal_gpu_(out, self.tseed(TAG_GU), 0, self.cfg.w_sigma)

    def down_gpu(self, out) -> None:
        normal_gpu_(out, self.tseed(TAG_DN), 0, self.cfg.w_sigma)

    def shared_gate_up_gpu(self, out) -> None:
        normal_gpu_(out, self.tseed(TAG_SH_GU), 0, self.cfg.w_sigma)

    def shared_down_gpu(self, out) -> None:
        normal_gpu_(out, self.tseed(TAG_SH_DN), 0, self.cfg.w_sigma)


def zipf_log_prior(E: int, s: float, seed: int) -> np.ndarray:
    """ln p(rank_e) with p(r) proportional to r^-s over ranks 1..E and a seeded rank permutation."""
    keys = np.array([hash64(seed, e) for e in range(E)], dtype=np.uint64)
    order = np.argsort(keys, kind="stable")          # expert order[r] gets rank r+1
    ranks = np.empty(E, dtype=np.int64)
    ranks[order] = np.arange(1, E + 1)
    p = ranks.astype(np.float64) ** (-s)
    p /= p.sum()
    return np.log(p).astype(np.float32)
