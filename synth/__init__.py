"""Seeded synthetic inputs for the block-quantised routed MoE layer.

This package is the one input source shared by the fp64 oracle's tests and by
the CUDA path's tests and benchmark.  It draws Gaussian numbers from a
counter-based generator (SplitMix64 into a normal-quantile table), rounds them
to the storage types and encodes weights into the canonical block formats
(see synth.c for the byte layouts).  It holds none of the layer's arithmetic.

Workloads (the MoE layer of a Qwen3.8-Flash-Next-style model as described by
the "Qwen3.8-Flash-Next UD-IQ2_XS (L4 fix) for Basalt" model card, section
"What was changed": routed experts in Q8_0, Q5_1, IQ4_NL or NVFP4 read by a
device-planned tail of grouped kernels):

  tiny_q8       H=1024 E=64  I=256 k=8  Q8_0 gate/up and down, fp32 x, T=1
  model_decode  H=2048 E=512 I=512 k=10 + shared expert, IQ4_NL gate/up,
                Q5_1 down, bf16 x, T=1
  spec_verify   48 layers of model_decode, T=8 correlated tokens (b + 0.3 eps)
  zipf_batch    48 layers, NVFP4, T=64, router biased to Zipf(1.1) popularity
  prefill       T=8192, Zipf(1.1), NVFP4 (and the same with Q8_0)
"""
import ctypes
import math
import os
from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

from . import build as _build

FMT_Q8_0, FMT_Q5_1, FMT_IQ4_NL, FMT_NVFP4, FMT_Q5_0 = 1, 2, 3, 4, 5
DT_F32, DT_BF16 = 1, 2
FMT_NAMES = {FMT_Q8_0: "q8_0", FMT_Q5_1: "q5_1", FMT_IQ4_NL: "iq4_nl", FMT_NVFP4: "nvfp4",
             FMT_Q5_0: "q5_0"}

# Synthetic IQ4_NL table: the 16 Lloyd-Max levels of N(0,1) (J. Max, "Quantizing
# for minimum distortion", IRE Trans. IT-6, 1960), scaled so the outermost level
# is 127 and rounded.  `lloyd_max_table()` recomputes it; it makes no claim of
# equality with any other engine's table, which the kernels take as an input.
IQ4NL_TABLE = np.array([-127, -96, -75, -58, -44, -31, -18, -6, 6, 18, 31, 44, 58, 75, 96, 127],
                       dtype=np.int8)

# Zipf popularity bias: Wr[e, H-1] = -ZIPF_BETA * s * ln(rank).  ZIPF_BETA was
# chosen with calibrate_zipf.py so that the realised top-10 selection counts of
# the 512-expert router follow rank^-1.1 (fitted log-log slope 1.1 +- 0.05).
ZIPF_BETA = 0.39


def lloyd_max_table(levels=16, peak=127, iters=2000):
    phi = lambda t: math.exp(-t * t / 2) / math.sqrt(2 * math.pi) if math.isfinite(t) else 0.0
    cdf = lambda t: 0.5 * math.erfc(-t / math.sqrt(2)) if math.isfinite(t) else float(t > 0)
    y = [-2.5 + 5 * i / (levels - 1) for i in range(levels)]
    for _ in range(iters):
        t = [-math.inf] + [(y[i] + y[i + 1]) / 2 for i in range(levels - 1)] + [math.inf]
        y = [(phi(t[i]) - phi(t[i + 1])) / (cdf(t[i + 1]) - cdf(t[i])) for i in range(levels)]
    s = peak / max(abs(v) for v in y)
    return np.array([int(round(v * s)) for v in y], dtype=np.int8)


@dataclass(frozen=True)
class Workload:
    name: str
    hidden: int
    n_experts: int
    inter: int
    top_k: int
    has_shared: bool
    fmt_gate_up: int
    fmt_down: int
    x_dtype: int
    tokens: int
    layers: int = 1
    corr: float = 0.0          # >0: x = b + corr * eps
    zipf_s: float = 0.0        # >0: popularity bias feature in column H-1
    sigma_w: float = 0.02
    sigma_r: float = 0.02
    margin: float = 1e-3
    seed: int = 0

    @property
    def n_packed(self):
        return self.n_experts + (1 if self.has_shared else 0)

    def gate_up_bytes(self):
        return row_bytes(self.fmt_gate_up, self.hidden) * 2 * self.inter

    def down_bytes(self):
        return row_bytes(self.fmt_down, self.inter) * self.hidden

    def expert_bytes(self):
        """HBM bytes of one expert's blocks (NVFP4 adds its two fp32 scales)."""
        extra = 8 if FMT_NVFP4 in (self.fmt_gate_up, self.fmt_down) else 0
        return self.gate_up_bytes() + self.down_bytes() + extra

    def with_(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    "tiny_q8": Workload("tiny_q8", 1024, 64, 256, 8, False, FMT_Q8_0, FMT_Q8_0, DT_F32, 1),
    "model_decode": Workload("model_decode", 2048, 512, 512, 10, True, FMT_IQ4_NL, FMT_Q5_1,
                             DT_BF16, 1),
    "spec_verify": Workload("spec_verify", 2048, 512, 512, 10, True, FMT_IQ4_NL, FMT_Q5_1,
                            DT_BF16, 8, layers=48, corr=0.3),
    "zipf_batch": Workload("zipf_batch", 2048, 512, 512, 10, False, FMT_NVFP4, FMT_NVFP4, DT_BF16,
                           64, layers=48, zipf_s=1.1),
    "prefill_nvfp4": Workload("prefill_nvfp4", 2048, 512, 512, 10, False, FMT_NVFP4, FMT_NVFP4,
                              DT_BF16, 8192, zipf_s=1.1),
    "prefill_q8": Workload("prefill_q8", 2048, 512, 512, 10, False, FMT_Q8_0, FMT_Q8_0, DT_BF16,
                           8192, zipf_s=1.1),
    # the model-shaped layer's formats (IQ4_NL gate/up, Q5_1 down, shared expert) in a prefill chunk
    "prefill_iq4nl_q51": Workload("prefill_iq4nl_q51", 2048, 512, 512, 10, True, FMT_IQ4_NL, FMT_Q5_1,
                                  DT_BF16, 8192, zipf_s=1.1),
}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u64, i64, i32, f32, f64, vp = (ctypes.c_uint64, ctypes.c_int64, ctypes.c_int,
                                       ctypes.c_float, ctypes.c_double, ctypes.c_void_p)
        L.synth_key.restype = u64
        L.synth_key.argtypes = [u64, u64, u64, u64, u64]
        L.synth_normal_f32.argtypes = [u64, i64, f32, vp]
        L.synth_normal_table.restype = vp
        L.synth_row_bytes.restype = i64
        L.synth_row_bytes.argtypes = [i32, i64]
        L.synth_encode.restype = i32
        L.synth_encode.argtypes = [i32, vp, i64, i64, vp, vp, vp]
        L.synth_round_bf16.argtypes = [vp, i64, vp]
        L.synth_expert.restype = i32
        L.synth_expert.argtypes = [u64, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp, vp, vp, vp]
        L.synth_layer_experts.restype = i32
        L.synth_layer_experts.argtypes = [u64, i32, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp,
                                          vp, vp, i32]
        L.synth_router.argtypes = [u64, i32, i32, i32, f32, f32, f32, vp, vp]
        L.synth_tokens.restype = i64
        L.synth_tokens.argtypes = [u64, i32, i32, i32, i32, i32, f32, i32, vp, i32, i32, f64, vp,
                                   i32]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def row_bytes(fmt, cols):
    return {FMT_Q8_0: cols // 32 * 34, FMT_Q5_1: cols // 32 * 24, FMT_IQ4_NL: cols // 32 * 18,
            FMT_NVFP4: cols // 16 * 9, FMT_Q5_0: cols // 32 * 22}[fmt]


def normal(key, n, sigma=1.0):
    out = np.empty(n, np.float32)
    lib().synth_normal_f32(key, n, sigma, _p(out))
    return out


def key(seed, a, b, c, d):
    return lib().synth_key(seed, a, b, c, d)


def bf16_bits(x):
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().synth_round_bf16(_p(x), x.size, _p(out))
    return out


def bf16_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def encode(fmt, w, table=None):
    """Encode a float matrix [rows, cols] into canonical blocks.
    Returns (uint8 [rows, row_bytes], tensor_scale or None)."""
    w = np.ascontiguousarray(w, np.float32)
    rows, cols = w.shape
    out = np.zeros((rows, row_bytes(fmt, cols)), np.uint8)
    ts = np.zeros(1, np.float32)
    tab = None if table is None else np.ascontiguousarray(table, np.int8)
    rc = lib().synth_encode(fmt, _p(w), rows, cols, _p(tab), _p(out), _p(ts))
    if rc:
        raise ValueError(f"synth_encode failed ({rc})")
    return out, (float(ts[0]) if fmt == FMT_NVFP4 else None)


@dataclass
class LayerInputs:
    """Host-side canonical inputs of one layer."""
    wl: Workload
    layer: int
    router: np.ndarray            # uint16 bf16 bits [E, H]
    gate_up: np.ndarray           # uint8 [n_packed, gate_up_bytes]
    down: np.ndarray              # uint8 [n_packed, down_bytes]
    gate_up_scale: Optional[np.ndarray]  # float32 [n_packed] (NVFP4) or None
    down_scale: Optional[np.ndarray]
    table: Optional[np.ndarray]   # int8 [16] (IQ4_NL) or None
    rank: Optional[np.ndarray]    # int32 [E] popularity rank (Zipf) or None


def router(wl: Workload, layer=0):
    wr = np.empty((wl.n_experts, wl.hidden), np.uint16)
    rank = np.zeros(wl.n_experts, np.int32) if wl.zipf_s > 0 else None
    lib().synth_router(wl.seed, layer, wl.n_experts, wl.hidden, wl.sigma_r, wl.zipf_s, ZIPF_BETA,
                       _p(wr), _p(rank))
    return wr, rank


def experts(wl: Workload, layer=0, e0=0, n=None, nthreads=0):
    """Blocks of experts [e0, e0+n); expert index n_experts is the shared one."""
    n = wl.n_packed - e0 if n is None else n
    gu = np.empty((n, wl.gate_up_bytes()), np.uint8)
    dn = np.empty((n, wl.down_bytes()), np.uint8)
    gts = np.ones(n, np.float32) if wl.fmt_gate_up == FMT_NVFP4 else None
    dts = np.ones(n, np.float32) if wl.fmt_down == FMT_NVFP4 else None
    tab = IQ4NL_TABLE if FMT_IQ4_NL in (wl.fmt_gate_up, wl.fmt_down) else None
    rc = lib().synth_layer_experts(wl.seed, layer, e0, n, wl.fmt_gate_up, wl.fmt_down, wl.hidden,
                                   wl.inter, wl.sigma_w, _p(tab), _p(gu), _p(dn), _p(gts), _p(dts),
                                   nthreads)
    if rc:
        raise RuntimeError(f"synth_layer_experts failed ({rc})")
    return gu, dn, gts, dts


def layer_inputs(wl: Workload, layer=0, nthreads=0) -> LayerInputs:
    wr, rank = router(wl, layer)
    gu, dn, gts, dts = experts(wl, layer, nthreads=nthreads)
    tab = IQ4NL_TABLE.copy() if FMT_IQ4_NL in (wl.fmt_gate_up, wl.fmt_down) else None
    return LayerInputs(wl, layer, wr, gu, dn, gts, dts, tab, rank)


def tokens(wl: Workload, wr, layer=0, step=0, n_tokens=None, max_attempts=4000):
    """Token vectors [T, H]: float32 for fp32 workloads, bf16 bits (uint16) otherwise."""
    T = wl.tokens if n_tokens is None else n_tokens
    dt = np.float32 if wl.x_dtype == DT_F32 else np.uint16
    out = np.empty((T, wl.hidden), dt)
    r = lib().synth_tokens(wl.seed, layer, step, T, wl.hidden, wl.x_dtype, wl.corr,
                           1 if wl.zipf_s > 0 else 0, _p(np.ascontiguousarray(wr, np.uint16)),
                           wl.n_experts, wl.top_k, wl.margin, _p(out), max_attempts)
    if r < 0:
        raise RuntimeError("synth_tokens: a token found no draw with the required top-k margin")
    return out


def tokens_f64(wl: Workload, x):
    """Token vectors as float64 (exact: they are fp32 or bf16 values)."""
    return (bf16_to_f32(x) if wl.x_dtype == DT_BF16 else np.asarray(x, np.float32)).astype(np.float64)
