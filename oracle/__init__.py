"""fp64 CPU oracle of the routed block-quantised MoE layer.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import this package.  It is a ctypes binding
of oracle.c (plain C, fp64), which states what it computes and which passages
it follows; it shares no code with the CUDA path.
"""
import ctypes

import numpy as np

from . import build as _build

Q8_0, Q5_1, IQ4_NL, NVFP4, Q5_0 = 1, 2, 3, 4, 5

_lib = None


class _Desc(ctypes.Structure):
    _fields_ = [("n_experts", ctypes.c_int), ("hidden", ctypes.c_int), ("inter", ctypes.c_int),
                ("has_shared", ctypes.c_int), ("fmt_gate_up", ctypes.c_int),
                ("fmt_down", ctypes.c_int), ("gate_up", ctypes.c_void_p),
                ("down", ctypes.c_void_p), ("gate_up_scale", ctypes.c_void_p),
                ("down_scale", ctypes.c_void_p), ("table", ctypes.c_void_p)]


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build())
        vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        for name in ("oracle_fp16", "oracle_bf16"):
            getattr(L, name).restype = f64
            getattr(L, name).argtypes = [ctypes.c_uint16]
        for name in ("oracle_e4m3", "oracle_e2m1"):
            getattr(L, name).restype = f64
            getattr(L, name).argtypes = [i32]
        L.oracle_row_bytes.restype = i64
        L.oracle_row_bytes.argtypes = [i32, i64]
        L.oracle_decode_row.restype = i32
        L.oracle_decode_row.argtypes = [i32, vp, i64, vp, f64, vp]
        L.oracle_route.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp]
        L.oracle_act_quant_nvfp4.argtypes = [vp, i64, vp]
        L.oracle_expert.restype = i32
        L.oracle_expert.argtypes = [ctypes.POINTER(_Desc), i32, vp, vp, i32]
        L.oracle_layer.restype = i32
        L.oracle_layer.argtypes = [ctypes.POINTER(_Desc), vp, vp, i32, i32, vp, vp, vp, i32]
        L.oracle_threads.restype = i32
        L.oracle_set_threads.argtypes = [i32]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def fp16(u):
    return lib().oracle_fp16(int(u))


def bf16(u):
    return lib().oracle_bf16(int(u))


def e4m3(c):
    return lib().oracle_e4m3(int(c))


def e2m1(c):
    return lib().oracle_e2m1(int(c))


def threads():
    return lib().oracle_threads()


def set_threads(n):
    """OpenMP threads of later layer calls (timing on one core: 1)."""
    lib().oracle_set_threads(int(n))


def decode_row(fmt, row, cols, table=None, tensor_scale=1.0):
    row = np.ascontiguousarray(row, np.uint8)
    out = np.empty(cols, np.float64)
    tab = None if table is None else np.ascontiguousarray(table, np.int8)
    rc = lib().oracle_decode_row(fmt, _p(row), cols, _p(tab), float(tensor_scale), _p(out))
    if rc:
        raise ValueError(f"oracle_decode_row failed ({rc})")
    return out


def decode_matrix(fmt, blocks, rows, cols, table=None, tensor_scale=1.0):
    blocks = np.ascontiguousarray(blocks, np.uint8).reshape(rows, -1)
    return np.stack([decode_row(fmt, blocks[r], cols, table, tensor_scale) for r in range(rows)])


def route(x, wr, k):
    """x: float64 [T, H]; wr: uint16 bf16 bits [E, H].  Returns idx int32 [T, k]
    (descending logit, ties to the lower index), gates float64 [T, k], logits [T, E]."""
    x = np.ascontiguousarray(x, np.float64)
    wr = np.ascontiguousarray(wr, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float64)
    logits = np.empty((T, E), np.float64)
    lib().oracle_route(_p(x), _p(wr), T, H, E, k, _p(idx), _p(gate), _p(logits))
    return idx, gate, logits


def act_quant_nvfp4(v):
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty_like(v)
    lib().oracle_act_quant_nvfp4(_p(v), v.size, _p(out))
    return out


class Experts:
    """Expert blocks handed to the oracle: row e of the block arrays holds expert e,
    row n_experts the shared expert (when there is one)."""

    def __init__(self, n_experts, hidden, inter, has_shared, fmt_gate_up, fmt_down, gate_up, down,
                 gate_up_scale=None, down_scale=None, table=None):
        self.keep = [np.ascontiguousarray(gate_up, np.uint8), np.ascontiguousarray(down, np.uint8)]
        gs = None if gate_up_scale is None else np.ascontiguousarray(gate_up_scale, np.float64)
        ds = None if down_scale is None else np.ascontiguousarray(down_scale, np.float64)
        tab = None if table is None else np.ascontiguousarray(table, np.int8)
        self.keep += [gs, ds, tab]
        self.desc = _Desc(n_experts, hidden, inter, 1 if has_shared else 0, fmt_gate_up, fmt_down,
                          _p(self.keep[0]), _p(self.keep[1]), _p(gs), _p(ds), _p(tab))
        self.hidden = hidden
        self.n_experts = n_experts

    @classmethod
    def from_layer(cls, li, gate_up=None, down=None, gate_up_scale=None, down_scale=None):
        wl = li.wl
        return cls(wl.n_experts, wl.hidden, wl.inter, wl.has_shared, wl.fmt_gate_up, wl.fmt_down,
                   li.gate_up if gate_up is None else gate_up, li.down if down is None else down,
                   li.gate_up_scale if gate_up_scale is None else gate_up_scale,
                   li.down_scale if down_scale is None else down_scale, li.table)

    def expert(self, e, x, act_quant=0):
        x = np.ascontiguousarray(x, np.float64)
        y = np.empty(self.hidden, np.float64)
        rc = lib().oracle_expert(ctypes.byref(self.desc), e, _p(x), _p(y), act_quant)
        if rc:
            raise ValueError(f"oracle_expert failed ({rc})")
        return y

    def layer(self, x, wr, k, act_quant=0):
        """Returns out float64 [T, H], idx int32 [T, k], gates float64 [T, k]."""
        x = np.ascontiguousarray(x, np.float64)
        wr = np.ascontiguousarray(wr, np.uint16)
        T = x.shape[0]
        out = np.empty((T, self.hidden), np.float64)
        idx = np.empty((T, k), np.int32)
        gate = np.empty((T, k), np.float64)
        rc = lib().oracle_layer(ctypes.byref(self.desc), _p(x), _p(wr), T, k, _p(out), _p(idx),
                                _p(gate), act_quant)
        if rc:
            raise ValueError(f"oracle_layer failed ({rc})")
        return out, idx, gate
