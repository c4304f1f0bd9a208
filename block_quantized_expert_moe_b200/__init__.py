"""Python binding of libmoe, the C-ABI library of the block-quantised routed
MoE layer for B200 (include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Device buffers are torch CUDA tensors (PyTorch provides memory and
streams); weights enter as canonical blocks in host numpy arrays.  The library
must be built (build.py, or __graft_entry__.build()); importing this module
without it raises, there is no other implementation.
"""
import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_FMT_MISMATCH = 0, 1, 2, 3
MOE_ERR_OOM, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE, MOE_ERR_RANGE = 4, 5, 6, 7, 8
MOE_FMT_FROM_PACK, MOE_FMT_Q8_0, MOE_FMT_Q5_1, MOE_FMT_IQ4_NL, MOE_FMT_NVFP4, MOE_FMT_Q5_0 = 0, 1, 2, 3, 4, 5
MOE_DT_F32, MOE_DT_BF16 = 1, 2
MOE_PATH_AUTO, MOE_PATH_DECODE, MOE_PATH_PREFILL, MOE_PATH_DENSE, MOE_PATH_GROUPED = 0, 1, 2, 3, 4
MOE_PATH_DECODE_STAGED, MOE_PATH_TAIL, MOE_PATH_PREFILL_BF16 = 5, 6, 7


class MoeError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {moe_status_string(status)} ({status})")


class moe_pack_desc(ctypes.Structure):
    _fields_ = [("n_experts", ctypes.c_int), ("hidden", ctypes.c_int), ("inter", ctypes.c_int),
                ("has_shared", ctypes.c_int), ("max_tokens", ctypes.c_int),
                ("max_top_k", ctypes.c_int), ("fmt_gate_up", ctypes.c_int),
                ("fmt_down", ctypes.c_int), ("gate_up_blocks", ctypes.c_void_p),
                ("down_blocks", ctypes.c_void_p), ("gate_up_tensor_scale", ctypes.c_void_p),
                ("down_tensor_scale", ctypes.c_void_p), ("iq4nl_table", ctypes.c_void_p),
                ("shared_gate_up_blocks", ctypes.c_void_p),
                ("shared_down_blocks", ctypes.c_void_p), ("flags", ctypes.c_int),
                ("expert_begin", ctypes.c_int), ("expert_end", ctypes.c_int)]


MOE_PACK_DENSE = 1


class moe_pack_info(ctypes.Structure):
    _fields_ = [("gate_up_bytes_per_expert", ctypes.c_int64),
                ("down_bytes_per_expert", ctypes.c_int64), ("expert_bytes", ctypes.c_int64),
                ("arena_bytes", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64),
                ("device", ctypes.c_int), ("code_table_masked", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmoe.so is not built ({LIB_PATH}); run block_quantized_expert_moe_b200/build.py")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [i32]
    L.moe_pack_experts.restype = i32
    L.moe_pack_experts.argtypes = [ctypes.POINTER(moe_pack_desc), i32, ctypes.POINTER(vp)]
    L.moe_pack_free.restype = i32
    L.moe_pack_free.argtypes = [vp]
    L.moe_pack_query.restype = i32
    L.moe_pack_query.argtypes = [vp, ctypes.POINTER(moe_pack_info)]
    L.moe_route_workspace_bytes.restype = sz
    L.moe_route_workspace_bytes.argtypes = [i32, i32]
    L.moe_route_topk.restype = i32
    L.moe_route_topk.argtypes = [vp, i32, vp, i32, i32, i32, i32, vp, vp, vp, sz, vp]
    L.moe_route_topk_noalloc.restype = i32
    L.moe_route_topk_noalloc.argtypes = [vp, i32, vp, i32, i32, i32, i32, vp, vp, vp]
    L.moe_route_noalloc_status.restype = i32
    L.moe_route_noalloc_status.argtypes = []
    L.moe_debug_noalloc_wait_timeout.restype = i32
    L.moe_debug_noalloc_wait_timeout.argtypes = [vp]
    L.moe_layer_forward.restype = i32
    L.moe_layer_forward.argtypes = [vp, i32, vp, vp, i32, i32, i32, vp, vp]
    L.moe_layer_forward_ex.restype = i32
    L.moe_layer_forward_ex.argtypes = [vp, i32, vp, vp, i32, i32, i32, vp, i32, vp]
    L.moe_debug_wait_timeout.restype = i32
    L.moe_debug_wait_timeout.argtypes = [vp, vp]
    L.moe_debug_act_quant_nvfp4.restype = i32
    L.moe_debug_act_quant_nvfp4.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
    L.moe_debug_dequant_rows.restype = i32
    L.moe_debug_dequant_rows.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp]
    L.moe_debug_tail_plan.restype = i32
    L.moe_debug_tail_plan.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32, i32, vp]
    L.moe_debug_fail_alloc_after.restype = i32
    L.moe_debug_fail_alloc_after.argtypes = [i32]
    L.moe_read_routing.restype = i32
    L.moe_read_routing.argtypes = [vp, i32, i32, vp, vp, vp, vp]
    L.moe_profile_begin.restype = i32
    L.moe_profile_begin.argtypes = [vp, i32]
    L.moe_profile_end.restype = i32
    L.moe_profile_end.argtypes = [vp, vp, vp]
    L.moe_get_device_error.restype = i32
    L.moe_get_device_error.argtypes = [vp]
    return L


lib = _load()


def moe_status_string(status):
    return lib.moe_status_string(int(status)).decode()


def _check(status, what):
    if status != MOE_OK:
        raise MoeError(status, what)


def _np_ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _stream_ptr(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _shape2(t, name):
    shape = tuple(getattr(t, "shape", ()))
    if len(shape) != 2:
        raise ValueError(f"{name} must be 2-D, not of shape {shape}")
    return shape


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return MOE_DT_F32
    if t.dtype == torch.bfloat16:
        return MOE_DT_BF16
    raise TypeError(f"activations must be float32 or bfloat16, not {t.dtype}")


def _check_tensor(t, name, dtypes, shape):
    """What the C ABI cannot check from a pointer: type, dtype, shape, contiguity."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor, not {type(t).__name__}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must be {' or '.join(str(d) for d in dtypes)}, not {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _device_ptrs(named, device):
    """Device pointers of already checked tensors, all in CUDA memory on `device`
    (default: the first tensor's); raises before any library call."""
    ptrs = []
    for name, t in named:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor: the library reads and writes device memory")
        if device is None:
            device = t.device.index
        if t.device.index != device:
            raise ValueError(f"{name} is on cuda:{t.device.index}, expected cuda:{device}")
        ptrs.append(t.data_ptr())
    return ptrs


def _act_dtypes():
    import torch
    return (torch.float32, torch.bfloat16)


def _bf16_bits_dtypes():
    import torch
    return (torch.bfloat16, torch.int16, torch.uint16)


class Pack:
    """An uploaded expert pack (owns device memory until free())."""

    def __init__(self, handle, desc, device=0):
        self.handle = handle
        self.device = device
        self.n_experts = desc.n_experts
        self.hidden = desc.hidden
        self.inter = desc.inter
        self.has_shared = bool(desc.has_shared)
        self.max_tokens = desc.max_tokens
        self.max_top_k = desc.max_top_k
        self.fmt_gate_up = desc.fmt_gate_up
        self.fmt_down = desc.fmt_down

    def info(self):
        return moe_pack_query(self)

    def free(self):
        if self.handle:
            _check(lib.moe_pack_free(self.handle), "moe_pack_free")
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def moe_pack_experts(n_experts, hidden, inter, fmt_gate_up, fmt_down, gate_up_blocks, down_blocks,
                     gate_up_tensor_scale=None, down_tensor_scale=None, iq4nl_table=None,
                     shared_gate_up_blocks=None, shared_down_blocks=None, max_tokens=64,
                     max_top_k=None, device=0, flags=0, expert_window=None):
    """Upload a layer's experts.  Blocks are host uint8 arrays in the canonical
    layout of include/moe.h (expert-major); NVFP4 scales float32 [E(+1)].
    expert_window=(begin, end): the blocks hold only those routed experts (expert
    parallelism: the forward computes that window's share of the layer)."""
    keep = [np.ascontiguousarray(gate_up_blocks, np.uint8), np.ascontiguousarray(down_blocks, np.uint8)]
    opt = lambda a, dt: None if a is None else np.ascontiguousarray(a, dt)
    gts, dts = opt(gate_up_tensor_scale, np.float32), opt(down_tensor_scale, np.float32)
    tab = opt(iq4nl_table, np.int8)
    sgu, sdn = opt(shared_gate_up_blocks, np.uint8), opt(shared_down_blocks, np.uint8)
    keep += [gts, dts, tab, sgu, sdn]
    d = moe_pack_desc(n_experts, hidden, inter, 1 if sgu is not None else 0, max_tokens,
                      max_top_k if max_top_k is not None else n_experts, fmt_gate_up, fmt_down,
                      _np_ptr(keep[0]), _np_ptr(keep[1]), _np_ptr(gts), _np_ptr(dts), _np_ptr(tab),
                      _np_ptr(sgu), _np_ptr(sdn), flags,
                      *((0, 0) if expert_window is None else expert_window))
    h = ctypes.c_void_p()
    _check(lib.moe_pack_experts(ctypes.byref(d), device, ctypes.byref(h)), "moe_pack_experts")
    return Pack(h, d, device)


def moe_pack_free(pack):
    pack.free()


def moe_pack_query(pack):
    info = moe_pack_info()
    _check(lib.moe_pack_query(pack.handle, ctypes.byref(info)), "moe_pack_query")
    return {f: getattr(info, f) for f, _ in moe_pack_info._fields_}


def moe_debug_wait_timeout(pack, stream=None):
    """Tests only: a kernel's bounded wait runs out (~1 s) and records MOE_ERR_TIMEOUT in the pack."""
    _check(lib.moe_debug_wait_timeout(pack.handle, _stream_ptr(stream)), "moe_debug_wait_timeout")


def moe_debug_fail_alloc_after(n):
    """Tests only: the (n+1)-th device allocation of moe_pack_experts from now fails once (-1: off)."""
    _check(lib.moe_debug_fail_alloc_after(n), "moe_debug_fail_alloc_after")


def moe_debug_act_quant_nvfp4(x, stream=None):
    """Tests only: the NVFP4 prefill's activation quantiser on the rows of x (CUDA
    [rows, cols]; bf16: the gate/up activations' quantiser, float32: the down
    activations').  Returns CUDA tensors (codes uint8 [rows, cols/2], E4M3 scales
    uint8 [rows, cols/16], row scales float32 [rows])."""
    import torch
    rows, cols = _shape2(x, "x")
    _check_tensor(x, "x", _act_dtypes(), (rows, cols))
    dev = x.device
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(rows, max(cols // 16, 1), dtype=torch.uint8, device=dev)
    row_scale = torch.empty(rows, dtype=torch.float32, device=dev)
    px, pc, ps, pr = _device_ptrs([("x", x), ("codes", codes), ("scales", scales), ("row_scale", row_scale)], None)
    _check(lib.moe_debug_act_quant_nvfp4(px, _dtype_code(x), rows, cols, pc, ps, pr, _stream_ptr(stream)),
           "moe_debug_act_quant_nvfp4")
    return codes, scales, row_scale


def moe_debug_dequant_rows(pack, proj, slot, row0, nrows, kind, cols, stream=None):
    """Tests only: the block decoders on rows of a packed projection (proj 0 gate/up,
    1 down; kind 0: the tensor-core decode's fp16 expansion, returned as float16;
    kind 1: the bf16-dequantising prefill's fp32 values).  cols: the projection's
    row length (H for gate/up, I for down).  Returns a CUDA tensor [nrows, cols]."""
    import torch
    dt = torch.float16 if kind == 0 else torch.float32
    out = torch.empty(nrows, cols, dtype=dt, device=f"cuda:{pack.device}")
    _check(lib.moe_debug_dequant_rows(pack.handle, proj, slot, row0, nrows, kind, out.data_ptr(), _stream_ptr(stream)),
           "moe_debug_dequant_rows")
    return out


def moe_debug_tail_plan(n_tokens, max_tokens, hidden, n_experts, inter, top_k, x_dtype, fmt_gate_up, fmt_down,
                        grid):
    """Tests only (no device): the one-launch tail's shared-memory plan, a dict (fits False
    when the tail does not take the shape)."""
    out = (ctypes.c_int64 * 8)()
    _check(lib.moe_debug_tail_plan(n_tokens, max_tokens, hidden, n_experts, inter, top_k, x_dtype, fmt_gate_up,
                                   fmt_down, grid, out), "moe_debug_tail_plan")
    keys = ("fits", "raw_stages", "b_slots", "raw_stage_bytes", "b_slot_bytes", "rings_bytes", "smem_bytes",
            "a_stages")
    d = dict(zip(keys, list(out)))
    d["fits"] = bool(d["fits"])
    return d


def moe_route_workspace_bytes(n_tokens, n_experts):
    return lib.moe_route_workspace_bytes(n_tokens, n_experts)


def moe_route_topk(x, router_w, top_k, idx_out, gate_out, workspace, stream=None):
    """x: CUDA [T, H] float32/bfloat16; router_w: CUDA [E, H] bf16 bits (bfloat16,
    int16 or uint16 tensor); idx_out int32 [T, k]; gate_out float32 [T, k];
    workspace: CUDA uint8 tensor of moe_route_workspace_bytes(T, E) bytes."""
    T, H, E, named = _route_tensors(x, router_w, top_k, idx_out, gate_out)
    _check_tensor(workspace, "workspace", (workspace.dtype,), tuple(getattr(workspace, "shape", ())))
    px, pw, pi, pg, pws = _device_ptrs(named + [("workspace", workspace)], None)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.moe_route_topk(px, _dtype_code(x), pw, T, H, E, top_k, pi, pg, pws, ws_bytes,
                              _stream_ptr(stream)), "moe_route_topk")


def moe_route_topk_noalloc(x, router_w, top_k, idx_out, gate_out, stream=None):
    """moe_route_topk for callers that cannot allocate: the scratch is a fixed
    array inside the library (n_tokens * n_experts <= 65536; calls that overlap
    on the GPU race; the first call on a device must precede any capture)."""
    T, H, E, named = _route_tensors(x, router_w, top_k, idx_out, gate_out)
    px, pw, pi, pg = _device_ptrs(named, None)
    _check(lib.moe_route_topk_noalloc(px, _dtype_code(x), pw, T, H, E, top_k, pi, pg, _stream_ptr(stream)),
           "moe_route_topk_noalloc")


def moe_route_noalloc_status():
    """Status of the last moe_route_topk_noalloc call on the current device (MOE_OK
    or MOE_ERR_TIMEOUT); synchronises the device and clears it."""
    return lib.moe_route_noalloc_status()


def moe_debug_noalloc_wait_timeout(stream=None):
    """Tests only: a bounded wait runs out (~1 s) and records MOE_ERR_TIMEOUT in the
    allocation-free router's error word."""
    _check(lib.moe_debug_noalloc_wait_timeout(_stream_ptr(stream)), "moe_debug_noalloc_wait_timeout")


def _route_tensors(x, router_w, top_k, idx_out, gate_out):
    import torch
    T, H = _shape2(x, "x")
    E = _shape2(router_w, "router_w")[0]
    _check_tensor(x, "x", _act_dtypes(), (T, H))
    _check_tensor(router_w, "router_w", _bf16_bits_dtypes(), (E, H))
    _check_tensor(idx_out, "idx_out", (torch.int32,), (T, top_k))
    _check_tensor(gate_out, "gate_out", (torch.float32,), (T, top_k))
    return T, H, E, [("x", x), ("router_w", router_w), ("idx_out", idx_out), ("gate_out", gate_out)]


def _forward_ptrs(x, router_w, pack, out):
    import torch
    T = _shape2(x, "x")[0]
    H, E = pack.hidden, pack.n_experts
    _check_tensor(x, "x", _act_dtypes(), (T, H))
    _check_tensor(router_w, "router_w", _bf16_bits_dtypes(), (E, H))
    _check_tensor(out, "out", (torch.float32,), (T, H))
    px, pw, po = _device_ptrs([("x", x), ("router_w", router_w), ("out", out)], pack.device)
    return T, px, pw, po


def moe_layer_forward(x, router_w, pack, fmt, top_k, out, stream=None):
    """out[T, H] (float32 CUDA) = the MoE layer on x[T, H] (float32/bfloat16 CUDA)."""
    T, px, pw, po = _forward_ptrs(x, router_w, pack, out)
    _check(lib.moe_layer_forward(px, _dtype_code(x), pw, pack.handle, fmt, T, top_k, po, _stream_ptr(stream)),
           "moe_layer_forward")


def moe_layer_forward_ex(x, router_w, pack, fmt, top_k, out, path, stream=None):
    T, px, pw, po = _forward_ptrs(x, router_w, pack, out)
    _check(lib.moe_layer_forward_ex(px, _dtype_code(x), pw, pack.handle, fmt, T, top_k, po, path,
                                    _stream_ptr(stream)), "moe_layer_forward_ex")


def moe_read_routing(pack, n_tokens, top_k, stream=None):
    """Routing of the last forward on `pack`, to host: (idx [T,k], gate [T,k], counts [E+1])."""
    idx = np.empty((n_tokens, top_k), np.int32)
    gate = np.empty((n_tokens, top_k), np.float32)
    counts = np.empty(pack.n_experts + 1, np.int32)
    _check(lib.moe_read_routing(pack.handle, n_tokens, top_k, _np_ptr(idx), _np_ptr(gate),
                                _np_ptr(counts), _stream_ptr(stream)), "moe_read_routing")
    return idx, gate, counts


def moe_profile_begin(pack, max_forwards):
    _check(lib.moe_profile_begin(pack.handle, max_forwards), "moe_profile_begin")


def moe_profile_end(pack):
    """-> (ms[32] summed over recorded forwards: route+plan, gate/up, down, combine,
    fused, prefill, the fused kernel's nine phases, then the streaming kernel's
    grid events and its first CTA's sub-step times; n_forwards)."""
    ms = np.zeros(32, np.float64)
    n = ctypes.c_int(0)
    _check(lib.moe_profile_end(pack.handle, _np_ptr(ms), ctypes.byref(n)), "moe_profile_end")
    return ms, n.value


def moe_get_device_error(pack):
    return lib.moe_get_device_error(pack.handle)


def pack_layer(li, max_tokens=64, max_top_k=None, device=0, flags=0, expert_window=None, shared=True):
    """Pack a synth.LayerInputs-like object (router, gate_up, down, scales, table).
    expert_window=(begin, end) packs only those routed experts (and the shared
    expert if the layer has one and `shared`)."""
    wl = li.wl
    E = wl.n_experts
    b, e = (0, E) if expert_window is None else expert_window
    has_sh = wl.has_shared and shared
    idx = list(range(b, e)) + ([E] if has_sh else [])
    gs = None if li.gate_up_scale is None else li.gate_up_scale[idx]
    ds = None if li.down_scale is None else li.down_scale[idx]
    return moe_pack_experts(E, wl.hidden, wl.inter, wl.fmt_gate_up, wl.fmt_down, li.gate_up[b:e],
                            li.down[b:e], gs, ds, li.table,
                            li.gate_up[E] if has_sh else None,
                            li.down[E] if has_sh else None, max_tokens,
                            max_top_k if max_top_k is not None else wl.top_k, device, flags,
                            None if expert_window is None else (b, e))
