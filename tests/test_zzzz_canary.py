"""Canary-padded caller buffers: every path writes exactly the T rows of `out`
(and the router exactly the T rows of idx / gate) that the call names.  The
buffers handed to the library are row slices of larger tensors whose first and
last rows hold a sentinel that must survive the call; the rows in between must
be finite (NaN-filled before the call, so an unwritten row shows up too).
The file sorts last: it repeats paths the parity tests cover, with offset buffers."""
import numpy as np
import pytest

import synth
from harness import router_to_device, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _padded(T, C, dtype, fill, sentinel):
    """(full, rows): `rows` = T rows of C, between `pad` sentinel rows on each side;
    pad keeps the slice 16-byte aligned, as the C ABI asks of device pointers."""
    esize = torch.empty((), dtype=dtype).element_size()
    pad = next(p for p in range(1, 17) if (p * C * esize) % 16 == 0)
    full = torch.full((T + 2 * pad, C), fill, dtype=dtype, device="cuda")
    full[:pad] = sentinel
    full[T + pad:] = sentinel
    rows = full[pad:T + pad]
    assert rows.data_ptr() % 16 == 0
    return full, rows, pad


def _sentinels_intact(full, pad, sentinel):
    return bool((full[:pad] == sentinel).all() and (full[-pad:] == sentinel).all())


@pytest.mark.parametrize("name,T,path,flags", [
    ("tiny_q8", 1, "auto", 0),          # single-token streaming kernel
    ("model_decode", 1, "auto", 0),     # single-token streaming kernel, shared expert
    ("spec_verify", 8, "auto", 0),      # the one-launch tail (route, plan, tensor-core units, combine)
    ("zipf_batch", 64, "auto", 0),      # the one-launch tail at its largest token count
    ("spec_verify", 8, "staged", 0),    # router + tensor-core grouped decode + combine as separate launches
    ("tiny_q8", 5, "grouped", 0),       # plain grouped kernels
    ("zipf_batch", 16, "dense", 1),     # dense-batched comparison variant
    ("prefill_nvfp4", 300, "auto", 0),  # tensor-core prefill (output accumulated in place)
    ("prefill_q8", 130, "auto", 0),     # bf16-dequantising prefill
])
def test_forward_writes_exactly_its_rows(name, T, path, flags):
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS[name]
    li = synth.layer_inputs(wl, 0)
    x = to_device(synth.tokens(wl, li.router, 0, 0, T))
    wr = router_to_device(li.router)
    pack = bq.pack_layer(li, max_tokens=T, max_top_k=wl.top_k, flags=flags)
    try:
        full, out, pad = _padded(T, wl.hidden, torch.float32, float("nan"), -7.0)
        p = {"auto": bq.MOE_PATH_AUTO, "grouped": bq.MOE_PATH_GROUPED, "dense": bq.MOE_PATH_DENSE,
             "staged": bq.MOE_PATH_DECODE_STAGED}[path]
        bq.moe_layer_forward_ex(x, wr, pack, bq.MOE_FMT_FROM_PACK, wl.top_k, out, p)
        torch.cuda.synchronize()
        assert bq.moe_get_device_error(pack) == bq.MOE_OK
        assert _sentinels_intact(full, pad, -7.0)
        assert torch.isfinite(out).all()
    finally:
        pack.free()


def test_router_writes_exactly_its_rows():
    import block_quantized_expert_moe_b200 as bq
    for name, T in (("spec_verify", 8), ("zipf_batch", 64), ("prefill_nvfp4", 100)):
        wl = synth.WORKLOADS[name]
        wr_np, _ = synth.router(wl)
        x = to_device(synth.tokens(wl, wr_np, 0, 0, T))
        wr = router_to_device(wr_np)
        ifull, idx, ipad = _padded(T, wl.top_k, torch.int32, -1, -7)
        gfull, gate, gpad = _padded(T, wl.top_k, torch.float32, float("nan"), -7.0)
        ws = torch.empty(bq.moe_route_workspace_bytes(T, wl.n_experts), dtype=torch.uint8, device="cuda")
        bq.moe_route_topk(x, wr, wl.top_k, idx, gate, ws)
        torch.cuda.synchronize()
        assert _sentinels_intact(ifull, ipad, -7), name
        assert _sentinels_intact(gfull, gpad, -7.0), name
        i = idx.cpu().numpy()
        assert ((i >= 0) & (i < wl.n_experts)).all(), name
        assert np.allclose(gate.cpu().numpy().sum(axis=1), 1.0, atol=1e-5), name
