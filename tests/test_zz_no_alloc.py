"""The allocation-free router entry point (moe_route_topk_noalloc) against the
workspace one (moe_route_topk) and the oracle, through the C ABI.

moe_route_topk_noalloc serves callers that cannot allocate device memory: code
running while a global-mode stream capture is open, where cudaMalloc is an
illegal call, or a framework that forbids cudaMalloc once it serves requests
because it can synchronise the device.  Its scratch is a fixed array inside the
library (at most 65,536 logits), shared by every call on a device.  This file is
collected after the parity tests so a run that stops at the first failure has
run them first."""
import numpy as np
import pytest

import synth
from harness import GATE_TOL, router_to_device, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _both(bq, wl, wr, x, T):
    idx_ws = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
    gate_ws = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
    ws = torch.empty(bq.moe_route_workspace_bytes(T, wl.n_experts), dtype=torch.uint8, device="cuda")
    bq.moe_route_topk(x, wr, wl.top_k, idx_ws, gate_ws, ws)
    idx_na = torch.full((T, wl.top_k), -1, dtype=torch.int32, device="cuda")
    gate_na = torch.full((T, wl.top_k), -1.0, dtype=torch.float32, device="cuda")
    bq.moe_route_topk_noalloc(x, wr, wl.top_k, idx_na, gate_na)
    torch.cuda.synchronize()
    assert bq.moe_route_noalloc_status() == bq.MOE_OK
    return idx_ws.cpu().numpy(), gate_ws.cpu().numpy(), idx_na.cpu().numpy(), gate_na.cpu().numpy()


@pytest.mark.parametrize("name,T", [("model_decode", 8), ("tiny_q8", 3)])
def test_noalloc_route_matches_workspace_route(name, T):
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS[name]
    wr_np, _ = synth.router(wl)
    wr = router_to_device(wr_np)
    for call in range(2):  # two calls in a row share the library's scratch
        x = to_device(synth.tokens(wl, wr_np, 0, call, T))
        idx_ws, gate_ws, idx_na, gate_na = _both(bq, wl, wr, x, T)
        assert np.array_equal(idx_na, idx_ws), call
        assert np.abs(gate_na - gate_ws).max() <= GATE_TOL, call


def test_noalloc_route_at_the_scratch_limit_then_a_smaller_call():
    """128 bf16 tokens x 512 experts fill the 65,536 logits exactly; above 64 bf16
    tokens moe_route_topk runs its tensor-core GEMM while this entry point keeps the
    CUDA-core router, so both are checked against the oracle.  Then a call with
    fewer experts (64) reads only its own logits, not the larger call's leftovers."""
    import block_quantized_expert_moe_b200 as bq
    import oracle
    for name, T in (("model_decode", 128), ("tiny_q8", 5), ("model_decode", 128)):
        wl = synth.WORKLOADS[name]
        assert name != "model_decode" or T * wl.n_experts == 65536
        wr_np, _ = synth.router(wl)
        x_np = synth.tokens(wl, wr_np, 0, 3, T)
        idx_ws, gate_ws, idx_na, gate_na = _both(bq, wl, router_to_device(wr_np), to_device(x_np), T)
        ridx, rgate, _ = oracle.route(synth.tokens_f64(wl, x_np), wr_np, wl.top_k)
        assert np.array_equal(idx_na, ridx) and np.array_equal(idx_ws, ridx), name
        assert np.abs(gate_na - rgate).max() <= GATE_TOL and np.abs(gate_ws - rgate).max() <= GATE_TOL


def test_noalloc_route_writes_exactly_its_rows():
    """idx_out and gate_out as row slices of larger buffers: the sentinel rows around
    them survive, every row in between is written."""
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS["model_decode"]
    wr_np, _ = synth.router(wl)
    T, k, pad = 7, wl.top_k, 2  # 2 rows of 10 int32 / fp32 = 80 bytes: slices stay 16-byte aligned
    x = to_device(synth.tokens(wl, wr_np, 0, 1, T))
    idx_full = torch.full((T + 2 * pad, k), -5, dtype=torch.int32, device="cuda")
    gate_full = torch.full((T + 2 * pad, k), -5.0, dtype=torch.float32, device="cuda")
    idx, gate = idx_full[pad:T + pad], gate_full[pad:T + pad]
    assert idx.data_ptr() % 16 == 0 and gate.data_ptr() % 16 == 0
    bq.moe_route_topk_noalloc(x, router_to_device(wr_np), k, idx, gate)
    torch.cuda.synchronize()
    for full in (idx_full, gate_full):
        assert (full[:pad] == -5).all() and (full[T + pad:] == -5).all()
    assert (idx >= 0).all() and (idx < wl.n_experts).all()
    assert torch.allclose(gate.sum(1), torch.ones(T, device="cuda"), atol=1e-5)


def test_noalloc_route_reports_a_timed_out_wait():
    """The diagnostic bounded wait (nothing ever arrives) records MOE_ERR_TIMEOUT in the
    allocation-free router's error word; the status call reports it once and clears
    it, and the router then works again."""
    import block_quantized_expert_moe_b200 as bq
    bq.moe_debug_noalloc_wait_timeout()
    assert bq.moe_route_noalloc_status() == bq.MOE_ERR_TIMEOUT
    assert bq.moe_route_noalloc_status() == bq.MOE_OK
    wl = synth.WORKLOADS["tiny_q8"]
    wr_np, _ = synth.router(wl)
    x = to_device(synth.tokens(wl, wr_np, 0, 0, 2))
    idx_ws, _, idx_na, _ = _both(bq, wl, router_to_device(wr_np), x, 2)
    assert np.array_equal(idx_na, idx_ws)


def test_noalloc_route_rejects_more_than_its_scratch_holds():
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS["model_decode"]
    wr = torch.zeros(wl.n_experts, wl.hidden, dtype=torch.int16, device="cuda")
    x = torch.zeros(129, wl.hidden, dtype=torch.bfloat16, device="cuda")  # 129 * 512 > 65536
    idx = torch.empty(129, wl.top_k, dtype=torch.int32, device="cuda")
    gate = torch.empty(129, wl.top_k, dtype=torch.float32, device="cuda")
    with pytest.raises(bq.MoeError) as e:
        bq.moe_route_topk_noalloc(x, wr, wl.top_k, idx, gate)
    assert e.value.status == bq.MOE_ERR_INVALID_ARG
