"""The allocation-free router entry point (moe_route_topk_noalloc) against the
workspace one (moe_route_topk), through the C ABI, on two calls in a row.

moe_route_topk_noalloc serves callers that cannot allocate device memory
(an open global-mode stream capture, or a framework that forbids cudaMalloc
after start-up); its scratch is a fixed array inside the library.  This file is
collected after the parity tests so a run that stops at the first failure has
run them first."""
import numpy as np
import pytest

import synth
from harness import GATE_TOL, router_to_device, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,T", [("model_decode", 8), ("tiny_q8", 3)])
def test_noalloc_route_matches_workspace_route(name, T):
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS[name]
    wr_np, _ = synth.router(wl)
    wr = router_to_device(wr_np)
    for call in range(2):  # two calls in a row share the library's scratch
        x = to_device(synth.tokens(wl, wr_np, 0, call, T))
        idx_ws = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
        gate_ws = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
        ws = torch.empty(bq.moe_route_workspace_bytes(T, wl.n_experts), dtype=torch.uint8, device="cuda")
        bq.moe_route_topk(x, wr, wl.top_k, idx_ws, gate_ws, ws)
        idx_na = torch.full((T, wl.top_k), -1, dtype=torch.int32, device="cuda")
        gate_na = torch.full((T, wl.top_k), -1.0, dtype=torch.float32, device="cuda")
        bq.moe_route_topk_noalloc(x, wr, wl.top_k, idx_na, gate_na)
        torch.cuda.synchronize()
        assert np.array_equal(idx_na.cpu().numpy(), idx_ws.cpu().numpy()), call
        assert np.abs(gate_na.cpu().numpy() - gate_ws.cpu().numpy()).max() <= GATE_TOL, call


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
