"""Host-side fault injection: a device allocation inside moe_pack_experts fails
(moe_debug_fail_alloc_after).  Every allocation point must return MOE_ERR_OOM
with no pack, free what it had allocated, and leave the library able to pack
and run a layer that matches the oracle.  The failure is made on the host: no
kernel runs while it is armed."""
import numpy as np
import pytest

import synth
from harness import DECODE_TOL, assert_routing_equal, gpu_layer, normwise_err, oracle_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_pack_reports_each_injected_allocation_failure_and_recovers():
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS["tiny_q8"]
    li = synth.layer_inputs(wl)
    bq.pack_layer(li, max_tokens=4).free()  # device set up before measuring
    free_before = torch.cuda.mem_get_info()[0]
    failures = 0
    try:
        for n in range(64):
            bq.moe_debug_fail_alloc_after(n)
            try:
                pack = bq.pack_layer(li, max_tokens=4)
            except bq.MoeError as e:
                assert e.status == bq.MOE_ERR_OOM
                failures += 1
                continue
            pack.free()  # n reached the pack's allocation count: it packed normally
            break
        else:
            pytest.fail("every pack attempt failed")
    finally:
        bq.moe_debug_fail_alloc_after(-1)
    # Q8_0: the code and scale planes of both projections, then the workspace (five here)
    assert failures >= 5, failures
    torch.cuda.synchronize()
    # the failed packs freed their allocations (a leaked code plane would be 17-34 MB;
    # the slack covers the driver's page granularity for the small ones)
    assert torch.cuda.mem_get_info()[0] >= free_before - (8 << 20)
    x = synth.tokens(wl, li.router, 0, 0, 4)
    out, idx, gate, _ = gpu_layer(li, x, wl.top_k)
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k)
    assert_routing_equal(idx, gate, ridx, rgate)
    assert normwise_err(out, ref) <= DECODE_TOL
