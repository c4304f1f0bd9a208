"""Failure paths, made without faulting the GPU.

* A device allocation inside moe_pack_experts fails (moe_debug_fail_alloc_after,
  made on the host): every allocation point returns MOE_ERR_OOM with no pack and
  frees what it had, and the library still packs and runs a layer that matches
  the oracle.
* A device-side bounded wait runs out (moe_debug_wait_timeout: an mbarrier that
  nothing arrives on): the kernel gives up after about a second, the pack's
  error word reads MOE_ERR_TIMEOUT once, and the same pack then runs a forward
  that matches the oracle.
The file sorts after the parity tests: it arms process-wide fault injection and
spends about a second in a deliberately exhausted wait.
"""
import time

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


def test_bounded_wait_runs_out_records_timeout_and_the_context_stays_usable():
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS["tiny_q8"]
    li = synth.layer_inputs(wl)
    pack = bq.pack_layer(li, max_tokens=4)
    try:
        assert bq.moe_get_device_error(pack) == bq.MOE_OK
        t0 = time.perf_counter()
        bq.moe_debug_wait_timeout(pack)
        torch.cuda.synchronize()
        waited = time.perf_counter() - t0
        assert bq.moe_get_device_error(pack) == bq.MOE_ERR_TIMEOUT
        assert bq.moe_get_device_error(pack) == bq.MOE_OK  # reading clears the word
        assert 0.2 < waited < 10.0, waited  # 2^31 SM clocks: about a second
        x = synth.tokens(wl, li.router, 0, 1, 4)
        out, idx, gate, _ = gpu_layer(li, x, wl.top_k, pack=pack)
        ref, ridx, rgate = oracle_layer(li, x, wl.top_k)
        assert_routing_equal(idx, gate, ridx, rgate)
        assert normwise_err(out, ref) <= DECODE_TOL
    finally:
        pack.free()
