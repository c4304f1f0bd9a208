"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Routing: the selected expert set of every token must equal the oracle's
(inputs carry a top-k logit margin >= 1e-3) and gates agree within 1e-5.
Outputs: normwise max relative error per token <= 2e-3 (fp32-accumulate
decode kernels).
"""
import numpy as np
import pytest

import synth
from harness import (DECODE_TOL, assert_routing_equal, expected_counts, gpu_layer, normwise_err,
                     oracle_layer, router_to_device, to_device)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _layer(name, layer=0, **kw):
    wl = synth.WORKLOADS[name].with_(**kw) if kw else synth.WORKLOADS[name]
    return wl, synth.layer_inputs(wl, layer)


def _check(li, x, k, tol=DECODE_TOL, path=None):
    out, idx, gate, counts = gpu_layer(li, x, k, path=path)
    ref, ridx, rgate = oracle_layer(li, x, k)
    assert_routing_equal(idx, gate, ridx, rgate)
    assert np.array_equal(counts, expected_counts(ridx, li.wl.n_experts, x.shape[0], li.wl.has_shared))
    err = normwise_err(out, ref)
    assert err <= tol, err
    return err


@pytest.mark.parametrize("layer", [0, 1, 2])
def test_tiny_q8_decode_one_token(layer):
    wl, li = _layer("tiny_q8", layer)
    _check(li, synth.tokens(wl, li.router, layer), wl.top_k)


@pytest.mark.parametrize("step", [0, 1])
def test_model_decode_iq4nl_q51_shared_one_token(step):
    wl, li = _layer("model_decode")
    _check(li, synth.tokens(wl, li.router, 0, step), wl.top_k)


def test_spec_verify_eight_correlated_tokens():
    wl, li = _layer("spec_verify", layer=5)
    err = _check(li, synth.tokens(wl, li.router, 5), wl.top_k)
    # the tensor-core decode rounds weights and h to fp16: the margin to 2e-3 is printed
    print(f"spec_verify (8 tokens, tensor-core decode): normwise err {err:.3e} of {DECODE_TOL:.0e}")


def test_zipf_batch_nvfp4_64_tokens():
    wl, li = _layer("zipf_batch", layer=2)
    err = _check(li, synth.tokens(wl, li.router, 2), wl.top_k)
    print(f"zipf_batch (64 tokens, NVFP4, tensor-core decode): normwise err {err:.3e} of {DECODE_TOL:.0e}")


@pytest.mark.parametrize("name,layer,T", [("spec_verify", 3, 8), ("zipf_batch", 4, 64), ("model_decode", 2, 1),
                                          ("tiny_q8", 1, 17)])
def test_one_launch_tail_matches_oracle_and_staged_path(name, layer, T):
    """The device-planned tail in one launch (route, plan, tensor-core gate/up and down,
    combine) against the oracle, and against the same tensor-core work run as separate
    launches: both round weights, x and h to fp16 the same way, only the order of the
    fp32 sums differs."""
    import block_quantized_expert_moe_b200 as bq
    wl, li = _layer(name, layer)
    x = synth.tokens(wl, li.router, layer, 5, T)
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k)
    out_t, idx, gate, counts = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_TAIL)
    assert_routing_equal(idx, gate, ridx, rgate)
    assert np.array_equal(counts, expected_counts(ridx, wl.n_experts, T, wl.has_shared))
    err = normwise_err(out_t, ref)
    assert err <= DECODE_TOL, err
    print(f"{name} ({T} tokens, one-launch tail): normwise err {err:.3e} of {DECODE_TOL:.0e}")
    if T >= 2:
        out_s, _, _, _ = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_DECODE_STAGED)
        assert normwise_err(out_s, ref) <= DECODE_TOL
        assert normwise_err(out_t, out_s) <= 1e-4


@pytest.mark.parametrize("name,T", [("model_decode", 100), ("tiny_q8", 150)])
def test_grouped_path_above_64_tokens_matches_oracle(name, T):
    """MOE_PATH_GROUPED (fp32 CUDA-core matvecs) is not limited to decode batches:
    checked against the oracle at more than 64 tokens (bf16 and fp32 x)."""
    import block_quantized_expert_moe_b200 as bq
    wl, li = _layer(name, 2)
    _check(li, synth.tokens(wl, li.router, 2, 1, T), wl.top_k, path=bq.MOE_PATH_GROUPED)


@pytest.mark.parametrize("fmt", [synth.FMT_Q8_0, synth.FMT_Q5_1, synth.FMT_IQ4_NL, synth.FMT_NVFP4, synth.FMT_Q5_0])
def test_every_format_on_both_projections(fmt):
    wl = synth.Workload("fmt", 1024, 32, 256, 4, True, fmt, fmt, synth.DT_BF16, 13, seed=fmt)
    li = synth.layer_inputs(wl)
    _check(li, synth.tokens(wl, li.router), wl.top_k)


@pytest.mark.parametrize("fmt_gu,fmt_dn", [(synth.FMT_Q8_0, synth.FMT_Q8_0), (synth.FMT_Q5_1, synth.FMT_Q5_1),
                                           (synth.FMT_IQ4_NL, synth.FMT_IQ4_NL), (synth.FMT_NVFP4, synth.FMT_NVFP4),
                                           (synth.FMT_NVFP4, synth.FMT_Q5_1), (synth.FMT_IQ4_NL, synth.FMT_Q5_0)])
def test_single_token_streaming_kernel_every_format(fmt_gu, fmt_dn):
    """One token with whole-row bulk copies (hidden and inter multiples of 256):
    fewer experts than SMs, so many CTAs own no router row and a few pairs."""
    wl = synth.Workload("s1", 1024, 32, 256, 4, True, fmt_gu, fmt_dn, synth.DT_BF16, 1, seed=20 + fmt_gu)
    li = synth.layer_inputs(wl)
    for step in range(2):
        _check(li, synth.tokens(wl, li.router, 0, step), wl.top_k)


def test_single_token_streaming_kernel_sixteen_experts_no_shared():
    wl = synth.Workload("s1k16", 512, 64, 256, 16, False, synth.FMT_IQ4_NL, synth.FMT_Q8_0, synth.DT_F32, 1,
                        seed=31)
    li = synth.layer_inputs(wl)
    _check(li, synth.tokens(wl, li.router), 16)


def test_ragged_shapes_and_k_equals_E():
    # hidden 96 (3 units per row), inter 64, top_k = E, shared expert, 3 tokens
    wl = synth.Workload("ragged", 96, 5, 64, 5, True, synth.FMT_IQ4_NL, synth.FMT_Q5_1, synth.DT_F32, 3,
                        seed=4)
    li = synth.layer_inputs(wl)
    _check(li, synth.tokens(wl, li.router), 5)
    # hidden 1056 (33 units: one lane of 32 takes two), top_k = 1
    wl = synth.Workload("odd", 1056, 9, 96, 1, False, synth.FMT_Q8_0, synth.FMT_NVFP4, synth.DT_BF16, 17,
                        seed=5)
    li = synth.layer_inputs(wl)
    _check(li, synth.tokens(wl, li.router), 1)


def test_route_topk_bit_exact_sets_and_gates():
    import block_quantized_expert_moe_b200 as bq
    # fp32 x with 200 tokens stays on the CUDA-core router: 25 token blocks over 14 block groups
    for name, T in (("tiny_q8", 1), ("model_decode", 1), ("zipf_batch", 64), ("spec_verify", 8), ("tiny_q8", 200)):
        wl, li = _layer(name)
        x = synth.tokens(wl, li.router, 0, 0, T)
        xt, wr = to_device(x), router_to_device(li.router)
        idx = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
        gate = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
        ws = torch.empty(bq.moe_route_workspace_bytes(T, wl.n_experts), dtype=torch.uint8, device="cuda")
        bq.moe_route_topk(xt, wr, wl.top_k, idx, gate, ws)
        torch.cuda.synchronize()
        import oracle
        ridx, rgate, _ = oracle.route(synth.tokens_f64(wl, x), li.router, wl.top_k)
        assert np.array_equal(idx.cpu().numpy(), ridx)  # margin-guarded: order is unique too
        assert np.abs(gate.cpu().numpy() - rgate).max() <= 1e-5


def test_outputs_are_bitwise_reproducible():
    wl, li = _layer("zipf_batch")
    x = synth.tokens(wl, li.router)
    outs, _, _, _ = gpu_layer(li, x, wl.top_k, repeat=3)
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_fmt_argument_is_checked():
    import block_quantized_expert_moe_b200 as bq
    wl, li = _layer("tiny_q8")
    pack = bq.pack_layer(li, max_tokens=4)
    x = to_device(synth.tokens(wl, li.router))
    out = torch.empty(1, wl.hidden, device="cuda")
    with pytest.raises(bq.MoeError) as e:
        bq.moe_layer_forward(x, router_to_device(li.router), pack, bq.MOE_FMT_NVFP4, wl.top_k, out)
    assert e.value.status == bq.MOE_ERR_FMT_MISMATCH
    with pytest.raises(bq.MoeError) as e:  # more tokens than the pack was sized for
        bq.moe_layer_forward(torch.zeros(5, wl.hidden, device="cuda"), router_to_device(li.router), pack,
                             0, wl.top_k, torch.empty(5, wl.hidden, device="cuda"))
    assert e.value.status == bq.MOE_ERR_INVALID_ARG
    pack.free()


def test_empty_batch_is_a_no_op():
    """Zero tokens: every entry point returns MOE_OK, enqueues nothing and leaves the
    routing record of the previous forward in place."""
    import block_quantized_expert_moe_b200 as bq
    wl, li = _layer("tiny_q8")
    x = synth.tokens(wl, li.router, 0, 0, 3)
    pack = bq.pack_layer(li, max_tokens=8)
    wr = router_to_device(li.router)
    out = torch.empty(3, wl.hidden, device="cuda")
    bq.moe_layer_forward(to_device(x), wr, pack, bq.MOE_FMT_FROM_PACK, wl.top_k, out)
    before = bq.moe_read_routing(pack, 3, wl.top_k)
    empty_x = torch.empty(0, wl.hidden, device="cuda")
    empty_out = torch.empty(0, wl.hidden, device="cuda")
    for path in (bq.MOE_PATH_AUTO, bq.MOE_PATH_DECODE, bq.MOE_PATH_GROUPED):
        bq.moe_layer_forward_ex(empty_x, wr, pack, bq.MOE_FMT_FROM_PACK, wl.top_k, empty_out, path)
    idx = torch.empty(0, wl.top_k, dtype=torch.int32, device="cuda")
    gate = torch.empty(0, wl.top_k, dtype=torch.float32, device="cuda")
    ws = torch.empty(bq.moe_route_workspace_bytes(0, wl.n_experts), dtype=torch.uint8, device="cuda")
    bq.moe_route_topk(empty_x, wr, wl.top_k, idx, gate, ws)
    torch.cuda.synchronize()
    after = bq.moe_read_routing(pack, 3, wl.top_k)
    assert all(np.array_equal(a, b) for a, b in zip(before, after))
    assert bq.moe_get_device_error(pack) == bq.MOE_OK
    pack.free()


def test_pack_rejects_nan_block_scale():
    import block_quantized_expert_moe_b200 as bq
    wl = synth.Workload("nan", 64, 4, 32, 2, False, synth.FMT_NVFP4, synth.FMT_NVFP4, synth.DT_BF16, 1)
    li = synth.layer_inputs(wl)
    li.gate_up[1, 9 * 3] = 0x7F  # E4M3 NaN scale in expert 1
    with pytest.raises(bq.MoeError) as e:
        bq.pack_layer(li)
    assert e.value.status == bq.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("name,layer,T", [("tiny_q8", 3, 1), ("model_decode", 1, 1), ("spec_verify", 2, 8),
                                          ("model_decode", 4, 3)])
def test_fused_and_grouped_decode_paths_both_match_the_oracle(name, layer, T):
    import block_quantized_expert_moe_b200 as bq
    wl, li = _layer(name, layer)
    x = synth.tokens(wl, li.router, layer, 7, T)
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k)
    outs = {}
    for path in (bq.MOE_PATH_DECODE, bq.MOE_PATH_GROUPED):
        out, idx, gate, counts = gpu_layer(li, x, wl.top_k, path=path)
        assert_routing_equal(idx, gate, ridx, rgate)
        assert np.array_equal(counts, expected_counts(ridx, wl.n_experts, T, wl.has_shared))
        err = normwise_err(out, ref)
        assert err <= DECODE_TOL, (path, err)
        outs[path] = out
    # one token: the same fp32 arithmetic in a different order, close but not
    # necessarily bitwise; two or more: the decode path runs the tensor cores on
    # fp16 operands (weights and h rounded to 11 significant bits, 2^-12
    # relative each), the grouped path stays in fp32
    assert normwise_err(outs[bq.MOE_PATH_DECODE], outs[bq.MOE_PATH_GROUPED]) <= (1e-5 if T == 1 else 1e-3)


def test_fused_decode_ragged_shapes():
    for T in (1, 3, 5, 8):
        wl = synth.Workload("ragged_fused", 96, 7, 64, 3, True, synth.FMT_NVFP4, synth.FMT_Q5_1, synth.DT_BF16,
                            T, seed=10 + T)
        li = synth.layer_inputs(wl)
        _check(li, synth.tokens(wl, li.router), wl.top_k)


@pytest.mark.parametrize("name,T,kw", [("prefill_nvfp4", 300, {}),
                                       ("prefill_nvfp4", 130, dict(n_experts=200, hidden=96, top_k=5))])
def test_tensor_core_router_matches_oracle(name, T, kw):
    """More than 64 bf16 tokens: the router runs as a tcgen05 GEMM (ragged M, N and K tiles here)."""
    import block_quantized_expert_moe_b200 as bq
    import oracle
    wl = synth.WORKLOADS[name].with_(**kw)
    wr_np, _ = synth.router(wl)
    x = synth.tokens(wl, wr_np, 0, 0, T)
    xt, wr = to_device(x), router_to_device(wr_np)
    idx = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
    ws = torch.zeros(bq.moe_route_workspace_bytes(T, wl.n_experts), dtype=torch.uint8, device="cuda")
    bq.moe_route_topk(xt, wr, wl.top_k, idx, gate, ws)
    torch.cuda.synchronize()
    assert ws[4:8].view(torch.int32).item() == 0  # no timed-out wait
    ridx, rgate, rlog = oracle.route(synth.tokens_f64(wl, x), wr_np, wl.top_k)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.abs(gate.cpu().numpy() - rgate).max() <= 1e-5
    logits = ws[256:256 + 4 * T * wl.n_experts].view(torch.float32).view(T, wl.n_experts).cpu().numpy()
    assert np.abs(logits - rlog).max() <= 1e-4 * np.abs(rlog).max()


@pytest.mark.parametrize("name,T", [("zipf_batch", 64), ("model_decode", 5)])
def test_dense_batched_variant_matches_oracle(name, T):
    """Every active expert multiplies the whole batch (zero gates where not routed)."""
    import block_quantized_expert_moe_b200 as bq
    wl, li = _layer(name, 1)
    x = synth.tokens(wl, li.router, 1, 3, T)
    out, idx, gate, counts = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_DENSE, flags=bq.MOE_PACK_DENSE)
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k)
    assert_routing_equal(idx, gate, ridx, rgate)
    assert normwise_err(out, ref) <= DECODE_TOL


def test_grouped_cuda_core_path_when_weights_are_not_fp16_normal():
    """Block scales below 2^-14 make some weights fp16 subnormals: the pack turns
    the tensor-core decode off and 2-64 tokens run the CUDA-core grouped kernels."""
    wl = synth.Workload("tiny_scales", 2048, 64, 512, 8, True, synth.FMT_Q8_0, synth.FMT_Q8_0, synth.DT_BF16, 8,
                        sigma_w=3e-4, seed=21)
    li = synth.layer_inputs(wl)
    _check(li, synth.tokens(wl, li.router), wl.top_k)


def test_tensor_core_decode_reports_h_outside_fp16_range():
    """Weights large enough that h = silu(G x) (U x) passes 65,504: the tensor-core
    decode records MOE_ERR_RANGE; the fp32 grouped path computes the layer."""
    import block_quantized_expert_moe_b200 as bq
    wl = synth.Workload("big_h", 1024, 32, 256, 4, True, synth.FMT_Q8_0, synth.FMT_Q8_0, synth.DT_BF16, 8,
                        sigma_w=1000.0, seed=22)
    li = synth.layer_inputs(wl)
    x = synth.tokens(wl, li.router)
    pack = bq.pack_layer(li, max_tokens=8, max_top_k=wl.top_k)
    out = torch.zeros(8, wl.hidden, device="cuda")
    bq.moe_layer_forward(to_device(x), router_to_device(li.router), pack, bq.MOE_FMT_FROM_PACK, wl.top_k, out)
    torch.cuda.synchronize()
    assert bq.moe_get_device_error(pack) == bq.MOE_ERR_RANGE
    pack.free()
    out_g, idx, gate, _ = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_GROUPED)
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k)
    assert_routing_equal(idx, gate, ridx, rgate)
    assert normwise_err(out_g, ref) <= DECODE_TOL


def test_tensor_core_decode_with_fp32_tokens():
    """fp32 x (rounded to fp16 in the gather, 2^-12 relative) through the tensor-core decode."""
    wl, li = _layer("tiny_q8")
    x = synth.tokens(wl, li.router, 0, 0, 6)
    _check(li, x, wl.top_k)


def test_tensor_core_decode_sixty_four_identical_tokens():
    """The largest group the tensor-core decode takes: 64 copies of one token send all 64
    to the same k experts (N = 64 per tile).  Tokens are independent, so every output row
    must equal the first, bit for bit, and match the oracle."""
    wl, li = _layer("model_decode", layer=1)
    x = np.repeat(synth.tokens(wl, li.router, 1, 0, 1), 64, axis=0)
    out, idx, gate, counts = gpu_layer(li, x, wl.top_k)
    ref, ridx, rgate = oracle_layer(li, x[:1], wl.top_k)
    assert_routing_equal(idx[:1], gate[:1], ridx, rgate)
    assert (idx == idx[0]).all() and (gate == gate[0]).all()
    assert np.array_equal(counts, expected_counts(np.repeat(ridx, 64, axis=0), wl.n_experts, 64, wl.has_shared))
    assert (out == out[0]).all()
    assert normwise_err(out[:1], ref) <= DECODE_TOL
