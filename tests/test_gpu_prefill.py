"""Tensor-core prefill (NVFP4 block-scaled tcgen05 GEMMs) vs the fp64 oracle.

The prefill quantises activations to NVFP4 with a per-token scale (x before
gate/up, h before down), so the reference is the oracle's act_quant = 1 mode;
the tolerance is the 2e-2 of tensor-core prefill.  Routing (tensor-core
router GEMM) must still select exactly the oracle's experts.
"""
import numpy as np
import pytest

import synth
from harness import (PREFILL_TOL, assert_routing_equal, expected_counts, gpu_layer, normwise_err,
                     oracle_layer)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _run(wl, T, layer=0, sample=None):
    import block_quantized_expert_moe_b200 as bq
    li = synth.layer_inputs(wl, layer)
    x = synth.tokens(wl, li.router, layer, 0, T)
    out, idx, gate, counts = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_PREFILL)
    tok = np.arange(T) if sample is None else np.asarray(sample)
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k, tokens=tok, act_quant=1)
    assert_routing_equal(idx[tok], gate[tok], ridx, rgate)
    if sample is None:
        assert np.array_equal(counts, expected_counts(ridx, wl.n_experts, T, wl.has_shared))
    err = normwise_err(out[tok], ref)
    assert err <= PREFILL_TOL, err
    return li, x, out, err


def test_prefill_nvfp4_ragged_batch():
    wl = synth.WORKLOADS["prefill_nvfp4"]
    li, x, out, err = _run(wl, 300)
    # the exact (unquantised-activation) layer differs by the NVFP4 rounding of x and h
    exact, _, _ = oracle_layer(li, x, wl.top_k)
    print(f"prefill NVFP4 T=300: err vs act-quant oracle {err:.2e}, vs exact oracle {normwise_err(out, exact):.2e}")


def test_prefill_nvfp4_with_shared_expert():
    wl = synth.WORKLOADS["prefill_nvfp4"].with_(has_shared=True, zipf_s=0.0, tokens=130)
    _run(wl, 130, layer=3)


def test_prefill_matches_grouped_decode_path():
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS["prefill_nvfp4"]
    li = synth.layer_inputs(wl, 1)
    x = synth.tokens(wl, li.router, 1, 0, 200)
    pf, idx_p, _, _ = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_PREFILL)
    gr, idx_g, _, _ = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_GROUPED)
    assert all(sorted(a) == sorted(b) for a, b in zip(idx_p.tolist(), idx_g.tolist()))
    # the grouped decode path keeps x and h in fp32; the prefill rounds both to
    # NVFP4 (E2M1 codes, one E4M3 scale per 16): measured ~0.25 normwise on B200
    assert normwise_err(pf, gr) <= 0.4


def test_prefill_full_chunk_sampled():
    """The full 8192-token chunk in the launch configuration the benchmark uses; the
    oracle checks 24 sampled tokens (tokens are independent)."""
    wl = synth.WORKLOADS["prefill_nvfp4"]
    rng = np.random.default_rng(0)
    sample = np.sort(rng.choice(8192, 24, replace=False))
    _run(wl, 8192, sample=sample)


def _run_q8(T, sample=None, layer=0):
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS["prefill_q8"]
    li = synth.layer_inputs(wl, layer)
    x = synth.tokens(wl, li.router, layer, 0, T)
    out, idx, gate, counts = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_PREFILL)
    tok = np.arange(T) if sample is None else np.asarray(sample)
    # weights and h are rounded to bf16 for the tensor cores; the oracle stays exact
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k, tokens=tok)
    assert_routing_equal(idx[tok], gate[tok], ridx, rgate)
    err = normwise_err(out[tok], ref)
    assert err <= PREFILL_TOL, err
    return err


def test_prefill_q8_bf16_dequant_ragged_batch():
    err = _run_q8(300)
    print(f"prefill Q8_0 -> bf16 T=300: err vs exact oracle {err:.2e}")


def test_prefill_q8_full_chunk_sampled():
    rng = np.random.default_rng(1)
    _run_q8(8192, sample=np.sort(rng.choice(8192, 16, replace=False)))


def _run_dq(wl, T, layer=0, sample=None):
    import block_quantized_expert_moe_b200 as bq
    li = synth.layer_inputs(wl, layer)
    x = synth.tokens(wl, li.router, layer, 0, T)
    out, idx, gate, counts = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_PREFILL)
    tok = np.arange(T) if sample is None else np.asarray(sample)
    # weights and h are rounded to bf16 for the tensor cores; the oracle stays exact
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k, tokens=tok)
    assert_routing_equal(idx[tok], gate[tok], ridx, rgate)
    if sample is None:
        assert np.array_equal(counts, expected_counts(ridx, wl.n_experts, T, wl.has_shared))
    err = normwise_err(out[tok], ref)
    assert err <= PREFILL_TOL, err
    return err


def test_prefill_iq4nl_q51_dequant_ragged_batch():
    """The model-shaped layer's formats through the bf16-dequantising tensor-core path (shared expert)."""
    err = _run_dq(synth.WORKLOADS["prefill_iq4nl_q51"], 300)
    print(f"prefill IQ4_NL/Q5_1 -> bf16 T=300: err vs exact oracle {err:.2e}")


def test_prefill_mixed_formats_small_shapes():
    # Q5_1 gate/up with an IQ4_NL down projection, and Q8_0 with Q5_1: 4-bit and 8-bit dequantisers
    # Q5_0 runs through the Q5_1 planes (m = -16 d)
    for gu, dn, seed in ((synth.FMT_Q5_1, synth.FMT_IQ4_NL, 41), (synth.FMT_Q8_0, synth.FMT_Q5_1, 42),
                         (synth.FMT_Q5_0, synth.FMT_IQ4_NL, 43)):
        wl = synth.Workload("mixed", 1024, 48, 256, 6, True, gu, dn, synth.DT_BF16, 200, zipf_s=1.1, seed=seed)
        _run_dq(wl, 200)


def test_prefill_iq4nl_q51_full_chunk_sampled():
    rng = np.random.default_rng(2)
    _run_dq(synth.WORKLOADS["prefill_iq4nl_q51"], 8192, sample=np.sort(rng.choice(8192, 16, replace=False)))



def test_prefill_nvfp4_through_bf16_dequant_against_the_exact_oracle():
    """NVFP4 weights dequantised to bf16 in shared memory (exact), x left in bf16, bf16
    MMA: the variant of the NVFP4 prefill that the exact oracle (no activation
    quantisation) checks, beside the native FP4 GEMM that rounds x and h to NVFP4."""
    import block_quantized_expert_moe_b200 as bq
    wl = synth.WORKLOADS["prefill_nvfp4"]
    li = synth.layer_inputs(wl, 2)
    x = synth.tokens(wl, li.router, 2, 0, 300)
    out, idx, gate, counts = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_PREFILL_BF16)
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k)
    assert_routing_equal(idx, gate, ridx, rgate)
    assert np.array_equal(counts, expected_counts(ridx, wl.n_experts, 300, wl.has_shared))
    err = normwise_err(out, ref)
    assert err <= PREFILL_TOL, err
    print(f"prefill NVFP4 -> bf16 T=300: err vs exact oracle {err:.2e}")
    # the full 8192-token chunk, 16 sampled tokens
    x = synth.tokens(wl, li.router, 2, 0, 8192)
    out, idx, gate, _ = gpu_layer(li, x, wl.top_k, path=bq.MOE_PATH_PREFILL_BF16)
    tok = np.sort(np.random.default_rng(3).choice(8192, 16, replace=False))
    ref, ridx, rgate = oracle_layer(li, x, wl.top_k, tokens=tok)
    assert_routing_equal(idx[tok], gate[tok], ridx, rgate)
    assert normwise_err(out[tok], ref) <= PREFILL_TOL
