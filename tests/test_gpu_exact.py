"""Bitwise sub-step pins: every CUDA path against the fp64 oracle on layers whose
every intermediate is exact (tests/exact_layers.py).

Integer tokens, integer-or-dyadic weights with power-of-two block scales, gate
pre-activations >= 40 (SiLU is the identity there in fp32 and fp64) and top-1
routing (gate exactly 1): the matvec sums are exact in any order, so the layer
output of each kernel must equal the oracle's bit for bit.  A dropped or
doubled block, a wrong scale, a misplaced fifth bit or a table lookup that
picks the wrong entry changes the output by at least one unit and fails here,
where the 2e-3 tolerance of the ordinary parity tests could let it pass.  The
IQ4_NL table of these layers makes the decode kernels use their masked lookup
(no bias splits its entries evenly); the pack reports that mode.
"""
import numpy as np
import pytest

import synth
from exact_layers import assert_exact_bounds, exact_layer, exact_tokens
from harness import gpu_layer, oracle_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

PAIRS = [(synth.FMT_Q8_0, synth.FMT_Q8_0), (synth.FMT_IQ4_NL, synth.FMT_Q5_1), (synth.FMT_NVFP4, synth.FMT_NVFP4),
         (synth.FMT_Q5_0, synth.FMT_IQ4_NL), (synth.FMT_Q5_1, synth.FMT_Q8_0), (synth.FMT_IQ4_NL, synth.FMT_IQ4_NL)]


def _bitwise(li, x, path=None, max_tokens=None, h_max=2048):
    assert_exact_bounds(li, x, h_max)
    ref, ridx, rgate = oracle_layer(li, x, 1)
    import block_quantized_expert_moe_b200 as bq
    pack = bq.pack_layer(li, max_tokens=max_tokens or max(x.shape[0], 1), max_top_k=1)
    try:
        out, idx, gate, _ = gpu_layer(li, x, 1, path=path, pack=pack)
        info = pack.info()
    finally:
        pack.free()
    assert np.array_equal(idx, ridx) and (gate == 1.0).all()
    bad = np.argwhere(out != ref)
    assert bad.size == 0, (len(bad), bad[:4].tolist(), out[tuple(bad[0])], ref[tuple(bad[0])])
    return info


@pytest.mark.parametrize("fmt_gu,fmt_dn", PAIRS)
@pytest.mark.parametrize("T", [1, 5, 64])
def test_decode_default_path_is_bitwise_exact(fmt_gu, fmt_dn, T):
    """One token: the single-token streaming kernel; 2-64: the one-launch tail."""
    li = exact_layer(fmt_gu, fmt_dn, seed=10 * fmt_gu + fmt_dn)
    info = _bitwise(li, exact_tokens(li, T, seed=T))
    if synth.FMT_IQ4_NL in (fmt_gu, fmt_dn):
        assert info["code_table_masked"] == ((fmt_gu == synth.FMT_IQ4_NL) | 2 * (fmt_dn == synth.FMT_IQ4_NL))


@pytest.mark.parametrize("fmt_gu,fmt_dn", PAIRS)
@pytest.mark.parametrize("T,path", [(1, "tail"), (13, "tail"), (3, "staged"), (40, "staged")])
def test_tail_and_staged_tensor_core_decode_are_bitwise_exact(fmt_gu, fmt_dn, T, path):
    """The one-launch tail also at one token, and the same tensor-core work as
    separate launches (route and plan, x gather, gate/up, down, combine)."""
    import block_quantized_expert_moe_b200 as bq
    li = exact_layer(fmt_gu, fmt_dn, seed=10 * fmt_gu + fmt_dn + 3)
    p = {"tail": bq.MOE_PATH_TAIL, "staged": bq.MOE_PATH_DECODE_STAGED}[path]
    _bitwise(li, exact_tokens(li, T, seed=T + 100), path=p)


def test_tail_on_many_experts_and_every_sm_partition():
    """64 experts, top-1, 64 tokens: about 60 groups, so the units of a tile meet
    ranges of several CTAs and most tiles are summed from pieces; then 3 tokens,
    where fewer units than SMs leave some CTAs without work."""
    import block_quantized_expert_moe_b200 as bq
    li = exact_layer(synth.FMT_IQ4_NL, synth.FMT_Q5_1, n_experts=64, seed=77)
    for T in (64, 3):
        _bitwise(li, exact_tokens(li, T, seed=T + 7), path=bq.MOE_PATH_TAIL, max_tokens=64)


@pytest.mark.parametrize("fmt_gu,fmt_dn", PAIRS)
def test_grouped_cuda_core_path_is_bitwise_exact(fmt_gu, fmt_dn):
    import block_quantized_expert_moe_b200 as bq
    li = exact_layer(fmt_gu, fmt_dn, seed=10 * fmt_gu + fmt_dn + 1)
    for T in (1, 7):
        _bitwise(li, exact_tokens(li, T, seed=T), path=bq.MOE_PATH_GROUPED)


@pytest.mark.parametrize("fmt_gu,fmt_dn", [p for p in PAIRS if p[0] != synth.FMT_NVFP4])
def test_streamed_grouped_fallback_is_bitwise_exact(fmt_gu, fmt_dn):
    """An extra expert outside the fp16 range turns the tensor-core decode off: 2-64
    tokens take the TMA-fed CUDA-core grouped kernels."""
    li = exact_layer(fmt_gu, fmt_dn, fp16_fallback=True, seed=10 * fmt_gu + fmt_dn + 2)
    for T in (3, 8, 20):
        _bitwise(li, exact_tokens(li, T, seed=T))


def test_fp32_tokens_and_no_shared_expert_are_bitwise_exact():
    li = exact_layer(synth.FMT_Q8_0, synth.FMT_IQ4_NL, has_shared=False, x_dtype=synth.DT_F32, seed=3)
    for T in (1, 4, 33):
        _bitwise(li, exact_tokens(li, T, seed=T))


def test_small_ragged_shapes_are_bitwise_exact():
    """hidden 96 and inter 64 (no whole-row bulk copies, no 256-row tiles): the fused
    cooperative kernel and the plain grouped matvecs."""
    import block_quantized_expert_moe_b200 as bq
    for fmt_gu, fmt_dn in ((synth.FMT_IQ4_NL, synth.FMT_Q5_1), (synth.FMT_NVFP4, synth.FMT_Q8_0)):
        li = exact_layer(fmt_gu, fmt_dn, hidden=96, inter=64, n_experts=5, n_gate=48, seed=7 + fmt_gu)
        for T in (1, 6):
            _bitwise(li, exact_tokens(li, T, seed=T))
            _bitwise(li, exact_tokens(li, T, seed=T), path=bq.MOE_PATH_GROUPED)


@pytest.mark.parametrize("fmt_gu,fmt_dn", [(synth.FMT_Q8_0, synth.FMT_Q8_0), (synth.FMT_IQ4_NL, synth.FMT_Q5_1),
                                           (synth.FMT_Q5_1, synth.FMT_IQ4_NL), (synth.FMT_NVFP4, synth.FMT_NVFP4),
                                           (synth.FMT_NVFP4, synth.FMT_Q5_1)])
def test_bf16_dequant_prefill_is_bitwise_exact(fmt_gu, fmt_dn):
    """More than 64 tokens: the bf16-dequantising tensor-core prefill (NVFP4 included:
    its weights are exact in bf16).  bf16 keeps 8 significant bits, so h stays below
    256 here (one +-1 per up row)."""
    import block_quantized_expert_moe_b200 as bq
    li = exact_layer(fmt_gu, fmt_dn, n_gate=40, n_up=1, seed=10 * fmt_gu + fmt_dn + 5)
    x = exact_tokens(li, 200, seed=11)
    _bitwise(li, x, path=bq.MOE_PATH_PREFILL_BF16, h_max=256)
