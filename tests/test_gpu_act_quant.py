"""The NVFP4 prefill's activation quantisers on the GPU against the oracle's
act_quant mode, bit for bit.

Block-scaled FP4 MMA needs both operands in NVFP4, so the tensor-core prefill
rounds x (before gate/up) and h (before down) per token: scale s = amax/(6*448)
in fp32, E4M3 block scales and E2M1 codes, each rounded to nearest even and
saturating.  The layer tests see this only through the 2e-2 prefill tolerance;
here the quantisers run alone (moe_debug_act_quant_nvfp4) and every value
s * e4m3(scale) * e2m1(code) must equal the oracle's (an exact product in
fp64), including ties of both rounding steps, subnormal and zero block scales
and the saturating block that holds the row maximum.
"""
import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

E2M1_TIES = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0]  # in units of the block's step; ties to even


def crafted_row(cols, rng):
    """One row with s = 2^-10 (amax 2.625 = 2688 * 2^-10): blocks of E2M1 ties, an E4M3
    tie (1.0625 and 1.1875 of 6s), a subnormal block scale (2^-8), a subnormal tie
    (1.5 * 2^-9), a scale below the smallest subnormal (rounds to 0), a zero block and
    the saturating block (448); the rest small random values.  Every value is exact
    in bf16."""
    s = 2.0 ** -10
    v = np.round(rng.standard_normal(cols) * 64) / 64 * 0.01
    blocks = []
    sb = 8.0  # block scale 8: step s * 8 = 2^-7
    blocks.append(np.array([sg * t * s * sb for t in E2M1_TIES for sg in (1, -1)]))
    for r in (1.0625, 1.1875):  # E4M3 ties: block max = r * 6 s
        b = np.zeros(16)
        b[3] = r * 6 * s
        b[7] = -0.5 * r * 6 * s
        blocks.append(b)
    for r in (2.0 ** -8, 1.5 * 2.0 ** -9, 2.0 ** -11):  # subnormal, subnormal tie, below the smallest
        b = np.zeros(16)
        b[0] = r * 6 * s
        b[9] = -r * 3 * s
        blocks.append(b)
    blocks.append(np.zeros(16))
    b = rng.uniform(-2.6, 2.6, 16)
    b[5] = 2.625  # the row maximum: block scale 448
    blocks.append(b)
    for i, b in enumerate(blocks):
        v[16 * (2 * i + 1):16 * (2 * i + 2)] = b
    return v


def gpu_values(x):
    import block_quantized_expert_moe_b200 as bq
    codes, scales, row_scale = bq.moe_debug_act_quant_nvfp4(x)
    torch.cuda.synchronize()
    codes, scales, row_scale = codes.cpu().numpy(), scales.cpu().numpy(), row_scale.cpu().numpy()
    e2m1 = np.array([oracle.e2m1(c) for c in range(16)])
    e4m3 = np.array([oracle.e4m3(c) for c in range(256)])
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[0], -1)
    sb = np.repeat(e4m3[scales], 16, axis=1)
    return row_scale.astype(np.float64)[:, None] * sb * e2m1[nib], row_scale


def oracle_values(rows):
    return np.stack([oracle.act_quant_nvfp4(r) for r in rows])


@pytest.mark.parametrize("cols", [2048, 512])
def test_quantisers_match_the_oracle_bitwise(cols):
    rng = np.random.default_rng(cols)
    rand = rng.standard_normal((40, cols)) * rng.choice([1e-3, 1.0, 30.0], (40, 1))
    rows = np.concatenate([np.stack([crafted_row(cols, rng) for _ in range(3)]), rand, np.zeros((1, cols))])
    rows_bf16 = synth.bf16_to_f32(synth.bf16_bits(rows)).astype(np.float64)  # exact bf16 values
    ref = oracle_values(rows_bf16)
    xb = torch.from_numpy(synth.bf16_bits(rows_bf16).view(np.int16)).cuda().view(torch.bfloat16)
    xf = torch.from_numpy(rows_bf16.astype(np.float32)).cuda()
    for x in (xb, xf):  # the gate/up activations' quantiser, then the down activations'
        got, row_scale = gpu_values(x)
        amax = np.abs(rows_bf16).max(1).astype(np.float32)
        assert np.array_equal(row_scale, amax / np.float32(6 * 448))
        bad = np.argwhere(got != ref)
        assert bad.size == 0, (x.dtype, len(bad), bad[:4].tolist())
    # the crafted rows reach every case they were built for
    q = ref[0] / 2.0 ** -10
    assert q[16:32].tolist() == [sg * t * 8 for t in (0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0) for sg in (1, -1)]
