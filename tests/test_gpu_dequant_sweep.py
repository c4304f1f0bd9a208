"""Device block decoders against the oracle's decoders, weight by weight.

Each format's blocks are filled with every code and a sweep of block scales
(every finite fp16 exponent, subnormals and zero included; Q5_1 also a sweep of
offsets m; NVFP4 every positive E4M3 byte), packed as a layer, and decoded on
the device from the pack's own planes by moe_debug_dequant_rows:

  kind 0  the tensor-core decode's fp16 expansion, one rounding of each weight:
          equal to the fp16 round-to-nearest-even of the oracle's exact value
          (overflow to infinity included)
  kind 1  the bf16-dequantising prefill's fp32 values before their bf16
          rounding: equal to the fp32 rounding of the oracle's exact value

bit for bit.  The block layouts and the values they encode are those of the
Unsloth dynamic-quantisation page ("Quantization types") and the UD-IQ2_XS
model card ("What was changed"); NVFP4 comes out as 2 x E2M1 x E4M3 (the
kernels apply the halving and the matrix scale in their epilogues).
"""
import numpy as np
import pytest

import oracle
import synth
from exact_layers import EXACT_IQ4NL_TABLE

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

H, I, E = 512, 256, 2


def _f16_sweep(rng, n, max_exp_field=30):
    """fp16 bit patterns: every exponent field 0 .. max_exp_field (0: zero and
    subnormals), random mantissas and signs, plus the edge values in range."""
    exp = rng.integers(0, max_exp_field + 1, n)
    bits = (exp << 10) | rng.integers(0, 1024, n) | (rng.integers(0, 2, n) << 15)
    edges = [0x0000, 0x8000, 0x0001, 0x03FF, 0x0400, 0x3C00, 0xBC00, 0x7BFF, 0xFBFF, 0x3555]
    edges = [e for e in edges if (e >> 10) & 31 <= max_exp_field]
    bits[:len(edges)] = edges
    return bits.astype(np.uint16)


def _encode(fmt, rng, rows, K):
    """Canonical blocks (uint8 [rows, row_bytes]) with random codes (every code
    appears) and swept scales."""
    if fmt == synth.FMT_NVFP4:
        nb = K // 16
        sc = rng.integers(0, 0x7F, (rows, nb)).astype(np.uint8)  # positive E4M3, NaN excluded
        sc.flat[:0x7F] = np.arange(0x7F, dtype=np.uint8)           # every byte at least once
        codes = rng.integers(0, 16, (rows, nb, 16))
        packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
        return np.concatenate([sc[..., None], packed], axis=2).reshape(rows, -1)
    nb = K // 32
    # Q5_0 is packed with m = -16 d, which must stay finite in fp16: |d| < 2048
    d = _f16_sweep(rng, rows * nb, 25 if fmt == synth.FMT_Q5_0 else 30).reshape(rows, nb)
    d_bytes = d.view(np.uint8).reshape(rows, nb, 2)
    if fmt == synth.FMT_Q8_0:
        q = rng.integers(-128, 128, (rows, nb, 32)).astype(np.int8)
        return np.concatenate([d_bytes, q.view(np.uint8)], axis=2).reshape(rows, -1)
    if fmt == synth.FMT_IQ4_NL:
        idx = rng.integers(0, 16, (rows, nb, 32))
        qs = (idx[..., :16] | (idx[..., 16:] << 4)).astype(np.uint8)
        return np.concatenate([d_bytes, qs], axis=2).reshape(rows, -1)
    q = rng.integers(0, 32, (rows, nb, 32))
    qh = ((q >> 4) & 1).astype(np.uint64) << np.arange(32, dtype=np.uint64)
    qh = qh.sum(axis=2).astype(np.uint32).view(np.uint8).reshape(rows, nb, 4)
    qs = ((q[..., :16] & 15) | ((q[..., 16:] & 15) << 4)).astype(np.uint8)
    parts = [d_bytes]
    if fmt == synth.FMT_Q5_1:
        parts.append(_f16_sweep(rng, rows * nb).reshape(rows, nb).view(np.uint8).reshape(rows, nb, 2))
    return np.concatenate(parts + [qh, qs], axis=2).reshape(rows, -1)


def _layer(fmt, table, seed):
    rng = np.random.default_rng(seed)
    wl = synth.Workload("sweep", H, E, I, 1, False, fmt, fmt, synth.DT_BF16, 1, seed=seed)
    gu = np.stack([_encode(fmt, rng, 2 * I, H).ravel() for _ in range(E)])
    dn = np.stack([_encode(fmt, rng, H, I).ravel() for _ in range(E)])
    assert gu.shape[1] == 2 * I * oracle.lib().oracle_row_bytes(fmt, H)
    assert dn.shape[1] == H * oracle.lib().oracle_row_bytes(fmt, I)
    ts = np.ones(E, np.float32) if fmt == synth.FMT_NVFP4 else None
    router = np.zeros((E, H), np.uint16)
    return synth.LayerInputs(wl, 0, router, gu, dn, ts, None if ts is None else ts.copy(), table, None)


def _expected(fmt, blocks, rows, cols, table):
    ref = oracle.decode_matrix(fmt, blocks, rows, cols, table, 1.0)
    return 2.0 * ref if fmt == synth.FMT_NVFP4 else ref


CASES = [(synth.FMT_Q8_0, None), (synth.FMT_Q5_1, None), (synth.FMT_Q5_0, None),
         (synth.FMT_IQ4_NL, synth.IQ4NL_TABLE), (synth.FMT_IQ4_NL, EXACT_IQ4NL_TABLE), (synth.FMT_NVFP4, None)]


@pytest.mark.parametrize("fmt,table", CASES, ids=["q8_0", "q5_1", "q5_0", "iq4nl_xor", "iq4nl_masked", "nvfp4"])
def test_device_decoders_match_the_oracle_bitwise(fmt, table):
    import block_quantized_expert_moe_b200 as bq
    li = _layer(fmt, None if table is None else np.asarray(table, np.int8), seed=100 + fmt)
    pack = bq.pack_layer(li, max_tokens=8, max_top_k=1)
    try:
        if table is not None:
            masked = table is EXACT_IQ4NL_TABLE
            assert pack.info()["code_table_masked"] == (3 if masked else 0)
        for proj, blocks, rows, cols in ((0, li.gate_up, 2 * I, H), (1, li.down, H, I)):
            for slot in range(E):
                ref = _expected(fmt, blocks[slot], rows, cols, li.table)
                with np.errstate(over="ignore"):
                    ref16, ref32 = ref.astype(np.float16), ref.astype(np.float32)
                got16 = bq.moe_debug_dequant_rows(pack, proj, slot, 0, rows, 0, cols).cpu().numpy()
                got32 = bq.moe_debug_dequant_rows(pack, proj, slot, 0, rows, 1, cols).cpu().numpy()
                torch.cuda.synchronize()
                for got, want, what in ((got16.view(np.uint16), ref16.view(np.uint16), "fp16"),
                                        (got32.view(np.uint32), ref32.view(np.uint32), "fp32")):
                    # both zeros of E2M1 (codes 0 and 8) decode to +0 on the device: the
                    # sign of a zero weight is the one difference allowed
                    zero = (got.view(ref16.dtype if what == "fp16" else np.float32) == 0) & (ref == 0)
                    bad = np.argwhere((got != want) & ~zero)
                    assert bad.size == 0, (what, proj, slot, len(bad), bad[:3].tolist(),
                                           got.view(ref16.dtype if what == "fp16" else np.float32)[tuple(bad[0])],
                                           ref[tuple(bad[0])])
        assert bq.moe_get_device_error(pack) == bq.MOE_OK
    finally:
        pack.free()


def test_dequant_rows_checks_its_arguments():
    import block_quantized_expert_moe_b200 as bq
    li = _layer(synth.FMT_Q8_0, None, seed=7)
    pack = bq.pack_layer(li, max_tokens=8, max_top_k=1)
    try:
        out = torch.empty(4, H, dtype=torch.float32, device="cuda")
        for proj, slot, row0, n, kind in ((2, 0, 0, 1, 0), (0, E, 0, 1, 0), (0, 0, 2 * I - 1, 2, 0),
                                          (0, 0, 0, 0, 0), (0, 0, 0, 1, 2), (0, -1, 0, 1, 1)):
            st = bq.lib.moe_debug_dequant_rows(pack.handle, proj, slot, row0, n, kind, out.data_ptr(), None)
            assert st == bq.MOE_ERR_INVALID_ARG, (proj, slot, row0, n, kind)
    finally:
        pack.free()
