"""Pins of the fp64 oracle against facts fixed outside it: closed-form block
decodes, library conversions (numpy fp16, torch fp8), brute force on tiny
inputs, and identities of the layer (dense sum, permutation, k = 1, linearity).
CPU only."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].strip()
        if line:
            rows.append(line.split())
    return rows


# ---------------------------------------------------------------- scalars


def test_fp16_all_codes_match_numpy():
    codes = np.arange(65536, dtype=np.uint16)
    ref = codes.view(np.float16).astype(np.float64)
    got = np.array([oracle.fp16(c) for c in codes])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_bf16_all_codes_match_float32_upper_half():
    codes = np.arange(65536, dtype=np.uint32)
    ref = (codes << 16).view(np.float32).astype(np.float64)
    got = np.array([oracle.bf16(int(c)) for c in codes])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])


def test_e4m3_all_codes_match_torch_and_closed_form():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])
    for c in range(127):  # closed form of the non-negative finite codes
        e, m = c >> 3, c & 7
        want = m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        assert oracle.e4m3(c) == want
    for kind, code, val in _golden("e2m1_e4m3.txt"):
        if kind == "e4m3":
            assert oracle.e4m3(int(code, 16)) == float(val)


def test_e2m1_all_codes():
    table = {int(c): float(v) for k, c, v in _golden("e2m1_e4m3.txt") if k == "e2m1"}
    for c in range(16):
        mag = table[c & 7]
        assert oracle.e2m1(c) == (-mag if c & 8 else mag)
        assert math.copysign(1.0, oracle.e2m1(c)) == (-1.0 if c & 8 else 1.0)


# ---------------------------------------------------------------- blocks


def _q8_block(d_bits, q):
    return np.concatenate([np.array([d_bits & 255, d_bits >> 8], np.uint8),
                           np.asarray(q, np.int8).view(np.uint8)])


def test_q8_0_closed_form():
    q = np.arange(-128, 128, dtype=np.int64)
    for d_bits, d in ((0x3C00, 1.0), (0x0400, 2.0 ** -14), (0x0001, 2.0 ** -24), (0xC000, -2.0)):
        row = np.concatenate([_q8_block(d_bits, q[i:i + 32]) for i in range(0, 256, 32)])
        assert row.size == 8 * 34
        got = oracle.decode_row(oracle.Q8_0, row, 256)
        assert np.array_equal(got, d * q.astype(np.float64))


def _q5_1_block(d_bits, m_bits, q):
    q = np.asarray(q)
    qs = np.zeros(16, np.uint8)
    qh = 0
    for j in range(32):
        lo = int(q[j]) & 15
        if j < 16:
            qs[j] |= lo
        else:
            qs[j - 16] |= lo << 4
        qh |= ((int(q[j]) >> 4) & 1) << j
    head = [d_bits & 255, d_bits >> 8, m_bits & 255, m_bits >> 8,
            qh & 255, (qh >> 8) & 255, (qh >> 16) & 255, (qh >> 24) & 255]
    return np.concatenate([np.array(head, np.uint8), qs])


def test_q5_1_closed_form_and_high_bit_walk():
    q = np.arange(32)
    blk = _q5_1_block(0x3C00, 0xCC00, q)  # d = 1, m = -16
    assert blk.size == 24
    assert np.array_equal(oracle.decode_row(oracle.Q5_1, blk, 32), q - 16.0)
    for j in range(32):  # one high bit at a time: only element j reaches 16 + low bits
        qj = np.zeros(32, np.int64)
        qj[j] = 16 + (j % 16)
        got = oracle.decode_row(oracle.Q5_1, _q5_1_block(0x3C00, 0x0000, qj), 32)
        want = np.zeros(32)
        want[j] = 16 + (j % 16)
        assert np.array_equal(got, want), j


def _q5_0_block(d_bits, q):
    # the Q5_1 block without m: d, qh, qs
    b = _q5_1_block(d_bits, 0, q)
    return np.concatenate([b[:2], b[4:]])


def test_q5_0_closed_form_high_bit_walk_and_negative_scale():
    q = np.arange(32)
    blk = _q5_0_block(0x3C00, q)  # d = 1
    assert blk.size == 22
    assert np.array_equal(oracle.decode_row(oracle.Q5_0, blk, 32), q - 16.0)
    # d = -0.5: the code is centred, then scaled (sign included)
    assert np.array_equal(oracle.decode_row(oracle.Q5_0, _q5_0_block(0xB800, q), 32), -0.5 * (q - 16.0))
    for j in range(32):  # one fifth bit at a time: only element j leaves -16 + low bits
        qj = np.zeros(32, np.int64)
        qj[j] = 16 + (j % 16)
        got = oracle.decode_row(oracle.Q5_0, _q5_0_block(0x3C00, qj), 32)
        want = np.full(32, -16.0)
        want[j] = j % 16
        assert np.array_equal(got, want), j


def test_q5_0_equals_q5_1_with_m_minus_16d():
    # the identity the pack uses to serve Q5_0 through the Q5_1 planes
    rng = np.random.default_rng(3)
    for d_bits, m_bits in ((0x3C00, 0xCC00), (0x2E66, 0xBE66), (0x0401, 0x9401)):  # d, -16 d exactly
        q = rng.integers(0, 32, 32)
        a = oracle.decode_row(oracle.Q5_0, _q5_0_block(d_bits, q), 32)
        b = oracle.decode_row(oracle.Q5_1, _q5_1_block(d_bits, m_bits, q), 32)
        assert np.array_equal(a, b), hex(d_bits)


def _iq4_block(d_bits, idx):
    qs = np.zeros(16, np.uint8)
    for j in range(32):
        if j < 16:
            qs[j] |= idx[j]
        else:
            qs[j - 16] |= idx[j] << 4
    return np.concatenate([np.array([d_bits & 255, d_bits >> 8], np.uint8), qs])


def test_iq4_nl_decodes_to_table():
    T = synth.IQ4NL_TABLE
    idx = np.concatenate([np.arange(16), np.arange(15, -1, -1)])
    want = T[idx].astype(np.float64)
    assert np.array_equal(oracle.decode_row(oracle.IQ4_NL, _iq4_block(0x3C00, idx), 32, T), want)
    assert np.array_equal(oracle.decode_row(oracle.IQ4_NL, _iq4_block(0xBC00, idx), 32, T), -want)
    odd = np.arange(16, dtype=np.int8) * 3 - 20  # a non-monotone table is decoded as given
    odd[[3, 9]] = odd[[9, 3]]
    assert np.array_equal(oracle.decode_row(oracle.IQ4_NL, _iq4_block(0x4000, idx), 32, odd),
                          2.0 * odd[idx])


def _nvfp4_block(sb, codes):
    b = np.zeros(9, np.uint8)
    b[0] = sb
    for i in range(8):
        b[1 + i] = codes[2 * i] | (codes[2 * i + 1] << 4)
    return b


def test_nvfp4_codes_and_scale_sweep():
    codes = np.arange(16)
    e2 = np.array([oracle.e2m1(c) for c in codes])
    got = oracle.decode_row(oracle.NVFP4, _nvfp4_block(0x38, codes), 16)
    assert np.array_equal(got, e2)
    assert np.array_equal(oracle.decode_row(oracle.NVFP4, _nvfp4_block(0x38, codes), 16,
                                            tensor_scale=0.375), 0.375 * e2)
    for sb in range(127):
        e, m = sb >> 3, sb & 7
        sv = m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        got = oracle.decode_row(oracle.NVFP4, _nvfp4_block(sb, np.full(16, 5)), 16, tensor_scale=2.0)
        assert np.all(got == 2.0 * sv * 3.0), sb


def test_sizes_match_pages():
    bpw = {f: float(v) for f, v in _golden("format_sizes.txt")}
    assert oracle.lib().oracle_row_bytes(oracle.IQ4_NL, 32) * 8 / 32 == bpw["IQ4_NL"]
    # Q5_0 (d + 32 five-bit values) is 22 B per 32; Q5_1 adds the fp16 m
    assert oracle.lib().oracle_row_bytes(oracle.Q5_0, 32) * 8 / 32 == bpw["Q5_0"]
    assert oracle.lib().oracle_row_bytes(oracle.Q5_1, 32) == oracle.lib().oracle_row_bytes(oracle.Q5_0, 32) + 2
    assert oracle.lib().oracle_row_bytes(oracle.Q8_0, 32) == 34
    assert oracle.lib().oracle_row_bytes(oracle.NVFP4, 16) * 8 / 16 == 4.5
    g = {k: float(v) for k, v in _golden("expert_bytes.txt")}
    per_expert_pages = g["gib"] * 2 ** 30 / g["experts"]
    ours = synth.WORKLOADS["model_decode"].expert_bytes()
    assert ours == 1_966_080
    assert abs(ours / per_expert_pages - 1) < 0.1


# ---------------------------------------------------------------- routing


def test_topk_matches_brute_force_sort():
    rng = np.random.default_rng(1)
    E, H, T, k = 37, 64, 20, 6
    wr = synth.bf16_bits(rng.normal(0, 0.1, (E, H)))
    x = synth.bf16_to_f32(synth.bf16_bits(rng.normal(0, 1, (T, H)))).astype(np.float64)
    idx, gate, logits = oracle.route(x, wr, k)
    wf = synth.bf16_to_f32(wr).astype(np.float64)
    for t in range(T):
        lt = [sum(float(wf[e, h]) * float(x[t, h]) for h in range(H)) for e in range(E)]
        order = sorted(range(E), key=lambda e: (-lt[e], e))[:k]
        assert list(idx[t]) == order
        ex = [math.exp(lt[e] - lt[order[0]]) for e in order]
        assert np.allclose(gate[t], [v / sum(ex) for v in ex], rtol=1e-12, atol=0)


def test_topk_ties_go_to_lower_index_and_two_gate_closed_form():
    H = 32
    wr = np.zeros((6, H), np.uint16)
    one = synth.bf16_bits(np.array([1.0]))[0]
    half = synth.bf16_bits(np.array([0.5]))[0]
    wr[1, 0] = one
    wr[4, 0] = one      # experts 1 and 4 tie at the top
    wr[2, 0] = half
    x = np.zeros((1, H))
    x[0, 0] = 2.0
    idx, gate, logits = oracle.route(x, wr, 3)
    assert list(idx[0]) == [1, 4, 2]
    e1 = math.exp(-1.0)
    assert np.allclose(gate[0], [1 / (2 + e1), 1 / (2 + e1), e1 / (2 + e1)], rtol=1e-15)
    idx, gate, _ = oracle.route(x, wr, 2)
    assert np.array_equal(gate[0], [0.5, 0.5])


# ---------------------------------------------------------------- experts / layer


def _tiny_q8_expert(rng, H, I, scale_exp=-7):
    """Float matrices exactly representable in Q8_0 with d = 2^scale_exp."""
    d = 2.0 ** scale_exp
    mats = [rng.integers(-127, 128, size=s) * d for s in ((2 * I, H), (H, I))]
    d_bits = int(np.float16(d).view(np.uint16))
    enc = []
    for m in mats:
        rows = []
        for r in range(m.shape[0]):
            q = np.rint(m[r] / d).astype(np.int64)
            rows.append(np.concatenate([_q8_block(d_bits, q[c:c + 32]) for c in range(0, m.shape[1], 32)]))
        enc.append(np.stack(rows))
    return mats, enc


def test_expert_matches_numpy_brute_force():
    rng = np.random.default_rng(7)
    H, I = 64, 32
    (GU, D), (gu_b, dn_b) = _tiny_q8_expert(rng, H, I)
    ex = oracle.Experts(1, H, I, False, oracle.Q8_0, oracle.Q8_0, gu_b[None], dn_b[None])
    x = rng.normal(0, 1, H)
    a, b = GU[:I] @ x, GU[I:] @ x
    want = D @ (a / (1 + np.exp(-a)) * b)
    got = ex.expert(0, x)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-14)


def _small_layer(fmt_gu=oracle.Q8_0, fmt_dn=oracle.Q8_0, shared=True, E=12, H=64, I=32, k=3, seed=3):
    wl = synth.Workload("pin", H, E, I, k, shared, fmt_gu, fmt_dn, synth.DT_BF16, 5, seed=seed)
    return wl, synth.layer_inputs(wl)


def test_expert_of_every_format_is_the_ffn_of_its_decoded_matrices():
    """The expert FFN assembled from the pinned block decoders, for every format pair and the
    shared expert's slot: gate rows first then up rows, SwiGLU, down, each projection with its
    own NVFP4 tensor scale and the layer's IQ4_NL table.  A swapped gate/up half, a wrong
    scale index or a transposed down matrix in any format's path fails here."""
    rng = np.random.default_rng(11)
    pairs = ((oracle.Q8_0, oracle.Q8_0), (oracle.Q5_1, oracle.Q5_1), (oracle.Q5_0, oracle.Q5_0),
             (oracle.IQ4_NL, oracle.IQ4_NL), (oracle.NVFP4, oracle.NVFP4), (oracle.IQ4_NL, oracle.Q5_1),
             (oracle.Q5_0, oracle.IQ4_NL), (oracle.NVFP4, oracle.Q8_0))
    for fgu, fdn in pairs:
        wl, li = _small_layer(fgu, fdn, E=3, seed=10 * fgu + fdn)
        ex = oracle.Experts.from_layer(li)
        H, I = wl.hidden, wl.inter
        for e in range(wl.n_experts + 1):  # slot n_experts holds the shared expert
            gs = 1.0 if li.gate_up_scale is None else float(li.gate_up_scale[e])
            ds = 1.0 if li.down_scale is None else float(li.down_scale[e])
            GU = oracle.decode_matrix(fgu, li.gate_up[e], 2 * I, H, li.table, gs)
            D = oracle.decode_matrix(fdn, li.down[e], H, I, li.table, ds)
            x = rng.normal(0, 1, H)
            a, b = GU[:I] @ x, GU[I:] @ x
            want = D @ (a / (1 + np.exp(-a)) * b)
            got = ex.expert(e, x)
            assert np.allclose(got, want, rtol=1e-12, atol=1e-13 * np.abs(want).max()), (fgu, fdn, e)


def test_layer_is_the_gate_weighted_sum_of_its_selected_experts():
    """The layer restated in numpy from its definition: bf16 router logits, the k largest
    (lower index on ties), softmax renormalised over the selection, each selected expert
    weighted by its own gate, plus the shared expert with gate 1.  Gates differ from
    one another here, so a combine that pairs an expert with another selection's gate fails."""
    for fmts in ((oracle.Q8_0, oracle.Q8_0), (oracle.IQ4_NL, oracle.Q5_1), (oracle.NVFP4, oracle.NVFP4)):
        wl, li = _small_layer(*fmts, k=4)
        ex = oracle.Experts.from_layer(li)
        x = synth.tokens_f64(wl, synth.tokens(wl, li.router))
        out, idx, gate = ex.layer(x, li.router, wl.top_k)
        wf = synth.bf16_to_f32(li.router).astype(np.float64)
        for t in range(x.shape[0]):
            lt = [sum(float(wf[e, h]) * float(x[t, h]) for h in range(wl.hidden)) for e in range(wl.n_experts)]
            sel = sorted(range(wl.n_experts), key=lambda e: (-lt[e], e))[:wl.top_k]
            w = [math.exp(lt[e] - lt[sel[0]]) for e in sel]
            g = [v / sum(w) for v in w]
            assert max(g) - min(g) > 1e-3  # distinct gates: the pairing matters
            want = sum(gj * ex.expert(e, x[t]) for gj, e in zip(g, sel)) + ex.expert(wl.n_experts, x[t])
            assert list(idx[t]) == sel
            assert np.allclose(gate[t], g, rtol=1e-12, atol=0)
            assert np.allclose(out[t], want, rtol=1e-11, atol=1e-13 * np.abs(want).max())


def test_dense_sum_identity_when_k_equals_E_and_uniform_gates():
    for fmts in ((oracle.Q8_0, oracle.Q8_0), (oracle.IQ4_NL, oracle.Q5_1), (oracle.NVFP4, oracle.NVFP4)):
        wl, li = _small_layer(*fmts)
        ex = oracle.Experts.from_layer(li)
        x = synth.tokens_f64(wl, synth.tokens(wl.with_(margin=0.0), li.router))
        zero_router = np.zeros_like(li.router)
        out, idx, gate = ex.layer(x, zero_router, wl.n_experts)
        assert np.all(gate == 1.0 / wl.n_experts)
        for t in range(x.shape[0]):
            assert sorted(idx[t]) == list(range(wl.n_experts))
            ys = [ex.expert(e, x[t]) for e in range(wl.n_experts)]
            want = np.mean(ys, axis=0) + ex.expert(wl.n_experts, x[t])
            assert np.allclose(out[t], want, rtol=1e-12, atol=1e-15)


def test_token_permutation_invariance_bitwise():
    wl, li = _small_layer(oracle.IQ4_NL, oracle.Q5_1)
    ex = oracle.Experts.from_layer(li)
    x = synth.tokens_f64(wl, synth.tokens(wl, li.router))
    out, idx, gate = ex.layer(x, li.router, wl.top_k)
    p = np.array([3, 0, 4, 1, 2])
    out_p, idx_p, gate_p = ex.layer(x[p], li.router, wl.top_k)
    assert np.array_equal(out_p, out[p])
    assert np.array_equal(idx_p, idx[p])


def test_top1_equals_argmax_expert():
    wl, li = _small_layer(shared=False)
    ex = oracle.Experts.from_layer(li)
    x = synth.tokens_f64(wl, synth.tokens(wl.with_(top_k=1), li.router))
    out, idx, gate = ex.layer(x, li.router, 1)
    assert np.all(gate == 1.0)
    for t in range(x.shape[0]):
        assert np.array_equal(out[t], ex.expert(int(idx[t, 0]), x[t]))


def test_linearity_in_down_scales_bitwise():
    wl, li = _small_layer(shared=True)
    ex = oracle.Experts.from_layer(li)
    x = synth.tokens_f64(wl, synth.tokens(wl, li.router))
    out, _, _ = ex.layer(x, li.router, wl.top_k)
    dn2 = li.down.copy().reshape(li.down.shape[0], wl.hidden, -1, 34)
    d = dn2[..., 0].astype(np.uint16) | (dn2[..., 1].astype(np.uint16) << 8)
    d2 = (d.view(np.float16) * np.float16(2)).view(np.uint16)  # exact: exponent + 1
    dn2[..., 0], dn2[..., 1] = d2 & 255, d2 >> 8
    ex2 = oracle.Experts.from_layer(li, down=dn2.reshape(li.down.shape))
    out2, _, _ = ex2.layer(x, li.router, wl.top_k)
    assert np.array_equal(out2, 2 * out)


# ---------------------------------------------------------------- activation quantisation


def _e2m1_nearest_even(v):
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    a = min(abs(v), 6.0)
    best = min(range(8), key=lambda c: (abs(a - mags[c]), c & 1))  # ties to even mantissa
    return math.copysign(mags[best], v)


def test_act_quant_nvfp4_brute_force():
    rng = np.random.default_rng(11)
    for trial in range(20):
        v = rng.normal(0, 1, 64) * (10.0 ** rng.uniform(-3, 3))
        got = oracle.act_quant_nvfp4(v)
        s = np.float32(np.max(np.abs(v.astype(np.float32)))) / np.float32(6 * 448)
        grid = sorted({torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item()
                       for c in range(127)})
        for b in range(4):
            blk = v[b * 16:(b + 1) * 16].astype(np.float32)
            q = np.float32(np.max(np.abs(blk))) / (np.float32(6) * s)
            # nearest E4M3 by brute force, ties to the even code
            cands = sorted(range(127), key=lambda c: (abs(grid[c] - float(q)), c & 1))
            sb = grid[cands[0]]
            den = np.float32(s) * np.float32(sb)
            want = [float(s) * sb * _e2m1_nearest_even(float(np.float32(x) / den)) for x in blk]
            assert np.array_equal(got[b * 16:(b + 1) * 16], want), (trial, b)


def test_act_quant_nvfp4_exact_values_and_ties():
    s = 1.0  # amax = 6 * 448 makes the per-vector scale exactly 1
    v = np.zeros(16)
    v[0] = 6 * 448
    v[1:8] = [0.25 * 448, 0.75 * 448, 1.25 * 448, 2.5 * 448, 5 * 448, 3.5 * 448, 1.75 * 448]
    got = oracle.act_quant_nvfp4(v)
    assert got[0] == 6 * 448 * s
    assert list(got[1:8] / 448) == [0.0, 1.0, 1.0, 2.0, 4.0, 4.0, 2.0]


def test_act_quant_nvfp4_block_scale_ties_and_subnormals():
    """Block scales on exact E4M3 ties, worked by hand.  v[0] = 6 * 448 makes the
    per-vector scale exactly 1, so a block scale is (block max) / 6 rounded to E4M3:
      block 1: max 63 -> 10.5, halfway between 10 and 11 -> 10 (even mantissa);
               63 / 10 = 6.3 -> E2M1 6 -> 60;  -35 / 10 = -3.5, halfway -> -4 -> -40
      block 2: max 21 * 2^-9 -> 3.5 * 2^-9, halfway between the subnormal steps
               3 and 4 * 2^-9 -> 4 * 2^-9 = 2^-7;  21 * 2^-9 / 2^-7 = 5.25 -> 6 -> 0.046875"""
    v = np.zeros(48)
    v[0] = 6 * 448
    v[16], v[17] = 63.0, -35.0
    v[32] = 21 * 2.0 ** -9
    got = oracle.act_quant_nvfp4(v)
    want = np.zeros(48)
    want[0] = 6 * 448
    want[16], want[17] = 60.0, -40.0
    want[32] = 0.046875
    assert np.array_equal(got, want), got[np.nonzero(got != want)]


def test_oracle_ctypes_descriptor_matches_its_header(repo_tmp):
    """The oracle's ctypes descriptor puts every field where the C compiler does, so the
    oracle reads the blocks, scales and table it is handed."""
    import ctypes
    import subprocess
    desc = oracle._Desc
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "oracle.h"', "int main(void)", "{",
             '    printf("size %zu\\n", sizeof(oracle_desc));']
    for field, _ in desc._fields_:
        lines.append(f'    printf("{field} %zu\\n", offsetof(oracle_desc, {field}));')
    lines += ["    return 0;", "}"]
    src, exe = repo_tmp / "odesc.c", repo_tmp / "odesc"
    src.write_text("\n".join(lines) + "\n")
    here = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(here, "oracle"), str(src), "-o",
                    str(exe)], check=True, capture_output=True, text=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], check=True, capture_output=True,
                                                        text=True).stdout.splitlines())
    assert int(got["size"]) == ctypes.sizeof(desc)
    for field, _ in desc._fields_:
        assert int(got[field]) == getattr(desc, field).offset, field
