"""Layers whose every intermediate is exact in fp16, bf16, fp32 and fp64.

The layer's matvecs are sums of products of weights and activations.  When the
weights are small integers times powers of two, the tokens small integers, and
every partial sum stays below 2^24 units of its finest power of two, each such
sum is exact in any order and any of those precisions.  SwiGLU is exact too
when every gate pre-activation g is at least 40: exp(-g) < 2^-57, so
1 + exp(-g) rounds to 1 in fp32 and fp64 and silu(g) = g.  With top_k = 1 the
renormalised gate is exp(0) / exp(0) = 1.  So the whole layer output is one
exact value that the fp64 oracle and every CUDA path must reproduce bit for bit
(the tensor-core decode rounds weights, tokens and h to fp16 and the prefill to
bf16: the builders keep all of them representable there).

The builders place chosen codes and scales into the canonical block bytes of
include/moe.h (the byte layout only; no arithmetic of the layer).

Row recipe (hidden H, inter I, tokens x in {1, 2}):
  gate rows  n_gate (>= 40) entries of +1, the rest 0   -> g in [n_gate, 2 n_gate]
  up rows    n_up entries of +-1, the rest 0             -> |u| <= 2 n_up
  down rows  dense small values (format codes times a power-of-two scale)
"""
import numpy as np

import synth

F16_ONE = 0x3C00


def f16_bits(v):
    return int(np.array(v, np.float16).view(np.uint16))


def e4m3_pow2(e):
    """E4M3 byte of 2^e (normal range e in [-6, 8])."""
    assert -6 <= e <= 8
    return (e + 7) << 3


# IQ4_NL table of the exact layers: it holds 0 and +-1 (sparse rows) and small
# values for the down rows; 0, 1 and -1 appear twice each, so every candidate
# bias of the decode kernels' lookup splits the biased bytes' top bits oddly
# (seven entries >= 2, none equal to -2; 100 rules out the bias 192) and the
# kernels use their masked lookup.  The order is not monotone.
EXACT_IQ4NL_TABLE = np.array([0, 0, 1, 1, -1, -1, 2, 3, -3, 4, -4, 5, -5, 100, -100, -6], np.int8)
E2M1 = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def e2m1_code(v):
    c = E2M1[abs(v)]
    return c | (8 if v < 0 else 0)


def _row_values(rng, kind, K, n_gate, n_up):
    if kind == "gate":
        v = np.zeros(K)
        v[rng.choice(K, n_gate, replace=False)] = 1.0
        return v
    v = np.zeros(K)
    v[rng.choice(K, n_up, replace=False)] = rng.choice([-1.0, 1.0], n_up)
    return v


def encode_rows(fmt, rng, kinds, K):
    """Blocks (uint8 [rows, row_bytes]) of rows of the given kinds, plus the
    matrix scale for NVFP4 (1.0).  kinds: list of ("gate"|"up", n_gate, n_up) or
    ("down",) per row."""
    rows = []
    for kind in kinds:
        if kind[0] == "down":
            rows.append(_down_row(fmt, rng, K))
        else:
            rows.append(_sparse_row(fmt, _row_values(rng, kind[0], K, kind[1], kind[2])))
    return np.stack(rows)


def _sparse_row(fmt, v):
    """Values in {-1, 0, 1} with unit scale."""
    K = v.size
    out = bytearray()
    if fmt == synth.FMT_NVFP4:
        for b in range(K // 16):
            codes = [e2m1_code(x) for x in v[16 * b:16 * b + 16]]
            out.append(e4m3_pow2(0))
            out += bytes(codes[2 * i] | (codes[2 * i + 1] << 4) for i in range(8))
        return np.frombuffer(bytes(out), np.uint8)
    for b in range(K // 32):
        blk = v[32 * b:32 * b + 32]
        if fmt == synth.FMT_Q8_0:
            out += F16_ONE.to_bytes(2, "little") + blk.astype(np.int8).tobytes()
        elif fmt == synth.FMT_IQ4_NL:
            tab = list(EXACT_IQ4NL_TABLE)
            idx = [tab.index(int(x)) for x in blk]
            out += F16_ONE.to_bytes(2, "little") + bytes(idx[i] | (idx[i + 16] << 4) for i in range(16))
        elif fmt in (synth.FMT_Q5_1, synth.FMT_Q5_0):
            q = [int(x) + 16 for x in blk]  # d = 1, m = -16 (Q5_1) / w = q - 16 (Q5_0)
            qh = sum(((c >> 4) & 1) << j for j, c in enumerate(q))
            qs = bytes((q[i] & 15) | ((q[i + 16] & 15) << 4) for i in range(16))
            head = F16_ONE.to_bytes(2, "little")
            if fmt == synth.FMT_Q5_1:
                head += f16_bits(-16.0).to_bytes(2, "little")
            out += head + qh.to_bytes(4, "little") + qs
        else:
            raise ValueError(fmt)
    return np.frombuffer(bytes(out), np.uint8)


def _down_row(fmt, rng, K):
    """Dense values with a power-of-two block scale: at most 8 units of 2^-3 in
    magnitude (IQ4_NL: a few +-100 / 8 as well)."""
    out = bytearray()
    if fmt == synth.FMT_NVFP4:
        mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
        for b in range(K // 16):
            vals = rng.choice(mags, 16) * rng.choice([-1.0, 1.0], 16)
            codes = [e2m1_code(x) for x in vals]
            out.append(e4m3_pow2(int(rng.integers(-3, 0))))
            out += bytes(codes[2 * i] | (codes[2 * i + 1] << 4) for i in range(8))
        return np.frombuffer(bytes(out), np.uint8)
    for b in range(K // 32):
        if fmt == synth.FMT_Q8_0:
            d = f16_bits(2.0 ** -int(rng.integers(2, 5)))
            q = rng.integers(-8, 9, 32).astype(np.int8)
            out += d.to_bytes(2, "little") + q.tobytes()
        elif fmt == synth.FMT_IQ4_NL:
            d = f16_bits(2.0 ** -3)
            idx = rng.integers(0, 16, 32)
            big = [i for i, t in enumerate(EXACT_IQ4NL_TABLE) if abs(int(t)) > 10]
            small = [i for i in range(16) if i not in big]
            idx = np.where(rng.random(32) < 0.05, rng.choice(big, 32), rng.choice(small, 32))
            out += d.to_bytes(2, "little") + bytes(int(idx[i]) | (int(idx[i + 16]) << 4) for i in range(16))
        elif fmt in (synth.FMT_Q5_1, synth.FMT_Q5_0):
            e = int(rng.integers(2, 5))
            q = [int(c) for c in rng.integers(0, 32, 32)]
            qh = sum(((c >> 4) & 1) << j for j, c in enumerate(q))
            qs = bytes((q[i] & 15) | ((q[i + 16] & 15) << 4) for i in range(16))
            head = f16_bits(2.0 ** -e).to_bytes(2, "little")
            if fmt == synth.FMT_Q5_1:
                # m a power-of-two multiple of d (w = d q + m); -16 d or -8 d
                head += f16_bits(-(2.0 ** -e) * (16 if rng.random() < 0.5 else 8)).to_bytes(2, "little")
            out += head + qh.to_bytes(4, "little") + qs
        else:
            raise ValueError(fmt)
    return np.frombuffer(bytes(out), np.uint8)


def exact_layer(fmt_gu, fmt_dn, hidden=1024, inter=256, n_experts=8, has_shared=True, n_gate=48, n_up=10,
                x_dtype=synth.DT_BF16, fp16_fallback=False, seed=0):
    """A synth.LayerInputs of an exact layer (top_k = 1).  fp16_fallback adds one
    never-selected expert whose block scale is an fp16 subnormal, so the pack
    turns the tensor-core decode off and 2-64 tokens take the CUDA-core kernels."""
    rng = np.random.default_rng(seed)
    E = n_experts + (1 if fp16_fallback else 0)
    wl = synth.Workload("exact", hidden, E, inter, 1, has_shared, fmt_gu, fmt_dn, x_dtype, 1, seed=seed)
    n_packed = E + (1 if has_shared else 0)
    gu_kinds = [("gate", n_gate, n_up)] * inter + [("up", n_gate, n_up)] * inter
    gate_up = np.stack([encode_rows(fmt_gu, rng, gu_kinds, hidden).ravel() for _ in range(n_packed)])
    down = np.stack([encode_rows(fmt_dn, rng, [("down",)] * hidden, inter).ravel() for _ in range(n_packed)])
    if fp16_fallback:
        # first block of the extra expert: Q8_0 / IQ4_NL a subnormal d; Q5_1 an m
        # beyond the fp16 budget; Q5_0 a d with 47 |d| > 60000 (its m is -16 d)
        patch = {synth.FMT_Q8_0: (0, 2.0 ** -20), synth.FMT_IQ4_NL: (0, 2.0 ** -20),
                 synth.FMT_Q5_1: (2, 65000.0), synth.FMT_Q5_0: (0, 2048.0)}[fmt_gu]
        gate_up[n_experts, patch[0]:patch[0] + 2] = np.frombuffer(f16_bits(patch[1]).to_bytes(2, "little"), np.uint8)
    gs = np.ones(n_packed, np.float32) if fmt_gu == synth.FMT_NVFP4 else None
    ds = np.ones(n_packed, np.float32) if fmt_dn == synth.FMT_NVFP4 else None
    table = EXACT_IQ4NL_TABLE.copy() if synth.FMT_IQ4_NL in (fmt_gu, fmt_dn) else None
    # router: integer multiples of 2^-6 in bf16, so logits of integer tokens are exact
    wr_f = rng.integers(-4, 5, (E, hidden)).astype(np.float32) / 64.0
    if fp16_fallback:
        wr_f[n_experts] = -4.0 / 64.0  # never the top expert of a positive token
    router = synth.bf16_bits(wr_f)
    return synth.LayerInputs(wl, 0, router, gate_up, down, gs, ds, table, None)


def exact_tokens(li, T, seed=1):
    """T tokens in {1, 2} (bf16 bits or fp32) whose top-1 router logit wins by at
    least 2^-6 (logits are exact)."""
    rng = np.random.default_rng(seed)
    wr = synth.bf16_to_f32(li.router).astype(np.float64)
    rows = []
    while len(rows) < T:
        x = rng.integers(1, 3, li.wl.hidden).astype(np.float64)
        lg = np.sort(wr @ x)
        if lg[-1] - lg[-2] >= 2.0 ** -6:
            rows.append(x)
    x = np.stack(rows).astype(np.float32)
    return synth.bf16_bits(x) if li.wl.x_dtype == synth.DT_BF16 else x


def assert_exact_bounds(li, x, h_max=2048):
    """Preconditions of the bitwise pins, from the oracle's block decoders: every
    gate pre-activation >= 40, |h| <= h_max (integers: exact in fp16 up to 2048,
    in bf16 up to 256) and, per output row, sum_i |D_ri| |h_i| < 2^20, so every
    partial sum is an exact multiple of 2^-4 in fp32 (D's values are multiples
    of 2^-4)."""
    import oracle
    wl = li.wl
    xf = synth.tokens_f64(wl, x)
    for e in range(wl.n_packed):
        gs = 1.0 if li.gate_up_scale is None else float(li.gate_up_scale[e])
        ds = 1.0 if li.down_scale is None else float(li.down_scale[e])
        G = oracle.decode_matrix(wl.fmt_gate_up, li.gate_up[e], 2 * wl.inter, wl.hidden, li.table, gs)
        D = oracle.decode_matrix(wl.fmt_down, li.down[e], wl.hidden, wl.inter, li.table, ds)
        assert np.array_equal(D * 16, np.round(D * 16))
        g, u = xf @ G[:wl.inter].T, xf @ G[wl.inter:].T
        h = g * u
        if e < wl.n_experts and (synth.bf16_to_f32(li.router[e]) < 0).all():
            continue  # the fp16 fallback's expert: never selected by positive tokens
        assert g.min() >= 40 and np.abs(h).max() <= h_max, (e, g.min(), np.abs(h).max())
        assert (np.abs(D) @ np.abs(h).T).max() < 2 ** 20, e
