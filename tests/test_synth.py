"""The seeded input generator: determinism, regenerating one expert alone,
quantiser round-trip bounds (decoded with the oracle), the top-k margin and
the Zipf popularity of the biased router.  CPU only."""
import numpy as np

import oracle
import synth


def test_normal_table_is_standard_normal():
    z = synth.normal(synth.key(0, 1, 2, 3, 4), 1 << 20)
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1) < 5e-3
    assert np.array_equal(z, synth.normal(synth.key(0, 1, 2, 3, 4), 1 << 20))
    assert not np.array_equal(z[:64], synth.normal(synth.key(0, 1, 2, 3, 5), 64))


def test_single_expert_regenerates_identically():
    wl = synth.WORKLOADS["zipf_batch"].with_(n_experts=16)
    gu, dn, gts, dts = synth.experts(wl, layer=3)
    gu1, dn1, gts1, dts1 = synth.experts(wl, layer=3, e0=9, n=1)
    assert np.array_equal(gu[9], gu1[0]) and np.array_equal(dn[9], dn1[0])
    assert gts[9] == gts1[0] and dts[9] == dts1[0]
    gu2, _, _, _ = synth.experts(wl, layer=4, e0=9, n=1)
    assert not np.array_equal(gu1, gu2)


def _roundtrip(fmt, rows=64, cols=256, sigma=0.02, seed=5):
    w = synth.normal(synth.key(seed, 9, 9, 9, 9), rows * cols, sigma).reshape(rows, cols)
    tab = synth.IQ4NL_TABLE
    blocks, ts = synth.encode(fmt, w, tab)
    deq = oracle.decode_matrix(fmt, blocks, rows, cols, tab, ts if ts is not None else 1.0)
    return w.astype(np.float64), deq, blocks, ts


def test_q8_0_roundtrip_within_half_step():
    w, deq, blocks, _ = _roundtrip(synth.FMT_Q8_0)
    d = blocks.reshape(64, -1, 34)[..., :2].copy().view(np.float16)[..., 0].astype(np.float64)
    err = np.abs(w - deq).reshape(64, -1, 32)
    assert np.all(err <= d[..., None] / 2 * (1 + 1e-3) + 1e-12)


def test_q5_1_roundtrip_within_half_step():
    w, deq, blocks, _ = _roundtrip(synth.FMT_Q5_1)
    d = blocks.reshape(64, -1, 24)[..., :2].copy().view(np.float16)[..., 0].astype(np.float64)
    err = np.abs(w - deq).reshape(64, -1, 32)
    assert np.all(err <= d[..., None] / 2 * (1 + 1e-3) + 1e-6)


def test_q5_0_roundtrip_within_half_step_and_extreme_exact():
    w, deq, blocks, _ = _roundtrip(synth.FMT_Q5_0)
    d = blocks.reshape(64, -1, 22)[..., :2].copy().view(np.float16)[..., 0].astype(np.float64)
    err = np.abs(w - deq).reshape(64, -1, 32)
    ad = np.abs(d[..., None])
    # codes run -16 .. 15 around zero: an element opposite the extreme one can
    # need +16 and is clamped to 15 (error at most one step); the rest round
    clamped = w.reshape(64, -1, 32) / d[..., None] > 15.5
    assert np.all(err <= ad * (1 + 1e-3) + 1e-6)
    assert np.all(err[~clamped] <= ad[..., 0:1].repeat(32, -1)[~clamped] / 2 * (1 + 1e-3) + 1e-6)
    # the element of largest magnitude gets code 0: it decodes to -16 d
    wb = w.reshape(64, -1, 32)
    jx = np.abs(wb).argmax(-1)
    ext = np.take_along_axis(deq.reshape(64, -1, 32), jx[..., None], -1)[..., 0]
    assert np.array_equal(ext, -16.0 * d)


def test_iq4_nl_picks_nearest_level():
    w, deq, blocks, _ = _roundtrip(synth.FMT_IQ4_NL)
    d = blocks.reshape(64, -1, 18)[..., :2].copy().view(np.float16)[..., 0].astype(np.float64)
    levels = d[..., None, None] * synth.IQ4NL_TABLE.astype(np.float64)  # [64, nb, 1, 16]
    dist = np.abs(w.reshape(64, -1, 32)[..., None] - levels)
    best = dist.min(-1)
    mine = np.abs(w - deq).reshape(64, -1, 32)
    assert np.all(mine <= best + 1e-7 * np.abs(d[..., None]) + 1e-12)


def test_nvfp4_picks_nearest_code_at_block_scale():
    w, deq, blocks, ts = _roundtrip(synth.FMT_NVFP4)
    assert abs(ts - np.abs(w).max() / (6 * 448)) <= 1e-6 * ts
    sb = blocks.reshape(64, -1, 9)[..., 0]
    scale = ts * np.vectorize(oracle.e4m3)(sb)                    # [64, nb]
    codes = np.array([oracle.e2m1(c) for c in range(16)])
    dist = np.abs(w.reshape(64, -1, 16)[..., None] - scale[..., None, None] * codes)
    mine = np.abs(w - deq).reshape(64, -1, 16)
    assert np.all(mine <= dist.min(-1) * (1 + 1e-5) + 1e-12)


def test_tokens_keep_the_topk_margin():
    wl = synth.WORKLOADS["model_decode"]
    wr, _ = synth.router(wl)
    x = synth.tokens(wl, wr, n_tokens=16)
    _, _, logits = oracle.route(synth.tokens_f64(wl, x), wr, wl.top_k)
    srt = -np.sort(-logits, axis=1)
    assert np.all(srt[:, wl.top_k - 1] - srt[:, wl.top_k] >= wl.margin)


def test_correlated_tokens_share_a_base():
    wl = synth.WORKLOADS["spec_verify"]
    wr, _ = synth.router(wl)
    x = synth.tokens_f64(wl, synth.tokens(wl, wr))
    c = np.corrcoef(x)
    off = c[~np.eye(len(c), dtype=bool)]
    assert off.min() > 0.8  # 1 / (1 + 0.3^2) ~ 0.92 for b + 0.3 eps


def test_zipf_router_popularity_slope():
    wl = synth.WORKLOADS["prefill_nvfp4"]
    wr, rank = synth.router(wl)
    x = synth.tokens(wl.with_(margin=0.0), wr, n_tokens=2048)
    idx, _, _ = oracle.route(synth.tokens_f64(wl, x), wr, wl.top_k)
    counts = np.bincount(idx.ravel(), minlength=wl.n_experts)
    by_rank = np.zeros(wl.n_experts)
    by_rank[rank - 1] = counts
    r = np.arange(1, wl.n_experts + 1)
    m = by_rank >= 5
    slope = -np.polyfit(np.log(r[m]), np.log(by_rank[m]), 1)[0]
    assert abs(slope - 1.1) < 0.1, slope
