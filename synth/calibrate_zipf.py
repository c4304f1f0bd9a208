"""Choose the popularity-bias strength ZIPF_BETA for the Zipf-routed workloads.

The router bias column gives expert e the logit offset -beta*s*ln(rank(e)).
For each candidate beta this script draws the 512-expert router and a batch of
tokens from the seeded generator, selects each token's top-k experts from fp64
logits (numpy), counts selections per popularity rank and fits the log-log slope
of count against rank.  It prints the slope per beta; ZIPF_BETA in
synth/__init__.py is the value whose slope is closest to the target s.
Input generation only: nothing here is used by the layer or its oracle.
"""
import argparse
import dataclasses

import numpy as np

import synth


def realised_counts(wl, beta, n_tokens, layer=0):
    old = synth.ZIPF_BETA
    synth.ZIPF_BETA = beta
    try:
        wr, rank = synth.router(wl, layer)
    finally:
        synth.ZIPF_BETA = old
    x = synth.tokens(dataclasses.replace(wl, margin=0.0), wr, layer, 0, n_tokens)
    xf = synth.tokens_f64(wl, x)
    logits = xf @ synth.bf16_to_f32(wr).astype(np.float64).T
    sel = np.argpartition(-logits, wl.top_k - 1, axis=1)[:, :wl.top_k]
    counts = np.bincount(sel.ravel(), minlength=wl.n_experts)
    by_rank = np.zeros(wl.n_experts)
    by_rank[rank - 1] = counts
    return by_rank


def fit_slope(by_rank, min_count=5):
    r = np.arange(1, by_rank.size + 1)
    m = by_rank >= min_count
    return -np.polyfit(np.log(r[m]), np.log(by_rank[m]), 1)[0]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=8192)
    ap.add_argument("--betas", type=float, nargs="*", default=[0.6, 0.8, 1.0, 1.2, 1.4, 1.6, 1.8, 2.0])
    a = ap.parse_args()
    wl = synth.WORKLOADS["prefill_nvfp4"]
    for b in a.betas:
        c = realised_counts(wl, b, a.tokens)
        print(f"beta={b:.2f} slope={fit_slope(c):.3f} top={int(c[0])} active={int((c > 0).sum())} "
              f"min_active={int(c[c > 0].min())}")


if __name__ == "__main__":
    main()
