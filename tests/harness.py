"""Shared helpers of the parity tests: run the CUDA layer through the C ABI and
the fp64 oracle on the same seeded inputs, and compare them."""
import numpy as np

import oracle
import synth

DECODE_TOL = 2e-3   # fp32-accumulate decode: normwise max relative error per token
PREFILL_TOL = 2e-2  # tensor-core prefill
GATE_TOL = 1e-5     # gates compared per expert id, absolute


def to_device(x_np):
    import torch
    if x_np.dtype == np.uint16:
        return torch.from_numpy(x_np.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x_np)).cuda()


def router_to_device(wr):
    import torch
    return torch.from_numpy(np.ascontiguousarray(wr).view(np.int16)).cuda()


def gpu_layer(li, x_np, k, path=None, pack=None, repeat=1, flags=0):
    """Run the layer through the C ABI.  Returns (out [T,H] float64, idx, gate, counts)."""
    import torch
    import block_quantized_expert_moe_b200 as bq
    T = x_np.shape[0]
    own = pack is None
    if own:
        pack = bq.pack_layer(li, max_tokens=T, max_top_k=k, flags=flags)
    xt = to_device(x_np)
    wr = router_to_device(li.router)
    out = torch.full((T, li.wl.hidden), float("nan"), device="cuda")
    outs = []
    for _ in range(repeat):
        if path is None:
            bq.moe_layer_forward(xt, wr, pack, bq.MOE_FMT_FROM_PACK, k, out)
        else:
            bq.moe_layer_forward_ex(xt, wr, pack, bq.MOE_FMT_FROM_PACK, k, out, path)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy().astype(np.float64))
    idx, gate, counts = bq.moe_read_routing(pack, T, k)
    assert bq.moe_get_device_error(pack) == bq.MOE_OK
    if own:
        pack.free()
    return (outs[0] if repeat == 1 else outs), idx, gate, counts


def oracle_layer(li, x_np, k, tokens=None, act_quant=0):
    ex = oracle.Experts.from_layer(li)
    xf = synth.tokens_f64(li.wl, x_np)
    if tokens is not None:
        xf = xf[tokens]
    return ex.layer(xf, li.router, k, act_quant)


def normwise_err(got, ref):
    """max over tokens of max_i |got - ref| / max_i |ref|."""
    num = np.abs(got - ref).max(axis=1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float((num / den).max())


def assert_routing_equal(idx_gpu, gate_gpu, idx_ref, gate_ref):
    for t in range(idx_ref.shape[0]):
        assert sorted(idx_gpu[t].tolist()) == sorted(idx_ref[t].tolist()), t
        g = dict(zip(idx_gpu[t].tolist(), gate_gpu[t].tolist()))
        for e, gr in zip(idx_ref[t].tolist(), gate_ref[t].tolist()):
            assert abs(g[e] - gr) <= GATE_TOL, (t, e, g[e], gr)


def expected_counts(idx, n_experts, T, has_shared):
    c = np.bincount(idx.ravel(), minlength=n_experts).astype(np.int64)
    return np.concatenate([c, [T if has_shared else 0]])
