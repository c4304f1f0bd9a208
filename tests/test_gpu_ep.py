"""Expert parallelism of the CUDA path on one GPU: the packs of two (and three)
expert windows run one after another on the same GPU (independent launches,
nothing waits on another rank), and their outputs must sum to the layer: bit
for bit on an exact layer (tests/exact_layers.py), within the decode tolerance
on the model-shaped one.  The multi-GPU all-reduce of those shares is
block_quantized_expert_moe_b200/ep.py (its arithmetic is checked on gloo ranks
in test_ep_dist.py)."""
import numpy as np
import pytest

import synth
from exact_layers import exact_layer, exact_tokens
from harness import DECODE_TOL, normwise_err, oracle_layer, router_to_device, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _shares(li, x, k, world, T):
    import block_quantized_expert_moe_b200 as bq
    from block_quantized_expert_moe_b200 import ep
    xt, wr = to_device(x), router_to_device(li.router)
    total = np.zeros((T, li.wl.hidden))
    counts = np.zeros(li.wl.n_experts + 1, np.int64)
    for r in range(world):
        pack = ep.pack_rank(li, r, world, max_tokens=T, max_top_k=k)
        try:
            out = torch.full((T, li.wl.hidden), float("nan"), device="cuda")
            bq.moe_layer_forward(xt, wr, pack, bq.MOE_FMT_FROM_PACK, k, out)
            torch.cuda.synchronize()
            assert bq.moe_get_device_error(pack) == bq.MOE_OK
            total += out.cpu().numpy().astype(np.float64)
            _, _, c = bq.moe_read_routing(pack, T, k)
            b, e = ep.expert_window(r, world, li.wl.n_experts)
            assert (c[:b] == 0).all() and (c[e:li.wl.n_experts] == 0).all()  # only its own experts
            counts += c
        finally:
            pack.free()
    return total, counts


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("T", [1, 6, 64])
def test_expert_windows_sum_to_the_exact_layer_bitwise(world, T):
    li = exact_layer(synth.FMT_IQ4_NL, synth.FMT_Q5_1, n_experts=8, seed=31)
    x = exact_tokens(li, T, seed=T + 3)
    total, _ = _shares(li, x, 1, world, T)
    ref, _, _ = oracle_layer(li, x, 1)
    assert np.array_equal(total, ref)


def test_expert_windows_of_the_model_shaped_layer():
    wl = synth.WORKLOADS["spec_verify"]
    li = synth.layer_inputs(wl, 7)
    x = synth.tokens(wl, li.router, 7, 1, 8)
    total, counts = _shares(li, x, wl.top_k, 2, 8)
    ref, ridx, _ = oracle_layer(li, x, wl.top_k)
    assert normwise_err(total, ref) <= DECODE_TOL
    exp = np.bincount(ridx.ravel(), minlength=wl.n_experts)
    assert np.array_equal(counts[:wl.n_experts], exp) and counts[wl.n_experts] == 8  # the shared expert: rank 0 only


def test_windowed_pack_refuses_other_paths():
    import block_quantized_expert_moe_b200 as bq
    li = exact_layer(synth.FMT_Q8_0, synth.FMT_Q8_0, n_experts=8, seed=5)
    x = exact_tokens(li, 4)
    pack = bq.pack_layer(li, max_tokens=4, max_top_k=1, expert_window=(2, 6))
    try:
        out = torch.empty(4, li.wl.hidden, device="cuda")
        for path in (bq.MOE_PATH_GROUPED, bq.MOE_PATH_DECODE_STAGED, bq.MOE_PATH_PREFILL):
            with pytest.raises(bq.MoeError) as e:
                bq.moe_layer_forward_ex(to_device(x), router_to_device(li.router), pack, bq.MOE_FMT_FROM_PACK, 1,
                                        out, path)
            assert e.value.status == bq.MOE_ERR_UNSUPPORTED
    finally:
        pack.free()
