"""Expert parallelism of the MoE layer over ranks (one GPU per rank).

Every rank holds the whole router and a window of each layer's routed experts
(moe_pack_desc.expert_begin / expert_end); rank 0 also holds the shared expert.
A forward on a windowed pack computes that window's share of the layer, the
gate-weighted sum over the selected experts that fall in the window (plus the
shared expert on rank 0), so the layer output is the sum of the ranks' outputs:
one all-reduce of [T x hidden] fp32 per layer, the only exchange of the step.
The weights never move; every expert stays resident in its rank's HBM.
"""
from . import MOE_FMT_FROM_PACK, moe_layer_forward, pack_layer


def expert_window(rank, world, n_experts):
    """The routed experts [begin, end) of `rank` among `world` ranks."""
    return rank * n_experts // world, (rank + 1) * n_experts // world


def holds_shared(rank):
    """The shared (always-on) expert lives on rank 0 only, so it is summed once."""
    return rank == 0


def pack_rank(li, rank, world, **kw):
    """This rank's pack of a synth.LayerInputs-like layer."""
    return pack_layer(li, expert_window=expert_window(rank, world, li.wl.n_experts), shared=holds_shared(rank), **kw)


def combine(out, group=None):
    """Sum the ranks' shares of the layer in place (torch.distributed all-reduce)."""
    import torch.distributed as dist
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def ep_layer_forward(x, router_w, pack, top_k, out, group=None, stream=None):
    """out = the whole layer: this rank's share, then the sum over ranks."""
    moe_layer_forward(x, router_w, pack, MOE_FMT_FROM_PACK, top_k, out, stream)
    return combine(out, group)
