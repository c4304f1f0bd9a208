"""Expert parallelism on the host: two gloo ranks, each taking its window of the
experts (ep.expert_window, the shared expert on rank 0 only), compute their
share of the layer with the oracle's pieces; ep.combine (the all-reduce the GPU
ranks use) must give the oracle's whole layer.  This pins the partition and the
sum; the GPU kernels' windowed plan is checked on one GPU in test_gpu_ep.py."""
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import oracle
    import synth
    from block_quantized_expert_moe_b200 import ep  # loads on a CPU host: no CUDA call at import
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        dist.init_process_group("gloo", rank=rank, world_size=world)
        wl = synth.Workload("ep", 256, 12, 64, 3, True, synth.FMT_IQ4_NL, synth.FMT_Q5_1, synth.DT_BF16, 5, seed=9)
        li = synth.layer_inputs(wl)
        x = synth.tokens(wl, li.router, 0, 0, 5)
        xf = synth.tokens_f64(wl, x)
        ex = oracle.Experts.from_layer(li)
        idx, gate, _ = oracle.route(xf, li.router, wl.top_k)
        b, e = ep.expert_window(rank, world, wl.n_experts)
        part = np.zeros((5, wl.hidden))
        for t in range(5):
            for j in range(wl.top_k):
                if b <= idx[t, j] < e:
                    part[t] += gate[t, j] * ex.expert(int(idx[t, j]), xf[t])
            if ep.holds_shared(rank):
                part[t] += ex.expert(wl.n_experts, xf[t])
        out = torch.from_numpy(part)
        ep.combine(out)
        full, _, _ = ex.layer(xf, li.router, wl.top_k)
        q.put((rank, float(np.abs(out.numpy() - full).max() / np.abs(full).max()), (b, e)))
        dist.destroy_process_group()
    except Exception as exc:  # report to the parent instead of hanging it
        q.put((rank, repr(exc), None))


def test_two_rank_expert_windows_sum_to_the_layer():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = [q.get(timeout=240) for _ in ps]
    for p in ps:
        p.join(timeout=60)
    res.sort()
    assert all(isinstance(r[1], float) for r in res), res
    assert [r[2] for r in res] == [(0, 6), (6, 12)]
    for _, err, _ in res:
        assert err < 1e-12, err
