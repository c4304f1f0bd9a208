#!/usr/bin/env python
"""Throughput of the block-quantised routed MoE layer on B200.

One step = one forward (route, plan, gate/up + SwiGLU, down, combine) of each
of L distinct synthetic layers on its own batch of T tokens, replayed as one
CUDA graph.  The L layers' selected experts (L x ~23.7 MB for the
model-shaped decode layer) are far larger than the 126 MB L2, so no step finds
its weights in L2.  value = layer-tokens per second = K * L * T / time (max
over ranks); the expert-weight GB/s and the roofline of the dominant kernel
come from the same inputs.  Everything is seeded and synthetic (synth/).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
STAGES = ["route_plan", "gate_up", "down", "combine", "fused", "prefill"]
KERNEL_NAMES = {"route_plan": "route_kernel", "gate_up": "matvec_kernel<gate/up>",
                "down": "matvec_kernel<down>", "combine": "combine_kernel",
                "fused": "fused_decode_kernel", "prefill": "prefill sequence"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="model_decode", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--layers", type=int, default=48, help="distinct layers per step")
    ap.add_argument("--tokens", type=int, default=0, help="override tokens per layer")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="headline only (default: also the 8-token stack and both prefill chunks)")
    ap.add_argument("--quick", action="store_true", help="for profiler runs: few steps, no baselines")
    ap.add_argument("--path", choices=["auto", "grouped", "dense", "tail", "staged", "prefill_bf16"], default="auto",
                    help="kernel path (dense: the dense-batched comparison variant; tail: the one-launch tail, "
                         "also at one token; staged: its tensor-core work as separate launches; prefill_bf16: "
                         "the bf16-dequantising prefill for every format)")
    return ap.parse_args()


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index):
        self.samples = []
        self.stop_ev = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report it rather than guess
            self.err = str(e)

    def _run(self):
        while not self.stop_ev.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop_ev.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"nvml unavailable: {self.err}"]}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = statistics.median(s[0] for s in self.samples)
        seen = set()
        for _, rs in self.samples:
            for name, bit in self.REASONS.items():
                if rs & bit:
                    seen.add(name)
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": sorted(seen),
                "samples": len(self.samples)}


def peaks():
    try:
        p = json.load(open(PEAKS_FILE))
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak(kind):
    """Dense tensor peak in TFLOP/s for bf16 or fp4 (fp4 = bf16 x 4, the nominal
    2.25 -> 9 PFLOP/s ratio), sustained figure (prefill runs inside long steps)."""
    try:
        p = json.load(open(PEAKS_FILE))
        bf16, src = float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured sustained bf16"
    except Exception:
        bf16, src = 1400.0, "fallback sustained bf16"
    return (bf16 * 4.0, src + " x4 (nominal fp4/bf16)") if kind == "fp4" else (bf16, src)


def kernel_traffic(stage, wl_name):
    """Per-launch DRAM bytes from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path)).get(f"{stage}:{wl_name}")
    except Exception:
        return None
    if not rec:
        return None
    if rec.get("source_sha") != kernel_source_sha(rec.get("source_files")):
        return None
    return rec.get("bytes_per_launch")


def traffic_source(stage, wl_name):
    """Where roofline.traffic comes from, or why it is null."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path)).get(f"{stage}:{wl_name}")
    except Exception:
        rec = None
    if not rec:
        return {"status": f"no ncu capture recorded for {stage}:{wl_name}", "kernel_source_sha": kernel_source_sha()}
    cur = kernel_source_sha(rec.get("source_files"))
    same = rec.get("source_sha") == cur
    return {"status": "captured on this kernel source" if same
            else "kernel source changed since the capture: null until it is retaken",
            "captured_sha": rec.get("source_sha"), "kernel_source_sha": cur, "source_files": rec.get("source_files"),
            "kernel": rec.get("kernel"), "command": rec.get("command")}


def kernel_source_sha(files=None):
    """Hash of the kernel sources a capture depends on: the given .cu files (all of
    them when None) and every shared header."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_quantized_expert_moe_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith(".cuh") or (f.endswith(".cu") and (files is None or f in files)):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------- CPU oracle


def oracle_rate(li, wl, budget_s, max_s=30.0):
    """Oracle layer-tokens/s on a bounded sample of the workload's tokens."""
    import oracle
    ex = oracle.Experts.from_layer(li)
    done, spent, n, step = 0, 0.0, 4, 0
    while spent < budget_s:
        x = synth.tokens(wl, li.router, li.layer, 1000 + step, n)
        t0 = time.perf_counter()
        ex.layer(synth.tokens_f64(wl, x), li.router, wl.top_k)
        dt = time.perf_counter() - t0
        done += n
        spent += dt
        step += 1
        rate = n / max(dt, 1e-9)
        n = int(max(1, min(rate * (budget_s - spent), rate * (max_s - spent), 4096)))
        if spent >= max_s or n < 1:
            break
    return done / spent, done, spent, oracle.threads()


def workload_config(wl, layers, tokens, world):
    """The workload keys both arms report in `config`."""
    return {"workload": wl.name, "layers_per_step": layers, "tokens_per_layer": tokens,
            "hidden": wl.hidden, "experts": wl.n_experts, "inter": wl.inter, "top_k": wl.top_k,
            "shared_expert": wl.has_shared,
            "formats": f"{synth.FMT_NAMES[wl.fmt_gate_up]}/{synth.FMT_NAMES[wl.fmt_down]}",
            "parallelism": f"replicas x{world}"}


def reference_arm(a, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    li = synth.layer_inputs(wl, 0)
    import oracle
    ex = oracle.Experts.from_layer(li)
    n = max(1, a.tokens or wl.tokens)
    per_step = []
    total_tok = 0
    for s in range(a.warmup + a.steps):
        x = synth.tokens(wl, li.router, 0, 2000 + s, n)
        t0 = time.perf_counter()
        ex.layer(synth.tokens_f64(wl, x), li.router, wl.top_k)
        dt = time.perf_counter() - t0
        if s >= a.warmup:
            per_step.append(dt)
            total_tok += n
    secs = sum(per_step)
    v = total_tok / secs
    sample = f"{a.steps} steps x {n} tokens of layer 0 ({wl.name}), fp64 oracle"
    line = {"metric": METRIC, "value": v, "unit": "tokens/s",
            "impl": "reference", "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": secs / a.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(wl, 1, n, a.gpus), path="oracle",
                           l2="host memory: one layer per step, fp64 oracle on the host cores"),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- replicas across ranks


def sync_barrier(dist, device_sync):
    """Device sync, then a process barrier, then device sync (no-op barrier at N=1)."""
    device_sync()
    if dist is not None:
        dist.barrier()
    device_sync()


def reduce_max(dist, v, device):
    """Maximum of a per-rank float over all ranks (the slowest replica times the job)."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, steps, layers, tokens, ms_max):
    """Whole-job layer-tokens/s: every rank runs its own replica of the step."""
    return world * steps * layers * tokens / (ms_max / 1e3)


# ---------------------------------------------------------------- GPU arm


METRIC = "MoE layer tokens/s and expert-weight HBM GB/s (% of roofline), 1 B200"


def _to_dev_x(x_np):
    import torch
    if x_np.dtype == np.uint16:
        return torch.from_numpy(x_np.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x_np)).cuda()


def measure(a, bq, torch, wl, layers, T, dist, world, dev, e2e=True):
    """Time K replays of one CUDA graph holding a forward of every layer (T tokens
    each, drawn for workload `wl`), then the same work with an event around each
    kernel.  Returns the measurement as a dict (max over ranks)."""
    L = len(layers)
    k = wl.top_k
    H, E, I = wl.hidden, wl.n_experts, wl.inter
    xbytes = 2 if wl.x_dtype == synth.DT_BF16 else 4
    for l, ly in enumerate(layers):
        x = synth.tokens(wl, ly["router_np"], l, 0, T)
        ly.update(x=_to_dev_x(x), xh=x, out=torch.empty(T, H, device="cuda"))
    info = layers[0]["pack"].info()
    path = {"auto": bq.MOE_PATH_AUTO, "grouped": bq.MOE_PATH_GROUPED, "dense": bq.MOE_PATH_DENSE,
            "tail": bq.MOE_PATH_TAIL, "staged": bq.MOE_PATH_DECODE_STAGED,
            "prefill_bf16": bq.MOE_PATH_PREFILL_BF16}[a.path]

    def fwd(ly):
        bq.moe_layer_forward_ex(ly["x"], ly["wr"], ly["pack"], bq.MOE_FMT_FROM_PACK, k, ly["out"], path)

    # routing of every layer (deterministic): active experts and slots
    n_active, slots = [], []
    for ly in layers:
        fwd(ly)
        idx, gate, counts = bq.moe_read_routing(ly["pack"], T, k)
        n_active.append(int((counts[:E] > 0).sum()) + (1 if wl.has_shared else 0))
        slots.append(T * k + (T if wl.has_shared else 0))
    torch.cuda.synchronize()
    gu_b, dn_b = info["gate_up_bytes_per_expert"], info["down_bytes_per_expert"]
    exp_b = info["expert_bytes"]
    stage_bytes = {
        "route_plan": [E * H * 2 + T * H * xbytes + 2 * T * E * 4 for _ in layers],
        "gate_up": [na * gu_b + T * H * xbytes + s * I * 4 for na, s in zip(n_active, slots)],
        "down": [na * dn_b + s * I * 4 + s * H * 4 for na, s in zip(n_active, slots)],
        "combine": [s * H * 4 + T * H * 4 for s in slots],
    }
    # the one-launch kernels read the router, every active expert's blocks and x,
    # write and re-read h, and write out
    stage_bytes["fused"] = [E * H * 2 + na * exp_b + T * H * xbytes + 2 * s * I * 4 + T * H * 4
                            for na, s in zip(n_active, slots)]
    prefill_flops = [2.0 * T * H * E + 2.0 * s * H * 2 * I + 2.0 * s * I * H for s in slots]
    unique_bytes_step = sum(na * exp_b + E * H * 2 for na in n_active)

    def barrier():
        sync_barrier(dist, torch.cuda.synchronize)

    def max_over_ranks(v):
        return reduce_max(dist, v, "cuda")

    # ---- timed region: K replays of the one-step graph
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for ly in layers:
            fwd(ly)
    for _ in range(max(a.warmup, 3)):
        g.replay()
    barrier()
    st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        st.record()
        for _ in range(a.steps):
            g.replay()
        en.record()
        en.synchronize()
    ms = max_over_ranks(st.elapsed_time(en))
    barrier()
    value = job_throughput(world, a.steps, L, T, ms)
    expert_gbs = world * a.steps * unique_bytes_step / (ms / 1e3) / 1e9
    layer_us = ms / a.steps / L * 1e3  # timed graph: one layer's forward

    # ---- kernel-stage durations: the same work with event records around each kernel
    kp = max(1, min(a.steps, 10))
    for ly in layers:
        bq.moe_profile_begin(ly["pack"], kp)
    gp = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gp):
        for _ in range(kp):
            for ly in layers:
                fwd(ly)
    gp.replay()
    torch.cuda.synchronize()
    stage_ms = np.zeros(32)
    nf = 0
    for ly in layers:
        m, n = bq.moe_profile_end(ly["pack"])
        stage_ms += m
        nf += n
    del gp
    prefill_kernels = 7 if wl.fmt_gate_up == synth.FMT_NVFP4 else 6  # route GEMM, top-k, plan, gather, GEMMs (+ h quant)
    # grouped decode: route, (x gather,) gate/up, down, combine; the x gather runs
    # with the tensor-core kernels (2-64 tokens, H and I multiples of 256)
    tc_path = a.path in ("auto", "staged", "tail") and 2 <= T <= 64 and H % 256 == 0 and I % 256 == 0
    launches_per_fwd = 1 if stage_ms[4] > 0 else (prefill_kernels if stage_ms[5] > 0 else (5 if tc_path else 4))
    stage_us = {s: float(stage_ms[i] / nf * 1e3) for i, s in enumerate(STAGES) if stage_ms[i] > 0}
    phase_names = ["stage_x", "router", "logit_poll_topk", "issue", "gate_up", "h_poll", "down", "-", "tail"]
    # the one-launch tail: chosen explicitly, or by the automatic path for 2-64 tokens
    one_launch_tail = stage_ms[4] > 0 and (a.path == "tail" or (a.path == "auto" and T >= 2))
    if one_launch_tail:
        # CTA 0's steps in the one-launch tail
        fused_phase_us = {n: float(stage_ms[6 + i] / nf * 1e3) for i, n in enumerate(
            ["wait_route", "barrier", "topk", "plan", "x_rows", "units", "combine"])}
    elif stage_ms[4] > 0 and T == 1:
        fused_phase_us = {n: float(stage_ms[6 + i] / nf * 1e3) for i, n in enumerate(phase_names) if n != "-"}
    else:
        fused_phase_us = None
    grid_names = (["last_start", "first_router", "last_router", "first_issue", "last_issue",
                   "first_gate_up", "last_gate_up", "first_end", "last_end"] if not one_launch_tail else
                  # the one-launch tail: routed (grid barrier reached), planned, units done, combined
                  ["last_start", "first_routed", "last_routed", "first_planned", "last_planned",
                   "first_units_done", "last_units_done", "first_end", "last_end"])
    grid_event_us = ({n: float(stage_ms[15 + i] / nf * 1e3) for i, n in enumerate(grid_names)}
                     if stage_ms[4] > 0 and stage_ms[15] > 0 else None)
    if grid_event_us is not None:
        # stream1: CTA 0 at eight internal points; tail: CTA 0's first four units, raw
        # stage landed (4) then MMAs issued (4); from the kernel's start
        grid_event_us["cta0_points"] = [round(float(v / nf * 1e3), 3) for v in stage_ms[24:32]]
    elif stage_ms[0] > 0 and stage_ms[15] > 0:
        route_names = ["last_start", "first_staged", "last_staged", "first_logits", "last_logits",
                       "first_topk_end", "last_topk_end", "first_plan_end", "last_plan_end"]
        grid_event_us = {"route_" + n: float(stage_ms[15 + i] / nf * 1e3) for i, n in enumerate(route_names)}
        step_names = ["stage_logits", "select", "topk_rest", "ticket", "counts", "scans", "groups",
                      "slot_order", "tail"]
        fused_phase_us = {"route_" + n: float(stage_ms[6 + i] / nf * 1e3) for i, n in enumerate(step_names)}
    dom = max(stage_us, key=lambda s: stage_us[s])
    kname = KERNEL_NAMES[dom]
    if dom == "fused":
        kname = ("tail_kernel" if one_launch_tail else "stream1_kernel" if T == 1 else "fused_decode_kernel")
    if a.path in ("auto", "staged") and T >= 2 and dom in ("gate_up", "down"):
        kname = f"dtc_kernel<{dom.replace('_', '/')}>" if tc_path else f"sgm_kernel<{dom.replace('_', '/')}>"
    hbm, peak_src = peaks()
    traffic = kernel_traffic(dom, wl.name)
    if launches_per_fwd == 1:
        # one launch per layer: its duration inside the timed region is the
        # timed graph's time per layer
        launch_us, launch_src = layer_us, "timed graph: ms_per_step / layers (one launch per layer)"
    else:
        # several launches per layer: the event-bracketed replay (no overlap between
        # launches) gives each kernel's share; scaled so that the shares add up to the
        # timed graph's time per layer
        prof_sum = sum(stage_us.values())
        launch_us = stage_us[dom] * layer_us / prof_sum
        launch_src = (f"timed graph share: event-bracketed {stage_us[dom]:.2f} us of {prof_sum:.2f} us per "
                      f"layer, scaled to the timed {layer_us:.2f} us per layer")
    if dom == "prefill":
        kind = "fp4" if wl.fmt_gate_up == synth.FMT_NVFP4 else "bf16"
        tpk, tsrc = tensor_peak(kind)
        fl = float(np.mean(prefill_flops))
        achieved = fl / (layer_us * 1e-6) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": tpk, "unit": "TFLOP/s",
                    "frac": achieved / tpk, "traffic": traffic, "kernel": KERNEL_NAMES[dom],
                    "peak_source": tsrc, "algorithmic_flops_per_launch": fl, "avg_launch_us": layer_us,
                    "launch_time_source": "timed graph: ms_per_step / layers (the whole prefill sequence)"}
    else:
        dom_bytes = float(np.mean(stage_bytes[dom]))
        achieved = dom_bytes / (launch_us * 1e-6) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "traffic": traffic, "kernel": kname,
                    "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                    else "fallback 6650 GB/s",
                    "algorithmic_bytes_per_launch": dom_bytes, "avg_launch_us": launch_us,
                    "launch_time_source": launch_src}
    roofline["traffic_source"] = traffic_source(dom, wl.name)

    # ---- end to end: pinned host input -> forward -> host output, every layer, every step
    e2e_rec = None
    if e2e and not a.no_e2e:
        xh = [torch.from_numpy(ly["xh"].view(np.int16) if ly["xh"].dtype == np.uint16 else ly["xh"]).pin_memory()
              for ly in layers]
        oh = [torch.empty(T, H, dtype=torch.float32).pin_memory() for _ in layers]
        ge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge):
            for ly, xin, o in zip(layers, xh, oh):
                ly["x"].view(xin.dtype).copy_(xin, non_blocking=True)
                fwd(ly)
                o.copy_(ly["out"], non_blocking=True)
        for _ in range(max(a.warmup, 3)):
            ge.replay()
        barrier()
        st.record()
        for _ in range(a.steps):
            ge.replay()
        en.record()
        en.synchronize()
        ems = max_over_ranks(st.elapsed_time(en))
        barrier()
        e2e_rec = {"value": world * a.steps * L * T / (ems / 1e3), "unit": "tokens/s",
                   "h2d_bytes_per_step": L * T * H * xbytes, "d2h_bytes_per_step": L * T * H * 4,
                   "ms_per_step": ems / a.steps}
        del ge
    del g
    return {"value": value, "ms_per_step": ms / a.steps, "layer_us": layer_us,
            "config": workload_config(wl, L, T, world),
            "l2": f"inputs larger than L2: {L} distinct layers, "
                  f"{unique_bytes_step / 1e6:.0f} MB of selected expert weights per step",
            "expert_gbs": expert_gbs, "expert_gbs_frac": expert_gbs / hbm,
            "unique_expert_bytes_per_step": unique_bytes_step,
            "active_experts_per_layer": float(np.mean(n_active)),
            "stage_us": stage_us, "profiled_layer_us": float(sum(stage_us.values())),
            "fused_phase_us": fused_phase_us, "grid_event_us": grid_event_us, "roofline": roofline,
            "clocks": clk.summary(), "e2e": e2e_rec, "gpu_launches": launches_per_fwd * L * a.steps,
            "launches_per_layer": launches_per_fwd}


def build_layers(bq, torch, wl, L, max_tokens, dev, flags=0):
    layers = []
    for l in range(L):
        li = synth.layer_inputs(wl, l)
        pack = bq.pack_layer(li, max_tokens=max_tokens, max_top_k=wl.top_k, device=dev, flags=flags)
        layers.append({"pack": pack, "router_np": li.router,
                       "wr": torch.from_numpy(li.router.view(np.int16)).cuda(), "li": li if l == 0 else None})
        del li
    return layers


def free_layers(layers):
    for ly in layers:
        ly["pack"].free()


# configurations measured beside the headline in the default run: the 48-layer
# speculative-verify stack on the headline's own layers (same weights: the
# generator keys them by layer), and the prefill chunk with NVFP4 and Q8_0 weights
EXTRA_PREFILL = ("prefill_nvfp4", "prefill_q8")


def ours_arm(a, wl):
    import torch
    import block_quantized_expert_moe_b200 as bq
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.cuda.current_device()
    T = a.tokens or wl.tokens
    L = a.layers
    extras = not a.no_extra and wl.name == "model_decode" and not a.tokens
    sv = synth.WORKLOADS["spec_verify"]
    t0 = time.time()
    layers = build_layers(bq, torch, wl, L, max(T, sv.tokens) if extras else T, dev,
                          bq.MOE_PACK_DENSE if a.path == "dense" else 0)
    gen_s = time.time() - t0
    log(f"[bench] rank {rank}: built {L} layers of {wl.name} in {gen_s:.1f} s")
    li0 = layers[0]["li"]
    head = measure(a, bq, torch, wl, layers, T, dist, world, dev)
    extra = {}
    if extras:
        extra["spec_verify"] = measure(a, bq, torch, sv, layers, sv.tokens, dist, world, dev, e2e=False)
    free_layers(layers)
    del layers
    if extras:
        for name in EXTRA_PREFILL:
            pw = synth.WORKLOADS[name]
            pl = build_layers(bq, torch, pw, 2, pw.tokens, dev)
            extra[name] = measure(a, bq, torch, pw, pl, pw.tokens, dist, world, dev, e2e=False)
            free_layers(pl)
            del pl

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline and not a.quick:
        import oracle
        v, n, secs, cores = oracle_rate(li0, wl, a.cpu_seconds)
        oracle.set_threads(1)
        v1, n1, secs1, _ = oracle_rate(li0, wl, a.cpu_seconds / 2)
        oracle.set_threads(cores)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} tokens of layer 0 ({wl.name}) in {secs:.1f} s, fp64 oracle, "
                         f"OpenMP over tokens",
               "value_1core": v1, "sample_1core": f"{n1} tokens of layer 0 in {secs1:.1f} s on one thread"}

    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": dict(head["config"], path=a.path, l2=head["l2"])}
        for key in ("expert_gbs", "expert_gbs_frac", "unique_expert_bytes_per_step", "active_experts_per_layer",
                    "layer_us", "stage_us", "profiled_layer_us", "fused_phase_us", "grid_event_us", "roofline",
                    "clocks", "e2e", "gpu_launches", "launches_per_layer"):
            line[key] = head[key]
        line["cpu_baseline"] = cpu
        line["gen_seconds"] = gen_s
        if extra:
            line["workloads"] = {n: {kk: vv for kk, vv in m.items() if kk not in ("e2e", "l2")}
                                 for n, m in extra.items()}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    a = parse()
    wl = synth.WORKLOADS[a.workload]
    if a.quick:
        a.no_e2e = True
        a.no_cpu_baseline = True
        a.no_extra = True
    if a.impl == "reference":
        reference_arm(a, wl)
    else:
        ours_arm(a, wl)


if __name__ == "__main__":
    main()
