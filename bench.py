#!/usr/bin/env python3
"""Benchmark of the routed-MoE layer forward on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload decode80b|decode35b|prefill|pool_int4|pool_int8|gdn80b|gdn80b_b8]
                    [--tokens T] [--impl ours|reference] [--parallel replicas|ep] [--no-cpu-baseline]
                    [--policy lfu_recency|lru|lfu] [--slots S] [--store host|file|file_direct] [--overlap]

Default workload: the 80B-like decode stack -- hidden 2048, 512 experts, top-10,
intermediate 512, shared expert 512, int4 group 64, one token per step through 48
stacked layers with independent seeded weights, a router bias giving Zipf(1.0)
popularity, all 512 x 48 experts resident (43.5 GB of blobs).  A step is one token
through all 48 layers; the input of layer l+1 is bf16(x_0 + moe_l(x_l)) (x_0 = the step's
token), which keeps the serial dependence between layers and unit-scale activations (a plain
residual chain x_l + moe_l(x_l) grows without bound under random weights).

Timing: W untimed warm-up steps, then K steps timed with CUDA events on the launching
stream, bracketed by a barrier and a device synchronize; the max over ranks is taken.
Each step reads >1 GB of distinct expert blobs, larger than the 126 MB L2, so no flush is
needed between steps.  With N > 1 every rank runs an independent replica by default (weak
scaling; one token stream's layer has no exchange step); `--parallel ep` splits every layer's
experts over the ranks instead (strong scaling, one NCCL all-reduce per layer).  Rank 0 prints
one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per layer of the fused decode
# kernel, from an ncu capture of a 2-layer stack of the same workload (the full stack is too
# large to capture; every layer reads its own blobs, so traffic scales with the layers).  Keyed
# by (kernel, workload, tokens); an entry is dropped whenever the kernel changes and comes back
# with the next capture.
NCU_TRAFFIC_PER_LAYER = {("k_fused_decode", "decode80b", 1): 21_664_640}
# DRAM traffic per launch of the prefill gate/up GEMM on the prefill workload (full-size,
# one-pass capture).  Dropped whenever the kernel changes.
NCU_TRAFFIC_PREFILL_GATEUP = {("prefill", 4096): 829_933_568}


# --------------------------------------------------------------------------------------
# distributed plumbing (host-side helpers are importable for the CPU tests)
# --------------------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


def init_dist(backend: str):
    import torch.distributed as dist
    import datetime
    rank, _, ws = dist_env()
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, ws


def reduce_max(value: float, device) -> float:
    """Max over ranks of a per-rank measurement (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_step_seed(rank: int, step: int) -> int:
    """Activation seed of (rank, step): ranks draw disjoint token streams."""
    return rank * 1_000_003 + step


# --------------------------------------------------------------------------------------
# measurement helpers
# --------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"]
        except Exception:
            sel = []
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [c.strip() for c in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def event_ms(a: torch.cuda.Event, b: torch.cuda.Event) -> float:
    """Elapsed ms between two events (recorded by the library's profiling hook)."""
    return float(a.elapsed_time(b))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def cpu_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# --------------------------------------------------------------------------------------
# decode workloads (our arm)
# --------------------------------------------------------------------------------------
class DecodeStack:
    """All layers of a decode workload resident on one GPU, plus per-step inputs."""

    def __init__(self, w: synth.Workload, T: int, device, n_inputs: int, rank: int = 0):
        from int4_expert_gemv_router_b200 import abi
        self.abi = abi
        self.w, self.T, self.dev = w, T, device
        self.shape = abi.shape_of(w)
        self.stride = synth.blob_stride(w.hidden, w.inter, w.bits)
        E, nL = w.n_experts, w.layers
        self.pool_all = torch.empty(nL * E, self.stride, dtype=torch.uint8, device=device)
        self.layers = []
        for l in range(nL):
            L = synth.make_layer(w, l, device, pool_out=self.pool_all[l * E:(l + 1) * E])
            self.layers.append(L)
        self.slot_table = torch.arange(E, dtype=torch.int32, device=device)
        ws_bytes = abi.moe_workspace_size(self.shape, T)
        self.ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=device)
        self.bufs = [torch.zeros(T, w.hidden, dtype=torch.bfloat16, device=device) for _ in range(nL + 1)]
        self.idx = [torch.zeros(T, w.top_k, dtype=torch.int32, device=device) for _ in range(nL)]
        self.p = [torch.zeros(T, w.top_k, dtype=torch.float32, device=device) for _ in range(nL)]
        self.inputs = torch.stack([synth.activations(w, rank_step_seed(rank, s), tokens=T, device=device)
                                   for s in range(n_inputs)])
        torch.cuda.synchronize(device)

    def descs(self):
        a, w = self.abi, self.w
        return [a.layer_desc(x=self.bufs[l], w_router=L.w_router, router_bias=L.router_bias, pool=L.pool,
                             slot_table=self.slot_table, n_slots=w.n_experts, shared_blob=L.shared,
                             w_shared_gate=L.w_sg, residual=self.bufs[0], out=self.bufs[l + 1],
                             topk_idx_out=self.idx[l], topk_w_out=self.p[l])
                for l, L in enumerate(self.layers)]

    def layer_calls(self):
        """One step: every layer in one moe_stack_forward call."""
        self.abi.moe_stack_forward(self.shape, self.T, self.descs(), self.ws)

    def unique_experts(self):
        """Distinct routed experts per layer of the last step."""
        return [len(set(i.cpu().numpy().reshape(-1).tolist())) for i in self.idx]

    def step_bytes(self, uniq):
        """Algorithmic HBM bytes of one step: every distinct selected blob and the shared blob
        once per layer, router weights (+bias), shared gate, x, residual and out."""
        w, T = self.w, self.T
        act = 3 * T * w.hidden * 2
        router = w.n_experts * w.hidden * 2 + (w.n_experts * 4 if w.router == "zipf" else 0) + w.hidden * 2
        return sum((u + 1) * self.stride + router + act for u in uniq)

    def gateup_bytes(self, uniq):
        """Algorithmic bytes of the gate/up kernels of one step: gate and up codes + scales/biases
        of every distinct selected expert and the shared expert, and x."""
        w = self.w
        per = 2 * w.inter * w.hidden * w.bits // 8 + 4 * w.inter * (w.hidden // 64) * 2
        return sum((u + 1) * per + self.T * w.hidden * 2 for u in uniq)


def run_decode(args, w, T, device, rank, ws_n):
    from int4_expert_gemv_router_b200 import abi, build
    build.build()
    K, W = args.steps, args.warmup
    st = DecodeStack(w, T, device, n_inputs=K + W, rank=rank)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize(device)
    # capture one step (all layers) into a CUDA graph
    with torch.cuda.stream(stream):
        st.layer_calls()  # warm (sets kernel attributes outside capture)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    graph_ok = True
    try:
        with torch.cuda.graph(g, stream=stream):
            st.layer_calls()
    except Exception as ex:  # capture of the cooperative launch not available: launch eagerly
        graph_ok = False
        print(f"graph capture failed ({ex}); launching eagerly", file=sys.stderr)
        torch.cuda.synchronize(device)
    gpu_launches_per_step = 1  # the whole stack is one persistent kernel

    def step(i):
        st.bufs[0].copy_(st.inputs[i], non_blocking=True)
        if graph_ok:
            g.replay()
        else:
            st.layer_calls()

    with torch.cuda.stream(stream):
        for i in range(W):
            step(i)
    stream.synchronize()
    barrier(device)
    torch.cuda.synchronize(device)
    clk = ClockSampler(device.index)
    clk.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(K):
            step(W + i)
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize(device)
    clocks = clk.stop()
    barrier(device)
    ms = e0.elapsed_time(e1)
    ms_max = reduce_max(ms, device)
    uniq = st.unique_experts()
    flags = abi.moe_ws_check(st.ws, stream)

    # kernel duration: the same step, eager, with the library's profiling hook recording
    # events on the launching stream around its kernel launch(es).  A GPU sleep issued first
    # lets the host enqueue the step before the device reaches it.
    n_k = 3
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n_k)]
    for ev in evs:  # torch creates the CUDA event lazily, on its first record
        ev.record(stream)
    descs = st.descs()
    kern_ms = {0: [], 1: [], 2: []}
    for r in range(5):
        with torch.cuda.stream(stream):
            st.bufs[0].copy_(st.inputs[r % (K + W)], non_blocking=True)
            torch.cuda._sleep(20_000_000)
            abi.moe_profile_events(evs, n_k)
            abi.moe_stack_forward(st.shape, T, descs, st.ws)
            abi.moe_profile_events(None)
        stream.synchronize()
        kern_ms[0].append(event_ms(evs[0], evs[1]))
    kern_avg_us = {kk: 1e3 * statistics.mean(v) for kk, v in kern_ms.items() if v}

    # end to end through the public call with host buffers: pinned H2D of the token(s),
    # the step, D2H of the result, every step
    x_host = st.inputs.cpu().pin_memory()
    out_host = torch.empty(T, w.hidden, dtype=torch.bfloat16).pin_memory()
    barrier(device)
    torch.cuda.synchronize(device)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for i in range(K):
            st.bufs[0].copy_(x_host[(W + i) % (K + W)], non_blocking=True)
            if graph_ok:
                g.replay()
            else:
                st.layer_calls()
            out_host.copy_(st.bufs[-1], non_blocking=True)
        f1.record(stream)
    f1.synchronize()
    e2e_ms = reduce_max(f0.elapsed_time(f1), device)

    res = dict(graph=graph_ok, ms=ms_max, clocks=clocks, uniq=uniq, flags=flags, kern_us=kern_avg_us, e2e_ms=e2e_ms,
               gpu_launches=gpu_launches_per_step * K, step_bytes=st.step_bytes(uniq),
               gateup_bytes=st.gateup_bytes(uniq), stack=st)
    return res


def run_ep(args, w, T, device, rank, world):
    """Expert-parallel layer stack: rank r holds the experts e % world == r of every layer
    (its pool shard), router and shared expert replicated; per layer the partial forward (the
    fused decode kernel for T <= 8, the prefill path above that), one NCCL sum all-reduce of
    the [T, H] fp32 partials, and the combine kernel.  All ranks work on the same tokens, so
    the job's tokens per step are T (strong scaling)."""
    from int4_expert_gemv_router_b200 import abi, build, ep
    build.build()
    K, W = args.steps, args.warmup
    shape = abi.shape_of(w)
    E, nL = w.n_experts, w.layers
    mine = ep.local_experts(E, rank, world)
    stride = synth.blob_stride(w.hidden, w.inter, w.bits)
    pool_all = torch.empty(nL * len(mine), stride, dtype=torch.uint8, device=device)
    table = ep.local_slot_table(E, rank, world, device)
    layers = []
    for l in range(nL):
        pool = pool_all[l * len(mine):(l + 1) * len(mine)]
        synth.make_blobs(w, l, mine, device, out=pool)
        shared = synth.make_blobs(w, l, [0], device, shared=True)[0]
        wr, b, wsg = synth.router_weights(w, l, device)
        layers.append(ep.EPLayer(shape, wr, b, pool, table, shared, wsg, rank, world, T, device))
    bufs = [torch.zeros(T, w.hidden, dtype=torch.bfloat16, device=device) for _ in range(nL + 1)]
    inputs = torch.stack([synth.activations(w, rank_step_seed(0, s), tokens=T, device=device) for s in range(K + W)])
    stream = torch.cuda.current_stream(device)
    torch.cuda.synchronize(device)

    def step(i):
        bufs[0].copy_(inputs[i], non_blocking=True)
        for l, Ly in enumerate(layers):
            Ly.forward(bufs[l], bufs[0], bufs[l + 1])

    for i in range(W):
        step(i)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    clk = ClockSampler(device.index)
    clk.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        step(W + i)
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize(device)
    clocks = clk.stop()
    barrier(device)
    ms = reduce_max(e0.elapsed_time(e1), device)
    flags = max(abi.moe_ws_check(Ly.ws) for Ly in layers)
    x_host = inputs.cpu().pin_memory()
    out_host = torch.empty(T, w.hidden, dtype=torch.bfloat16).pin_memory()
    barrier(device)
    torch.cuda.synchronize(device)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(K):
        bufs[0].copy_(x_host[(W + i) % (K + W)], non_blocking=True)
        for l, Ly in enumerate(layers):
            Ly.forward(bufs[l], bufs[0], bufs[l + 1])
        out_host.copy_(bufs[-1], non_blocking=True)
    f1.record(stream)
    f1.synchronize()
    e2e_ms = reduce_max(f0.elapsed_time(f1), device)
    value = T * K / (ms / 1e3)
    return {
        "metric": ("routed-MoE layer tokens/s; tensor % (prefill)" if w.name == "prefill"
                   else "routed-MoE layer tokens/s; achieved HBM GB/s (decode)"),
        "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms / K, 4), "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": f"int{w.bits} weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded; weights ~N(0,0.02) quantised, x ~N(0,1))",
        "config": dict(workload_config(args, w, T, world), parallelism=f"ep{world}"),
        "launch": ("per call: the prefill path over this rank's experts (fp32 partial), NCCL all-reduce, "
                   "combine kernel" if w.name == "prefill" else
                   "per layer: partial kernel, NCCL all-reduce of the fp32 partial, combine kernel"),
        "clocks": clocks,
        "e2e": {"value": round(T * K / (e2e_ms / 1e3), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": T * w.hidden * 2, "d2h_bytes_per_step": T * w.hidden * 2},
        "gpu_launches": (12 if w.name == "prefill" else 2) * nL * K,
        "device_error_flags": flags,
    }


# ======================================================================================
# Gated DeltaNet decode step (the linear-attention layers' recurrence)
# ======================================================================================
def run_gdn(args, name, device, rank):
    """One step = one token of B sequences through the recurrence of every linear-attention
    layer (36 launches, one per layer, in a CUDA graph; each layer has its own resident fp32
    state and its own seeded q/k/v/gates).  Per-launch durations come from an eager pass with
    events around each launch."""
    from int4_expert_gemv_router_b200 import abi, build
    build.build()
    c = synth.GDN_WORKLOADS[name]
    Hk, Hv, dk, dv, nL, B = c["n_k_heads"], c["n_v_heads"], c["d_k"], c["d_v"], c["layers"], c["batch"]
    K, W = args.steps, args.warmup
    shape = abi.moe_gdn_shape(Hk, Hv, dk, dv)
    states = [synth.gdn_state(Hv, dk, dv, B, c["seed"] + 1000 * rank + l, device) for l in range(nL)]
    ins = [synth.gdn_inputs(Hk, Hv, dk, dv, B, 1, c["seed"] + 1000 * rank + 100 + l, device) for l in range(nL)]
    ins = [tuple(t[0].contiguous() for t in x) for x in ins]
    # every layer's q, k, v, g, beta as views of one flat byte buffer (two of them, for the
    # end-to-end pipeline), and every layer's output as a slice of one [layers, B, Hv, dv] tensor
    sizes = [t.numel() * t.element_size() for t in ins[0]]
    per_layer = sum((n + 15) // 16 * 16 for n in sizes)
    flat = [torch.empty(nL * per_layer, dtype=torch.uint8, device=device) for _ in range(2)]

    def views(buf):
        res = []
        for l in range(nL):
            off, vs = l * per_layer, []
            for t, n in zip(ins[l], sizes):
                vs.append(buf[off:off + n].view(t.dtype).view(t.shape))
                off += (n + 15) // 16 * 16
            res.append(tuple(vs))
        return res

    ins_b = [views(flat[0]), views(flat[1])]
    for b in range(2):
        for l in range(nL):
            for dst, src in zip(ins_b[b][l], ins[l]):
                dst.copy_(src)
    ins = ins_b[0]
    outs_b = [torch.empty(nL, B, Hv, dv, dtype=torch.bfloat16, device=device) for _ in range(2)]
    outs = outs_b[0]
    stream = torch.cuda.Stream(device)

    def layer_calls(b=0):
        # each layer's step reads its own state early, while the previous layer finishes
        # (consecutive layers never share a state)
        for l in range(nL):
            q, k, v, g, beta = ins_b[b][l]
            abi.moe_gdn_decode_step(shape, B, states[l], q, k, v, g, beta, outs_b[b][l], flags=abi.MOE_GDN_EARLY_STATE)

    with torch.cuda.stream(stream):
        layer_calls()
    stream.synchronize()
    g_ = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_, stream=stream):
        layer_calls()
    with torch.cuda.stream(stream):
        for _ in range(W):
            g_.replay()
    stream.synchronize()
    barrier(device)
    clk = ClockSampler(device.index)
    clk.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(K):
            g_.replay()
        e1.record(stream)
    e1.synchronize()
    clocks = clk.stop()
    ms = reduce_max(e0.elapsed_time(e1), device)
    # per-launch duration on the launching stream (a GPU sleep first, so the launches queue up)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nL)]
    with torch.cuda.stream(stream):
        torch.cuda._sleep(20_000_000)
        for l in range(nL):
            q, k, v, g, beta = ins[l]
            evs[l][0].record(stream)
            abi.moe_gdn_decode_step(shape, B, states[l], q, k, v, g, beta, outs[l])
            evs[l][1].record(stream)
    stream.synchronize()
    launch_us = 1e3 * statistics.mean(a.elapsed_time(b) for a, b in evs)
    # end to end: every step's inputs of all layers come up from pinned host memory in one copy
    # and all outputs go back in one, pipelined over two buffer sets (one graph per set)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        layer_calls(1)
    graphs = [g_, g2]
    host_in = flat[0].cpu().pin_memory()
    host_out = [torch.empty(nL, B, Hv, dv, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    barrier(device)
    e2e_ms = pipelined_e2e(device, stream, K, lambda i, b: flat[b].copy_(host_in, non_blocking=True),
                           lambda i, b: graphs[b].replay(),
                           lambda i, b: host_out[b].copy_(outs_b[b], non_blocking=True))
    in_bytes = per_layer  # the flat upload, padding included
    return dict(c=c, ms=ms, clocks=clocks, launch_us=launch_us, e2e_ms=e2e_ms, in_bytes=in_bytes * nL,
                out_bytes=nL * B * Hv * dv * 2, state=states[0], ins=ins[0])


def cpu_baseline_gdn(r, budget_s=10.0):
    """The fp64 oracle as it stands: one sequence's step through layers until ~budget_s, scaled."""
    import oracle
    c = r["c"]
    q, k, v, g, beta = (t[0].float().double().cpu().numpy() for t in r["ins"])
    S = r["state"][0].double().cpu().numpy()
    t_total, n = 0.0, 0
    while t_total < budget_s and n < 10 * c["layers"]:
        t0 = time.perf_counter()
        oracle.gdn_step(S, q, k, v, g, beta)
        t_total += time.perf_counter() - t0
        n += 1
    per_layer = t_total / n
    return {"value": round(1.0 / (per_layer * c["layers"]), 3), "unit": "tokens/s", "cores": cpu_threads(),
            "kind": "oracle", "sample": f"{n} single-sequence layer steps (fp64 numpy oracle, {per_layer * 1e3:.1f} ms "
                                        f"each), scaled to a {c['layers']}-layer token"}


def run_reference_gdn(args, name):
    """Reference arm of the Gated DeltaNet workloads: the fp64 oracle as it stands on the host
    cores; each step is one token of one sequence through one layer's recurrence (cycling over
    the layers' seeded inputs), scaled to the workload's tokens/s."""
    import oracle
    c = synth.GDN_WORKLOADS[name]
    K, W = args.steps, args.warmup
    times = []
    for s_ in range(W + K):
        l = s_ % c["layers"]
        q, k, v, g, beta = (t[0, 0].double().numpy() for t in synth.gdn_inputs(
            c["n_k_heads"], c["n_v_heads"], c["d_k"], c["d_v"], 1, 1, c["seed"] + 100 + l))
        S = synth.gdn_state(c["n_v_heads"], c["d_k"], c["d_v"], 1, c["seed"] + l)[0].double().numpy()
        t0 = time.perf_counter()
        oracle.gdn_step(S, q, k, v, g, beta)
        if s_ >= W:
            times.append(time.perf_counter() - t0)
    per = statistics.mean(times)
    value = 1.0 / (per * c["layers"])
    return {"impl": "reference", "metric": "Gated DeltaNet decode-step tokens/s; achieved HBM GB/s",
            "value": round(value, 3), "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": round(per * 1e3, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": name, "n_k_heads": c["n_k_heads"], "n_v_heads": c["n_v_heads"], "d_k": c["d_k"],
                       "d_v": c["d_v"], "layers": c["layers"], "sequences": c["batch"], "parallelism": "replicas1"},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"each step: one sequence's token through one layer (fp64 numpy oracle, "
                                       f"{per * 1e3:.1f} ms measured), scaled to a {c['layers']}-layer token"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def gdn_line(args, name, r, n_gpus, peaks, peak_kind, cpu_base):
    c = r["c"]
    K = args.steps
    B, nL = c["batch"], c["layers"]
    per_launch = 2 * 4 * B * c["n_v_heads"] * c["d_v"] * c["d_k"] + 2 * B * (2 * c["n_k_heads"] * c["d_k"] +
                                                                             2 * c["n_v_heads"] * c["d_v"]) + 8 * B * c["n_v_heads"]
    hbm = peaks["hbm_gbs"]
    # average duration of one launch inside the timed region: the graph's time per step over
    # its launches (the gaps between back-to-back launches included)
    launch_us = r["ms"] * 1e3 / K / nL
    achieved = per_launch / (launch_us * 1e-6) / 1e9
    line = {
        "metric": "Gated DeltaNet decode-step tokens/s; achieved HBM GB/s",
        "value": round(n_gpus * B * K / (r["ms"] / 1e3), 1), "unit": "tokens/s", "n_gpus": n_gpus, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(r["ms"] / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp32 state, bf16 q/k/v/out", "data": "synthetic (seeded)",
        "config": {"workload": name, "n_k_heads": c["n_k_heads"], "n_v_heads": c["n_v_heads"], "d_k": c["d_k"],
                   "d_v": c["d_v"], "layers": nL, "sequences": B, "parallelism": f"replicas{n_gpus}",
                   "l2": f"{nL * B * c['n_v_heads'] * c['d_v'] * c['d_k'] * 4 / 1e6:.0f} MB of state per step"},
        "roofline": {"bound": "hbm", "kernel": "k_gdn_step (one layer)", "achieved": round(achieved, 1), "peak": hbm,
                     "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": None,
                     "launch_us": round(launch_us, 3), "launch_us_isolated": round(r["launch_us"], 3),
                     "bytes_per_launch": per_launch, "peak_kind": f"{peak_kind} hbm_gbs (burst copy)"},
        "clocks": r["clocks"],
        "e2e": {"value": round(n_gpus * B * K / (r["e2e_ms"] / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": r["in_bytes"], "d2h_bytes_per_step": r["out_bytes"],
                "copies": "one upload and one download per step (all layers), two buffer sets, on copy "
                          "streams overlapping the neighbouring steps"},
        "gpu_launches": nL * K,
    }
    if cpu_base is not None:
        line["cpu_baseline"] = cpu_base
    return line


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def cpu_baseline_decode(w, T, device, stack, budget_s=12.0):
    """The fp64 oracle as it stands, on host cores, on a bounded sample: the first step's
    token(s) through as many layers as fit in ~budget_s, scaled to tokens/s of the full stack.
    Copying the layer's bytes to the host is not timed."""
    import oracle
    x = stack.inputs[0]
    x0b = _bits(x)
    t_total, n = 0.0, 0
    for l in range(w.layers):
        L = stack.layers[l]
        xb, wr, wsg = _bits(x), _bits(L.w_router), _bits(L.w_sg)
        b = None if L.router_bias is None else L.router_bias.cpu().numpy()
        shared = L.shared.cpu().numpy()
        pre, _ = oracle.route(oracle.router_logits(xb, wr, b), w.top_k)
        blobs = {int(e): L.pool[int(e)].cpu().numpy() for e in set(pre.reshape(-1).tolist())}
        t0 = time.perf_counter()
        r = oracle.layer_forward(xb, wr, b, w.top_k, lambda e: blobs[e], shared, wsg, w.hidden, w.inter,
                                 w.shared_inter, w.bits, residual_bits=x0b)
        t_total += time.perf_counter() - t0
        n += 1
        x = torch.from_numpy(oracle.f64_to_bf16_bits(r["out"]).view(np.int16)).view(torch.bfloat16).to(device)
        if t_total > budget_s:
            break
    per_layer = t_total / n
    return {"value": round(T / (per_layer * w.layers), 4), "unit": "tokens/s", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": f"{T} token(s) through {n} of {w.layers} layers (fp64 numpy oracle, "
                      f"{per_layer * 1e3:.0f} ms/layer), scaled to the {w.layers}-layer step"}


def workload_config(args, w, T, n_gpus):
    """The `config` object of a result line: the workload alone, identical in both arms."""
    cfg = {"workload": w.name, "hidden": w.hidden, "n_experts": w.n_experts, "top_k": w.top_k,
           "inter": w.inter, "shared_inter": w.shared_inter, "bits": w.bits, "group": 64,
           "router": w.router, "parallelism": f"replicas{n_gpus}"}
    if w.name.startswith("pool"):
        cfg.update({"tokens_per_step": 1, "layers": 1, "n_slots": w.n_slots, "slot_fraction": w.n_slots / w.n_experts,
                    "steps_total": max(1024, args.steps + args.warmup),
                    "policy": {"lfu_recency": "LFU + recency", "lru": "LRU", "lfu": "LFU"}[args.policy],
                    "miss_path": {"host": "pinned host -> cudaMemcpyAsync on a side stream",
                                  "file": "pread from a file -> pinned staging -> cudaMemcpyAsync",
                                  "file_direct": "O_DIRECT pread from a file -> pinned staging -> cudaMemcpyAsync"}[
                                      getattr(args, "store", "host")],
                    "overlap": bool(args.overlap),
                    "l2": "one layer; misses come over PCIe, hits from the slot pool"})
    elif w.name == "prefill":
        cfg.update({"tokens_per_call": T, "layers": 1,
                    "l2": "inputs exceed L2 (906 MB of expert blobs per call)"})
    else:
        cfg.update({"tokens_per_step": T, "layers": w.layers,
                    "l2": "inputs exceed L2 (>1 GB distinct blobs per step)"})
    return cfg


def decode_line(args, w, T, r, n_gpus, peaks, peak_kind, cpu_base):
    K = args.steps
    tok = T * K * n_gpus
    value = tok / (r["ms"] / 1e3)
    step_s = r["ms"] / 1e3 / K
    hbm = peaks["hbm_gbs"]
    k_us = r["kern_us"][0]
    k_bytes = r["step_bytes"]  # the fused kernel moves the whole step's bytes per launch
    achieved = k_bytes / (k_us * 1e-6) / 1e9
    line = {
        "metric": "routed-MoE layer tokens/s; achieved HBM GB/s (decode)",
        "value": round(value, 2), "unit": "tokens/s", "n_gpus": n_gpus, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(r["ms"] / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": f"int{w.bits} weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded; weights ~N(0,0.02) quantised, x ~N(0,1))",
        "config": workload_config(args, w, T, n_gpus),
        "launch": "one persistent kernel per step" + (" in a CUDA graph" if r["graph"] else ""),
        "hbm_step": {"bytes_per_step": r["step_bytes"], "achieved_gbs": round(r["step_bytes"] / step_s / 1e9, 1),
                     "frac_of_measured": round(r["step_bytes"] / step_s / 1e9 / hbm, 4),
                     "mean_distinct_experts_per_layer": round(float(np.mean(r["uniq"])), 2)},
        "roofline": {"bound": "hbm", "kernel": f"k_fused_decode (whole {w.layers}-layer step, one launch)",
                     "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "traffic": (NCU_TRAFFIC_PER_LAYER.get(("k_fused_decode", w.name, T), 0) * w.layers) or None,
                     "launch_us": round(k_us, 3), "bytes_per_launch": int(k_bytes),
                     "peak_kind": f"{peak_kind} hbm_gbs (burst copy)"},
        "clocks": r["clocks"],
        "e2e": {"value": round(tok / (r["e2e_ms"] / 1e3), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": T * w.hidden * 2, "d2h_bytes_per_step": T * w.hidden * 2},
        "gpu_launches": r["gpu_launches"],
        "device_error_flags": r["flags"],
    }
    if cpu_base is not None:
        line["cpu_baseline"] = cpu_base
    return line


# ======================================================================================
# prefill workload (many tokens in one call)
# ======================================================================================
def prefill_flops(w, T):
    """Algorithmic FLOPs of one call (padding excluded): router, routed experts, shared expert."""
    H, I, Is, E, k = w.hidden, w.inter, w.shared_inter, w.n_experts, w.top_k
    router = 2 * T * H * (E + 1)
    gateup = 2 * T * k * 2 * H * I + 2 * T * 2 * H * Is
    down = 2 * T * k * I * H + 2 * T * Is * H
    return router, gateup, down


def pipelined_e2e(device, stream, K, upload, compute, download):
    """Device time of K steps end to end, with two buffers each way: upload(i, b) copies step
    i's inputs from pinned host memory into device buffer b (b = i % 2), compute(i, b) runs the
    step on buffer b and download(i, b) copies its result back to pinned host memory.  Uploads
    run on one copy stream and downloads on another, so that step i + 1's upload and step
    i - 1's download overlap step i's compute; events keep a buffer from being overwritten
    before the step that reads it is done.  The timed region runs from before the first upload
    to after the last download."""
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    in_free, out_free = [f0, f0], [f0, f0]
    for i in range(K):
        b = i % 2
        up.wait_event(in_free[b])
        with torch.cuda.stream(up):
            upload(i, b)
        ready = torch.cuda.Event()
        ready.record(up)
        stream.wait_event(ready)
        stream.wait_event(out_free[b])
        with torch.cuda.stream(stream):
            compute(i, b)
        done = torch.cuda.Event()
        done.record(stream)
        in_free[b] = done
        down.wait_event(done)
        with torch.cuda.stream(down):
            download(i, b)
        read = torch.cuda.Event()
        read.record(down)
        out_free[b] = read
    stream.wait_event(out_free[0])
    stream.wait_event(out_free[1])
    f1.record(stream)
    f1.synchronize()
    return reduce_max(f0.elapsed_time(f1), device)


def run_prefill(args, w, T, device, rank):
    from int4_expert_gemv_router_b200 import abi, build
    build.build()
    K, W = args.steps, args.warmup
    L = synth.make_layer(w, 0, device)
    shape = abi.shape_of(w)
    n_in = 3
    xs = [synth.activations(w, rank_step_seed(rank, s), tokens=T, device=device) for s in range(n_in)]
    xbuf = torch.empty_like(xs[0])
    out = torch.empty(T, w.hidden, dtype=torch.bfloat16, device=device)
    idx = torch.empty(T, w.top_k, dtype=torch.int32, device=device)
    p = torch.empty(T, w.top_k, dtype=torch.float32, device=device)
    slots = torch.arange(w.n_experts, dtype=torch.int32, device=device)
    ws = torch.zeros(abi.moe_workspace_size(shape, T), dtype=torch.uint8, device=device)
    stream = torch.cuda.Stream(device)

    def call():
        abi.moe_layer_forward(shape, xbuf, T, L.w_router, L.router_bias, None, None, L.pool, slots, w.n_experts,
                              L.shared, L.w_sg, xbuf, out, idx, p, ws)

    def step(i):
        xbuf.copy_(xs[i % n_in], non_blocking=True)
        call()

    with torch.cuda.stream(stream):
        for i in range(W):
            step(i)
    stream.synchronize()
    barrier(device)
    clk = ClockSampler(device.index)
    clk.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(K):
            step(i)
        e1.record(stream)
    e1.synchronize()
    clocks = clk.stop()
    barrier(device)
    ms = reduce_max(e0.elapsed_time(e1), device)
    flags = abi.moe_ws_check(ws, stream)
    # per-kernel durations through the library's events hook (5 groups, see moe_profile_events)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
    for ev in evs:
        ev.record(stream)
    kern = [[] for _ in range(5)]
    for r in range(3):
        with torch.cuda.stream(stream):
            xbuf.copy_(xs[r % n_in], non_blocking=True)
            torch.cuda._sleep(20_000_000)
            abi.moe_profile_events(evs, 5)
            call()
            abi.moe_profile_events(None)
        stream.synchronize()
        for g in range(5):
            kern[g].append(event_ms(evs[2 * g], evs[2 * g + 1]))
    kern_us = [1e3 * statistics.mean(v) for v in kern]
    # end to end: every step's x comes up from pinned host memory and its output goes back,
    # as a serving loop runs it: two device buffers each way, step i + 1's upload and step
    # i - 1's download on two copy streams while step i computes
    x_host = [x.cpu().pin_memory() for x in xs]
    out_host = [torch.empty(T, w.hidden, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xb = [xbuf, torch.empty_like(xbuf)]
    ob = [out, torch.empty_like(out)]

    def call_on(b):
        abi.moe_layer_forward(shape, xb[b], T, L.w_router, L.router_bias, None, None, L.pool, slots, w.n_experts,
                              L.shared, L.w_sg, xb[b], ob[b], idx, p, ws)

    barrier(device)
    e2e_ms = pipelined_e2e(device, stream, K, lambda i, b: xb[b].copy_(x_host[i % n_in], non_blocking=True),
                           lambda i, b: call_on(b), lambda i, b: out_host[b].copy_(ob[b], non_blocking=True))
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=w.n_experts)
    return dict(ms=ms, clocks=clocks, flags=flags, kern_us=kern_us, e2e_ms=e2e_ms, layer=L, x=xs[0],
                tokens_per_expert=(float(counts.mean()), int(counts.min()), int(counts.max())))


def cpu_baseline_prefill(w, T, r, n_sample=32):
    """The fp64 oracle as it stands on host cores: routing and outputs of a seeded sample of
    the call's tokens (copies to the host not timed), scaled to tokens/s."""
    import oracle
    L = r["layer"]
    sample = np.sort(np.random.default_rng(0).choice(T, n_sample, replace=False))
    x = r["x"][torch.from_numpy(sample).to(r["x"].device)]
    xb, wr, wsg = _bits(x), _bits(L.w_router), _bits(L.w_sg)
    pre, _ = oracle.route(oracle.router_logits(xb, wr, None), w.top_k)
    blobs = {int(e): L.pool[int(e)].cpu().numpy() for e in set(pre.reshape(-1).tolist())}
    shared = L.shared.cpu().numpy()
    t0 = time.perf_counter()
    oracle.layer_forward(xb, wr, None, w.top_k, lambda e: blobs[e], shared, wsg, w.hidden, w.inter,
                         w.shared_inter, w.bits, residual_bits=xb)
    dt = time.perf_counter() - t0
    return {"value": round(n_sample / dt, 3), "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{n_sample} of the {T} tokens (seeded), routing + experts + shared expert, fp64 numpy "
                      f"oracle ({dt:.1f} s), scaled to tokens/s"}


def prefill_line(args, w, T, r, n_gpus, peaks, peak_kind, cpu_base):
    K = args.steps
    router_f, gu_f, dn_f = prefill_flops(w, T)
    total_f = router_f + gu_f + dn_f
    step_s = r["ms"] / 1e3 / K
    value = n_gpus * T * K / (r["ms"] / 1e3)
    peak = peaks["bf16_tflops"]
    gu_us = r["kern_us"][2]
    achieved = gu_f / (gu_us * 1e-6) / 1e12
    line = {
        "metric": "routed-MoE layer tokens/s; tensor % (prefill)",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": n_gpus, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(r["ms"] / K, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"int{w.bits} weights dequantised to bf16, bf16 x bf16 -> fp32 (tcgen05)",
        "data": "synthetic (seeded; weights ~N(0,0.02) quantised, x ~N(0,1))",
        "config": workload_config(args, w, T, n_gpus),
        "tokens_per_expert_mean_min_max": r["tokens_per_expert"],
        "tensor_step": {"flops_per_call": total_f, "achieved_tflops": round(total_f / step_s / 1e12, 1),
                        "frac_of_measured": round(total_f / step_s / 1e12 / peak, 4)},
        "roofline": {"bound": "tensor", "kernel": "k_gemm<GATEUP> (gate/up grouped GEMM + SwiGLU)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": NCU_TRAFFIC_PREFILL_GATEUP.get((w.name, T)),
                     "launch_us": round(gu_us, 2),
                     "flops_per_launch": gu_f, "peak_kind": f"{peak_kind} bf16_tflops (burst)"},
        "kernels_us": {"router+topk": round(r["kern_us"][0], 2), "group": round(r["kern_us"][1], 2),
                       "gateup_gemm": round(r["kern_us"][2], 2), "down_gemm": round(r["kern_us"][3], 2),
                       "finalize": round(r["kern_us"][4], 2)},
        "clocks": r["clocks"],
        "e2e": {"value": round(n_gpus * T * K / (r["e2e_ms"] / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": T * w.hidden * 2, "d2h_bytes_per_step": T * w.hidden * 2,
                "copies": "two buffers each way, uploads and downloads on copy streams overlapping the "
                          "neighbouring steps"},
        "gpu_launches": 8 * K,
        "device_error_flags": r["flags"],
    }
    if cpu_base is not None:
        line["cpu_baseline"] = cpu_base
    return line


# ======================================================================================
# bounded slot pool (25% of experts resident, LFU + recency, misses from pinned host)
# ======================================================================================
def run_pool(args, w, device, rank, total_steps=1024):
    """Decode steps of one layer through the bounded pool: router -> moe_expert_pool_load (reads
    the ids back, loads the misses on the pool's side stream) -> layer forward on the slots.
    W warm-up steps, then the timed steps; at least total_steps steps run for the hit rate."""
    from int4_expert_gemv_router_b200 import abi, build
    build.build()
    K, W = args.steps, args.warmup
    n_total = max(total_steps, K + W)
    L = synth.make_layer(w, 0, device)
    host_blobs = L.pool.cpu().pin_memory()
    stride = L.pool.shape[1]
    del L.pool
    torch.cuda.empty_cache()
    shape = abi.shape_of(w)
    dev_pool = torch.zeros(w.n_slots, stride, dtype=torch.uint8, device=device)
    table = torch.empty(w.n_experts, dtype=torch.int32, device=device)
    store_path = None
    if args.store == "host":
        pool = abi.moe_pool_create(shape, w.n_slots, host_blobs, dev_pool, table)
    else:
        # the storage tier: the blobs in a file, misses read with one pread each
        fd, store_path = tempfile.mkstemp(suffix=".blobs", dir=os.environ.get("MOE_STORE_DIR"))
        os.close(fd)
        host_blobs.numpy().tofile(store_path)
        pool = abi.moe_pool_create_file(shape, w.n_slots, store_path, dev_pool, table,
                                        direct=(args.store == "file_direct"))
    abi.moe_pool_set_policy(pool, args.policy)
    abi.moe_pool_set_overlap(pool, args.overlap)
    T = 1
    # n_total steps on device-resident inputs (warm-up, hit-rate steps, timed steps), then K
    # end-to-end steps on inputs of their own
    xs = torch.stack([synth.activations(w, rank_step_seed(rank, s), tokens=T, device=device)
                      for s in range(n_total + K)])
    out = torch.empty(T, w.hidden, dtype=torch.bfloat16, device=device)
    idx = torch.empty(T, w.top_k, dtype=torch.int32, device=device)
    p = torch.empty(T, w.top_k, dtype=torch.float32, device=device)
    ws = torch.zeros(abi.moe_workspace_size(shape, T), dtype=torch.uint8, device=device)
    stream = torch.cuda.Stream(device)
    popularity = np.zeros(w.n_experts, dtype=np.int64)

    def step(i):
        x = xs[i]
        abi.moe_router_topk(shape, x, T, L.w_router, L.router_bias, idx, p, ws)
        abi.moe_expert_pool_load(pool, idx, T)
        abi.moe_layer_forward(shape, x, T, L.w_router, L.router_bias, idx, p, dev_pool, table, w.n_slots,
                              L.shared, L.w_sg, x, out, None, None, ws)

    t_start = n_total - K
    with torch.cuda.stream(stream):
        for i in range(t_start):
            step(i)
            if i >= W:
                popularity[idx.cpu().numpy().reshape(-1)] += 1
    stream.synchronize()
    st0 = abi.moe_pool_stats(pool)
    barrier(device)
    clk = ClockSampler(device.index)
    clk.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(t_start, n_total):
            step(i)
        e1.record(stream)
    e1.synchronize()
    clocks = clk.stop()
    ms = reduce_max(e0.elapsed_time(e1), device)
    st1 = abi.moe_pool_stats(pool)
    flags = abi.moe_ws_check(ws, stream)
    # end to end: every step's x comes up from pinned host memory and its output goes back
    # (two device buffers each way, copies on two copy streams), the pool carrying on from
    # the timed steps
    x_host = xs[n_total:].cpu().pin_memory()
    xb = [torch.empty_like(xs[0]) for _ in range(2)]
    ob = [out, torch.empty_like(out)]
    out_host = [torch.empty(T, w.hidden, dtype=torch.bfloat16).pin_memory() for _ in range(2)]

    def step_on(b):
        abi.moe_router_topk(shape, xb[b], T, L.w_router, L.router_bias, idx, p, ws)
        abi.moe_expert_pool_load(pool, idx, T)
        abi.moe_layer_forward(shape, xb[b], T, L.w_router, L.router_bias, idx, p, dev_pool, table, w.n_slots,
                              L.shared, L.w_sg, xb[b], ob[b], None, None, ws)

    barrier(device)
    e2e_ms = pipelined_e2e(device, stream, K, lambda i, b: xb[b].copy_(x_host[i], non_blocking=True),
                           lambda i, b: step_on(b), lambda i, b: out_host[b].copy_(ob[b], non_blocking=True))
    flags |= abi.moe_ws_check(ws, stream)
    abi.moe_pool_destroy(pool)
    if store_path:
        os.unlink(store_path)
    hits = st1["hits"] - st0["hits"]
    look = st1["lookups"] - st0["lookups"]
    # Zipf exponent fitted to the measured popularity (log count vs log rank)
    cnt = np.sort(popularity)[::-1]
    cnt = cnt[cnt > 0]
    rk = np.arange(1, len(cnt) + 1)
    zipf_s = float(-np.polyfit(np.log(rk), np.log(cnt), 1)[0]) if len(cnt) > 2 else None
    L.shared_host = L.shared.cpu().numpy()
    return dict(ms=ms, clocks=clocks, flags=flags, K=K, n_total=n_total, stats=st1, e2e_ms=e2e_ms,
                io_bytes=T * w.hidden * 2,
                hit_rate_all=st1["hits"] / max(1, st1["lookups"]), hit_rate_timed=hits / max(1, look),
                h2d_timed=st1["h2d_bytes"] - st0["h2d_bytes"], zipf_s=zipf_s, stride=stride,
                layer=L, host_blobs=host_blobs, xs=xs[:64])


def cpu_baseline_pool(w, r, budget_s=10.0):
    """The fp64 oracle as it stands on host cores: one token per step through the layer (every
    expert readable from host memory, no pool), as many steps as fit in ~budget_s."""
    import oracle
    L = r["layer"]
    wr, wsg = _bits(L.w_router), _bits(L.w_sg)
    b = None if L.router_bias is None else L.router_bias.cpu().numpy()
    shared = L.shared_host
    t_total, n = 0.0, 0
    while t_total < budget_s and n < 200:
        xb = _bits(r["xs"][n % r["xs"].shape[0]])
        t0 = time.perf_counter()
        oracle.layer_forward(xb, wr, b, w.top_k, lambda e: r["host_blobs"][e].numpy(), shared, wsg, w.hidden,
                             w.inter, w.shared_inter, w.bits, residual_bits=xb)
        t_total += time.perf_counter() - t0
        n += 1
    return {"value": round(n / t_total, 4), "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{n} decode steps (one token through the layer, fp64 numpy oracle, "
                      f"{1e3 * t_total / n:.0f} ms/step), all experts in host memory"}


def pool_line(args, w, r, n_gpus, cpu_base=None):
    K = r["K"]
    value = n_gpus * K / (r["ms"] / 1e3)
    line = {
        "metric": "routed-MoE layer tokens/s with a bounded slot pool; expert-cache hit rate",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": n_gpus, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(r["ms"] / K, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"int{w.bits} weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded; Zipf(1.0) router bias)",
        "config": workload_config(args, w, 1, n_gpus),
        "timing": "events around the timed steps; each step waits on the host for the ids",
        "pool": {"hit_rate_all_steps": round(r["hit_rate_all"], 4), "hit_rate_timed": round(r["hit_rate_timed"], 4),
                 "stats": r["stats"], "h2d_bytes_timed": r["h2d_timed"],
                 "h2d_gbs_timed": round(r["h2d_timed"] / (r["ms"] / 1e3) / 1e9, 2),
                 "fitted_zipf_s": None if r["zipf_s"] is None else round(r["zipf_s"], 3)},
        "clocks": r["clocks"],
        "e2e": {"value": round(n_gpus * K / (r["e2e_ms"] / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": r["io_bytes"], "d2h_bytes_per_step": r["io_bytes"],
                "note": "x uploaded from pinned host memory and the output read back every step; the "
                        "library's own read-back of the ids and copies of the misses are inside the timing too"},
        "gpu_launches": 6 * K,
        "device_error_flags": r["flags"],
    }
    if cpu_base is not None:
        line["cpu_baseline"] = cpu_base
    return line


# --------------------------------------------------------------------------------------
# reference arm: the fp64 oracle on host cores
# --------------------------------------------------------------------------------------
def run_reference(args, w, T):
    """The reference arm: the fp64 oracle as it stands, timed on the host cores.  Each step is
    a bounded sample of the workload: decode -- the step's T token(s) through one layer
    (cycling over the first four layers), tokens/s scaled to the whole stack; prefill -- 32
    seeded tokens of the call through the layer; pool -- one decode token through the layer.
    ms_per_step is the time the timed steps actually took."""
    import oracle
    rank, _, n_ranks = dist_env()
    if rank != 0:
        return None
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    K, W = args.steps, args.warmup
    layers = {}

    def layer(l):
        if l not in layers:
            L = synth.make_layer(w, l, dev)
            layers[l] = dict(wr=L.w_router.cpu(), b=None if L.router_bias is None else L.router_bias.cpu().numpy(),
                             wsg=L.w_sg.cpu(), shared=L.shared.cpu().numpy(), pool=L.pool)
        return layers[l]

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    prefill = w.name == "prefill"
    n_tok = 32 if prefill else (1 if w.name.startswith("pool") else T)
    times = []
    for s in range(W + K):
        l = 0 if (prefill or w.name.startswith("pool")) else s % min(w.layers, 4)
        d = layer(l)
        if prefill:
            x = synth.activations(w, rank_step_seed(0, s % 3), tokens=T, device=dev)
            sel = np.sort(np.random.default_rng(s).choice(T, n_tok, replace=False))
            x = x[torch.from_numpy(sel).to(dev)].cpu()
        else:
            x = synth.activations(w, rank_step_seed(0, s), tokens=n_tok, device=dev).cpu()
        logits = oracle.router_logits(bits(x), bits(d["wr"]), d["b"])
        idx, _ = oracle.route(logits, w.top_k)
        blobs = {int(e): d["pool"][int(e)].cpu().numpy() for e in set(idx.reshape(-1).tolist())}
        t0 = time.perf_counter()
        oracle.layer_forward(bits(x), bits(d["wr"]), d["b"], w.top_k, lambda e: blobs[e], d["shared"], bits(d["wsg"]),
                             w.hidden, w.inter, w.shared_inter, w.bits, residual_bits=bits(x))
        dt = time.perf_counter() - t0
        if s >= W:
            times.append(dt)
    per_step = statistics.mean(times)
    if prefill:
        value = n_tok / per_step
        sample = (f"each step: {n_tok} seeded tokens of the {T}-token call through the layer (fp64 numpy oracle, "
                  f"{per_step * 1e3:.0f} ms), scaled to tokens/s")
        metric = "routed-MoE layer tokens/s; tensor % (prefill)"
    elif w.name.startswith("pool"):
        value = 1.0 / per_step
        sample = (f"each step: one token through the layer (fp64 numpy oracle, {per_step * 1e3:.0f} ms), "
                  f"every expert in host memory")
        metric = "routed-MoE layer tokens/s with a bounded slot pool; expert-cache hit rate"
    else:
        value = T / (per_step * w.layers)
        sample = (f"each step: {T} token(s) through one layer (cycling layers 0-3) with the fp64 numpy oracle "
                  f"({per_step * 1e3:.0f} ms measured per step); tokens/s scaled to the {w.layers}-layer stack")
        metric = "routed-MoE layer tokens/s; achieved HBM GB/s (decode)"
    return {"impl": "reference", "metric": metric,
            "value": round(value, 4), "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": round(per_step * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": workload_config(args, w, T, n_ranks),
            "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------------------------
def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode80b",
                    choices=["decode80b", "decode35b", "prefill", "pool_int4", "pool_int8", "gdn80b", "gdn80b_b8"])
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--policy", choices=["lfu_recency", "lru", "lfu"], default="lfu_recency",
                    help="pool workloads: eviction policy (the pages' LFU + recency by default)")
    ap.add_argument("--slots", type=int, default=None, help="pool workloads: number of slots (default 128)")
    ap.add_argument("--store", choices=["host", "file", "file_direct"], default="host",
                    help="pool workloads: where misses come from (pinned host memory, or a file read with pread)")
    ap.add_argument("--overlap", action="store_true",
                    help="pool workloads: the forward starts while the step's misses are still being copied")
    ap.add_argument("--parallel", choices=["replicas", "ep"], default="replicas",
                    help="decode and prefill workloads with --gpus N: N independent replicas (default, weak "
                         "scaling) or expert parallelism (each rank holds 1/N of every layer's experts, strong "
                         "scaling)")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the stack depth (profiling of a small case only; not a bench value)")
    return ap.parse_args(argv)


def main_gdn(args):
    rank, local, n_ranks = dist_env()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference_gdn(args, args.workload)), flush=True)
        return 0
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist("nccl")
    peaks, peak_kind = load_peaks()
    r = run_gdn(args, args.workload, device, rank)
    cpu_base = cpu_baseline_gdn(r) if (rank == 0 and n_ranks == 1 and not args.no_cpu_baseline) else None
    line = gdn_line(args, args.workload, r, n_ranks, peaks, peak_kind, cpu_base)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.workload.startswith("gdn"):
        return main_gdn(args)
    w = synth.WORKLOADS[args.workload]
    if args.layers:
        w = w.with_(layers=args.layers)
    if args.slots and w.name.startswith("pool"):
        w = w.with_(n_slots=args.slots)
    T = args.tokens or w.tokens
    if args.impl == "reference":
        line = run_reference(args, w, T)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    rank, local, ws = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist("nccl")
    peaks, peak_kind = load_peaks()
    cpu_base = None
    want_cpu = rank == 0 and ws == 1 and not args.no_cpu_baseline
    if args.parallel == "ep" and not w.name.startswith("pool"):
        line = run_ep(args, w, T, device, rank, ws)
    elif w.name == "prefill":
        r = run_prefill(args, w, T, device, rank)
        if want_cpu:
            cpu_base = cpu_baseline_prefill(w, T, r)
        line = prefill_line(args, w, T, r, ws, peaks, peak_kind, cpu_base)
    elif w.name.startswith("pool"):
        r = run_pool(args, w, device, rank)
        if want_cpu:
            cpu_base = cpu_baseline_pool(w, r)
        line = pool_line(args, w, r, ws, cpu_base)
    else:
        r = run_decode(args, w, T, device, rank, ws)
        if want_cpu:
            cpu_base = cpu_baseline_decode(w, T, device, r["stack"])
        line = decode_line(args, w, T, r, ws, peaks, peak_kind, cpu_base)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
