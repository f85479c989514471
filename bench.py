#!/usr/bin/env python3
"""Benchmark of the routed-MoE layer forward on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode80b|decode35b|pool_int4|pool_int8]
                    [--tokens T] [--impl ours|reference]

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
needed between steps.  With N > 1 every rank runs an independent replica (weak scaling;
the path has no exchange step).  Rank 0 prints one JSON line.
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

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per layer-token of the kernel the
# bench times, from the ncu capture summarised in profiles/k_fused_decode_decode80b_2layer_full.md
# (2-layer case, scaled by layers).  Must be re-captured whenever the kernel changes.
NCU_TRAFFIC_PER_LAYER = {("k_fused_decode", "decode80b", 1): 21_639_120}


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
        "config": {"workload": w.name, "hidden": w.hidden, "n_experts": w.n_experts, "top_k": w.top_k,
                   "inter": w.inter, "shared_inter": w.shared_inter, "bits": w.bits, "group": 64,
                   "tokens_per_step": T, "layers": w.layers, "router": w.router,
                   "parallelism": f"replicas{n_gpus}", "l2": "inputs exceed L2 (>1 GB distinct blobs per step)",
                   "launch": "one persistent kernel per step" + (" in a CUDA graph" if r["graph"] else "")},
        "hbm_step": {"bytes_per_step": r["step_bytes"], "achieved_gbs": round(r["step_bytes"] / step_s / 1e9, 1),
                     "frac_of_measured": round(r["step_bytes"] / step_s / 1e9 / hbm, 4),
                     "mean_distinct_experts_per_layer": round(float(np.mean(r["uniq"])), 2)},
        "roofline": {"bound": "hbm", "kernel": "k_fused_decode (whole 48-layer step, one launch)",
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


# --------------------------------------------------------------------------------------
# reference arm: the fp64 oracle on host cores
# --------------------------------------------------------------------------------------
def run_reference(args, w, T):
    import oracle
    rank, _, ws = dist_env()
    if rank != 0:
        return None
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    K, W = args.steps, args.warmup
    # inputs: the same generator as our arm; only the sampled layer is materialised
    layers = {}

    def layer(l):
        if l not in layers:
            L = synth.make_layer(w, l, dev)
            layers[l] = dict(wr=L.w_router.cpu(), b=None if L.router_bias is None else L.router_bias.cpu().numpy(),
                             wsg=L.w_sg.cpu(), shared=L.shared.cpu().numpy(), pool=L.pool)
        return layers[l]

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    times = []
    for s in range(W + K):
        l = s % min(w.layers, 4)
        d = layer(l)
        x = synth.activations(w, rank_step_seed(0, s), tokens=T, device=dev).cpu()
        logits = oracle.router_logits(bits(x), bits(d["wr"]), d["b"])
        idx, _ = oracle.route(logits, w.top_k)
        blobs = {int(e): d["pool"][int(e)].cpu().numpy() for e in set(idx.reshape(-1).tolist())}
        t0 = time.perf_counter()
        oracle.layer_forward(bits(x), bits(d["wr"]), d["b"], w.top_k, lambda e: blobs[e], d["shared"], bits(d["wsg"]),
                             w.hidden, w.inter, w.shared_inter, w.bits, residual_bits=bits(x))
        dt = time.perf_counter() - t0
        if s >= W:
            times.append(dt)
    per_layer = statistics.mean(times)
    value = T / (per_layer * w.layers)
    sample = (f"each step: {T} token(s) through one layer (cycling layers 0-3) with the fp64 numpy oracle; "
              f"tokens/s scaled to the {w.layers}-layer stack")
    return {"impl": "reference", "metric": "routed-MoE layer tokens/s; achieved HBM GB/s (decode)",
            "value": round(value, 4), "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": round(per_layer * w.layers * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": w.name, "hidden": w.hidden, "n_experts": w.n_experts, "top_k": w.top_k,
                       "tokens_per_step": T, "layers": w.layers, "bits": w.bits},
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
    ap.add_argument("--workload", default="decode80b", choices=["decode80b", "decode35b"])
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the stack depth (profiling of a small case only; not a bench value)")
    return ap.parse_args(argv)


def main(argv=None):
    args = parse(argv)
    if args.warmup < 3:
        args.warmup = 3
    w = synth.WORKLOADS[args.workload]
    if args.layers:
        w = w.with_(layers=args.layers)
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
    r = run_decode(args, w, T, device, rank, ws)
    cpu_base = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
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
