"""Benchmark of the PBD window-attention path on B200.

One step = one PBD decode step of the workload: for every layer, the window K/V append and
the window attention (``la_pbd_step`` through the C ABI). Default workload: the long-context
batch (8 sequences, prefix 32768, window 6, 16 query / 2 KV heads, d = 128, per-sequence K
mean offset), seed 4, the largest of the target configurations; the other workloads are timed
in the sweep, each with its own roofline block.

Timing: inputs resident in HBM, several full copies of the workload rotated so that every step
reads data that is not in L2 (working set > 2 x L2); the step is captured in a CUDA graph; W
untimed warm-up steps; K timed steps between CUDA events on the launching stream with a
barrier and synchronize on both sides; max over ranks. `e2e` repeats the measurement through
the same C ABI with the step's inputs (Q, new K/V of every layer) copied from pinned host
memory and the output copied back inside the timed region (graph replays, copies on a second
stream); `e2e_eager` does the same with the C-ABI calls made eagerly inside the timed region
(no CUDA graph), as a caller without graphs would.

`algo_compare` times the attention call of every workload with each attention kernel (tcgen05
and CUDA cores) under the same protocol; the automatic kernel choice follows that table.

Multi-GPU: replicas only (each rank runs its own independent batch; no collective on the data
path; the timing uses one max-reduction).

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "PBD window-steps/sec and achieved HBM GB/s (% of B200 peak) vs prefix length"
UNIT = "window-steps/s"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# The sources the decode attention and merge kernels are compiled from (the stored traffic
# figures are theirs; the prefill kernel and the host code do not affect them).
DECODE_SOURCES = ("attn_tc.cu", "combine.cu", "pbd_common.cuh", "pbd_kernels.h", "tc_util.cuh",
                  "tma_util.h")


def kernel_sources_digest():
    """SHA-256 over the decode kernels' CUDA sources (order fixed), to tell whether a stored
    ncu traffic figure was taken on the kernels that run now."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_masked_window_b200", "csrc")
    for name in DECODE_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def stored_traffic(workload):
    """DRAM bytes per attention call measured by ncu (dram__bytes_read.sum +
    dram__bytes_write.sum of the attention and merge kernels of one call), from
    profiles/traffic.json, if it was taken on the current sources and this workload."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f)
        if d.get("sources_sha256") != kernel_sources_digest():
            return None
        e = d["workloads"].get(workload)
        return None if e is None else float(e["dram_bytes_per_call"])
    except Exception:
        return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- setup
def build_device_inputs(wi, copies, device):
    """Stack every layer's tensors and make `copies` independent copies on the device."""
    import torch
    L = len(wi.layers)
    stack = lambda name: torch.stack([getattr(li, name) for li in wi.layers])  # noqa: E731
    host = {n: stack(n) for n in ("q", "k_cache", "v_cache", "k_new", "v_new")}
    dev = []
    for c in range(copies):
        d = {n: t.to(device) for n, t in host.items()}
        d["out"] = torch.empty_like(d["q"])
        dev.append(d)
    seq = wi.seq_lens.to(device)
    return host, dev, seq, L


def run_step(bmw, cfg, d, seq, W, ws, L):
    for layer in range(L):
        bmw.la_pbd_step(cfg, d["q"][layer], d["k_new"][layer], d["v_new"][layer],
                        d["k_cache"][layer], d["v_cache"][layer], seq, W, d["out"][layer], ws)


def run_attn_only(bmw, cfg, d, seq, W, ws, L):
    for layer in range(L):
        bmw.la_pbd_attn(cfg, d["q"][layer], d["k_cache"][layer], d["v_cache"][layer], seq, W,
                        d["out"][layer], ws)


def capture(torch, fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm (kernel attributes, tensor-map encoder)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_graphs(torch, graphs, steps, warmup, barrier):
    # Every graph is replayed at least once before timing: a graph's first launch uploads it
    # to the device and would otherwise land in the timed region.
    for i in range(max(warmup, len(graphs))):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        graphs[i % len(graphs)].replay()
    end.record()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    return start.elapsed_time(end)


ALGO_NAMES = {1: "tcgen05", 2: "cuda_cores"}


def supported_algos(wl):
    """Attention kernels that take this workload: tcgen05 up to W * G = 80 query rows per KV
    head, the CUDA-core kernel up to 128."""
    R = wl.window * (wl.num_q_heads // wl.num_kv_heads)
    return [a for a, lim in ((1, 80), (2, 128)) if R <= lim]


def time_attention(args, bmw, torch, cfg_for, dev, seq, W, L, seq_of, ngraphs, inner, warmup,
                   steps, barrier, max_over_ranks, device):
    """Per-call time (us) of the attention call (attention + merge) of every layer, timed back
    to back over the rotating copies, for the configuration `cfg_for`."""
    ws = bmw.Workspace(cfg_for, W, device=device)
    graphs = [capture(torch, lambda ds=seq_of(i): [run_attn_only(bmw, cfg_for, d, seq, W, ws, L) for d in ds])
              for i in range(ngraphs)]
    reps = max(1, math.ceil(max(steps, 20) / inner))
    ms = max_over_ranks(time_graphs(torch, graphs, reps, warmup, barrier))
    if bmw.la_pbd_check(ws) != 0:
        raise RuntimeError("device-side status not OK after the attention timing")
    del graphs
    return ms * 1e3 / (reps * inner * L)


def measure(args, rank, world, device, bmw, torch, wl, barrier, max_over_ranks, e2e=True,
            compare=True):
    wi = workloads.generate(wl)
    B, W = wl.batch, wl.window
    per_copy = (2 * wi.layers[0].k_cache.numel() * 2 + 3 * wi.layers[0].q.numel() * 2) * len(wi.layers)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    copies = max(2, min(args.max_copies, math.ceil(2.5 * l2 / max(per_copy, 1))))
    host, dev, seq, L = build_device_inputs(wi, copies, device)
    make_cfg = lambda algo: bmw.Config.make(B, wl.num_q_heads, wl.num_kv_heads, wi.max_seq,  # noqa: E731
                                            algo=algo)
    cfg = make_cfg(args.algo)
    R = W * (wl.num_q_heads // wl.num_kv_heads)
    uses_tc = bmw.chosen_algo(cfg, W) == bmw.LA_ALGO_TCGEN05
    ws = bmw.Workspace(cfg, W, device=device)

    # One graph replay runs `inner` consecutive steps, each on the next copy in the rotation
    # (so every call still reads its inputs from HBM), so that workloads of a single layer
    # call are timed back to back like the 36 layer calls of a decode step, not one call per
    # graph launch.
    inner = max(d for d in range(1, max(1, math.ceil(8 / L)) + 1) if args.steps % d == 0)
    def seq_of(i):
        return [dev[(i * inner + j) % copies] for j in range(inner)]
    ngraphs = copies if inner == 1 else max(1, copies // math.gcd(copies, inner))
    step_graphs = [capture(torch, lambda ds=seq_of(i): [run_step(bmw, cfg, d, seq, W, ws, L) for d in ds])
                   for i in range(ngraphs)]
    steps, warmup = args.steps, args.warmup
    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    replays = steps // inner   # exactly `steps` steps
    ms = time_graphs(torch, step_graphs, replays, warmup, barrier)
    clk = clocks.stop()
    ms = max_over_ranks(ms)
    ms_per_step = ms / (replays * inner)
    value = aggregate_throughput(world, B, replays * inner, ms)

    # Launch floor: a graph of as many empty kernels as one replay of the step graph launches
    # (programmatic dependent launch, one CTA of 224 threads per SM), timed the same way.
    per_step_launches = L * (2 if uses_tc else 3)
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    floor_graph = capture(torch, lambda: bmw.la_noop_chain(inner * per_step_launches, sms, 224))
    ms_floor = max_over_ranks(time_graphs(torch, [floor_graph], replays, warmup, barrier))
    launch_floor = {"ms_per_step": ms_floor / (replays * inner),
                    "launches_per_step": per_step_launches,
                    "kernel": f"empty, programmatic dependent launch, {sms} CTAs x 224 threads"}
    del floor_graph

    # Dominant kernel: the attention call of one layer (attention + split merge), timed alone
    # over the same rotating copies, with the kernel the step used; then every supported
    # kernel, forced, for the comparison table.
    launch_us = time_attention(args, bmw, torch, cfg, dev, seq, W, L, seq_of, ngraphs, inner,
                               warmup, steps, barrier, max_over_ranks, device)
    algo_us = {}
    if compare:
        for a in supported_algos(wl):
            algo_us[ALGO_NAMES[a]] = time_attention(args, bmw, torch, make_cfg(a), dev, seq, W, L,
                                                    seq_of, ngraphs, inner, warmup, steps, barrier,
                                                    max_over_ranks, device)
    alg_bytes = workloads.algorithmic_bytes(wi.seq_lens.tolist(), W, wl.num_q_heads,
                                            wl.num_kv_heads, wl.head_dim)
    achieved = alg_bytes / (launch_us * 1e-6) / 1e9
    step_bytes = L * (alg_bytes + workloads.append_bytes(B, W, wl.num_kv_heads, wl.head_dim))
    if bmw.la_pbd_check(ws) != 0:
        raise RuntimeError("device-side status not OK after the benchmark")

    # End to end through the same API: inputs from pinned host memory, output back to host.
    e2e_res = e2e_eager = None
    if e2e:
        # One step per replay here: each step copies its own inputs in and its output out.
        one_step = step_graphs if inner == 1 else [
            capture(torch, lambda d=d: run_step(bmw, cfg, d, seq, W, ws, L)) for d in dev]
        h_in = {n: host[n].pin_memory() for n in ("q", "k_new", "v_new")}
        h_out = torch.empty_like(host["q"]).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in h_in.values())
        d2h = h_out.numel() * h_out.element_size()
        # Serving-loop pipelining: step i+1's inputs are copied in on a copy stream while step
        # i computes, and step i's output is read back while step i+1 computes. Every step
        # still moves its own inputs host -> device and its output device -> host inside the
        # timed region; a buffer is reused only after the step that last used it finished.
        comp_s, copy_s = torch.cuda.current_stream(), torch.cuda.Stream()
        in_ready = [torch.cuda.Event() for _ in range(copies)]
        done = [torch.cuda.Event() for _ in range(copies)]
        used = [False] * copies

        def upload(i):
            k = i % copies
            if used[k]:
                copy_s.wait_event(done[k])
            with torch.cuda.stream(copy_s):
                for n in h_in:
                    dev[k][n].copy_(h_in[n], non_blocking=True)
            in_ready[k].record(copy_s)
            used[k] = True

        def run(n_steps, graphed):
            upload(0)
            for i in range(n_steps):
                k = i % copies
                comp_s.wait_event(in_ready[k])
                if graphed:
                    one_step[k].replay()
                else:
                    run_step(bmw, cfg, dev[k], seq, W, ws, L)
                done[k].record(comp_s)
                if i + 1 < n_steps:
                    upload(i + 1)
                copy_s.wait_event(done[k])
                with torch.cuda.stream(copy_s):
                    h_out.copy_(dev[k]["out"], non_blocking=True)
            comp_s.wait_stream(copy_s)

        def timed(graphed):
            nonlocal used
            run(warmup, graphed)
            torch.cuda.synchronize()
            barrier()
            used = [False] * copies
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(comp_s)
            run(steps, graphed)
            e1.record(comp_s)
            torch.cuda.synchronize()
            barrier()
            ms_e = max_over_ranks(e0.elapsed_time(e1))
            return {"value": aggregate_throughput(world, B, steps, ms_e), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": ms_e / steps}

        e2e_res = timed(True)
        e2e_res["how"] = "CUDA graph of the step's C-ABI calls per step; copies on a second stream"
        e2e_eager = timed(False)
        e2e_eager["how"] = "C-ABI calls made eagerly inside the timed region; copies on a second stream"
        if bmw.la_pbd_check(ws) != 0:
            raise RuntimeError("device-side status not OK after the end-to-end timing")
        del one_step
    del step_graphs
    return {
        "wi": wi, "ms_per_step": ms_per_step, "value": value, "clocks": clk,
        "launch_us": launch_us, "alg_bytes": alg_bytes, "achieved_gbs": achieved,
        "step_bytes": step_bytes, "copies": copies, "e2e": e2e_res, "e2e_eager": e2e_eager,
        "layers": L, "algo_us": algo_us, "algo": ALGO_NAMES[bmw.chosen_algo(cfg, W)],
        # per layer: attention (with the append fused in on the tcgen05 path) + merge; the
        # CUDA-core path runs the append kernel too
        "launches_per_step": per_step_launches, "launch_floor": launch_floor,
    }


def roofline_block(res, peak, peak_kind, name):
    """Roofline of the dominant kernel (the attention call: attention + merge) of a workload."""
    return {"bound": "hbm", "achieved": res["achieved_gbs"], "peak": peak, "unit": "GB/s",
            "frac": res["achieved_gbs"] / peak, "peak_kind": peak_kind,
            "frac_of_8tbs": res["achieved_gbs"] / 8000.0,
            "traffic": stored_traffic(name),
            "kernel": f"la_pbd_attn ({res['algo']} split-KV attention + merge), one layer",
            "bytes_per_launch": res["alg_bytes"], "launch_us": res["launch_us"]}


def measure_prefill(args, device, bmw, torch, barrier, max_over_ranks, T=16384, bs=6):
    """Block-causal prefill (the pages' long contexts): one sequence of T tokens, 16 query /
    2 KV heads, block size 6, timed back to back in a CUDA graph over two copies of the inputs
    (> L2 together). Algorithmic FLOPs: 4 * D * Hq * sum_i visible(i) (QK^T and PV)."""
    pi = workloads.prefill_case((T,), seed=71)
    cfg = bmw.Config.make(1, pi.q.shape[2], pi.k_cache.shape[1], pi.k_cache.shape[2])
    copies = [{n: getattr(pi, n).to(device) for n in ("q", "k_cache", "v_cache", "seq_lens")}
              for _ in range(2)]
    for d in copies:
        d["out"] = torch.empty_like(d["q"])
    ws = bmw.PrefillWorkspace(cfg, T, device=device)
    run = lambda d: bmw.la_block_prefill(cfg, d["q"], d["k_cache"], d["v_cache"], d["seq_lens"],  # noqa: E731
                                          bs, d["out"], ws)
    graphs = [capture(torch, lambda d=d: run(d)) for d in copies]
    reps = max(4, min(args.steps, 10))
    ms = max_over_ranks(time_graphs(torch, graphs, reps, args.warmup, barrier)) / reps
    if bmw.la_pbd_check(ws) != 0:
        raise RuntimeError("device-side status not OK after the prefill benchmark")
    i = torch.arange(T, dtype=torch.float64)
    visible = torch.minimum(torch.full_like(i, T), (torch.floor(i / bs) + 1) * bs).sum().item()
    flops = 4.0 * 128 * pi.q.shape[2] * visible
    tflops = flops / (ms * 1e-3) / 1e12
    peak = None
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak = float(json.load(f)["bf16_tflops"])
    except Exception:
        peak = 1590.0
    return {"workload": f"block prefill T={T} bs={bs} 16q/2kv d128", "ms": ms,
            "tflops": tflops, "bound": "tensor", "peak_tflops": peak,
            "frac_of_measured_bf16": tflops / peak, "flops_per_call": flops}


def dist_helpers(world, device):
    """Barrier and max-over-ranks reduction for the timing (the only collective used: the
    replicas share no data)."""
    if world <= 1:
        return (lambda: None), (lambda x: x)
    import torch
    import torch.distributed as dist

    def barrier():
        dist.barrier()

    def max_over_ranks(x):
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return barrier, max_over_ranks


def aggregate_throughput(world, batch, steps, max_ms):
    """Whole-job window-steps/s: every replica runs `batch` sequences for `steps` steps; the
    job takes as long as its slowest rank."""
    return world * batch * steps / (max_ms / 1e3)


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def _oracle_sample(wl, wi, budget_s):
    """Whole-layer oracle calls until the budget is spent (at most 4 steps' worth)."""
    import oracle
    done, t0 = 0, time.perf_counter()
    while True:
        li = wi.layers[done % len(wi.layers)]
        oracle.pbd_step(li.q, li.k_cache, li.v_cache, li.k_new, li.v_new, wi.seq_lens, wl.scale)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or done >= 4 * wl.layers:
            return done, el


def cpu_baseline(wl, budget_s):
    """The fp64 oracle on a bounded sample of the workload (whole layers), timed with the
    host's default BLAS threading and with BLAS limited to one thread (half the budget). The
    faster of the two is the baseline; the other is reported beside it."""
    wi = workloads.generate(wl, layers=min(wl.layers, 4))
    try:
        threads = len(os.sched_getaffinity(0))
    except Exception:
        threads = os.cpu_count()
    done, el = _oracle_sample(wl, wi, budget_s)
    runs = [{"value": wl.batch / (el / done * wl.layers), "unit": UNIT, "cores": threads,
             "sample": f"{done} layer calls of the {wl.name} workload ({el:.1f} s), scaled to "
                       f"{wl.layers}-layer steps; numpy fp64, all host threads"}]
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            done1, el1 = _oracle_sample(wl, wi, budget_s / 2)
        runs.append({"value": wl.batch / (el1 / done1 * wl.layers), "unit": UNIT, "cores": 1,
                     "sample": f"{done1} layer calls of the {wl.name} workload ({el1:.1f} s), "
                               f"scaled to {wl.layers}-layer steps; numpy fp64, BLAS limited "
                               f"to one thread"})
    except ImportError:
        pass
    runs.sort(key=lambda r: r["value"], reverse=True)
    best = dict(runs[0], kind="oracle", cpu_model=cpu_model())
    best["other"] = runs[1] if len(runs) > 1 else None
    return best


def workload_label(wl, world):
    """The workload a line measures (identical in both arms' lines)."""
    return {"workload": wl.name, "batch": wl.batch, "layers": wl.layers,
            "prefix": wl.prefix if wl.prefix is not None else "ragged U{512..4096}+U{1..5}",
            "window": wl.window, "q_heads": wl.num_q_heads, "kv_heads": wl.num_kv_heads,
            "head_dim": wl.head_dim, "seed": wl.seed, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (rotating copies of the whole workload)"}


DEFAULT_SWEEP = "tiny,single_image,max_context,max_context_w1,ragged,ragged_w10"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--algo", type=int, default=0, help="0 auto, 1 tcgen05, 2 CUDA cores")
    ap.add_argument("--sweep", default=DEFAULT_SWEEP,
                    help="extra workloads measured for the prefix-length sweep ('' for none)")
    ap.add_argument("--max-copies", type=int, default=16)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-compare", action="store_true", help="skip the per-kernel timing table")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-baseline leg")
    ap.add_argument("--no-prefill", action="store_true", help="skip the block-prefill line")
    ap.add_argument("--prefill-tokens", type=int, default=16384,
                    help="sequence length of the block-prefill line")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.steps = max(args.steps, 1)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = workloads.WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return
        cb = cpu_baseline(wl, args.cpu_budget)
        line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * wl.batch / cb["value"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": workload_label(wl, args.gpus), "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    import block_masked_window_b200 as bmw
    bmw.load()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        device = torch.device("cuda", local_rank)
    else:
        device = torch.device("cuda", 0)
        torch.cuda.set_device(0)
    barrier, max_over_ranks = dist_helpers(world, device)

    compare = not args.no_compare
    res = measure(args, rank, world, device, bmw, torch, wl, barrier, max_over_ranks,
                  e2e=not args.no_e2e, compare=compare)
    peak, peak_kind = measured_peaks()
    sweep = []
    algo_compare = {wl.name: res["algo_us"]} if compare else {}
    for name in [s for s in args.sweep.split(",") if s and s != wl.name]:
        swl = workloads.WORKLOADS[name]
        sargs = argparse.Namespace(**vars(args))
        sargs.steps = max(10, min(args.steps, 20))
        r = measure(sargs, rank, world, device, bmw, torch, swl, barrier, max_over_ranks,
                    e2e=False, compare=compare)
        if compare:
            algo_compare[name] = r["algo_us"]
        sweep.append({
            "workload": name, "prefix": swl.prefix if swl.prefix is not None else "ragged",
            "batch": swl.batch, "window": swl.window, "layers": swl.layers,
            "window_steps_per_s": r["value"], "ms_per_step": r["ms_per_step"],
            "attn_launch_us": r["launch_us"], "attn_bytes_per_launch": r["alg_bytes"],
            "launch_floor_ms_per_step": r["launch_floor"]["ms_per_step"],
            "roofline": roofline_block(r, peak, peak_kind, name), "clocks": r["clocks"],
        })

    prefill = None if args.no_prefill else measure_prefill(args, device, bmw, torch, barrier,
                                                           max_over_ranks, T=args.prefill_tokens)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    cb = cpu_baseline(wl, args.cpu_budget) if (world == 1 and not args.no_cpu) else None
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V, per the workload recipe)",
        "config": workload_label(wl, world),
        "run": {"graph": "CUDA graph per step", "algo": res["algo"], "algo_arg": args.algo,
                "copies": res["copies"]},
        "roofline": roofline_block(res, peak, peak_kind, wl.name),
        "gpu_launches": res["launches_per_step"] * args.steps,
        "e2e": res["e2e"], "e2e_eager": res["e2e_eager"], "clocks": res["clocks"],
        "cpu_baseline": cb,
        "launch_floor": res["launch_floor"],
        "step_bytes": res["step_bytes"],
        "step_gbs": res["step_bytes"] / (res["ms_per_step"] * 1e-3) / 1e9,
        "sweep": sweep,
        "algo_compare_us": algo_compare,
        "prefill": prefill,
    }
    print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
