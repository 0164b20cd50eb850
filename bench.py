"""Throughput of the routed-expert MoE layer on B200.

Workload (default): the BF16 decode layer -- E=128 experts, top-8, d=2048,
SwiGLU intermediate 768, weights ~N(0, 0.02^2) in bf16, router logits N(0,1)
plus a per-expert bias N(0, 0.5^2), T=64 tokens per step, every expert
resident in HBM.  One step = route -> permute -> expert FFN -> combine over
one batch, captured in a CUDA graph.  R independent replicas of the layer
(weights, routing, activations) are cycled so that the bytes read between two
uses of a replica exceed the 126 MB L2 several times.

Output: one JSON line on rank 0 (see the keys below).  `--impl reference`
times the CPU oracle instead, on a bounded sample of the same workload.
Multi-GPU: launch with torchrun; every rank runs its own replica set
(independent batches, no data-path collective), timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s; decode HBM GB/s and prefill FP4 TFLOPS vs B200 peak"
L2_BYTES = 126 * 1024 * 1024


def kernel_traffic(kernel_file, key):
    """DRAM bytes (read + write) per launch of a kernel from the ncu capture
    recorded in profiles/traffic.json -- only while the kernel's source file
    still has the hash recorded there (None once the kernel has changed)."""
    import hashlib
    rec_path = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "expert_offload_serving_b200", "csrc", kernel_file)
    if not (os.path.exists(rec_path) and os.path.exists(src)):
        return None
    rec = json.load(open(rec_path)).get(key)
    if not rec:
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return rec["bytes_per_launch"] if rec.get("source_sha256_16") == h else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if "hbm_gbs" in d:
            return d["hbm_gbs"], "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 100 ms, each with nvidia-smi's own timestamp)
    of SM clock and throttle reasons while the bench runs; summary() keeps the
    samples that fall inside the given wall-clock windows."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    @staticmethod
    def now():
        return time.time()

    def _samples(self):
        import datetime
        out = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                out.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        return out

    def summary(self, windows=None):
        """Median SM clock, max clock and the throttle reasons seen, over the
        samples inside `windows` ([(t0, t1)] wall-clock seconds; all if None)."""
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for ts, clk, cmax, flags in self._samples():
            if windows is not None and not any(a - 0.05 <= ts <= b + 0.05 for a, b in windows):
                continue
            sm.append(clk)
            mx.append(cmax)
            for n, v in zip(names, flags):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_info():
    """Host CPU model and its physical core count (unique (package, core)
    pairs in /proc/cpuinfo), next to the threads this process may use."""
    model, cores = None, set()
    try:
        phys = core = None
        for ln in open("/proc/cpuinfo"):
            k, _, v = ln.partition(":")
            k, v = k.strip(), v.strip()
            if k == "model name" and model is None:
                model = v
            elif k == "physical id":
                phys = v
            elif k == "core id":
                core = v
            elif not k and phys is not None:
                cores.add((phys, core))
                phys = core = None
    except OSError:
        pass
    return {"cpu_model": model, "physical_cores": len(cores) or None, "threads_available": _cpu_cores()}


# ---------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- workload
def build_replicas(cfg, T, R, seed0=0, routed_only=False):
    """R independent resident layers with their inputs on the device.
    routed_only: materialise only the experts the batch's top-k selects (the
    slot table maps them; the others are never read)."""
    from expert_offload_serving_b200.layer import MoeLayer, pack_pool
    reps = []
    for r in range(R):
        seed = seed0 + r
        logits, x = synth.make_routing(cfg, T, seed)
        if routed_only:
            experts = sorted(set(torch.topk(logits, cfg.k, dim=1).indices.ravel().tolist()))
        else:
            experts = list(range(cfg.E))
        w = synth.make_experts(cfg, experts, seed, device="cuda")
        pool = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, {k: v.cpu() for k, v in w.items()},
                         experts, pin=False).cuda()
        del w
        layer = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, device_pool=pool)
        if routed_only:
            layer.slot.fill_(-1)
            layer.slot[torch.tensor(experts, device=layer.slot.device)] = torch.arange(
                len(experts), dtype=torch.int32, device=layer.slot.device)
        reps.append(dict(layer=layer, logits=logits.cuda(), x=x.cuda(), logits_h=logits.pin_memory(),
                         x_h=x.pin_memory()))
    return reps


def steps_per_graph(K, R, cap=32):
    """Steps captured into one CUDA graph: the largest divisor of K that is a
    multiple of R and at most cap (1 when there is none), so that K steps are
    exactly K / G replays and one launch covers several small steps."""
    for g in range(min(K, cap), 0, -1):
        if K % g == 0 and g % R == 0:
            return g
    return 1


def capture_cycle(fns, G, stream):
    """One CUDA graph running G calls fns[0], fns[1], ... (cycling)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(G):
            fns[i % len(fns)]()
    return g


def experts_touched(layer):
    """Distinct experts of the last step (non-empty groups of the layer's
    offsets): the algorithmic weight bytes are this count x blob bytes."""
    off = layer.offsets.cpu()
    return int(((off[1:] - off[:-1]) > 0).sum())


def decode_point(cfg, T, R, warmup, steps, stream, routed_only=False):
    """Device-timed decode_bf16 layer steps at T tokens (graph replay over R
    replicas) and the expert-FFN time alone, for the secondary T points."""
    import expert_offload_serving_b200 as moe
    blob = moe.moe_expert_blob_bytes(moe.shape(cfg.E, cfg.d, cfg.I, cfg.fmt))
    reps = build_replicas(cfg, T, R, seed0=500 + T, routed_only=routed_only)
    U = []
    for r in reps:
        r["layer"].forward(r["logits"], r["x"])
        torch.cuda.synchronize()
        U.append(experts_touched(r["layer"]))
    G = steps_per_graph(steps, R)
    with torch.cuda.stream(stream):
        step_fns = [lambda r=r: r["layer"].forward(r["logits"], r["x"]) for r in reps]
        ffn_fns = [lambda r=r: r["layer"].ffn(r["x"]) for r in reps]
        for f in step_fns + ffn_fns:
            f()
        stream.synchronize()
        g_step = capture_cycle(step_fns, G, stream)
        g_ffn = capture_cycle(ffn_fns, G, stream)
        for _ in range(max(1, warmup // G)):
            g_step.replay()
            g_ffn.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps // G):
            g_step.replay()
        e1.record(stream)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(steps // G):
            g_ffn.replay()
        f1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    ffn_ms = f0.elapsed_time(f1) / steps
    del g_step, g_ffn
    gbs = sum(U) / R * blob / (ffn_ms / 1e3) / 1e9
    hbm, _ = peaks()
    del reps
    return {"tokens_per_s": round(T / (ms / 1e3), 1), "ms_per_step": round(ms, 5), "ffn_ms": round(ffn_ms, 5),
            "ffn_gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4), "experts_touched": U}


def run_gpu(args, rank, world, local):
    """The GPU arm, with nvidia-smi sampling clocks over the whole run."""
    idx = local if world > 1 else 0
    props = torch.cuda.get_device_properties(idx)
    smi_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(idx)
    with ClockSampler(smi_id) as clk:
        return _run_gpu(args, rank, world, local, clk, [])


def _run_gpu(args, rank, world, local, clk, timed_windows):
    import expert_offload_serving_b200 as moe
    moe.lib()
    cfg = synth.CONFIGS[args.config]
    T = args.tokens
    routed_only = cfg.fmt != "bf16"   # the 256-expert MXFP4 layer: only the routed experts are materialised
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    blob = moe.moe_expert_blob_bytes(moe.shape(cfg.E, cfg.d, cfg.I, cfg.fmt))
    # replicas: the bytes between two uses of one replica >= 4 x L2
    per_step = None
    R = args.replicas
    reps = build_replicas(cfg, T, R, seed0=1000 * rank, routed_only=routed_only)
    U = []
    for r in reps:
        r["layer"].forward(r["logits"], r["x"])
        torch.cuda.synchronize()
        U.append(experts_touched(r["layer"]))
    per_step = [u * blob for u in U]
    if R > 1 and min(sum(per_step) - p for p in per_step) < 4 * L2_BYTES:
        print(f"warning: replicas stream only {min(sum(per_step) - p for p in per_step) / 1e6:.0f} MB "
              "between reuses", file=sys.stderr)
    stream = torch.cuda.Stream(device=dev)
    # kernels per step: route, permute, the FFN's (the library reports them:
    # one cooperative GEMV launch or gate/up + down, plus MXFP4's split of x
    # into E4M3 terms; a one-launch counter reset is a memset node), combine
    ffn_launches = moe.moe_expert_ffn_launches(moe.shape(cfg.E, cfg.d, cfg.I, cfg.fmt), T, cfg.k)
    two = ffn_launches - (1 if cfg.fmt == "mxfp4" else 0) == 2
    launches_per_step = 3 + ffn_launches

    def step_fn(r):
        L = r["layer"]
        L.forward(r["logits"], r["x"])

    # one CUDA graph of G consecutive steps cycling over the replicas (G divides
    # K, so the K timed steps are K / G replays; small steps are not bound by
    # the host's launch rate)
    G = steps_per_graph(args.steps, R)
    with torch.cuda.stream(stream):
        for r in reps:                      # warm the code paths once before capture
            step_fn(r)
        stream.synchronize()
        g_steps = capture_cycle([lambda r=r: step_fn(r) for r in reps], G, stream)
    torch.cuda.synchronize()

    # ---- device-timed steps (W warm-up steps, rounded up to whole graphs)
    with torch.cuda.stream(stream):
        for _ in range((args.warmup + G - 1) // G):
            g_steps.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = ClockSampler.now()
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps // G):
            g_steps.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    timed_windows.append((w0, ClockSampler.now()))
    ms = ev0.elapsed_time(ev1)
    barrier(world)
    ms_max = max_over_ranks(ms, world)
    value = world * args.steps * T / (ms_max / 1e3)

    # ---- dominant kernel: moe_expert_ffn (gate/up + down launches), timed alone,
    # as graph replays of G calls on the bench stream
    # each replay (G calls cycling the R replicas) timed on its own; the line
    # reports the median replay
    with torch.cuda.stream(stream):
        g_ffn = capture_cycle([lambda r=r: r["layer"].ffn(r["x"]) for r in reps], G, stream)
        for _ in range(max(1, (max(3, args.warmup) + G - 1) // G)):
            g_ffn.replay()
        n_rep = max(20, (args.steps + G - 1) // G)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_rep)]
        w0 = ClockSampler.now()
        for a, b in evs:
            a.record(stream)
            g_ffn.replay()
            b.record(stream)
    torch.cuda.synchronize()
    timed_windows.append((w0, ClockSampler.now()))
    del g_ffn
    rep_ms = sorted(a.elapsed_time(b) for a, b in evs)
    ffn_avg_ms = statistics.median(rep_ms) / G
    ffn_spread = (round(rep_ms[0] / G, 5), round(rep_ms[-1] / G, 5))
    alg_bytes = sum(per_step[i % R] for i in range(G)) / G
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hbm_peak, peak_src = peaks()
    achieved = alg_bytes / (ffn_avg_ms / 1e3) / 1e9

    # ---- end to end through the public API with host buffers: every step
    # uploads its logits and x from pinned host memory and downloads its out,
    # pipelined as a serving loop would run it -- the copies go on a copy
    # stream (uploads one step ahead, downloads behind), ordered by events,
    # and the timed region closes when the last download has landed
    e2e_steps = max(3, min(args.steps, 50))
    outs_h = [torch.empty((T, cfg.d), dtype=torch.float32, pin_memory=True) for _ in range(R)]
    copy = torch.cuda.Stream(device=dev)
    in_ready = [torch.cuda.Event() for _ in range(R)]
    out_done = [torch.cuda.Event() for _ in range(R)]
    out_copied = [torch.cuda.Event() for _ in range(R)]
    for ev in out_done + out_copied:
        ev.record(stream)                   # give every event a handle before it is waited on

    def upload(i):
        r = reps[i % R]
        with torch.cuda.stream(copy):
            copy.wait_event(out_done[i % R])          # the replica's previous step has read its inputs
            r["logits"].copy_(r["logits_h"], non_blocking=True)
            r["x"].copy_(r["x_h"], non_blocking=True)
            in_ready[i % R].record(copy)

    def compute(i):
        r = reps[i % R]
        stream.wait_event(in_ready[i % R])
        stream.wait_event(out_copied[i % R])          # its previous out has been downloaded
        r["out_dev"] = r["layer"].forward(r["logits"], r["x"], stream=stream)
        out_done[i % R].record(stream)

    def download(i):
        r = reps[i % R]
        with torch.cuda.stream(copy):
            copy.wait_event(out_done[i % R])
            outs_h[i % R].copy_(r["out_dev"], non_blocking=True)
            out_copied[i % R].record(copy)

    def run_e2e(n, first):
        upload(first)
        for i in range(first, first + n):
            if i + 1 < first + n:
                upload(i + 1)
            compute(i)
            download(i)

    with torch.cuda.stream(stream):
        run_e2e(max(3, args.warmup), 0)
        torch.cuda.synchronize()
        barrier(world)
        e0.record(stream)
        copy.wait_event(e0)
        run_e2e(e2e_steps, 0)
        stream.wait_event(out_copied[(e2e_steps - 1) % R])
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = world * e2e_steps * T / (e2e_ms / 1e3)
    h2d = T * cfg.E * 4 + T * cfg.d * 2
    d2h = T * cfg.d * 4

    st = reps[0]["layer"].status
    moe.moe_check_status(st)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, T)

    streamed = None
    if not args.no_prefill and not args.no_cached and world == 1:
        streamed = run_streamed_prefill()
    prefill = None
    if not args.no_prefill:
        prefill = run_prefill(Ts=(4096,) if (args.no_sweep or world > 1) else (4096, 16384, 32768),
                              windows=timed_windows)
    sweep = None
    if not args.no_sweep and world == 1:
        sweep = {}
        for t in (1, 16):
            if t == T:
                continue
            # T=1 touches ~75 MB: 8 replicas stream >= 4x L2 between two uses of one
            sweep[f"T{t}"] = decode_point(cfg, t, max(R, 8) if t == 1 else R, args.warmup,
                                          min(args.steps, 2000), stream)
    mx = None
    if not args.no_sweep and world == 1:
        cmx = synth.CONFIGS["decode_mxfp4"]
        mx = {f"T{t}": decode_point(cmx, t, 8, args.warmup, min(args.steps, 1000), stream, routed_only=True)
              for t in cmx.T}
    cached = split = layered = None
    if not args.no_cached and world == 1:
        hp = cached_host_pool()
        cached = [run_cached_decode(hp, T=t) for t in (1, 8)]
        split = run_split_sweep(hp)
        layered = run_layered_cache(hp)
        del hp

    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.fmt == "bf16" else "mxfp4 weights x bf16 activations",
        "data": "synthetic",
        "config": {
            "workload": f"{cfg.name}: E={cfg.E} k={cfg.k} d={cfg.d} I={cfg.I} T={T}, "
                        + ("the routed experts resident" if routed_only else "all experts resident"),
            "global_batch": T * world,
            "replicas": R,
            "l2": f"inputs larger than L2: {R} replicas, >= {min(sum(per_step) - p for p in per_step) / 1e6:.0f} MB "
                  "read between reuses" if R > 1 else "single replica",
            "experts_touched_per_step": U,
            "parallelism": f"dp{world} (independent batches)",
            "cuda_graph": f"{G} steps per graph, cycling the replicas",
        },
        "roofline": {
            "kernel": "moe_expert_ffn: " + ("gemv_mx_kernel" if cfg.fmt == "mxfp4" else "gemv_tc_kernel")
                      + (" gate/up + down (two launches)" if two else " (both GEMVs, one launch)"),
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": hbm_peak,
            "peak_source": peak_src,
            "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4),
            "traffic": kernel_traffic("ffn_decode_tc.cu", f"{cfg.name}_T{T}"),
            "algorithmic_bytes_per_launch": int(alg_bytes),
            "avg_launch_ms": round(ffn_avg_ms, 5),
            "timing": f"median of {n_rep} graph replays of {G} calls (per-call min/max over replays: "
                      f"{ffn_spread[0]} / {ffn_spread[1]} ms)",
        },
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(timed_windows),
        "clocks_whole_run": clk.summary(),
    }
    if cpu is not None:
        result["cpu_baseline"] = cpu
    if prefill is not None:
        result["prefill"] = prefill[0]
        if len(prefill) > 1:
            result["prefill_T_sweep"] = prefill[1:]
    if cached is not None:
        result["decode_mxfp4_cached"] = cached
    if split is not None:
        result["split_merge_q_sweep"] = split
    if layered is not None:
        result["layered_cache"] = layered
    if streamed is not None:
        result["prefill_streamed"] = streamed
    if sweep:
        result["decode_bf16_T_sweep"] = sweep
    if mx:
        result["decode_mxfp4_resident"] = mx
    return result


# ---------------------------------------------------------------- prefill (FP4 tensor cores)
def prefill_kernels(cfg, T):
    """The kernels the library runs for an FP4 prefill step of T tokens: single
    CTAs with at most 128 token rows per expert on average, else CTA pairs
    (or what MOE_PREFILL_TILES forces)."""
    forced = os.environ.get("MOE_PREFILL_TILES")
    single = forced == "cta" if forced in ("cta", "pair") else T * cfg.k <= 128 * cfg.E
    if single:
        return "quant_tokens_cta_kernel, gather_x128_kernel, gemm_fp4_cta_kernel<1>, gemm_fp4_cta_kernel<2> (single CTAs)"
    return "quant_tokens_kernel, gather_x_kernel, gemm_fp4_kernel<1>, gemm_fp4_kernel<2> (CTA pairs)"


def run_prefill(iters=20, warmup=5, Ts=(4096,), E=None, windows=None):
    """The NVFP4 prefill layer (E=256, k=6, d=4096, I=2048, NVFP4 activations
    on tcgen05) at each token count in Ts: whole-layer time and the expert-FFN
    time alone.  The 3.6 GB of weights exceed L2 many times over, so no
    replicas.  T=4096 is bound by the weight read; at 16384 and 32768 tokens
    the FP4 contraction dominates."""
    import expert_offload_serving_b200 as moe
    from expert_offload_serving_b200.layer import MoeLayer, pack_pool
    cfg = synth.CONFIGS["prefill_nvfp4"]
    if E is not None and E != cfg.E:
        # a smaller expert count at the same d, I, k (for short profiler captures)
        cfg = dataclasses.replace(cfg, E=E)
    w = synth.make_experts(cfg, range(cfg.E), 0, device="cuda")
    pool = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, {k: v.cpu() for k, v in w.items()}, range(cfg.E),
                     pin=False).cuda()
    del w
    layer = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, max(Ts), device_pool=pool, act="nvfp4")
    have_peaks = os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json"))
    d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if have_peaks else {}
    bf16 = d.get("bf16_tflops", 1590.0)
    fp4_peak = 4.0 * bf16          # dense FP4 = 4 x dense BF16 (nominal 9 / 2.25 PFLOP/s)
    fp4_src = ("4 x measured bf16 (MEASURED_PEAKS.json bf16_tflops)" if "bf16_tflops" in d
               else "4 x fallback bf16 1590 TFLOP/s (no measured peaks file)")
    hbm, _ = peaks()
    out = []
    for T in Ts:
        logits, x = synth.make_routing(cfg, T, 0)
        lg, xx = logits.cuda(), x.cuda()
        stream = torch.cuda.Stream()
        n = max(20, iters)
        ev = lambda: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        le = [ev() for _ in range(n)]
        fe = [ev() for _ in range(n)]
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                layer.forward(lg, xx)
            w0 = time.time()
            for a, b in le:                     # each call timed on its own: the median is reported
                a.record(stream)
                layer.forward(lg, xx)
                b.record(stream)
            for a, b in fe:
                a.record(stream)
                layer.ffn(xx)
                b.record(stream)
        torch.cuda.synchronize()
        if windows is not None:
            windows.append((w0, time.time()))
        layer_all = sorted(a.elapsed_time(b) for a, b in le)
        ffn_all = sorted(a.elapsed_time(b) for a, b in fe)
        layer_ms = statistics.median(layer_all)
        ffn_ms = statistics.median(ffn_all)
        moe.moe_check_status(layer.status)
        flops = 2.0 * 3 * cfg.d * cfg.I * T * cfg.k
        off = layer.offsets.cpu()
        U = int(((off[1:] - off[:-1]) > 0).sum())
        wbytes = U * moe.moe_expert_blob_bytes(moe.shape(cfg.E, cfg.d, cfg.I, cfg.fmt))
        tf = flops / (ffn_ms / 1e3) / 1e12
        gbs = wbytes / (ffn_ms / 1e3) / 1e9
        roof_ms = max(wbytes / (hbm * 1e9), flops / (fp4_peak * 1e12)) * 1e3
        out.append({
            "workload": f"prefill_nvfp4: E={cfg.E} k={cfg.k} d={cfg.d} I={cfg.I} T={T}, "
                        "NVFP4 weights and activations",
            "tokens_per_s": round(T / (layer_ms / 1e3), 1),
            "layer_ms": round(layer_ms, 4),
            "ffn_ms": round(ffn_ms, 4),
            "tflops": round(tf, 1),
            "fp4_peak_tflops": round(fp4_peak, 1),
            "fp4_peak_source": fp4_src,
            "frac_fp4_peak": round(tf / fp4_peak, 4),
            "weight_gbs": round(gbs, 1),
            "frac_hbm": round(gbs / hbm, 4),
            "roofline_ms": round(roof_ms, 4),
            "frac_roofline": round(roof_ms / ffn_ms, 4),
            "experts_touched": U,
            "timed_iters": n,
            "timing": f"median of {n} individually timed calls (FFN min/max {ffn_all[0]:.4f} / {ffn_all[-1]:.4f} ms)",
            "kernels": prefill_kernels(cfg, T),
        })
        del lg, xx
    return out


# ---------------------------------------------------------------- prefill streamed from host memory
def run_streamed_prefill(Ts=(4096, 8192, 16384), n_layers=4, reps=2):
    """Prefill through n_layers NVFP4 layers (E=256, k=6, d=4096, I=2048)
    whose 3.6 GB expert pools stay in pinned host memory (every layer reads
    the same pool here; its bytes cross PCIe once per layer either way): each
    layer's pool is copied into one of two full-layer device buffers while
    the GPU computes the previous layer from the other, against the same
    layers with each copy issued only after the previous compute (the pages'
    ablation of double buffering).  Device-timed per chunk of T tokens."""
    import expert_offload_serving_b200 as moe
    from expert_offload_serving_b200.layer import StreamedPrefill, pack_pool
    cfg = synth.CONFIGS["prefill_nvfp4"]
    w = synth.make_experts(cfg, range(cfg.E), 0, device="cuda")
    host = pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, {k: v.cpu() for k, v in w.items()}, range(cfg.E), pin=True)
    del w
    sp = StreamedPrefill(cfg.E, cfg.d, cfg.I, cfg.k, max(Ts), [host] * n_layers)
    B = host.numel()
    rows = []
    st = torch.cuda.current_stream()
    for T in Ts:
        inputs = []
        for l in range(n_layers):
            lg, x = synth.make_routing(cfg, T, 700 + l)
            inputs.append((lg.cuda(), x.cuda()))
        r = {"T": T}
        for mode in (True, False):
            sp.run(inputs, double_buffer=mode)          # warm-up
            times = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(st)
                sp.copy.wait_event(a)
                sp.run(inputs, double_buffer=mode)
                st.wait_stream(sp.copy)
                b.record(st)
                torch.cuda.synchronize()
                times.append(a.elapsed_time(b))
            ms = statistics.median(times)
            r["double_buffered" if mode else "serial"] = {
                "ms_per_chunk": round(ms, 3), "tokens_per_s": round(T / (ms / 1e3), 1),
                "h2d_gbs": round(n_layers * B / (ms / 1e3) / 1e9, 1)}
        # the compute alone: the layers run from a buffer already on the device
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for l in range(n_layers):
            sp.layers[0].forward(*inputs[l])
        b.record(st)
        torch.cuda.synchronize()
        r["compute_only_ms"] = round(a.elapsed_time(b), 3)
        db, se = r["double_buffered"]["tokens_per_s"], r["serial"]["tokens_per_s"]
        r["throughput_loss_without_double_buffering"] = round(1.0 - se / db, 4)
        rows.append(r)
        del inputs
    for L_ in sp.layers:
        moe.moe_check_status(L_.status)
    del sp, host
    return {"workload": f"prefill_nvfp4 x {n_layers} layers: E={cfg.E} k={cfg.k} d={cfg.d} I={cfg.I}, each layer's "
                        "3.6 GB pool streamed from pinned host memory into two full-layer buffers",
            "timing": f"median of {reps} device-timed passes over the {n_layers} layers", "chunks": rows}


# ---------------------------------------------------------------- decode with the expert cache
def cached_host_pool():
    """The 256 MXFP4 experts of the cached-decode workload, packed into one
    pinned host pool in expert order."""
    from expert_offload_serving_b200.layer import pack_pool
    cfg = synth.CONFIGS["decode_mxfp4"]
    w = synth.make_experts(cfg, range(cfg.E), 0, device="cuda")
    return pack_pool(cfg.E, cfg.d, cfg.I, cfg.fmt, {k: v.cpu() for k, v in w.items()}, range(cfg.E), pin=True)


def run_cached_decode(host_pool, T=1, steps=64, warm=32):
    """MXFP4 decode with 64 GPU slots over a drifting routing trace (E=256,
    k=6, d=4096, I=2048): per step the host reads the routing, the LRU fills
    misses from the pinned host pool over PCIe on a side stream, then
    permute -> FFN -> combine.  Timed on the device over `steps` steps after
    `warm` warm-up steps (fills included)."""
    import expert_offload_serving_b200 as moe
    from expert_offload_serving_b200.layer import MoeLayer
    cfg = synth.CONFIGS["decode_mxfp4"]
    B = host_pool.shape[1]
    # pinned host -> device copy bandwidth of whole blobs (the fill path)
    dst = torch.empty((8, B), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        for i in range(8):
            dst[i].copy_(host_pool[i], non_blocking=True)
        e0.record(s)
        for rep in range(4):
            for i in range(8):
                dst[i].copy_(host_pool[8 * rep + i], non_blocking=True)
        e1.record(s)
    torch.cuda.synchronize()
    h2d_gbs = 32 * B / (e0.elapsed_time(e1) / 1e3) / 1e9
    del dst
    layer = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, host_pool=host_pool, n_slots=cfg.n_slots)
    trace = synth.make_trace(cfg, T, steps=warm + steps, seed=0)
    lgs = [lg.cuda() for lg, _ in trace]
    xs = [x.cuda() for _, x in trace]
    main = torch.cuda.Stream()
    hits = misses = 0
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(main):
        for t in range(warm + steps):
            if t == warm:
                t0.record(main)
            layer.route(lgs[t])
            U = sorted(set(layer.idx[:T].cpu().numpy().ravel().tolist()))
            fills = layer.prepare(t, U, stream=main)
            layer.permute(T)
            layer.ffn(xs[t])
            layer.combine(T)
            if t >= warm:
                misses += len(fills)
                hits += len(U) - len(fills)
        t1.record(main)
    torch.cuda.synchronize()
    moe.moe_check_status(layer.status)
    ms = t0.elapsed_time(t1) / steps
    return {
        "workload": f"decode_mxfp4: E={cfg.E} k={cfg.k} d={cfg.d} I={cfg.I} T={T}, {cfg.n_slots} slots, "
                    f"AR(1) drifting trace, LRU fills from pinned host memory",
        "tokens_per_s": round(T / (ms / 1e3), 1),
        "ms_per_step": round(ms, 4),
        "miss_rate": round(misses / max(1, hits + misses), 4),
        "fills_per_step": round(misses / steps, 2),
        "fill_mb_per_step": round(misses / steps * B / 1e6, 2),
        "h2d_pinned_gbs": round(h2d_gbs, 1),
        "steps": steps,
    }


# ---------------------------------------------------------------- one cache shared by many layers
def _route_on_gpu(cfg, trace, k):
    """Routing of a trace through moe_route_topk (device), read back."""
    import expert_offload_serving_b200 as moe
    lg = torch.cat([l for l, _ in trace]).cuda()
    idx = torch.empty((lg.shape[0], k), dtype=torch.int32, device="cuda")
    gate = torch.empty((lg.shape[0], k), dtype=torch.float32, device="cuda")
    moe.moe_route_topk(lg, k, idx, gate)
    return idx.cpu().numpy()


def run_layered_cache(host_pool, n_sim_layers=43, slots_per_layer=16, T_sim=1, sim_steps=128,
                      n_gpu_layers=4, gpu_slots_per_layer=None, steps=48, warm=16):
    """The pages' global LRU (one expert cache whose decisions are shared by
    all MoE layers) against per-layer caches of equal total capacity.
    (a) Miss rates from the cache planner alone (plan-only handles) for
        n_sim_layers layers (43, DeepSeek-V4-Flash's depth) of E=256, k=6
        experts, T=1 decode: per-layer routing traces with their own AR(1)
        drifting bias and bias spreads 0.25 ... 1.5 across layers (layers with
        sharper routing need fewer slots), each layer's routing from
        moe_route_topk.
    (b) On the GPU: n_gpu_layers MXFP4 layers (E=256, d=4096, I=2048) over one
        pinned host pool, one shared cache of n_gpu_layers * S slots vs S per
        layer (S = 16 at T=1, 64 at T=8, where a step can route to 48
        experts): step time for all layers and miss rate.
    (c) Elastic resize of the shared T=8 cache to half and back, on a full
        cache, device-timed (moves only, no host copy)."""
    import expert_offload_serving_b200 as moe
    from expert_offload_serving_b200.layer import ExpertCache, MoeLayer
    base = synth.CONFIGS["decode_mxfp4"]
    s = moe.shape(base.E, base.d, base.I, base.fmt)
    # (a) planner-only miss rates
    spreads = np.linspace(0.25, 1.5, n_sim_layers)
    idxs = []
    for l in range(n_sim_layers):
        cfg_l = dataclasses.replace(base, bias_std=float(spreads[l]))
        idxs.append(_route_on_gpu(cfg_l, synth.make_trace(cfg_l, T_sim, steps=sim_steps, seed=300 + l), base.k))
    glob = moe.MoeCache(s, n_sim_layers * slots_per_layer, n_layers=n_sim_layers)
    per = [moe.MoeCache(s, slots_per_layer) for _ in range(n_sim_layers)]
    acc = {"global": [0, 0], "per_layer": [0, 0]}
    for t in range(sim_steps):
        for l in range(n_sim_layers):
            U = sorted(set(idxs[l][t * T_sim:(t + 1) * T_sim].ravel().tolist()))
            clock = t * n_sim_layers + l
            fg = glob.fill(U, clock, protect=U, layer=l)
            fp = per[l].fill(U, t, protect=U)
            if t >= sim_steps // 4:                     # after the cold start
                acc["global"][0] += len(fg)
                acc["per_layer"][0] += len(fp)
                acc["global"][1] += len(U)
                acc["per_layer"][1] += len(U)
    glob.close()
    for c in per:
        c.close()
    sim = {k: round(v[0] / v[1], 4) for k, v in acc.items()}
    # (b) GPU step time with the cache shared or split
    res_gpu = {}
    for mode in ("global", "per_layer"):
        for T in (1, 8):
            per_layer_slots = gpu_slots_per_layer or (16 if T == 1 else 64)
            gpu_slots = per_layer_slots * n_gpu_layers
            torch.cuda.synchronize()
            if mode == "global":
                caches = [ExpertCache(s, gpu_slots, [host_pool] * n_gpu_layers)]
                layers = [MoeLayer(s.E, s.d, s.I, base.fmt, base.k, T, cache=caches[0], layer_id=l)
                          for l in range(n_gpu_layers)]
            else:
                caches = [ExpertCache(s, gpu_slots // n_gpu_layers, host_pool) for _ in range(n_gpu_layers)]
                layers = [MoeLayer(s.E, s.d, s.I, base.fmt, base.k, T, cache=caches[l], layer_id=0)
                          for l in range(n_gpu_layers)]
            traces = [synth.make_trace(dataclasses.replace(base, bias_std=float(0.25 + 1.25 * l / 3)), T,
                                       steps=warm + steps, seed=400 + l) for l in range(n_gpu_layers)]
            idx_h = [_route_on_gpu(base, tr, base.k) for tr in traces]
            lgs = [[lg.cuda() for lg, _ in tr] for tr in traces]
            xs = [[x.cuda() for _, x in tr] for tr in traces]
            misses = looked = 0
            st = torch.cuda.current_stream()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for t in range(warm + steps):
                if t == warm:
                    e0.record(st)
                for l in range(n_gpu_layers):
                    U = sorted(set(idx_h[l][t * T:(t + 1) * T].ravel().tolist()))
                    clock = t * n_gpu_layers + l if mode == "global" else t
                    f = layers[l].prepare(clock, U, protect=U)
                    layers[l].forward(lgs[l][t], xs[l][t])
                    if t >= warm:
                        misses += len(f)
                        looked += len(U)
            e1.record(st)
            torch.cuda.synchronize()
            for L_ in layers:
                moe.moe_check_status(L_.status)
            ms = e0.elapsed_time(e1) / steps
            res_gpu[f"{mode}_T{T}"] = {"ms_per_step_all_layers": round(ms, 4), "miss_rate": round(misses / looked, 4)}
            # (c) resize timing on the full shared cache
            if mode == "global" and T == 8:
                rs = []
                for n in (gpu_slots // 2, gpu_slots):
                    # the new pool is allocated before the timed region: the
                    # events bracket the device moves on the bench stream only
                    new_pool = torch.empty((n, host_pool.shape[1]), dtype=torch.uint8, device=caches[0].dev)
                    torch.cuda.synchronize()
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(st)
                    kept = caches[0].resize(n, stream=st, new_pool=new_pool)
                    b.record(st)
                    torch.cuda.synchronize()
                    del new_pool
                    rs.append({"to_slots": n, "kept": len(kept), "ms": round(a.elapsed_time(b), 4),
                               "moved_gb": round(len(kept) * host_pool.shape[1] / 1e9, 3)})
                res_gpu["resize"] = rs
            for c in caches:
                c.close()
            del layers, caches, lgs, xs
    return {
        "planner_miss_rate": {
            "workload": f"{n_sim_layers} layers x E={base.E} k={base.k}, T={T_sim}, {sim_steps} steps (first quarter "
                        f"excluded), AR(1) routing bias per layer, spreads 0.25..1.5; capacity "
                        f"{n_sim_layers * slots_per_layer} slots: global vs {slots_per_layer} per layer",
            **sim},
        "gpu": {"workload": f"{n_gpu_layers} MXFP4 layers (E={base.E} d={base.d} I={base.I} k={base.k}) over one pinned "
                            f"host pool; {n_gpu_layers} x S slots shared vs S per layer (S = 16 at T=1, 64 at T=8); "
                            f"{steps} steps after {warm}", **res_gpu},
    }


# ---------------------------------------------------------------- q sweep of the miss split
def run_split_sweep(host_pool, T=8, steps=32, warm=16, threads=0):
    """The split/merge workload at its configured shapes (E=256, k=6, d=4096,
    I=2048, MXFP4, 64 slots, the AR(1) trace, T=8): each step's cache misses
    are split, a fraction q filled over PCIe on the side stream while the CPU
    computes the rest from the pinned host pool (moe_host_expert_ffn), merged
    by the combine.  For q = 0, 0.1, ..., 1 and for q* (from the bandwidths
    moe_profile_bandwidth measures first): step wall time (host sync to
    host sync), host-kernel and fill times, and the merge's deviation from the
    all-GPU layer on the same step."""
    import expert_offload_serving_b200 as moe
    from expert_offload_serving_b200.layer import MoeLayer
    cfg = synth.CONFIGS["split_merge"]
    s = moe.shape(cfg.E, cfg.d, cfg.I, cfg.fmt)
    B = host_pool.shape[1]
    dev_buf = torch.empty((4, B), dtype=torch.uint8, device="cuda")
    bw = moe.moe_profile_bandwidth(s, host_pool, 16, dev_buf.view(-1), n_threads=threads)
    del dev_buf
    full = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, device_pool=host_pool.cuda())   # all-GPU reference
    trace = synth.make_trace(cfg, T, steps=warm + steps, seed=0)
    lgs = [lg.cuda() for lg, _ in trace]
    xs = [x.cuda() for _, x in trace]
    rows = []
    for q in [i / 10 for i in range(11)] + [None]:
        layer = MoeLayer(cfg.E, cfg.d, cfg.I, cfg.fmt, cfg.k, T, host_pool=host_pool, n_slots=cfg.n_slots)
        step_ms, host_ms, n_fill, n_host, n_miss = [], [], 0, 0, 0
        dev_max = dev_mean = 0.0
        for t in range(warm + steps):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            res = layer.split_step(t, lgs[t], xs[t], q=q, bw=bw, threads=threads)
            torch.cuda.synchronize()
            dt = (time.perf_counter() - t0) * 1e3
            if t < warm:
                continue
            step_ms.append(dt)
            host_ms.append(res["host_ms"])
            n_fill += len(res["fills"])
            n_host += len(res["host"])
            n_miss += len(res["filled"]) + len(res["host"])
            if t == warm + steps - 1:
                out = layer.out[:T].clone()
                ref = full.forward(lgs[t], xs[t]).clone()
                err = (out - ref).abs()
                dev_max = float(err.max() / ref.abs().max())
                dev_mean = float(err.mean() / ref.abs().mean())
        moe.moe_check_status(layer.status)
        layer.cache.close()
        rows.append({"q": "q*" if q is None else q, "step_ms": round(statistics.median(step_ms), 3),
                     "tokens_per_s": round(T / (statistics.median(step_ms) / 1e3), 1),
                     "host_ms": round(statistics.median(host_ms), 3),
                     "misses_per_step": round(n_miss / steps, 2), "fills_per_step": round(n_fill / steps, 2),
                     "host_experts_per_step": round(n_host / steps, 2),
                     "merge_vs_all_gpu": {"max_rel": float(f"{dev_max:.3e}"), "mean_rel": float(f"{dev_mean:.3e}")}})
    del full
    best = min(r["step_ms"] for r in rows if r["q"] != "q*")
    qs = next(r for r in rows if r["q"] == "q*")
    return {
        "workload": f"split_merge: E={cfg.E} k={cfg.k} d={cfg.d} I={cfg.I} T={T}, {cfg.n_slots} slots, AR(1) "
                    f"trace; misses split by q, host share on the CPU ({threads or 'all'} threads) concurrently "
                    "with the fills",
        "bandwidth_profile": {"h2d_pinned_gbs": round(bw[0], 1), "host_kernel_gbs": round(bw[1], 1)},
        "steps": steps, "warmup_steps": warm, "timing": "median step wall time, host sync to host sync",
        "sweep": rows,
        "q_star_step_ms_over_best": round(qs["step_ms"] / best, 3),
    }


# ---------------------------------------------------------------- CPU oracle arms
def _cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_step(cfg, T_sample, seed, weights_cache):
    from oracle import moe as M
    logits, x = synth.make_routing(cfg, T_sample, seed)

    def w(e):
        if e not in weights_cache:
            ww = synth.make_experts(cfg, [e], 0, device="cpu")
            weights_cache[e] = M.dequant_expert(cfg.fmt, ww, 0)
        return weights_cache[e]
    return M.moe_layer(x.double().numpy(), logits.numpy(), cfg.k, w)


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return _cpu_cores()


def cpu_baseline(cfg, T, seconds=10.0):
    """The oracle as it stands, on the host cores: repeated float64 layer
    passes over one batch of T tokens of the same workload until `seconds`
    have elapsed (expert weights generated and dequantised before timing)."""
    from oracle import moe as M
    cache = {}
    logits, x = synth.make_routing(cfg, T, 99)
    idx, _ = M.route_topk(logits.numpy(), cfg.k)
    for e in sorted(set(idx.ravel().tolist())):
        ww = synth.make_experts(cfg, [e], 0, device="cpu")
        cache[e] = M.dequant_expert(cfg.fmt, ww, 0)
    xs, ls = x.double().numpy(), logits.numpy()
    passes = 0
    t0 = time.perf_counter()
    while True:
        M.moe_layer(xs, ls, cfg.k, lambda e: cache[e])
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= seconds or passes >= 1000:
            break
    return {"value": round(passes * T / dt, 2), "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{passes} float64 oracle passes over one batch of T={T} tokens of the decode_bf16 "
                      f"workload ({len(cache)} experts; weights dequantised before timing)",
            "seconds": round(dt, 2), **cpu_info()}


def run_reference(args, rank, world):
    """The reference arm: the float64 oracle on the host cores, on the GPU
    arm's workload and batch (decode_bf16, T = --tokens), each step one batch
    with fresh routing.  The timed steps are capped so that the arm ends
    within a few minutes; the line reports how many ran."""
    if rank != 0:
        return None
    cfg = synth.CONFIGS["decode_bf16"]
    T_s = args.tokens
    from oracle import moe as M
    # every expert generated and dequantised before timing (as for
    # cpu_baseline): the timed steps are the oracle's layer passes only
    cache = {}
    for e in range(cfg.E):
        ww = synth.make_experts(cfg, [e], 0, device="cpu")
        cache[e] = M.dequant_expert(cfg.fmt, ww, 0)
    for i in range(min(args.warmup, 3)):
        oracle_step(cfg, T_s, 5000 + i, cache)
    budget_s = 150.0
    t0 = time.perf_counter()
    done = 0
    for i in range(args.steps):
        oracle_step(cfg, T_s, 6000 + i, cache)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    v = done * T_s / dt
    workload = f"{cfg.name}: E={cfg.E} k={cfg.k} d={cfg.d} I={cfg.I} T={T_s}, all experts resident"
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": done, "steps_requested": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / done * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload, "global_batch": T_s, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(v, 2), "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
                         "sample": f"{done} steps of {T_s} tokens (fresh routing each step, capped at "
                                   f"{budget_s:.0f} s); all {cfg.E} experts' weights generated and dequantised "
                                   "before timing", **cpu_info()},
        "e2e": {"value": round(v, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--tokens", type=int, default=64, help="tokens per step (1, 16 or 64)")
    ap.add_argument("--replicas", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the FP4 prefill measurement")
    ap.add_argument("--config", default="decode_bf16", choices=["decode_bf16", "decode_mxfp4"],
                    help="decode workload of the main line (default: decode_bf16)")
    ap.add_argument("--only-prefill", action="store_true", help="print only the FP4 prefill measurement")
    ap.add_argument("--prefill-T", type=int, default=0, help="with --only-prefill: this token count only")
    ap.add_argument("--prefill-E", type=int, default=None,
                    help="with --only-prefill: this many experts instead of 256 (smaller captures)")
    ap.add_argument("--no-cached", action="store_true", help="skip the expert-cache decode measurement")
    ap.add_argument("--no-sweep", action="store_true", help="skip the T=1 and T=16 decode points")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus)
    if args.only_prefill:
        Ts = (args.prefill_T,) if args.prefill_T else ((4096,) if args.no_sweep else (4096, 16384, 32768))
        res = run_prefill(iters=max(3, min(args.steps, 50)), warmup=args.warmup, Ts=Ts, E=args.prefill_E)
        print(json.dumps(res[0] if len(res) == 1 else res), flush=True)
        return
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_gpu(args, rank, world, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
