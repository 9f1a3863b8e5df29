"""Benchmark of the FP4 W4A16 decode GEMM on the LLaMA-7B-shaped decode
workload (three weight matrices 4096x4096, 11008x4096, 4096x11008, E2M1,
group 128, fp16 scales; activations with M in {1, 8, 16, 64} rows).

One step = the decode sweep: fp4_gemm for every (M, matrix) pair, 12 calls,
on weights already quantized and resident in HBM.  The metric is weight
GB/s: packed codes + scales streamed per step / step time (all ranks).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Also measured in the same run and reported under "parts": the quantize
pass (GB/s), the prefill GEMM at M = 2048 (TFLOP/s) on the LLaMA-7B
prefill workload with the pre-shift, the format/bias search on a
LLaMA-13B-shaped 5120x5120 matrix, and passes over the full 40-layer
LLaMA-13B-shaped linear stack (6.54 GB packed): decode at M in {1, 4, 16,
64} (weight GB/s, tokens/s-equivalent) and prefill at M = 2048.
``--impl reference`` times the CPU oracle on a bounded sample of the same
workload, in the same unit.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fp4_gemm decode weight-GB/s vs HBM peak; prefill TFLOP/s vs bf16 tensor peak"
SHAPES = ((4096, 4096), (11008, 4096), (4096, 11008))
MS = (1, 8, 16, 64)
GROUP = 128


def weight_bytes(N, K, group=GROUP, scale_bytes=2):
    return N * K // 2 + N * (K // group) * scale_bytes


def step_weight_bytes():
    return sum(weight_bytes(N, K) for (N, K) in SHAPES) * len(MS)


# Nominal B200 figures, reported beside the measured denominators: HBM3e
# 8 TB/s (DGX datasheet), dense bf16 2.25 PFLOP/s (half the 2:4-sparse figure).
SPEC_HBM_GBS = 8000.0
SPEC_BF16_TFLOPS = 2250.0


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _code_only(text):
    """C++ source without comments and blank lines (string literals kept)."""
    import re
    pat = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', re.S)
    text = pat.sub(lambda m: m.group(0) if m.group(0).startswith('"') else "", text)
    return "\n".join(l.rstrip() for l in text.splitlines() if l.strip())


def kernel_sources_sha():
    """Digest of the CUDA sources' code (comments and blank lines dropped):
    per-launch DRAM traffic recorded under profiles/ is valid only for the
    kernels it was measured on."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "w4a16_gemm_fp4_b200", "csrc")
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh")):
            h.update(f.encode())
            h.update(_code_only(open(os.path.join(d, f), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(key):
    """DRAM bytes (read + write) of one launch, from an ncu capture recorded
    in profiles/traffic.json; None when absent or taken on other sources."""
    try:
        d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    except Exception:
        return None
    e = d.get("launches", {}).get(key)
    if not e or d.get("sources_sha") != kernel_sources_sha():
        return None
    return e["dram_bytes"]


def rowblk_fits(M, K):
    """Whether the library's group-128 row-block decode kernel takes this
    shape (its shared-memory plan: activations staged once per CTA, 16-row
    block buffers of codes and scale rows, the cross-warp reduction area)."""
    if K > 24576 or M > 16:
        return False

    def smem(nw, nbuf):
        return nbuf * (16 * (K // 2) + 16 * (K // 128) * 4) + M * (2 * K + 64) + \
            2 * nw * 32 * 4 * 4 * (2 if M > 8 else 1) + 128
    return any(2 * (smem(8, nb) + 1024 + 128) <= 228 * 1024 or smem(16, nb) <= 226 * 1024 for nb in (2, 1))


def gemm_kernel_name(api, M, N, K):
    """Kernel that serves an E2M1 group-128 GEMM of this shape (automatic
    engine): the row-block or streaming decode kernel, or the tensor
    engine's token tile."""
    if api.gemm_engine_for(M, N, K, GROUP) == api.ENGINE_DECODE:
        return "gemm_rowblk_kernel" if rowblk_fits(M, K) else "gemm_skinny_kernel"
    return "gemm_tcg_kernel<%d>" % (16 if M <= 16 else 32 if M <= 32 else 64 if M <= 64 else 128)


def launches_per_call(api, M, N, K):
    """Kernels one such call launches: the tensor engine's E2M1 token tiles
    other than 64 tokens take an activation pre-pass (f16 rows) first."""
    if api.gemm_engine_for(M, N, K, GROUP) == api.ENGINE_DECODE:
        return 1
    return 1 if 32 < M <= 64 else 2


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- distributed

def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value):
    """The largest of the ranks' values (device time: the slowest rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world, bytes_per_rank_step, steps, ms_max):
    """Weight GB/s of the whole job: the bytes every rank streamed over the
    slowest rank's time (replicas: each rank runs the full sweep)."""
    return world * bytes_per_rank_step * steps / (ms_max * 1e-3) / 1e9


# --------------------------------------------------------------- our arm

def build_workload(api, torch, copies):
    """Quantize the three matrices once, then replicate the packed weights
    into `copies` buffers so that consecutive steps read different memory
    (total > L2)."""
    from w4a16_gemm_fp4_b200 import synth
    cases = synth.llama7b_decode()
    mats = []
    for (N, K), case in zip(SHAPES, cases):
        W = torch.from_numpy(case["W"]).cuda()
        q = api.quantize(W, GROUP, api.E2M1, False, None, "f16")
        del W
        reps = [(q["packed"].clone(), q["scales"].clone()) for _ in range(copies)]
        xs = {M: torch.from_numpy(case["X"][M].view(np.int16)).cuda().view(torch.bfloat16) for M in MS}
        mats.append({"N": N, "K": K, "reps": reps, "X": xs})
    return mats, cases


def capture(torch, fn, stream):
    """Capture fn() (a sequence of library calls) into a CUDA graph."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def run_ours(args, world, rank):
    import torch
    from w4a16_gemm_fp4_b200 import api, build
    build.build()
    api.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = read_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per_copy = sum(weight_bytes(N, K) for (N, K) in SHAPES)
    copies = max(4, int(np.ceil(4 * l2 / per_copy)))
    mats, cases = build_workload(api, torch, copies)
    keys = [(i, M) for M in MS for i in range(len(mats))]
    outs = {(i, M): torch.empty((M, mats[i]["N"]), dtype=torch.bfloat16, device=dev) for (i, M) in keys}
    wss = {}
    for (i, M) in keys:
        nb = api.gemm_workspace_size(M, mats[i]["N"], mats[i]["K"])
        wss[(i, M)] = torch.zeros(max(nb, 16), dtype=torch.uint8, device=dev) if nb else None
    stream = torch.cuda.Stream()

    def sweep(c):
        for (i, M) in keys:
            packed, scales = mats[i]["reps"][c]
            api.gemm(mats[i]["X"][M], packed, scales, api.E2M1, GROUP, out=outs[(i, M)], workspace=wss[(i, M)])

    with torch.cuda.stream(stream):
        for s in range(args.warmup):          # eager warm-up (also loads modules, sets attributes)
            sweep(s % copies)
    torch.cuda.synchronize()
    # one graph per weight copy holding the 12 launches back to back (the
    # timed step); per-launch durations come from separate graphs that each
    # hold one call, back to back over the weight copies (no event nodes
    # between launches, so the launches overlap as they do in the step)
    graphs = [capture(torch, lambda c=c: sweep(c), stream) for c in range(copies)]

    def one_call(key, c):
        i, M = key
        packed, scales = mats[i]["reps"][c]
        api.gemm(mats[i]["X"][M], packed, scales, api.E2M1, GROUP, out=outs[key], workspace=wss[key])
    call_graphs = {k: capture(torch, lambda k=k: [one_call(k, c) for c in range(copies)], stream) for k in keys}
    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            graphs[s % copies].replay()
    torch.cuda.synchronize()
    api.device_status(clear=True)

    # clock sampler: soak ~1.5 s of the same replays so that nvidia-smi has
    # samples under this load, then the timed region
    clocks = ClockSampler(dev.index)
    clocks.start()
    t_end = time.time() + args.soak_s
    with torch.cuda.stream(stream):
        s = 0
        while time.time() < t_end:
            for _ in range(50):
                graphs[s % copies].replay()
                s += 1
            stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        for s in range(args.steps):
            graphs[s % copies].replay()
        t1.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(world, t0.elapsed_time(t1))
    # per-launch durations: each call's graph replayed back to back
    per = {}
    reps = max(3, min(40, args.steps // 50))
    with torch.cuda.stream(stream):
        for k in keys:
            call_graphs[k].replay()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                call_graphs[k].replay()
            b.record()
            b.synchronize()
            per[k] = a.elapsed_time(b) / (reps * copies)
    torch.cuda.synchronize()
    del call_graphs
    st = api.device_status(clear=True)
    if st:
        raise RuntimeError("device status %#x during the timed region" % st)

    value = whole_job_gbs(world, step_weight_bytes(), args.steps, ms)
    per_sum_ms = sum(per.values())

    groups = {}
    for (i, M), t in per.items():
        eng = "/".join(sorted({"decode" if api.gemm_engine_for(M, N, K, GROUP) == api.ENGINE_DECODE else "tensor"
                               for (N, K) in SHAPES}))
        g = groups.setdefault((eng, M), {"ms": 0.0, "bytes": 0.0, "launches": 0})
        g["ms"] += t
        g["launches"] += 1
    # roofline of the dominant launch: algorithmic bytes (packed codes +
    # scales + activations + output) over its average duration
    (idom, Mdom) = max(per, key=lambda k: per[k])
    Nd, Kd = mats[idom]["N"], mats[idom]["K"]
    alg = weight_bytes(Nd, Kd) + Mdom * Kd * 2 + Mdom * Nd * 2
    achieved = alg / (per[(idom, Mdom)] * 1e-3) / 1e9
    kname = gemm_kernel_name(api, Mdom, Nd, Kd)
    key = "%s %dx%d M=%d" % (kname, Nd, Kd, Mdom)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "frac_of_spec": round(achieved / SPEC_HBM_GBS, 4),
                "traffic": recorded_traffic(key),
                "kernel": key, "algorithmic_bytes": alg, "us_per_launch": round(per[(idom, Mdom)] * 1e3, 2),
                "peak_source": peaks["source"] + " (burst copy)",
                "share_of_step": round(per[(idom, Mdom)] / sum(per.values()), 3)}
    per_m = {}
    for (eng_, M), gg in sorted(groups.items(), key=lambda kv: kv[0][1]):
        per_m[str(M)] = {"engine": eng_, "us_per_3_matrices": round(gg["ms"] * 1e3, 2),
                         "weight_gbs": round(sum(weight_bytes(N, K) for (N, K) in SHAPES) / (gg["ms"] * 1e-3) / 1e9,
                                             1),
                         "us_per_launch": [round(per[(i, M)] * 1e3, 2) for i in range(len(mats))]}

    e2e = None if args.no_e2e else run_e2e(api, torch, mats, args, stream, world)
    parts = {}
    if not args.no_parts and rank == 0:
        parts = run_parts(api, torch, peaks, dev, stream)
        if not args.no_stack:
            try:
                parts["llama13b_stack"] = run_stack(api, torch, peaks, dev, stream)
            except Exception as exc:  # reported, never fatal to the bench line
                parts["llama13b_stack"] = {"error": "%s: %s" % (type(exc).__name__, exc)}
    return {
        "value": value, "ms_per_step": ms / args.steps, "roofline": roofline, "clocks": clk, "e2e": e2e,
        "per_launch_sum_ms": per_sum_ms,
        "gpu_launches": sum(launches_per_call(api, k[1], *SHAPES[k[0]]) for k in keys) * args.steps, "per_m": per_m, "parts": parts, "copies": copies,
        "copy_bytes": per_copy * copies, "l2_bytes": l2,
    }


def run_e2e(api, torch, mats, args, stream, world):
    """The same sweep through the public API with host buffers: every step
    copies each X from pinned host memory to the device and reads every Y
    back (captured once into graphs, replayed per step)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    keys = [(i, M) for M in MS for i in range(len(mats))]
    hx, hy, dx, dy = {}, {}, {}, {}
    h2d = d2h = 0
    for (i, M) in keys:
        hx[(i, M)] = mats[i]["X"][M].cpu().pin_memory()
        hy[(i, M)] = torch.empty((M, mats[i]["N"]), dtype=torch.bfloat16).pin_memory()
        dx[(i, M)] = torch.empty_like(mats[i]["X"][M])
        dy[(i, M)] = torch.empty((M, mats[i]["N"]), dtype=torch.bfloat16, device=dev)
        h2d += hx[(i, M)].numel() * 2
        d2h += hy[(i, M)].numel() * 2
    copies = len(mats[0]["reps"])
    wss = {k: (lambda nb: torch.zeros(max(nb, 16), dtype=torch.uint8, device=dev) if nb else None)(
        api.gemm_workspace_size(k[1], mats[k[0]]["N"], mats[k[0]]["K"])) for k in keys}

    def step(c):
        for (i, M) in keys:
            dx[(i, M)].copy_(hx[(i, M)], non_blocking=True)
            packed, scales = mats[i]["reps"][c]
            api.gemm(dx[(i, M)], packed, scales, api.E2M1, GROUP, out=dy[(i, M)], workspace=wss[(i, M)])
            hy[(i, M)].copy_(dy[(i, M)], non_blocking=True)

    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            step(s % copies)
    torch.cuda.synchronize()
    graphs = [capture(torch, lambda c=c: step(c), stream) for c in range(copies)]
    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            graphs[s % copies].replay()
    torch.cuda.synchronize()
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        for s in range(args.steps):
            graphs[s % copies].replay()
        t1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(world, t0.elapsed_time(t1))
    v = step_weight_bytes() * args.steps * world / (ms * 1e-3) / 1e9
    return {"value": round(v, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def time_graph(torch, fn, stream, iters, warm=3):
    """Mean time of fn() replayed from a CUDA graph (no host overhead)."""
    with torch.cuda.stream(stream):
        for _ in range(warm):
            fn()
    torch.cuda.synchronize()
    g = capture(torch, fn, stream)
    with torch.cuda.stream(stream):
        g.replay()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            g.replay()
        b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def run_parts(api, torch, peaks, dev, stream):
    from w4a16_gemm_fp4_b200 import synth
    out = {}
    # quantize pass (E2M1, group 128, fp16 scales) over the three decode matrices
    rng = np.random.default_rng(1)
    Ws = [torch.from_numpy(synth.lognormal_row_weights(rng, N, K)).cuda() for (N, K) in SHAPES]
    outs = [api.quantize(W, GROUP, api.E2M1) for W in Ws]

    def qpass():
        for W, o in zip(Ws, outs):
            api.quantize_into(W, o["packed"], o["scales"], o["choice"], GROUP, api.E2M1)
    ms = time_graph(torch, qpass, stream, 20)
    qbytes = sum(N * K * 4 + weight_bytes(N, K) for (N, K) in SHAPES)
    out["quantize"] = {"workload": "3 LLaMA-7B decode matrices, E2M1 g128 fp16 scales", "ms": round(ms, 4),
                       "gbs": round(qbytes / (ms * 1e-3) / 1e9, 1),
                       "frac_hbm": round(qbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    del Ws, outs
    # prefill with the pre-shift: GEMM M = 2048 on 4096x4096 and 11008x4096
    case = synth.llama7b_prefill()
    X = torch.from_numpy(case["X"].view(np.int16)).cuda().view(torch.bfloat16)
    shift, rho = api.preshift_calibrate(X)
    Xt = api.preshift_apply(X, shift, rho)
    qs = [api.quantize(torch.from_numpy(W).cuda(), GROUP, api.E2M1, False, shift) for W in case["W"]]
    ys = [torch.empty((X.shape[0], W.shape[0]), dtype=torch.bfloat16, device=dev) for W in case["W"]]

    def prefill():
        for q, y in zip(qs, ys):
            api.gemm(Xt, q["packed"], q["scales"], api.E2M1, GROUP, x_scale=rho, out=y)
    ms = time_graph(torch, prefill, stream, 20)
    flops = sum(2.0 * X.shape[0] * N * K for (N, K) in ((4096, 4096), (11008, 4096)))
    tf = flops / (ms * 1e-3) / 1e12
    out["prefill"] = {"workload": "LLaMA-7B prefill X 2048x4096 (1% outlier channels x50), pre-shift on, "
                                  "W 4096x4096 + 11008x4096; each call includes its f16 activation pre-pass",
                      "ms": round(ms, 4), "tflops": round(tf, 1),
                      "peak_tflops": peaks["bf16_tflops"], "frac": round(tf / peaks["bf16_tflops"], 4),
                      "frac_of_spec": round(tf / SPEC_BF16_TFLOPS, 4)}
    ws_cal = torch.zeros(api.lib().fp4_preshift_workspace_size(*X.shape), dtype=torch.uint8, device=dev)
    ms_pro = time_graph(torch, lambda: api.preshift_apply(X, shift, rho, out=Xt), stream, 20)
    out["preshift_apply"] = {"ms": round(ms_pro, 4), "gbs": round(2 * 2 * X.numel() / (ms_pro * 1e-3) / 1e9, 1)}
    # the same prefill with 4-bit activations: activation codes against the
    # calibrated per-tensor scale (the channel powers of two are in the
    # weights), then the W4A4 product on the same weights
    ap, a_scale = api.act_quantize(X, rho, api.E2M1, 0, shift)
    ms_aq = time_graph(torch, lambda: api.act_quantize(X, rho, api.E2M1, 0, shift, out=ap, a_scale=a_scale),
                       stream, 20)
    aq_bytes = 2.5 * X.numel()
    out["act_quantize"] = {"workload": "X bf16 2048x4096 (1% outlier channels x50) -> E2M1 codes, pre-shift on",
                           "ms": round(ms_aq, 4), "gbs": round(aq_bytes / (ms_aq * 1e-3) / 1e9, 1),
                           "frac_hbm": round(aq_bytes / (ms_aq * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    ws4 = torch.zeros(max(api.gemm_w4a4_workspace_size(X.shape[0], N, K) for (N, K) in
                          ((4096, 4096), (11008, 4096))), dtype=torch.uint8, device=dev)

    def prefill_w4a4():
        api.act_quantize(X, rho, api.E2M1, 0, shift, out=ap, a_scale=a_scale)
        for q, y in zip(qs, ys):
            api.gemm_w4a4(ap, a_scale, q["packed"], q["scales"], api.E2M1, api.E2M1, GROUP, out=y, workspace=ws4)
    ms = time_graph(torch, prefill_w4a4, stream, 20)
    tf = flops / (ms * 1e-3) / 1e12
    out["w4a4_prefill"] = {"workload": "LLaMA-7B prefill in W4A4: act_quantize of X 2048x4096 + the product on "
                                       "W 4096x4096 + 11008x4096; each call includes its activation expansion",
                           "ms": round(ms, 4), "tflops": round(tf, 1), "frac": round(tf / peaks["bf16_tflops"], 4)}
    del X, Xt, qs, ys, ws_cal, ap, a_scale, ws4
    # LLaMA-13B search workload: the per-tensor format/bias search (3 formats
    # x 8 bias candidates, then the pack) on each Student-t matrix, then the
    # W4A16 GEMM at M = 512 on the searched weights
    case = synth.llama13b_search()
    X = torch.from_numpy(case["X"].view(np.int16)).cuda().view(torch.bfloat16)
    out["search"] = {}
    out["gemm_m512"] = {}
    for W_np in case["W"]:
        N, K = W_np.shape
        W = torch.from_numpy(W_np).cuda()
        o = api.quantize(W, GROUP, api.AUTO, True)
        ms = time_graph(torch, lambda: api.quantize_into(W, o["packed"], o["scales"], o["choice"], GROUP,
                                                         api.AUTO, True), stream, 5, warm=1)
        fmt = int(o["choice"][0].item())
        out["search"]["%dx%d" % (N, K)] = {
            "workload": "%dx%d Student-t(5)*0.015, 3 formats x 8 bias candidates + group-128 pack" % (N, K),
            "ms": round(ms, 3), "candidate_evals_per_s": round(24 * W.numel() / (ms * 1e-3), 0),
            "format_chosen": fmt}
        del W
        Y = torch.empty((X.shape[0], N), dtype=torch.bfloat16, device=dev)
        ms = time_graph(torch, lambda: api.gemm(X, o["packed"], o["scales"], fmt, GROUP, out=Y), stream, 20)
        tf = 2.0 * X.shape[0] * N * K / (ms * 1e-3) / 1e12
        out["gemm_m512"]["%dx%d" % (N, K)] = {
            "workload": "X bf16 512x5120 ~ N(0,1) . searched %dx%d weights (format %d, g128, fp16 scales)" % (
                N, K, fmt),
            "ms": round(ms, 4), "tflops": round(tf, 1), "frac": round(tf / peaks["bf16_tflops"], 4),
            "frac_of_spec": round(tf / SPEC_BF16_TFLOPS, 4)}
        del o, Y
    # scale granularity on the 13B projections: one scale per attention
    # head (40 heads of 128 rows) with the bias searched per head on the q
    # projection, and one per output channel on the gate projection
    out["quantize_blocks"] = {}
    for (W_np, gran, heads, bias, name) in ((case["W"][0], api.GRAN_HEAD, 40, -1, "head40_search"),
                                            (case["W"][1], api.GRAN_CHANNEL, 0, 0, "channel")):
        N, K = W_np.shape
        W = torch.from_numpy(W_np).cuda()
        ms = time_graph(torch, lambda: api.quantize_blocks(W, GROUP, gran, heads, api.E2M1, bias), stream, 5,
                        warm=1)
        out["quantize_blocks"]["%dx%d_%s" % (N, K, name)] = {
            "workload": "%dx%d Student-t(5)*0.015, E2M1, scales per %s%s" % (
                N, K, "attention head (40 x 128 rows)" if heads else "output channel",
                ", bias index searched per block" if bias < 0 else ""),
            "ms": round(ms, 4), "weight_gbs_read": round(4.0 * N * K / (ms * 1e-3) / 1e9, 1)}
        del W
    return out


def run_stack(api, torch, peaks, dev, stream, layers=40):
    """The full LLaMA-13B-shaped linear stack: 40 layers x {q, k, v, o
    5120x5120; gate, up 13824x5120; down 5120x13824}, weights drawn on the
    GPU and quantized to E2M1 g128 fp16 scales (6.54 GB packed, far beyond
    L2).  One pass = the 280 fp4_gemm calls in layer order; decode passes at
    M in {1, 4, 16, 64} give weight GB/s and tokens/s-equivalent (M rows per
    pass, linear layers only), one prefill pass at M = 2048 gives TFLOP/s."""
    from w4a16_gemm_fp4_b200 import synth
    mats = []
    fused = []  # per layer: q, k, v, o, gate/up interleaved (SiLU-gated), down
    for layer in range(layers):
        lay = {}
        for name, w in synth.stack_layer_weights(layer, device=dev):
            q = api.quantize(w, GROUP, api.E2M1)
            mats.append((q["packed"], q["scales"], w.shape[0], w.shape[1]))
            lay[name] = mats[-1]
            del w, q
        g, u = lay["gate"], lay["up"]
        # quantization is per row, so the interleaved rows are the quantized
        # rows interleaved: row 2i = gate row i, row 2i+1 = up row i
        gu_p = torch.stack((g[0], u[0]), dim=1).reshape(2 * g[2], g[0].shape[1])
        gu_s = torch.stack((g[1], u[1]), dim=1).reshape(2 * g[2], g[1].shape[1])
        for name in ("q", "k", "v", "o"):
            fused.append(lay[name] + (api.ACT_NONE,))
        fused.append((gu_p, gu_s, 2 * g[2], g[3], api.ACT_SILU_GATE))
        fused.append(lay["down"] + (api.ACT_NONE,))
    torch.cuda.synchronize()
    wbytes = sum(weight_bytes(N, K) for (_, _, N, K) in mats)
    dims = sorted({K for (_, _, _, K) in mats} | {N for (_, _, N, _) in mats})
    gen = torch.Generator(device=dev)
    gen.manual_seed(4)
    out = {"workload": "llama13b_stack: %d layers x 7 matrices, E2M1 g128 fp16 scales, weights ~ N(0, 0.02^2) "
                       "drawn on the GPU; X ~ N(0, 1) bf16" % layers,
           "matrices": len(mats), "weight_bytes": wbytes}
    for M in (1, 4, 16, 64, 2048):
        xs = {d: torch.randn((M, d), generator=gen, device=dev).to(torch.bfloat16) for d in dims}
        ys = {d: torch.empty((M, d), dtype=torch.bfloat16, device=dev) for d in dims}

        def one_pass():
            for (pk, sc, N, K) in mats:
                api.gemm(xs[K], pk, sc, api.E2M1, GROUP, out=ys[N])

        def fused_pass():
            for (pk, sc, N, K, act) in fused:
                api.gemm(xs[K], pk, sc, api.E2M1, GROUP, out=ys[N // 2] if act else ys[N], act=act)
        ms = time_graph(torch, one_pass, stream, 3 if M < 2048 else 2, warm=1)
        if M < 2048:
            gbs = wbytes / (ms * 1e-3) / 1e9
            out["decode_M%d" % M] = {"ms_per_pass": round(ms, 4), "weight_gbs": round(gbs, 1),
                                     "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                     "frac_hbm_spec": round(gbs / SPEC_HBM_GBS, 4),
                                     "tokens_per_s_equiv": round(M / (ms * 1e-3), 1)}
            # the same pass with each layer's gate and up projections fused in
            # one call (interleaved rows, SiLU-gated epilogue): 240 calls
            ms = time_graph(torch, fused_pass, stream, 3, warm=1)
            gbs = wbytes / (ms * 1e-3) / 1e9
            out["decode_M%d_fused_mlp" % M] = {"ms_per_pass": round(ms, 4), "weight_gbs": round(gbs, 1),
                                               "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                               "tokens_per_s_equiv": round(M / (ms * 1e-3), 1)}
        else:
            tf = sum(2.0 * M * N * K for (_, _, N, K) in mats) / (ms * 1e-3) / 1e12
            out["prefill_M2048"] = {"ms_per_pass": round(ms, 3), "tflops": round(tf, 1),
                                    "frac": round(tf / peaks["bf16_tflops"], 4),
                                    "frac_of_spec": round(tf / SPEC_BF16_TFLOPS, 4)}
        del xs, ys
    del mats, fused
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------- CPU oracle

SAMPLE_ROW_DIV = 16  # the CPU sample: every sweep call on the first 1/16 of each matrix's rows


def oracle_sample(row_div=SAMPLE_ROW_DIV, threads=None):
    """Time the CPU oracle (fp64 GEMM on dequantized weights) on a bounded
    sample of the decode sweep: all 12 calls (every M, every matrix), each
    on the first N/row_div rows of its matrix.  The oracle's work is linear
    in the row count, so the sample's time x row_div is the sweep's time.
    Returns (weight GB/s of the sweep, threads used, description)."""
    import oracle
    from w4a16_gemm_fp4_b200 import synth
    oracle.build()
    if threads is not None:
        oracle.set_num_threads(threads)
    cores = oracle.num_threads()
    cases = synth.llama7b_decode()
    quant = [oracle.quantize(c["W"][: c["W"].shape[0] // row_div], GROUP, oracle.E2M1) for c in cases]
    t_total = 0.0
    for M in MS:
        for c, q in zip(cases, quant):
            t0 = time.perf_counter()
            oracle.gemm(c["X"][M], q["packed"], q["scales"], oracle.E2M1, GROUP)
            t_total += time.perf_counter() - t0
    sweep_s = t_total * row_div
    gbs = step_weight_bytes() / sweep_s / 1e9
    return gbs, cores, ("oracle fp64 GEMM, all 12 sweep calls on the first 1/%d of each matrix's rows (%.2f s), "
                        "scaled to the full sweep by the row count" % (row_div, t_total))


def cpu_baselines():
    """The oracle on all host cores and on one thread, same sample."""
    import oracle
    gbs, cores, desc = oracle_sample()
    gbs1, _, desc1 = oracle_sample(threads=1)
    oracle.set_num_threads(cores)
    return {"value": round(gbs, 5), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc,
            "host_cores": host_cores(),
            "single_thread": {"value": round(gbs1, 5), "unit": "GB/s", "cores": 1, "sample": desc1}}


def cpu_configs(threads_list=(0, 1), emit=None, single_row_div=16):
    """The oracle on the host cores for every configuration: configs 1-4
    (quantize/search/pack and GEMM, as the workloads define them) and config
    5 extrapolated from one matrix of each of its three shapes (x 4, 2 and 1
    per layer, x 40 layers; its M = 2048 prefill GEMM from the first 64
    rows, the oracle's work being linear in M).  threads 0 = all host
    cores: everything in full.  At one thread the quantizers run in full and
    each GEMM on the first 1/single_row_div of its weight rows, scaled by
    the row count (the oracle GEMM is linear in N), so the run stays within
    tens of minutes.  emit(record) receives each configuration's record as
    soon as it is done; the dict of all records is returned."""
    import oracle
    from w4a16_gemm_fp4_b200 import synth
    oracle.build()
    all_cores = oracle.num_threads()
    out = {"host_cores": host_cores(), "runs": {}}

    def t(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    for th in threads_list:
        nth = th if th > 0 else all_cores
        oracle.set_num_threads(nth)
        div = 1 if nth == all_cores and th == 0 else single_row_div
        r = {}

        def done(name, rec):
            rec["threads"] = nth
            rec["gemm_row_sample"] = "full" if div == 1 else "first 1/%d of the weight rows, x%d" % (div, div)
            r[name] = rec
            if emit:
                emit({"config": name, **rec})

        def gemm_s(X, q, N, fmt=oracle.E2M1, rho=1.0):
            n = max(1, N // div)
            return t(lambda: oracle.gemm(X, q["packed"][:n], q["scales"][:n], fmt, GROUP, rho)) * (N / n)

        c1 = synth.tiny()
        q = oracle.quantize(c1["W"], GROUP, oracle.E2M1, scale_dtype="f32")
        done("cfg1_tiny", {"quantize_s": t(lambda: oracle.quantize(c1["W"], GROUP, oracle.E2M1, scale_dtype="f32")),
                           "gemm_s": t(lambda: oracle.gemm(c1["X"], q["packed"], q["scales"], oracle.E2M1, GROUP))})
        c2 = synth.llama7b_decode()
        qs = []
        tq = 0.0
        for c in c2:
            t0 = time.perf_counter()
            qs.append(oracle.quantize(c["W"], GROUP, oracle.E2M1))
            tq += time.perf_counter() - t0
        tg = sum(gemm_s(c["X"][M], qq, c["W"].shape[0]) for M in MS for c, qq in zip(c2, qs))
        done("cfg2_llama7b_decode", {"quantize_s": tq, "gemm_sweep_s": tg,
                                     "weight_gbs": step_weight_bytes() / tg / 1e9})
        del c2, qs
        c3 = synth.llama7b_prefill()
        tc = t(lambda: oracle.preshift_calibrate(c3["X"]))
        shift, rho = oracle.preshift_calibrate(c3["X"])
        ta = t(lambda: oracle.preshift_apply(c3["X"], shift, rho))
        Xt = oracle.preshift_apply(c3["X"], shift, rho)
        tq = 0.0
        tg = 0.0
        flops = 0.0
        for W in c3["W"]:
            t0 = time.perf_counter()
            qq = oracle.quantize(W, GROUP, oracle.E2M1, shift=shift)
            tq += time.perf_counter() - t0
            tg += gemm_s(Xt, qq, W.shape[0], rho=rho)
            flops += 2.0 * Xt.shape[0] * W.shape[0] * W.shape[1]
        done("cfg3_llama7b_prefill", {"calibrate_s": tc, "apply_s": ta, "quantize_s": tq, "gemm_s": tg,
                                      "gflops": flops / tg / 1e9})
        del c3, Xt
        c4 = synth.llama13b_search()
        ts = 0.0
        tg = 0.0
        flops = 0.0
        for W in c4["W"]:
            t0 = time.perf_counter()
            qq = oracle.quantize(W, GROUP, oracle.AUTO, bias_search=True)
            ts += time.perf_counter() - t0
            tg += gemm_s(c4["X"], qq, W.shape[0], fmt=qq["choice"][0])
            flops += 2.0 * c4["X"].shape[0] * W.shape[0] * W.shape[1]
        done("cfg4_llama13b_search", {"search_and_pack_s": ts, "gemm_m512_s": tg, "gflops": flops / tg / 1e9})
        del c4
        # config 5: one matrix of each shape, counts per layer 4, 2, 1
        rng = np.random.default_rng(4)
        shapes = ((5120, 5120, 4), (13824, 5120, 2), (5120, 13824, 1))
        per_layer = {"quantize_s": 0.0}
        for M in (1, 4, 16, 64, 2048):
            per_layer["gemm_M%d_s" % M] = 0.0
        for (N, K, cnt) in shapes:
            W = synth.normal_weights(rng, N, K)
            t0 = time.perf_counter()
            qq = oracle.quantize(W, GROUP, oracle.E2M1)
            per_layer["quantize_s"] += cnt * (time.perf_counter() - t0)
            del W
            for M in (1, 4, 16, 64, 2048):
                Mt = min(M, 64)
                X = synth.activations(rng, Mt, K)
                per_layer["gemm_M%d_s" % M] += cnt * gemm_s(X, qq, N) * (M / Mt)
        rec = {k: v * 40 for k, v in per_layer.items()}
        rec["note"] = "one matrix of each shape timed, x {4,2,1} per layer x 40 layers; M=2048 from its first 64 rows"
        done("cfg5_llama13b_stack_extrapolated", rec)
        out["runs"]["threads_%d" % nth] = r
    oracle.set_num_threads(all_cores)
    return out


def run_reference(args, world, rank):
    if rank != 0:
        return None
    import oracle
    oracle.build()
    # each step is one bounded sample of the sweep: the cpu_baseline sample
    # (1/16 of the rows) when the run is short, fewer rows when many steps
    # are asked for, so that the run ends within a few minutes
    n = args.warmup + args.steps
    row_div = SAMPLE_ROW_DIV
    while n * 1.0 * SAMPLE_ROW_DIV / row_div > 40 and row_div < 1024:
        row_div *= 2
    vals = []
    desc = ""
    cores = 1
    for s in range(n):
        gbs, cores, desc = oracle_sample(row_div=row_div)
        if s >= args.warmup:
            vals.append(gbs)
    v = statistics.median(vals)
    return {"impl": "reference", "metric": METRIC, "value": round(v, 5), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_weight_bytes() / (v * 1e9) * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded PCG64 draws standing in for LLaMA-7B weights/activations)",
            "config": {"workload": "llama7b_decode: W 4096x4096, 11008x4096, 4096x11008 E2M1 g128 fp16 "
                                   "scales; M in {1,8,16,64}", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": round(v, 5), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": round(v, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def profile_case(case):
    """One configuration, three eager calls (the first loads modules and sets
    attributes; captures skip it)."""
    import torch
    from w4a16_gemm_fp4_b200 import api, build, synth
    build.build()
    kind, *dims = case.split(":")
    dims = [int(d) for d in dims]
    rng = np.random.default_rng(1)
    if kind == "gemm":
        N, K, M = dims
        W = torch.from_numpy(synth.lognormal_row_weights(rng, N, K)).cuda()
        q = api.quantize(W, GROUP, api.E2M1)
        del W
        X = torch.from_numpy(synth.activations(rng, M, K).view(np.int16)).cuda().view(torch.bfloat16)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            api.gemm(X, q["packed"], q["scales"], api.E2M1, GROUP, out=Y)
    elif kind == "w4a4":
        # the W4A4 product: outlier activations calibrated and coded to E2M1,
        # weights quantized with the same channel shift
        N, K, M = dims
        W = torch.from_numpy(synth.lognormal_row_weights(rng, N, K)).cuda()
        Xb, _ = synth.outlier_activations(rng, M, K)
        X = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)
        shift, rho = api.preshift_calibrate(X)
        q = api.quantize(W, GROUP, api.E2M1, False, shift)
        del W
        ap, a_scale = api.act_quantize(X, rho, api.E2M1, 0, shift)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            api.gemm_w4a4(ap, a_scale, q["packed"], q["scales"], api.E2M1, api.E2M1, GROUP, out=Y)
    elif kind == "quantize":
        N, K = dims
        W = torch.from_numpy(synth.lognormal_row_weights(rng, N, K)).cuda()
        o = api.quantize(W, GROUP, api.E2M1)
        for _ in range(3):
            api.quantize_into(W, o["packed"], o["scales"], o["choice"], GROUP, api.E2M1)
    else:
        raise SystemExit("unknown profile case " + case)
    torch.cuda.synchronize()
    st = api.device_status(clear=True)
    print("profile case %s done, device status %d" % (case, st))


def traffic_cmds():
    """One counter capture per kernel of the sweep (exact name, as many
    launches as the first eager warm-up sweep has of it), each a single-pass
    pair of DRAM byte counters."""
    from w4a16_gemm_fp4_b200 import api
    counts = {}
    for M in MS:
        for (N, K) in SHAPES:
            base = gemm_kernel_name(api, M, N, K).split("<")[0]
            counts[base] = counts.get(base, 0) + 1
    return {base: ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none -k regex:%s "
                   "-c %d --csv --log-file traffic_%s.csv python bench.py --steps 1 --warmup 3 --soak-s 0 "
                   "--no-parts --no-e2e --no-cpu-baseline" % (base, n, base))
            for base, n in sorted(counts.items())}


def record_traffic(csv_paths):
    """profiles/traffic.json from the per-kernel captures of traffic_cmds():
    each CSV lists its kernel's launches of the first eager warm-up sweep in
    key order (for M in MS, for each matrix); ncu flushes the caches before
    each profiled launch, so the bytes are cold-cache."""
    import csv
    from w4a16_gemm_fp4_b200 import api
    keys = [(i, M) for M in MS for i in range(len(SHAPES))]
    out = {}
    for path in csv_paths.split(","):
        vals, order = {}, []
        with open(path) as f:
            lines = [l for l in f if l.startswith('"')]
        for row in csv.DictReader(lines):
            lid = int(row["ID"])
            if lid not in vals:
                vals[lid] = {"name": row["Kernel Name"]}
                order.append(lid)
            v = float(row["Metric Value"].replace(",", ""))
            scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}.get(row.get("Metric Unit", "byte"), 1)
            vals[lid][row["Metric Name"]] = v * scale
        if not order:
            raise SystemExit("no launches in " + path)
        base = vals[order[0]]["name"].split("<")[0].split("(")[0].strip()
        mine = [k for k in keys if gemm_kernel_name(api, k[1], *SHAPES[k[0]]).split("<")[0] in base]
        if len(order) < len(mine):
            raise SystemExit("expected %d launches in %s, found %d" % (len(mine), path, len(order)))
        for (i, M), lid in zip(mine, order):
            N, K = SHAPES[i]
            kname = gemm_kernel_name(api, M, N, K)
            assert kname.split("<")[0] in vals[lid]["name"], (kname, vals[lid]["name"])
            d = vals[lid]
            out["%s %dx%d M=%d" % (kname, N, K, M)] = {
                "dram_bytes": int(d["dram__bytes_read.sum"] + d["dram__bytes_write.sum"]),
                "algorithmic_bytes": weight_bytes(N, K) + M * K * 2 + M * N * 2}
    doc = {"sources_sha": kernel_sources_sha(), "commands": traffic_cmds(), "launches": out}
    path = os.path.join(ROOT, "profiles", "traffic.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)
    print("wrote", path)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-parts", action="store_true", help="skip the quantize/prefill/search/stack legs")
    ap.add_argument("--no-stack", action="store_true", help="skip the 40-layer 13B-shaped stack leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg")
    ap.add_argument("--soak-s", type=float, default=1.5,
                    help="seconds of untimed replays before the timed region (clock sampling)")
    ap.add_argument("--profile-case", metavar="CASE",
                    help="run one case a few times and exit, for ncu captures: gemm:N:K:M (E2M1 g128 fp16 "
                         "scales, synthetic weights and activations), w4a4:N:K:M (4-bit activations) or "
                         "quantize:N:K")
    ap.add_argument("--cpu-configs", action="store_true",
                    help="time the CPU oracle on every configuration (1 thread and all cores), print JSON, exit")
    ap.add_argument("--record-traffic", metavar="CSV[,CSV]",
                    help="write profiles/traffic.json from the per-kernel ncu CSVs of traffic_cmds() "
                         "(dram__bytes_read.sum, dram__bytes_write.sum), then exit")
    ap.add_argument("--traffic-cmds", action="store_true", help="print the per-kernel traffic captures, exit")
    args = ap.parse_args()
    if args.record_traffic:
        record_traffic(args.record_traffic)
        return
    if args.traffic_cmds:
        for cmd in traffic_cmds().values():
            print(cmd)
        return
    if args.cpu_configs:
        cpu_configs(emit=lambda rec: print(json.dumps(rec), flush=True))
        return
    if args.profile_case:
        profile_case(args.profile_case)
        return
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    world, rank, local = dist_setup(args)
    res = run_ours(args, world, rank)
    if rank == 0:
        cpu = None if args.no_cpu_baseline else cpu_baselines()
        line = {
            "metric": METRIC, "value": round(res["value"], 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(res["ms_per_step"], 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded PCG64 draws standing in for LLaMA-7B weights/activations)",
            "config": {"workload": "llama7b_decode: W 4096x4096, 11008x4096, 4096x11008 E2M1 g128 fp16 scales; "
                                   "M in {1,8,16,64}; one step = 12 fp4_gemm calls",
                       "global_batch": sum(MS), "parallelism": "replicas" if world > 1 else "single",
                       "l2": "weights rotate over %d copies (%.0f MB) > 4x L2 (%d MB)" % (
                           res["copies"], res["copy_bytes"] / 1e6, res["l2_bytes"] // 2 ** 20)},
            "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": res["e2e"], "gpu_launches": res["gpu_launches"],
            "clocks": res["clocks"], "per_m": res["per_m"],
            "per_launch_sum_ms": round(res["per_launch_sum_ms"], 5),
            "per_launch_sum_over_step": round(res["per_launch_sum_ms"] / res["ms_per_step"], 3),
            "parts": res["parts"],
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
