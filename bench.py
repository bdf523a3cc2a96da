"""Benchmark: the weight-only quantized Linear of a DiT attention projection.

Workload (seeded, synthetic): W [4096, 4096] ~ N(0, 0.02) fp32 with 1% of the
input columns x20, RTN int8 per output channel; x bf16 [M, 4096] ~ N(0, 1)
for M in {16, 256, 4096}; bias [4096] ~ N(0, 0.01).  One step is one pass of
the whole path: quantize W and pack it (one fused pass), then the Linear at
M = 16, 256 and 4096
(inputs already in HBM; L2 flushed between steps).  value = total Linear
FLOPs (2 M N K) of all ranks / the max over ranks of the device time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun every rank runs an independent replica (weak scaling); there
is no collective on the data path.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import wlq_inputs as wi  # noqa: E402

N_OUT, K_IN, BITS, GROUP = 4096, 4096, 8, 0
MS = (16, 256, 4096)
METRIC = "quantized-linear TFLOP/s and HBM GB/s vs B200 roofline, M=16..4096"
WORKLOAD = ("DiT attention projection W8A16: W[4096,4096] fp32 N(0,0.02), 1% input columns x20, "
            "RTN int8 per output channel; x bf16 [M,4096] N(0,1), M in {16,256,4096}; bias N(0,0.01); "
            "step = quantize + pack (one fused pass over W) + Linear at the three M")
PROFILE = os.path.join(ROOT, "profiles", "gemm_w8_attn_m4096.txt")


def linear_flops():
    return sum(2.0 * M * N_OUT * K_IN for M in MS)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_only_quantized_rtn_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the M=4096 GEMM from the committed ncu summary,
    or None when the kernel sources changed since that capture."""
    if not os.path.exists(PROFILE):
        return None
    vals = {}
    for line in open(PROFILE):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.25)
        self.p.terminate()
        try:
            self.p.wait(5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [v for v in sm if v > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


def cpu_baseline(n_rows_per_m=(48, 192, 2832)):
    """The oracle as it stands on this host's cores: quantize the whole W, then
    the Linear for a bounded sample of rows of each M batch."""
    import oracle
    d = wi.attn_w8(1)
    W = d["W"]
    t0 = time.perf_counter()
    codes, scales = oracle.quantize(W, BITS, GROUP)
    flops = 0.0
    for M, nr in zip(MS, n_rows_per_m):
        x = wi.attn_w8(M)["x"][:nr]
        oracle.linear(x, codes, scales, GROUP, d["b"])
        flops += 2.0 * x.shape[0] * N_OUT * K_IN
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": int(os.environ.get("OMP_NUM_THREADS", cores)),
            "kind": "oracle", "seconds": round(dt, 3),
            "sample": "quantize all of W + Linear on %s rows of the M=%s batches (fp64 C, OpenMP)"
                      % ("/".join(map(str, n_rows_per_m)), "/".join(map(str, MS)))}


def max_over_ranks(values, dist=None, device="cpu"):
    """Each value's maximum over all ranks: a job's time is its slowest rank's.
    Every rank must call it with the same number of values (one collective)."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_tflops(world, flops_per_rank, ms):
    """Whole-job throughput of independent replicas (weak scaling): the work
    of all ranks over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ---------------------------------------------------------------------------
# Every configured workload, timed in the launch configuration of a model's
# layer sequence: a CUDA graph of back-to-back units (one unit = the
# workload's Linear calls), kernels chained by programmatic dependent launch,
# the units rotating over enough copies of the packed weights that every unit
# reads its weights from HBM, not from L2 (L2 is also flushed before each
# replay).  Per unit: device time, TFLOP/s, algorithmic GB/s and both roofline
# fractions against the measured peaks.
# ---------------------------------------------------------------------------
L2_BYTES = 126 * 2 ** 20


def workload_entries():
    """(key, M, layers, wiring) for every configured workload.  layers:
    (name, N, K, bits, group, r); wiring: 'each' (every layer on x), 'chain'
    (down on up's bf16 output) or 'block' (q, k, v, o and up on x, down on
    up's bf16 output)."""
    H, F = wi.HIDDEN, wi.MLP
    out = [("tiny_w8_m64", 64, [("lin", 512, 256, 8, 0, 0)], "each")]
    for M in (16, 256, 4096):
        out.append(("attn_w8_m%d" % M, M, [("proj", H, H, 8, 0, 0)], "each"))
    for M in (16, 1560, 6240):
        out.append(("mlp_w4g64_up_m%d" % M, M, [("up", F, H, 4, 64, 0)], "each"))
        out.append(("mlp_w4g64_down_m%d" % M, M, [("down", H, F, 4, 64, 0)], "each"))
        out.append(("mlp_w4g64_chained_m%d" % M, M, [("up", F, H, 4, 64, 0), ("down", H, F, 4, 64, 0)], "chain"))
    out.append(("mixed_block_m4096", 4096, [(n, N, K, b, g, 0) for n, N, K, b, g in wi.MIXED_LAYERS], "block"))
    for M in (256, 4096):
        out.append(("svdq_w4g64_lr32_m%d" % M, M, [("lr", H, H, 4, 64, wi.RANK)], "each"))
    return out


def _layer_weight(key, name, N, K):
    """The workload's seeded fp32 weight for this layer (timing only needs its
    shape and value range; the recipe is the parity tests')."""
    if key.startswith("tiny"):
        return wi.tiny_w8()["W"]
    if key.startswith("attn"):
        return wi.attn_w8(1)["W"]
    if key.startswith("mlp"):
        return wi.mlp_w4(1, name)["W"]
    if key.startswith("mixed"):
        i = [n for n, *_ in wi.MIXED_LAYERS].index(name)
        return wi.weight(3, 10 * (i + 1), N, K)
    return wi.svdq_w4_lr(1)["W"]


def time_workloads(wlq, torch, dev, evict_l2, hbm_peak, tc_peak, reps=3):
    res = {}
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    for key, M, layers, wiring in workload_entries():
        K0 = layers[0][2]
        x = bf(wi.activations(5, 1, M, K0))
        wbytes = sum(wlq.packed_bytes(N, K, b, g) for _, N, K, b, g, _ in layers)
        copies = int(min(16, max(1, -(-3 * L2_BYTES // wbytes))))
        units = max(8, copies)
        L = []
        for name, N, K, bits, group, r in layers:
            W = torch.from_numpy(_layer_weight(key, name, N, K)).to(dev)
            _, p = wlq.quantize_pack(W, bits, group)
            del W
            ps = [p] + [p.clone() for _ in range(copies - 1)]
            b = bf(wi.bias(5, 2, N))
            L1 = bf(wi.normal_bf16(wi.rng(5, 3), (K, r), 0.05)) if r else None
            L2 = bf(wi.normal_bf16(wi.rng(5, 4), (r, N), 0.05)) if r else None
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = wlq.new_workspace(M, N, K, bits, group, r, device=dev)
            L.append(dict(name=name, N=N, K=K, bits=bits, group=group, r=r, ps=ps, b=b, L1=L1, L2=L2, y=y, ws=ws))

        def unit(i):
            for j, l in enumerate(L):
                inp = x
                if wiring == "chain" and j == 1:
                    inp = L[0]["y"]
                if wiring == "block" and l["name"] == "down":
                    inp = [u for u in L if u["name"] == "up"][0]["y"]
                wlq.linear_into(l["y"], inp, l["ps"][i % copies], l["N"], l["K"], l["bits"], l["group"], l["b"],
                                l["L1"], l["L2"], workspace=l["ws"])

        for i in range(3):
            unit(i)
        torch.cuda.synchronize()
        wlq.check_status()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(units):
                unit(i)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            evict_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e-3 / units)
        wlq.check_status()
        t = statistics.median(ts)
        flops = sum(2.0 * M * l["N"] * l["K"] + (2.0 * M * l["r"] * (l["K"] + l["N"]) if l["r"] else 0.0) for l in L)
        byts = sum(wlq.packed_bytes(l["N"], l["K"], l["bits"], l["group"]) + 2 * M * l["K"] + 2 * M * l["N"] + 2 * l["N"]
                   + (2 * l["r"] * (l["K"] + l["N"]) if l["r"] else 0) for l in L)
        res[key] = {"M": M, "layers": ["%s %dx%d int%d %s%s" % (l["name"], l["N"], l["K"], l["bits"],
                                                                "gs%d" % l["group"] if l["group"] else "per-channel",
                                                                " r=%d" % l["r"] if l["r"] else "") for l in L],
                    "wiring": wiring, "us": round(t * 1e6, 2), "tflops": round(flops / t / 1e12, 1),
                    "hbm_gbs": round(byts / t / 1e9, 1), "tensor_frac": round(flops / t / 1e12 / tc_peak, 4),
                    "hbm_frac": round(byts / t / 1e9 / hbm_peak, 4), "algorithmic_bytes": int(byts),
                    "flops": flops, "weight_copies": copies, "units_per_replay": units}
        del L, g
        torch.cuda.empty_cache()
    return res


def time_lowrank_producer(wlq, torch, dev, evict_l2, reps=3):
    """The step before the low-rank branch on the SVDQuant workload's weight
    (W = (L1 L2)^T + R, [4096, 4096], r = 32): the GPU top-r split (sketch of
    64 columns, two power passes), the residual R = W - (L1 L2)^T and its
    quantize-pack (int4 gs64), each timed alone after an L2 flush."""
    d = wi.svdq_w4_lr(1)
    l1p = (d["L1"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    l2p = (d["L2"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    W = torch.from_numpy(((l1p @ l2p).T + d["W"].astype(np.float64)).astype(np.float32)).to(dev)
    N, K = W.shape
    omega = torch.from_numpy(wi.normal_f32(wi.rng(9, 2), (N, 64), 1.0)).to(dev)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            evict_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            out = fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        wlq.check_status()
        return statistics.median(ts), out

    t_split, (L1, L2, _) = timed(lambda: wlq.lowrank_split(W, 32, omega, power_iters=2))
    t_res, R = timed(lambda: wlq.lowrank_residual(W, L1, L2))
    t_qp, _ = timed(lambda: wlq.quantize_pack(R, 4, 64))
    return {"workload": "SVDQuant-style weight W = (L1 L2)^T + R, [4096, 4096], r = 32 (planted N(0,0.05) bf16 "
                        "factors, R ~ N(0, 0.02)); sketch l = 64, 2 power passes",
            "split_us": round(t_split, 1), "residual_us": round(t_res, 1), "quantize_pack_us": round(t_qp, 1),
            "residual_gbs": round(2 * N * K * 4 / t_res / 1e3, 1),  # W read + R written
            "timing": "each call alone, L2 flushed before, CUDA events, median of %d" % reps}


def time_w4a4(wlq, torch, dev, evict_l2, tc_peak, reps=3):
    """The NVFP4 W4A4 forward on the SVDQuant projection ([4096, 4096], r = 32):
    x quantized to NVFP4, the low-rank pre-pass, the block-scaled GEMM with the
    low-rank accumulator; graphs of back-to-back forwards over weight copies
    (> 3x L2), L2 flushed before each replay.  FP4 peak: the measured bf16
    figure x 4 (the nominal dense fp4 / bf16 ratio, 9 / 2.25)."""
    N = K = wi.HIDDEN
    r = wi.RANK
    W = torch.from_numpy(wi.svdq_w4_lr(1)["W"]).to(dev)
    wq, ws, wg = wlq.nvfp4_quantize(W)
    del W
    wbytes = wq.numel() + ws.numel()
    copies = int(min(16, max(1, -(-3 * L2_BYTES // wbytes))))
    units = max(8, copies)
    ops = [(wq, ws, wg)] + [(wq.clone(), ws.clone(), wg.clone()) for _ in range(copies - 1)]
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    L1 = bf(wi.normal_bf16(wi.rng(5, 3), (K, r), 0.05))
    L2 = bf(wi.normal_bf16(wi.rng(5, 4), (r, N), 0.05))
    b = bf(wi.bias(5, 2, N))
    out = {}
    fp4_peak = 4.0 * tc_peak
    for M in (256, 4096):
        x = bf(wi.activations(5, 1, M, K))
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        wsp = wlq.w4a4_workspace(M, N, K, r, device=dev)

        def unit(i):
            q, s_, g_ = ops[i % copies]
            wlq.w4a4_linear_into(y, x, q, s_, g_, N, K, b, L1, L2, workspace=wsp)

        for i in range(3):
            unit(i)
        torch.cuda.synchronize()
        wlq.check_status()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(units):
                unit(i)
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            evict_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e-3 / units)
        wlq.check_status()
        t = statistics.median(ts)
        flops = 2.0 * M * N * K + 2.0 * M * r * (K + N)
        out["m%d" % M] = {"M": M, "us": round(t * 1e6, 2), "tflops": round(flops / t / 1e12, 1),
                          "fp4_tensor_frac": round(flops / t / 1e12 / fp4_peak, 4),
                          "bf16_tensor_frac": round(flops / t / 1e12 / tc_peak, 4)}
        del g
    out["workload"] = ("W4A4 NVFP4 forward, [4096, 4096] weight (SVDQuant recipe's residual), r = 32, bf16 x "
                       "quantized per call; weight copies %d, units per replay %d" % (copies, units))
    out["fp4_peak_tflops"] = round(fp4_peak, 1)
    out["fp4_peak_source"] = "measured bf16 burst x 4 (nominal dense fp4 / bf16 ratio)"
    return out


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    d = wi.attn_w8(1)
    xs = {M: wi.attn_w8(M)["x"][:16] for M in MS}
    times, flops = [], 0.0
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        codes, scales = oracle.quantize(d["W"], BITS, GROUP)
        f = 0.0
        for M in MS:
            oracle.linear(xs[M], codes, scales, GROUP, d["b"])
            f += 2.0 * xs[M].shape[0] * N_OUT * K_IN
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            flops = f
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    sample = "per step: quantize all of W + Linear on 16 rows of each M batch (fp64 C oracle, OpenMP)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": list(MS), "N": N_OUT, "K": K_IN, "sampled_rows_per_M": 16},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args):
    import torch
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import weight_only_quantized_rtn_b200 as wlq
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    # ---- inputs, resident in HBM before the timed region
    base = wi.attn_w8(1)
    W = torch.from_numpy(base["W"]).to(dev)
    b = torch.from_numpy(base["b"].view(np.int16)).to(dev).view(torch.bfloat16)
    xs = {M: torch.from_numpy(wi.attn_w8(M)["x"].view(np.int16)).to(dev).view(torch.bfloat16) for M in MS}
    scales = torch.empty((N_OUT, 1), dtype=torch.float32, device=dev)
    packed = torch.empty(wlq.packed_bytes(N_OUT, K_IN, BITS, GROUP), dtype=torch.uint8, device=dev)
    ys = {M: torch.empty((M, N_OUT), dtype=torch.bfloat16, device=dev) for M in MS}
    wss = {M: wlq.new_workspace(M, N_OUT, K_IN, BITS, GROUP, 0, device=dev) for M in MS}
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    lib, ptr = wlq.lib, wlq._ptr

    def evict_l2():
        # Write a buffer twice the L2, then read it back: afterwards L2 holds
        # none of the step's data and no dirty line whose write-back the next
        # timed step would pay for.
        flush.zero_()
        flush.view(torch.float32).sum()

    def quantize_pack():
        # RTN quantization straight into the packed operand (one pass over W)
        st = wlq._stream(torch.cuda.current_stream())
        wlq._check(lib.wlq_quantize_pack(ptr(W), N_OUT, K_IN, BITS, GROUP, ptr(scales), ptr(packed), st))

    def linear(M):
        wlq.linear_into(ys[M], xs[M], packed, N_OUT, K_IN, BITS, GROUP, bias=b, workspace=wss[M])

    def step():
        quantize_pack()
        for M in MS:
            linear(M)

    launches_per_step = 1 + len(MS)  # quantize-and-pack, one GEMM per M

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    wlq.check_status()

    # The step runs as one CUDA-graph replay (host launch overhead off the
    # device timeline), timed by events around the replay.  Its kernels are
    # launched with programmatic dependent launch, so each may start while
    # the previous one finishes; a second graph of the same step, with timing
    # events recorded between its phases (which serialise them), gives the
    # split of a step into phases.
    phases = ["qp"] + list(MS)
    inner = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(phases) + 1)]
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    g_phases = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_phases):
        inner[0].record()
        quantize_pack()
        inner[1].record()
        for j, M in enumerate(MS):
            linear(M)
            inner[j + 2].record()
    graphs = {}
    for M in MS:  # one graph per Linear, for the isolated timings
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            linear(M)
        graphs[M] = g
    torch.cuda.synchronize()
    for _ in range(2):
        g_step.replay()
        g_phases.replay()
        for g in graphs.values():
            g.replay()
    torch.cuda.synchronize()
    wlq.check_status()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    phase_ms = {ph: 0.0 for ph in phases}
    for i in range(args.steps):
        evict_l2()  # between steps, outside the timed events
        torch.cuda.nvtx.range_push("timed_step")
        outer[i][0].record(stream)
        g_step.replay()
        outer[i][1].record(stream)
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    for i in range(args.steps):
        evict_l2()
        g_phases.replay()
        torch.cuda.synchronize()  # the in-graph events are re-recorded by the next replay
        for j, ph in enumerate(phases):
            phase_ms[ph] += inner[j].elapsed_time(inner[j + 1]) / args.steps
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    wlq.check_status()

    ms_step = sum(a.elapsed_time(c) for a, c in outer) / args.steps
    per_ms = phase_ms
    per_m_ms = {M: per_ms[M] for M in MS}
    red = max_over_ranks([ms_step] + [per_m_ms[M] for M in MS], dist, dev)
    ms_step = red[0]
    per_m_ms = {M: red[1 + i] for i, M in enumerate(MS)}

    # ---- per-M kernels in isolation (L2 flushed before every launch)
    iso = {}
    for M in MS:
        pairs = []
        for _ in range(max(5, args.steps)):
            evict_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graphs[M].replay()
            e1.record(stream)
            pairs.append((e0, e1))
        torch.cuda.synchronize()
        iso[M] = statistics.median(a.elapsed_time(c) for a, c in pairs)

    # ---- the dominant kernel sustained: the M=4096 Linear replayed back to
    # back for about two seconds while the clocks are sampled, so that its
    # time can be read beside the SM clock it actually ran at
    g4 = graphs[4096]
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    n_probe = 0
    while time.perf_counter() - t0 < 0.05:
        g4.replay()
        torch.cuda.synchronize()
        n_probe += 1
    per = (time.perf_counter() - t0) / max(1, n_probe)
    reps_sus = int(max(50, min(40000, 2.0 / max(per, 1e-6))))
    sampler2 = ClockSampler(local)
    sampler2.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps_sus):
        g4.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks_sus = sampler2.stop()
    sus_us = e0.elapsed_time(e1) * 1e3 / reps_sus
    sustained = {"launches": reps_sus, "us_per_launch": round(sus_us, 2),
                 "tflops": round(2.0 * 4096 * N_OUT * K_IN / (sus_us * 1e-6) / 1e12, 1),
                 "clocks": clocks_sus,
                 "note": "back-to-back replays of the M=4096 Linear (weights stay in L2): time beside the SM clock under load"}
    if clocks_sus and clocks_sus.get("sm_mhz"):
        sustained["us_x_mhz"] = round(sus_us * clocks_sus["sm_mhz"], 1)

    # ---- end to end through the public API with pinned host buffers
    W_h = torch.from_numpy(base["W"]).pin_memory()
    x_h = {M: xs[M].cpu().pin_memory() for M in MS}
    y_h = {M: torch.empty((M, N_OUT), dtype=torch.bfloat16).pin_memory() for M in MS}
    h2d = W_h.numel() * 4 + sum(x_h[M].numel() * 2 for M in MS)
    d2h = sum(y_h[M].numel() * 2 for M in MS)
    e2e_steps = max(3, min(args.steps, 20))
    # One plain step first: its outputs are what every pipelined step must reproduce.
    torch.cuda.synchronize()
    W.copy_(W_h, non_blocking=True)
    for M in MS:
        xs[M].copy_(x_h[M], non_blocking=True)
    step()
    for M in MS:
        y_h[M].copy_(ys[M], non_blocking=True)
    torch.cuda.synchronize()
    y_first = {M: y_h[M].clone() for M in MS}
    # Steps run back to back as a pipeline over three streams: host-to-device
    # copies, compute, device-to-host copies.  Step i+1's uploads overlap step
    # i's compute and downloads (the link is full duplex); every step still
    # uploads all of W and x and downloads every y, and each buffer is reused
    # only after the step that last touched it is done with it.
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    qp_done, lin_done, y_read = None, None, None
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e_start.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for i in range(e2e_steps):
        with torch.cuda.stream(s_in):
            if qp_done is not None:
                s_in.wait_event(qp_done)    # the previous step has read W
            W.copy_(W_h, non_blocking=True)
            w_in = ev(); w_in.record(s_in)
            if lin_done is not None:
                s_in.wait_event(lin_done)   # the previous step has read x
            for M in MS:
                xs[M].copy_(x_h[M], non_blocking=True)
            x_in = ev(); x_in.record(s_in)
        stream.wait_event(w_in)
        quantize_pack()
        qp_done = ev(); qp_done.record(stream)
        stream.wait_event(x_in)
        if y_read is not None:
            stream.wait_event(y_read)       # the previous step's y are downloaded
        for M in MS:
            linear(M)
        lin_done = ev(); lin_done.record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(lin_done)
            for M in MS:
                y_h[M].copy_(ys[M], non_blocking=True)
            y_read = ev(); y_read.record(s_out)
    stream.wait_event(y_read)
    e_end.record(stream)
    torch.cuda.synchronize()
    for M in MS:
        if not torch.equal(y_h[M], y_first[M]):
            raise RuntimeError("pipelined end-to-end steps changed the output at M=%d" % M)
    e2e_ms = e_start.elapsed_time(e_end) / e2e_steps
    e2e_ms = max_over_ranks([e2e_ms], dist, dev)[0]
    wlq.check_status()

    hbm_peak, tc_peak, tc_sust, peak_src = measured_peaks()
    flops = linear_flops()
    value = job_tflops(world, flops, ms_step)
    per_m = {}
    for M in MS:
        f = 2.0 * M * N_OUT * K_IN
        byts = wlq.packed_bytes(N_OUT, K_IN, BITS, GROUP) + M * K_IN * 2 + M * N_OUT * 2 + N_OUT * 2
        t_iso = iso[M] * 1e-3
        per_m[str(M)] = {
            "in_step_us": round(per_m_ms[M] * 1e3, 2), "isolated_us": round(iso[M] * 1e3, 2),
            "tflops": round(f / t_iso / 1e12, 1), "hbm_gbs": round(byts / t_iso / 1e9, 1),
            "tensor_frac": round(f / t_iso / 1e12 / tc_peak, 4), "hbm_frac": round(byts / t_iso / 1e9 / hbm_peak, 4),
            "algorithmic_bytes": int(byts)}
    # roofline of the dominant kernel (the M=4096 GEMM, one launch), timed live in the step
    t_dom = per_m_ms[4096] * 1e-3
    achieved = 2.0 * 4096 * N_OUT * K_IN / t_dom / 1e12
    roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tc_peak, "unit": "TFLOP/s",
            "frac": round(achieved / tc_peak, 4), "traffic": profiled_traffic(),
            "peak_source": peak_src + " bf16_tflops (burst); sustained %s" % tc_sust,
            "kernel": "gemm_kernel<FMT_W8> at M=4096 (one launch per step)"}
    line = {"metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": list(MS), "N": N_OUT, "K": K_IN, "bits": BITS,
                       "group": "per-channel", "out": "bf16", "parallelism": "replicas x%d" % world,
                       "l2": "flushed between steps: 256 MiB written then read back, outside the timed events (no step data and no dirty line left in L2)",
                       "timing": "one CUDA-graph replay per step between CUDA events (kernels chained by programmatic dependent launch); phases from replays of a second graph of the step with events between its phases"},
            "per_m": per_m, "roofline": roof, "clocks": clocks, "sustained_m4096": sustained,
            "quantize_pack_us": round(per_ms["qp"] * 1e3, 2),
            "e2e": {"value": round(job_tflops(world, flops, e2e_ms), 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "ms_per_step": round(e2e_ms, 4),
                    "schedule": "steps back to back on three streams (uploads, compute, downloads overlap across steps); outputs checked equal to a plain step's"},
            "gpu_launches": launches_per_step * args.steps}
    if not args.no_configs:
        line["configs"] = time_workloads(wlq, torch, dev, evict_l2, hbm_peak, tc_peak)
        line["lowrank_producer"] = time_lowrank_producer(wlq, torch, dev, evict_l2)
        line["w4a4_nvfp4"] = time_w4a4(wlq, torch, dev, evict_l2, tc_peak)
        line["configs_timing"] = ("per unit = one CUDA-graph replay of back-to-back units / units; units rotate over "
                                  "weight copies totalling >= 3x L2 and L2 is flushed before each replay; "
                                  "median of 3 replays; bf16 outputs")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload timings")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
