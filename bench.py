#!/usr/bin/env python
"""Benchmark of the B200 BitStack residual-block linear (bs_linear).

Headline (default): one decode call y = x W_hat^T of a 4096 x 4096 linear with n = 8
loaded residual blocks, k = 16, batch 1, fp16 x -- microseconds per call and the
fraction of the HBM / tensor roofline.  A step is one bs_linear call; steps rotate
over enough distinct stacks (each with its own x and y) that the bytes touched
between two uses of one stack exceed three times the L2 size.  Steps are replayed
from CUDA graphs and timed with CUDA events on the launching stream; nvidia-smi
clocks are sampled during the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (torchrun, one process per GPU) every rank runs the same workload on its
own GPU (the path needs no exchange between GPUs: replicas); the time is the max over
ranks and the value is that time divided by all calls of all ranks.

--impl reference times the CPU oracle (float64 NumPy) on the same workload, on a
bounded sample, on the host cores.  The blocks are synthetic (random signs and
factors of decomposition-like scale): timing depends only on shapes and bytes.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "bs_linear µs/call & % roofline (HBM/tensor) at 4096², n=8, k=16, batch 1"
UNIT = "us/call"
M_HEAD, D_HEAD, N_HEAD, K_HEAD, B_HEAD = 4096, 4096, 8, 16, 1
L2_FALLBACK = 126 * 2 ** 20


# ------------------------------------------------------------------ helpers -------
def max_over_ranks(values, device=None):
    """Each value's maximum over all ranks (one all-reduce); unchanged for one rank.
    Timing a multi-GPU job by its slowest rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_us_per_call(ms_total, steps, world):
    """Whole-job figure: the (slowest rank's) time over the calls of all ranks."""
    return ms_total * 1000.0 / (steps * world)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), \
            "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def algorithmic(m, d, k, n, b):
    """Bytes and FLOPs one call must move / do (the roofline's numerators)."""
    block = m * d // 8 + 2 * k * (m + d)
    nbytes = n * block + 2 * b * d + 2 * b * m + 4 * d
    flops_factored = 2 * m * d * k * b * n      # the +-1 contraction S_i (x' (.) V_i)
    flops_rebuild = 2 * m * d * (k * n + b)      # rank-k rebuild + dense product
    return nbytes, flops_factored, flops_rebuild


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu_index), "-lms", "50"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxes.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(sms)}


def source_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def dram_traffic(kind):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kind}_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        src = [os.path.join(ROOT, "residual_block_decomp_b200", "csrc", s) for s in rec["sources"]]
        if rec["source_sha"] != source_sha(src):
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


# --------------------------------------------------------------- CUDA arm ---------
def make_records(m, d, k, n, gen):
    """n synthetic block records: random sign words (random bits in any bit order
    are random bits) followed by fp16 U and V of decomposition-like scale."""
    from residual_block_decomp_b200.layer import record_from_parts
    recs = []
    for i in range(n):
        words = gen.integers(0, 2 ** 32, size=m * d // 32, dtype=np.uint64).astype(np.uint32)
        U = wl.random_factors(m, k, gen, 0.12 / np.sqrt(i + 1.0))
        V = wl.random_factors(d, k, gen, 0.12 / np.sqrt(i + 1.0))
        recs.append(record_from_parts(words, U, V))
    return recs


def run_cuda(args, rank, world, local_rank):
    import torch
    import residual_block_decomp_b200 as R
    from residual_block_decomp_b200 import BitStackLinear

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    m, d, k, n, b = args.m, args.d, K_HEAD, args.n, args.batch
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 0) or L2_FALLBACK)
    nbytes, flops_f, flops_r = algorithmic(m, d, k, n, b)
    n_stacks = max(2, int(np.ceil(3 * l2 / nbytes)) + 1)

    gen = wl.generator(2, 100 + rank, "blocks")
    inv_s = wl.synthetic_inv_scale(d, gen)
    layers, xs, ys = [], [], []
    for j in range(n_stacks):
        layer = BitStackLinear(m, d, n, inv_s, device=dev)
        for rec in make_records(m, d, k, n, gen):
            layer.add_record(rec)
        layer.set_loaded(n)
        layers.append(layer)
        xs.append(torch.from_numpy(wl.activations(b, d, gen).astype(np.float16)).to(dev))
        ys.append(torch.empty((b, m), dtype=torch.float16, device=dev))
    ws = torch.zeros(R.bs_workspace_bytes(m, d, k, n, b), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize(dev)

    stream = torch.cuda.Stream(dev)

    def step(j):
        layers[j % n_stacks].forward(xs[j % n_stacks], n, out=ys[j % n_stacks], workspace=ws, stream=stream)

    # warm-up (eager), then graphs of whole rotations
    with torch.cuda.stream(stream):
        for j in range(max(args.warmup, 3)):
            step(j)
    stream.synchronize()
    per_graph = min(args.steps, n_stacks * max(1, 2000 // n_stacks))
    reps, rem = divmod(args.steps, per_graph)

    def capture(count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for j in range(count):
                step(j)
        return g

    g_main = capture(per_graph)
    g_rem = capture(rem) if rem else None
    with torch.cuda.stream(stream):     # replay() launches on the current stream
        g_main.replay()
    stream.synchronize()
    assert layers[0].device_error() == 0, "device error during warm-up"

    def timed(run):
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                          os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]) as cs:
            with torch.cuda.stream(stream):
                e0.record(stream)
                run()
                e1.record(stream)
            e1.synchronize()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1), cs.summary()

    def run_main():
        for _ in range(reps):
            g_main.replay()
        if g_rem is not None:
            g_rem.replay()

    ms, clocks = timed(run_main)
    for layer in layers[:1]:
        assert layer.device_error() == 0, "device error in the timed region"

    # ------------------------------------------------------------------ e2e ----
    # through the C ABI with host buffers: every call copies its x from pinned host memory,
    # runs bs_linear and copies its y back to pinned host memory.  As a serving loop would,
    # the copies run on their own streams and overlap the neighbouring calls' kernels: call
    # j's kernel waits for its x, its y copy waits for its kernel, and a buffer is reused
    # (x refilled, y overwritten) only after its previous call has consumed it.
    xh = [torch.empty((b, d), dtype=torch.float16, pin_memory=True) for _ in range(n_stacks)]
    yh = [torch.empty((b, m), dtype=torch.float16, pin_memory=True) for _ in range(n_stacks)]
    for j in range(n_stacks):
        xh[j].copy_(xs[j].cpu())
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(n_stacks)]     # x of buffer jj landed
    ev_done = [torch.cuda.Event() for _ in range(n_stacks)]   # its call finished (x read, y written)
    ev_out = [torch.cuda.Event() for _ in range(n_stacks)]    # its y copied out

    def e2e_step(j):
        jj = j % n_stacks
        with torch.cuda.stream(h2d):
            if j >= n_stacks:
                h2d.wait_event(ev_done[jj])
            xs[jj].copy_(xh[jj], non_blocking=True)
            ev_in[jj].record(h2d)
        stream.wait_event(ev_in[jj])
        if j >= n_stacks:
            stream.wait_event(ev_out[jj])
        step(jj)
        ev_done[jj].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_done[jj])
            yh[jj].copy_(ys[jj], non_blocking=True)
            ev_out[jj].record(d2h)

    def capture_e2e(count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            h2d.wait_stream(stream)
            d2h.wait_stream(stream)
            for j in range(count):
                e2e_step(j)
            stream.wait_stream(h2d)
            stream.wait_stream(d2h)
        return g

    e2e_steps = args.e2e_steps or args.steps
    per_e = min(e2e_steps, per_graph)
    reps_e, rem_e = divmod(e2e_steps, per_e)
    ge_main = capture_e2e(per_e)
    ge_rem = capture_e2e(rem_e) if rem_e else None
    with torch.cuda.stream(stream):
        ge_main.replay()
    stream.synchronize()

    def run_e2e():
        for _ in range(reps_e):
            ge_main.replay()
        if ge_rem is not None:
            ge_rem.replay()

    ms_e2e, _ = timed(run_e2e)

    ms, ms_e2e = max_over_ranks([ms, ms_e2e], device=dev)

    out = {
        "ms": ms, "ms_e2e": ms_e2e, "steps": args.steps, "e2e_steps": e2e_steps, "clocks": clocks,
        "n_stacks": n_stacks, "l2": l2, "bytes": nbytes, "flops_factored": flops_f, "flops_rebuild": flops_r,
        "e2e_h2d": b * d * 2, "e2e_d2h": b * m * 2,
    }
    if args.extras and rank == 0:
        out["extras"] = extras(args, dev, stream, layers[0], ws, inv_s)
    for layer in layers:
        layer.close()
    if args.extras and rank == 0:
        out["extras"].update(extras_workloads(args, dev, stream, l2))
    return out


def extras(args, dev, stream, layer, ws, inv_s):
    """Secondary figures (not the headline): n sweep, batch 4, prefill, block load."""
    import torch
    res = {}
    m, d, k = args.m, args.d, K_HEAD

    def time_calls(fn, count=200):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(count):
                fn()
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) * 1000.0 / count

    x1 = torch.randn((1, d), device=dev).half()
    y1 = torch.empty((1, m), device=dev, dtype=torch.float16)
    res["decode_b1_us_by_n"] = {
        str(nn): round(time_calls(lambda nn=nn: layer.forward(x1, nn, out=y1, workspace=ws, stream=stream)), 3)
        for nn in range(1, args.n + 1)}
    x4 = torch.randn((4, d), device=dev).half()
    y4 = torch.empty((4, m), device=dev, dtype=torch.float16)
    ws4 = torch.zeros(layer.workspace(args.n, 4).numel(), dtype=torch.uint8, device=dev)
    res["decode_b4_n8_us"] = round(time_calls(lambda: layer.forward(x4, args.n, out=y4, workspace=ws4,
                                                                     stream=stream)), 3)
    for M in (512, 4096):
        xM = torch.randn((M, d), device=dev).bfloat16()
        yM = torch.empty((M, m), device=dev, dtype=torch.bfloat16)
        us = time_calls(lambda: layer.forward(xM, args.n, out=yM, stream=stream), count=20)
        res[f"prefill_M{M}_us"] = round(us, 2)
        res[f"prefill_M{M}_gemm_tflops"] = round(2.0 * M * m * d / (us * 1e-6) / 1e12, 1)
    # block load: one record H2D (pinned host -> device) per append
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    layer.set_loaded(0)
    torch.cuda.synchronize(dev)
    t0.record(torch.cuda.current_stream(dev))
    layer.set_loaded(args.n)
    t1.record(torch.cuda.current_stream(dev))
    t1.synchronize()
    per_block = t0.elapsed_time(t1) * 1000.0 / args.n
    res["append_us_per_block"] = round(per_block, 1)
    res["append_gbs"] = round(layer.block_bytes / (per_block * 1e-6) / 1e9, 1)
    return res


def _graph_us(dev, stream, step, count, reps=3):
    """Per-step µs of `count` steps replayed from one CUDA graph (best of `reps`)."""
    import torch
    for j in range(3):
        step(j)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for j in range(count):
            step(j)
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1) * 1000.0 / count)
    del g
    return best


def _stacks(m, d, n, count, gen, dev, plain=False, kp=None):
    from residual_block_decomp_b200 import BitStackLinear
    import residual_block_decomp_b200 as R
    layers = []
    for _ in range(count):
        inv_s = wl.synthetic_inv_scale(d, gen)
        if plain:
            L = BitStackLinear(m, d, n, inv_s, k=kp, device=dev, plain=True)
            for i in range(n):
                U = wl.random_factors(m, kp, gen, 0.05 / np.sqrt(i + 1.0))
                V = wl.random_factors(d, kp, gen, 0.05 / np.sqrt(i + 1.0))
                L.add_record(np.concatenate([U.view(np.uint8).reshape(-1), V.view(np.uint8).reshape(-1)]))
        else:
            L = BitStackLinear(m, d, n, inv_s, device=dev)
            for rec in make_records(m, d, K_HEAD, n, gen):
                L.add_record(rec)
        L.set_loaded(n)
        layers.append(L)
    return layers


def extras_workloads(args, dev, stream, l2):
    """The other workloads: the MLP linears (config 3), prefill shapes (config 4), the
    whole-model token through a grouped launch (config 5), "w/o AVD" stacks, and the
    headline call's latency with L2 flushed before every call."""
    import torch
    import residual_block_decomp_b200 as R
    res = {}
    gen = wl.generator(3, 0, "blocks")

    # headline call, L2 flushed (a 4x-L2 buffer written) before every timed call
    layers = _stacks(M_HEAD, D_HEAD, N_HEAD, 1, gen, dev)
    x = torch.randn((1, D_HEAD), device=dev).half()
    y = torch.empty((1, M_HEAD), device=dev, dtype=torch.float16)
    ws = torch.zeros(R.bs_workspace_bytes(M_HEAD, D_HEAD, K_HEAD, N_HEAD, 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(4 * l2 // 4, dtype=torch.float32, device=dev)
    times = []
    with torch.cuda.stream(stream):
        for j in range(33):
            flush.fill_(float(j))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            layers[0].forward(x, N_HEAD, out=y, workspace=ws, stream=stream)
            e1.record(stream)
            e1.synchronize()
            if j >= 3:
                times.append(e0.elapsed_time(e1) * 1000.0)
    res["decode_l2_flushed_single_call_us"] = round(statistics.median(times), 3)
    # eager end-to-end: pinned x in, one binding call, y out, no graph, per call
    xh = torch.empty((1, D_HEAD), dtype=torch.float16, pin_memory=True)
    yh = torch.empty((1, M_HEAD), dtype=torch.float16, pin_memory=True)
    xh.copy_(x.cpu())
    with torch.cuda.stream(stream):
        for _ in range(20):
            x.copy_(xh, non_blocking=True)
            layers[0].forward(x, N_HEAD, out=y, workspace=ws, stream=stream)
            yh.copy_(y, non_blocking=True)
        stream.synchronize()
        t0 = time.perf_counter()
        for _ in range(500):
            x.copy_(xh, non_blocking=True)
            layers[0].forward(x, N_HEAD, out=y, workspace=ws, stream=stream)
            yh.copy_(y, non_blocking=True)
        stream.synchronize()
        res["decode_e2e_eager_us"] = round((time.perf_counter() - t0) * 1e6 / 500, 2)
    for L in layers:
        L.close()
    del flush

    # config 3: MLP linears, 12-block stacks, n per matrix drawn from 2..12, L2-rotated
    for (m, d) in ((14336, 4096), (4096, 14336)):
        count = max(2, int(np.ceil(3 * l2 / (12 * R.bs_block_bytes(m, d, K_HEAD)))) + 1)
        layers = _stacks(m, d, 12, count, gen, dev)
        ns = wl.n_loaded_draws(count, gen, 2, 12).tolist()
        for b in (1, 4, 16):
            xs = [torch.randn((b, d), device=dev).half() for _ in range(count)]
            ys = [torch.empty((b, m), device=dev, dtype=torch.float16) for _ in range(count)]
            wss = [L.workspace(12, b) for L in layers]

            def step(j, layers=layers, xs=xs, ys=ys, wss=wss, ns=ns):
                k = j % len(layers)
                layers[k].forward(xs[k], ns[k], out=ys[k], workspace=wss[k], stream=stream)
            us = _graph_us(dev, stream, step, 10 * count)
            nbytes = np.mean([n * R.bs_block_bytes(m, d, K_HEAD) for n in ns])
            res[f"mlp_{m}x{d}_b{b}_us"] = round(us, 2)
            res[f"mlp_{m}x{d}_b{b}_hbm_frac"] = round(nbytes / (us * 1e-6) / 1e9 / peaks()[0], 4)
        res[f"mlp_{m}x{d}_n_loaded"] = ns
        for L in layers:
            L.close()

    # config 4: prefill, n = 8, M in {512, 2048, 4096}, bf16 tokens
    for (m, d) in ((4096, 4096), (14336, 4096)):
        layers = _stacks(m, d, 8, 1, gen, dev)
        for M in (512, 2048, 4096):
            xM = torch.randn((M, d), device=dev).bfloat16()
            yM = torch.empty((M, m), device=dev, dtype=torch.bfloat16)
            us = _graph_us(dev, stream, lambda j: layers[0].forward(xM, 8, out=yM, stream=stream), 5)
            res[f"prefill_{m}x{d}_M{M}_us"] = round(us, 1)
            res[f"prefill_{m}x{d}_M{M}_tensor_frac"] = round(2.0 * M * m * d / (us * 1e-6) / 1e12 / peaks()[1], 4)
        layers[0].close()

    # "w/o AVD": vanilla rank-k' blocks of the same bytes, 4096 x 4096, n = 8, batch 1
    kp = R.bs_plain_rank(M_HEAD, D_HEAD, K_HEAD)
    pbytes = N_HEAD * R.bs_plain_block_bytes(M_HEAD, D_HEAD, kp)
    count = max(2, int(np.ceil(3 * l2 / pbytes)) + 1)
    layers = _stacks(M_HEAD, D_HEAD, N_HEAD, count, gen, dev, plain=True, kp=kp)
    x1 = torch.randn((1, D_HEAD), device=dev).half()
    y1 = torch.empty((1, M_HEAD), device=dev, dtype=torch.float16)
    wsp = layers[0].workspace(N_HEAD, 1)
    us = _graph_us(dev, stream, lambda j: layers[j % count].forward(x1, N_HEAD, out=y1, workspace=wsp,
                                                                    stream=stream), 10 * count)
    res["plain_4096x4096_kp144_n8_b1_us"] = round(us, 3)
    res["plain_4096x4096_kp144_n8_b1_hbm_frac"] = round(pbytes / (us * 1e-6) / 1e9 / peaks()[0], 4)
    for L in layers:
        L.close()
    torch.cuda.synchronize(dev)

    # the offline step on the GPU: decomposition of a 4096 x 4096 weight into 8 blocks
    W = torch.randn((M_HEAD, D_HEAD), device=dev) * 0.02
    sc = torch.rand(D_HEAD, device=dev) + 0.5
    bb = R.bs_block_bytes(M_HEAD, D_HEAD, K_HEAD)
    recs = torch.zeros(N_HEAD * bb, dtype=torch.uint8, device=dev)
    norms = torch.zeros(N_HEAD + 1, dtype=torch.float64, device=dev)
    dws = torch.empty(R.bs_decompose_workspace_bytes(M_HEAD, D_HEAD), dtype=torch.uint8, device=dev)
    R.bs_decompose(W, sc, N_HEAD, recs, norms, dws, stream=stream)
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        R.bs_decompose(W, sc, N_HEAD, recs, norms, dws, stream=stream)
        e1.record(stream)
    e1.synchronize()
    res["decompose_4096x4096_n8_ms"] = round(e0.elapsed_time(e1), 2)
    del W, recs, dws

    res.update(extras_model(dev, stream))
    return res


def extras_model(dev, stream, budgets_mib=(3000, 2000, 4500), tokens=20):
    """Config 5: 224 Llama-3-8B-shaped linears with 16-block stacks; per-linear loaded
    counts from the greedy fill of each budget over a Greedy global order (the
    library's planner on seeded per-block scores); blocks dropped / appended between
    budgets (timed); then one decode token through all linears, as one grouped launch
    and as one launch per linear."""
    import torch
    import residual_block_decomp_b200 as R
    from residual_block_decomp_b200 import BitStackLinear
    mats = wl.llama3_8b_matrices()
    shapes = [(m, d) for (_, _, m, d) in mats]
    gen = wl.generator(5, 0, "blocks")
    # one storage copy per (shape, level), shared by the stacks of that shape
    pinned = {}
    for (m, d) in sorted(set(shapes)):
        recs = []
        for rec in make_records(m, d, K_HEAD, 16, gen):
            t = torch.empty(rec.size, dtype=torch.uint8, pin_memory=True)
            t.copy_(torch.from_numpy(rec))
            recs.append(t)
        pinned[(m, d)] = recs
    layers = []
    for (m, d) in shapes:
        L = BitStackLinear(m, d, 16, wl.synthetic_inv_scale(d, gen), device=dev)
        for t in pinned[(m, d)]:
            L.add_pinned_record(t)
        layers.append(L)
    sizes = np.array([R.bs_block_bytes(m, d, K_HEAD) for (m, d) in shapes], dtype=np.uint64)
    # per-block scores: energy drop per byte from seeded geometric residual-norm decays
    sgen = wl.generator(5, 0, "plan")
    norms = np.cumprod(np.concatenate([np.ones((len(shapes), 1)), sgen.uniform(0.8, 0.99, (len(shapes), 16))], 1), 1)
    scores = (norms[:, :-1] ** 2 - norms[:, 1:] ** 2) / sizes[:, None].astype(np.float64)
    order_w, _ = R.bs_plan_order([16] * len(shapes), R.BS_ORDER_GREEDY, scores=scores)
    xs = [torch.randn((1, d), device=dev).half() for (_, d) in shapes]
    ys = [torch.empty((1, m), device=dev, dtype=torch.float16) for (m, _) in shapes]
    handles = [L.handle for L in layers]
    ws = None
    out = {"model_linears": len(shapes)}
    for mib in budgets_mib:
        counts = R.bs_plan_budget(order_w, sizes, int(mib) * 2 ** 20).tolist()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        moved = sum(abs(c - L.n_blocks) * int(sz) for c, L, sz in zip(counts, layers, sizes))
        with torch.cuda.stream(stream):
            e0.record(stream)
            for L, c in zip(layers, counts):
                L.set_loaded(c, stream=stream)
            e1.record(stream)
        e1.synchronize()
        loaded = int(np.sum(np.array(counts, dtype=np.uint64) * sizes))
        out[f"model_{mib}MiB_budget_change_ms"] = round(e0.elapsed_time(e1), 3)
        out[f"model_{mib}MiB_bytes_moved"] = int(moved)
        need = R.bs_group_workspace_bytes(handles, counts, 1)
        if ws is None or ws.numel() < need:
            ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        us_g = _graph_us(dev, stream, lambda j: R.bs_linear_group(handles, xs, counts, ys, ws, stream), tokens)
        wss = [L.workspace(max(c, 1), 1) for L, c in zip(layers, counts)]

        def token_singles(j):
            for L, x, y, c, w in zip(layers, xs, ys, counts, wss):
                L.forward(x, c, out=y, workspace=w, stream=stream)
        us_s = _graph_us(dev, stream, token_singles, 3)
        hbm = peaks()[0]
        out[f"model_{mib}MiB_loaded_bytes"] = loaded
        out[f"model_{mib}MiB_token_grouped_us"] = round(us_g, 1)
        out[f"model_{mib}MiB_token_per_linear_launches_us"] = round(us_s, 1)
        out[f"model_{mib}MiB_grouped_hbm_frac"] = round(loaded / (us_g * 1e-6) / 1e9 / hbm, 4)
    assert layers[0].device_error() == 0
    for L in layers:
        L.close()
    return out


# -------------------------------------------------------------- oracle arm --------
def run_oracle(args, budget_s):
    """Times the oracle's two float64 forms of the linear on the headline workload, each
    for about half of `budget_s`, with the BLAS pool pinned to the host's cores: the
    factored form (the sign contraction per block) is the reported value, the explicit
    form (rebuild the weight, then one product) is reported beside it."""
    from oracle import linear
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(limits=cores)
    except Exception:
        limiter = None
    m, d, k, n, b = args.m, args.d, K_HEAD, args.n, args.batch
    gen = wl.generator(2, 900, "blocks")
    negs, Us, Vs = [], [], []
    for i in range(n):
        neg, U, V = wl.synthetic_block(m, d, k, gen, level=i)
        negs.append(neg)
        Us.append(U)
        Vs.append(V)
    inv_s = wl.synthetic_inv_scale(d, gen)
    x = wl.activations(b, d, gen).astype(np.float16)
    timed = {}
    for name, fn in (("factored", linear.linear_factored), ("explicit", linear.linear_explicit)):
        calls = 0
        t0 = time.perf_counter()
        while True:
            fn(x, negs, Us, Vs, inv_s, n, m)
            calls += 1
            if time.perf_counter() - t0 >= budget_s / 2:
                break
        timed[name] = (time.perf_counter() - t0, calls)
    if limiter is not None:
        limiter.restore_original_limits()
    el, calls = timed["factored"]
    ee, ce = timed["explicit"]
    return {"value": el * 1e6 / calls, "unit": UNIT, "cores": cores, "kind": "oracle",
            "explicit_value": ee * 1e6 / ce,
            "sample": f"{calls} call(s) of the float64 factored oracle ({el:.1f} s) and {ce} of the explicit "
                      f"oracle ({ee:.1f} s) on the full {m}x{d}, n={n}, k={k}, batch {b} workload; BLAS threads "
                      f"pinned to the {cores} host cores"}


# ---------------------------------------------------------------------- main ------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--e2e-steps", type=int, default=0)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--m", type=int, default=M_HEAD)
    ap.add_argument("--d", type=int, default=D_HEAD)
    ap.add_argument("--n", type=int, default=N_HEAD)
    ap.add_argument("--batch", type=int, default=B_HEAD)
    ap.add_argument("--no-extras", dest="extras", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    kind = "decode" if args.batch <= 4 else "prefill"
    workload = f"{kind} {args.m}x{args.d} n={args.n} k={K_HEAD} batch={args.batch} fp16"
    config = {"workload": workload, "m": args.m, "d": args.d, "n_loaded": args.n, "k": K_HEAD,
              "batch": args.batch, "parallelism": f"replicas x{world}"}

    if args.impl == "reference":
        if rank != 0:
            return
        cpu = run_oracle(args, budget_s=args.cpu_seconds)
        v = cpu["value"]
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1000.0, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": cpu, "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_cuda(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    hbm, bf16, bf16_sus, src = peaks()
    us_step = res["ms"] * 1000.0 / args.steps                 # per call on one GPU
    value = job_us_per_call(res["ms"], args.steps, world)      # whole job: all calls of all ranks
    nbytes = res["bytes"]
    achieved = nbytes / (us_step * 1e-6) / 1e9                 # GB/s of the decode kernel
    i8_peak = bf16 * 2.0                                       # int8 dense = 2x bf16 (nominal ratio 4.5 / 2.25)
    t_roof = max(nbytes / (hbm * 1e9), res["flops_factored"] / (bf16 * 1e12))
    traffic = dram_traffic("decode")
    cpu = run_oracle(args, budget_s=args.cpu_seconds) if args.cpu_seconds > 0 else None
    if kind == "decode":
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": traffic, "peak_source": src,
                "t_roof_us": round(t_roof * 1e6, 3), "frac_of_roofline_time": round(t_roof * 1e6 / us_step, 4),
                "bytes_per_launch": nbytes,
                "tensor_i8_frac": round(2 * res["flops_factored"] * 1.0 / (us_step * 1e-6) / (i8_peak * 1e12), 4)}
    else:
        # the prefill kernel is a dense fp16/bf16 contraction: its roofline is the tensor
        # peak, counted on the product's 2 batch m d FLOPs alone (the rank-k rebuild's
        # 2 m d k n are extra work the kernel also does); the burst peak, the lower
        # fraction of the two
        gemm_flops = 2.0 * args.batch * args.m * args.d
        tflops = gemm_flops / (us_step * 1e-6) / 1e12
        roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": bf16, "unit": "TFLOP/s",
                "frac": round(tflops / bf16, 4), "traffic": dram_traffic("prefill"), "peak_source": src,
                "flops_per_launch": gemm_flops, "rebuild_flops_per_launch": res["flops_rebuild"] - gemm_flops,
                "bytes_per_launch": nbytes}
    line = {
        "metric": METRIC if args.batch == B_HEAD else METRIC.replace(f"batch {B_HEAD}", f"batch {args.batch}"),
        "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": us_step / 1000.0, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8" if kind == "decode" else "f16", "data": "synthetic",
        "config": dict(config, l2_policy=f"inputs larger than L2: {res['n_stacks']} distinct stacks "
                                         f"({res['n_stacks'] * nbytes / 2**20:.0f} MiB) rotated, L2 "
                                         f"{res['l2'] / 2**20:.0f} MiB", timing="CUDA graph replays, CUDA events"),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": round(job_us_per_call(res["ms_e2e"], res["e2e_steps"], world), 4), "unit": UNIT,
                "h2d_bytes_per_step": res["e2e_h2d"], "d2h_bytes_per_step": res["e2e_d2h"]},
        "gpu_launches": args.steps,       # one kernel (decode or prefill) per call
        "clocks": res["clocks"],
        "tokens_per_s": round(args.batch * 1e6 / value, 1),
        "weights_per_s": round(args.m * args.d * 1e6 / value, 1),
    }
    if "extras" in res:
        line["extras"] = res["extras"]
    print(json.dumps(line))


if __name__ == "__main__":
    main()
