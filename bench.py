#!/usr/bin/env python
"""Benchmark of the NVFP4 KV-cache hot path on B200.

Workload ("layer step", the 5B video DiT shape at 1280x704): one layer of
streaming generation per step -- NVFP4-quantize the new 7040-token chunk's K
and V ([7040, 24, 128] bf16) into the cache (K-smoothing, Four-Over-Six),
evict what left the window, then sink-window attention of the chunk's queries
Q [7040, 24, 128] over the global sink (chunk 0), the shot sink (chunk 4) and
the window of 3 chunks: 5 x 7040 = 35,200 keys.  Inputs are seeded synthetic
tensors (synth/), a rotating pool of 4 (K, V, Q) sets (520 MB, larger than
the 126 MB L2).

Printed (rank 0, one JSON line): value = sink-window attention TFLOP/s of the
whole step (4*T_q*L*d*H FLOPs per step over the step's device time, summed
over ranks); the quantizer's GB/s (algorithmic bytes: bf16 K, V read once,
codes + scales + mean + tensor scales written once) and both kernels'
roofline fractions; e2e = the same metric through the public API with host
buffers (pinned host -> device copies of K, V, Q and the device -> host copy of
O inside the timed region).

--impl reference times the CPU oracle on a bounded sample of the same step
(see cpu_baseline in the line).  Multi-GPU: one process per GPU (torchrun),
independent replicas (no collective on the data path), weak scaling.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

CFG = dict(H=24, d=128, T_c=7040, S_g=1, S_s=1, W=3, seed=2, shot_start=4, prefill=9, pool=4)
METRIC = "KV quantize GB/s and sink-window attention TFLOP/s (% of roofline), 1 B200"
WORKLOAD = ("one layer step: NVFP4-quantize K,V [7040,24,128] bf16 into the cache, then "
            "sink-window attention Q [7040,24,128] over S_g=1, S_s=1, W=3 chunks (35,200 keys)")
MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu
# capture of the layer step (summaries under profiles/), valid only for the kernel
# source it was taken on: a changed source reports null until it is captured again.
NCU_TRAFFIC = {
    "attention": ("sink_window_video_b200/csrc/attention_ws.cu",
                  "9b32bdc98dc3116b0a96d8fe5309c1a00aabf18bc35389e901e98f84d158d67b", 226354688),
    "matrix_1d": ("sink_window_video_b200/csrc/matrix_quant.cu",
                  "3286f4378a02393756ca9d2ec0164e9ec70777adf69cdacefd0d340704548b10", 43654912),
    "quantize": ("sink_window_video_b200/csrc/quant.cu",
                 "6a3a95c215cb0d9dd447332b23b0bcaf29d066650881108d9bb1c8938d060cfa", 97882112),
    "attention_fp4": ("sink_window_video_b200/csrc/attention_fp4.cu",
                      "385b563baf2156d9f340a5b351f880de978d2ecddd7e92a3ddefc57bd36f4a2b", 194231296),
    "rope": ("sink_window_video_b200/csrc/rope.cu",
             "99749510966436bda09ff494d743697066680af300e7be7131e030868f696f84", 45756160),
    "dequantize": ("sink_window_video_b200/csrc/dequant.cu",
                   "7dd04c898e146642244e3c647f75a4c6d746e2fad0c7c310a2255267bb2fd8f6", 51334400),
}


def ncu_traffic(which):
    path, sha, nbytes = NCU_TRAFFIC[which]
    try:
        with open(os.path.join(ROOT, path), "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    return nbytes if digest == sha else None


def keys_per_step():
    return (CFG["S_g"] + CFG["S_s"] + CFG["W"]) * CFG["T_c"]


def attn_flops(T_q=None, L=None):
    T_q = CFG["T_c"] if T_q is None else T_q
    L = keys_per_step() if L is None else L
    return 4.0 * T_q * L * CFG["d"] * CFG["H"]


def quant_bytes():
    n = CFG["T_c"] * CFG["H"] * CFG["d"]
    return 2 * n * 2 + n * 9 // 8 + CFG["H"] * CFG["d"] * 4 + 8


def load_peaks():
    try:
        with open(MEASURED_PEAKS) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
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
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x, world):
    """The maximum of x over all ranks (NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_step_per_rank, steps, world, ms_max):
    """Aggregate throughput of a weak-scaling run: every rank does the same work
    per step; the job takes the slowest rank's time."""
    return work_per_step_per_rank * steps * world / (ms_max / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ our arm

def make_inputs(rank):
    cfg = dict(CFG, seed=CFG["seed"] + 1000 * rank)
    return [synth.layer_chunk(cfg, rank, p, T_c=CFG["T_c"], H=CFG["H"], d=CFG["d"])
            for p in range(CFG["pool"])]


def run_ours(args, rank, world, local):
    import torch
    import sink_window_video_b200 as swv

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    swv.load()
    host = make_inputs(rank)

    def to_dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    pool = [tuple(to_dev(x) for x in s) for s in host]
    pinned = [tuple(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
                    for x in s) for s in host]
    T, H, d = CFG["T_c"], CFG["H"], CFG["d"]
    cache = swv.KVCache(1, H, T, CFG["S_g"], CFG["S_s"], CFG["W"])
    O = torch.empty((T, H, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    # fill the cache up to the steady state: chunks 0..8, shot switch at chunk 4
    for c in range(CFG["prefill"]):
        if c == CFG["shot_start"]:
            cache.rebind_shot_sink(c)
        K, V, _ = pool[c % CFG["pool"]]
        cache.append(0, K, V)
    torch.cuda.synchronize()

    def step(i, ev=None):
        K, V, Q = pool[i % CFG["pool"]]
        if ev is not None:
            ev[0].record(stream)
        cache.append(0, K, V)
        if ev is not None:
            ev[1].record(stream)
        cache.attention(0, Q, O)
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert cache.keyset(0) == sorted({0, CFG["shot_start"]} | set(range(
        cache.num_chunks(0) - CFG["W"], cache.num_chunks(0))))
    if cache.check_status() != swv.OK:
        raise RuntimeError("device status not OK after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(args.steps):
        step(i, evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms_total = t0.elapsed_time(t1)
    ms_quant = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    ms_attn = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    if cache.check_status() != swv.OK:
        raise RuntimeError("device status not OK after the timed steps")
    ms_total = max_over_ranks(ms_total, world)

    # end to end through the public API with host buffers: every step copies
    # its K, V, Q from pinned host memory and reads its O back; the copies run
    # on two copy streams into double buffers, so step i+1's inputs and step
    # i-1's output cross the host link while step i computes
    e2e_ms = None
    if not args.no_e2e:
        up = torch.cuda.Stream(device=dev)        # host -> device (its own copy engine)
        down = torch.cuda.Stream(device=dev)      # device -> host
        dbuf = [tuple(torch.empty_like(x) for x in pool[0]) for _ in range(2)]
        obuf = [torch.empty_like(O) for _ in range(2)]
        O_host = [torch.empty((T, H, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        loaded = [torch.cuda.Event() for _ in range(2)]
        consumed = [torch.cuda.Event() for _ in range(2)]
        drained = [torch.cuda.Event() for _ in range(2)]
        n_e2e = args.e2e_steps

        def upload(i):
            b = i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(consumed[b])          # step i-2 no longer reads this buffer
                for dst, src in zip(dbuf[b], pinned[i % CFG["pool"]]):
                    dst.copy_(src, non_blocking=True)
                loaded[b].record(up)

        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        upload(0)
        for i in range(n_e2e):
            b = i % 2
            if i + 1 < n_e2e:
                upload(i + 1)
            stream.wait_event(loaded[b])
            if i >= 2:
                stream.wait_event(drained[b])            # step i-2's O has left obuf[b]
            K, V, Q = dbuf[b]
            cache.append(0, K, V)
            cache.attention(0, Q, obuf[b])
            consumed[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(consumed[b])
                O_host[b].copy_(obuf[b], non_blocking=True)
                drained[b].record(down)
        stream.wait_stream(down)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / n_e2e

    matrix = run_matrix_quant(swv, pool, stream) if not args.no_matrix else None
    dequant = run_dequant(swv, cache, stream) if not args.no_matrix else None
    qonly = run_quantize_only(swv, stream) if not args.no_quantize_only else None
    fp4q = run_fp4q(swv, cache, pool, O, stream) if not args.no_fp4q else None
    rope = run_rope(swv, pool, stream) if not args.no_rope else None

    rollouts = None
    if not args.no_rollout:
        rollouts = [run_rollout(swv, cfg, pool, O, stream, world) for cfg in ROLLOUTS]

    return dict(ms_total=ms_total, ms_quant=ms_quant, ms_attn=ms_attn, clocks=clocks,
                e2e_ms=e2e_ms, rollouts=rollouts, matrix=matrix, dequant=dequant,
                quantize_only=qonly, fp4q=fp4q, rope=rope,
                attn_launches=swv.attention_launches(len(cache.keyset(0)), T, H, T))


# ------------------------------------------------------------------ quantize-only workload

def run_quantize_only(swv, stream, n_chunks=100):
    """The quantize-only workload as stated: 100 distinct chunks K, V [7040, 24,
    128] bf16 (seeds 1..100; K with per-channel offsets ~N(0, 4) and 1% outliers
    x20, V ~ N(0, 1)), drawn on the device by synth.device (8.7 GB resident,
    far beyond L2) and quantized back to back into 100 distinct chunk buffers.
    CUDA events around the whole run (the figure) and, in a second pass, around
    each launch."""
    import torch

    import synth.device as sd
    peaks, src = load_peaks()
    hpeak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    T, H, d = CFG["T_c"], CFG["H"], CFG["d"]
    chunks = [sd.quant_chunk(i, "cuda") for i in range(n_chunks)]
    # the device generator draws the host generator's bits (a slice of chunk 0)
    Kh, Vh = synth.quant_chunk(0, T_c=64)
    if not (np.array_equal(chunks[0][0][:64].view(torch.int16).cpu().numpy().view(np.uint16), Kh)
            and np.array_equal(chunks[0][1][:64].view(torch.int16).cpu().numpy().view(np.uint16),
                               Vh)):
        raise RuntimeError("device input generator differs from the host one")
    outs = [swv.ChunkBuffer(T, H) for _ in range(n_chunks)]
    ws = swv.new_workspace(T, H)
    for i in range(3):
        swv.quantize_chunk(chunks[i][0], chunks[i][1], outs[i], ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n_chunks):
        swv.quantize_chunk(chunks[i][0], chunks[i][1], outs[i], ws)
    e1.record(stream)
    torch.cuda.synchronize()
    us = 1e3 * e0.elapsed_time(e1) / n_chunks
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n_chunks)]
    for i, (a, b) in enumerate(ev):
        a.record(stream)
        swv.quantize_chunk(chunks[i][0], chunks[i][1], outs[i], ws)
        b.record(stream)
    torch.cuda.synchronize()
    if swv.workspace_status(ws) != swv.OK:
        raise RuntimeError("device status not OK after the quantize-only run")
    us_launch = 1e3 * sum(a.elapsed_time(b) for a, b in ev) / n_chunks
    nbytes = quant_bytes()
    gbs = nbytes / (us / 1e6) / 1e9
    del chunks, outs
    torch.cuda.empty_cache()
    return {"workload": ("quantize-only: 100 chunks K, V [7040, 24, 128] bf16, seeds 1..100, "
                         "K offsets ~N(0,4) + 1% outliers x20, device-resident (8.7 GB)"),
            "kernel": "nvfp4kv_quantize_chunk", "chunks": n_chunks,
            "us_per_chunk": us, "us_per_launch_events": us_launch,
            "bytes_per_chunk": nbytes, "achieved": gbs, "unit": "GB/s", "peak": hpeak,
            "frac": gbs / hpeak, "bound": "hbm", "peak_source": f"{src} hbm",
            "gpu_launches": 2 * n_chunks}


# ------------------------------------------------------------------ standalone de-quantization

def run_dequant(swv, cache, stream, launches=40):
    """nvfp4kv_dequantize of K and V of the cache's chunks to bf16 (rotating over
    the 5 chunks of the key set): reads codes, scales, mean and tensor scales,
    writes 2 x [7040, 24, 128] bf16."""
    import torch
    peaks, src = load_peaks()
    hpeak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    T, H, d = CFG["T_c"], CFG["H"], CFG["d"]
    chunks = [cache.chunk(0, n) for n in cache.keyset(0)]
    Ko = torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda")
    Vo = torch.empty_like(Ko)
    for i in range(3):
        swv.dequantize(chunks[i % len(chunks)], Ko, Vo)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(launches)]
    torch.cuda.synchronize()
    for i, (e0, e1) in enumerate(ev):
        e0.record(stream)
        swv.dequantize(chunks[i % len(chunks)], Ko, Vo)
        e1.record(stream)
    torch.cuda.synchronize()
    us = 1e3 * sum(e0.elapsed_time(e1) for e0, e1 in ev) / launches
    n = T * H * d
    nbytes = 2 * (n // 2 + n // 16) + H * d * 4 + 8 + 2 * 2 * n
    gbs = nbytes / (us / 1e6) / 1e9
    return {"kernel": "nvfp4kv_dequantize (K and V to bf16)", "us_per_launch": us,
            "bytes_per_launch": nbytes, "achieved": gbs, "unit": "GB/s", "peak": hpeak,
            "frac": gbs / hpeak, "bound": "hbm", "gpu_launches_per_call": 1,
            "traffic": ncu_traffic("dequantize"), "peak_source": f"{src} hbm"}


# ------------------------------------------------------------------ rotary position embedding

ROPE_GRID = (8, 22, 40)          # frames per chunk, latent rows, latent columns: 7040 tokens
ROPE_CHUNK = 9                   # the layer step's chunk: frames 72..79 of a single shot


def run_rope(swv, pool, stream, launches=40):
    """The 3D rotary embedding of the layer step's chunk: its cos/sin table, the
    rotation of the queries [7040, 24, 128] (rotating over the pool's Q tensors,
    larger than L2), and the chunk quantizer with the rotation fused into its
    reads of K, beside the quantizer alone and the unfused composition (rotate,
    then quantize).  CUDA events around each launch."""
    import torch
    peaks, src = load_peaks()
    hpeak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    T, H, d = CFG["T_c"], CFG["H"], CFG["d"]
    F, R, C = ROPE_GRID
    tab = swv.RopeTable(F, R, C)
    p0 = swv.rope_frame_position(ROPE_CHUNK, F, 0, 0)
    ws = swv.new_workspace(T, H)
    out = swv.ChunkBuffer(T, H)
    Y = torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda")
    n = len(pool)

    def timed(fn):
        for i in range(3):
            fn(i)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(launches)]
        torch.cuda.synchronize()
        for i, (e0, e1) in enumerate(ev):
            e0.record(stream)
            fn(i)
            e1.record(stream)
        torch.cuda.synchronize()
        return 1e3 * sum(e0.elapsed_time(e1) for e0, e1 in ev) / launches

    t_table = timed(lambda i: tab.fill(p0))
    t_rope = timed(lambda i: swv.rope(pool[i % n][2], tab, Y=Y))
    t_q = timed(lambda i: swv.quantize_chunk(pool[i % n][0], pool[i % n][1], out, ws))
    t_qr = timed(lambda i: swv.quantize_chunk_rope(pool[i % n][0], pool[i % n][1], tab, out, ws))
    if swv.workspace_status(ws) != swv.OK:
        raise RuntimeError("device status not OK after the rotary quantizer")
    rb = 4 * T * H * d                         # bf16 in and out
    qb = quant_bytes()
    return {"workload": f"chunk {ROPE_CHUNK} of a single shot: {F} frames of {R} x {C} tokens, "
                        f"frame coordinates {p0}..{p0 + F - 1}",
            "table_us": t_table,
            "rope": {"kernel": "nvfp4kv_rope (queries [7040, 24, 128] bf16)", "us_per_launch": t_rope,
                     "bytes_per_launch": rb, "achieved": rb / (t_rope / 1e6) / 1e9, "unit": "GB/s",
                     "peak": hpeak, "frac": rb / (t_rope / 1e6) / 1e9 / hpeak, "bound": "hbm",
                     "traffic": ncu_traffic("rope"), "peak_source": f"{src} hbm"},
            "quantize_rope": {"kernel": "nvfp4kv_quantize_chunk_rope (rotation fused)",
                              "us_per_launch": t_qr, "bytes_per_launch": qb,
                              "achieved": qb / (t_qr / 1e6) / 1e9, "unit": "GB/s", "peak": hpeak,
                              "frac": qb / (t_qr / 1e6) / 1e9 / hpeak, "bound": "hbm",
                              "peak_source": f"{src} hbm",
                              "quantize_alone_us": t_q, "unfused_us": t_rope + t_q}}


# ------------------------------------------------------------------ FP4-operand attention

# Dense tensor-core throughput of FP4 (kind::mxf4nvf4) over bf16 on B200: 9 vs
# 2.25 PFLOP/s nominal.
FP4_OVER_BF16 = 4.0


def run_fp4q(swv, cache, pool, O, stream, launches=30):
    """nvfp4kv_attention_fp4q over the layer step's key set (5 x 7040 keys):
    the queries quantized to NVFP4, Q K^T on the block-scaled FP4 tensor
    cores, P V in fp16.  Q rotates over the pool's 4 query tensors; CUDA
    events around each call (query quantizer + attention kernel (+ merge)).
    Roofline: the call's tensor time at the measured peaks -- Q K^T's FLOPs at
    the FP4 rate (measured bf16 x 4, the nominal ratio) plus P V's at the bf16
    rate -- over the measured time."""
    import torch
    peaks, src = load_peaks()
    T, H, d = CFG["T_c"], CFG["H"], CFG["d"]
    ids = cache.keyset(0)
    chunks = [cache.chunk(0, n) for n in ids]
    qb = swv.Fp4QBuffer(T, H)
    ws = cache.ws
    for i in range(3):
        swv.attention_fp4q(chunks, pool[i % len(pool)][2], O, qb, ws)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(launches)]
    torch.cuda.synchronize()
    for i, (e0, e1) in enumerate(ev):
        e0.record(stream)
        swv.attention_fp4q(chunks, pool[i % len(pool)][2], O, qb, ws)
        e1.record(stream)
    torch.cuda.synchronize()
    if swv.workspace_status(ws) != swv.OK:
        raise RuntimeError("device status not OK after the FP4-operand attention")
    ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / launches
    # how far the FP4 queries move the output from the fp16-product path
    O16 = torch.empty_like(O)
    Q = pool[0][2]
    swv.attention_fp4q(chunks, Q, O, qb, ws)
    cache.attention(0, Q, O16)
    torch.cuda.synchronize()
    rel = float(torch.linalg.vector_norm((O.float() - O16.float())) /
                torch.linalg.vector_norm(O16.float()))
    flops = attn_flops()
    tf = flops / (ms / 1e3) / 1e12
    timed_ms = ms * launches
    bpeak, bname = tensor_peak(peaks, src, timed_ms)
    fp4_peak = bpeak * FP4_OVER_BF16
    t_ideal = (flops / 2) / (fp4_peak * 1e12) + (flops / 2) / (bpeak * 1e12)
    return {"kernel": "nvfp4kv_attention_fp4q (query quantizer + attention)",
            "ms_per_launch": ms, "flops_per_launch": flops, "achieved": tf,
            "unit": "TFLOP/s", "bound": "tensor",
            "peak": flops / t_ideal / 1e12,
            "frac": (t_ideal * 1e3) / ms,
            "peak_source": f"{bname}; Q K^T at x{FP4_OVER_BF16:g} (FP4 nominal ratio)",
            "gpu_launches_per_call": swv.attention_fp4q_launches(len(ids), T, H, T),
            "traffic": ncu_traffic("attention_fp4"),
            "rel_l2_vs_f16_queries": rel}


# ------------------------------------------------------------------ weights / activations

MATRIX_SHAPES = (("activations [7040, 3072] bf16, 16-element row blocks", 1, 7040, 3072),
                 ("weights [3072, 3072] bf16, 16 x 16 tiles", 2, 3072, 3072))


def run_matrix_quant(swv, pool, stream, launches=40):
    """NVFP4 quantization of the 5B DiT's activation and weight shapes; inputs
    rotate over 8 distinct device tensors (the pool's K and V, 151-346 MB,
    larger than L2), CUDA events around each launch."""
    import torch
    peaks, src = load_peaks()
    hpeak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    ws = swv.new_matrix_workspace()
    res = []
    for name, mode, M, N in MATRIX_SHAPES:
        srcs = [t.view(-1)[:M * N].view(M, N) for s3 in pool for t in s3[:2]]
        out = swv.MatrixBuffer(M, N, mode)
        for i in range(3):
            swv.quantize_matrix(srcs[i % len(srcs)], out, ws)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(launches)]
        torch.cuda.synchronize()
        for i, (e0, e1) in enumerate(ev):
            e0.record(stream)
            swv.quantize_matrix(srcs[i % len(srcs)], out, ws)
            e1.record(stream)
        torch.cuda.synchronize()
        if swv.workspace_status(ws) != swv.OK:
            raise RuntimeError("device status not OK after the matrix quantizer")
        us = 1e3 * sum(e0.elapsed_time(e1) for e0, e1 in ev) / launches
        nbytes = 2 * M * N + M * N // 2 + (M * N // 16 if mode == 1 else M * N // 256) + 4
        gbs = nbytes / (us / 1e6) / 1e9
        res.append({"workload": name, "us_per_launch": us, "bytes_per_launch": nbytes,
                    "achieved": gbs, "unit": "GB/s", "peak": hpeak, "frac": gbs / hpeak,
                    "bound": "hbm", "peak_source": f"{src} hbm",
                    "traffic": ncu_traffic("matrix_1d") if mode == 1 else None})
    return res


# ------------------------------------------------------------------ rollouts

ROLLOUTS = (synth.ROLLOUT, synth.MULTISHOT)


def rollout_keyset_sizes(swv, cfg):
    """Chunks attended at each step of the schedule (the same in every layer),
    from the cache's own bookkeeping (advance + keyset, no device work)."""
    c = swv.KVCache(1, CFG["H"], CFG["T_c"], cfg["S_g"], cfg["S_s"], cfg["W"])
    sizes = []
    for n in range(cfg["chunks"]):
        if n in cfg["switches"]:
            c.rebind_shot_sink(n)
        c.advance(0)
        sizes.append(len(c.keyset(0)))
    return sizes


def run_rollout(swv, cfg, pool, O, stream, world):
    """One streaming rollout: every chunk of the schedule through every layer
    (quantize into the cache, then sink-window attention), shot switches
    re-binding A_s; inputs rotate over the device-resident pool."""
    import torch
    T, H = CFG["T_c"], CFG["H"]
    layers, chunks = cfg["layers"], cfg["chunks"]
    sizes = rollout_keyset_sizes(swv, cfg)
    flops = sum(sizes) * layers * attn_flops(T_q=T, L=T)
    n_quant = chunks * layers
    cache = swv.KVCache(layers, H, T, cfg["S_g"], cfg["S_s"], cfg["W"])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for n in range(chunks):
        if n in cfg["switches"]:
            cache.rebind_shot_sink(n)
        for layer in range(layers):
            K, V, Q = pool[(n * layers + layer) % len(pool)]
            cache.append(layer, K, V)
            cache.attention(layer, Q, O)
    e1.record(stream)
    torch.cuda.synchronize()
    if cache.check_status() != swv.OK:
        raise RuntimeError("device status not OK after the rollout")
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    del cache
    peaks, src = load_peaks()
    tpeak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    hpeak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    t_roof = flops / (tpeak * 1e12) + n_quant * quant_bytes() / (hpeak * 1e9)
    value = chunks * world / (ms / 1e3)
    return {"workload": (f"{cfg['name']}: {chunks} chunks x {layers} layers of [{T},{H},128], "
                         f"S_g={cfg['S_g']}, S_s={cfg['S_s']}, W={cfg['W']}, shot switches at "
                         f"{list(cfg['switches']) or 'none'}"),
            "chunks_per_s": value, "ms": ms, "attention_flops": flops,
            "gpu_launches": n_quant + sum(swv.attention_launches(k, T, H, T) for k in sizes) * layers,
            "quantizations": n_quant, "keyset_sizes": sizes,
            "roofline_chunks_per_s": chunks * world / t_roof, "frac": value * t_roof / (chunks * world),
            "roofline_basis": f"{src} bf16 sustained + {src} hbm, attention and quantizer serial"}


# ------------------------------------------------------------------ oracle (CPU)

class OracleSample:
    """The oracle on a bounded sample of the step, prepared once: the float64
    attention of `rows` query rows of head 0 over the 5 key chunks, and the NVFP4
    quantization of a `slice_tokens`-token slice of the chunk (all 24 heads).
    The quantization is per chunk; its cost is prorated to the sampled
    (row, head) pairs: t_quant_chunk * rows / (7040 * 24)."""

    def __init__(self, rows=32, slice_tokens=704, rank=0):
        import oracle
        self.oracle = oracle
        cfg = dict(CFG, seed=CFG["seed"] + 1000 * rank)
        K, V, Q = synth.layer_chunk(cfg, rank, 0)
        K2, V2, _ = synth.layer_chunk(cfg, rank, 1)
        self.Ks, self.Vs = K[:slice_tokens].copy(), V[:slice_tokens].copy()
        self.slice_tokens = slice_tokens
        h = slice(0, 1)

        def head0(q):
            return dict(q, k_codes=q["k_codes"][h], k_scales=q["k_scales"][h],
                        k_mean=q["k_mean"][h], v_codes=q["v_codes"][h], v_scales=q["v_scales"][h])
        old = head0(oracle.quantize_chunk(K2, V2))
        cur = head0(oracle.quantize_chunk(K, V))
        self.chunks = [old] * 4 + [cur]
        self.Q = np.ascontiguousarray(Q[:, h, :])
        self.rows = np.linspace(0, CFG["T_c"] - 1, rows).astype(np.int32)

    def run(self):
        """(TFLOP/s of the sample, its prorated seconds, attention seconds,
        seconds per chunk quantization, wall seconds of this call)."""
        t0 = t = time.perf_counter()
        self.oracle.quantize_chunk(self.Ks, self.Vs)
        tq_chunk = (time.perf_counter() - t) * CFG["T_c"] / self.slice_tokens
        t = time.perf_counter()
        self.oracle.attention_f64(self.chunks, self.Q, rows=self.rows)
        ta = time.perf_counter() - t
        wall = time.perf_counter() - t0
        R = len(self.rows)
        t_sample = ta + tq_chunk * R / (CFG["T_c"] * CFG["H"])
        flops = 4.0 * R * keys_per_step() * CFG["d"]
        return flops / t_sample / 1e12, t_sample, ta, tq_chunk, wall

    def entry(self, value, ta, tq_chunk):
        return {"value": value, "unit": "TFLOP/s", "cores": self.oracle.get_threads(),
                "kind": "oracle",
                "sample": (f"oracle float64 attention of {len(self.rows)} of 7040 query rows, "
                           f"head 0 of 24, over 35,200 keys ({ta:.3f} s), plus NVFP4 "
                           f"quantization of a {self.slice_tokens}-token slice of the chunk "
                           f"scaled to the chunk ({tq_chunk:.3f} s per chunk) and prorated per "
                           f"(row, head)")}

    def quantize_rates(self):
        """The oracle's chunk quantizer alone on the slice, one thread and all
        threads: GB/s of the chunk's algorithmic bytes (the slice's time
        scaled to the chunk)."""
        nbytes = quant_bytes()
        threads = self.oracle.get_threads()
        out = {"unit": "GB/s", "threads": threads,
               "sample": f"{self.slice_tokens}-token slice of the 7040 x 24 x 128 chunk, "
                         f"scaled to the chunk's {nbytes} algorithmic bytes"}
        try:
            for key, n in (("one_thread", 1), ("all_threads", threads)):
                self.oracle.set_threads(n)
                t = time.perf_counter()
                self.oracle.quantize_chunk(self.Ks, self.Vs)
                t_chunk = (time.perf_counter() - t) * CFG["T_c"] / self.slice_tokens
                out[key] = nbytes / t_chunk / 1e9
        finally:
            self.oracle.set_threads(threads)
        return out

    def baseline(self, budget_s=12.0):
        """Repeat the sample for about budget_s seconds; median value."""
        vals, t0 = [], time.perf_counter()
        while not vals or time.perf_counter() - t0 < budget_s:
            v, _, ta, tq, _ = self.run()
            vals.append(v)
        entry = self.entry(statistics.median(vals), ta, tq)
        entry["quantize"] = self.quantize_rates()
        return entry


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    smp = OracleSample(rows=args.ref_rows)
    for _ in range(args.warmup):
        smp.run()
    vals, times = [], []
    for _ in range(args.steps):
        v, _, ta, tq, wall = smp.run()
        vals.append(v)
        times.append(wall)
    value = statistics.median(vals)
    entry = smp.entry(value, ta, tq)
    sample_s = statistics.median(times)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            # each timed step is one bounded sample of the layer step (what ran)
            "ms_per_step": 1000.0 * sample_s, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded SplitMix64 + Box-Muller, 5B video DiT shapes)",
            "config": step_config(args.gpus),
            "cpu_baseline": dict(entry, sample_seconds=sample_s),
            "extrapolated": {"extrapolated": True,
                             "ms_per_full_step": 1000.0 * attn_flops() / (value * 1e12),
                             "basis": "the sample's TFLOP/s applied to the whole layer step"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ------------------------------------------------------------------ main

def wants_cpu_baseline(args, world):
    """The oracle's timing runs on rank 0 of a one-GPU run only: a bounded
    sample on the host cores, which a multi-GPU run would only keep the other
    ranks waiting for."""
    return world == 1 and not args.no_cpu_baseline


def step_config(world):
    """The workload both arms report (identical dicts, so the two lines compare)."""
    return {"workload": WORKLOAD, "global_batch": world, "seq_len": CFG["T_c"],
            "keys": keys_per_step(), "heads": CFG["H"], "head_dim": CFG["d"],
            "parallelism": f"replicas x{world}",
            "l2": "inputs rotate over 4 sets of K,V,Q (520 MB) > 126 MB L2",
            "arithmetic": "attention MMAs on fp16 operands (the de-quantized cache "
                          "exactly; bf16 Q scaled by 2^-e), fp32 accumulation and "
                          "softmax; quantizer in fp32"}


# A kernel timed over a region shorter than this runs at the burst clock; a
# longer region settles under the power cap at the sustained rate.
SUSTAINED_AFTER_MS = 1000.0


def tensor_peak(peaks, peak_src, timed_ms):
    """(peak TFLOP/s, its name) for a tensor-bound kernel timed over timed_ms:
    the burst GEMM figure for a short region, the sustained one for a long one."""
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if timed_ms < SUSTAINED_AFTER_MS:
        return burst, f"{peak_src} bf16 burst (timed region {timed_ms:.0f} ms)"
    return sust, f"{peak_src} bf16 sustained (timed region {timed_ms:.0f} ms)"


def build_line(args, r, world, peaks, peak_src):
    """The JSON line of our arm from run_ours' measurements r (every key but
    cpu_baseline, which main adds)."""
    K = args.steps
    value = whole_job_rate(attn_flops(), K, world, r["ms_total"]) / 1e12
    attn_tf = attn_flops() / (r["ms_attn"] / 1e3) / 1e12
    quant_gbs = quant_bytes() / (r["ms_quant"] / 1e3) / 1e9
    tpeak, tpeak_name = tensor_peak(peaks, peak_src, r["ms_total"])
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    hpeak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": r["ms_total"] / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded SplitMix64 + Box-Muller, 5B video DiT shapes)",
        "config": step_config(world),
        "roofline": {"bound": "tensor", "kernel": "sink_window_attention",
                     "achieved": attn_tf, "peak": tpeak, "unit": "TFLOP/s",
                     "frac": attn_tf / tpeak, "frac_burst": attn_tf / burst,
                     "frac_sustained": attn_tf / sust, "traffic": ncu_traffic("attention"),
                     "peak_source": tpeak_name},
        "quantize": {"kernel": "nvfp4kv_quantize_chunk", "bound": "hbm",
                     "achieved": quant_gbs, "peak": hpeak, "unit": "GB/s",
                     "frac": quant_gbs / hpeak, "bytes_per_launch": quant_bytes(),
                     "traffic": ncu_traffic("quantize"),
                     "ms_per_launch": r["ms_quant"], "peak_source": f"{peak_src} hbm"},
        "attention": {"ms_per_launch": r["ms_attn"], "flops_per_launch": attn_flops(),
                      "tflops": attn_tf},
        "gpu_launches": K * (1 + r["attn_launches"]),
        "clocks": r["clocks"],
    }
    if r["e2e_ms"] is not None:
        n = CFG["T_c"] * CFG["H"] * CFG["d"]
        line["e2e"] = {"value": attn_flops() * world / (r["e2e_ms"] / 1e3) / 1e12,
                       "unit": "TFLOP/s", "h2d_bytes_per_step": 3 * n * 2,
                       "d2h_bytes_per_step": n * 2, "ms_per_step": r["e2e_ms"]}
    if r["rollouts"] is not None:
        line["rollouts"] = r["rollouts"]
    if r["matrix"] is not None:
        line["matrix_quantize"] = r["matrix"]
    if r["dequant"] is not None:
        line["dequantize"] = r["dequant"]
    if r.get("quantize_only") is not None:
        line["quantize_only"] = r["quantize_only"]
    if r.get("fp4q") is not None:
        line["attention_fp4q"] = r["fp4q"]
    if r.get("rope") is not None:
        line["rope"] = r["rope"]
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rollout", action="store_true")
    ap.add_argument("--no-matrix", action="store_true")
    ap.add_argument("--no-quantize-only", action="store_true")
    ap.add_argument("--no-fp4q", action="store_true")
    ap.add_argument("--no-rope", action="store_true")
    ap.add_argument("--ref-rows", type=int, default=32)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    if args.impl == "reference":
        run_reference(args)
        return

    rank, world, local = dist_setup(args.gpus)
    r = run_ours(args, rank, world, local)
    peaks, peak_src = load_peaks()
    if rank == 0:
        line = build_line(args, r, world, peaks, peak_src)
        if wants_cpu_baseline(args, world):
            line["cpu_baseline"] = OracleSample(rows=args.ref_rows).baseline()
        print(json.dumps(line))
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
