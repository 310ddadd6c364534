#!/usr/bin/env python
"""Benchmark of the mixed-precision KV-cache hot path on B200.

Headline workload (one GPU): decode attention at 64k context over a kvarn4 cache with a
1024-token BF16 tail, 8 KV heads x 128, 40 query heads, batch 1.  One step = append one
token (tail write, spill of the oldest tail token into its kvarn group, WHT, Sinkhorn,
quantize) + decode attention (Q rotation, split-K over the quantized pages and the tail,
merge with the inverse rotation of the V accumulator), issued as one kvq_append_decode call
(the decode overlaps the spill).  Steps cycle over `--layers`
independent layer caches (8 x 81.6 MB by default) so that every step reads its cache from
HBM, not L2.  The metric is decode KV bytes read per second (algorithmic bytes: codes,
scales and tail rows of every K/V stream at the step's context length).

`--impl reference` times the CPU oracle (oracle/, plain C) on the same workload instead.
Multi-GPU (torchrun): every rank runs the same workload on its own GPU (no collective on
the data path: independent sequences / layers); rank 0 prints the max-over-ranks time.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn KV GB/s (% of HBM peak) at 64k ctx; append Mtok/s; vs CPU oracle"
D = 128
REPS_APPEND = 5


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=512)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--type", default="kvarn4")
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--quick", action="store_true", help="skip the per-type sweep and the append workload")
    ap.add_argument("--part", default="all", choices=["all", "append", "prefill"],
                    help="append / prefill: only the batched append or the chunk-attention workload "
                         "(for a profiler run)")
    return ap.parse_args()


# ---------------------------------------------------------------------------------------
# algorithmic bytes

def decode_bytes(calc, type_, n, tail, hkv, hq):
    """Algorithmic bytes of one decode step at context n: every K/V stream once (packed codes,
    fp16 scales, kvarn channel scales, BF16 tail rows) plus q in and out (fp32).  `calc` is
    a payload calculator: the library's (our arm) or the oracle's (reference arm)."""
    per_stream = calc.payload_bytes(type_, 1, 1, n, tail) / 2.0
    return 2 * hkv * per_stream + 2 * hq * D * 4


class LibCalc:
    """The library's host-only payload calculator (kvq_payload_bytes)."""

    def __init__(self, kvq):
        self.kvq = kvq

    def payload_bytes(self, type_, n_layers, n_kv_heads, n, tail):
        return self.kvq.kvq_payload_bytes(type_, n_layers, n_kv_heads, n, tail)


# ---------------------------------------------------------------------------------------
# clocks

class ClockSampler:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.f.flush()
        rows = []
        with open(self.f.name) as fh:
            for line in fh:
                c = [x.strip() for x in line.split(",")]
                if len(c) < 10:
                    continue
                try:
                    rows.append(dict(sm=float(c[2]), smax=float(c[3]), power=float(c[4]), hw=c[6], hwt=c[7],
                                     swt=c[8], swp=c[9]))
                except ValueError:
                    continue
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        reasons = set()
        for r in rows:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                            ("swp", "sw_power_cap")):
                if r[k].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------------------------------
# distributed plumbing (one process per GPU; measurement only, no data-path collective)

def dist_init(args):
    import torch

    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        if torch.cuda.is_available():
            torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(ws, x):
    """The largest x over all ranks (every rank gets it): the job's time is its slowest rank's."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(ws, bytes_per_rank, ms_max):
    """Whole-job throughput (GB/s) of ws independent replicas that each moved bytes_per_rank,
    timed by the slowest rank."""
    return ws * bytes_per_rank / (ms_max * 1e-3) / 1e9


# ---------------------------------------------------------------------------------------
# our implementation

def dev_bf16(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def build_decode_workload(torch, kvq, cfg, type_, layers, tokens_per_layer):
    """Cache with `layers` layer copies of the 64k workload, each prefilled to
    n - tokens_per_layer tokens; returns the cache and device inputs."""
    n, hkv, hq, tail = cfg["n"], cfg["hkv"], cfg["hq"], cfg["tail"]
    cache = kvq.KVCache(n_layers=layers, n_seqs=1, n_kv_heads=hkv, max_ctx=n, type_k=type_, type_v=type_,
                        tail=tail)
    from bit_kv_cache_17_b200 import synth

    kt = dev_bf16(torch, synth.token_major(cfg["k"]))
    vt = dev_bf16(torch, synth.token_major(cfg["v"]))
    P = n - tokens_per_layer
    for l in range(layers):
        cache.append(l, [0], [P], kt[:P], vt[:P])
    torch.cuda.synchronize()
    return cache, kt, vt, P


def graph_upload(torch, g):
    """Uploads an instantiated CUDA graph to the device (cudaGraphUpload on the current
    stream), so that its first replay inside a timed region does not include the upload."""
    import ctypes

    rt = ctypes.CDLL("libcudart.so.12")
    rt.cudaGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    rc = rt.cudaGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()),
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, f"cudaGraphUpload: {rc}"


def run_ours(args, ws, rank):
    import torch

    from bit_kv_cache_17_b200 import kvq, synth

    calc = LibCalc(kvq)
    cfg = synth.config2()
    hkv, hq, tail, n = cfg["hkv"], cfg["hq"], cfg["tail"], cfg["n"]
    L = args.layers
    W, K = args.warmup, args.steps
    K_e2e = max(8, min(K, 256))
    per_layer = math.ceil((W + K + K_e2e) / L)
    assert per_layer <= 4096, "too many steps for the 64k context window"
    cache, kt, vt, P = build_decode_workload(torch, kvq, cfg, args.type, L, per_layer)
    qdev = torch.from_numpy(cfg["q"][:, 0]).cuda()  # [128, hq, 128]
    out = torch.empty((W + K, 1, hq, D), dtype=torch.float32, device="cuda")
    cache.workspace(1, hq)

    def step(s, out_row):
        layer, tok = s % L, P + s // L
        cache.append_decode(layer, [0], [1], kt[tok:tok + 1], vt[tok:tok + 1], qdev[s % qdev.shape[0]][None],
                            out=out_row)

    def ctx(s):
        return P + s // L + 1

    # warm-up steps run eagerly (first launches set kernel attributes), then the timed
    # steps are captured into CUDA graphs and replayed once
    for s in range(W):
        step(s, out[s])
    torch.cuda.synchronize()
    launches0 = kvq.kvq_launch_count()
    graphs = []
    chunk = 1024
    for c0 in range(W, W + K, chunk):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for s in range(c0, min(W + K, c0 + chunk)):
                step(s, out[s])
        graphs.append(g)
    launches = kvq.kvq_launch_count() - launches0
    for g in graphs:
        graph_upload(torch, g)

    # decode-only graph (state unchanged) for the kernel's own duration and a clock soak
    dec_out = torch.empty((1, hq, D), dtype=torch.float32, device="cuda")
    gd = torch.cuda.CUDAGraph()
    ND = 64
    with torch.cuda.graph(gd):
        for i in range(ND):
            cache.decode(i % L, [0], qdev[i % qdev.shape[0]][None], out=dec_out)
    torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    sampler = ClockSampler("GPU-" + str(props.uuid))
    sampler.start()
    # soak ~1 s so that the clocks sampled below describe a GPU under this load
    t_end = time.time() + 1.0
    while time.time() < t_end:
        gd.replay()
        torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 20
    e0.record()
    for _ in range(reps):
        gd.replay()
    e1.record()
    torch.cuda.synchronize()
    dec_ms = e0.elapsed_time(e1) / (reps * ND)

    barrier(ws)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for g in graphs:
        g.replay()
    t1.record()
    torch.cuda.synchronize()
    barrier(ws)
    ms = t0.elapsed_time(t1)
    clocks = sampler.stop()
    ms_max = max_over_ranks(ws, ms)

    bytes_steps = sum(decode_bytes(calc, args.type, ctx(s), tail, hkv, hq) for s in range(W, W + K))
    value = weak_value(ws, bytes_steps, ms_max)
    dec_bytes = decode_bytes(calc, args.type, ctx(W + K - 1), tail, hkv, hq)
    assert cache.status() == 0

    # end to end through the public API with host buffers, every step: one H2D copy of the
    # step's inputs (token K and V rows, then q) from pinned memory into a device staging
    # buffer, kvq_append_decode, and a D2H copy of the output into pinned memory
    kb, qb = hkv * D * 2, hq * D * 4
    kall = np.ascontiguousarray(synth.token_major(cfg["k"])[P:]).view(np.uint8).reshape(-1, kb)
    vall = np.ascontiguousarray(synth.token_major(cfg["v"])[P:]).view(np.uint8).reshape(-1, kb)
    qall = np.ascontiguousarray(cfg["q"][:, 0]).view(np.uint8).reshape(-1, qb)
    s0 = W + K
    hstage = np.empty((K_e2e, 2 * kb + qb), dtype=np.uint8)
    for j in range(K_e2e):
        s = s0 + j
        tok = s // L
        hstage[j, :kb] = kall[tok]
        hstage[j, kb:2 * kb] = vall[tok]
        hstage[j, 2 * kb:] = qall[s % qall.shape[0]]
    hstage = torch.from_numpy(hstage).pin_memory()
    hout = torch.empty((K_e2e, 1, hq, D), dtype=torch.float32).pin_memory()
    dstage = torch.empty(2 * kb + qb, dtype=torch.uint8, device="cuda")
    dk = dstage[:kb].view(torch.bfloat16).view(1, hkv, D)
    dv = dstage[kb:2 * kb].view(torch.bfloat16).view(1, hkv, D)
    dq = dstage[2 * kb:].view(torch.float32).view(1, hq, D)
    do = torch.empty((1, hq, D), dtype=torch.float32, device="cuda")
    barrier(ws)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for j in range(K_e2e):
        dstage.copy_(hstage[j], non_blocking=True)
        cache.append_decode((s0 + j) % L, [0], [1], dk, dv, dq, out=do)
        hout[j].copy_(do, non_blocking=True)
    a1.record()
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = max_over_ranks(ws, a0.elapsed_time(a1))
    e2e_bytes = sum(decode_bytes(calc, args.type, ctx(s0 + j), tail, hkv, hq) for j in range(K_e2e))
    e2e = {"value": round(weak_value(ws, e2e_bytes, e2e_ms), 2), "unit": "GB/s",
           "h2d_bytes_per_step": int(2 * hkv * D * 2 + hq * D * 4), "d2h_bytes_per_step": int(hq * D * 4),
           "steps": K_e2e, "ms_per_step": round(e2e_ms / K_e2e, 4)}

    peaks = load_peaks()
    achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
    roof = {"kernel": "k_decode (split-K decode + merge)", "bound": "hbm", "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "peak_source": peaks["source"], "avg_launch_us": round(dec_ms * 1e3, 2),
            "bytes_per_launch": int(dec_bytes), "traffic": traffic_for("decode", args.type)}

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": W,
        "ms_per_step": round(ms_max / K, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic (seeded AR(1) K/V, N(0,1) queries; see bit_kv_cache_17_b200/synth.py)",
        "config": {"workload": f"decode @64k: {args.type}, context {P + 1}..{ctx(W + K - 1)}, tail {tail} BF16, "
                               f"{hkv} KV heads x 128, {hq} query heads, batch 1, 1 token appended per step",
                   "layer_caches_cycled": L, "hbm_frac_of_peak": round(value / ws / peaks["hbm_gbs"], 4),
                   "l2": f"inputs larger than L2: {L} layer caches x {dec_bytes / 1e6:.1f} MB cycled",
                   "parallelism": f"weak: {ws} independent replicas, no collective on the data path"},
        "roofline": roof, "e2e": e2e, "gpu_launches": int(launches), "clocks": clocks,
    }
    del graphs, gd
    return result, cfg, cache


def run_type_sweep(args, kvq, torch, synth, cfg):
    calc = LibCalc(kvq)
    out = {}
    for t in ("kvarn2", "kvarn3", "kvarn4", "kvarn5", "kvarn6", "kvarn8", "q4_0", "bf16"):
        L = args.layers
        cache, kt, vt, P = build_decode_workload(torch, kvq, cfg, t, L, 1)
        # fill the last token so that every layer holds exactly 65536 tokens
        for l in range(L):
            cache.append(l, [0], [1], kt[P:P + 1], vt[P:P + 1])
        qdev = torch.from_numpy(cfg["q"][0, 0]).cuda()[None]
        o = torch.empty_like(qdev)
        cache.workspace(1, cfg["hq"])
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(4 * L):
                cache.decode(i % L, [0], qdev, out=o)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (40 * L)
        b = decode_bytes(calc, t, cfg["n"], cfg["tail"] if t != "bf16" else 0, cfg["hkv"], cfg["hq"])
        out[t] = {"decode_us": round(us, 2), "GB_per_s": round(b / us / 1e3, 1), "bytes": int(b)}
        del cache, g
        torch.cuda.empty_cache()
    return out


def graph_time_us(torch, fn, reps=10):
    """Mean duration in microseconds of one replay of a CUDA graph of fn() (after one
    untimed replay)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / reps


def run_formats(args, kvq, torch, synth):
    """Plain block formats at context 16384 with tails 0 / 1024 / 2048 (8 KV heads, 32 query
    heads): decode GB/s, cycling enough layer caches that every decode reads from HBM."""
    calc = LibCalc(kvq)
    cfg = synth.config1()
    n, hkv, hq = cfg["n"], cfg["hkv"], cfg["hq"]
    kt = dev_bf16(torch, synth.token_major(cfg["k"]))
    vt = dev_bf16(torch, synth.token_major(cfg["v"]))
    qdev = torch.from_numpy(cfg["q"][0, 0]).cuda()[None]
    o = torch.empty_like(qdev)
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    out = {}
    for t in cfg["types"]:
        for tail in cfg["tails"]:
            b = decode_bytes(calc, t, n, tail, hkv, hq)
            L = max(2, math.ceil(4 * l2 / b))
            cache = kvq.KVCache(n_layers=L, n_seqs=1, n_kv_heads=hkv, max_ctx=n, type_k=t, type_v=t, tail=tail)
            for l in range(L):
                cache.append(l, [0], [n], kt, vt)
            cache.workspace(1, hq)

            def fn():
                for i in range(4 * L):
                    cache.decode(i % L, [0], qdev, out=o)

            us = graph_time_us(torch, fn) / (4 * L)
            out[f"{t}/T{tail}"] = {"decode_us": round(us, 2), "GB_per_s": round(b / us / 1e3, 1), "bytes": int(b),
                                   "layers_cycled": L}
            assert cache.status() == 0
            del cache
            torch.cuda.empty_cache()
    return {"workload": f"context {n}, {hkv} KV heads x 128, {hq} query heads, batch 1, tails {cfg['tails']}",
            "per_format": out}


def run_page1_shape(args, kvq, torch, synth):
    """64 layers x 8 KV heads x 128, 64 query heads, context 240000: one decode over all 64
    layers (one CUDA graph), kvarn2 and q4_0 with a 1024-token tail, and all-BF16.  The
    seeded data of layer 0 is appended to every layer (the kernels' timing does not depend
    on the values)."""
    calc = LibCalc(kvq)
    cfg = synth.config4_layer(0)
    n, hkv, hq, tail = cfg["n"], cfg["hkv"], cfg["hq"], cfg["tail"]
    NL = 64
    kt = dev_bf16(torch, synth.token_major(cfg["k"]))
    vt = dev_bf16(torch, synth.token_major(cfg["v"]))
    qdev = torch.from_numpy(cfg["q"][0, 0]).cuda()[None]
    o = torch.empty((NL, 1, hq, D), dtype=torch.float32, device="cuda")
    out = {}
    for t in cfg["types"]:
        tl = tail if t != "bf16" else 0
        cache = kvq.KVCache(n_layers=NL, n_seqs=1, n_kv_heads=hkv, max_ctx=n, type_k=t, type_v=t, tail=tl)
        for l in range(NL):
            cache.append(l, [0], [n], kt, vt)
        cache.workspace(1, hq)

        def fn():
            for l in range(NL):
                cache.decode(l, [0], qdev, out=o[l])

        us = graph_time_us(torch, fn, reps=3)
        b = NL * decode_bytes(calc, t, n, tl, hkv, hq)
        out[t] = {"decode_64_layers_ms": round(us / 1e3, 3), "GB_per_s": round(b / us / 1e3, 1), "bytes": int(b),
                  "cache_bytes": int(cache.nbytes)}
        assert cache.status() == 0
        del cache
        torch.cuda.empty_cache()
    return {"workload": f"{NL} layers, context {n}, {hkv} KV heads x 128, {hq} query heads, batch 1, "
                        f"tail {tail} (quantized types); layer 0's seeded data in every layer", "per_type": out}


def run_prefill(args, kvq, torch, synth):
    """Chunk attention (kvq_prefill_attn): a 64k-context kvarn4 cache (the headline data) takes
    a chunk of 16 new tokens, whose 16 queries then attend causally; timed in a CUDA graph
    cycling layer caches.  Each 64-token tile of the cache is read and rebuilt once for all query
    rows (tcgen05 tensor cores, accumulators in tensor memory)."""
    calc = LibCalc(kvq)
    cfg = synth.config2()
    n, hkv, hq, tail = cfg["n"], cfg["hkv"], cfg["hq"], cfg["tail"]
    M, L = 16, 4
    cache, kt, vt, P = build_decode_workload(torch, kvq, cfg, "kvarn4", L, M)
    for l in range(L):
        cache.append(l, [0], [M], kt[P:P + M], vt[P:P + M])
    q = torch.from_numpy(np.ascontiguousarray(cfg["q"][:M, 0])).cuda()  # [M, hq, 128]
    o = torch.empty_like(q)
    cache.workspace(M, hq)

    def fn():
        for i in range(2 * L):
            cache.prefill_attn(i % L, 0, q, out=o)

    us = graph_time_us(torch, fn) / (2 * L)
    b = sum(decode_bytes(calc, "kvarn4", n - M + 1 + i, tail, hkv, 0) for i in range(M)) + 2 * M * hq * D * 4
    assert cache.status() == 0
    del cache
    return {"workload": f"context {n}, kvarn4, tail {tail}, {hkv} KV heads, {hq} query heads, a chunk of {M} "
                        f"queries (causal)", "us_per_chunk": round(us, 2), "query_rows_per_s": round(M / us * 1e6),
            "GB_per_s_per_row_reads": round(b / us / 1e3, 1)}


def run_quality(args, kvq, torch, synth):
    """Side report (not a target): attention KL(P_bf16 || P_q) and the relative L2 error of the
    attention output of a quantized cache against the BF16 cache of the same data (context
    16384, 8 KV heads, 32 query heads, 4 query draws).  The cache is read back through
    kvq_dequant (original basis); the attention itself is plain fp32 torch, outside the
    product path.  Data sets: the formats workload's AR(1) data with four K outlier channels
    x20 (every type, tails 0..2048), and two i.i.d. N(0, 1) sets at tails 0 and 1024 for the
    2- to 4-bit types: with K channels 7 and 63 x16 (the PR1 data) and with no outliers, which
    separate what the outlier channels do to the rotated types from the types themselves."""
    cfg = synth.config1()
    n, hkv, hq = cfg["n"], cfg["hkv"], cfg["hq"]
    G = hq // hkv
    rng = np.random.default_rng(11)
    q = torch.from_numpy(rng.standard_normal((4, hq, D)).astype(np.float32)).cuda()

    def attend(kf, vf):  # kf, vf: [n, hkv, D] fp32 -> probabilities [4, hq, n], out [4, hq, D]
        kk = kf.permute(1, 0, 2).repeat_interleave(G, 0)  # [hq, n, D]
        vv = vf.permute(1, 0, 2).repeat_interleave(G, 0)
        s = torch.einsum("bhd,hnd->bhn", q, kk) / math.sqrt(D)
        p = torch.softmax(s, -1)
        return p, torch.einsum("bhn,hnd->bhd", p, vv)

    def sweep(kbits, vbits, types, tails):
        kt = dev_bf16(torch, synth.token_major(kbits))
        vt = dev_bf16(torch, synth.token_major(vbits))
        p0, o0 = attend(kt.float(), vt.float())
        lp0 = torch.log(p0.clamp_min(1e-38))
        out = {}
        for t in types:
            row = {}
            for tail in tails:
                cache = kvq.KVCache(n_layers=1, n_seqs=1, n_kv_heads=hkv, max_ctx=n, type_k=t, type_v=t, tail=tail)
                cache.append(0, [0], [n], kt, vt)
                kf = cache.dequant(0, 0, 0, 0, n)
                vf = cache.dequant(0, 0, 1, 0, n)
                p1, o1 = attend(kf, vf)
                kl = (p0 * (lp0 - torch.log(p1.clamp_min(1e-38)))).sum(-1)  # [4, hq]
                rel = (o1 - o0).norm(dim=-1) / o0.norm(dim=-1)
                row[f"T{tail}"] = {"kl_mean": float(kl.mean()), "kl_median": float(kl.median()),
                                   "out_rel_l2_mean": float(rel.mean())}
                del cache
            out[t] = row
        return out

    types = ["q2_0", "q3_0", "q4_0", "q5_0", "q6_0", "q8_0", "q4_1", "q2_1", "q3_1", "q5_1", "q6_1",
             "kvarn2", "kvarn3", "kvarn4", "kvarn5", "kvarn6", "kvarn8"]
    res = {"workload": f"context {n}, {hkv} KV heads, {hq} query heads, 4 query draws (seed 11)",
           "ar1_outliers20": sweep(cfg["k"], cfg["v"], types, (0, 256, 512, 1024, 2048))}
    low = ["q2_0", "q3_0", "q4_0", "kvarn2", "kvarn3", "kvarn4"]
    k, v = synth.kv_iid(np.random.default_rng(12), hkv, n)
    res["iid_outliers16"] = sweep(k, v, low, (0, 1024))
    k, v = synth.kv_iid(np.random.default_rng(13), hkv, n, outlier_channels=())
    res["iid_plain"] = sweep(k, v, low, (0, 1024))
    return res


def run_append(args, kvq, torch, synth):
    """Batched prefill-append: 16 sequences built to L_i ~ U[4096, 32768], then one timed
    append of 4096 tokens per sequence (kvarn4, tail 1024), then 64 batched decode steps
    (one token appended to every sequence, then decode of all 16)."""
    NSTEP = 64
    cfg = synth.config3(steps=NSTEP)
    hkv, hq, tail = cfg["hkv"], cfg["hq"], cfg["tail"]
    Ls = cfg["lengths"]
    S = len(Ls)
    cache = kvq.KVCache(n_layers=1, n_seqs=S, n_kv_heads=hkv, max_ctx=max(Ls) + cfg["prefill"] + 64,
                        type_k="kvarn4", type_v="kvarn4", tail=tail)
    ks = [dev_bf16(torch, synth.token_major(k)) for k in cfg["k"]]
    vs = [dev_bf16(torch, synth.token_major(v)) for v in cfg["v"]]
    cache.append(0, list(range(S)), Ls, torch.cat([k[:l] for k, l in zip(ks, Ls)]),
                 torch.cat([v[:l] for v, l in zip(vs, Ls)]))
    P = cfg["prefill"]
    kin = torch.cat([k[l:l + P] for k, l in zip(ks, Ls)])
    vin = torch.cat([v[l:l + P] for v, l in zip(vs, Ls)])
    torch.cuda.synchronize()
    # the state before the append: every replay of the captured append starts from it (the
    # restore is a device copy larger than L2, outside the timed region)
    snap = cache.storage.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cache.append(0, list(range(S)), [P] * S, kin, vin)
    graph_upload(torch, g)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for _ in range(REPS_APPEND):
        cache.storage.copy_(snap)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    del snap
    ms = statistics.median(times)
    assert cache.status() == 0

    # batched decode steps: append one token per sequence, then decode all of them
    calc = LibCalc(kvq)
    qd = torch.from_numpy(cfg["q"]).cuda()  # [steps, S, hq, 128]
    od = torch.empty((S, hq, D), dtype=torch.float32, device="cuda")
    cache.workspace(S, hq)
    ksteps = torch.stack([torch.cat([k[l + P + j:l + P + j + 1] for k, l in zip(ks, Ls)]) for j in range(NSTEP)])
    vsteps = torch.stack([torch.cat([v[l + P + j:l + P + j + 1] for v, l in zip(vs, Ls)]) for j in range(NSTEP)])
    gs = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gs):
        for j in range(NSTEP):
            cache.append_decode(0, list(range(S)), [1] * S, ksteps[j], vsteps[j], qd[j], out=od)
    e0.record()
    gs.replay()
    e1.record()
    torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / NSTEP
    assert cache.status() == 0
    ctx_end = [l + P + NSTEP for l in Ls]
    dec_b = sum(decode_bytes(calc, "kvarn4", c, tail, hkv, hq) for c in ctx_end)
    dec_us = graph_time_us(torch, lambda: cache.decode(0, list(range(S)), qd[0], out=od))
    batched = {"steps": NSTEP, "ms_per_step": round(step_ms, 4),
               "step_GB_per_s": round(dec_b / (step_ms * 1e-3) / 1e9, 1),
               "decode_us": round(dec_us, 2), "decode_GB_per_s": round(dec_b / dec_us / 1e3, 1),
               "decode_bytes": int(dec_b),
               "workload": f"{S} sequences at {min(ctx_end)}..{max(ctx_end)} tokens, kvarn4, tail {tail}, "
                           f"{hkv} KV heads, {hq} query heads; step = append 1 token to each + decode all"}
    # algorithmic bytes: new rows in, the old tail + open-group rows re-read, quantized
    # tokens and the new tail out (per stream)
    tb = 75.0
    moved = 0.0
    for l in Ls:
        q0 = l - tail
        q1 = l + P - tail
        staged = q0 - (q0 // 256) * 256
        moved += 2 * hkv * (P * 256 + (tail + staged) * 256 + (q1 - (q0 // 256) * 256) * tb + tail * 256)
    peaks = load_peaks()
    gbs = moved / (ms * 1e-3) / 1e9
    roof = {"kernel": "kvq_append (k_spill_kvarn + k_tail_write)", "bound": "alu (kvarn: WHT + Sinkhorn)",
            "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
            "ms_per_launch_median": round(ms, 4), "ms_all": [round(x, 4) for x in times],
            "bytes_per_launch": int(moved), "traffic": traffic_for("spill_bulk_cfg3", "kvarn4")}
    return {"metric": "append Mtok/s", "value": round(S * P / (ms * 1e-3) / 1e6, 2), "unit": "Mtok/s",
            "ms": round(ms, 4), "GB_per_s": round(gbs, 1), "bytes": int(moved), "roofline": roof,
            "workload": f"{S} sequences, lengths {min(Ls)}..{max(Ls)}, +{P} tokens each in one call, kvarn4, "
                        f"tail {tail}, 8 KV heads x 128", "batched_decode": batched}


# ---------------------------------------------------------------------------------------
# measured peaks and committed ncu traffic

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured (MEASURED_PEAKS.json)"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


def traffic_for(kernel, type_):
    """dram bytes per launch from the committed ncu summary, or None when the kernel source
    changed since the counters were taken."""
    import hashlib

    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(f"{kernel}:{type_}")
    if not ent:
        return None
    src = os.path.join(ROOT, "bit_kv_cache_17_b200", "csrc", ent["source"])
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return ent["dram_bytes_per_launch"] if h == ent["source_sha256_16"] else None


# ---------------------------------------------------------------------------------------
# the CPU oracle

def _oracle_rows(oracle, type_, hist, tail):
    """fp64 rows of one stream as the oracle's decode reads them: the quantized region
    dequantized in the original basis, then the BF16 tail exactly."""
    st = oracle.stream_state(type_, hist, tail)
    Q = st["Q"]
    rows = np.empty((hist.shape[0], D), np.float64)
    rows[:Q] = oracle.dequant(type_, st, basis=0)
    rows[Q:] = oracle.bf16_to_f32(hist[Q:])
    return rows


def _oracle_decode_job(job):
    """One KV head: its state is built untimed, then the oracle's fp64 attention of the G
    query heads over it is timed (runs in a spawned worker); returns seconds."""
    import oracle

    type_, k, v, tail, q = job
    kr = _oracle_rows(oracle, type_, k, tail)
    vr = _oracle_rows(oracle, type_, v, tail)
    t0 = time.perf_counter()
    oracle.attend(q, kr, vr, 1.0 / math.sqrt(D))
    return time.perf_counter() - t0


def _oracle_append_job(job):
    """One stream of the append sample: the oracle quantizes `n_new` tokens (WHT, Sinkhorn,
    block quantization of whole groups) behind a BF16 tail; returns seconds."""
    import oracle

    type_, hist, tail = job
    t0 = time.perf_counter()
    oracle.stream_state(type_, hist, tail)
    return time.perf_counter() - t0


def cpu_baseline(cfg, type_):
    """The oracle on the host cores, in spawned worker processes (no worker inherits a CUDA
    context), one KV head (decode) or one stream (append) per job:
      - decode: one decode step at 64k over a state built before the timed call (the
        oracle's fp64 attention over its dequantized rows), all KV heads;
      - append: a sample of the batched append workload, 4096 new tokens of one sequence
        (8 KV heads x K and V) quantized behind the 1024-token BF16 tail."""
    import multiprocessing as mp

    import oracle as calc

    n, hkv = cfg["n"], cfg["hkv"]
    G = cfg["hq"] // hkv
    q = cfg["q"][0, 0]
    cores = len(os.sched_getaffinity(0))
    nproc = max(1, min(cores, 2 * hkv))
    dec_jobs = [(type_, cfg["k"][h, :n], cfg["v"][h, :n], cfg["tail"], q[h * G:(h + 1) * G]) for h in range(hkv)]
    n_new, tail = 4096, cfg["tail"]
    app_jobs = [(type_, x[h, :n_new + tail], tail) for h in range(hkv) for x in (cfg["k"], cfg["v"])]
    with mp.get_context("spawn").Pool(nproc) as pool:
        pool.map(_oracle_append_job, [(type_, cfg["k"][0, :300], 0)] * nproc)  # start the workers untimed
        t0 = time.perf_counter()
        dec = pool.map(_oracle_decode_job, dec_jobs)
        dec_wall = time.perf_counter() - t0  # includes the untimed state builds: not used
        t0 = time.perf_counter()
        app = pool.map(_oracle_append_job, app_jobs)
        app_wall = time.perf_counter() - t0
    b = decode_bytes(calc, type_, n, cfg["tail"], hkv, cfg["hq"])
    dec_cpu = sum(dec)
    par = min(nproc, hkv)
    dec_par_s = max(dec) if par >= hkv else dec_cpu / par
    return {"value": round(b / dec_par_s / 1e9, 4), "unit": "GB/s", "cores": par, "kind": "oracle",
            "single_thread_value": round(b / dec_cpu / 1e9, 4),
            "sample": f"decode: one step at context {n} ({type_}, {hkv} KV heads, {cfg['hq']} query heads), "
                      f"state built untimed, one KV head per worker on {par} of {cores} host cores "
                      f"({dec_cpu:.2f} s CPU in attention); append: {n_new} new tokens of one sequence "
                      f"(8 KV heads x K/V, behind a {tail}-token tail), one stream per worker",
            "append": {"value": round(n_new / app_wall / 1e6, 5), "unit": "Mtok/s", "cores": nproc,
                       "single_thread_value": round(n_new / sum(app) / 1e6, 6),
                       "seconds_cpu": round(sum(app), 2), "seconds_wall": round(app_wall, 2)}}


def run_reference(args, ws, rank):
    """The CPU oracle as the reference arm.  Each step is a bounded sample of the workload:
    the decode of one KV head over a 4096-token window of its 64k stream (3072 quantized
    tokens + the 1024-token BF16 tail), windows and heads cycling, so that the whole run
    ends within minutes on one core."""
    import oracle
    from bit_kv_cache_17_b200 import synth

    calc = oracle
    cfg = synth.config2()
    win, hkv, G = 4096, cfg["hkv"], cfg["hq"] // cfg["hkv"]
    q = cfg["q"][0, 0]
    steps = []
    for s in range(args.warmup + args.steps):
        h = s % hkv
        a = (s // hkv * win) % (cfg["n"] - win)
        a -= a % 256
        t0 = time.perf_counter()
        oracle.decode_head(args.type, args.type, cfg["k"][h, a:a + win], cfg["v"][h, a:a + win], cfg["tail"],
                           q[h * G:(h + 1) * G])
        if s >= args.warmup:
            steps.append(time.perf_counter() - t0)
    b = decode_bytes(calc, args.type, win, cfg["tail"], 1, G)
    tot = sum(steps)
    value = b * len(steps) / tot / 1e9
    sample = (f"each step: decode of 1 of {hkv} KV heads over a {win}-token window (3072 {args.type} + 1024 BF16 "
              f"tail) of the 64k stream, single-threaded C oracle")
    return {"metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(tot / len(steps) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": f"decode @64k: {args.type}, context {cfg['n']}, tail {cfg['tail']} BF16, "
                                   f"{hkv} KV heads x 128, {cfg['hq']} query heads, batch 1"},
            "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def compact(x, digits=4):
    """Floats rounded to `digits` significant digits, recursively."""
    if isinstance(x, float):
        return float(f"{x:.{digits}g}")
    if isinstance(x, dict):
        return {k: compact(v, digits) for k, v in x.items()}
    if isinstance(x, list):
        return [compact(v, digits) for v in x]
    return x


def summary(result):
    """The side workloads as roofline fractions of the measured HBM peak (and their times),
    compact enough to travel with the roofline object."""
    peak = load_peaks()["hbm_gbs"]
    out = {}
    a = result.get("append")
    if a:
        out["append_cfg3"] = {"Mtok_per_s": a["value"], "ms": a["ms"], "GB_per_s": a["GB_per_s"],
                              "frac": a["roofline"]["frac"], "traffic": a["roofline"]["traffic"],
                              "bytes_per_launch": a["bytes"]}
        b = a["batched_decode"]
        out["batched_decode_cfg3"] = {"step_ms": b["ms_per_step"], "decode_us": b["decode_us"],
                                      "decode_frac": round(b["decode_GB_per_s"] / peak, 4)}
    t = result.get("per_type_decode_64k")
    if t:
        out["decode_64k_frac"] = {k: round(v["GB_per_s"] / peak, 4) for k, v in t.items()}
        out["decode_64k_us"] = {k: v["decode_us"] for k, v in t.items()}
    f = result.get("formats_16k")
    if f:
        out["decode_16k_frac"] = {k: round(v["GB_per_s"] / peak, 3) for k, v in f["per_format"].items()}
    p = result.get("page1_shape_240k")
    if p:
        out["page1_240k_64_layers"] = {k: {"ms": v["decode_64_layers_ms"], "frac": round(v["GB_per_s"] / peak, 4)}
                                       for k, v in p["per_type"].items()}
    c = result.get("prefill_chunk_64k")
    if c:
        out["chunk16_64k_us"] = c["us_per_chunk"]
    return out


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        print(json.dumps(run_reference(args, ws, rank)))
        return 0
    ws, rank, local = dist_init(args)
    import torch

    from bit_kv_cache_17_b200 import kvq, synth

    if args.part in ("append", "prefill"):
        r = (run_append if args.part == "append" else run_prefill)(args, kvq, torch, synth)
        if rank == 0:
            print(json.dumps(r))
        return 0
    result, cfg, cache = run_ours(args, ws, rank)
    del cache
    torch.cuda.empty_cache()
    if not args.quick:
        result["per_type_decode_64k"] = run_type_sweep(args, kvq, torch, synth, cfg)
        torch.cuda.empty_cache()
        result["append"] = run_append(args, kvq, torch, synth)
        torch.cuda.empty_cache()
        result["formats_16k"] = run_formats(args, kvq, torch, synth)
        torch.cuda.empty_cache()
        result["page1_shape_240k"] = run_page1_shape(args, kvq, torch, synth)
        torch.cuda.empty_cache()
        result["prefill_chunk_64k"] = run_prefill(args, kvq, torch, synth)
        torch.cuda.empty_cache()
        result["quality"] = compact(run_quality(args, kvq, torch, synth))
        result["roofline"]["others"] = summary(result)
    if rank == 0 and ws == 1:
        result["cpu_baseline"] = cpu_baseline(cfg, args.type)
    elif rank == 0:
        result["cpu_baseline"] = None
    if "quality" in result:  # the long side report goes last on the line
        result["quality"] = result.pop("quality")
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))
    return 0


if __name__ == "__main__":
    sys.exit(main())
