#!/usr/bin/env python
"""Benchmark of the TurboQuant decode hot path on B200.

A step is one decode step of the long-context workload (B=4, Hq=16/Hkv=8,
d=128, 102400 compressed tokens per sequence) through the library's C ABI,
tq_append_attend: encode one new K and one new V vector per (batch, kv head)
into the cache and attend over the whole compressed cache (query prologue,
split-K attention, combine), the five kernels chained on one stream.  The headline
metric is the achieved bandwidth on the compressed-cache bytes the step must
read (118 B per token per kv head); the encode-only workload (B=1, 8 kv heads,
32768 bf16 tokens) gives the KV encode throughput in Mvectors/s.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica on its own GPU (the workload shards by sequence with no exchange), and
rank 0 prints one JSON line with the whole-job numbers (max time over ranks).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_vector_14_b200 import synthetic  # noqa: E402

METRIC = "decode-attn achieved HBM GB/s (% of B200 peak); KV encode Mvectors/s"
UNIT = "GB/s"
BYTES_PER_TOKEN_HEAD = {64: 36 + 26, 128: 68 + 50, 256: 132 + 98}   # packed K + V record per token per kv head
ENCODE_BYTES_PER_VECTOR = {("k", 128): 68, ("v", 128): 50}

# DRAM traffic of the split-K kernel (read + write bytes per launch) from one
# ncu capture, valid only while the kernel sources are unchanged (sha256 over
# DECODE_SOURCES at capture time).
NCU_TRAFFIC = {"source_sha256": "b92fbfb91599ce7faae1a3c9cf92f313b8878332d27044e65647f74a8e4377fc",
               "bytes_per_launch": 387270144 + 3134208,
               "capture": "profiles/tq_decode_mma_d128_long_context_b4_hq16_hkv8_t102400.md"}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def bf16_peak_tflops() -> float:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


DECODE_SOURCES = ("kv_cache_vector_14_b200/csrc/tq_decode_mma.cu", "kv_cache_vector_14_b200/csrc/tq_frag.cuh",
                  "kv_cache_vector_14_b200/csrc/tq_internal.h")


def source_sha(rels) -> str:
    h = hashlib.sha256()
    for rel in rels:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.proc = None
        self.out = None
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
            if uuid:
                cmd += ["-i", uuid]
            self.out = open(os.devnull if not os.path.isdir("/tmp") else f"/tmp/tq_clocks_{os.getpid()}.csv", "w+")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.count(",") >= 8]
        self.out.close()
        try:
            os.unlink(self.out.name)
        except Exception:
            pass
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" == r[5 + i].strip()})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- multi-rank plumbing

def max_over_ranks(x: float, dist, device) -> float:
    """Largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, seconds_local: float, world: int, dist, device) -> float:
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return world * units_per_rank / max_over_ranks(seconds_local, dist, device)


# ----------------------------------------------------------------------------- CPU oracle (baseline)

def host_cpu() -> dict:
    """Model name and logical CPU count of the host the oracle runs on."""
    name = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    name = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": name, "nproc": os.cpu_count()}


def oracle_decode_rate(w, seconds: float, tokens: int | None = None, threads: int = 0):
    """Time the float64 oracle's decode attention on host cores over a bounded
    sample: the G query heads of kv head 0 of sequence 0, over its first
    `tokens` compressed tokens (the oracle encodes them itself), on `threads`
    threads (0: every core; the oracle splits the scores over tokens and the
    value sum over coordinates).  Returns (GB/s on the algorithmic bytes,
    threads, sample text, seconds of work)."""
    import oracle as O
    tokens = tokens or w.T
    O.set_threads(0)
    prm = O.params(w.d, 0)
    xk = synthetic.kv(w, "k", 0, tokens, batches=[0])[0, 0].astype(np.float64)
    xv = synthetic.kv(w, "v", 0, tokens, batches=[0])[0, 0].astype(np.float64)
    ek, ev = O.encode(xk, prm, True), O.encode(xv, prm, False)
    kc = {"idx": ek["idx"], "sig": ek["sig"], "nh": ek["nh"], "gh": ek["gh"]}
    vc = {"idx": ev["idx"], "nh": ev["nh"]}
    G = w.Hq // w.Hkv
    q = synthetic.queries(w)[0, :G].astype(np.float64)
    O.set_threads(threads)
    used = O.num_threads()
    t0 = time.perf_counter()
    n = 0
    while True:
        O.attend(prm, q, kc, vc, w.scale)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    O.set_threads(0)
    nbytes = n * tokens * BYTES_PER_TOKEN_HEAD[w.d]
    sample = (f"oracle attention of {G} query heads over {tokens} tokens of one kv head "
              f"(float64, {n} repetitions, {el:.1f} s)")
    return nbytes / el / 1e9, used, sample, el


def oracle_encode_rate(w, seconds: float, threads: int = 0):
    """The oracle's encode (K and V of 4096 tokens x 8 kv heads of the encode-only
    workload, repeated) on `threads` host threads (0: every core)."""
    import oracle as O
    prm = O.params(w.d, 0)
    x = synthetic.kv(w, "k", 0, 4096, batches=[0])[0].reshape(-1, w.d).astype(np.float64)
    O.set_threads(threads)
    used = O.num_threads()
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < seconds:
        O.encode(x, prm, True)
        O.encode(x, prm, False)
        n += 2 * x.shape[0]
    el = time.perf_counter() - t0
    O.set_threads(0)
    return n / el / 1e6, used, f"oracle encode of {x.shape[0]} K and V vectors, repeated ({el:.1f} s)"


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    w = synthetic.WORKLOADS["c4"]
    budget = 120.0 / max(args.steps + args.warmup, 1)       # seconds per step
    # calibrate tokens per step so the whole run stays within a few minutes
    probe = 2048
    rate, _, _, _ = oracle_decode_rate(w, 0.5, probe)
    tok = int(max(256, min(w.T, rate * 1e9 * budget * 0.8 / BYTES_PER_TOKEN_HEAD[w.d])))
    tok = tok // 64 * 64
    import oracle as O
    prm = O.params(w.d, 0)
    xk = synthetic.kv(w, "k", 0, tok, batches=[0])[0, 0].astype(np.float64)
    xv = synthetic.kv(w, "v", 0, tok, batches=[0])[0, 0].astype(np.float64)
    ek, ev = O.encode(xk, prm, True), O.encode(xv, prm, False)
    kc = {"idx": ek["idx"], "sig": ek["sig"], "nh": ek["nh"], "gh": ek["gh"]}
    vc = {"idx": ev["idx"], "nh": ev["nh"]}
    G = w.Hq // w.Hkv
    q = synthetic.queries(w)[0, :G].astype(np.float64)
    for _ in range(args.warmup):
        O.attend(prm, q, kc, vc, w.scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.attend(prm, q, kc, vc, w.scale)
    el = time.perf_counter() - t0
    value = args.steps * tok * BYTES_PER_TOKEN_HEAD[w.d] / el / 1e9
    threads = O.num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.title, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.d, "T": w.T,
                   "l2": "n/a (host)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", **host_cpu(),
                         "sample": f"per step: oracle attention of {G} query heads over {tok} tokens of one kv head"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm

def measure_encode(h, dev, world: int, dist, passes: int = 30) -> dict:
    """Encode-only workload (B=1, 8 kv heads, 32768 bf16 tokens): K and V of
    every token per pass, L2 flushed between passes.  Returns the fields of the
    'encode' object."""
    import torch
    from kv_cache_vector_14_b200 import tq
    we = synthetic.WORKLOADS["c2"]
    xk = torch.from_numpy(synthetic.kv(we, "k")).to(dev).to(torch.bfloat16)
    xv = torch.from_numpy(synthetic.kv(we, "v")).to(dev).to(torch.bfloat16)
    ekc = tq.Cache(we.d, True, we.B, we.Hkv, we.T)
    evc = tq.Cache(we.d, False, we.B, we.Hkv, we.T)
    for _ in range(3):
        tq.tq_encode_k(h, xk, ekc, 0)
        tq.tq_encode_v(h, xv, evc, 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)      # 2x L2: evict between passes
    enc_ms, k_ms = [], []
    # A pass is the two calls back to back, as a caller issues them (no event between them:
    # the V encode's set-up may overlap the end of the K encode); the K encode alone is
    # timed in passes of its own.
    for _ in range(passes):
        flush.zero_()
        a, b = (torch.cuda.Event(enable_timing=True) for _ in range(2))
        a.record()
        tq.tq_encode_k(h, xk, ekc, 0)
        tq.tq_encode_v(h, xv, evc, 0)
        b.record()
        torch.cuda.synchronize()
        enc_ms.append(a.elapsed_time(b))
    for _ in range(passes):
        flush.zero_()
        a, b = (torch.cuda.Event(enable_timing=True) for _ in range(2))
        a.record()
        tq.tq_encode_k(h, xk, ekc, 0)
        b.record()
        torch.cuda.synchronize()
        k_ms.append(a.elapsed_time(b))
    enc_med = statistics.median(enc_ms)
    nvec = 2 * we.B * we.Hkv * we.T
    enc_bytes = we.B * we.Hkv * we.T * (2 * we.d * 2 + ENCODE_BYTES_PER_VECTOR[("k", 128)] +
                                        ENCODE_BYTES_PER_VECTOR[("v", 128)])
    enc_mvps = whole_job_rate(nvec, enc_med * 1e-3, world, dist, dev) / 1e6
    return {"workload": we.title, "value": enc_mvps, "unit": "Mvectors/s", "ms_per_pass": enc_med,
            "k_ms": statistics.median(k_ms), "vectors_per_pass": nvec, "algorithmic_bytes_per_pass": enc_bytes,
            "achieved_gbs": enc_bytes / (enc_med * 1e-3) / 1e9,
            "l2": "256 MB buffer written between passes"}


def measure_loop(dev, world: int, dist, replays: int = 5) -> dict:
    """Append-and-attend workload (B=16, Hq=32/Hkv=8, d=256, cache from 8192
    tokens, 256 steps of tq_append_attend: encode the step's K and V per
    (batch, kv head) at position T, attend over T+1 tokens).  The 256-step
    sequence is captured once in a CUDA graph and replayed; each replay
    rewrites the same cache positions with the same values, so every replay
    does the full work.  The ~250 MB cache exceeds L2.  Also timed eagerly, and
    as a graph of the same steps made of three separate calls each."""
    import torch
    from kv_cache_vector_14_b200 import tq
    w = synthetic.WORKLOADS["c5"]
    d, B, Hq, Hkv, T0, S = w.d, w.B, w.Hq, w.Hkv, w.T, w.steps
    Tend = T0 + S
    Tcap = (Tend + 63) // 64 * 64
    h = tq.tq_init(d, 0)
    kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    news = []
    for which, cache in (("k", kc), ("v", vc)):
        x = torch.from_numpy(synthetic.kv(w, which)).to(dev)
        (tq.tq_encode_k if which == "k" else tq.tq_encode_v)(h, x[:, :, :T0], cache, 0)
        news.append(x[:, :, T0:].clone())
        del x
    kn, vn = news
    q = torch.from_numpy(synthetic.queries_all(w)).to(dev)
    q = q.to(torch.bfloat16) if w.q_dtype == "bf16" else q
    out = torch.empty((S, B, Hq, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, Tend), dtype=torch.uint8, device=dev)

    def sequence(fused=True):
        for s in range(S):
            T = T0 + s
            if fused:
                tq.tq_append_attend(h, kn[:, :, s:s + 1], vn[:, :, s:s + 1], kc, vc, T, q[s], out[s], ws,
                                    scale=w.scale)
                continue
            tq.tq_encode_k(h, kn[:, :, s:s + 1], kc, T)
            tq.tq_encode_v(h, vn[:, :, s:s + 1], vc, T)
            tq.tq_attend_decode(h, q[s], kc, vc, out[s], ws, T=T + 1, scale=w.scale)

    sequence()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    sequence()
    e1.record()
    torch.cuda.synchronize()
    eager_ms = e0.elapsed_time(e1)
    ref = out.clone()
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        sequence()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        sequence()
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    same = bool(torch.equal(out, ref))
    times = []
    for _ in range(replays):
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    graph_ms = statistics.median(times)
    graph_ms_max = max_over_ranks(graph_ms, dist, dev)
    del graph
    graph = torch.cuda.CUDAGraph()              # the same steps as three separate calls each
    with torch.cuda.graph(graph):
        sequence(fused=False)
    graph.replay()
    torch.cuda.synchronize()
    same_sep = bool(torch.equal(out, ref))
    times = []
    for _ in range(replays):
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    graph_sep_ms = statistics.median(times)
    path = tq.tq_attend_path(h, Hq, Hkv)
    status = tq.tq_status_string(tq.tq_device_status(h))
    del graph
    tq.tq_destroy(h)
    nbytes = sum(B * Hkv * (T0 + s + 1) * BYTES_PER_TOKEN_HEAD[d] for s in range(S))
    return {"workload": w.title, "steps": S, "decode_path": path,
            "graph_ms_total": graph_ms, "graph_us_per_step": graph_ms * 1e3 / S,
            "eager_ms_total": eager_ms, "eager_us_per_step": eager_ms * 1e3 / S,
            "graph_us_per_step_separate_calls": graph_sep_ms * 1e3 / S,
            "separate_calls_output_equal": same_sep,
            "achieved_gbs": whole_job_rate(nbytes, graph_ms * 1e-3, world, dist, dev) / 1e9,
            "decode_tokens_per_s": world * S * B / (graph_ms_max * 1e-3),
            "kernels_per_step": 5, "graph_output_equals_eager": same,
            "l2": "cache (~250 MB) larger than L2; no flush between replays", "device_status": status}


def exact_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Softmax attention in float64 over unquantised keys and values (ground
    truth for the quality comparison, not the method): q [G, d], k, v [T, d]."""
    s = (q.astype(np.float64) @ k.astype(np.float64).T) * scale
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p / p.sum(axis=1, keepdims=True)) @ v.astype(np.float64)


def measure_polar(h, dev, w, vc, q, out_qjl, ws, n_calls: int) -> dict:
    """PolarQuant-only K on the long-context workload: the K vectors encoded
    without the QJL bit (codes and norm, 50 B per token at d=128), attention timed
    on its own (split-K kernel by events, and the whole call), and the output
    error of both K flows against exact attention over the unquantised data
    for one sequence and kv head."""
    import torch
    from kv_cache_vector_14_b200 import tq
    d, B, Hq, Hkv, T = w.d, w.B, w.Hq, w.Hkv, w.T
    kp = tq.Cache(d, False, B, Hkv, T)
    x = torch.from_numpy(synthetic.kv(w, "k")).to(dev)
    tq.tq_encode_v(h, x, kp, 0)
    del x
    out = torch.empty_like(out_qjl)
    for _ in range(5):
        tq.tq_attend_decode_polar(h, q, kp, vc, out, ws, T=T, scale=w.scale)
    torch.cuda.synchronize()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_calls)]
    for a_, b_ in kev:
        a_.record()
        b_.record()
    torch.cuda.synchronize()
    for i in range(n_calls):
        tq.tq_set_decode_events(h, kev[i][0], kev[i][1])
        tq.tq_attend_decode_polar(h, q, kp, vc, out, ws, T=T, scale=w.scale)
    torch.cuda.synchronize()
    tq.tq_set_decode_events(h, None, None)
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_calls):
        tq.tq_attend_decode_polar(h, q, kp, vc, out, ws, T=T, scale=w.scale)
    e1.record()
    torch.cuda.synchronize()
    call_ms = e0.elapsed_time(e1) / n_calls
    G = Hq // Hkv
    kx = synthetic.kv(w, "k", batches=[0])[0, 0]
    vx = synthetic.kv(w, "v", batches=[0])[0, 0]
    qx = q[0, :G].float().cpu().numpy()
    ref = exact_attention(qx, kx, vx, w.scale)

    def rel(o):        # mean over the query heads of ||o - ref||_2 / ||ref||_2
        return float((np.linalg.norm(o - ref, axis=1) / np.linalg.norm(ref, axis=1)).mean())

    nbytes = B * Hkv * T * 100          # 50 B K + 50 B V per token per kv head at d=128
    del kp
    return {"workload": w.title + ", K without the QJL bit (3.125 b/dim)", "bytes_per_token_head": 100,
            "kernel_ms": kern_ms, "call_ms": call_ms, "achieved_gbs": nbytes / (kern_ms * 1e-3) / 1e9,
            "quality_vs_exact_attention": {
                "sample": f"batch 0, kv head 0: {G} query heads over {T} tokens, float64 softmax attention "
                          "over the unquantised K and V",
                "metric": "mean over query heads of relative L2 error of the attention output",
                "qjl_k": rel(out_qjl[0, :G].cpu().numpy().astype(np.float64)),
                "polar_k": rel(out[0, :G].cpu().numpy().astype(np.float64))}}


def measure_paged(h, dev, w, kc, vc, q, out_ref, ws, n_calls: int) -> dict:
    """Paged caches on the long-context workload: the same K and V blocks
    scattered over two pools by a random permutation (block tables
    [B*Hkv][T/64]), attention timed on its own (split-K kernel by events)
    and its output compared with the contiguous caches' bit for bit."""
    import torch
    from kv_cache_vector_14_b200 import tq
    d, B, Hq, Hkv, T = w.d, w.B, w.Hq, w.Hkv, w.T
    nblk = B * Hkv * (T // 64)
    gen = torch.Generator().manual_seed(1234)
    caches = []
    for src, is_k in ((kc, True), (vc, False)):
        perm = torch.randperm(nblk, generator=gen).to(torch.int32)
        table = perm.view(B * Hkv, T // 64).to(dev)
        pc = tq.Cache(d, is_k, B, Hkv, T, block_table=table, pool_blocks=nblk)
        bb = tq.tq_block_bytes(d, is_k)
        pc.buf[:nblk * bb].view(nblk, bb).index_copy_(0, perm.to(dev).long(), src.buf[:nblk * bb].view(nblk, bb))
        caches.append(pc)
    kp, vp = caches
    out = torch.empty_like(out_ref)
    for _ in range(5):
        tq.tq_attend_decode(h, q, kp, vp, out, ws, T=T, scale=w.scale)
    torch.cuda.synchronize()
    same = bool(torch.equal(out, out_ref))
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_calls)]
    for a_, b_ in kev:
        a_.record()
        b_.record()
    torch.cuda.synchronize()
    for i in range(n_calls):
        tq.tq_set_decode_events(h, kev[i][0], kev[i][1])
        tq.tq_attend_decode(h, q, kp, vp, out, ws, T=T, scale=w.scale)
    torch.cuda.synchronize()
    tq.tq_set_decode_events(h, None, None)
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    del kp, vp, caches
    nbytes = B * Hkv * T * BYTES_PER_TOKEN_HEAD[d]
    return {"workload": w.title + ", K and V blocks scattered over pools by random block tables",
            "kernel_ms": kern_ms, "achieved_gbs": nbytes / (kern_ms * 1e-3) / 1e9,
            "output_equals_contiguous": same}


def measure_d64(dev, world: int, dist, n_calls: int = 200) -> dict:
    """head_dim 64 on the long-context shape (B=4, Hq=16/Hkv=8, T=102400,
    bf16 K/V with outlier channels and log-normal norms): the bulk encode of
    the whole cache (K then V, timed by events) and decode attention over it
    (split-K kernel by events, and the whole call).  62 bytes of packed cache
    per (token, kv head)."""
    import torch
    from kv_cache_vector_14_b200 import tq
    base = synthetic.WORKLOADS["c4"]
    w = synthetic.Workload("d64", "head_dim 64, long context: B=4, Hq=16/Hkv=8, T=102400",
                           B=base.B, Hq=base.Hq, Hkv=base.Hkv, d=64, T=base.T, kv_dtype="bf16", q_dtype="bf16",
                           lognormal_norms=True, seed=640, scale=0.125)
    d, B, Hq, Hkv, T = w.d, w.B, w.Hq, w.Hkv, w.T
    h = tq.tq_init(d, 0)
    kc, vc = tq.Cache(d, True, B, Hkv, T), tq.Cache(d, False, B, Hkv, T)
    xk = torch.from_numpy(synthetic.kv(w, "k")).to(dev).to(torch.bfloat16)
    xv = torch.from_numpy(synthetic.kv(w, "v")).to(dev).to(torch.bfloat16)
    ek = []
    for i in range(8):
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        tq.tq_encode_k(h, xk, kc, 0)
        e1.record()
        tq.tq_encode_v(h, xv, vc, 0)
        e2.record()
        torch.cuda.synchronize()
        if i >= 3:
            ek.append((e0.elapsed_time(e1), e1.elapsed_time(e2)))
    k_ms = statistics.median(a for a, _ in ek)
    v_ms = statistics.median(b for _, b in ek)
    del xk, xv
    q = torch.from_numpy(synthetic.queries(w)).to(dev).to(torch.bfloat16)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, T), dtype=torch.uint8, device=dev)
    for _ in range(10):
        tq.tq_attend_decode(h, q, kc, vc, out, ws, T=T, scale=w.scale)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_calls)]
    for a_, b_ in kev:
        a_.record()
        b_.record()
    torch.cuda.synchronize()
    for i in range(n_calls):
        tq.tq_set_decode_events(h, kev[i][0], kev[i][1])
        tq.tq_attend_decode(h, q, kc, vc, out, ws, T=T, scale=w.scale)
    torch.cuda.synchronize()
    tq.tq_set_decode_events(h, None, None)
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record()
    for _ in range(n_calls):
        tq.tq_attend_decode(h, q, kc, vc, out, ws, T=T, scale=w.scale)
    c1.record()
    torch.cuda.synchronize()
    call_ms = c0.elapsed_time(c1) / n_calls
    status = tq.tq_status_string(tq.tq_device_status(h))
    path = tq.tq_attend_path(h, Hq, Hkv)
    tq.tq_destroy(h)
    nbytes = B * Hkv * T * BYTES_PER_TOKEN_HEAD[d]
    nvec = B * Hkv * T
    return {"workload": w.title + ", bf16 K/V with outlier channels and log-normal norms",
            "decode_path": path, "kernel_ms": kern_ms, "call_ms": call_ms,
            "achieved_gbs": world * nbytes / (max_over_ranks(kern_ms, dist, dev) * 1e-3) / 1e9,
            "call_gbs": world * nbytes / (max_over_ranks(call_ms, dist, dev) * 1e-3) / 1e9,
            "encode_k_ms": k_ms, "encode_v_ms": v_ms,
            "encode_mvec_s": world * 2 * nvec / (max_over_ranks(k_ms + v_ms, dist, dev) * 1e-3) / 1e6,
            "device_status": status}


def measure_gqa(dev, world: int, dist, n_calls: int = 300, copies: int = 7) -> dict:
    """Decode attention on the GQA workload (B=1, Hq=32/Hkv=8, d=128, 40960
    tokens; bf16 K/V with outlier channels and log-normal norms, bf16 query,
    scale 1/sqrt(128)).  Its compressed cache (38.7 MB) fits in the 126 MB L2,
    so the headline figure rotates over `copies` identical caches (7 x 38.7 MB
    = 271 MB, more than twice the L2): each call reads a cache last touched six
    calls earlier.  The same calls on one cache give the L2-warm figure,
    reported separately.  The split-K kernel is timed by events the library
    records around it, the whole call (prologue, kernel, combine) by events
    around the calls."""
    import torch
    from kv_cache_vector_14_b200 import tq
    w = synthetic.WORKLOADS["c3"]
    d, B, Hq, Hkv, T = w.d, w.B, w.Hq, w.Hkv, w.T
    h = tq.tq_init(d, 0)
    kc, vc = tq.Cache(d, True, B, Hkv, T), tq.Cache(d, False, B, Hkv, T)
    for which, cache in (("k", kc), ("v", vc)):
        x = torch.from_numpy(synthetic.kv(w, which)).to(dev).to(torch.bfloat16)
        (tq.tq_encode_k if which == "k" else tq.tq_encode_v)(h, x, cache, 0)
        del x
    caches = [(kc, vc)]
    for _ in range(copies - 1):
        k2, v2 = tq.Cache(d, True, B, Hkv, T), tq.Cache(d, False, B, Hkv, T)
        k2.buf.copy_(kc.buf)
        v2.buf.copy_(vc.buf)
        caches.append((k2, v2))
    q = torch.from_numpy(synthetic.queries(w)).to(dev).to(torch.bfloat16)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, T), dtype=torch.uint8, device=dev)

    def timed(rotate: bool):
        for i in range(2 * copies):
            k_, v_ = caches[i % copies] if rotate else caches[0]
            tq.tq_attend_decode(h, q, k_, v_, out, ws, T=T, scale=w.scale)
        kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_calls)]
        for a_, b_ in kev:
            a_.record()
            b_.record()
        torch.cuda.synchronize()
        for i in range(n_calls):
            k_, v_ = caches[i % copies] if rotate else caches[0]
            tq.tq_set_decode_events(h, kev[i][0], kev[i][1])
            tq.tq_attend_decode(h, q, k_, v_, out, ws, T=T, scale=w.scale)
        torch.cuda.synchronize()
        tq.tq_set_decode_events(h, None, None)
        kern = statistics.mean(a.elapsed_time(b) for a, b in kev)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record()
        for i in range(n_calls):
            k_, v_ = caches[i % copies] if rotate else caches[0]
            tq.tq_attend_decode(h, q, k_, v_, out, ws, T=T, scale=w.scale)
        c1.record()
        torch.cuda.synchronize()
        return kern, c0.elapsed_time(c1) / n_calls

    kern_ms, call_ms = timed(True)
    warm_kern_ms, warm_call_ms = timed(False)
    status = tq.tq_status_string(tq.tq_device_status(h))
    path = tq.tq_attend_path(h, Hq, Hkv)
    tq.tq_destroy(h)
    nbytes = B * Hkv * T * BYTES_PER_TOKEN_HEAD[d]
    gbs = lambda ms: world * nbytes / (max_over_ranks(ms, dist, dev) * 1e-3) / 1e9
    return {"workload": w.title, "decode_path": path, "algorithmic_bytes_per_call": nbytes,
            "l2": f"{copies} identical caches rotated ({copies * nbytes / 1e6:.0f} MB > 2x L2)",
            "kernel_ms": kern_ms, "call_ms": call_ms, "achieved_gbs": gbs(kern_ms), "call_gbs": gbs(call_ms),
            "l2_warm": {"kernel_ms": warm_kern_ms, "call_ms": warm_call_ms, "achieved_gbs": gbs(warm_kern_ms),
                        "call_gbs": gbs(warm_call_ms)},
            "device_status": status}


def measure_single_head(dev, world: int, dist, n_calls: int = 2000) -> dict:
    """The single-head workload (d=128, 1024 fp32 K/V vectors with outlier
    channels, one fp32 query): microseconds per call of tq_encode_k and
    tq_encode_v over the 1024 vectors and of one tq_attend_decode over them,
    each timed alone over n_calls back-to-back calls.  Latency-bound: the data
    (1.17 MB in, 120.8 KB packed) stays in L2."""
    import torch
    from kv_cache_vector_14_b200 import tq
    w = synthetic.WORKLOADS["c1"]
    d, T = w.d, w.T
    h = tq.tq_init(d, 0)
    kc, vc = tq.Cache(d, True, w.B, w.Hkv, T), tq.Cache(d, False, w.B, w.Hkv, T)
    xk = torch.from_numpy(synthetic.kv(w, "k")).to(dev)
    xv = torch.from_numpy(synthetic.kv(w, "v")).to(dev)
    q = torch.from_numpy(synthetic.queries(w)).to(dev)
    out = torch.empty((w.B, w.Hq, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, w.B, w.Hq, w.Hkv, T), dtype=torch.uint8, device=dev)
    calls = {"encode_k": lambda: tq.tq_encode_k(h, xk, kc, 0), "encode_v": lambda: tq.tq_encode_v(h, xv, vc, 0),
             "attend": lambda: tq.tq_attend_decode(h, q, kc, vc, out, ws, T=T, scale=w.scale)}
    res = {}
    for name, fn in calls.items():
        for _ in range(20):
            fn()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record()
        for _ in range(n_calls):
            fn()
        c1.record()
        torch.cuda.synchronize()
        res[name + "_us"] = max_over_ranks(c0.elapsed_time(c1) / n_calls, dist, dev) * 1e3
    res["total_us"] = res["encode_k_us"] + res["encode_v_us"] + res["attend_us"]
    status = tq.tq_status_string(tq.tq_device_status(h))
    tq.tq_destroy(h)
    return {"workload": w.title, **res, "calls_timed": n_calls, "device_status": status}


def measure_prefill(dev, world: int, dist, reps: int = 20, Lq: int = 512, d: int = 128) -> dict:
    """Chunked prefill on the GQA workload's cache (B=1, Hq=32/Hkv=8, 40960
    tokens; head_dim d, 128 as in the workload or 64 with the same data
    recipe): the last Lq tokens' queries as one chunk, query i attending
    causally over tokens [0, T - Lq + i].  Timed per call (prologue, prefill
    kernel, combine).  Work: 3 contractions of d multiply-adds per (query row,
    visible token) pair: 6 d flops."""
    import dataclasses
    import torch
    from kv_cache_vector_14_b200 import tq
    w = synthetic.WORKLOADS["c3"]
    if d != w.d:
        w = dataclasses.replace(w, d=d, scale=1.0 / math.sqrt(d))
    B, Hq, Hkv, T = w.B, w.Hq, w.Hkv, w.T
    T0 = T - Lq
    h = tq.tq_init(d, 0)
    kc, vc = tq.Cache(d, True, B, Hkv, T), tq.Cache(d, False, B, Hkv, T)
    for which, cache in (("k", kc), ("v", vc)):
        x = torch.from_numpy(synthetic.kv(w, which)).to(dev).to(torch.bfloat16)
        (tq.tq_encode_k if which == "k" else tq.tq_encode_v)(h, x, cache, 0)
        del x
    q = torch.from_numpy(synthetic.gaussian((B, Lq, Hq, d), seed=11)).to(dev).to(torch.bfloat16)
    out = torch.empty((B, Lq, Hq, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_prefill_workspace_bytes(h, B, Lq, Hq), dtype=torch.uint8, device=dev)
    for _ in range(3):
        tq.tq_attend_prefill(h, q, kc, vc, T0, out, ws, scale=w.scale)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        tq.tq_attend_prefill(h, q, kc, vc, T0, out, ws, scale=w.scale)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    status = tq.tq_status_string(tq.tq_device_status(h))
    tq.tq_destroy(h)
    pairs = B * Hq * (Lq * T0 + Lq * (Lq + 1) // 2)
    flops = 6 * d * pairs
    return {"workload": f"chunked prefill: B=1, Hq=32/Hkv=8, d={d}, {Lq} queries after {T0} cached tokens",
            "ms_per_call": ms, "query_token_pairs": pairs, "algorithmic_flops": flops,
            "tflops": world * flops / (max_over_ranks(ms, dist, dev) * 1e-3) / 1e12,
            "device_status": status}


def run_ours(args, rank: int, world: int, dist):
    import torch
    from kv_cache_vector_14_b200 import build, tq

    build.build()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    w = synthetic.WORKLOADS["c4"]
    d, B, Hq, Hkv, T = w.d, w.B, w.Hq, w.Hkv, w.T
    h = tq.tq_init(d, 0)
    if args.only == "encode":          # profiling aid: the encode-only workload alone
        enc = measure_encode(h, dev, world, dist, passes=args.steps)
        tq.tq_destroy(h)
        if rank == 0:
            print(json.dumps({"encode": enc}), flush=True)
        return
    if args.only == "prefill":         # profiling aid: the chunked-prefill workload alone
        tq.tq_destroy(h)
        pf = measure_prefill(dev, world, dist, reps=args.steps)
        if rank == 0:
            print(json.dumps({"prefill": pf}), flush=True)
        return
    if args.only == "d64":             # profiling aid: the head_dim 64 workload alone
        tq.tq_destroy(h)
        r = measure_d64(dev, world, dist, n_calls=args.steps)
        r["prefill"] = measure_prefill(dev, world, dist, reps=5, d=64)
        r["prefill_d256"] = measure_prefill(dev, world, dist, reps=5, d=256)
        if rank == 0:
            print(json.dumps({"d64": r}), flush=True)
        return
    if args.only == "gqa":             # profiling aid: the GQA decode and the single-head latencies
        tq.tq_destroy(h)
        r = {"c3": measure_gqa(dev, world, dist, n_calls=args.steps), "c1": measure_single_head(dev, world, dist)}
        if rank == 0:
            print(json.dumps(r), flush=True)
        return
    if args.only == "loop":            # profiling aid: the append-and-attend workload alone
        tq.tq_destroy(h)
        loop = measure_loop(dev, world, dist, replays=args.steps)
        if rank == 0:
            print(json.dumps({"loop": loop}), flush=True)
        return
    kc, vc = tq.Cache(d, True, B, Hkv, T), tq.Cache(d, False, B, Hkv, T)
    for which, cache in (("k", kc), ("v", vc)):
        x = torch.from_numpy(synthetic.kv(w, which)).to(dev)
        (tq.tq_encode_k if which == "k" else tq.tq_encode_v)(h, x, cache, 0)
        torch.cuda.synchronize()
        if which == "k":
            k_new = x[:, :, T - 1:T].clone()
        else:
            v_new = x[:, :, T - 1:T].clone()
        del x
    q = torch.from_numpy(synthetic.queries(w)).to(dev).to(torch.bfloat16)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, T), dtype=torch.uint8, device=dev)
    path = tq.tq_attend_path(h, Hq, Hkv)

    def step(kn, vn, qq, o):
        tq.tq_append_attend(h, kn, vn, kc, vc, T - 1, qq, o, ws, scale=w.scale)

    def step_separate(kn, vn, qq, o):
        tq.tq_encode_k(h, kn, kc, T - 1)
        tq.tq_encode_v(h, vn, vc, T - 1)
        tq.tq_attend_decode(h, qq, kc, vc, o, ws, T=T, scale=w.scale)

    def barrier():
        if dist is not None:
            dist.barrier()


    for _ in range(args.warmup):
        step(k_new, v_new, q, out)
        step_separate(k_new, v_new, q, out)
    torch.cuda.synchronize()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    # ---- timed region (device-resident inputs): the fused step, nothing else on the stream
    sampler = ClockSampler(uuid) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        step(k_new, v_new, q, out)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = max_over_ranks(ms, dist, dev)
    bytes_step = B * Hkv * T * BYTES_PER_TOKEN_HEAD[d]
    value = whole_job_rate(bytes_step, ms * 1e-3, world, dist, dev) / 1e9

    # ---- the split-K kernel alone, timed by events the library records around
    # it (the events break the launch chain, so this is a separate pass)
    n_kern = max(1, min(args.steps, 500))
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_kern)]
    for a_, b_ in kev:           # torch creates the CUDA events on first record; the library re-records them
        a_.record()
        b_.record()
    torch.cuda.synchronize()
    for i in range(n_kern):
        tq.tq_set_decode_events(h, kev[i][0], kev[i][1])
        step(k_new, v_new, q, out)
    torch.cuda.synchronize()
    tq.tq_set_decode_events(h, None, None)
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)

    # ---- the same step as three separate calls (encode K, encode V, attend)
    e0.record()
    for i in range(n_kern):
        step_separate(k_new, v_new, q, out)
    e1.record()
    torch.cuda.synchronize()
    ms_separate = e0.elapsed_time(e1) / n_kern

    if args.only == "step":            # profiling aid: the timed decode steps alone
        tq.tq_destroy(h)
        if rank == 0:
            print(json.dumps({"ms_per_step": ms_max, "kernel_ms": kern_ms, "ms_per_step_separate_calls": ms_separate,
                              "decode_path": path}), flush=True)
        return

    # ---- end to end: pinned host inputs copied in, the output read back, every step.
    # The step's new K, V and query sit in one pinned host buffer and go to the
    # device in one copy (one transfer instead of three on the step's stream).
    parts = [k_new.contiguous(), v_new.contiguous(), q.contiguous()]
    offs, off = [], 0
    for t_ in parts:
        offs.append(off)
        off += (t_.numel() * t_.element_size() + 255) // 256 * 256
    hbuf = torch.empty(off, dtype=torch.uint8).pin_memory()
    dbuf = torch.empty(off, dtype=torch.uint8, device=dev)
    views_h, views_d = [], []
    for t_, o_ in zip(parts, offs):
        nb = t_.numel() * t_.element_size()
        views_h.append(hbuf[o_:o_ + nb].view(t_.dtype).view(t_.shape))
        views_d.append(dbuf[o_:o_ + nb].view(t_.dtype).view(t_.shape))
    for vh_, t_ in zip(views_h, parts):
        vh_.copy_(t_.cpu())
    kh, vh, qh = views_h
    kd, vd, qd = views_d
    oh = torch.empty_like(out, device="cpu").pin_memory()
    n_e2e = max(1, min(args.steps, 2000))
    for _ in range(3):
        dbuf.copy_(hbuf, non_blocking=True)
        step(kd, vd, qd, out)
        oh.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record()
    for _ in range(n_e2e):
        dbuf.copy_(hbuf, non_blocking=True)
        step(kd, vd, qd, out)
        oh.copy_(out, non_blocking=True)
    e3.record()
    torch.cuda.synchronize()
    ms_e2e_local = e2.elapsed_time(e3) / n_e2e
    ms_e2e = max_over_ranks(ms_e2e_local, dist, dev)
    e2e_value = whole_job_rate(bytes_step, ms_e2e_local * 1e-3, world, dist, dev) / 1e9
    h2d = hbuf.numel()                  # the one packed copy (K and V fp32, q bf16, 256-byte aligned parts)
    d2h = oh.numel() * 4

    tq.tq_attend_decode(h, q, kc, vc, out, ws, T=T, scale=w.scale)     # QJL output for the quality check
    torch.cuda.synchronize()
    polar = measure_polar(h, dev, w, vc, q, out.clone(), ws, n_kern)
    paged = measure_paged(h, dev, w, kc, vc, q, out.clone(), ws, n_kern)
    enc = measure_encode(h, dev, world, dist)
    loop = measure_loop(dev, world, dist)
    gqa = measure_gqa(dev, world, dist)
    single = measure_single_head(dev, world, dist)
    prefill = measure_prefill(dev, world, dist)
    prefill64 = measure_prefill(dev, world, dist, d=64)
    prefill256 = measure_prefill(dev, world, dist, reps=10, d=256)
    d64 = measure_d64(dev, world, dist)

    peak, peak_kind = peaks()
    bf16_peak = bf16_peak_tflops()
    achieved = bytes_step / (kern_ms * 1e-3) / 1e9
    traffic = NCU_TRAFFIC["bytes_per_launch"] if (path == "mma" and
                                                  NCU_TRAFFIC["source_sha256"] == source_sha(DECODE_SOURCES)) else None

    cpu = None
    enc_cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        half = args.cpu_seconds / 2
        v, cores, sample, _ = oracle_decode_rate(w, half)
        v1, _, sample1, _ = oracle_decode_rate(w, half, threads=1)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample, **host_cpu(),
               "single_thread": {"value": v1, "unit": UNIT, "cores": 1, "sample": sample1}}
        ev_, ecores, esample = oracle_encode_rate(synthetic.WORKLOADS["c2"], min(5.0, half))
        ev1, _, esample1 = oracle_encode_rate(synthetic.WORKLOADS["c2"], min(5.0, half), threads=1)
        enc_cpu = {"value": ev_, "unit": "Mvectors/s", "cores": ecores, "kind": "oracle", "sample": esample,
                   "single_thread": {"value": ev1, "unit": "Mvectors/s", "cores": 1, "sample": esample1}}

    status = tq.tq_device_status(h)
    tq.tq_destroy(h)
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.title, "B": B, "Hq": Hq, "Hkv": Hkv, "head_dim": d, "T": T,
                   "step": "tq_append_attend: encode 1 K + 1 V per (batch, kv head) at position T-1, then "
                           "attention over the T-token compressed cache",
                   "ms_per_step_separate_calls": ms_separate,
                   "algorithmic_bytes_per_step": bytes_step, "decode_path": path,
                   "l2": "inputs larger than L2 (386.7 MB compressed cache read per step vs 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "kernel": f"tq_decode ({path})",
                     "kernel_ms": kern_ms, "peak_kind": f"{peak_kind} (copy bandwidth, burst)",
                     "frac_of_8000": achieved / 8000.0},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": ms_e2e},
        "gpu_launches": 5 * args.steps,
        "clocks": clocks,
        "encode": {**enc, "frac": enc["achieved_gbs"] / peak, "cpu_baseline": enc_cpu},
        "loop": {**loop, "frac": loop["achieved_gbs"] / peak},
        "c3": {**gqa, "frac": gqa["achieved_gbs"] / peak, "frac_of_8000": gqa["achieved_gbs"] / 8000.0,
               "call_frac": gqa["call_gbs"] / peak},
        "c1": single,
        "polar_k": {**polar, "frac": polar["achieved_gbs"] / peak},
        "paged": {**paged, "frac": paged["achieved_gbs"] / peak},
        "prefill": {**prefill, "peak_tflops": bf16_peak, "frac": prefill["tflops"] / bf16_peak,
                    "peak_kind": "measured bf16 dense GEMM (burst); the kernel uses mma.sync fp16/int8"},
        "d64": {**d64, "frac": d64["achieved_gbs"] / peak,
                "prefill": {**prefill64, "frac": prefill64["tflops"] / bf16_peak}},
        "prefill_d256": {**prefill256, "frac": prefill256["tflops"] / bf16_peak},
        "device_status": tq.tq_status_string(status),
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["step", "encode", "loop", "prefill", "d64", "gqa"], default=None,
                    help="run only the decode step (--steps steps), the encode-only workload (--steps "
                         "passes), the append-and-attend workload (--steps graph replays), the chunked "
                         "prefill (--steps calls) or the head_dim 64 workload (--steps decode calls); for "
                         "profiling")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    try:
        run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
