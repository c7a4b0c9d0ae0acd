#!/usr/bin/env python
"""Benchmark of compressed-KV decode attention on B200.

Metric: KV tokens*heads per second of tq_decode_attention on the
Llama-3-8B-shaped 32K-context decode (batch 16, 32 q / 8 kv heads,
head_dim 128, 1024 hot fp16 tokens + 31744 cold tokens at 3-bit keys /
4-bit values), with achieved HBM GB/s of the split-K attention kernel
against the measured copy bandwidth.  A step is one decode call over the
whole cache: query prep, split-K attention over hot and cold tokens,
cross-split combine.  The cold pages are written by tq_compress_append from
seeded synthetic K, V (N(0,1), 8 outlier channels x8 per kv head).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]

N > 1 runs under torchrun, one rank per GPU; every rank decodes its own
batch (weak scaling, no data-path collective); the time is the maximum
over ranks.  --impl reference times the CPU oracle on a bounded sample of
the same workload.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "llama3_8b_32k"
METRIC = "compressed-KV decode attention: KV tokens·heads/s and achieved HBM GB/s vs peak"
UNIT = "KV tokens*heads/s"
COLD_RECORD_BYTES = 118   # per cold token per kv head (d=128): 52 B key + 66 B value
HOT_RECORD_BYTES = 512    # per hot token per kv head: fp16 K and V


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per GPU (default: the workload's 16); smaller values only "
                         "size profiler captures and are not the benchmark line")
    ap.add_argument("--only", default=None,
                    choices=["gated", "monarch", "promotion", "tensor_cache", "stage1", "self_index",
                             "compress", "search"],
                    help="run one extra row alone and print it (sized for profiler captures; "
                         "not the benchmark line)")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def source_sha(source):
    """Hash of a CUDA source's code: comments and whitespace removed, so a
    comment edit keeps a capture valid and any code change voids it."""
    import re
    with open(os.path.join(ROOT, source)) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()[:16]


def kernel_traffic(kernel, source):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current code of the kernel's source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    return rec["bytes_per_launch"] if rec.get("src_sha") == source_sha(source) else None


class ClockSampler:
    """SM clock and throttle reasons read through NVML while the timed region runs."""

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nv is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv is not None:
            self._stop.set()
            self.t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# workload on the device
# ---------------------------------------------------------------------------
def build_state(torch, tq, W, rank, batch=None, workload=WORKLOAD, extra_pages=0):
    cfg = W.DECODE[workload]
    B, Hq, Hkv, d = batch or cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["d"]
    cold, hot = cfg["cold"], cfg["hot"]
    dev = torch.device("cuda")
    ctx = tq.Context(d, seed=0)
    max_pages = (cold + 127) // 128 + extra_pages
    n_pages = B * Hkv * max_pages
    page_bytes = ctx.page_bytes(True)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    pool = torch.empty((n_pages, page_bytes), dtype=torch.uint8, device=dev)
    table = torch.randperm(n_pages, generator=gen, device=dev).to(torch.int32).view(B, Hkv, max_pages)
    cold_len = torch.zeros(B, dtype=torch.int32, device=dev)
    chans = torch.stack([torch.randperm(d, generator=gen, device=dev)[:cfg["n_out"]] for _ in range(Hkv)])
    scale = torch.ones(Hkv, d, device=dev)
    scale.scatter_(1, chans, cfg["factor"])

    def kv(n):
        x = torch.randn((B, Hkv, n, d), generator=gen, device=dev) * scale[None, :, None, :]
        return x.to(torch.bfloat16)

    chunk = 2048
    for t0 in range(0, cold, chunk):
        n = min(chunk, cold - t0)
        tq.tq_compress_append(ctx.handle, kv(n), kv(n), pool, table, cold_len)
    torch.cuda.synchronize()
    ctx.check()
    k_hot = kv(hot).to(torch.float16)
    v_hot = kv(hot).to(torch.float16)
    hot_len = torch.full((B,), hot, dtype=torch.int32, device=dev)
    q = torch.randn((B, Hq, d), generator=gen, device=dev).to(getattr(torch, cfg["q_dtype"]))
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ws = ctx.workspace(B, Hq, Hkv, max_pages, hot)
    st = dict(ctx=ctx, pool=pool, table=table, cold_len=cold_len, k_hot=k_hot, v_hot=v_hot,
              hot_len=hot_len, q=q, out=out, ws=ws, B=B, Hq=Hq, Hkv=Hkv, d=d, cold=cold, hot=hot)
    return st


def measure_compress(torch, tq, reps=5, T=524288):
    """Compress/append throughput: 8 kv heads x 524288 bf16 vectors (d=128),
    x = N(0,1) * sigma[h, j], sigma ~ LogNormal(0,1), keys-only pages (T
    smaller only for profiler captures)."""
    dev = torch.device("cuda")
    H, d = 8, 128
    ctx = tq.Context(d, seed=0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(21)
    sigma = torch.exp(torch.randn((H, d), generator=gen, device=dev))
    x = (torch.randn((1, H, T, d), generator=gen, device=dev) * sigma[None, :, None, :]).to(torch.bfloat16)
    pages = H * T // 128
    pool = torch.empty((pages, ctx.page_bytes(False)), dtype=torch.uint8, device=dev)
    table = torch.arange(pages, dtype=torch.int32, device=dev).view(1, H, T // 128)
    cold = torch.zeros(1, dtype=torch.int32, device=dev)
    times = []
    for i in range(reps + 2):
        cold.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(), b.record()
        tq.tq_set_profile_events(ctx.handle, a, b)
        tq.tq_compress_append(ctx.handle, x, None, pool, table, cold)
        tq.tq_set_profile_events(ctx.handle, None, None)
        torch.cuda.synchronize()
        if i >= 2:
            times.append(a.elapsed_time(b))
    ctx.check()
    ms = statistics.median(times)
    n = H * T
    bytes_ = n * (2 * d + 52)
    flops = n * 2 * (d * d + d * d)
    return {"workload": "compress_4m (8 kv heads x %d bf16 vectors, d=128, keys-only)" % T,
            "vectors_per_s": n / (ms / 1e3), "kernel_ms": ms,
            "achieved_gbs": bytes_ / (ms / 1e3) / 1e9, "algorithmic_bytes": bytes_,
            "achieved_tflops": flops / (ms / 1e3) / 1e12, "algorithmic_flops": flops}


def measure_search(torch, tq, reps=3, N=1_000_000):
    """Compressed top-10 search: 10^6 database unit vectors (d=128, bf16
    input, keys-only pages) and 4096 unit queries (N smaller only for
    profiler captures)."""
    dev = torch.device("cuda")
    Q, d, k = 4096, 128, 10
    ctx = tq.Context(d, seed=0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(31)
    db = torch.randn((N, d), generator=gen, device=dev)
    db = (db / db.norm(dim=1, keepdim=True)).to(torch.bfloat16)
    pages = (N + 127) // 128
    pool = torch.zeros((pages, ctx.page_bytes(False)), dtype=torch.uint8, device=dev)
    table = torch.arange(pages, dtype=torch.int32, device=dev).view(1, 1, pages)
    cold = torch.zeros(1, dtype=torch.int32, device=dev)
    tq.tq_compress_append(ctx.handle, db.view(1, 1, N, d), None, pool, table, cold)
    qs = torch.randn((Q, d), generator=gen, device=dev)
    qs = qs / qs.norm(dim=1, keepdim=True)
    ids = torch.empty((Q, k), dtype=torch.int32, device=dev)
    sc = torch.empty((Q, k), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_topk_workspace_bytes(ctx.handle, Q, N, k), dtype=torch.uint8, device=dev)
    times = []
    for i in range(reps + 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(), b.record()
        tq.tq_set_profile_events(ctx.handle, a, b)
        tq.tq_score_topk(ctx.handle, qs, pool, N, k, ids, sc, ws)
        tq.tq_set_profile_events(ctx.handle, None, None)
        torch.cuda.synchronize()
        if i >= 1:
            times.append(a.elapsed_time(b))
    ctx.check()
    ms = statistics.median(times)
    flops = 2.0 * Q * N * (d + d)
    return {"workload": "search_1m (10^6 x 4096 queries, d=128, top-10)",
            "query_vectors_per_s": Q * N / (ms / 1e3), "kernel_ms": ms,
            "achieved_tflops": flops / (ms / 1e3) / 1e12, "algorithmic_flops": flops}


def graph_ms(torch, fn, reps=50):
    """Mean device time of fn (one step) replayed from a CUDA graph."""
    main = torch.cuda.current_stream()
    cap = torch.cuda.Stream()
    cap.wait_stream(main)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        fn()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=cap):
            fn()
    main.wait_stream(cap)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(main)
    for _ in range(reps):
        g.replay()
    b.record(main)
    b.synchronize()
    del g
    return a.elapsed_time(b) / reps


def gated_decode(tq, st, threshold, used):
    tq.tq_decode_attention_gated(st["ctx"].handle, st["q"], st["k_hot"], st["v_hot"],
                                 st["hot_len"], st["pool"], st["table"], st["cold_len"],
                                 threshold, st["out"], st["ws"], st["Hkv"], cold_used=used)


def measure_gated(torch, tq, st, reps=50):
    """Monarch's threshold gate on a decode state: step time with every head
    open, every head shut, and the threshold at the median of the per-head
    raw hot-score maxima (about half the heads read their cold tokens)."""
    G = st["Hq"] // st["Hkv"]
    qf = st["q"].float().view(st["B"], st["Hkv"], G, st["d"])
    hmax = torch.einsum("bhgd,bhtd->bhgt", qf, st["k_hot"].float()).amax(-1).reshape(st["B"], -1)
    used = torch.empty((st["B"], st["Hq"]), dtype=torch.int32, device=st["q"].device)
    res = {}
    for name, thr in (("open", float("inf")), ("median", float(hmax.median())),
                      ("shut", float("-inf"))):
        ms = graph_ms(torch, lambda: gated_decode(tq, st, thr, used), reps)
        u = used.view(st["B"], st["Hkv"], G)
        res[name] = {"ms_per_step": ms, "threshold": thr,
                     "heads_reading_cold": float(u.float().mean()),
                     "groups_reading_cold": float(u.any(-1).float().mean())}
    res["ungated_ms_per_step"] = graph_ms(torch, lambda: decode(tq, st), reps)
    st["ctx"].check()
    return res


def measure_monarch(torch, tq, W, workload, evict_block, thresholds=(float("inf"), float("-inf")),
                    steps=256, promotion=None):
    """Monarch decode steps (append, gated attention, eviction) on a decode
    workload: the hot ring holds W_max = the workload's hot length slots,
    window = W_max - E; the timed steps (replayed from a CUDA graph, one step
    per replay) include every eviction that falls due (one per E steps).
    promotion: None, or dict(threshold, sticky, max_per_step): the steps also
    count cold weights and move cold tokens back (tq_monarch_step_promote)."""
    # cold positions the steps can add: one token per step, plus every token
    # moved back (each can be evicted again into a new cold position)
    grow = (steps + 64) * (1 + (promotion["max_per_step"] if promotion else 0))
    st = build_state(torch, tq, W, 0, None, workload, extra_pages=grow // 128 + 3)
    ctx, B, Hq, Hkv, d = st["ctx"], st["B"], st["Hq"], st["Hkv"], st["d"]
    W_max, E = st["hot"], evict_block
    window = W_max - E
    dev = st["q"].device
    k_new = torch.randn((B, Hkv, d), device=dev).half()
    v_new = torch.randn((B, Hkv, d), device=dev).half()
    hot_start = torch.zeros(B, dtype=torch.int32, device=dev)
    ws = torch.empty(tq.tq_monarch_workspace_bytes(ctx.handle, B, Hq, Hkv, st["table"].shape[-1],
                                                   W_max, E), dtype=torch.uint8, device=dev)
    used = torch.empty((B, Hq), dtype=torch.int32, device=dev)
    res = {"workload": workload, "evict_block": E, "window": window, "hot_slots": W_max,
           "steps": steps}
    pr = None
    if promotion is not None:
        cap = st["table"].shape[-1] * tq.TQ_PAGE_TOKENS
        pr = dict(promotion, cold_mask=torch.zeros((B, cap // 32), dtype=torch.int32, device=dev),
                  counts=torch.zeros((B, cap), dtype=torch.uint8, device=dev),
                  logits=torch.empty((B, Hq, cap), dtype=torch.float32, device=dev))
        res["promotion"] = dict(promotion)
    for thr in thresholds:
        st["hot_len"].fill_(window)
        hot_start.zero_()
        st["cold_len"].fill_(st["cold"])
        if pr is not None:
            pr["cold_mask"].zero_()
            pr["counts"].zero_()

        def step():
            if pr is None:
                tq.tq_monarch_step(ctx.handle, st["q"], k_new, v_new, st["k_hot"], st["v_hot"],
                                   hot_start, st["hot_len"], st["pool"], st["table"],
                                   st["cold_len"], thr, window, E, st["out"], ws, Hkv,
                                   cold_used=used)
            else:
                tq.tq_monarch_step_promote(ctx.handle, st["q"], k_new, v_new, st["k_hot"],
                                           st["v_hot"], hot_start, st["hot_len"], st["pool"],
                                           st["table"], st["cold_len"], thr, window, E, pr,
                                           st["out"], ws, Hkv, cold_used=used)
        ms = graph_ms(torch, step, steps)
        ctx.check()
        tokens = B * Hkv * (W_max + st["cold"])
        row = {"us_per_step": ms * 1e3, "kv_tokens_heads_per_s": tokens / (ms / 1e3),
               "heads_reading_cold": float(used.float().mean())}
        if pr is not None:  # cold positions moved back over every step run (warm-up included)
            row["moved_back"] = int(sum(bin(int(w) & 0xFFFFFFFF).count("1")
                                        for w in pr["cold_mask"].flatten().tolist()))
        res["threshold_%s" % thr] = row
    del st
    torch.cuda.empty_cache()
    return res


def measure_tensor_cache(torch, tq, W, workload, steps=256):
    """Tensor Cache steps on a decode workload's shapes: the fp16 ring holds
    the workload's hot length W (full, so every step evicts one token per kv
    head into A), no cold pages; each step replayed from a CUDA graph."""
    cfg = W.DECODE[workload]
    B, Hq, Hkv, d, Wr = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["d"], cfg["hot"]
    ctx = tq.Context(d, seed=0)
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(51)
    k_ring = torch.randn((B, Hkv, Wr, d), generator=gen, device=dev).half()
    v_ring = torch.randn((B, Hkv, Wr, d), generator=gen, device=dev).half()
    A = torch.randn((B, Hkv, d, d), generator=gen, device=dev) * 0.01
    lam = torch.full((Hkv,), 0.95, device=dev)
    eta = torch.full((Hkv,), 0.1, device=dev)
    gate = torch.zeros(Hq, device=dev)
    q = torch.randn((B, Hq, d), generator=gen, device=dev).to(getattr(torch, cfg["q_dtype"]))
    k_new = torch.randn((B, Hkv, d), generator=gen, device=dev).half()
    v_new = torch.randn((B, Hkv, d), generator=gen, device=dev).half()
    rs = torch.zeros(B, dtype=torch.int32, device=dev)
    rl = torch.full((B,), Wr, dtype=torch.int32, device=dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_tensor_cache_workspace_bytes(ctx.handle, B, Hq, Hkv, Wr),
                     dtype=torch.uint8, device=dev)

    def step():
        tq.tq_tensor_cache_step(ctx.handle, q, k_new, v_new, k_ring, v_ring, rs, rl, A, lam, eta,
                                gate, out, ws, Hkv)
    ms = graph_ms(torch, step, steps)
    ctx.check()
    # bytes per step: the ring once (fp16 K and V), A read and written, q, out
    by = B * Hkv * (Wr * 4 * d + 8 * d * d) + B * Hq * d * 6
    return {"workload": workload + " shapes, fp16 ring of %d + d x d fp32 memory" % Wr,
            "us_per_step": ms * 1e3, "bytes_per_step": by,
            "achieved_gbs": by / (ms / 1e3) / 1e9}


def measure_self_index(torch, tq, reps=3, B=16):
    """Self-Indexing on the 32K decode's key shapes (B = 16 x 8 kv heads x
    32768 fp16 keys and values, d = 128, 32 query heads, top_k = 7.5 % of T):
    kernel times (CUDA events, median of reps) and GB/s over the algorithmic
    bytes -- keys read + codes and centroids written (build), codes read +
    scores written (scores), scores read + picked written (select), the 64
    sinks' and the picked tokens' key and value rows read per query head
    (attend).  A smaller B only sizes profiler captures."""
    Hkv, Hq, T, d = 8, 32, 32768, 128
    top_k = round(0.075 * T)
    ctx = tq.Context(d, seed=0)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(61)
    k = torch.randn((B, Hkv, T, d), generator=gen, device="cuda").half()
    q = torch.randn((B, Hq, d), generator=gen, device="cuda").to(torch.bfloat16)
    mu = torch.empty((B, Hkv, d), device="cuda")
    codes = torch.empty((B, Hkv, T, d // 4), dtype=torch.uint8, device="cuda")
    cent = torch.empty((B, Hkv, d // 4, 16, 4), device="cuda")
    scores = torch.empty((B, Hq, T), device="cuda")
    v = torch.randn((B, Hkv, T, d), generator=gen, device="cuda").half()
    picked = torch.empty((B, Hq, top_k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, Hq, d), device="cuda")
    times = {"build": [], "scores": [], "select": [], "attend": []}
    for i in range(reps + 1):
        for which, lst in times.items():
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            if which == "build":
                tq.tq_self_index_build(ctx.handle, k, mu, codes, cent)
            elif which == "scores":
                tq.tq_self_index_scores(ctx.handle, q, codes, cent, scores, Hkv)
            elif which == "select":
                tq.tq_self_index_select(ctx.handle, scores, picked)
            else:
                tq.tq_self_index_attend(ctx.handle, q, k, v, picked, out)
            b.record()
            torch.cuda.synchronize()
            if i > 0:
                lst.append(a.elapsed_time(b))
    ctx.check()
    algo = {"build": B * Hkv * T * (2 * d + d // 4),
            "scores": B * Hq * T * (d // 4 + 4),
            "select": B * Hq * (T * 4 + top_k * 4),
            "attend": B * Hq * ((64 + top_k) * 2 * d * 2 + top_k * 4 + d * 2 + d * 4)}
    peak = float(measured_peaks()[0]["hbm_gbs"])
    row = {"workload": "%d x 8 kv heads x 32768 fp16 keys and values, d=128; 32 query "
                       "heads; top_k = %d (7.5%% of T) + 64 sinks" % (B, top_k)}
    for which, lst in times.items():
        m = statistics.median(lst)
        row[which + "_ms"] = m
        row[which + "_gbs"] = algo[which] / (m / 1e3) / 1e9
        row[which + "_hbm_frac"] = algo[which] / (m / 1e3) / 1e9 / peak
    return row


def measure_stage1(torch, tq, N=1 << 20, reps=5):
    """Stage-1 variants on 2^20 rotated fp32 vectors (d = 128, N(0,1)):
    encode and decode kernel times (CUDA events, median of reps) with their
    HBM bytes, and the distortion of encode -> decode (relative MSE, and the
    RMS inner-product error against 64 random unit queries) on the first
    65536 vectors."""
    d = 128
    ctx = tq.Context(d, seed=0)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(41)
    x = torch.randn((N, d), generator=gen, device="cuda")
    q = torch.randn((64, d), generator=gen, device="cuda", dtype=torch.float64)
    q /= q.norm(dim=1, keepdim=True)
    xh = torch.empty_like(x)
    peaks, _ = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    res = []
    for kind, b1, b2, name in ((tq.TQ_STAGE1_POLAR, 4, 2, "polar b1=4 b2=2"),
                               (tq.TQ_STAGE1_MSE, 3, 0, "mse b=3"),
                               (tq.TQ_STAGE1_MSE, 2, 0, "mse b=2"),
                               (tq.TQ_STAGE1_MSE, 4, 0, "mse b=4")):
        cb = tq.tq_stage1_code_bytes(ctx.handle, kind, b1, b2)
        codes = torch.empty((N, cb), dtype=torch.uint8, device="cuda")
        norms = torch.empty(N, dtype=torch.int16, device="cuda")
        times = {"encode": [], "decode": []}
        for i in range(reps + 1):
            for what in ("encode", "decode"):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                if what == "encode":
                    tq.tq_stage1_encode(ctx.handle, kind, b1, b2, x, codes, norms)
                else:
                    tq.tq_stage1_decode(ctx.handle, kind, b1, b2, codes, norms, xh)
                b.record()
                torch.cuda.synchronize()
                if i > 0:
                    times[what].append(a.elapsed_time(b))
        n_s = 65536
        xs, hs = x[:n_s].double(), xh[:n_s].double()
        rel = ((hs - xs) ** 2).sum(1) / (xs ** 2).sum(1)
        ip = (hs - xs) @ q.T
        row = {"variant": name, "code_bytes_per_vector": cb + 2,
               "bits_per_coordinate": 8.0 * (cb + 2) / d,
               "relative_mse": float(rel.mean()), "ip_rms_error": float(ip.pow(2).mean().sqrt())}
        for what in ("encode", "decode"):
            ms = statistics.median(times[what])
            by = N * (d * 4 + cb + 2)
            row[what + "_ms"] = ms
            row[what + "_gbs"] = by / (ms / 1e3) / 1e9
            row[what + "_hbm_frac"] = row[what + "_gbs"] / peak
        res.append(row)
        del codes, norms
    ctx.check()
    return {"workload": "2^20 rotated N(0,1) vectors, d=128, fp32", "variants": res}


def decode(tq, st, q=None, out=None):
    tq.tq_decode_attention(st["ctx"].handle, st["q"] if q is None else q, st["k_hot"],
                           st["v_hot"], st["hot_len"], st["pool"], st["table"], st["cold_len"],
                           st["out"] if out is None else out, st["ws"], st["Hkv"])


def reduce_max(torch, x, world):
    """The maximum of x over ranks (a time: the slowest rank's)."""
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


def cpu_baseline(sample_groups=None):
    """The oracle, as it stands, on a bounded sample of the workload: a few
    (batch, kv head) groups of the 32K decode with random cold records."""
    import oracle as O
    from compressed_kv_decode_b200 import workloads as W
    cfg = W.DECODE[WORKLOAD]
    d, G = cfg["d"], cfg["Hq"] // cfg["Hkv"]
    cores = os.cpu_count() or 1
    n = sample_groups or max(1, min(cfg["B"] * cfg["Hkv"], cores))
    P = O.Params(d, seed=0)
    nbytes, _ = O.page_layout(d, d, True)
    max_pages = cfg["cold"] // 128
    table = np.arange(n * max_pages, dtype=np.int32).reshape(n, 1, max_pages)
    pool = W.random_page_bytes(7, n * max_pages, nbytes, O.norm_slots(d, d, True))
    rng = np.random.default_rng(8)
    k_hot = rng.standard_normal((n, 1, cfg["hot"], d)).astype(np.float16).astype(np.float64)
    v_hot = rng.standard_normal((n, 1, cfg["hot"], d)).astype(np.float16).astype(np.float64)
    q = W.queries(13, n, G, d, "bfloat16")
    lens_c = np.full(n, cfg["cold"], np.int32)
    lens_h = np.full(n, cfg["hot"], np.int32)
    threads = O.max_threads()
    t0 = time.perf_counter()
    O.attention(P, q, 1, 1.0 / math.sqrt(d), k_hot, v_hot, lens_h, pool.reshape(-1), nbytes,
                table, lens_c, threads=threads)
    dt = time.perf_counter() - t0
    t1 = time.perf_counter()  # one thread, one group
    O.attention(P, q[:1], 1, 1.0 / math.sqrt(d), k_hot[:1], v_hot[:1], lens_h[:1],
                pool.reshape(-1), nbytes, table[:1], lens_c[:1], threads=1)
    dt1 = time.perf_counter() - t1
    units = n * (cfg["cold"] + cfg["hot"])
    return {"value": units / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "value_1_thread": (cfg["cold"] + cfg["hot"]) / dt1,
            "sample": "%d of %d (batch, kv head) groups of the 32K decode (%d tokens each), "
                      "random cold records, %.2f s; 1 thread: 1 group, %.2f s"
                      % (n, cfg["B"] * cfg["Hkv"], cfg["cold"] + cfg["hot"], dt, dt1)}


def cpu_baseline_compress(n=1 << 18, n1=1 << 14):
    """The oracle's encoder (rotation, codes, residual, QJL sketch, keys) on a
    bounded sample of the compress workload: n of its 4194304 vectors on all
    host threads, n1 of them on one thread."""
    import oracle as O
    from compressed_kv_decode_b200 import workloads as W
    d, H = 128, 8
    P = O.Params(d, seed=0)
    scales = W.compress_scales(21, H, d)
    x = W.compress_data(22, scales, 524288, rows=(0, 0, n))[0]
    threads = O.max_threads()
    t0 = time.perf_counter()
    O.encode(P, x, True, threads=threads)
    dt = time.perf_counter() - t0
    t1 = time.perf_counter()
    O.encode(P, x[:n1], True, threads=1)
    dt1 = time.perf_counter() - t1
    return {"value": n / dt, "unit": "vectors/s", "cores": threads, "kind": "oracle",
            "value_1_thread": n1 / dt1,
            "sample": "%d of the 4194304 vectors (head 0), %.2f s; 1 thread: %d vectors, %.2f s"
                      % (n, dt, n1, dt1)}


def cpu_baseline_search(nq=256, nq1=16):
    """The oracle's search (estimated inner products with every database
    record, exact top-10) for nq of the 4096 queries against the full 10^6
    database, which the oracle's encoder writes; nq1 queries on one thread."""
    import oracle as O
    from compressed_kv_decode_b200 import workloads as W
    d, N, k = 128, 1_000_000, 10
    P = O.Params(d, seed=0)
    threads = O.max_threads()
    db = W.unit_vectors(31, N, d)
    rec = O.encode(P, db, True, threads=threads)
    nb, _ = O.page_layout(d, d, False)
    pool = np.zeros(((N + 127) // 128) * nb, np.uint8)
    idx = np.arange(N)
    O.pack(pool, nb, d, d, False, idx // 128, idx % 128,
           {f: rec[f] for f in ("sign", "mag", "qbits", "n", "gamma")})
    del rec
    qs = W.unit_vectors(32, 4096, d)
    t0 = time.perf_counter()
    O.topk(P, qs[:nq], pool, nb, N, k, threads=threads)
    dt = time.perf_counter() - t0
    t1 = time.perf_counter()
    O.topk(P, qs[:nq1], pool, nb, N, k, threads=1)
    dt1 = time.perf_counter() - t1
    return {"value": nq * N / dt, "unit": "query*vectors/s", "cores": threads, "kind": "oracle",
            "value_1_thread": nq1 * N / dt1,
            "sample": "%d of the 4096 queries against the full 10^6 database, %.2f s; "
                      "1 thread: %d queries, %.2f s" % (nq, dt, nq1, dt1)}


def run_reference(args, rank, world):
    if rank != 0:
        return
    steps = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline()
        if i >= args.warmup:
            steps.append(r)
    vals = [s["value"] for s in steps]
    value = statistics.mean(vals)
    cb = dict(steps[-1])
    cb["value"] = value
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "ms_per_step": None, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch
    import compressed_kv_decode_b200 as tq
    from compressed_kv_decode_b200 import workloads as W
    torch.cuda.set_device(local_rank)
    st = build_state(torch, tq, W, rank, args.batch)
    ctx = st["ctx"]
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        decode(tq, st)
    torch.cuda.synchronize()
    ctx.check()

    # one decode step (3 launches) captured once in a CUDA graph; the timed
    # region replays it K times, bracketed by barrier + sync
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        decode(tq, st)  # first call outside capture: one-time kernel attributes
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=cap):
            decode(tq, st)
    stream.wait_stream(cap)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for i in range(args.steps):
            graph.replay()
        e1.record(stream)
        e1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ctx.check()
    ms_total = reduce_max(torch, e0.elapsed_time(e1), world)

    # the attention kernel alone, per launch, with CUDA events recorded by the
    # library on the launching stream around that kernel (K more steps)
    ev_k = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk_k:
        for i in range(args.steps):
            # torch reports only events it recorded itself: record both once;
            # the library re-records them around the attention kernel
            ev_k[i][0].record(stream)
            ev_k[i][1].record(stream)
            tq.tq_set_profile_events(ctx.handle, ev_k[i][0], ev_k[i][1])
            decode(tq, st)
        tq.tq_set_profile_events(ctx.handle, None, None)
        torch.cuda.synchronize()
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_k)

    # end to end: q from pinned host memory, output back to pinned host memory
    q_host = st["q"].cpu().pin_memory()
    out_host = torch.empty(st["out"].shape, dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(st["q"])
    for _ in range(3):
        q_dev.copy_(q_host, non_blocking=True)
        decode(tq, st, q=q_dev)
        out_host.copy_(st["out"], non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        q_dev.copy_(q_host, non_blocking=True)
        decode(tq, st, q=q_dev)
        out_host.copy_(st["out"], non_blocking=True)
    f1.record(stream)
    f1.synchronize()
    barrier(world)
    e2e_ms = reduce_max(torch, f0.elapsed_time(f1), world)
    ctx.check()

    units_per_step = st["B"] * st["Hkv"] * (st["cold"] + st["hot"])
    value = units_per_step * world * args.steps / (ms_total / 1e3)
    e2e_value = units_per_step * world * args.steps / (e2e_ms / 1e3)
    peaks, peak_kind = measured_peaks()
    algo_bytes = (st["B"] * st["Hkv"] * (st["cold"] * COLD_RECORD_BYTES + st["hot"] * HOT_RECORD_BYTES)
                  + st["table"].numel() * 4)
    achieved = algo_bytes / (attn_ms / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    meta = {k: st[k] for k in ("B", "Hkv", "Hq", "d", "hot", "cold")}
    q_bytes = st["q"].numel() * st["q"].element_size()
    out_bytes = st["out"].numel() * 4
    if rank != 0:
        return
    cb = cpu_baseline() if world == 1 else None
    rows = {}
    if world == 1:
        rows["gated_decode"] = measure_gated(torch, tq, st)
        rows["gated_decode"]["workload"] = WORKLOAD + " with Monarch's threshold gate"
        del st, graph
        torch.cuda.empty_cache()
        rows["tensor_cache_step"] = [measure_tensor_cache(torch, tq, W, "tinyllama"),
                                     measure_tensor_cache(torch, tq, W, WORKLOAD)]
        torch.cuda.empty_cache()
        rows["monarch_step"] = [measure_monarch(torch, tq, W, "tinyllama", 128),
                                measure_monarch(torch, tq, W, "tinyllama", 1),
                                measure_monarch(torch, tq, W, WORKLOAD, 128),
                                measure_monarch(torch, tq, W, "tinyllama", 128,
                                                thresholds=(float("inf"),),
                                                promotion=dict(threshold=0.15, sticky=3,
                                                               max_per_step=8)),
                                measure_monarch(torch, tq, W, "tinyllama", 128,
                                                thresholds=(float("inf"),),
                                                promotion=dict(threshold=0.002, sticky=3,
                                                               max_per_step=8))]
        torch.cuda.empty_cache()
        rows["compress"] = measure_compress(torch, tq)
        rows["compress"]["cpu_baseline"] = cpu_baseline_compress()
        torch.cuda.empty_cache()
        rows["search"] = measure_search(torch, tq)
        rows["search"]["cpu_baseline"] = cpu_baseline_search()
        torch.cuda.empty_cache()
        rows["stage1"] = measure_stage1(torch, tq)
        torch.cuda.empty_cache()
        rows["self_index"] = measure_self_index(torch, tq)
        peak_tf = float(peaks.get("bf16_tflops", 1590.0))
        rows["compress"]["hbm_frac"] = rows["compress"]["achieved_gbs"] / peak
        rows["compress"]["tensor_frac"] = rows["compress"]["achieved_tflops"] / peak_tf
        rows["search"]["tensor_frac"] = rows["search"]["achieved_tflops"] / peak_tf
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp16/fp32 (3-bit keys, 4-bit values)",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": meta["B"] * world, "kv_heads": meta["Hkv"],
                   "q_heads": meta["Hq"], "head_dim": meta["d"], "hot_tokens": meta["hot"],
                   "cold_tokens": meta["cold"], "parallelism": "dp%d" % world,
                   "l2": "inputs larger than L2 (%.0f MB per step)" % (algo_bytes / 1e6)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind + " hbm_gbs",
                     "kernel": "attn_kernel", "kernel_ms": attn_ms,
                     "algorithmic_bytes_per_launch": algo_bytes,
                     "traffic": kernel_traffic("attn_kernel_llama3_8b_32k",
                                               "compressed_kv_decode_b200/csrc/tq_decode.cu")},
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": q_bytes, "d2h_bytes_per_step": out_bytes},
        "gpu_launches": 3 * args.steps,
        "step": "one decode call (query prep, split-K attention, combine) replayed from a CUDA graph",
        "clocks": clk.summary(),
        "clocks_kernel_pass": clk_k.summary(),
        "cpu_baseline": cb,
        "rows": rows,
    }
    print(json.dumps(line), flush=True)


def run_only(args):
    """One extra row alone, for profiler captures of its kernels."""
    import torch
    import compressed_kv_decode_b200 as tq
    from compressed_kv_decode_b200 import workloads as W
    if args.only == "gated":
        st = build_state(torch, tq, W, 0, args.batch)
        res = measure_gated(torch, tq, st, reps=args.steps)
    elif args.only == "monarch":
        res = measure_monarch(torch, tq, W, "tinyllama", 128, steps=args.steps)
    elif args.only == "promotion":
        res = measure_monarch(torch, tq, W, "tinyllama", 128, steps=args.steps,
                              thresholds=(float("inf"),),
                              promotion=dict(threshold=0.002, sticky=3, max_per_step=8))
    elif args.only == "tensor_cache":
        res = measure_tensor_cache(torch, tq, W, WORKLOAD, steps=args.steps)
    elif args.only == "self_index":  # --batch b: b sequences (default 16)
        res = measure_self_index(torch, tq, reps=max(1, args.steps), B=args.batch or 16)
    elif args.only == "compress":  # --batch b: 8 heads x b * 65536 vectors
        res = measure_compress(torch, tq, reps=max(1, args.steps), T=65536 * (args.batch or 8))
    elif args.only == "search":  # --batch b: b * 100000 database vectors
        res = measure_search(torch, tq, reps=max(1, args.steps), N=100_000 * (args.batch or 10))
    else:
        res = measure_stage1(torch, tq, reps=max(1, args.steps))
    print(json.dumps({"only": args.only, "row": res}), flush=True)


def main():
    args = parse()
    rank, world, local_rank = dist_env()
    if args.only:
        run_only(args)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
