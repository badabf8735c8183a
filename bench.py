#!/usr/bin/env python
"""Throughput of the RTPurbo attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--no-prefill] [--no-cpu-baseline]

One step = one decode token for the whole mixed layer on the 128K-cache,
batch-8 workload (32 query / 4 kv heads, 1 retrieval kv head, p = 0.95,
window 4096 + 4 sinks): indexer projection of the new token (q16 + k16 append),
exact top-p over the 128K k16 cache, gathered sparse attention on the retrieval
heads, sink+window attention on the local heads.  `value` is decode tokens/s
(batch / step time) summed over ranks; each rank decodes its own batch (weak
scaling, no data-path collective).  The prefill of the 128K workload (1 x 131072
tokens, chained needles) is timed in the same run and reported in `prefill`.

Timing: W untimed warm-up steps, then exactly K steps, each bracketed by CUDA
events on the launching stream with an L2 flush between steps (outside the
events: 256 MB written, then 256 MB read, so that no dirty line of the flush is
written back inside a timed step); a barrier + synchronize on both sides; the
max over ranks.

--impl reference times the fp64 CPU oracle on this host's cores on the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill & decode tokens/s per layer at 128K (1 B200); % of HBM / tensor roofline"
DECODE_WL = "decode_128k_b8"
PREFILL_WL = "prefill_128k"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-steps", type=int, default=3)
    ap.add_argument("--no-1m", action="store_true", help="skip the 1M prefill workload")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the block top-p / top-k / ring-cache decode lines")
    ap.add_argument("--case", default=None, choices=["decode", "select", "prefill", "dense"],
                    help="run one small case twice and exit (for profilers)")
    ap.add_argument("--L", type=int, default=16384, help="sequence length for --case")
    return ap.parse_args()


def run_case(args):
    """One case, run twice (the second is the one to capture), then exit."""
    import torch
    from long_context_sparse_rtp_b200 import (build, rtp_dense_attn, rtp_index_scores,
                                              rtp_layer_prefill, rtp_topp_select, synth)
    build.build()
    torch.cuda.set_device(0)
    if args.case == "decode":
        st = decode_state(0)
        for _ in range(2):
            decode_step(st, None, None)
    else:
        w = synth.WORKLOADS[PREFILL_WL]
        inp = synth.make_inputs(w, "cuda", L=args.L)
        q, k, v, Wq, Wk, role = (inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
        for _ in range(2):
            if args.case == "select":
                q16, k16 = rtp_index_scores(q, k, Wq, Wk, role)
                rtp_topp_select(q16, k16, role, w.p, H=w.H)
            elif args.case == "prefill":
                rtp_layer_prefill(q, k, v, Wq, Wk, role, p=w.p, window=w.window,
                                  n_sink=w.n_sink)
            else:
                rtp_dense_attn(q, k, v)
    torch.cuda.synchronize()
    print(f"case {args.case} ok")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sus=d["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ helpers
def dist_setup():
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
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time (device tensor under nccl, host tensor under gloo)."""
    import torch
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own replica of the workload (weak scaling)."""
    return seed + 1000 * rank


def profiled_traffic(summary: str):
    """DRAM bytes per launch from a committed ncu summary under profiles/, or None
    when the summary is missing or the kernel's source has changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    traffic = src = sha = None
    for ln in open(path):
        if ln.startswith("traffic_bytes_per_launch:"):
            traffic = int(ln.split(":")[1])
        elif ln.startswith("source:"):
            parts = ln.split()
            src, sha = parts[1], parts[-1]
    if traffic is None or src is None:
        return None
    fn = os.path.join(ROOT, src)
    if not os.path.exists(fn):
        return None
    if hashlib.sha256(open(fn, "rb").read()).hexdigest()[:len(sha)] != sha:
        return None
    return traffic


def trace_read():
    from long_context_sparse_rtp_b200 import rtp

    class Entry(ctypes.Structure):
        _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64),
                    ("total_ms", ctypes.c_double)]
    L = rtp.lib()
    L.rtp_trace_read.restype = ctypes.c_int
    arr = (Entry * 64)()
    n = L.rtp_trace_read(arr, 64)
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(max(n, 0))}


def trace_timeline():
    """(name, start us, end us) of each launch recorded since the last reset."""
    from long_context_sparse_rtp_b200 import rtp

    class Launch(ctypes.Structure):
        _fields_ = [("name", ctypes.c_char * 48), ("start_ms", ctypes.c_double),
                    ("end_ms", ctypes.c_double)]
    L = rtp.lib()
    L.rtp_trace_timeline.restype = ctypes.c_int
    arr = (Launch * 256)()
    n = L.rtp_trace_timeline(arr, 256)
    return [(arr[i].name.decode(), round(arr[i].start_ms * 1e3, 2), round(arr[i].end_ms * 1e3, 2))
            for i in range(max(n, 0))]


def trace(on: bool):
    from long_context_sparse_rtp_b200 import rtp
    rtp.lib().rtp_trace_reset()
    rtp.lib().rtp_trace_enable(1 if on else 0)


# ------------------------------------------------------------------ decode (ours)
def decode_state(rank: int):
    import torch
    from long_context_sparse_rtp_b200 import rtp_index_scores, synth
    w = synth.WORKLOADS[DECODE_WL]
    w = w.with_(seed=rank_seed(w.seed, rank))
    inp = synth.make_inputs(w, "cuda")
    q, k, v, Wq, Wk, role = (inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
    L = k.shape[1]
    # the k16 cache a prefill would have written (state, not part of a step)
    _, k16 = rtp_index_scores(q, k, Wq, Wk, role)
    torch.cuda.synchronize()
    return dict(w=w, q=q, k=k, v=v, Wq=Wq, Wk=Wk, role=role, k16=k16, L=L)


def decode_step(st, o, lse):
    from long_context_sparse_rtp_b200 import rtp_layer_decode
    L = st["L"]
    w = st["w"]
    return rtp_layer_decode(st["q"], st["k"][:, L - 1:], st["k"], st["v"], st["k16"], st["Wq"],
                            st["Wk"], st["role"], pos=L - 1, p=w.p, window=w.window,
                            n_sink=w.n_sink)


L2_FLUSH = ("256 MB written, then another 256 MB read, between timed steps (outside the "
            "events): the L2 (126 MB) holds none of the step's data and no dirty lines")


def make_l2_flush():
    """Between timed steps: write a buffer twice the L2 size, then read another
    one.  The read evicts the written lines, so their write-back to HBM happens
    here and not inside the next timed step."""
    import torch
    wbuf = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    rbuf = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")

    def flush():
        wbuf.fill_(1.0)
        rbuf.sum()

    return flush


def time_steps(fn, steps, warmup, world, flush, traced=False):
    """Per-step CUDA events, L2 flush between steps (outside the events)."""
    import torch
    for _ in range(warmup):
        fn()
        flush()
    trace(traced)
    barrier(world)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        flush()
        evs[i][0].record()
        fn()
        evs[i][1].record()
    barrier(world)
    ms = sum(a.elapsed_time(b) for a, b in evs)
    per_kernel = trace_read() if traced else None
    trace(False)
    return ms, per_kernel


def decode_bytes(st, sel_count_union):
    """Algorithmic HBM bytes of one decode step."""
    w = st["w"]
    B, L = st["q"].shape[0], st["L"]
    k16 = B * L * w.H_ret * 16 * 2
    local = B * (w.Hkv - len(w.ret_kv)) * min(L, w.window + w.n_sink) * 2 * 128 * 2
    gather = sel_count_union * 2 * 128 * 2
    small = B * w.H * 128 * 2 * 2 + B * w.Hkv * 128 * 2 * 2 + B * w.Hkv * 128 * 2
    return dict(k16=k16, local=local, gather=gather, small=small,
                total=k16 + local + gather + small)


def union_size(st, sel):
    """Sum over (batch, retrieval kv head) of the union of the kept keys, derived
    on the device from the thresholds (reporting only)."""
    import torch
    w = st["w"]
    q16 = sel["q16"].float()[:, 0]                          # [B, H_ret, 16]
    k16 = st["k16"][:, :st["L"]].float()                    # [B, L, H_ret, 16]
    s = torch.einsum("bjhc,bhc->bhj", k16, q16)
    thr = sel["sel"]["thr"][..., None]
    jt = sel["sel"]["jtie"][..., None]
    j = torch.arange(st["L"], device=s.device)[None, None]
    keep = (s > thr) | ((s == thr) & (j <= jt))
    tot = 0
    for r in range(len(w.ret_kv)):
        tot += int(keep[:, r * w.G:(r + 1) * w.G].any(dim=1).sum())
    return tot, int(sel["sel"]["count"].sum())


def bench_decode(args, world, rank, local, pk):
    """Device time of the decode step, replayed from one CUDA graph."""
    import torch
    from long_context_sparse_rtp_b200 import DecodeGraph
    st = decode_state(rank)
    w, L = st["w"], st["L"]
    flush = make_l2_flush()

    def make(trace_on=False):
        g = DecodeGraph(st["k"], st["v"], st["k16"], st["Wq"], st["Wk"], st["role"], H=w.H,
                        pos=L - 1, p=w.p, window=w.window, n_sink=w.n_sink, trace=trace_on)
        g.q.copy_(st["q"])
        return g

    g = make()
    clocks = ClockSampler(local)
    clocks.start()
    ms, _ = time_steps(g.replay, args.steps, args.warmup, world, flush)
    clk = clocks.stop()
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    # per-kernel device times: a second graph whose trace events are graph nodes
    gt = make(trace_on=True)
    kern = {}
    for _ in range(args.steps):
        flush()
        gt.replay()
        torch.cuda.synchronize()
        for name, (n, t) in trace_read().items():
            a0, a1 = kern.get(name, (0, 0.0))
            kern[name] = (a0 + n, a1 + t)
    timeline = trace_timeline()  # the last replay: each launch's start and end
    trace(False)
    res = decode_step(st, None, None)
    torch.cuda.synchronize()
    from long_context_sparse_rtp_b200 import rtp_check_device
    rtp_check_device()  # no kernel recorded an error during the timed steps
    union, compute_sel = union_size(st, res)
    B = st["q"].shape[0]
    nbytes = decode_bytes(st, union)
    return dict(st=st, ms_step=ms_step, clocks=clk, kern=kern, union=union,
                compute_sel=compute_sel, bytes=nbytes, B=B, flush=flush, graph=g,
                timeline=timeline)


def bench_decode_e2e(dec, args, world):
    """Through the public API with host buffers: H2D of the new token's q/k/v
    rows from pinned memory, one DecodeGraph step, D2H of the output."""
    import torch
    st = dec["st"]
    g = dec["graph"]
    L = st["L"]
    hq = st["q"].cpu().pin_memory()
    hk = st["k"][:, L - 1:].contiguous().cpu().pin_memory()
    hv = st["v"][:, L - 1:].contiguous().cpu().pin_memory()
    ho = torch.empty_like(hq).pin_memory()

    def step():
        g.step(hq, hk, hv, ho)

    ms, _ = time_steps(step, args.steps, args.warmup, world, dec["flush"])
    ms = max_over_ranks(ms, world)
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2
    d2h = ho.numel() * 2
    return ms / args.steps, h2d, d2h


def bench_decode_shared_k16(dec, args, world):
    """The same decode step with one k16 per retrieval kv head (the G query heads
    of a kv head share it: 1/8 of the k16 bytes at G = 8), replayed from a graph."""
    import torch
    from long_context_sparse_rtp_b200 import DecodeGraph, rtp_index_scores
    st = dec["st"]
    w, L = st["w"], st["L"]
    Wk = st["Wk"][[s for s in range(0, w.H_ret, w.G)]].contiguous()
    _, k16 = rtp_index_scores(st["q"], st["k"], st["Wq"], Wk, st["role"], k16_per_kv_head=1)
    g = DecodeGraph(st["k"], st["v"], k16, st["Wq"], Wk, st["role"], H=w.H, pos=L - 1, p=w.p,
                    window=w.window, n_sink=w.n_sink, k16_per_kv_head=1)
    g.q.copy_(st["q"])
    ms, _ = time_steps(g.replay, args.steps, args.warmup, world, dec["flush"])
    ms = max_over_ranks(ms, world) / args.steps
    B = st["q"].shape[0]
    k16_bytes = B * L * len(w.ret_kv) * 16 * 2
    del g, k16
    torch.cuda.empty_cache()
    return dict(ms_step=ms, tokens_per_s=B * world / (ms / 1e3), k16_bytes=k16_bytes)


def bench_decode_dense(dec, args):
    """The dense kernel on the same decode step: every query head attends to the
    whole cache (rtp_dense_attn with one query row), the baseline the sparse
    step replaces.  Algorithmic bytes: the K and V rows of every kv head."""
    import torch
    from long_context_sparse_rtp_b200 import rtp_dense_attn
    st = dec["st"]
    q, k, v, L = st["q"], st["k"], st["v"], st["L"]
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[2], 1, dtype=torch.float32, device=q.device)
    ms, _ = time_steps(lambda: rtp_dense_attn(q, k, v, q_pos0=L - 1, o=o, lse=lse),
                       args.steps, args.warmup, 1, dec["flush"])
    return dict(ms_step=ms / args.steps, bytes=k.shape[0] * L * k.shape[2] * 128 * 2 * 2)


def _keep_mask(scores, thr, jtie):
    import torch
    j = torch.arange(scores.shape[-1], device=scores.device)
    t, jt = thr[..., None], jtie[..., None]
    return (scores > t) | ((scores == t) & (j <= jt))


def bench_decode_variants(dec, args, world):
    """The same decode step with block-level top-p and with static top-k
    (k = 4096) on the retrieval heads (graph replay), and their recall of the
    exact top-p kept keys: the share of those keys, and of the indexer softmax
    mass, that each keeps."""
    import torch
    from long_context_sparse_rtp_b200 import (DecodeGraph, rtp_index_scores,
                                              rtp_sparse_attn_decode_select)
    st = dec["st"]
    w, L = st["w"], st["L"]
    out = {}
    for select in ("block_topp", "topk"):
        g = DecodeGraph(st["k"], st["v"], st["k16"], st["Wq"], st["Wk"], st["role"], H=w.H,
                        pos=L - 1, p=w.p, window=w.window, n_sink=w.n_sink, select=select,
                        top_k=4096)
        g.q.copy_(st["q"])
        ms, _ = time_steps(g.replay, args.steps, args.warmup, world, dec["flush"])
        ms = max_over_ranks(ms, world) / args.steps
        out[select] = {"ms_per_step": ms, "tokens_per_s": st["q"].shape[0] * world / (ms / 1e3)}
        del g
    q16, _ = rtp_index_scores(st["q"], None, st["Wq"], st["Wk"], st["role"], H=w.H)
    args_ = (st["q"], st["k"], st["v"], q16, st["k16"], st["role"])
    _, _, ex = rtp_sparse_attn_decode_select(*args_, "topp", p=w.p, want_scores=True)
    _, _, bl = rtp_sparse_attn_decode_select(*args_, "block_topp", p=w.p)
    _, _, tk = rtp_sparse_attn_decode_select(*args_, "topk", top_k=4096)
    s = ex["scores"]
    exact = _keep_mask(s, ex["thr"], ex["jtie"])
    masks = {"topk": _keep_mask(s, tk["thr"], tk["jtie"])}
    wb = bl["block_mask"].to(torch.int64) & 0xFFFFFFFF
    blk = ((wb[..., :, None] >> torch.arange(32, device=s.device)) & 1).flatten(-2)
    masks["block_topp"] = blk[..., torch.arange(s.shape[-1], device=s.device) // 64].bool()
    wgt = torch.exp(s - s.max(dim=-1, keepdim=True).values)
    for name, m in masks.items():
        out[name].update({
            "mean_keys": float(m.sum(-1).float().mean()),
            "token_recall_of_exact_topp": float((m & exact).sum() / exact.sum()),
            "indexer_mass_kept": float(((wgt * m).sum(-1) / wgt.sum(-1)).mean())})
    out["exact_topp_mean_keys"] = float(exact.sum(-1).float().mean())
    del s, ex, bl, tk, exact, masks, wgt
    torch.cuda.empty_cache()
    return out


def bench_decode_ring(dec, args, world):
    """The same decode step with the local heads on the window-only ring cache
    (written from the cache's first L - 1 positions; each step appends its token)."""
    import torch
    from long_context_sparse_rtp_b200 import DecodeGraph, local_ring_alloc, rtp_local_ring_write
    st = dec["st"]
    w, L = st["w"], st["L"]
    B = st["q"].shape[0]
    kr, vr = local_ring_alloc(B, st["role"], window=w.window, n_sink=w.n_sink, device="cuda")
    rtp_local_ring_write(st["k"][:, :L - 1], st["v"][:, :L - 1], kr, vr, st["role"],
                         window=w.window, n_sink=w.n_sink, pos0=0, H=w.H)
    g = DecodeGraph(st["k"], st["v"], st["k16"], st["Wq"], st["Wk"], st["role"], H=w.H,
                    pos=L - 1, p=w.p, window=w.window, n_sink=w.n_sink, local_ring=(kr, vr))
    g.q.copy_(st["q"])
    ms, _ = time_steps(g.replay, args.steps, args.warmup, world, dec["flush"])
    ms = max_over_ranks(ms, world) / args.steps
    n_lkv = int(sum(1 for x in st["role"] if int(x) == 0))
    ring_bytes = (kr.numel() + vr.numel()) * 2
    full_bytes = B * L * n_lkv * 128 * 2 * 2
    del g, kr, vr
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "tokens_per_s": B * world / (ms / 1e3),
            "local_kv_bytes_ring": ring_bytes, "local_kv_bytes_full_cache": full_bytes}


# ------------------------------------------------------------------ prefill (ours)
PREFILL_SET = ("prefill_2k", "prefill_32k", "prefill_128k", "prefill_1m")
PREFILL_DESC = {
    "prefill_2k": "causal prefill 1 x 2048, 8 q / 2 kv, kv0 retrieval, window 256+4, p=0.9, "
                  "8 needles per retrieval head",
    "prefill_32k": "causal prefill 1 x 32768, 32 q / 4 kv, kv0-1 retrieval, window 2048+4, "
                   "per-query temperature, p swept",
    "prefill_128k": "causal prefill 1 x 131072, 32 q / 4 kv, kv0 retrieval, window 4096+4, "
                    "p=0.95, 4-key needle chains",
    "prefill_1m": "causal prefill 1 x 1048576, 32 q / 4 kv, kv0 retrieval, window 4096+4, "
                  "p=0.95, needles per 4096-row group",
}
ATTN_FLOP_PER_PAIR = 4 * 128  # QK^T and PV: 2 x 2 x 128 per (query row, key)


def tile_pairs(L, window=None, n_sink=0):
    """(query row, key) pairs the 128 x 128 tile schedule of attn_tc computes per
    head: every causal tile (dense, sparse) or the sink and window tiles (local)."""
    import numpy as np
    nb = (L + 127) // 128
    rb = np.arange(nb, dtype=np.int64)
    P0 = rb * 128
    t_end = (np.minimum(L, P0 + 128) - 1) // 128
    if window is None:
        n = t_end + 1
    else:
        sink_end = np.full(nb, (n_sink + 127) // 128)
        win_begin = np.maximum(np.maximum(P0 - window + 1, 0) // 128, sink_end)
        sink_end = np.minimum(sink_end, t_end + 1)
        n = sink_end + np.maximum(0, t_end - win_begin + 1)
    return int(n.sum()) * 128 * 128


def local_pairs(L, window, n_sink):
    """Pairs of the sink + window rule per local head: sum over P of min(P + 1, n_sink + window)."""
    c = window + n_sink
    if L <= c:
        return L * (L + 1) // 2
    return c * (c + 1) // 2 + (L - c) * c


def measure_ex2_rate():
    """Sustained ex2.approx.f32 rate of the device (per second), from the
    library's probe kernel timed with CUDA events (best of 5 after a warm-up)."""
    import torch
    from long_context_sparse_rtp_b200.rtp import rtp_probe_ex2
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    blocks, iters = n_sm * 8, 4096
    out = torch.empty(blocks * 256, dtype=torch.float32, device="cuda")
    rtp_probe_ex2(blocks, iters, out)
    best = None
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        rtp_probe_ex2(blocks, iters, out)
        b.record()
        b.synchronize()
        t = a.elapsed_time(b) / 1e3
        best = t if best is None else min(best, t)
    return blocks * 256 * iters * 8 / best


def bench_prefill_config(name, args, world, rank, pk, ex2_rate, cpu=False):
    """One prefill workload: the whole layer (index, select, sparse, local) per p,
    the dense kernel and the summary's own prefill (retrieval heads dense) at
    the same L, per-kernel times and rooflines."""
    import torch
    from long_context_sparse_rtp_b200 import rtp_check_device, rtp_dense_attn, rtp_layer_prefill
    from long_context_sparse_rtp_b200 import synth
    w = synth.WORKLOADS[name]
    w = w.with_(seed=rank_seed(w.seed, rank))
    inp = synth.make_inputs(w, "cuda")
    q, k, v, Wq, Wk, role = (inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
    L = q.shape[1]
    big = L >= (1 << 20)
    steps = 1 if big else args.prefill_steps
    warm = 0 if big else 1  # a 1M layer runs for seconds; the kernels are loaded already
    flush = make_l2_flush()
    peak = pk["bf16_sus"] if big else pk["bf16"]
    peak_kind = "sustained" if big else "burst"
    causal = L * (L + 1) / 2
    dense_tiles = tile_pairs(L)
    loc_tiles = tile_pairs(L, w.window, w.n_sink)
    H_loc = w.H - w.H_ret
    out = {"workload": f"{name}: {PREFILL_DESC[name]}", "L": L, "steps": steps,
           "peak_kind": peak_kind}

    def tensor(kernel_ms, method_pairs, computed_pairs):
        t = kernel_ms / 1e3
        fm = method_pairs * ATTN_FLOP_PER_PAIR / t / 1e12
        ft = computed_pairs * ATTN_FLOP_PER_PAIR / t / 1e12
        return {"ms": kernel_ms, "tflops_method_pairs": fm, "frac_method_pairs": fm / peak,
                "tflops_computed_tiles": ft, "frac_computed_tiles": ft / peak}

    runs = []
    for p in (w.p_sweep or (w.p,)):
        def step(p=p):
            rtp_layer_prefill(q, k, v, Wq, Wk, role, p=p, window=w.window, n_sink=w.n_sink)
        ms, kern = time_steps(step, steps, warm, world, flush, traced=True)
        ms = max_over_ranks(ms, world) / steps
        per = {k_: t / n for k_, (n, t) in kern.items()}
        res = rtp_layer_prefill(q, k, v, Wq, Wk, role, p=p, window=w.window, n_sink=w.n_sink)
        torch.cuda.synchronize()
        rtp_check_device()
        kept = float(res["sel"]["count"].double().sum())
        del res
        r = {"p": p, "ms": ms, "tokens_per_s": L * world / (ms / 1e3), "per_kernel_ms": per,
             "kept_pairs": kept, "kept_share": kept / (w.H_ret * causal)}
        roof = {}
        if "attn_prefill_sparse" in per:
            roof["attn_prefill_sparse"] = tensor(per["attn_prefill_sparse"], kept,
                                                 w.H_ret * dense_tiles)
        if "attn_prefill_local" in per:
            roof["attn_prefill_local"] = tensor(per["attn_prefill_local"],
                                                H_loc * local_pairs(L, w.window, w.n_sink),
                                                H_loc * loc_tiles)
        if "topp_select" in per:
            t = per["topp_select"] / 1e3
            exp_ms = w.H_ret * causal / ex2_rate * 1e3
            roof["topp_select"] = {
                "ms": per["topp_select"], "bound": "alu (one exp per causal pair at least)",
                "exp_bound_ms": exp_ms, "frac_of_exp_bound": exp_ms / per["topp_select"],
                "tensor_frac_3_sweeps": 3 * 32 * w.H_ret * dense_tiles / t / 1e12 / peak}
        r["roofline"] = roof
        runs.append(r)
    out["runs"] = runs
    # the dense kernel on every head at the same L
    o = torch.empty_like(q)
    dms, _ = time_steps(lambda: rtp_dense_attn(q, k, v, o=o), 1, warm, world, flush)
    dms = max_over_ranks(dms, world)
    out["dense"] = {"ms": dms, "tokens_per_s": L / (dms / 1e3),
                    **{k_: v_ for k_, v_ in tensor(dms, w.H * causal, w.H * dense_tiles).items()
                       if k_ != "ms"}}
    for r in runs:
        r["speedup_vs_dense"] = dms / r["ms"]
    # the summary's own prefill: retrieval heads dense (with the k16 projection
    # the decode steps need), local heads sink + window
    pms, pk_ = time_steps(lambda: rtp_layer_prefill(q, k, v, Wq, Wk, role, p=w.p,
                                                    window=w.window, n_sink=w.n_sink,
                                                    retrieval="dense"),
                          1, warm, world, flush, traced=True)
    pms = max_over_ranks(pms, world)
    out["pages_mode"] = {
        "what": "retrieval heads dense, local heads sink + window (the summary's prefill)",
        "ms": pms, "tokens_per_s": L / (pms / 1e3), "speedup_vs_dense": dms / pms,
        "per_kernel_ms": {k_: t / n for k_, (n, t) in pk_.items()}}
    if cpu:
        try:
            out["cpu_baseline"] = oracle_prefill_baseline(w, inp)
        except Exception as e:  # report, never hide
            out["cpu_baseline"] = {"error": repr(e)}
    del o, inp, q, k, v
    torch.cuda.empty_cache()
    return out, w


def oracle_prefill_baseline(w, inp, n_pos=4):
    """The oracle on a seeded sample of one prefill workload, extrapolated to the
    whole layer: the k16 projection timed on up to 16384 key rows and scaled to
    every key and k16 slot; retrieval rows (full sort per row) at n_pos
    positions fitted to c * P * log2(P); local rows at n_pos positions fitted to
    c' * min(P + 1, window + n_sink); q16 projections scaled per row."""
    import numpy as np
    import oracle
    from long_context_sparse_rtp_b200 import synth
    L = inp["q"].shape[1]
    ret, loc = w.retrieval_q_heads(), w.local_q_heads()
    rng = np.random.default_rng(77)
    pos = sorted(set([L - 1] + [int(x) for x in rng.integers(L // 4, L, n_pos - 1)]))
    pidx = __import__("torch").as_tensor(pos, device="cuda")
    qb = synth.bits(inp["q"][:, pidx])
    kb, vb = synth.bits(inp["k"]), synth.bits(inp["v"])
    Wqb, Wkb = synth.bits(inp["Wq16"]), synth.bits(inp["Wk16"])
    scale = 1.0 / math.sqrt(128)
    nproj = min(L, 16384)
    t0 = time.perf_counter()
    oracle.project(kb[0, :nproj, ret[0] // w.G], Wkb[0])
    t_proj_row = (time.perf_counter() - t0) / nproj
    k16 = np.empty((1, L, len(ret), 16), np.uint16)
    t_k16 = 0.0
    for s, h in enumerate(ret):
        t0 = time.perf_counter()
        k16[0, :, s] = oracle.project(kb[0, :, h // w.G], Wkb[s])[0]
        t_k16 += time.perf_counter() - t0
    c_ret, c_loc, sample_s = [], [], t_k16
    for x, P in enumerate(pos):
        q16 = np.stack([oracle.project(qb[0, x, h][None], Wqb[s])[0][0]
                        for s, h in enumerate(ret)])[None, None]
        rows = np.array([(0, 0, h) for h in ret])
        t0 = time.perf_counter()
        oracle.retrieval_rows(qb[:, x:x + 1], kb, vb, q16, k16, rows, np.arange(len(ret)),
                              np.arange(len(ret)), H=w.H, Hkv=w.Hkv, q_pos0=P,
                              p=float(np.float32(w.p)), scale=scale)
        dt = time.perf_counter() - t0
        sample_s += dt
        c_ret.append(dt / len(ret) / ((P + 1) * math.log2(P + 2)))
        lrows = np.array([(0, 0, h) for h in loc])
        t0 = time.perf_counter()
        oracle.local_rows(qb[:, x:x + 1], kb, vb, lrows, H=w.H, Hkv=w.Hkv, q_pos0=P,
                          window=w.window, n_sink=w.n_sink, scale=scale)
        dt = time.perf_counter() - t0
        sample_s += dt
        c_loc.append(dt / len(loc) / min(P + 1, w.window + w.n_sink))
    Pv = np.arange(L, dtype=np.float64)
    t_ret = float(np.mean(c_ret)) * len(ret) * float(((Pv + 1) * np.log2(Pv + 2)).sum())
    t_loc = float(np.mean(c_loc)) * len(loc) * float(np.minimum(Pv + 1,
                                                                w.window + w.n_sink).sum())
    t_q16 = t_proj_row * L * len(ret)
    total = t_k16 + t_q16 + t_ret + t_loc
    return {"value": L / total, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
            "extrapolated": True, "sample_cpu_s": sample_s,
            "sample": f"{w.name}: k16 projection of all {L} keys x {len(ret)} slots timed; "
                      f"retrieval and local rows timed at positions {pos}, extrapolated to "
                      f"all {L} rows by c*P*log2(P) (retrieval) and c*min(P+1, W+S) (local)",
            "extrapolated_total_s": total}


# ------------------------------------------------------------------ CPU oracle
def oracle_decode_step_time(st_host, n_steps=1):
    """The oracle on one full decode step: q16 projection of the new token, the
    k16 append, top-p + exact attention on every retrieval row, sink+window
    attention on every local row."""
    import numpy as np
    import oracle
    w = st_host["w"]
    qb, kb, vb, Wqb, Wkb, k16o = (st_host[x] for x in ("qb", "kb", "vb", "Wqb", "Wkb", "k16o"))
    B, L = kb.shape[0], kb.shape[1]
    ret, loc = w.retrieval_q_heads(), w.local_q_heads()
    scale = 1.0 / math.sqrt(128)
    t0 = time.perf_counter()
    for _ in range(n_steps):
        q16 = np.zeros((B, 1, len(ret), 16), np.uint16)
        for b in range(B):
            for s, h in enumerate(ret):
                q16[b, 0, s] = oracle.project(qb[b, 0, h][None], Wqb[s])[0][0]
                k16o[b, L - 1, s] = oracle.project(kb[b, L - 1, h // w.G][None], Wkb[s])[0][0]
        rows = np.array([(b, 0, h) for b in range(B) for h in ret])
        slots = np.array([s for b in range(B) for s in range(len(ret))])
        oracle.retrieval_rows(qb, kb, vb, q16, k16o, rows, slots, slots, H=w.H, Hkv=w.Hkv,
                              q_pos0=L - 1, p=float(np.float32(w.p)), scale=scale)
        lrows = np.array([(b, 0, h) for b in range(B) for h in loc])
        oracle.local_rows(qb, kb, vb, lrows, H=w.H, Hkv=w.Hkv, q_pos0=L - 1, window=w.window,
                          n_sink=w.n_sink, scale=scale)
    return (time.perf_counter() - t0) / n_steps


def oracle_host_state(w, device="cpu"):
    import numpy as np
    import oracle
    from long_context_sparse_rtp_b200 import synth
    inp = synth.make_inputs(w, device)
    qb, kb, vb = synth.bits(inp["q"]), synth.bits(inp["k"]), synth.bits(inp["v"])
    Wqb, Wkb = synth.bits(inp["Wq16"]), synth.bits(inp["Wk16"])
    ret = w.retrieval_q_heads()
    B, L = kb.shape[0], kb.shape[1]
    k16o = np.empty((B, L, len(ret), 16), np.uint16)
    for b in range(B):
        for s, h in enumerate(ret):
            k16o[b, :, s] = oracle.project(kb[b, :, h // w.G], Wkb[s])[0]
    return dict(w=w, qb=qb, kb=kb, vb=vb, Wqb=Wqb, Wkb=Wkb, k16o=k16o)


def cpu_cores():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def run_reference(args, world, rank):
    if rank != 0:
        return
    from long_context_sparse_rtp_b200 import synth
    w = synth.WORKLOADS[DECODE_WL]
    st = oracle_host_state(w, "cuda" if _cuda() else "cpu")
    for _ in range(args.warmup):
        oracle_decode_step_time(st, 1)
    t = oracle_decode_step_time(st, args.steps)
    B = st["kb"].shape[0]
    value = B / t
    sample = f"{args.steps} full decode steps ({B} x {w.H_ret} retrieval rows + " \
             f"{B} x {w.H - w.H_ret} local rows each) of {DECODE_WL}"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": DECODE_WL, "global_batch": B, "seq_len": w.L,
                       "parallelism": "cpu-oracle"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def _cuda():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


# ------------------------------------------------------------------ main
def main():
    args = parse()
    if args.case is not None:
        run_case(args)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    import torch
    from long_context_sparse_rtp_b200 import build
    world, rank, local = dist_setup()
    if rank == 0:
        build.build()
    barrier(world)
    pk = peaks()
    dec = bench_decode(args, world, rank, local, pk)
    e2e_ms, h2d, d2h = bench_decode_e2e(dec, args, world)
    shared = bench_decode_shared_k16(dec, args, world)
    variants = ring = None
    if not args.no_variants:
        variants = bench_decode_variants(dec, args, world)
        ring = bench_decode_ring(dec, args, world)
    pres, ex2 = {}, None
    if not args.no_prefill:
        ex2 = measure_ex2_rate()
        for name in PREFILL_SET:
            if name == "prefill_1m" and args.no_1m:
                continue
            pres[name], _ = bench_prefill_config(
                name, args, world, rank, pk, ex2,
                cpu=(rank == 0 and world == 1 and not args.no_cpu_baseline))
    dense = None
    if world == 1:  # a reported baseline: no collective, so one rank only
        try:
            dense = bench_decode_dense(dec, args)
        except Exception as e:  # report, never hide
            dense = {"error": repr(e)}

    B = dec["B"]
    value = B * world / (dec["ms_step"] / 1e3)
    kern = dec["kern"]
    n_launch = sum(n for (n, _) in kern.values()) // args.steps  # our kernels per step
    score_ms = kern["dec_score"][1] / kern["dec_score"][0]
    score_bytes = dec["bytes"]["k16"]
    achieved = score_bytes / (score_ms / 1e3) / 1e9
    step_gbs = dec["bytes"]["total"] / (dec["ms_step"] / 1e3) / 1e9
    traffic = profiled_traffic("dec_score_decode_128k_b8.md")
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dec["ms_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{DECODE_WL}: decode 1 token/seq, batch 8, 131072-token cache, "
                               "32 q / 4 kv heads, 1 retrieval kv head, p=0.95, window 4096+4",
                   "global_batch": B * world, "seq_len": dec["st"]["L"],
                   "parallelism": f"dp{world}",
                   "l2": L2_FLUSH},
        "phase": "decode",
        "roofline": {"bound": "hbm", "kernel": "dec_score", "achieved": achieved,
                     "peak": pk["hbm"], "unit": "GB/s", "frac": achieved / pk["hbm"],
                     "traffic": traffic, "peak_source": pk["src"],
                     "algorithmic_bytes_per_launch": score_bytes},
        "step_roofline": {"bound": "hbm", "algorithmic_bytes": dec["bytes"],
                          "achieved": step_gbs, "frac": step_gbs / pk["hbm"],
                          "frac_of_8tbs": step_gbs / 8000.0},
        "per_kernel_ms": {k_: t / n for k_, (n, t) in kern.items()},
        "timeline_us": dec["timeline"],
        "selection": {"union_keys": dec["union"], "kept_pairs": dec["compute_sel"]},
        "gpu_launches": n_launch * args.steps,
        "clocks": dec["clocks"],
        "e2e": {"value": B * world / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "api": "DecodeGraph.step (pinned host q/k/v in, o out; one graph replay)"},
    }
    line["decode_shared_k16"] = {
        "workload": f"{DECODE_WL} with one k16 per retrieval kv head (k16_per_kv_head = 1)",
        "tokens_per_s": shared["tokens_per_s"], "ms_per_step": shared["ms_step"],
        "k16_bytes_per_step": shared["k16_bytes"]}
    if variants is not None:
        line["decode_variants"] = {
            "workload": f"{DECODE_WL} with block-level top-p (p = 0.95, 64-key blocks, 256 "
                        "bins) or static top-k (k = 4096) on the retrieval heads", **variants}
        line["decode_ring"] = {
            "workload": f"{DECODE_WL} with the local heads on the window-only ring cache",
            **ring}
    if pres:
        line["prefill"] = {
            "ex2_rate_per_s": ex2,
            "note": "per config: the whole mixed layer per p, the dense kernel on every head and "
                    "the summary's own prefill (retrieval heads dense) at the same L; "
                    "attention rooflines on the method's own pairs and on the computed tiles",
            **pres}
    if dense is not None:
        line["dense_decode"] = dense if "error" in dense else {
            "workload": f"{DECODE_WL} with every query head dense over the whole cache "
                        "(rtp_dense_attn, one query row)",
            "ms_per_step": dense["ms_step"], "tokens_per_s": B / (dense["ms_step"] / 1e3),
            "bytes_per_step": dense["bytes"],
            "achieved_gbs": dense["bytes"] / (dense["ms_step"] / 1e3) / 1e9,
            "frac_of_hbm": dense["bytes"] / (dense["ms_step"] / 1e3) / 1e9 / pk["hbm"],
            "sparse_step_speedup": dense["ms_step"] / dec["ms_step"]}
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        try:
            stc = oracle_host_state(dec["st"]["w"], "cuda")
            t = oracle_decode_step_time(stc, 1)
            line["cpu_baseline"] = {"value": B / t, "unit": "tokens/s", "cores": cpu_cores(),
                                    "kind": "oracle",
                                    "sample": f"1 full decode step of {DECODE_WL} "
                                              f"({B} x 8 retrieval + {B} x 24 local rows)"}
        except Exception as e:  # report, never hide
            line["cpu_baseline"] = {"error": repr(e)}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
