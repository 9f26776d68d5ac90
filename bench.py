#!/usr/bin/env python
"""Throughput of the indexer hot path on B200: query-key scores/s and Top-K queries/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline step = one pass of the flat DSA indexer (score, Eq. (1), + per-query Top-K,
Eq. (2)) over the largest single-GPU workload: a 262144-token causal prefill processed in
query chunks of 4096 against the growing key cache (H_I = 64 heads, d = 128, K = 2048, bf16
operands, anchor-structured synthetic data): 64 chunk calls, 3.44e10 (query, key) pairs.
Inputs are resident in HBM before the timed region and larger than L2 (q alone is 4 GiB), so
no L2 flush is needed. `e2e` times the same pass through the host-buffer entry point with the
copies inside the timed region. Under torchrun each rank runs its own replica (weak scaling,
no collective on the data path); the time is the max over ranks.

"rows" times every other workload of the hot path in the same run: the 256K prefill in group
mode and in FP8, the 16K flat prefill (bf16 and FP8), group mode on 64K tokens, decode with an
FP8 key cache, decode bank reuse (cycle and refine-only steps), MTP verification, calibration,
HISA and the group indexer. `cpu_baseline` is the fp64 oracle on the host cores (a thread per
core) on sampled rows of the headline workload; --impl reference times only that.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FLAT = dict(T=16384, H=64, d=128, K=2048, seed=1)
# smaller flat case for ncu captures: its operands (q 128 MiB, scores 256 MiB) still exceed L2
FLAT_SMALL = dict(T=8192, H=64, d=128, K=2048, seed=1)
# long rows for profiler captures of the long-row select: 1024 queries at the end of a
# 65536-token prefix (scores 256 MiB, still larger than L2)
LONG_ROWS = dict(T=1024, S=65536, H=64, d=128, K=2048, seed=1)
GROUP = dict(T=65536, H=64, d=128, K=2048, G=64, B=8192, Hg=16, seed=2)
# the same group mode at a quarter of the length (a profiling case)
GROUP_SMALL = dict(T=16384, H=64, d=128, K=2048, G=64, B=8192, Hg=16, seed=2)
DECODE = dict(Bs=32, S=131072, H=64, d=128, K=2048, Hg=16, B=8192, G=16, seed=3)
CHUNKED = dict(S=262144, chunk=4096, H=64, d=128, K=2048, G=64, B=8192, Hg=16, seed=4)
# rows per chunk of the host-buffer path (copies of one chunk overlap the work on another)
E2E_ROWS_PER_CHUNK = 1024
# HISA at the 64K context of the HISA paper's kernel benchmarks: 128-key blocks, 64 kept
HISA = dict(T=65536, H=64, d=128, K=2048, n_blocks=64, seed=13)
GROUP_INDEXER = dict(T=65536, G=64, d_c=1536, d_h=7168, H_S=16, d=128, seed=12)
# MTP target verification on the decode caches: one window of m draft tokens per sequence
MTP = dict(m=16, G=8, P=8192)


def flat_pairs(T, q_pos0=0):
    return sum(q_pos0 + t + 1 for t in range(T)) if q_pos0 else T * (T + 1) // 2


# ---------------------------------------------------------------------------------------
# infrastructure
# ---------------------------------------------------------------------------------------

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            timeout = datetime.timedelta(seconds=120)
            if torch.cuda.is_available():
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", timeout=timeout,
                                        device_id=torch.device("cuda", self.local))
            else:  # host-only ranks (the oracle arm, or tests without a GPU)
                dist.init_process_group("gloo", timeout=timeout)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x):
        if not self.pg:
            return x
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.3)
            self.proc.terminate()
            self.proc.wait()

    def summary(self):
        self.f.seek(0)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.f.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"],
                    bf16_sustained=p.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def kernel_traffic(name):
    """Per-launch DRAM bytes from the committed ncu summary of a kernel, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{name}.md")
    src = os.path.join(ROOT, "sparse_attention_token_indexer_b200", "csrc", "score_sm100.cu")
    if not os.path.exists(path):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(path):
        if ":" in line and line.startswith("- "):
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha256_16") != h:
        return None
    try:
        return float(vals["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


class StageTimer:
    """CUDA events the library records around its scoring and selection kernels."""

    def __init__(self, lib, steps):
        import ctypes
        self.ctypes, self.lib = ctypes, lib
        self.ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        for evs in self.ev:          # torch creates the CUDA event on its first record
            for e in evs:
                e.record()
        torch.cuda.synchronize()
        self.arr = []
        for evs in self.ev:
            a = (ctypes.c_void_p * 4)(*[e.cuda_event for e in evs])
            self.arr.append(a)

    def arm(self, i):
        self.lib.adx_set_timing_events(self.arr[i], 4)

    def disarm(self):
        self.lib.adx_set_timing_events(None, 0)

    def ms(self, a, b):
        return [evs[a].elapsed_time(evs[b]) for evs in self.ev]


def timed(fn, steps, warmup, dist, stage_timer=None):
    """W untimed steps, then exactly K timed steps between barriers; returns ms per step
    (max over ranks) and the library's launch count inside the timed region. With a stage
    timer, K more steps follow with the library's stage events armed: those events are extra
    stream operations between its kernels, so the timed steps run without them."""
    from sparse_attention_token_indexer_b200 import _lib
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = _lib.lib().adx_launch_count()
    start.record(s)
    for _ in range(steps):
        fn()
    end.record(s)
    torch.cuda.synchronize()
    launches = _lib.lib().adx_launch_count() - n0
    dist.barrier()
    ms = dist.max(start.elapsed_time(end)) / steps
    if stage_timer:
        for i in range(steps):
            stage_timer.arm(i)
            fn()
        stage_timer.disarm()
        torch.cuda.synchronize()
    return ms, launches


def timed_graph(fn, steps, warmup, dist):
    """Like timed(), with the step captured once in a CUDA graph and replayed: for steps of
    many short kernels, where the host's launch rate rather than the GPU bounds the plain
    loop. The launch count is the capture's, once per replayed step."""
    from sparse_attention_token_indexer_b200 import _lib
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    n0 = _lib.lib().adx_launch_count()
    with torch.cuda.graph(g):
        fn()
    per_step = _lib.lib().adx_launch_count() - n0
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s)
    for _ in range(steps):
        g.replay()
    end.record(s)
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(start.elapsed_time(end)) / steps
    del g
    return ms, per_step * steps


# ---------------------------------------------------------------------------------------
# workloads (our CUDA path)
# ---------------------------------------------------------------------------------------

def run_flat(args, dist, dtype="bf16", clocks=None):
    from sparse_attention_token_indexer_b200 import _lib, indexer, inputs
    c = {"flat_small": FLAT_SMALL, "long_rows": LONG_ROWS}.get(args.case, FLAT)
    p = inputs.anchor_prefill(c["T"], c["H"], c["d"], c["K"], seed=c["seed"], device="cuda",
                              dtype=dtype, S=c.get("S"))
    ws = indexer.Workspace("cuda")
    idx = torch.empty(c["T"], c["K"], dtype=torch.int32, device="cuda")

    def step():
        _call_prefill(p, c["K"], idx, ws)

    timer = StageTimer(_lib.lib(), args.steps)
    if clocks is not None:
        with clocks:
            ms, launches = timed(step, args.steps, args.warmup, dist, timer)
    else:
        ms, launches = timed(step, args.steps, args.warmup, dist, timer)
    score_ms = statistics.mean(timer.ms(0, 1))
    select_ms = statistics.mean(timer.ms(2, 3))
    pairs = flat_pairs(c["T"], p["q_pos0"])
    return dict(p=p, ms=ms, launches=launches, score_ms=score_ms, select_ms=select_ms,
                pairs=pairs, flops=pairs * 2 * c["H"] * c["d"], rows=c["T"])


def _call_prefill(p, K, idx, ws):
    import ctypes
    from sparse_attention_token_indexer_b200 import _lib as L, indexer
    ops = indexer.make_operands(p["q"], p["w"], p["k"], p["q_scale"], p["k_scale"], p["q_pos0"])
    buf = ws.get(indexer.workspace_size(L.ADX_OP_PREFILL, ops, K))
    L.check("adx_index_prefill", L.lib().adx_index_prefill(
        ctypes.byref(ops), K, ctypes.c_void_p(idx.data_ptr()), None, None, 0,
        ctypes.c_void_p(buf.data_ptr()), buf.numel(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))


def run_group(args, dist):
    from sparse_attention_token_indexer_b200 import indexer, inputs
    c = GROUP_SMALL if getattr(args, "case", "") == "group_small" else GROUP
    p = inputs.group_prefill(c["T"], c["H"], c["d"], c["K"], c["G"], c["B"], c["Hg"],
                             seed=c["seed"], device="cuda")
    ws = indexer.Workspace("cuda")
    steps = max(2, args.steps // 2)
    from sparse_attention_token_indexer_b200 import _lib
    tb, tr = StageTimer(_lib.lib(), steps), StageTimer(_lib.lib(), steps)

    def step(stage=None):
        # the group queries (mean-pooled by the library), the banks, the refinement
        qbar, wbar = indexer.group_query_mean(p["q"], p["w"], c["G"], c["Hg"])
        if stage is not None:
            tb.arm(stage)
        bank = indexer.group_bank(qbar, wbar, p["k"], c["G"], c["B"], "window", ws=ws)
        if stage is not None:
            tr.arm(stage)
        indexer.bank_refine(p["q"], p["w"], p["k"], bank, c["G"], c["B"], "window", c["K"],
                            ws=ws)
        if stage is not None:
            tr.disarm()

    ms, launches = timed(step, steps, args.warmup, dist)
    for i in range(steps):         # stage breakdown: a second pass with the events armed
        step(i)
    torch.cuda.synchronize()
    stages = {"bank_score_ms": statistics.mean(tb.ms(0, 1)),
              "bank_select_ms": statistics.mean(tb.ms(2, 3)),
              "refine_score_ms": statistics.mean(tr.ms(0, 1)),
              "refine_select_ms": statistics.mean(tr.ms(2, 3))}
    G, B, T = c["G"], c["B"], c["T"]
    scan = sum(g * G for g in range(T // G))
    refine = sum(min(B - G, g * G) * G + G * (G + 1) // 2 for g in range(T // G))
    return dict(ms=ms, launches=launches, scan_pairs=scan, refine_pairs=refine, rows=T,
                flops=scan * 2 * c["Hg"] * c["d"] + refine * 2 * c["H"] * c["d"], stages=stages,
                refine_tflops=refine * 2 * c["H"] * c["d"] / (stages["refine_score_ms"] * 1e-3) / 1e12)


def run_decode(args, dist, cycle=True):
    from sparse_attention_token_indexer_b200 import indexer, inputs
    c = DECODE
    prob = inputs.decode_problem(c["Bs"], c["S"], c["H"], c["d"], c["K"], c["Hg"],
                                 steps=c["G"], seed=c["seed"], device="cuda")
    ws = indexer.Workspace("cuda")
    seq0 = inputs.decode_seq_len(prob, 0)
    q0, w0 = prob["q_steps"][0], prob["w_steps"][0]

    def flat_step():
        indexer.index_decode(q0, w0, prob["k"], seq0, c["K"], k_scale=prob["k_scale"], ws=ws)

    from sparse_attention_token_indexer_b200 import _lib
    td = StageTimer(_lib.lib(), args.steps)
    ms_flat, l_flat = timed(flat_step, args.steps, args.warmup, dist, td)
    dstages = {"score_ms": statistics.mean(td.ms(0, 1)), "select_ms": statistics.mean(td.ms(2, 3))}
    # the same step replayed from a CUDA graph (how a serving loop issues it)
    ms_flat_graph, _ = timed_graph(flat_step, args.steps, args.warmup, dist)
    key_bytes = c["d"] + 4
    if not cycle:
        return dict(ms_flat=ms_flat, launches_flat=l_flat, bytes_flat=c["Bs"] * c["S"] * key_bytes,
                    stages=dstages, ms_flat_graph=ms_flat_graph)
    seqs = [inputs.decode_seq_len(prob, r) for r in range(c["G"])]

    def cycle():
        qb = prob["q_steps"][0][:, : c["Hg"]].contiguous()
        wb = prob["w_steps"][0][:, : c["Hg"]].contiguous()
        bank = indexer.group_bank(qb, wb, prob["k"], c["G"], c["B"], "paper",
                                  k_scale=prob["k_scale"], seq_len=seqs[0], ws=ws)
        for r in range(c["G"]):
            indexer.bank_refine(prob["q_steps"][r], prob["w_steps"][r], prob["k"], bank, c["G"],
                                c["B"], "paper", c["K"], k_scale=prob["k_scale"],
                                seq_len=seqs[r], ws=ws)

    ms_cycle, l_cycle = timed(cycle, max(2, args.steps // 4), args.warmup, dist)
    ms_cycle_graph, _ = timed_graph(cycle, max(2, args.steps // 4), args.warmup, dist)
    key_bytes = c["d"] + 4
    return dict(ms_flat=ms_flat, launches_flat=l_flat, ms_cycle=ms_cycle, launches_cycle=l_cycle,
                ms_cycle_graph=ms_cycle_graph, bytes_flat=c["Bs"] * c["S"] * key_bytes,
                steps_per_cycle=c["G"], stages=dstages, ms_flat_graph=ms_flat_graph)


def run_mtp(args, dist):
    """One verification round: each of the 32 sequences checks m = 16 draft tokens whose
    first one sees 131072 keys. Baseline: the plain indexer for the same 16 queries (16
    decode steps, one query per sequence each)."""
    from sparse_attention_token_indexer_b200 import indexer, inputs
    c, m, G, P = DECODE, MTP["m"], MTP["G"], MTP["P"]
    prob = inputs.decode_problem(c["Bs"], c["S"], c["H"], c["d"], c["K"], c["Hg"], steps=m,
                                 seed=c["seed"], device="cuda")
    ws = indexer.Workspace("cuda")
    k, ks = prob["k"], prob["k_scale"]
    q = prob["q_steps"].transpose(0, 1).reshape(c["Bs"] * m, c["H"], c["d"]).contiguous()
    w = prob["w_steps"].transpose(0, 1).reshape(c["Bs"] * m, c["H"]).contiguous()
    qbar, wbar = inputs.mean_pool_group_queries(q.float(), w, G, c["Hg"])
    qbar = qbar.to(torch.bfloat16).contiguous()
    seq = torch.full((c["Bs"],), c["S"] + m - 1, dtype=torch.int32, device="cuda")
    seqs = [inputs.decode_seq_len(prob, j) for j in range(m)]

    def mtp_round():
        indexer.index_mtp(q, w, k, seq, qbar, wbar, m, G, P, c["K"], k_scale=ks, ws=ws)

    def flat_round():
        for j in range(m):
            indexer.index_decode(prob["q_steps"][j], prob["w_steps"][j], k, seqs[j], c["K"],
                                 k_scale=ks, ws=ws)

    ms_mtp, l_mtp = timed(mtp_round, args.steps, args.warmup, dist)
    ms_flat, l_flat = timed(flat_round, max(2, args.steps // 2), args.warmup, dist)
    n0 = c["S"]                                   # keys the window's first query sees
    scan = c["Bs"] * sum(n0 + g * G for g in range(m // G))
    refine = c["Bs"] * sum(P + (j % G) for j in range(m))
    flat = c["Bs"] * sum(n0 + j for j in range(m))
    return dict(ms=ms_mtp, launches=l_mtp, ms_flat=ms_flat, launches_flat=l_flat, scan=scan,
                refine=refine, flat=flat, rows=c["Bs"] * m)


def run_calibration(args, dist):
    """Union sizes (Eq. (4)) of one layer's calibration Top-K rows for G = 4, 8 and 16: the
    flat prefill's own output at T = 16384, K = 2048."""
    from sparse_attention_token_indexer_b200 import calibration, indexer, inputs
    c = FLAT
    p = inputs.anchor_prefill(c["T"], c["H"], c["d"], c["K"], seed=c["seed"], device="cuda")
    idx, _, _ = indexer.index_prefill(p["q"], p["w"], p["k"], c["K"])
    del p

    def step():
        for G in calibration.GROUP_SIZES:
            calibration.union_sizes(idx, G, c["T"])

    ms, launches = timed(step, args.steps, args.warmup, dist)
    return dict(ms=ms, launches=launches, bytes=3 * idx.numel() * 4)


def run_hisa(args, dist, with_flat=True):
    """HISA prefill over 65536 tokens (block keys, block filter, token refinement), and the
    flat indexer on the same inputs."""
    from sparse_attention_token_indexer_b200 import _lib, indexer, inputs
    c = HISA
    p = inputs.anchor_prefill(c["T"], c["H"], c["d"], c["K"], seed=c["seed"], device="cuda")
    ws = indexer.Workspace("cuda")
    steps = max(2, args.steps // 2)

    def step():
        kbar, _ = indexer.hisa_block_keys(p["q"], p["w"], p["k"])
        indexer.index_hisa(p["q"], p["w"], p["k"], kbar, c["K"], n_blocks=c["n_blocks"], ws=ws)

    th = StageTimer(_lib.lib(), steps)
    ms, launches = timed(step, steps, args.warmup, dist, th)
    # the library's events mark its last score and select launches: the token refinement
    stages = {"refine_score_ms": statistics.mean(th.ms(0, 1)),
              "final_select_ms": statistics.mean(th.ms(2, 3))}
    T, nbk, B = c["T"], c["n_blocks"], 128
    blk_pairs = sum(t // B + 1 for t in range(T))
    tok_pairs = sum(min(nbk, t // B + 1) * B for t in range(T))
    out = dict(ms=ms, launches=launches, stages=stages, blk_pairs=blk_pairs, tok_pairs=tok_pairs,
               flops=2 * c["H"] * c["d"] * (blk_pairs + tok_pairs), rows=T)
    if with_flat:
        def flat():
            indexer.index_prefill(p["q"], p["w"], p["k"], c["K"], ws=ws)
        out["ms_flat"], _ = timed(flat, max(2, steps // 2), args.warmup, dist)
    return out


def run_hisa_decode(args, dist):
    """HISA decode step for 32 sequences of 131072 e4m3 keys: the last block key of every
    cache refreshed, the block filter, the token refinement (the block keys of the rest of
    the cache are built once, like the cache itself)."""
    from sparse_attention_token_indexer_b200 import indexer, inputs
    c = DECODE
    prob = inputs.decode_problem(c["Bs"], c["S"], c["H"], c["d"], c["K"], c["Hg"], steps=1,
                                 seed=c["seed"], device="cuda")
    ws = indexer.Workspace("cuda")
    seq0 = inputs.decode_seq_len(prob, 0)
    q0, w0, k, ks = prob["q_steps"][0], prob["w_steps"][0], prob["k"], prob["k_scale"]
    kbar, _ = indexer.hisa_block_keys(q0, w0, k, k_scale=ks, seq_len=seq0)

    def step():
        indexer.hisa_block_keys(q0, w0, k, k_scale=ks, seq_len=seq0, last_only=True,
                                out=(kbar, None))
        indexer.index_hisa(q0, w0, k, kbar, c["K"], n_blocks=HISA["n_blocks"], k_scale=ks,
                           seq_len=seq0, ws=ws)

    ms, launches = timed(step, args.steps, args.warmup, dist)
    ms_graph, _ = timed_graph(step, args.steps, args.warmup, dist)
    nb = (c["S"] + 127) // 128
    key_bytes = c["d"] + 4
    # the kept blocks' keys, the bf16 block keys and the refreshed last block's keys
    bytes_step = c["Bs"] * ((HISA["n_blocks"] * 128 + 128) * key_bytes + nb * c["d"] * 2)
    return dict(ms=ms, ms_graph=ms_graph, launches=launches, bytes=bytes_step)


def run_group_indexer(args, dist):
    """The trained group indexer's queries and gates (Eqs. (6)-(7)) for a 65536-token prefill
    with G = 64: d_c = 1536 query latents, d_h = 7168 hidden states, H_S = 16 heads of d = 128,
    synthetic weights. One step reads both activations once (1.14 GB, above L2)."""
    from sparse_attention_token_indexer_b200 import indexer, inputs
    c = GROUP_INDEXER
    p = inputs.group_indexer_problem(c["T"], c["d_c"], c["d_h"], c["H_S"], c["d"], seed=c["seed"],
                                     device="cuda")
    ws = indexer.Workspace("cuda")

    def step():
        indexer.group_indexer_queries(p["cq"], p["h"], p["w_pool"], p["w_q"], p["w_g"], c["G"],
                                      c["H_S"], c["d"], ws=ws)

    ms, launches = timed(step, args.steps, args.warmup, dist)
    ng = c["T"] // c["G"]
    flops = 2 * ng * (c["d_c"] * 3 * c["d_c"] + c["H_S"] * c["d"] * c["d_c"] + c["H_S"] * c["d_h"])
    act = c["T"] * (c["d_c"] + c["d_h"]) * 2
    return dict(ms=ms, launches=launches, groups=ng, act_bytes=act, flops=flops)


def chunked_inputs(dtype="bf16"):
    """The 256K chunked-prefill workload: q [S, 64, 128], w, k [S, 128] on the device (bf16,
    or e4m3 codes with per-token scales), and the group queries of every G = 64 tokens."""
    from sparse_attention_token_indexer_b200 import inputs
    c = CHUNKED
    S, G = c["S"], c["G"]
    st = inputs.AnchorStructure(c["d"], c["seed"], "cuda")
    kf = st.keys(S)
    q = torch.empty(S, c["H"], c["d"], dtype=torch.bfloat16, device="cuda")
    for c0 in range(0, S, 16384):  # generate in slices to bound the fp32 temporaries
        q[c0:c0 + 16384] = st.queries(16384, c["H"], pos0=c0).to(torch.bfloat16)
    w = st.gates(S, c["H"])
    qbar, wbar = inputs.mean_pool_group_queries(q, w, G, c["Hg"])
    qs = ks = qbs = None
    if dtype == "e4m3":
        k, ks = inputs.quantize_e4m3_rows(kf)
        qc = torch.empty(S, c["H"], c["d"], dtype=torch.uint8, device="cuda")
        qs = torch.empty(S, dtype=torch.float32, device="cuda")
        for c0 in range(0, S, 16384):
            qc[c0:c0 + 16384], qs[c0:c0 + 16384] = inputs.quantize_e4m3_rows(q[c0:c0 + 16384])
        q = qc
        qbar, qbs = inputs.quantize_e4m3_rows(qbar)
    else:
        k = kf.to(torch.bfloat16).contiguous()
        qbar = qbar.to(torch.bfloat16).contiguous()
    del kf
    return dict(q=q, w=w, k=k, q_scale=qs, k_scale=ks, qbar=qbar, wbar=wbar, qbar_scale=qbs,
                dtype=dtype)


def chunked_flat_pass(inp, ws, idx, timers=None):
    """One 256K prefill in query chunks of 4096, flat indexer; timers: one StageTimer slot per
    chunk (the library's events around each chunk's scoring and selection kernels)."""
    c = CHUNKED
    S, ch = c["S"], c["chunk"]
    q, w, k, qs, ks = inp["q"], inp["w"], inp["k"], inp["q_scale"], inp["k_scale"]
    for j, c0 in enumerate(range(0, S, ch)):
        if timers is not None:
            timers.arm(j)
        _call_prefill({"q": q[c0:c0 + ch], "w": w[c0:c0 + ch], "k": k,
                       "q_scale": None if qs is None else qs[c0:c0 + ch], "k_scale": ks,
                       "q_pos0": c0}, c["K"], idx, ws)
    if timers is not None:
        timers.disarm()


def chunked_group_pass(inp, ws):
    """One 256K prefill in query chunks of 4096, ADIndex group mode (WINDOW bank, G = 64,
    B = 8192): per chunk the group banks, then every query's refinement."""
    from sparse_attention_token_indexer_b200 import indexer
    c = CHUNKED
    S, ch, G = c["S"], c["chunk"], c["G"]
    gpc = ch // G
    q, w, k, qs, ks = inp["q"], inp["w"], inp["k"], inp["q_scale"], inp["k_scale"]
    qbar, wbar, qbs = inp["qbar"], inp["wbar"], inp["qbar_scale"]
    for c0 in range(0, S, ch):
        g0 = c0 // G
        bank = indexer.group_bank(qbar[g0:g0 + gpc], wbar[g0:g0 + gpc], k, G, c["B"], "window",
                                  qbar_scale=None if qbs is None else qbs[g0:g0 + gpc],
                                  k_scale=ks, q_pos0=c0, ws=ws)
        indexer.bank_refine(q[c0:c0 + ch], w[c0:c0 + ch], k, bank, G, c["B"], "window", c["K"],
                            q_scale=None if qs is None else qs[c0:c0 + ch], k_scale=ks,
                            q_pos0=c0, ws=ws)


def chunked_counts():
    c = CHUNKED
    S, G, B = c["S"], c["G"], c["B"]
    pairs = S * (S + 1) // 2
    scan = sum(g * G for g in range(S // G))
    refine = sum(min(B - G, g * G) * G + G * (G + 1) // 2 for g in range(S // G))
    return pairs, scan, refine


def run_chunked_flat(args, dist, inp, steps, clocks=None):
    """Times `steps` flat 256K passes, then one more pass with the per-chunk stage events
    armed; returns ms per pass, launches, and the summed scoring / selection kernel time of a
    pass."""
    from sparse_attention_token_indexer_b200 import _lib, indexer
    c = CHUNKED
    ws = indexer.Workspace("cuda")
    idx = torch.empty(c["chunk"], c["K"], dtype=torch.int32, device="cuda")
    n_chunks = c["S"] // c["chunk"]

    def step():
        chunked_flat_pass(inp, ws, idx)

    if clocks is not None:
        with clocks:
            ms, launches = timed(step, steps, args.warmup, dist)
    else:
        ms, launches = timed(step, steps, args.warmup, dist)
    timer = StageTimer(_lib.lib(), n_chunks)
    chunked_flat_pass(inp, ws, idx, timer)
    torch.cuda.synchronize()
    score_ms = sum(timer.ms(0, 1))
    select_ms = sum(timer.ms(2, 3))
    del ws
    return dict(ms=ms, launches=launches, score_ms=score_ms, select_ms=select_ms)


def run_chunked_group(args, dist, inp, steps):
    from sparse_attention_token_indexer_b200 import indexer
    ws = indexer.Workspace("cuda")

    def step():
        chunked_group_pass(inp, ws)

    ms, launches = timed(step, steps, args.warmup, dist)
    del ws
    return dict(ms=ms, launches=launches)


def run_chunked_e2e(args, dist, inp, steps):
    """The flat 256K prefill through the public host-buffer entry point (adx_index_prefill_host):
    the operands start in pinned host memory, chunks of 4096 rows are indexed longest first
    while the next chunk's queries and gates are copied in and the previous chunk's Top-K rows
    are copied out; every copy is inside the timed region."""
    from sparse_attention_token_indexer_b200 import indexer
    c = CHUNKED
    host = {n: inp[n].cpu().pin_memory() for n in ("q", "w", "k")}
    for n in ("q_scale", "k_scale"):
        host[n] = None if inp[n] is None else inp[n].cpu().pin_memory()
    out_h = torch.empty(c["S"], c["K"], dtype=torch.int32).pin_memory()
    ws = indexer.Workspace("cuda")

    def step():
        indexer.index_prefill_host(host["q"], host["w"], host["k"], c["K"], host["q_scale"],
                                   host["k_scale"], rows_per_chunk=c["chunk"], out=(out_h, None),
                                   ws=ws)

    ms, _ = timed(step, steps, args.warmup, dist)
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    d2h = out_h.numel() * out_h.element_size()
    del ws, host, out_h
    return ms, h2d, d2h


def run_decode_refine(args, dist):
    """Decode with bank reuse (the decode workload's variant): the refine-only steps between
    two refreshes, each over the bank of B = 8192 positions plus the keys appended since the
    refresh; one step = the refinement of all 32 sequences at one decode position. Timed two
    ways: the candidate keys gathered from the cache every step (tile::gather4), and the bank's
    keys packed once at the refresh and streamed (adx_pack_bank_keys, timed apart)."""
    from sparse_attention_token_indexer_b200 import indexer, inputs
    c = DECODE
    prob = inputs.decode_problem(c["Bs"], c["S"], c["H"], c["d"], c["K"], c["Hg"],
                                 steps=c["G"], seed=c["seed"], device="cuda")
    ws = indexer.Workspace("cuda")
    seqs = [inputs.decode_seq_len(prob, r) for r in range(c["G"])]
    qb = prob["q_steps"][0][:, : c["Hg"]].contiguous()
    wb = prob["w_steps"][0][:, : c["Hg"]].contiguous()
    bank = indexer.group_bank(qb, wb, prob["k"], c["G"], c["B"], "paper",
                              k_scale=prob["k_scale"], seq_len=seqs[0], ws=ws)
    r_mid = c["G"] // 2
    q, w, k, ks = prob["q_steps"][r_mid], prob["w_steps"][r_mid], prob["k"], prob["k_scale"]

    def refine():
        indexer.bank_refine(q, w, k, bank, c["G"], c["B"], "paper", c["K"], k_scale=ks,
                            seq_len=seqs[r_mid], ws=ws)

    packed = indexer.pack_bank_keys(q, w, k, bank, c["G"], c["B"], k_scale=ks, seq_len=seqs[0])

    def pack():
        indexer.pack_bank_keys(q, w, k, bank, c["G"], c["B"], k_scale=ks, seq_len=seqs[0],
                               out=packed)

    def refine_packed():
        indexer.bank_refine_packed(q, w, k, bank, packed[0], packed[1], c["G"], c["B"], c["K"],
                                   k_scale=ks, seq_len=seqs[r_mid], ws=ws)

    ms, launches = timed(refine, args.steps, args.warmup, dist)
    ms_graph, _ = timed_graph(refine, args.steps, args.warmup, dist)
    ms_p, launches_p = timed(refine_packed, args.steps, args.warmup, dist)
    ms_p_graph, _ = timed_graph(refine_packed, args.steps, args.warmup, dist)
    ms_pack, _ = timed(pack, args.steps, args.warmup, dist)
    # keys the step reads: the bank entries at or before the position plus the new keys
    keys = c["Bs"] * (c["B"] + r_mid)
    del prob, ws, packed
    return dict(ms=ms, ms_graph=ms_graph, launches=launches, ms_packed=ms_p,
                ms_packed_graph=ms_p_graph, launches_packed=launches_p, ms_pack=ms_pack,
                bytes=keys * (c["d"] + 4), rows=c["Bs"])


# ---------------------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------------------

def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def affinity_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleBaseline:
    """The fp64 oracle (as it stands) on the host cores: one query row per task on a thread
    pool with one thread per affinity core and one BLAS thread per call (numpy releases the
    interpreter lock inside its matrix products, maxima and sorts), on a stratified sample of
    the chunked prefill's query rows: the first and last positions, the rows around K, and
    positions drawn uniformly; scores/s = pairs scored / wall time."""

    def __init__(self, q, w, k, K, n_rows, seed=0, pos=None):
        """q, w: the workload's query rows and gates (all rows, or with `pos` given, just the
        rows sampled at those positions); k: its keys."""
        from concurrent.futures import ThreadPoolExecutor

        from threadpoolctl import threadpool_limits

        from oracle import fp_formats
        S = k.shape[0]
        if pos is None:
            rng = np.random.default_rng(seed)
            fixed = [0, 1, K - 1, K, K + 1, S - 2, S - 1]
            pos = np.array(fixed + rng.integers(0, S, max(0, n_rows - len(fixed))).tolist(),
                           dtype=np.int64)
            sel = torch.as_tensor(pos, device=q.device)
            q, w = q[sel], w[sel]

        def bits(t):
            return t.cpu().view(torch.int16).numpy().view(np.uint16)

        self.pos = np.asarray(pos, dtype=np.int64)
        self.k = fp_formats.bf16_bits_to_f64(bits(k))
        self.q = fp_formats.bf16_bits_to_f64(bits(q))
        self.w = w.cpu().double().numpy()
        self.K = K
        self.cores = affinity_cores()
        self.limits = threadpool_limits(1)
        self.pool = ThreadPoolExecutor(self.cores)

    def _row(self, j):
        from oracle import indexer as ox
        j %= len(self.pos)
        p = int(self.pos[j])
        ox.flat_topk_row(self.q[j], self.w[j], self.k, p, self.K)
        return p + 1

    def run(self, rows):
        """Scores the sampled rows with these indices; returns (pairs, rows, wall seconds)."""
        t0 = time.perf_counter()
        pairs = sum(self.pool.map(self._row, list(rows)))
        return pairs, len(rows), time.perf_counter() - t0

    def run_for(self, seconds, start=0):
        """Rows start, start+1, ... until about `seconds` of wall time: one batch of one row per
        thread first, to measure the row cost, then the rest in one go."""
        rows = list(range(start, start + self.cores))
        pairs, n, wall = self.run(rows)
        per_batch = max(wall, 1e-3)
        more = int(max(0.0, seconds - wall) / per_batch) * self.cores
        nxt = start + self.cores
        rows2 = list(range(nxt, nxt + more))
        if rows2:
            p2, n2, w2 = self.run(rows2)
            pairs, n, wall = pairs + p2, n + n2, wall + w2
        return pairs, n, wall, nxt + len(rows2)

    def close(self):
        self.pool.shutdown()
        self.limits.unregister()


# ---------------------------------------------------------------------------------------

def reference_arm(args, dist):
    """--impl reference: the fp64 oracle as it stands, on the host cores, on the headline's
    workload (the 256K chunked flat prefill), rank 0 only; each step a bounded sample of rows."""
    if dist.rank != 0:
        dist.close()
        return
    c = CHUNKED
    if torch.cuda.is_available():
        torch.cuda.set_device(dist.local)
        inp = chunked_inputs("bf16")      # the very operands the CUDA arm indexes
        ob = OracleBaseline(inp["q"], inp["w"], inp["k"], c["K"], 8192)
        del inp
        torch.cuda.empty_cache()
        where = "drawn on the GPU, the CUDA arm's operands"
    else:
        # no device: the same generator on the host (same shapes and distribution, other
        # values); query rows do not depend on their position, so only the sample is drawn
        from sparse_attention_token_indexer_b200 import inputs
        st = inputs.AnchorStructure(c["d"], c["seed"], "cpu")
        k = st.keys(c["S"]).to(torch.bfloat16)
        n = 4 * affinity_cores()
        rng = np.random.default_rng(0)
        pos = np.array([0, c["K"], c["S"] - 1] + rng.integers(0, c["S"], n - 3).tolist())
        ob = OracleBaseline(st.queries(n, c["H"]).to(torch.bfloat16), st.gates(n, c["H"]), k,
                            c["K"], n, pos=pos)
        where = "drawn on the host"
    per_step = min(10.0, max(0.5, args.cpu_seconds / max(1, args.steps)))
    start = 0
    for _ in range(args.warmup):
        _, _, _, start = ob.run_for(0.1, start)
    tot_pairs = tot_rows = 0
    tot_s = 0.0
    for _ in range(args.steps):
        pr, rw, wall, start = ob.run_for(per_step, start)
        tot_pairs, tot_rows, tot_s = tot_pairs + pr, tot_rows + rw, tot_s + wall
    ob.close()
    value = tot_pairs / tot_s
    sample = (f"{tot_rows} query rows of the 262144-token chunked prefill (first and last "
              f"positions, around K, uniform positions; inputs {where}), {tot_s:.1f} s wall "
              f"on {ob.cores} threads ({cpu_model()})")
    line = {"impl": "reference", "metric": "indexer query-key scores/s", "value": value,
            "unit": "scores/s", "n_gpus": dist.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (anchor-structured, seeded)",
            "config": headline_config(dist),
            "topk_queries_per_s": tot_rows / tot_s,
            "cpu_baseline": {"value": value, "unit": "scores/s", "cores": ob.cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "scores/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    dist.close()


def headline_config(dist):
    c = CHUNKED
    return {"workload": "chunked_prefill_flat_S262144_chunk4096_H64_d128_K2048_bf16",
            "S": c["S"], "chunk": c["chunk"], "H_I": c["H"], "d": c["d"], "K": c["K"],
            "seq_len": c["S"], "global_batch": dist.world,
            "parallelism": f"replicas{dist.world}",
            "l2": "inputs larger than L2 (q 4 GiB; per-chunk scores up to 4 GiB)"}


def quick_case(args, dist):
    """--quick: one workload's kernels only (no e2e, rows or CPU baseline), for profiling."""
    out = {"case": args.case}
    if args.case == "decode":
        dcd = run_decode(args, dist, cycle=False)
        out.update(ms_per_step=dcd["ms_flat"], stage_ms=dcd["stages"],
                   hbm_gbs=dcd["bytes_flat"] / (dcd["ms_flat"] * 1e-3) / 1e9,
                   graph_ms_per_step=dcd["ms_flat_graph"], gpu_launches=dcd["launches_flat"])
    elif args.case == "decode_refine":
        dr = run_decode_refine(args, dist)
        out.update(ms_per_step=dr["ms"], graph_ms_per_step=dr["ms_graph"],
                   packed_ms_per_step=dr["ms_packed"],
                   packed_graph_ms_per_step=dr["ms_packed_graph"], pack_ms=dr["ms_pack"],
                   hbm_gbs=dr["bytes"] / (dr["ms"] * 1e-3) / 1e9,
                   packed_hbm_gbs=dr["bytes"] / (dr["ms_packed"] * 1e-3) / 1e9,
                   gpu_launches=dr["launches"])
    elif args.case == "chunked":
        inp = chunked_inputs(args.dtype)
        fl = run_chunked_flat(args, dist, inp, args.steps)
        gr = run_chunked_group(args, dist, inp, args.steps)
        out.update(dtype=args.dtype, flat_ms=fl["ms"], score_ms=fl["score_ms"],
                   select_ms=fl["select_ms"], group_ms=gr["ms"])
    elif args.case == "decode_cycle":
        dcd = run_decode(args, dist)
        n = dcd["steps_per_cycle"]
        out.update(ms_per_step=dcd["ms_cycle"] / n, graph_ms_per_step=dcd["ms_cycle_graph"] / n,
                   gpu_launches=dcd["launches_cycle"])
    elif args.case == "mtp":
        mt = run_mtp(args, dist)
        out.update(ms_per_round=mt["ms"], flat_ms_per_round=mt["ms_flat"],
                   speedup_vs_flat=mt["ms_flat"] / mt["ms"], gpu_launches=mt["launches"])
    elif args.case in ("hisa", "hisa_small"):
        if args.case == "hisa_small":
            HISA["T"] = 16384
        hs = run_hisa(args, dist, with_flat=False)
        out.update(T=HISA["T"], ms_per_step=hs["ms"], stage_ms=hs["stages"],
                   gpu_launches=hs["launches"])
    elif args.case == "hisa_decode":
        hd = run_hisa_decode(args, dist)
        out.update(ms_per_step=hd["ms"], graph_ms_per_step=hd["ms_graph"],
                   gpu_launches=hd["launches"])
    elif args.case == "group_indexer":
        gi = run_group_indexer(args, dist)
        out.update(ms_per_step=gi["ms"], activation_gbs=gi["act_bytes"] / (gi["ms"] * 1e-3) / 1e9,
                   gpu_launches=gi["launches"])
    elif args.case in ("group", "group_small"):
        g = run_group(args, dist)
        out.update(ms_per_step=g["ms"], stage_ms=g["stages"],
                   refine_score_tflops=g["refine_tflops"], gpu_launches=g["launches"])
    else:  # flat / flat_small
        clocks = Clocks(dist.local)
        flat = run_flat(args, dist, args.dtype, clocks)
        out.update(dtype=args.dtype, ms_per_step=flat["ms"], score_ms=flat["score_ms"],
                   select_ms=flat["select_ms"],
                   score_tflops=flat["flops"] / flat["score_ms"] / 1e9,
                   gpu_launches=flat["launches"], clocks=clocks.summary())
    if dist.rank == 0:
        print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--case", default="all",
                    choices=["all", "flat", "flat_small", "long_rows", "chunked", "group",
                             "group_small", "decode",
                             "decode_refine", "decode_cycle", "mtp", "group_indexer", "hisa",
                             "hisa_small", "hisa_decode"],
                    help="all (default): the headline and every row; the others time one "
                         "workload's kernels alone (with --quick), for profiling")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "e4m3"])
    ap.add_argument("--quick", action="store_true",
                    help="with --case: time that workload's kernels only")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    dist = Dist()
    if args.impl == "reference":
        reference_arm(args, dist)
        return
    torch.cuda.set_device(dist.local)
    from sparse_attention_token_indexer_b200 import build
    build.build()
    if args.case != "all" or args.quick:
        quick_case(args, dist)
        dist.close()
        return

    pk = peaks()
    clocks = Clocks(dist.local)
    row_steps = max(2, args.steps // 5)
    n_chunks = CHUNKED["S"] // CHUNKED["chunk"]

    # ---- headline: the 256K chunked prefill, flat indexer, bf16 ---------------------------
    inp = chunked_inputs("bf16")
    fl = run_chunked_flat(args, dist, inp, args.steps, clocks)
    clk = clocks.summary()
    pairs, scan, refine = chunked_counts()
    flops = pairs * 2 * CHUNKED["H"] * CHUNKED["d"]
    score_tflops = flops / (fl["score_ms"] * 1e-3) / 1e12
    peak_s = pk["bf16_sustained"] or pk["bf16"]
    line = {
        "metric": "indexer query-key scores/s", "value": dist.world * pairs / (fl["ms"] * 1e-3),
        "unit": "scores/s", "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": fl["ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (anchor-structured, seeded)",
        "config": headline_config(dist),
        "topk_queries_per_s": dist.world * CHUNKED["S"] / (fl["ms"] * 1e-3),
        "stage_ms": {"score": fl["score_ms"], "select": fl["select_ms"]},
        "roofline": {"kernel": "score_kernel (tcgen05, bf16), 64 launches per step",
                     "bound": "tensor", "achieved": score_tflops, "peak": peak_s,
                     "unit": "TFLOP/s", "frac": score_tflops / peak_s,
                     "peak_source": f"{pk['source']} bf16 sustained (a kernel inside a long step)",
                     "traffic": kernel_traffic("score_kernel_chunked_prefill_S262144_bf16")},
        "gpu_launches": fl["launches"],
        "clocks": clk,
    }
    e2e_ms, h2d, d2h = run_chunked_e2e(args, dist, inp, args.steps)
    line["e2e"] = {"value": dist.world * pairs / (e2e_ms * 1e-3), "unit": "scores/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
    rows = {}
    gr = run_chunked_group(args, dist, inp, row_steps)
    rows["chunked_prefill_S262144_group_bf16"] = {
        "ms_per_pass": gr["ms"], "scores_per_s": (scan + refine) / (gr["ms"] * 1e-3),
        "topk_queries_per_s": CHUNKED["S"] / (gr["ms"] * 1e-3),
        "speedup_vs_flat": fl["ms"] / gr["ms"], "gpu_launches": gr["launches"]}
    ob = None
    if dist.rank == 0 and dist.world == 1:
        ob = OracleBaseline(inp["q"], inp["w"], inp["k"], CHUNKED["K"], 8192)
    del inp
    torch.cuda.empty_cache()
    inp8 = chunked_inputs("e4m3")
    f8 = run_chunked_flat(args, dist, inp8, row_steps)
    g8 = run_chunked_group(args, dist, inp8, row_steps)
    t8 = flops / (f8["score_ms"] * 1e-3) / 1e12
    rows["chunked_prefill_S262144_e4m3"] = {
        "flat_ms_per_pass": f8["ms"], "flat_scores_per_s": pairs / (f8["ms"] * 1e-3),
        "flat_stage_ms": {"score": f8["score_ms"], "select": f8["select_ms"]},
        "score_tflops": t8, "score_frac_e4m3_peak": t8 / (2 * peak_s),
        "group_ms_per_pass": g8["ms"], "group_speedup_vs_flat": f8["ms"] / g8["ms"],
        "peak_source": f"{pk['source']} bf16 sustained x 2 (e4m3 dense rate)",
        "gpu_launches": f8["launches"] + g8["launches"]}
    del inp8
    torch.cuda.empty_cache()

    # ---- the other workloads -------------------------------------------------------------
    for dt in ("bf16", "e4m3"):
        args.case = "flat"
        f = run_flat(args, dist, dt)
        f.pop("p")
        tf = f["flops"] / (f["score_ms"] * 1e-3) / 1e12
        pkf = pk["bf16"] * (2 if dt == "e4m3" else 1)
        rows[f"flat_prefill_T16384_{dt}"] = {
            "ms_per_step": f["ms"], "scores_per_s": f["pairs"] / (f["ms"] * 1e-3),
            "topk_queries_per_s": f["rows"] / (f["ms"] * 1e-3),
            "stage_ms": {"score": f["score_ms"], "select": f["select_ms"]},
            "score_tflops": tf, "score_frac": tf / pkf,
            "step_frac": f["flops"] / (f["ms"] * 1e-3) / 1e12 / pkf,
            "peak_tflops": pkf,
            "peak_source": f"{pk['source']} bf16 burst" + (" x 2" if dt == "e4m3" else ""),
            "gpu_launches": f["launches"]}
    args.case = "all"
    g = run_group(args, dist)
    rows["group_mode_T65536"] = {
        "ms_per_step": g["ms"], "scan_pairs": g["scan_pairs"], "refine_pairs": g["refine_pairs"],
        "scores_per_s": (g["scan_pairs"] + g["refine_pairs"]) / (g["ms"] * 1e-3),
        "topk_queries_per_s": g["rows"] / (g["ms"] * 1e-3), "stage_ms": g["stages"],
        "refine_score_tflops": g["refine_tflops"],
        "refine_score_frac": g["refine_tflops"] / pk["bf16"], "gpu_launches": g["launches"]}
    dcd = run_decode(args, dist)
    rows["decode_Bs32_S131072_e4m3"] = {
        "ms_per_step": dcd["ms_flat"],
        "scores_per_s": DECODE["Bs"] * DECODE["S"] / (dcd["ms_flat"] * 1e-3),
        "topk_queries_per_s": DECODE["Bs"] / (dcd["ms_flat"] * 1e-3),
        "hbm_gbs": dcd["bytes_flat"] / (dcd["ms_flat"] * 1e-3) / 1e9,
        "hbm_frac": dcd["bytes_flat"] / (dcd["ms_flat"] * 1e-3) / 1e9 / pk["hbm"],
        "score_kernel_hbm_frac": dcd["bytes_flat"] / (dcd["stages"]["score_ms"] * 1e-3) / 1e9
        / pk["hbm"], "stage_ms": dcd["stages"],
        "graph_ms_per_step": dcd["ms_flat_graph"],
        "graph_hbm_frac": dcd["bytes_flat"] / (dcd["ms_flat_graph"] * 1e-3) / 1e9 / pk["hbm"],
        "gpu_launches": dcd["launches_flat"]}
    rows["decode_bank_reuse_cycle16"] = {
        "ms_per_cycle": dcd["ms_cycle"],
        "ms_per_step": dcd["ms_cycle"] / dcd["steps_per_cycle"],
        "graph_ms_per_step": dcd["ms_cycle_graph"] / dcd["steps_per_cycle"],
        "topk_queries_per_s": DECODE["Bs"] * dcd["steps_per_cycle"] / (dcd["ms_cycle"] * 1e-3),
        "gpu_launches": dcd["launches_cycle"]}
    dr = run_decode_refine(args, dist)
    rows["decode_refine_step_Bs32_B8192_e4m3"] = {
        "ms_per_step": dr["ms_packed"], "graph_ms_per_step": dr["ms_packed_graph"],
        "bytes_per_step": dr["bytes"],
        "hbm_gbs": dr["bytes"] / (dr["ms_packed"] * 1e-3) / 1e9,
        "hbm_frac": dr["bytes"] / (dr["ms_packed"] * 1e-3) / 1e9 / pk["hbm"],
        "graph_hbm_frac": dr["bytes"] / (dr["ms_packed_graph"] * 1e-3) / 1e9 / pk["hbm"],
        "pack_ms_per_refresh": dr["ms_pack"],
        "gather_path": {"ms_per_step": dr["ms"], "graph_ms_per_step": dr["ms_graph"],
                        "hbm_frac": dr["bytes"] / (dr["ms"] * 1e-3) / 1e9 / pk["hbm"]},
        "topk_queries_per_s": dr["rows"] / (dr["ms_packed"] * 1e-3),
        "gpu_launches": dr["launches_packed"]}
    mt = run_mtp(args, dist)
    rows[f"mtp_round_Bs32_N131072_m{MTP['m']}_G{MTP['G']}_P{MTP['P']}"] = {
        "ms_per_round": mt["ms"], "scan_pairs": mt["scan"], "refine_pairs": mt["refine"],
        "scores_per_s": (mt["scan"] + mt["refine"]) / (mt["ms"] * 1e-3),
        "topk_queries_per_s": mt["rows"] / (mt["ms"] * 1e-3), "flat_ms_per_round": mt["ms_flat"],
        "speedup_vs_flat": mt["ms_flat"] / mt["ms"],
        "score_count_ratio": mt["flat"] / (mt["scan"] + mt["refine"]), "gpu_launches": mt["launches"]}
    cb = run_calibration(args, dist)
    rows["calibration_union_sizes_T16384_K2048"] = {
        "ms_per_layer": cb["ms"], "group_sizes": [4, 8, 16],
        "gbs_read": cb["bytes"] / (cb["ms"] * 1e-3) / 1e9,
        "hbm_frac": cb["bytes"] / (cb["ms"] * 1e-3) / 1e9 / pk["hbm"], "gpu_launches": cb["launches"]}
    hs = run_hisa(args, dist)
    rows["hisa_prefill_T65536_nb64"] = {
        "ms_per_step": hs["ms"], "flat_ms_per_step": hs["ms_flat"],
        "speedup_vs_flat": hs["ms_flat"] / hs["ms"],
        "scores_per_s": (hs["blk_pairs"] + hs["tok_pairs"]) / (hs["ms"] * 1e-3),
        "topk_queries_per_s": hs["rows"] / (hs["ms"] * 1e-3), "stage_ms": hs["stages"],
        "refine_score_tflops": 2 * HISA["H"] * HISA["d"] * hs["tok_pairs"]
        / (hs["stages"]["refine_score_ms"] * 1e-3) / 1e12, "gpu_launches": hs["launches"]}
    hd = run_hisa_decode(args, dist)
    rows["hisa_decode_Bs32_S131072_e4m3_nb64"] = {
        "ms_per_step": hd["ms"], "graph_ms_per_step": hd["ms_graph"],
        "flat_ms_per_step": dcd["ms_flat"], "speedup_vs_flat": dcd["ms_flat"] / hd["ms"],
        "topk_queries_per_s": DECODE["Bs"] / (hd["ms"] * 1e-3),
        "hbm_gbs": hd["bytes"] / (hd["ms"] * 1e-3) / 1e9, "gpu_launches": hd["launches"]}
    gi = run_group_indexer(args, dist)
    rows["group_indexer_queries_T65536_G64"] = {
        "ms_per_step": gi["ms"], "groups_per_s": gi["groups"] / (gi["ms"] * 1e-3),
        "activation_gbs": gi["act_bytes"] / (gi["ms"] * 1e-3) / 1e9,
        "hbm_frac": gi["act_bytes"] / (gi["ms"] * 1e-3) / 1e9 / pk["hbm"],
        "projection_gflop": gi["flops"] / 1e9, "gpu_launches": gi["launches"]}
    line["rows"] = rows
    if ob is not None:
        pr, rw, wall, _ = ob.run_for(args.cpu_seconds)
        ob.close()
        line["cpu_baseline"] = {
            "value": pr / wall, "unit": "scores/s", "cores": ob.cores, "kind": "oracle",
            "sample": f"{rw} query rows of the same 262144-token workload (first and last "
                      f"positions, around K, uniform positions), {wall:.1f} s wall on "
                      f"{ob.cores} threads ({cpu_model()})"}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
