"""Wave-index sparse decode benchmark (one decode step of one layer = one step).

Default workload: one Llama-3-8B-shaped layer, bf16 KV, batch 1, 32 q / 8 KV
heads, head_dim 128, 131072 tokens of context, segments of 8192, 16 tokens per
cluster (8192 clusters per KV head), 10 k-means rounds, steady zone 4 sinks +
64 recent tokens, top 1.8% of clusters retrieved (148 per KV head), page 16.

The index is built once on the GPU (timed separately, reported under
"build"), then cloned into R layer replicas; timed steps rotate through the
replicas so each step's ~44 MB working set was evicted from the 126 MB L2 by
the steps in between (R * step bytes > 2 * L2).

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--impl wave|reference]
Multi-GPU: one process per GPU under torch.distributed.run; every rank runs
its own independent replica workload (no collective on the data path), the
step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import tempfile
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-decode µs/step/layer + achieved HBM GB/s (% of roofline), 128K–1M ctx"
UNIT = "us/step/layer"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0   # dense bf16 tensor-core burst (cuBLAS) on this part


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS}, "fallback"


def kernel_source_sha256() -> str:
    """Hash of the CUDA sources (csrc/*.cu, *.cuh, *.h) in file-name order,
    comments and blank lines left out: a comment edit does not change the
    compiled kernels, so it keeps the measured traffic valid."""
    import glob
    import hashlib
    import re
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "retrieval_sparse_attention_wave_b200", "csrc", "*"))):
        if f.endswith((".cu", ".cuh", ".h")):
            with open(f) as fh:
                src = fh.read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            src = re.sub(r"//[^\n]*", "", src)
            src = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
            h.update(src.encode())
    return h.hexdigest()


def measured_traffic(cfg: int, kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary of this
    workload, or None when there is none or the kernels changed since."""
    p = os.path.join(ROOT, "profiles", f"traffic_config{cfg}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("kernel_source_sha256") != kernel_source_sha256():
        return None
    v = d.get("dram_bytes_per_launch", {}).get(kernel)
    return float(v) if v is not None else None


def workload_args(cfg: int):
    import wave_inputs as WI
    names = {1: "tiny fp32, T=4096, d=64, 1 q / 1 KV head",
             2: "Llama-3-8B-shaped layer, bf16, B=1, T=131072, 32q/8kv, d=128",
             3: "batched decode, bf16, B=16 x T=32768, 32q/8kv, d=128",
             4: "long context, bf16, B=1, T=1048576, 32q/8kv, d=128",
             5: "ragged paged batch, bf16, 8 seqs log-uniform in [4096, 262144]"}
    return names[cfg]


# ----------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix=f"wi_clocks_rank{index}_", suffix=".csv")
        os.close(fd)

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}",
                                          f"--query-gpu={self.QUERY}", "--format=csv,noheader",
                                          "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                mx = float(parts[2].split()[0])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- helpers

def algorithmic_bytes(index, params, info: np.ndarray, n_st_per_seq):
    """Bytes the method must move in one decode step, and the share of each
    launch: the steady kernel reads the steady positions' invperm entries;
    the scan reads every centroid, every value sum (not in the exact-only
    workload), the offsets and q; the gather reads the retrieved clusters'
    K/V rows with their perm entries, the steady K/V rows, and writes out and
    lse.  Workspace traffic (selection records, token lists, partial parts)
    and re-reads (the retrieved clusters' centroid and value-sum rows taken
    back out of the estimate) are not counted: they are not the method's
    bytes."""
    e = 2 if index.dtype == torch.bfloat16 else 4
    d = index.head_dim
    H = index.n_kv_heads
    per_stage = {"steady": 0, "scan": 0, "gather": 0}
    for b, T in enumerate(index.seq_lens):
        NC = index.nc[b]
        dense = bool(info[b * H, 6])
        st = T if dense else n_st_per_seq[b]
        sel_tok = int(sum(info[b * H + h, 3] for h in range(H)))
        if not dense:
            per_stage["steady"] += H * st * 4
            per_stage["scan"] += H * NC * d * e * (1 if params.exact_only else 2) \
                + H * (NC + 1) * 4 + params.n_q_heads * d * e
        per_stage["gather"] += sel_tok * (2 * d * e + 4) + H * st * 2 * d * e \
            + params.n_q_heads * (d + 1) * 4
    return sum(per_stage.values()), per_stage


def steady_count(T, n_sink, window):
    ns = min(n_sink, T)
    ws = max(T - window, ns)
    return ns + (T - ws)


def rank_seed(cfg: int, rank: int):
    """Seed of rank r's synthetic workload: rank 0 uses the workload's own
    seed, every other rank a distinct one, so the ranks' replicas differ."""
    return None if rank == 0 else 1000 * rank + cfg


def max_over_ranks(x: float, device) -> float:
    """The largest x over all ranks (a MAX all-reduce); x itself alone."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(ms_total_max: float, steps: int, world: int):
    """(device time per step on the slowest rank in us, whole-job value): with
    every rank decoding its own replica layer per step, the job advances
    `world` layer steps per step time, so the time per layer step is the
    slowest rank's step time divided by the number of ranks."""
    us_per_step = ms_total_max * 1e3 / steps
    return us_per_step, us_per_step / world


def clone_index(wx):
    import copy
    c = copy.copy(wx)
    for name in ["centroids", "value_sums", "offsets", "perm", "invperm", "labels", "k_pool",
                 "v_pool"]:
        setattr(c, name, getattr(wx, name).clone())
    return c


# ----------------------------------------------------------------- wave arm

def build_workload(cfg, dev, seed):
    """The workload's paged input cache and its GPU-built index (build timed
    once, cold, with events)."""
    import retrieval_sparse_attention_wave_b200 as W
    import wave_inputs as WI
    wl = WI.config(cfg, device=dev, seed=seed)
    bt, n_pages = WI.make_block_table(wl.seq_lens, wl.page_size,
                                      shuffle_seed=(5 if cfg == 5 else None))
    kv = W.KVCache(WI.to_pages(wl.keys, bt, n_pages, wl.page_size),
                   WI.to_pages(wl.values, bt, n_pages, wl.page_size),
                   torch.as_tensor(bt, device=dev), list(wl.seq_lens))
    wl.keys = wl.values = None
    bt_out, n_out = WI.make_block_table(wl.seq_lens, wl.page_size,
                                        shuffle_seed=(6 if cfg == 5 else None))
    bt_out = torch.as_tensor(bt_out, device=dev)
    W.build_index(kv, wl.seg_len, wl.cluster_size, 1, block_table=bt_out, n_pages=n_out)  # warm
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record()
    wx = W.build_index(kv, wl.seg_len, wl.cluster_size, wl.iters, block_table=bt_out,
                       n_pages=n_out)
    b1.record()
    torch.cuda.synchronize()
    assert W.read_device_status(wx._build_ws) == 0
    return wl, kv, wx, bt_out, n_out, b0.elapsed_time(b1)


def assign_round_us(W, wl, kv, wx, reps=10):
    """One k-means assignment round over every segment (the build's hot
    kernel pair), through the public assignment call, against the built
    index's fp32 centroids: mean of `reps` event-timed calls after a warm-up."""
    cent, _ = W.build_state(kv, wx)
    cent = cent.clone()
    ws = torch.empty(W.build_workspace_bytes(kv, wl.seg_len, wl.cluster_size), dtype=torch.uint8,
                     device=cent.device)
    W.kmeans_assign(kv, wl.seg_len, wl.cluster_size, cent, ws=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        W.kmeans_assign(kv, wl.seg_len, wl.cluster_size, cent, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / reps


class DecodeTimer:
    """Timed decode steps of one workload: R layer replicas of the index
    (R x step bytes > 2 x L2, so each step reads from HBM), one CUDA graph per
    replica and one with all R replicas back to back (a model step's layers);
    the decode's first kernel is a plain launch, so layers never overlap."""

    def __init__(self, W, wl, wx, params, dev, stream, replicas=0, graphs=True):
        self.W, self.wl, self.params, self.dev, self.stream = W, wl, params, dev, stream
        self.q = wl.q.to(dev)
        self.ws = W.decode_workspace(wx, params)
        self.lay = W.decode_layout(wx, params)
        W.decode(self.q, wx, params, ws=self.ws)
        torch.cuda.synchronize()
        self.info = W.unit_info(self.ws, self.lay, wl.batch * wl.n_kv_heads).cpu().numpy()
        n_st = [steady_count(T, wl.n_sink, wl.window) for T in wl.seq_lens]
        self.step_bytes, self.stage_bytes = algorithmic_bytes(wx, params, self.info, n_st)
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.l2 = l2
        R = max(1, math.ceil(2 * l2 / self.step_bytes)) + 1 if replicas <= 0 else replicas
        self.R = R
        self.reps = [wx] + [clone_index(wx) for _ in range(R - 1)]
        self.outs = [torch.empty(wl.batch, wl.n_q_heads, wl.head_dim, dtype=torch.float32,
                                 device=dev) for _ in range(R)]
        self.lses = [torch.empty(wl.batch, wl.n_q_heads, dtype=torch.float32, device=dev)
                     for _ in range(R)]
        self.graphs, self.full = [], None
        with torch.cuda.stream(stream):
            for r in range(R):                     # every replica runs once before capture
                self.decode(r)
            stream.synchronize()
            if graphs:
                for r in range(R):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        self.decode(r)
                    self.graphs.append(g)
                self.full = torch.cuda.CUDAGraph()
                with torch.cuda.graph(self.full, stream=stream):
                    for r in range(R):
                        self.decode(r)

    def decode(self, r, events=None):
        self.W.decode(self.q, self.reps[r], self.params, out=self.outs[r], lse=self.lses[r],
                      ws=self.ws, stream=self.stream, stage_events=events)

    def steps(self, n, per_layer_graphs=False):
        """Exactly n decode steps (layer r of step i is replica i % R)."""
        if not self.graphs:
            for i in range(n):
                self.decode(i % self.R)
            return
        if per_layer_graphs:
            for i in range(n):
                self.graphs[i % self.R].replay()
            return
        whole, rest = divmod(n, self.R)
        for _ in range(whole):
            self.full.replay()
        for r in range(rest):
            self.graphs[r].replay()

    def timed(self, n, per_layer_graphs=False) -> float:
        """Device ms of exactly n steps, CUDA events on the launching stream."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            e0.record(self.stream)
            self.steps(n, per_layer_graphs)
            e1.record(self.stream)
        self.stream.synchronize()
        return e0.elapsed_time(e1)

    def distribution(self, min_samples=100, min_seconds=1.0):
        """Per-step device time over at least min_samples samples and
        min_seconds: each sample replays the R-layer graph once (R steps) and
        counts its time / R; returns median, p10, p90 in us."""
        per, t_start = [], time.perf_counter()
        while len(per) < min_samples or time.perf_counter() - t_start < min_seconds:
            per.append(self.timed(self.R) * 1e3 / self.R)
            if len(per) > 100000:
                break
        a = np.asarray(per)
        return {"median": float(np.median(a)), "p10": float(np.percentile(a, 10)),
                "p90": float(np.percentile(a, 90)), "samples": int(len(a)),
                "steps_per_sample": self.R}

    def stage_us(self, n=100):
        """Per-kernel device time: launches serialised (no programmatic
        dependent launch), events recorded between them on the stream."""
        W = self.W
        nst = W.lib().wi_decode_stage_count()
        names = W.stage_names()
        acc = np.zeros(nst)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)]
        with torch.cuda.stream(self.stream):
            for i in range(n):
                self.decode(i % self.R, evs)
                evs[-1].synchronize()
                acc += [evs[j].elapsed_time(evs[j + 1]) for j in range(nst)]
        return {names[j]: acc[j] * 1e3 / n for j in range(nst)}

    def release(self):
        self.graphs, self.full = [], None
        self.reps = self.reps[:1]


def roofline_of(stage_us, stage_bytes, hbm, peak_kind, cfg):
    dom = max(stage_us, key=lambda k: stage_us[k])
    gbs = stage_bytes[dom] / (stage_us[dom] * 1e-6) / 1e9
    return {"bound": "hbm", "kernel": dom, "achieved": gbs, "peak": hbm, "unit": "GB/s",
            "frac": gbs / hbm, "traffic": measured_traffic(cfg, dom),
            "bytes_per_launch": stage_bytes[dom], "us_per_launch": stage_us[dom],
            "peak_kind": peak_kind}


def selection_recall(W, timer, wx, params_exact, params_sampled):
    """Mean recall of the sampled selection against the exact one on the same
    query and index (share of each unit's exact top-k it retrieves)."""
    wl = timer.wl
    ws_e = W.decode_workspace(wx, params_exact)
    ws_s = W.decode_workspace(wx, params_sampled)
    W.decode(timer.q, wx, params_exact, ws=ws_e)
    W.decode(timer.q, wx, params_sampled, ws=ws_s)
    torch.cuda.synchronize()
    lay_e, lay_s = W.decode_layout(wx, params_exact), W.decode_layout(wx, params_sampled)
    U = wl.batch * wl.n_kv_heads
    ie, is_ = W.unit_info(ws_e, lay_e, U).cpu().numpy(), W.unit_info(ws_s, lay_s, U).cpu().numpy()
    rec = []
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            u = b * wl.n_kv_heads + h
            a = W.selected_clusters(ws_e, lay_e, wx, b, h, int(ie[u, 0])).cpu().numpy()
            s_ = W.selected_clusters(ws_s, lay_s, wx, b, h, int(is_[u, 0])).cpu().numpy()
            if len(a):
                rec.append(len(np.intersect1d(a, s_)) / len(a))
    return float(np.mean(rec)) if rec else 1.0, float(np.min(rec)) if rec else 1.0


def run_wave(args, rank, world, local_rank):
    import retrieval_sparse_attention_wave_b200 as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl, kv, wx, bt_out, n_out, build_ms = build_workload(args.config, dev,
                                                         rank_seed(args.config, rank))

    if args.decode_only:
        return run_decode_only(args, W, wl, kv, wx, dev, build_ms)
    assign_us = assign_round_us(W, wl, kv, wx)
    # index extension: each sequence's last seg_len tokens arrive later (as a
    # decode appends them); the index of the shorter sequences grows to the
    # full ones, timed with events, and must equal the full build
    old_lens = [max(1, T - wl.seg_len) for T in wl.seq_lens]
    kv_old = W.KVCache(kv.k_pool, kv.v_pool, kv.block_table, old_lens)
    old = W.build_index(kv_old, wl.seg_len, wl.cluster_size, wl.iters, block_table=bt_out,
                        n_pages=n_out)
    W.extend_index(old, kv, wl.iters)                 # warm
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record()
    ext = W.extend_index(old, kv, wl.iters)
    x1.record()
    torch.cuda.synchronize()
    extend_ms = x0.elapsed_time(x1)
    assert torch.equal(ext.centroids, wx.centroids) and torch.equal(ext.perm, wx.perm)
    extend_tokens = sum(T - t for T, t in zip(wl.seq_lens, old_lens))
    # the block top-k workload's index: position blocks of cluster_size tokens
    bx = W.build_blocks(kv, wl.seg_len, wl.cluster_size, block_table=bt_out, n_pages=n_out)
    torch.cuda.synchronize()
    assert W.read_device_status(bx._build_ws) == 0
    del kv, kv_old, old, ext
    torch.cuda.empty_cache()

    params = W.DecodeParams(n_q_heads=wl.n_q_heads, n_sink=wl.n_sink, window=wl.window,
                            topk_clusters=wl.topk_clusters, topk_fraction=wl.topk_fraction)
    stream = torch.cuda.Stream(device=dev)
    T = DecodeTimer(W, wl, wx, params, dev, stream, args.replicas, not args.no_graph)
    with torch.cuda.stream(stream):
        T.steps(args.warmup)
        T.steps(args.warmup, per_layer_graphs=True)
    stream.synchronize()

    dist = world > 1
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    ms = T.timed(args.steps)                         # exactly K steps: the value
    spread = T.distribution()                        # >= 100 samples, >= 1 s
    clk = clocks.stop()
    per_layer_graph_us = max_over_ranks(T.timed(args.steps, per_layer_graphs=True), dev) \
        * 1e3 / args.steps
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(ms, dev)
    us_per_step, job_us = job_value(ms, args.steps, world)
    stage_us = T.stage_us(max(20, min(200, args.steps)))

    # end to end through the public API with host buffers
    q_h = wl.q.cpu().pin_memory()
    out_h = torch.empty(wl.batch, wl.n_q_heads, wl.head_dim, dtype=torch.float32).pin_memory()
    lse_h = torch.empty(wl.batch, wl.n_q_heads, dtype=torch.float32).pin_memory()
    n_e2e = max(10, min(args.steps, 200))
    with torch.cuda.stream(stream):
        # warm-up: every replica's call seen twice (the library captures a
        # call's copies and kernels into a graph the second time it sees it)
        for i in range(max(3, 2 * T.R)):
            W.decode_host(q_h, T.reps[i % T.R], params, out_h, lse_h, T.ws, stream=stream)
        stream.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(n_e2e):
            W.decode_host(q_h, T.reps[i % T.R], params, out_h, lse_h, T.ws, stream=stream)
            stream.synchronize()                 # the host reads this step's result
        f1.record(stream)
        stream.synchronize()
    e2e_us = f0.elapsed_time(f1) * 1e3 / n_e2e
    assert np.isfinite(out_h.numpy()).all()
    assert W.read_device_status(T.ws, stream) == 0

    # block top-k workload (exact attention over the top 1.8% blocks and the
    # steady zone, no estimation zone) on the block index, and the wave
    # decode under the same protocol: one CUDA graph per step, L2 flushed by
    # a 2 x L2 write outside each timed step
    bparams = W.DecodeParams(n_q_heads=wl.n_q_heads, n_sink=wl.n_sink, window=wl.window,
                             topk_clusters=wl.topk_clusters, topk_fraction=wl.topk_fraction,
                             exact_only=True)
    flush = torch.empty(2 * T.l2, dtype=torch.uint8, device=dev)

    def flushed_us(ix, prm, n=50):
        wsp = W.decode_workspace(ix, prm)
        o = torch.empty(wl.batch, wl.n_q_heads, wl.head_dim, dtype=torch.float32, device=dev)
        lo = torch.empty(wl.batch, wl.n_q_heads, dtype=torch.float32, device=dev)
        with torch.cuda.stream(stream):
            W.decode(T.q, ix, prm, out=o, lse=lo, ws=wsp, stream=stream)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                W.decode(T.q, ix, prm, out=o, lse=lo, ws=wsp, stream=stream)
            tot = 0.0
            for i in range(n + 3):
                flush.fill_(1)
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record(stream)
                g.replay()
                a1.record(stream)
                stream.synchronize()
                tot += a0.elapsed_time(a1) if i >= 3 else 0.0
        assert W.read_device_status(wsp, stream) == 0 and torch.isfinite(o).all()
        del g
        return tot * 1e3 / n

    block_us = flushed_us(bx, bparams)
    wave_flushed_us = flushed_us(wx, params)
    # stochastic radix top-k: same protocol, and its recall against the exact selection
    sparams = W.DecodeParams(n_q_heads=wl.n_q_heads, n_sink=wl.n_sink, window=wl.window,
                             topk_clusters=wl.topk_clusters, topk_fraction=wl.topk_fraction,
                             sampled=True, seed=12345)
    sampled_us = flushed_us(wx, sparams)
    rec_mean, rec_min = selection_recall(W, T, wx, params, sparams)
    del bx, flush

    peaks, peak_kind = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    step_gbs = T.step_bytes / (us_per_step * 1e-6) / 1e9
    tokens = sum(wl.seq_lens)
    assign_flop = 2.0 * sum(wl.seq_lens) * wl.n_kv_heads * (wl.seg_len // wl.cluster_size) \
        * wl.head_dim * wl.iters
    nst = W.lib().wi_decode_stage_count()
    result = {
        "metric": METRIC,
        "value": job_us,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": us_per_step / 1e3,
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded Gaussian-mixture keys, N(0,1) values)",
        "config": {"workload": workload_args(args.config), "batch": wl.batch,
                   "context": wl.seq_lens if wl.batch > 1 else wl.seq_lens[0],
                   "n_q_heads": wl.n_q_heads, "n_kv_heads": wl.n_kv_heads,
                   "head_dim": wl.head_dim, "seg_len": wl.seg_len,
                   "cluster_size": wl.cluster_size, "topk_fraction": wl.topk_fraction,
                   "n_sink": wl.n_sink, "window": wl.window,
                   "l2": f"rotate {T.R} layer replicas ({T.R * T.step_bytes / 1e6:.0f} MB per "
                         f"cycle > 2x L2)",
                   "cuda_graph": (f"{T.R} layer decodes per graph" if not args.no_graph
                                  else False),
                   "parallelism": f"replicas{world}"},
        "step_distribution_us": spread,
        "us_per_step_one_graph_per_layer": per_layer_graph_us,
        "tokens_per_s": tokens * world / (us_per_step * 1e-6),
        "hbm_gbs": step_gbs,
        "step_bytes": T.step_bytes,
        "stage_bytes": T.stage_bytes,
        "roofline_step": {"achieved": step_gbs, "peak": hbm, "unit": "GB/s",
                          "frac": step_gbs / hbm, "peak_kind": peak_kind},
        "roofline": roofline_of(stage_us, T.stage_bytes, hbm, peak_kind, args.config),
        "stage_us": stage_us,
        "gpu_launches": nst * args.steps,
        "e2e": {"value": e2e_us, "unit": UNIT,
                "h2d_bytes_per_step": int(q_h.numel() * q_h.element_size()),
                "d2h_bytes_per_step": int(out_h.numel() * 4 + lse_h.numel() * 4),
                "path": "wi_decode_host: q copied host to device; out and lse written by the "
                        "kernels into the pinned, device-mapped host buffers; a synchronise "
                        "per step"},
        "build": {"ms": build_ms, "iters": wl.iters, "assign_tflop": assign_flop / 1e12,
                  "assign_tflops_achieved": assign_flop / (build_ms * 1e-3) / 1e12,
                  "assign_round_us": assign_us,
                  # one assignment round (split + tensor-core kernel) against
                  # the bf16 peak: the tensor cores do two bf16 terms per
                  # centroid, twice the round's distance flops
                  "assign_roofline": {
                      "bound": "tensor",
                      "achieved": 2 * assign_flop / wl.iters / (assign_us * 1e-6) / 1e12,
                      "peak": float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)),
                      "unit": "TFLOP/s",
                      "frac": 2 * assign_flop / wl.iters / (assign_us * 1e-6) / 1e12
                              / float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)),
                      "peak_kind": peak_kind}},
        "block_topk": {"us_per_step": block_us, "wave_us_per_step_same_protocol": wave_flushed_us,
                       "note": "exact attention over the top blocks of cluster_size tokens "
                               "and the steady zone, no estimation; one graph per step, "
                               "L2 flushed between steps"},
        "stochastic_topk": {"us_per_step": sampled_us,
                            "exact_us_per_step_same_protocol": wave_flushed_us,
                            "recall_mean": rec_mean, "recall_min": rec_min,
                            "note": "threshold bin sampled by SplitMix64 draws (seed 12345); "
                                    "recall = share of each unit's exact top-k retrieved"},
        "extend": {"ms": extend_ms, "iters": wl.iters, "new_tokens": extend_tokens,
                   "note": "index grown by the last seg_len tokens of every sequence; "
                           "equals the full build"},
        "clocks": clk,
    }
    T.release()
    del T, wx
    torch.cuda.empty_cache()
    return result, wl


def run_decode_only(args, W, wl, kv, wx, dev, build_ms):
    """The decode steps alone (no extension, block or sampled workloads, no
    host-buffer run): the mode a kernel profile runs, so few launches come
    before the decode's own."""
    del kv
    torch.cuda.empty_cache()
    params = W.DecodeParams(n_q_heads=wl.n_q_heads, n_sink=wl.n_sink, window=wl.window,
                            topk_clusters=wl.topk_clusters, topk_fraction=wl.topk_fraction)
    stream = torch.cuda.Stream(device=dev)
    T = DecodeTimer(W, wl, wx, params, dev, stream, args.replicas, not args.no_graph)
    with torch.cuda.stream(stream):
        T.steps(args.warmup)
    stream.synchronize()
    ms = T.timed(args.steps)
    assert W.read_device_status(T.ws, stream) == 0
    us = ms * 1e3 / args.steps
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    gbs = T.step_bytes / (us * 1e-6) / 1e9
    res = {"metric": METRIC, "value": us, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
           "scaling": "weak", "vs_baseline": None,
           "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32",
           "data": "synthetic (seeded Gaussian-mixture keys, N(0,1) values)",
           "config": {"workload": workload_args(args.config), "mode": "decode only"},
           "step_bytes": T.step_bytes, "stage_bytes": T.stage_bytes,
           "roofline_step": {"achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                             "peak_kind": peak_kind},
           "build": {"ms": build_ms}, "gpu_launches": 3 * args.steps}
    T.release()
    return res, wl


def run_config_block(cfg, args, dev, hbm, peak_kind):
    """Decode timing of another workload (its own line of the metric's
    128K-1M range): exactly-K value, distribution, per-kernel time, roofline
    and the oracle's time on host cores."""
    import retrieval_sparse_attention_wave_b200 as W
    wl, kv, wx, _, _, build_ms = build_workload(cfg, dev, None)
    del kv
    torch.cuda.empty_cache()
    params = W.DecodeParams(n_q_heads=wl.n_q_heads, n_sink=wl.n_sink, window=wl.window,
                            topk_clusters=wl.topk_clusters, topk_fraction=wl.topk_fraction)
    stream = torch.cuda.Stream(device=dev)
    T = DecodeTimer(W, wl, wx, params, dev, stream, 0, True)
    with torch.cuda.stream(stream):
        T.steps(max(3, args.warmup))
    stream.synchronize()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    ms = T.timed(max(args.steps, T.R))
    spread = T.distribution(min_samples=100, min_seconds=0.5)
    clk = clocks.stop()
    us = ms * 1e3 / max(args.steps, T.R)
    stage_us = T.stage_us(50)
    assert W.read_device_status(T.ws, stream) == 0
    gbs = T.step_bytes / (us * 1e-6) / 1e9
    rf = roofline_of(stage_us, T.stage_bytes, hbm, peak_kind, cfg)
    block = {"workload": workload_args(cfg), "us_per_step": us, "steps": max(args.steps, T.R),
             "step_distribution_us": spread, "step_bytes": T.step_bytes,
             "stage_bytes": T.stage_bytes, "stage_us": stage_us,
             "tokens_per_s": sum(wl.seq_lens) / (us * 1e-6),
             "roofline_step": {"achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                               "peak_kind": peak_kind},
             "roofline": rf, "build_ms": build_ms, "replicas": T.R, "clocks": clk}
    if cfg == 4:
        # the top-k's share: the scan's tails run the per-head selection after
        # the streaming; reported as the scan kernel's share of the step
        block["scan_share_of_step"] = stage_us.get("scan", 0.0) / max(sum(stage_us.values()), 1e-9)
    if not args.no_cpu_baseline:
        block["cpu_baseline"] = oracle_decode_timing(W, wl, wx, params, budget_s=args.extra_cpu_budget)
    T.release()
    del T, wx
    torch.cuda.empty_cache()
    return block


# ----------------------------------------------------------------- oracle arm

def oracle_timing(cfg: int, budget_s: float):
    """Time the fp64 oracle decode on host cores on a bounded sample: the index
    of one (sequence, KV head) unit built by the oracle, then decode steps of
    that unit until the budget is spent; scaled to a whole layer step."""
    import oracle as O
    import wave_inputs as WI
    wl = WI.config(cfg, device="cpu")
    G = wl.n_q_heads // wl.n_kv_heads
    b, h = 0, 0
    K = wl.keys[b][h].to(torch.float64).numpy()
    V = wl.values[b][h].to(torch.float64).numpy()
    store = "bf16" if wl.dtype == torch.bfloat16 else "f32"
    t0 = time.perf_counter()
    ix = O.build_unit(K, V, wl.seg_len, wl.cluster_size, wl.iters, store)
    build_s = time.perf_counter() - t0
    qg = wl.q[b, h * G:(h + 1) * G].to(torch.float64).numpy()
    k = O.k_for(len(ix.centroids), wl.topk_clusters, wl.topk_fraction)
    n = 0
    t0 = time.perf_counter()
    while True:
        O.decode_unit(qg, ix, wl.n_sink, wl.window, k)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    units = wl.batch * wl.n_kv_heads
    us_step = el / n * units * 1e6
    cores = len(os.sched_getaffinity(0))
    return {"value": us_step, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"unit (b=0, kv head 0) of {units}; oracle-built index "
                      f"({wl.iters} rounds, {build_s:.1f} s); {n} decode steps in {el:.1f} s, "
                      f"x{units} units per layer step",
            "build_s_per_unit": build_s}


def oracle_decode_timing(W, wl, wx, params, budget_s: float):
    """Time the fp64 oracle's decode of one (sequence, KV head) unit of the
    GPU-built index (downloaded to the host) for a bounded time; scaled to a
    whole layer step (all units)."""
    import oracle as O
    b, h = 0, 0
    T, NC = wx.seq_lens[b], wx.nc[b]
    r, o, t = wx.cl_row(b, h), wx.off_row(b, h), wx.tok_row(b, h)
    slots = torch.arange(T, device=wx.block_table.device)
    pages = wx.block_table[b].long()[slots // wx.page_size]
    rows = slots % wx.page_size
    f32 = lambda x: x.to(torch.float32).cpu().numpy()
    i64 = lambda x: x.cpu().numpy().astype(np.int64)
    ix = O.UnitIndex(centroids=f32(wx.centroids[r:r + NC]).astype(np.float64),
                     value_sums=f32(wx.value_sums[r:r + NC]).astype(np.float64),
                     offsets=i64(wx.offsets[o:o + NC + 1]), perm=i64(wx.perm[t:t + T]),
                     invperm=i64(wx.invperm[t:t + T]), k_perm=f32(wx.k_pool[pages, h, rows]),
                     v_perm=f32(wx.v_pool[pages, h, rows]), labels=i64(wx.labels[t:t + T]),
                     centroids_exact=None, value_sums_exact=None)
    G = wl.n_q_heads // wl.n_kv_heads
    qg = wl.q[b, h * G:(h + 1) * G].to(torch.float64).cpu().numpy()
    k = O.k_for(NC, wl.topk_clusters, wl.topk_fraction)
    n = 0
    t0 = time.perf_counter()
    while True:
        O.decode_unit(qg, ix, wl.n_sink, wl.window, k)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    units = wl.batch * wl.n_kv_heads
    return {"value": el / n * units * 1e6, "unit": UNIT, "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"unit (b=0, kv head 0) of {units} of the GPU-built index; {n} oracle "
                      f"decode steps in {el:.1f} s, x{units} units per layer step"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--impl", default="wave", choices=["wave", "reference"])
    ap.add_argument("--replicas", type=int, default=0)
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra-configs", default="3,4,5",
                    help="other workloads of the metric's range timed after the headline "
                         "(one GPU only; '' for none)")
    ap.add_argument("--extra-cpu-budget", type=float, default=6.0)
    ap.add_argument("--decode-only", action="store_true",
                    help="time the decode steps alone (a profiling run): no extension, block, "
                         "sampled, host-buffer, CPU-baseline or other-workload timings")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # the oracle arm: rank 0 alone times the fp64 oracle on host cores
        if rank != 0:
            return
        steps = max(1, args.steps)
        cb = oracle_timing(args.config, budget_s=min(args.cpu_budget, 60.0))
        res = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT,
               "n_gpus": world, "steps": steps, "warmup": args.warmup,
               "ms_per_step": cb["value"] / 1e3, "higher_is_better": False,
               "scaling": "weak", "vs_baseline": None, "dtype": "f64",
               "data": "synthetic (seeded Gaussian-mixture keys, N(0,1) values)",
               "config": {"workload": workload_args(args.config)},
               "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
               "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                       "d2h_bytes_per_step": 0}}
        print(json.dumps(res))
        return

    if world > 1:
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        res, _ = run_wave(args, rank, world, local_rank)
        if args.decode_only:
            if rank == 0:
                print(json.dumps(res))
            return
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                cb = oracle_timing(args.config, budget_s=args.cpu_budget)
                res["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind",
                                                          "sample")}
            if world == 1 and args.extra_configs:
                peaks, peak_kind = measured_peaks()
                dev = torch.device("cuda", local_rank)
                res["configs"] = {}
                for c in [int(x) for x in args.extra_configs.split(",") if x.strip()]:
                    if c != args.config:
                        res["configs"][str(c)] = run_config_block(c, args, dev,
                                                                  float(peaks["hbm_gbs"]),
                                                                  peak_kind)
            print(json.dumps(res))
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
