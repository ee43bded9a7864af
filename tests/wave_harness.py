"""Test harness: moves workloads between the logical layout the oracle uses
and the paged layout the library uses, and compares results.

Layout only: nothing here computes any part of the method.
"""
from __future__ import annotations

import math
from typing import List, Optional

import numpy as np
import torch

import oracle as O
import retrieval_sparse_attention_wave_b200 as W
import wave_inputs as WI


def store_name(dtype: torch.dtype) -> str:
    return "bf16" if dtype == torch.bfloat16 else "f32"


def paged_kv(wl: WI.Workload, device="cuda", shuffle_seed: Optional[int] = None,
             page_size: Optional[int] = None) -> W.KVCache:
    P = page_size or wl.page_size
    bt, n_pages = WI.make_block_table(wl.seq_lens, P, shuffle_seed=shuffle_seed)
    keys = [k.to(device) for k in wl.keys]
    vals = [v.to(device) for v in wl.values]
    kp = WI.to_pages(keys, bt, n_pages, P)
    vp = WI.to_pages(vals, bt, n_pages, P)
    return W.KVCache(kp, vp, torch.as_tensor(bt, device=device), list(wl.seq_lens))


def out_block_table(wl: WI.Workload, device="cuda", shuffle_seed: Optional[int] = None,
                    page_size: Optional[int] = None):
    P = page_size or wl.page_size
    bt, n_pages = WI.make_block_table(wl.seq_lens, P, shuffle_seed=shuffle_seed, extra_pages=3)
    return torch.as_tensor(bt, device=device), n_pages


def host_rows(wl: WI.Workload):
    keys = [k.detach().to("cpu", torch.float64).numpy() for k in wl.keys]
    vals = [v.detach().to("cpu", torch.float64).numpy() for v in wl.values]
    return keys, vals


def oracle_build(wl: WI.Workload, iters: Optional[int] = None, units=None):
    """Oracle index for every unit (or for the given (b, h) units only)."""
    keys, vals = host_rows(wl)
    it = wl.iters if iters is None else iters
    out = {}
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            if units is not None and (b, h) not in units:
                continue
            out[(b, h)] = O.build_unit(keys[b][h], vals[b][h], wl.seg_len, wl.cluster_size, it,
                                       store_name(wl.dtype))
    return out


def empty_index(wl: WI.Workload, device="cuda", shuffle_seed=None, page_size=None) -> W.WaveIndex:
    bt, n_pages = out_block_table(wl, device, shuffle_seed, page_size)
    return W.WaveIndex(wl.seq_lens, wl.n_kv_heads, wl.head_dim, wl.dtype,
                       page_size or wl.page_size, wl.seg_len, wl.cluster_size, device,
                       block_table=bt, n_pages=n_pages)


def _slot_addr(wx: W.WaveIndex, b: int, T: int):
    slots = torch.arange(T, device=wx.block_table.device)
    pages = wx.block_table[b].long()[slots // wx.page_size]
    return pages, slots % wx.page_size


def upload_unit(wx: W.WaveIndex, b: int, h: int, ix: O.UnitIndex):
    """Write an oracle-built unit index into the library's buffers."""
    dev = wx.centroids.device
    T, NC = wx.seq_lens[b], wx.nc[b]
    assert len(ix.centroids) == NC and len(ix.perm) == T
    r = wx.cl_row(b, h)
    wx.centroids[r:r + NC] = torch.as_tensor(ix.centroids, device=dev).to(wx.dtype)
    wx.value_sums[r:r + NC] = torch.as_tensor(ix.value_sums, device=dev).to(wx.dtype)
    o = wx.off_row(b, h)
    wx.offsets[o:o + NC + 1] = torch.as_tensor(ix.offsets.astype(np.int32), device=dev)
    t = wx.tok_row(b, h)
    wx.perm[t:t + T] = torch.as_tensor(ix.perm.astype(np.int32), device=dev)
    wx.invperm[t:t + T] = torch.as_tensor(ix.invperm.astype(np.int32), device=dev)
    lab = np.empty(T, dtype=np.int64)                 # cluster of each position
    lab[ix.perm] = np.repeat(np.arange(NC), np.diff(ix.offsets))
    wx.labels[t:t + T] = torch.as_tensor(lab.astype(np.int32), device=dev)
    pages, rows = _slot_addr(wx, b, T)
    wx.k_pool[pages, h, rows] = torch.as_tensor(ix.k_perm, device=dev).to(wx.dtype)
    wx.v_pool[pages, h, rows] = torch.as_tensor(ix.v_perm, device=dev).to(wx.dtype)


def upload_index(wx: W.WaveIndex, units: dict):
    for (b, h), ix in units.items():
        upload_unit(wx, b, h, ix)


def download_unit(wx: W.WaveIndex, b: int, h: int) -> dict:
    """The library's index of unit (b, h) in logical layout (numpy, fp64 values)."""
    T, NC = wx.seq_lens[b], wx.nc[b]
    r, o, t = wx.cl_row(b, h), wx.off_row(b, h), wx.tok_row(b, h)
    pages, rows = _slot_addr(wx, b, T)
    f = lambda x: x.to(torch.float64).cpu().numpy()
    return dict(
        centroids=f(wx.centroids[r:r + NC]), value_sums=f(wx.value_sums[r:r + NC]),
        offsets=wx.offsets[o:o + NC + 1].cpu().numpy().astype(np.int64),
        perm=wx.perm[t:t + T].cpu().numpy().astype(np.int64),
        invperm=wx.invperm[t:t + T].cpu().numpy().astype(np.int64),
        labels=wx.labels[t:t + T].cpu().numpy().astype(np.int64),
        k_perm=f(wx.k_pool[pages, h, rows]), v_perm=f(wx.v_pool[pages, h, rows]))


def as_unit_index(d: dict) -> O.UnitIndex:
    return O.UnitIndex(centroids=d["centroids"], value_sums=d["value_sums"],
                       offsets=d["offsets"], perm=d["perm"], invperm=d["invperm"],
                       k_perm=d["k_perm"], v_perm=d["v_perm"], labels=d["labels"],
                       centroids_exact=None, value_sums_exact=None)


def q_host(wl: WI.Workload) -> np.ndarray:
    return wl.q.detach().to("cpu", torch.float64).numpy()


def params_of(wl: WI.Workload, **over) -> W.DecodeParams:
    p = W.DecodeParams(n_q_heads=wl.n_q_heads, n_sink=wl.n_sink, window=wl.window,
                       topk_clusters=wl.topk_clusters, topk_fraction=wl.topk_fraction)
    for k, v in over.items():
        setattr(p, k, v)
    return p


def rel_err(got: np.ndarray, ref: np.ndarray, dtype: torch.dtype) -> float:
    """Spec metric: fp32 configs max|d|/max|ref|, bf16 configs max|d|/rms(ref)."""
    d = np.max(np.abs(got - ref))
    if dtype == torch.float32:
        return float(d / max(np.max(np.abs(ref)), 1e-30))
    return float(d / max(math.sqrt(np.mean(ref * ref)), 1e-30))


TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


def assert_one_round_moves_are_near_ties(X: np.ndarray, lab_g: np.ndarray, lab_o: np.ndarray,
                                         seg_len: int, cluster_size: int) -> int:
    """After one round from the initial centroids, a position whose GPU
    cluster differs from the oracle's must be a near-tie under those initial
    centroids: its fp64 distance to the GPU's centroid lies within 1e-5
    relative of the distance to the oracle's.  lab_g / lab_o are global
    cluster ids per original position of one unit.  Returns the count."""
    moved = 0
    c0 = 0
    for s, n in O.segment_spans(len(X), seg_len):
        m = O.clusters_in_segment(n, cluster_size)
        g, o = lab_g[s:s + n] - c0, lab_o[s:s + n] - c0
        bad = np.nonzero(g != o)[0]
        if len(bad):
            assert g[bad].min() >= 0 and g[bad].max() < m, "moved outside its segment"
            D = O.kmeans_distances(X[s:s + n][bad], O.kmeans_init(X[s:s + n], cluster_size))
            dg = D[np.arange(len(bad)), g[bad]]
            do = D[np.arange(len(bad)), o[bad]]
            assert np.all(dg <= do * (1 + 1e-5)), "one-round assignment differs beyond near-ties"
            moved += len(bad)
        c0 += m
    return moved
