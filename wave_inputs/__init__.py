"""Seeded synthetic inputs for the wave-index decode and build paths.

This module draws random numbers and lays tensors out in pages. It holds none
of the method's arithmetic (no scores, no clustering, no attention), so both
the fp64 oracle and the CUDA path may take their inputs from here.

Workloads follow the key/value/query recipe of the five configurations the
wave-index hot path is measured on (a Gaussian-mixture key distribution, N(0,1)
values, queries drawn near a key centre).  The pages evaluate on long-context
suites with trained models; these synthetic draws stand in for them.

Generation order per configuration is fixed: centres -> per-channel scales ->
per-token centre ids -> key noise -> values -> per-q-head centre ids -> query
noise.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch


@dataclass
class Workload:
    """One synthetic decode/build workload (logical, unpaged layout).

    keys[b], values[b]: [n_kv_heads][T_b][head_dim] (torch, dtype `dtype`)
    q: [batch][n_q_heads][head_dim]
    """
    name: str
    dtype: torch.dtype
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_lens: List[int]
    seg_len: int
    cluster_size: int
    iters: int
    n_sink: int
    window: int
    topk_clusters: int          # >= 0: fixed k; < 0: use topk_fraction
    topk_fraction: float
    page_size: int
    keys: List[torch.Tensor] = field(default_factory=list)
    values: List[torch.Tensor] = field(default_factory=list)
    q: Optional[torch.Tensor] = None
    # generator state kept for drifting queries (long-context run)
    q_f32: Optional[torch.Tensor] = None

    @property
    def batch(self) -> int:
        return len(self.seq_lens)


def _mixture_keys(gen, n_kv_heads, T, d, n_centers, noise, outlier_sigma, device):
    centers = torch.randn(n_kv_heads, n_centers, d, generator=gen, device=device)
    if outlier_sigma > 0:
        scale = torch.exp(outlier_sigma * torch.randn(n_kv_heads, 1, d, generator=gen, device=device))
    else:
        scale = torch.ones(n_kv_heads, 1, d, device=device)
    ids = torch.randint(0, n_centers, (n_kv_heads, T), generator=gen, device=device)
    eps = torch.randn(n_kv_heads, T, d, generator=gen, device=device)
    k = torch.gather(centers, 1, ids.unsqueeze(-1).expand(-1, -1, d)) + noise * eps
    return centers, scale, k * scale


def _queries(gen, centers, scale, n_q_heads, noise, device):
    n_kv_heads, n_centers, d = centers.shape
    G = n_q_heads // n_kv_heads
    ids = torch.randint(0, n_centers, (n_kv_heads, G), generator=gen, device=device)
    eps = torch.randn(n_kv_heads, G, d, generator=gen, device=device)
    q = torch.gather(centers, 1, ids.unsqueeze(-1).expand(-1, -1, d)) + noise * eps
    return (q * scale).reshape(n_q_heads, d)


def mixture_workload(name, *, seq_lens, n_q_heads=32, n_kv_heads=8, head_dim=128,
                     n_centers=256, noise=0.3, outlier_sigma=0.5, dtype=torch.bfloat16,
                     seg_len=8192, cluster_size=16, iters=10, n_sink=4, window=64,
                     topk_clusters=-1, topk_fraction=0.018, page_size=16, seed=2,
                     device="cpu", per_seq_seed=False) -> Workload:
    """Gaussian-mixture keys times a per-head per-channel lognormal outlier scale.

    Each sequence draws its own centres, scales, keys, values and queries.
    With per_seq_seed the generator is re-seeded with seed+b for sequence b
    (the batched configuration's independent seeds).
    """
    wl = Workload(name=name, dtype=dtype, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads,
                  head_dim=head_dim, seq_lens=list(seq_lens), seg_len=seg_len,
                  cluster_size=cluster_size, iters=iters, n_sink=n_sink, window=window,
                  topk_clusters=topk_clusters, topk_fraction=topk_fraction, page_size=page_size)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    qs, qf = [], []
    for b, T in enumerate(seq_lens):
        if per_seq_seed:
            gen.manual_seed(seed + b)
        centers, scale, k = _mixture_keys(gen, n_kv_heads, T, head_dim, n_centers, noise,
                                          outlier_sigma, device)
        v = torch.randn(n_kv_heads, T, head_dim, generator=gen, device=device)
        q = _queries(gen, centers, scale, n_q_heads, noise, device)
        wl.keys.append(k.to(dtype))
        wl.values.append(v.to(dtype))
        qf.append(q)
        qs.append(q.to(dtype))
    wl.q = torch.stack(qs)
    wl.q_f32 = torch.stack(qf)
    return wl


def drift_queries(wl: Workload, gen: torch.Generator, sigma: float = 0.05) -> torch.Tensor:
    """Next query of a drifting decode run: q_{t+1} = q_t + N(0, sigma^2) in fp32,
    the rounded value fed to decode."""
    wl.q_f32 = wl.q_f32 + sigma * torch.randn(wl.q_f32.shape, generator=gen,
                                              device=wl.q_f32.device)
    wl.q = wl.q_f32.to(wl.dtype)
    return wl.q


def tiny_fp32_workload(seed=1, T=4096, head_dim=64, n_centers=32, noise=0.3) -> Workload:
    """fp32, one q head and one KV head, mixture of 32 N(0,1) centres, noise 0.3,
    drawn with numpy's default_rng(seed)."""
    rng = np.random.default_rng(seed)
    centers = rng.standard_normal((n_centers, head_dim))
    ids = rng.integers(0, n_centers, size=T)
    k = centers[ids] + noise * rng.standard_normal((T, head_dim))
    v = rng.standard_normal((T, head_dim))
    qid = rng.integers(0, n_centers)
    q = centers[qid] + noise * rng.standard_normal(head_dim)
    wl = Workload(name="tiny-fp32", dtype=torch.float32, n_q_heads=1, n_kv_heads=1,
                  head_dim=head_dim, seq_lens=[T], seg_len=1024, cluster_size=16, iters=10,
                  n_sink=4, window=64, topk_clusters=16, topk_fraction=0.0, page_size=16)
    wl.keys = [torch.from_numpy(k.astype(np.float32)).reshape(1, T, head_dim)]
    wl.values = [torch.from_numpy(v.astype(np.float32)).reshape(1, T, head_dim)]
    wl.q = torch.from_numpy(q.astype(np.float32)).reshape(1, 1, head_dim)
    wl.q_f32 = wl.q.clone()
    return wl


def ragged_lengths(seed: int, n: int = 8, lo: int = 4096, hi: int = 262144) -> List[int]:
    """Sequence lengths log-uniform in [lo, hi] (floor of exp(U(ln lo, ln hi)))."""
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    return [int(math.floor(math.exp(x))) for x in u]


def config(i: int, device="cpu", seed: Optional[int] = None, **over) -> Workload:
    """The five workloads: 1 tiny fp32, 2 one Llama-3-8B-shaped layer at 131072
    tokens, 3 a batch of 16 x 32768, 4 one layer at 1,048,576 tokens, 5 eight
    ragged sequences with a shared, randomly permuted page pool."""
    if i == 1:
        return tiny_fp32_workload(seed=1 if seed is None else seed)
    if i == 2:
        kw = dict(seq_lens=[131072], seed=2 if seed is None else seed)
    elif i == 3:
        kw = dict(seq_lens=[32768] * 16, seed=3 if seed is None else seed, per_seq_seed=True)
    elif i == 4:
        kw = dict(seq_lens=[1048576], seed=4 if seed is None else seed)
    elif i == 5:
        s = 5 if seed is None else seed
        kw = dict(seq_lens=ragged_lengths(s), seed=s)
    else:
        raise ValueError(f"no workload {i}")
    kw.update(over)
    return mixture_workload(f"config{i}", device=device, **kw)


# ----------------------------------------------------------------------------
# Paged layout (vTensor-style page pool + block table).  Layout only.
# ----------------------------------------------------------------------------

def pages_needed(T: int, page_size: int) -> int:
    return (T + page_size - 1) // page_size


def make_block_table(seq_lens, page_size, *, shuffle_seed: Optional[int] = None,
                     extra_pages: int = 0):
    """Assign each sequence ceil(T_b/page) pages of one shared pool.

    Returns (block_table [B][max_pages] int32, n_pages).  With shuffle_seed the
    pool order is a random permutation; unused entries are -1.
    """
    need = [pages_needed(T, page_size) for T in seq_lens]
    n_pages = sum(need) + extra_pages
    order = np.arange(n_pages)
    if shuffle_seed is not None:
        order = np.random.default_rng(shuffle_seed).permutation(n_pages)
    max_pages = max(need) if need else 0
    bt = np.full((len(seq_lens), max(max_pages, 1)), -1, dtype=np.int32)
    at = 0
    for b, n in enumerate(need):
        bt[b, :n] = order[at:at + n]
        at += n
    return bt, n_pages


def to_pages(rows: List[torch.Tensor], block_table: np.ndarray, n_pages: int,
             page_size: int) -> torch.Tensor:
    """Scatter per-sequence [Hkv][T_b][d] rows into a pool [n_pages][Hkv][page][d]."""
    Hkv, _, d = rows[0].shape
    dev = rows[0].device
    pool = torch.zeros(n_pages, Hkv, page_size, d, dtype=rows[0].dtype, device=dev)
    for b, x in enumerate(rows):
        T = x.shape[1]
        n = pages_needed(T, page_size)
        pad = n * page_size - T
        xp = torch.nn.functional.pad(x, (0, 0, 0, pad)) if pad else x
        xp = xp.reshape(Hkv, n, page_size, d).permute(1, 0, 2, 3)
        idx = torch.as_tensor(block_table[b, :n].astype(np.int64), device=dev)
        pool[idx] = xp
    return pool


def from_pages(pool: torch.Tensor, block_table: np.ndarray, seq_lens) -> List[torch.Tensor]:
    """Inverse of to_pages: per-sequence [Hkv][T_b][d] rows in slot order."""
    n_pages, Hkv, P, d = pool.shape
    out = []
    for b, T in enumerate(seq_lens):
        n = pages_needed(T, P)
        idx = torch.as_tensor(block_table[b, :n].astype(np.int64), device=pool.device)
        x = pool[idx].permute(1, 0, 2, 3).reshape(Hkv, n * P, d)[:, :T]
        out.append(x)
    return out
