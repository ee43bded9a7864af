"""wi_decode_noalloc, the decode entry point that allocates nothing.

Callers that cannot allocate device memory where they decode (code inside a
CUDA stream capture, serving loops whose device memory all belongs to a fixed
arena, C callers in runtimes without a device allocator) call
wi_decode_noalloc, whose workspace is a fixed array inside the library.  It
runs the same kernels as wi_decode on the same inputs, so its output must be
bit-identical to wi_decode's, call after call: the array keeps the previous
call's contents, so a second call with another query, and a third after a
call of another geometry, check that nothing stale leaks into the next
result.  (The refusal of oversized decodes is a host-side check, tested in
test_abi.py without a GPU.)
"""
import pytest
import torch

import retrieval_sparse_attention_wave_b200 as W
import wave_inputs as WI
from tests import wave_harness as H

pytestmark = pytest.mark.gpu
DEV = "cuda"


def small_index(seq_lens, seed, n_centers=48):
    wl = WI.mixture_workload("noalloc", seq_lens=list(seq_lens), n_q_heads=8, n_kv_heads=2,
                             head_dim=128, n_centers=n_centers, seg_len=1024, cluster_size=16,
                             iters=3, topk_fraction=0.05, seed=seed, device=DEV)
    kv = H.paged_kv(wl, DEV, shuffle_seed=3)
    wx = W.build_index(kv, wl.seg_len, wl.cluster_size, wl.iters)
    return wl, wx


def same_as_decode(q, wx, p):
    ref_out, ref_lse = W.decode(q, wx, p)
    out, lse = W.decode_noalloc(q, wx, p)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    assert torch.equal(lse, ref_lse)


def test_noalloc_matches_decode_on_two_calls():
    wl, wx = small_index([5000, 2900], seed=31)
    p = H.params_of(wl)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(5)
    queries = [wl.q.to(DEV), WI.drift_queries(wl, gen, sigma=0.5).to(DEV)]
    for q in queries:                       # two calls in a row, different queries
        same_as_decode(q, wx, p)


def test_noalloc_after_a_larger_decode_leaves_nothing_stale():
    big, wxb = small_index([9000, 7000, 3000], seed=41)
    small, wxs = small_index([2500], seed=43, n_centers=24)
    same_as_decode(big.q.to(DEV), wxb, H.params_of(big))
    same_as_decode(small.q.to(DEV), wxs, H.params_of(small))
    same_as_decode(big.q.to(DEV), wxb, H.params_of(big, topk_clusters=3))
