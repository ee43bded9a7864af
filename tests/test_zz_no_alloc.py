"""wi_decode_noalloc, the decode entry point that allocates nothing.

Callers that cannot allocate device memory where they decode (code inside a
CUDA stream capture, serving loops whose device memory all belongs to a fixed
arena, C callers in runtimes without a device allocator) call
wi_decode_noalloc, whose workspace is a fixed array inside the library.  Its
output must match wi_decode's on the same inputs, call after call: the array
keeps the previous call's contents, so a second call with another query
checks that nothing stale leaks into the next result.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import retrieval_sparse_attention_wave_b200 as W
import wave_inputs as WI
from tests import wave_harness as H

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_noalloc_matches_decode_on_two_calls():
    wl = WI.mixture_workload("noalloc", seq_lens=[5000, 2900], n_q_heads=8, n_kv_heads=2,
                             head_dim=128, n_centers=48, seg_len=1024, cluster_size=16,
                             iters=3, topk_fraction=0.05, seed=31, device=DEV)
    kv = H.paged_kv(wl, DEV, shuffle_seed=3)
    wx = W.build_index(kv, wl.seg_len, wl.cluster_size, wl.iters)
    p = H.params_of(wl)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(5)
    queries = [wl.q.to(DEV), WI.drift_queries(wl, gen, sigma=0.5).to(DEV)]
    for q in queries:                       # two calls in a row, different queries
        ref_out, ref_lse = W.decode(q, wx, p)
        out, lse = W.decode_noalloc(q, wx, p)
        torch.cuda.synchronize()
        ref = ref_out.cpu().numpy().astype(np.float64)
        got = out.cpu().numpy().astype(np.float64)
        assert H.rel_err(got, ref, wl.dtype) <= H.TOL[wl.dtype]
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=2e-6, atol=2e-5)


def test_noalloc_rejects_a_workspace_larger_than_its_scratch():
    """Sizes beyond the fixed scratch are refused on the host, before any GPU work."""
    seq = (C.c_int32 * 1)(4_000_000)
    ix = W.WiIndex()
    ix.dtype, ix.batch, ix.n_kv_heads, ix.head_dim = W.WI_BF16, 1, 8, 128
    ix.page_size, ix.seg_len, ix.cluster_size = 16, 8192, 16
    ix.seq_lens = C.cast(seq, C.POINTER(C.c_int32))
    fake = 0x7f0000000000
    for i, f in enumerate(["centroids", "value_sums", "offsets", "perm", "invperm", "labels",
                           "k_pool", "v_pool", "block_table"]):
        setattr(ix, f, fake + (i + 1) * 0x10000000)
    ix.n_pages, ix.max_pages = 250_000, 250_000
    prm = W.DecodeParams(n_q_heads=32).c_struct()
    n = C.c_size_t()
    assert W.lib().wi_decode_workspace_size(C.byref(ix), C.byref(prm), C.byref(n)) == W.WI_OK
    assert n.value > W.NOALLOC_SCRATCH_MIB << 20
    st = W.lib().wi_decode_noalloc(fake, C.byref(ix), C.byref(prm), fake, None, None)
    assert st == W.WI_ERR_WORKSPACE
