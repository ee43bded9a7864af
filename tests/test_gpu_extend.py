"""Index extension on the GPU (RetroInfer technical summary, section 2.A,
Segmented Clustering: segments are clustered independently, so an index grows
by clustering the segments its new tokens fill).

* extend(build(T), T') equals build(T') bit for bit: every index array and the
  permuted pools, with a partial and a whole old last segment, several
  sequences, bf16 d = 128 and fp32 d = 64, and with no new tokens at all.
* The extended index is valid against the host keys and values (the checks
  of the build parity test), and with one round from the initial centroids
  it equals the oracle's extension of the oracle's old index.
* A decode on the extended index equals one on the rebuilt index, bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle as O
import retrieval_sparse_attention_wave_b200 as W
import wave_inputs as WI
from tests import wave_harness as H
from tests.test_gpu_build import check_valid, ulp

pytestmark = pytest.mark.gpu
DEV = "cuda"
FIELDS = ("centroids", "value_sums", "offsets", "perm", "invperm", "labels", "k_pool", "v_pool")


def grow(new_lens, old_lens, dtype=torch.bfloat16, d=128, iters=4, seed=31):
    wl = WI.mixture_workload("extend", seq_lens=list(new_lens), n_q_heads=4, n_kv_heads=2,
                             head_dim=d, n_centers=40, dtype=dtype, seg_len=1024, cluster_size=16,
                             iters=iters, seed=seed, device=DEV)
    kv = H.paged_kv(wl, DEV, shuffle_seed=9)
    bt, n_pages = H.out_block_table(wl, DEV, shuffle_seed=4)   # pages for the longer sequences
    kv_old = W.KVCache(kv.k_pool, kv.v_pool, kv.block_table, list(old_lens))
    old = W.build_index(kv_old, wl.seg_len, wl.cluster_size, iters, block_table=bt, n_pages=n_pages)
    ext = W.extend_index(old, kv, iters)
    full = W.build_index(kv, wl.seg_len, wl.cluster_size, iters, block_table=bt, n_pages=n_pages)
    torch.cuda.synchronize()
    for x in (old, ext, full):
        assert W.read_device_status(x._build_ws) == 0
    return wl, kv, ext, full


@pytest.mark.parametrize("dtype,d,new_lens,old_lens", [
    (torch.bfloat16, 128, (4200, 3000), (2500, 1024)),   # partial and whole old last segment
    (torch.float32, 64, (3000, 2048, 1500), (2048, 100, 1500)),
    (torch.bfloat16, 128, (2500, 1024), (2500, 1024)),   # nothing new
])
def test_extension_equals_full_build(dtype, d, new_lens, old_lens):
    wl, kv, ext, full = grow(new_lens, old_lens, dtype, d)
    for f in FIELDS:
        assert torch.equal(getattr(ext, f), getattr(full, f)), f
    keys, vals = H.host_rows(wl)
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            check_valid(wl, ext, b, h, keys, vals)


def test_one_round_extension_equals_oracle():
    new_lens, old_lens = (3500, 2100), (1500, 2048)
    wl, kv, ext, _ = grow(new_lens, old_lens, iters=1)
    keys, vals = H.host_rows(wl)
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            T0 = old_lens[b]
            old = O.build_unit(keys[b][h][:T0], vals[b][h][:T0], wl.seg_len, wl.cluster_size, 1,
                               "bf16")
            ref = O.extend_unit(old, keys[b][h], vals[b][h], wl.seg_len, wl.cluster_size, 1,
                                "bf16")
            g = H.download_unit(ext, b, h)
            if np.array_equal(g["offsets"], ref.offsets) and np.array_equal(g["perm"], ref.perm):
                assert np.array_equal(g["labels"], ref.labels)
                assert np.all(np.abs(g["centroids"] - ref.centroids) <= ulp(ref.centroids, wl.dtype))
                assert np.all(np.abs(g["value_sums"] - ref.value_sums)
                              <= ulp(ref.value_sums, wl.dtype))
            else:   # a near-tie in the assignment: prove it for every moved token
                moved = H.assert_one_round_moves_are_near_ties(
                    keys[b][h], g["labels"], ref.labels, wl.seg_len, wl.cluster_size)
                assert 0 < moved <= 2


def test_decode_after_extension_equals_decode_after_build():
    wl, kv, ext, full = grow((4200, 3000), (2500, 1024))
    p = W.DecodeParams(n_q_heads=wl.n_q_heads, n_sink=4, window=64, topk_fraction=0.05)
    q = wl.q.to(DEV)
    o1, l1 = W.decode(q, ext, p)
    o2, l2 = W.decode(q, full, p)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.isfinite(o1).all()
