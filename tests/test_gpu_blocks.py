"""The block top-k workload on the GPU (Vortex summary, section 2.A:
forward_cache builds block centroids, forward_indexer selects the top-k
blocks and attends; its results name the workload "block top-k").

* The block index (wi_build_blocks) equals the oracle's: offsets, perm,
  invperm and labels exactly, rows copied bit-exactly, centroids and value
  sums within one unit in the last place of the KV dtype.
* Exact-only decode (no estimation zone) matches the oracle's exact-only
  decode, on a block index and on a k-means index, on the tensor-core path
  (bf16, d = 128) and the CUDA-core path (fp32, d = 64), with the retrieved
  sets identical up to near-ties; retrieving every block gives dense
  attention.
"""
import numpy as np
import pytest
import torch

import oracle as O
import retrieval_sparse_attention_wave_b200 as W
from tests import wave_harness as H
from tests.test_gpu_build import ulp
from tests.test_gpu_decode import STRICT, check_decode, small_wl

pytestmark = pytest.mark.gpu
DEV = "cuda"

SHAPES = [dict(), dict(dtype=torch.float32, d=64, Hq=16, Hkv=2, seq_lens=(1200, 2049, 17))]


def oracle_blocks(wl):
    keys, vals = H.host_rows(wl)
    return {(b, h): O.build_blocks_unit(keys[b][h], vals[b][h], wl.seg_len, wl.cluster_size,
                                        H.store_name(wl.dtype))
            for b in range(wl.batch) for h in range(wl.n_kv_heads)}


@pytest.mark.parametrize("shape", SHAPES)
def test_block_index_equals_oracle(shape):
    wl = small_wl(**shape)
    kv = H.paged_kv(wl, DEV, shuffle_seed=9)
    bt, n_pages = H.out_block_table(wl, DEV, shuffle_seed=4)
    wx = W.build_blocks(kv, wl.seg_len, wl.cluster_size, block_table=bt, n_pages=n_pages)
    torch.cuda.synchronize()
    assert W.read_device_status(wx._build_ws) == 0
    keys, vals = H.host_rows(wl)
    for (b, h), ref in oracle_blocks(wl).items():
        g = H.download_unit(wx, b, h)
        for f in ("offsets", "perm", "invperm", "labels"):
            assert np.array_equal(g[f], getattr(ref, f)), f
        np.testing.assert_array_equal(g["k_perm"], keys[b][h])
        np.testing.assert_array_equal(g["v_perm"], vals[b][h])
        assert np.all(np.abs(g["centroids"] - ref.centroids) <= ulp(ref.centroids, wl.dtype))
        assert np.all(np.abs(g["value_sums"] - ref.value_sums) <= ulp(ref.value_sums, wl.dtype))


@pytest.mark.parametrize("shape", SHAPES)
def test_exact_only_decode_on_block_index(shape):
    wl = small_wl(**shape)
    worst, _ = check_decode(wl, oracle_blocks(wl), H.params_of(wl, exact_only=True), shuffle_seed=5)
    assert worst <= STRICT[wl.dtype]


@pytest.mark.parametrize("shape", SHAPES)
def test_exact_only_decode_on_kmeans_index(shape):
    wl = small_wl(**shape)
    check_decode(wl, H.oracle_build(wl), H.params_of(wl, exact_only=True), shuffle_seed=5)


def test_exact_only_every_block_is_dense():
    wl = small_wl(seq_lens=(3100,))
    check_decode(wl, oracle_blocks(wl), H.params_of(wl, exact_only=True, topk_clusters=100000),
                 ref_dense=True)


def test_exact_only_on_the_gpu_built_block_index():
    """Exact-only decode over the index wi_build_blocks wrote (downloaded,
    then decoded by both sides from the same values)."""
    wl = small_wl()
    kv = H.paged_kv(wl, DEV, shuffle_seed=9)
    bt, n_pages = H.out_block_table(wl, DEV, shuffle_seed=4)
    wx = W.build_blocks(kv, wl.seg_len, wl.cluster_size, block_table=bt, n_pages=n_pages)
    torch.cuda.synchronize()
    units = {(b, h): H.as_unit_index(H.download_unit(wx, b, h))
             for b in range(wl.batch) for h in range(wl.n_kv_heads)}
    worst, _ = check_decode(wl, units, H.params_of(wl, exact_only=True), shuffle_seed=5)
    assert worst <= STRICT[wl.dtype]
