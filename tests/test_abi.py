"""The C-ABI boundary on the host: the library loads, exports every symbol
include/wi.h declares, and rejects bad arguments with status codes before any
CUDA call (so these run without a GPU)."""
import ctypes as C
import os
import re

import pytest

import retrieval_sparse_attention_wave_b200 as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x7f0000000000          # 256-byte aligned, never dereferenced


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "wi.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wi_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(W.lib(), n), n
    assert sorted(names) == sorted(W.EXPORTED)


def test_stage_names():
    assert W.stage_names() == ["steady", "scan", "gather"]
    assert W.lib().wi_decode_stage_name(99) is None


def test_index_clusters_counts():
    assert W.clusters_per_sequence([131072], 8192, 16) == [8192]
    assert W.clusters_per_sequence([4196, 1, 17], 1024, 16) == [263, 1, 2]
    tot = C.c_int64()
    arr = (C.c_int32 * 1)(100)
    assert W.lib().wi_index_clusters(1, arr, 30, 16, None, C.byref(tot)) == W.WI_ERR_INVALID_ARG
    assert W.lib().wi_index_clusters(1, arr, 32768, 16, None, C.byref(tot)) == W.WI_ERR_UNSUPPORTED


def kv_struct(**over):
    seq = over.pop("seq", [4096])
    s = W.WiKVCache()
    s.dtype = W.WI_BF16
    s.batch = len(seq)
    s.n_kv_heads, s.head_dim, s.page_size = 8, 128, 16
    s.n_pages = 4096
    s.k_pool = FAKE
    s.v_pool = FAKE + 0x10000000
    s.block_table = FAKE + 0x20000000
    s.max_pages = 4096
    s._seq = (C.c_int32 * len(seq))(*seq)
    s.seq_lens = C.cast(s._seq, C.POINTER(C.c_int32))
    for k, v in over.items():
        setattr(s, k, v)
    return s


def index_struct(**over):
    seq = over.pop("seq", [4096])
    s = W.WiIndex()
    s.dtype = W.WI_BF16
    s.batch = len(seq)
    s.n_kv_heads, s.head_dim, s.page_size, s.seg_len, s.cluster_size = 8, 128, 16, 1024, 16
    s._seq = (C.c_int32 * len(seq))(*seq)
    s.seq_lens = C.cast(s._seq, C.POINTER(C.c_int32))
    for i, f in enumerate(["centroids", "value_sums", "offsets", "perm", "invperm", "labels",
                           "k_pool", "v_pool", "block_table"]):
        setattr(s, f, FAKE + (i + 1) * 0x1000000)
    s.n_pages = 4096
    s.max_pages = 4096
    for k, v in over.items():
        setattr(s, k, v)
    return s


def params(**over):
    p = W.WiDecodeParams()
    p.n_q_heads, p.n_sink, p.window, p.topk_clusters, p.topk_fraction = 32, 4, 64, -1, 0.018
    for k, v in over.items():
        setattr(p, k, v)
    return p


def ws_size(ix, p):
    n = C.c_size_t()
    st = W.lib().wi_decode_workspace_size(C.byref(ix), C.byref(p), C.byref(n))
    return st, n.value


def test_decode_workspace_size_and_layout():
    st, n = ws_size(index_struct(), params())
    assert st == W.WI_OK and n > 0 and n % 256 == 0
    lay = W.WiDecodeLayout()
    assert W.lib().wi_decode_workspace_layout(C.byref(index_struct()), C.byref(params()),
                                              C.byref(lay)) == W.WI_OK
    assert lay.total_bytes == n and lay.status == 0
    assert 0 < lay.records < lay.selected < n and 0 < lay.unit_info < n
    assert lay.n_scan_ctas >= 1 and lay.n_gather_ctas >= 8 and lay.info_ints == 16


@pytest.mark.parametrize("dtype,d,seq,expect", [
    # 131072 tokens, 8 KV heads: 8192 clusters per head -> 128 chunks of 64,
    # 1024 chunks on 148 streaming CTAs; k = ceil(0.018 * 8192) = 148, so a
    # head expects 148 * 16 retrieved + 68 steady + 148 + 68 correction rows
    # = 2652 rows, plus half: 3978 -> 32 gather CTAs of 128 rows per head
    (W.WI_BF16, 128, [131072], dict(n_scan_ctas=148, n_gather_ctas=256)),
    # fp32: the same chunking (64-row tiles whatever the row size)
    (W.WI_F32, 128, [131072], dict(n_scan_ctas=148, n_gather_ctas=256)),
    # ragged batch: 256 clusters (4 chunks) and 19 clusters (1 chunk) per
    # head -> 40 chunks, 40 CTAs; 221 and 153 expected rows, plus half
    # (331, 229) -> 3 + 2 gather CTAs per head
    (W.WI_BF16, 128, [4096, 300], dict(n_scan_ctas=40, n_gather_ctas=40)),
])
def test_decode_plan_shapes(dtype, d, seq, expect):
    """The launch plan's CTA counts, from the geometry alone (host logic)."""
    lay = W.WiDecodeLayout()
    ix = index_struct(seq=seq, dtype=dtype, head_dim=d, n_pages=16384, max_pages=16384)
    assert W.lib().wi_decode_workspace_layout(C.byref(ix), C.byref(params()), C.byref(lay)) \
        == W.WI_OK
    for k, v in expect.items():
        assert getattr(lay, k) == v, (k, getattr(lay, k), v)
    # the exact-only workload keeps no estimation parts and fewer rows
    lay2 = W.WiDecodeLayout()
    assert W.lib().wi_decode_workspace_layout(C.byref(ix), C.byref(params(exact_only=1)),
                                              C.byref(lay2)) == W.WI_OK
    assert lay2.total_bytes < lay.total_bytes
    assert lay2.n_gather_ctas <= lay.n_gather_ctas


@pytest.mark.parametrize("over,expect", [
    (dict(n_q_heads=0), W.WI_ERR_INVALID_ARG),
    (dict(n_q_heads=31), W.WI_ERR_INVALID_ARG),       # not a multiple of Hkv
    (dict(n_q_heads=8 * 16), W.WI_ERR_UNSUPPORTED),   # G = 16
    (dict(n_q_heads=8 * 3), W.WI_ERR_UNSUPPORTED),    # G = 3
    (dict(n_sink=-1), W.WI_ERR_INVALID_ARG),
    (dict(window=-5), W.WI_ERR_INVALID_ARG),
    (dict(topk_clusters=-1, topk_fraction=1.5), W.WI_ERR_INVALID_ARG),
    (dict(n_sink=5000, window=5000), W.WI_OK),        # all steady (dense) is legal
    (dict(n_sink=8000, window=192), W.WI_OK),         # exactly WI_MAX_STEADY
    (dict(topk_mode=1, seed=7), W.WI_OK),              # sampled threshold bin
    (dict(topk_mode=2), W.WI_ERR_INVALID_ARG),         # no such selection mode
    (dict(scores_out=FAKE + 2), W.WI_ERR_INVALID_ARG),  # misaligned score buffer
])
def test_decode_param_validation(over, expect):
    st, _ = ws_size(index_struct(seq=[10000]), params(**over))
    assert st == expect


def test_steady_limit_is_reported():
    st, _ = ws_size(index_struct(seq=[100000], max_pages=8192), params(n_sink=5000, window=5000))
    assert st == W.WI_ERR_UNSUPPORTED
    st, _ = ws_size(index_struct(seq=[10000]), params(n_sink=8000, window=193))
    assert st == W.WI_ERR_UNSUPPORTED


@pytest.mark.parametrize("over,expect", [
    (dict(head_dim=96), W.WI_ERR_UNSUPPORTED),
    (dict(head_dim=0), W.WI_ERR_INVALID_ARG),
    (dict(page_size=12), W.WI_ERR_INVALID_ARG),
    (dict(dtype=7), W.WI_ERR_INVALID_ARG),
    (dict(centroids=None), W.WI_ERR_INVALID_ARG),
    (dict(perm=FAKE + 2), W.WI_ERR_INVALID_ARG),       # misaligned
    (dict(k_pool=FAKE + 8), W.WI_ERR_INVALID_ARG),     # not 16-byte aligned
    (dict(seg_len=1000), W.WI_ERR_INVALID_ARG),        # not a multiple of cluster_size
    (dict(seg_len=32768), W.WI_ERR_UNSUPPORTED),
    (dict(max_pages=10), W.WI_ERR_INVALID_ARG),        # 4096 tokens need 256 pages
    (dict(seq=[0]), W.WI_ERR_INVALID_ARG),
    (dict(seq=[16] * 300), W.WI_ERR_UNSUPPORTED),      # batch > WI_MAX_BATCH
])
def test_index_validation(over, expect):
    st, _ = ws_size(index_struct(**over), params())
    assert st == expect


def test_decode_rejects_before_any_cuda_call():
    ix, p = index_struct(), params()
    lib = W.lib()
    # null q / out
    assert lib.wi_decode(None, C.byref(ix), C.byref(p), FAKE, None, FAKE, 1 << 30, None) \
        == W.WI_ERR_INVALID_ARG
    assert lib.wi_decode(FAKE, C.byref(ix), C.byref(p), None, None, FAKE, 1 << 30, None) \
        == W.WI_ERR_INVALID_ARG
    # workspace missing, too small, misaligned
    _, need = ws_size(ix, p)
    assert lib.wi_decode(FAKE, C.byref(ix), C.byref(p), FAKE, None, None, need, None) \
        == W.WI_ERR_WORKSPACE
    assert lib.wi_decode(FAKE, C.byref(ix), C.byref(p), FAKE, None, FAKE, need - 1, None) \
        == W.WI_ERR_WORKSPACE
    assert lib.wi_decode(FAKE, C.byref(ix), C.byref(p), FAKE, None, FAKE + 16, need, None) \
        == W.WI_ERR_WORKSPACE
    assert lib.wi_decode_host(None, C.byref(ix), C.byref(p), FAKE, None, FAKE, need, None) \
        == W.WI_ERR_INVALID_ARG


def test_build_validation():
    lib = W.lib()
    kv = kv_struct()
    n = C.c_size_t()
    assert lib.wi_build_workspace_size(C.byref(kv), 1024, 16, C.byref(n)) == W.WI_OK
    assert n.value >= 8 * 4096 * 4
    out = index_struct()
    # iters < 1
    assert lib.wi_build_index(C.byref(kv), 1024, 16, 0, C.byref(out), FAKE, n.value, None) \
        == W.WI_ERR_INVALID_ARG
    # geometry mismatch between input and output
    assert lib.wi_build_index(C.byref(kv), 512, 16, 3, C.byref(out), FAKE, n.value, None) \
        == W.WI_ERR_INVALID_ARG
    # output pools aliasing the input pools
    alias = index_struct(k_pool=kv.k_pool)
    assert lib.wi_build_index(C.byref(kv), 1024, 16, 3, C.byref(alias), FAKE, n.value, None) \
        == W.WI_ERR_INVALID_ARG
    # workspace too small
    assert lib.wi_build_index(C.byref(kv), 1024, 16, 3, C.byref(out), FAKE, 1024, None) \
        == W.WI_ERR_WORKSPACE
    assert lib.wi_kmeans_assign(C.byref(kv), 1024, 16, None, FAKE, FAKE, n.value, None) \
        == W.WI_ERR_INVALID_ARG


def test_build_blocks_validation():
    lib = W.lib()
    kv = kv_struct()
    n = C.c_size_t()
    assert lib.wi_build_workspace_size(C.byref(kv), 1024, 16, C.byref(n)) == W.WI_OK
    out = index_struct()                       # cluster_size 16
    assert lib.wi_build_blocks(C.byref(kv), 1024, 32, C.byref(out), FAKE, n.value, None) \
        == W.WI_ERR_INVALID_ARG                # block size other than the index's
    alias = index_struct(k_pool=kv.k_pool)
    assert lib.wi_build_blocks(C.byref(kv), 1024, 16, C.byref(alias), FAKE, n.value, None) \
        == W.WI_ERR_INVALID_ARG
    assert lib.wi_build_blocks(C.byref(kv), 1024, 16, C.byref(out), FAKE, 1024, None) \
        == W.WI_ERR_WORKSPACE


def test_extend_validation():
    """wi_extend_index checks every argument before any launch."""
    lib = W.lib()
    kv = kv_struct(seq=[4096])
    n = C.c_size_t()
    assert lib.wi_build_workspace_size(C.byref(kv), 1024, 16, C.byref(n)) == W.WI_OK
    out = index_struct(seq=[4096])
    old = index_struct(seq=[3000], **{f: FAKE + (20 + i) * 0x1000000 for i, f in enumerate(
        ["centroids", "value_sums", "offsets", "perm", "invperm", "labels"])})
    ext = lambda o, k, it, x, nb: lib.wi_extend_index(o, k, it, x, FAKE, nb, None)
    assert ext(None, C.byref(kv), 3, C.byref(out), n.value) == W.WI_ERR_INVALID_ARG
    assert ext(C.byref(old), C.byref(kv), 0, C.byref(out), n.value) == W.WI_ERR_INVALID_ARG
    # the old index longer than the new sequences
    longer = index_struct(seq=[5000], **{f: getattr(old, f) for f in ["centroids", "value_sums",
                                                                      "offsets", "perm",
                                                                      "invperm", "labels"]})
    assert ext(C.byref(longer), C.byref(kv), 3, C.byref(out), n.value) == W.WI_ERR_INVALID_ARG
    # the new index reusing one of the old index's buffers
    reuse = index_struct(seq=[4096], perm=old.perm)
    assert ext(C.byref(old), C.byref(kv), 3, C.byref(reuse), n.value) == W.WI_ERR_INVALID_ARG
    # another segment length than the old index
    other = index_struct(seq=[3000], seg_len=512)
    assert ext(C.byref(other), C.byref(kv), 3, C.byref(out), n.value) == W.WI_ERR_INVALID_ARG
    # workspace too small
    assert ext(C.byref(old), C.byref(kv), 3, C.byref(out), 1024) == W.WI_ERR_WORKSPACE


def test_status_strings():
    lib = W.lib()
    for s in range(6):
        assert lib.wi_status_string(s)
    assert lib.wi_read_device_status(None, None, None, 0) == W.WI_ERR_INVALID_ARG


def test_selection_list_decoding_on_the_host():
    """The binding reads a unit's retrieved ids from its rows of the
    selection list (laid out like the centroids) and checks them."""
    import types

    import torch
    lay = types.SimpleNamespace(selected=256)
    index = types.SimpleNamespace(n_kv_heads=2, nc=[10, 7],
                                  cl_row=lambda b, h: 2 * sum([10, 7][:b]) + h * [10, 7][b])
    ws = torch.zeros(256 + 4 * 34, dtype=torch.uint8)
    ids = ws[256:].view(torch.int32)
    want = {(0, 1): [0, 3, 9], (1, 0): [2, 5, 6]}
    for (b, h), xs in want.items():
        r = index.cl_row(b, h)
        ids[r:r + len(xs)] = torch.tensor(xs, dtype=torch.int32)
    for (b, h), xs in want.items():
        assert W.selected_clusters(ws, lay, index, b, h, len(xs)).tolist() == xs
    assert W.selected_clusters(ws, lay, index, 0, 0, 0).tolist() == []
    with pytest.raises(RuntimeError):       # more than the unit's clusters
        W.selected_clusters(ws, lay, index, 1, 0, 8)
    ids[index.cl_row(1, 0)] = 9             # not ascending
    with pytest.raises(RuntimeError):
        W.selected_clusters(ws, lay, index, 1, 0, 3)


def test_noalloc_refuses_on_the_host():
    """wi_decode_noalloc refuses a decode whose workspace exceeds its fixed
    scratch, and bad q / out / lse, before any CUDA call: the pointers are
    never dereferenced."""
    lib = W.lib()
    seq = (C.c_int32 * 1)(4_000_000)
    ix = W.WiIndex()
    ix.dtype, ix.batch, ix.n_kv_heads, ix.head_dim = W.WI_BF16, 1, 8, 128
    ix.page_size, ix.seg_len, ix.cluster_size = 16, 8192, 16
    ix.seq_lens = C.cast(seq, C.POINTER(C.c_int32))
    for i, f in enumerate(["centroids", "value_sums", "offsets", "perm", "invperm", "labels",
                           "k_pool", "v_pool", "block_table"]):
        setattr(ix, f, FAKE + (i + 1) * 0x10000000)
    ix.n_pages, ix.max_pages = 250_000, 250_000
    prm = W.DecodeParams(n_q_heads=32).c_struct()
    n = C.c_size_t()
    assert lib.wi_decode_workspace_size(C.byref(ix), C.byref(prm), C.byref(n)) == W.WI_OK
    assert n.value > W.NOALLOC_SCRATCH_MIB << 20
    assert lib.wi_decode_noalloc(FAKE, C.byref(ix), C.byref(prm), FAKE, None, None) \
        == W.WI_ERR_WORKSPACE
    small = index_struct()
    p = params()
    assert lib.wi_decode_noalloc(None, C.byref(small), C.byref(p), FAKE, None, None) \
        == W.WI_ERR_INVALID_ARG
    assert lib.wi_decode_noalloc(FAKE, C.byref(small), C.byref(p), None, None, None) \
        == W.WI_ERR_INVALID_ARG
    assert lib.wi_decode_noalloc(FAKE + 8, C.byref(small), C.byref(p), FAKE, None, None) \
        == W.WI_ERR_INVALID_ARG
    assert lib.wi_decode_noalloc(FAKE, C.byref(small), C.byref(p), FAKE, FAKE + 2, None) \
        == W.WI_ERR_INVALID_ARG
