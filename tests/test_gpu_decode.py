"""Decode parity: the CUDA path through the C ABI against the fp64 oracle on
the same seeded inputs and the same (oracle-built) index.

Checked per unit: centroid scores (a1), the retrieved set (a2: identical
except clusters whose score lies within 1e-5 relative of the k-th), and the
merged output and lse (a3-a6) within the benchmark spec's tolerance: max|d|/max|ref|
<= 1e-5 for fp32 inputs, max|d|/rms(ref) <= 2e-2 for bf16 inputs.  A second,
tighter bound, 2e-4 of rms(ref), catches bugs the loose bf16 tolerance would
hide: both sides decode the same stored index values, and the GPU departs
from the oracle only by fp32 accumulation and the two-term bf16 split of the
softmax weights (about 2^-17 relative), far below it.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import retrieval_sparse_attention_wave_b200 as W
import wave_inputs as WI
from tests import wave_harness as H

pytestmark = pytest.mark.gpu
DEV = "cuda"
STRICT = {torch.float32: 1e-5, torch.bfloat16: 2e-4}


def check_decode(wl, units, params, *, shuffle_seed=None, page_size=None, ref_dense=False,
                 allow_near_ties=True):
    wx = H.empty_index(wl, DEV, shuffle_seed, page_size)
    H.upload_index(wx, units)
    q = wl.q.to(DEV)
    ws = W.decode_workspace(wx, params)
    params.scores_out = W.scores_buffer(wx, wl.n_q_heads)
    out, lse = W.decode(q, wx, params, ws=ws)
    torch.cuda.synchronize()
    assert W.read_device_status(ws) == 0
    lay = W.decode_layout(wx, params)
    U = wl.batch * wl.n_kv_heads
    info = W.unit_info(ws, lay, U).cpu().numpy()
    G = wl.n_q_heads // wl.n_kv_heads
    qh = H.q_host(wl)
    out_g = out.cpu().numpy().astype(np.float64)
    lse_g = lse.cpu().numpy().astype(np.float64)
    keys, vals = H.host_rows(wl) if ref_dense else (None, None)
    worst = 0.0
    for (b, h), ix in sorted(units.items()):
        u = b * wl.n_kv_heads + h
        NC = len(ix.centroids)
        k = O.k_for(NC, params.topk_clusters, params.topk_fraction)
        qg = qh[b, h * G:(h + 1) * G]
        est = not params.exact_only
        tr = O.decode_unit(qg, ix, params.n_sink, params.window, k, estimate=est)
        # (a1) scores
        sc = W.centroid_scores(params.scores_out, wx, b, h).cpu().numpy().astype(np.float64)
        if not info[u, 6]:
            smax = np.max(np.abs(tr.scores))
            assert np.max(np.abs(sc - tr.scores.T)) <= 1e-5 * max(smax, 1.0)
        # (a2) the retrieved set
        n_sel = int(info[u, 0])
        gsel = W.selected_clusters(ws, lay, wx, b, h, n_sel).cpu().numpy().astype(np.int64)
        assert n_sel == len(tr.selected), (n_sel, len(tr.selected))
        assert np.all(np.diff(gsel) > 0)
        if not np.array_equal(gsel, tr.selected):
            assert allow_near_ties
            diff = np.setxor1d(gsel, tr.selected)
            kth = np.sort(tr.sel_score[tr.selected])[0]
            assert np.all(np.abs(tr.sel_score[diff] - kth) <= 1e-5 * abs(kth)), \
                f"unit {(b, h)}: sets differ beyond near-ties"
            tr = O.decode_unit(qg, ix, params.n_sink, params.window, k, selected=gsel,
                               estimate=est)
        # the retrieved clusters' tokens, counted once each
        if info[u, 6]:
            assert int(info[u, 3]) == 0
        else:
            assert int(info[u, 3]) == int(sum(ix.offsets[c + 1] - ix.offsets[c] for c in gsel))
        # (a3-a6) output and lse
        og = out_g[b, h * G:(h + 1) * G]
        err = H.rel_err(og, tr.out, wl.dtype)
        worst = max(worst, err)
        assert err <= H.TOL[wl.dtype], (b, h, err)
        assert err <= STRICT[wl.dtype], (b, h, err)
        np.testing.assert_allclose(lse_g[b, h * G:(h + 1) * G], tr.lse, rtol=2e-6, atol=2e-5)
        if ref_dense:
            dense, dlse = O.dense_attention(qg, keys[b][h], vals[b][h])
            assert H.rel_err(og, dense, wl.dtype) <= STRICT[wl.dtype]
            np.testing.assert_allclose(lse_g[b, h * G:(h + 1) * G], dlse, rtol=2e-6, atol=2e-5)
    return worst, info


def small_wl(seq_lens=(5000, 3333), Hq=8, Hkv=2, d=128, dtype=torch.bfloat16, seg=1024, cs=16,
             iters=3, topk=-1, frac=0.05, n_sink=4, window=64, seed=11, page=16):
    return WI.mixture_workload("small", seq_lens=list(seq_lens), n_q_heads=Hq, n_kv_heads=Hkv,
                               head_dim=d, n_centers=48, dtype=dtype, seg_len=seg, cluster_size=cs,
                               iters=iters, n_sink=n_sink, window=window, topk_clusters=topk,
                               topk_fraction=frac, page_size=page, seed=seed, device=DEV)


def test_tiny_fp32_config_full_size():
    """The tiny fp32 workload (T=4096, d=64, one head) at its full size."""
    wl = WI.config(1)
    units = H.oracle_build(wl)
    worst, _ = check_decode(wl, units, H.params_of(wl))
    assert worst <= 1e-5


@pytest.mark.parametrize("shape", [
    dict(),                                                   # bf16 d128 G4, ragged pair
    dict(d=64, Hq=8, Hkv=1, seq_lens=(2500,), seg=512),       # bf16 d64 G8
    dict(dtype=torch.float32, Hq=4, Hkv=2, seq_lens=(3000, 700)),  # fp32 d128 G2
    dict(Hq=3, Hkv=3, seq_lens=(1900,), page=64),             # G1, page 64
    dict(dtype=torch.float32, d=64, Hq=16, Hkv=2, seq_lens=(1200, 2049, 17)),  # fp32 d64 G8
])
def test_decode_shapes(shape):
    wl = small_wl(**shape)
    units = H.oracle_build(wl)
    check_decode(wl, units, H.params_of(wl), shuffle_seed=5)


@pytest.fixture(scope="module")
def base():
    wl = small_wl(seq_lens=(4100,), Hq=8, Hkv=2)
    return wl, H.oracle_build(wl)


@pytest.mark.parametrize("over", [
    dict(topk_clusters=0),                       # estimation + steady only
    dict(topk_clusters=1),
    dict(topk_clusters=100000),                  # everything retrieved: dense
    dict(n_sink=0, window=0),                    # no steady zone
    dict(n_sink=4100, window=0),                 # all steady: dense
    dict(n_sink=0, window=5000),
    dict(n_sink=2000, window=2100),              # steady covers all by union
    dict(n_sink=37, window=333),
    dict(topk_clusters=-1, topk_fraction=1.0),
    dict(topk_clusters=-1, topk_fraction=0.0),
])
def test_decode_edge_cases(base, over):
    wl, units = base
    p = H.params_of(wl, **over)
    dense = over.get("topk_clusters", 0) >= 100000 or over.get("n_sink", 0) >= 4100 \
        or over.get("window", 0) >= 4100 or over.get("topk_fraction", 0) == 1.0 \
        or (over.get("n_sink", 0) + over.get("window", 0) >= 4100)
    check_decode(wl, units, p, ref_dense=dense)


def test_whole_clusters_inside_the_window():
    """Segments of one cluster each: the window swallows whole clusters,
    which then are neither candidates nor estimated."""
    wl = small_wl(seq_lens=(1000,), seg=16, cs=16, topk=5)
    units = H.oracle_build(wl)
    _, info = check_decode(wl, units, H.params_of(wl))
    assert np.all(info[:, 5] >= 4)   # at least the 4 window clusters are affected


def test_one_token_clusters_are_exact():
    """cluster_size 1: the estimate is exact, so any budget gives dense attention."""
    wl = small_wl(seq_lens=(700,), cs=1, seg=256, topk=9, dtype=torch.float32)
    units = H.oracle_build(wl)
    check_decode(wl, units, H.params_of(wl), ref_dense=True)


@pytest.mark.parametrize("seq_lens", [(1,), (7,), (16,), (17, 1, 40)])
def test_tiny_sequences(seq_lens):
    wl = small_wl(seq_lens=seq_lens, topk=1, n_sink=2, window=3)
    units = H.oracle_build(wl)
    check_decode(wl, units, H.params_of(wl))


def test_page_size_one():
    wl = small_wl(seq_lens=(600, 301), page=1)
    units = H.oracle_build(wl)
    check_decode(wl, units, H.params_of(wl), shuffle_seed=3, page_size=1)


def test_decode_host_buffers_match_device_call(base):
    wl, units = base
    p = H.params_of(wl)
    wx = H.empty_index(wl, DEV)
    H.upload_index(wx, units)
    ws = W.decode_workspace(wx, p)
    out_d, lse_d = W.decode(wl.q.to(DEV), wx, p, ws=ws)
    qh = wl.q.cpu().pin_memory()
    out_h = torch.empty(out_d.shape, dtype=torch.float32).pin_memory()
    lse_h = torch.empty(lse_d.shape, dtype=torch.float32).pin_memory()
    W.decode_host(qh, wx, p, out_h, lse_h, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())


def test_decode_host_pageable_and_unaligned_outputs(base):
    """Pageable host buffers take the copy path; pinned outputs that are
    only 4-byte aligned are written directly, by scalar stores.  Both give
    the device call's result bit for bit."""
    wl, units = base
    p = H.params_of(wl)
    wx = H.empty_index(wl, DEV)
    H.upload_index(wx, units)
    ws = W.decode_workspace(wx, p)
    out_d, lse_d = W.decode(wl.q.to(DEV), wx, p, ws=ws)
    torch.cuda.synchronize()
    n, m = out_d.numel(), lse_d.numel()
    out_h = torch.full(out_d.shape, float("nan"), dtype=torch.float32)
    lse_h = torch.full(lse_d.shape, float("nan"), dtype=torch.float32)
    W.decode_host(wl.q.cpu(), wx, p, out_h, lse_h, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())
    buf = torch.full((n + m + 2,), float("nan"), dtype=torch.float32).pin_memory()
    out_u = buf[1:1 + n].view(out_d.shape)          # 4 bytes past a 16-byte boundary
    lse_u = buf[1 + n:1 + n + m].view(lse_d.shape)
    W.decode_host(wl.q.cpu().pin_memory(), wx, p, out_u, lse_u, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_u, out_d.cpu()) and torch.equal(lse_u, lse_d.cpu())
    assert torch.isnan(buf[0]) and torch.isnan(buf[-1])   # nothing written outside
    out_x = torch.full((n + 1,), float("nan"), dtype=torch.float32, device=DEV)[1:].view(out_d.shape)
    W.decode(wl.q.to(DEV), wx, p, out=out_x, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(out_x, out_d)
    assert W.read_device_status(ws) == 0


def test_decode_host_graph_replays_match(base):
    """Repeated host-buffer calls with the same buffers on a side stream: the
    second captures a graph of the copies and kernels, the later ones replay
    it; every call's output equals the device call's, also after q changes
    (the graph copies the host buffer's current contents)."""
    wl, units = base
    p = H.params_of(wl)
    wx = H.empty_index(wl, DEV)
    H.upload_index(wx, units)
    ws = W.decode_workspace(wx, p)
    q2 = (wl.q.float() * 0.5).to(wl.q.dtype)
    ref = [W.decode(x.to(DEV), wx, p, ws=ws) for x in (wl.q, q2)]
    torch.cuda.synchronize()
    qh = wl.q.cpu().pin_memory()
    out_h = torch.empty(ref[0][0].shape, dtype=torch.float32).pin_memory()
    lse_h = torch.empty(ref[0][1].shape, dtype=torch.float32).pin_memory()
    st = torch.cuda.Stream()
    for i in range(5):
        src = wl.q if i < 3 else q2
        qh.copy_(src)
        out_h.zero_()
        W.decode_host(qh, wx, p, out_h, lse_h, ws, stream=st)
        st.synchronize()
        o, l = ref[0] if i < 3 else ref[1]
        assert torch.equal(out_h, o.cpu()) and torch.equal(lse_h, l.cpu()), i
    assert W.read_device_status(ws) == 0


def test_repeat_runs_are_bit_identical(base):
    wl, units = base
    p = H.params_of(wl)
    wx = H.empty_index(wl, DEV)
    H.upload_index(wx, units)
    ws = W.decode_workspace(wx, p)
    a, la = W.decode(wl.q.to(DEV), wx, p, ws=ws)
    a, la = a.clone(), la.clone()
    b, lb = W.decode(wl.q.to(DEV), wx, p, ws=ws)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_corrupt_block_table_is_flagged_not_faulted(base):
    """Device-side index checks: an out-of-range page id is skipped and
    reported in the status word; the context stays usable."""
    wl, units = base
    p = H.params_of(wl)
    wx = H.empty_index(wl, DEV)
    H.upload_index(wx, units)
    # the page holding the slot of position 0 (a sink token, always attended)
    slot0 = int(wx.invperm[wx.tok_row(0, 0)].item())
    wx.block_table[0, slot0 // wx.page_size] = wx.k_pool.shape[0] + 1000
    ws = W.decode_workspace(wx, p)
    W.decode(wl.q.to(DEV), wx, p, ws=ws)
    flags = W.read_device_status(ws)
    assert flags & W.WI_DEV_BAD_PAGE
    assert W.read_device_status(ws) == 0          # cleared
    torch.cuda.synchronize()
