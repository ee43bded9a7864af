"""Build parity at the workloads' own segment size (8192 tokens, 512 centroids
per segment) on sampled (KV head, segment) pairs of the 131072- and the
1,048,576-token workloads (RetroInfer technical summary, section 2.A,
Segmented Clustering).

The oracle cannot cluster a whole 1M-token index in seconds, so the GPU
builds everything and the oracle checks sampled segments:

* one round from the initial centroids gives the oracle's segment exactly
  (labels, hence offsets and perm; stored centroids and value sums within one
  unit in the last place of bf16), except tokens whose two candidate
  centroids are near-ties (fp64 distances within 1e-5 relative), which are
  shown to be near-ties;
* round by round (r = 1, 5, 9): the fp32 working centroids the GPU left after
  round r are the correctly rounded means of its round-r assignment, and the
  GPU assignment of round r + 1 from those very centroids equals the
  oracle's, up to near-ties;
* after the full ten rounds the sampled segments are a valid index on their
  own terms: a permutation of the segment's positions, clusters in slot
  ranges with ascending members, rows copied bit-exactly, stored centroid /
  value sum = the rounded mean / sum of the cluster's members.
"""
import numpy as np
import pytest
import torch

import oracle as O
import retrieval_sparse_attention_wave_b200 as W
import wave_inputs as WI
from tests import wave_harness as H

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (KV head, segment) pairs of sequence 0: the first segment of head 0 and the
# last segment of the last head, plus one in the middle for the long context
PICKS = {2: [(0, 0), (7, 15)], 4: [(3, 57), (7, 127)]}


def ulp(x, bits):
    ax = np.maximum(np.abs(x), 1e-30)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(int) - (bits - 1))


def segment_rows(wl, h, g):
    s = g * wl.seg_len
    n = min(wl.seg_len, wl.seq_lens[0] - s)
    f = lambda t: t[h, s:s + n].to("cpu", torch.float64).numpy()
    return s, n, f(wl.keys[0]), f(wl.values[0])


def gpu_segment(wx, h, g, s, n):
    """Offsets, perm, invperm, labels, stored centroids / value sums and the
    permuted K/V rows of segment g of unit (0, h), segment-local."""
    S, cs = wx.seg_len, wx.cluster_size
    c0, m = g * (S // cs), O.clusters_in_segment(n, cs)
    r, o, t = wx.cl_row(0, h), wx.off_row(0, h), wx.tok_row(0, h)
    slots = torch.arange(s, s + n, device=wx.block_table.device)
    pages = wx.block_table[0].long()[slots // wx.page_size]
    rows = slots % wx.page_size
    f = lambda x: x.to(torch.float64).cpu().numpy()
    i64 = lambda x: x.cpu().numpy().astype(np.int64)
    return dict(off=i64(wx.offsets[o + c0:o + c0 + m + 1]) - s,
                perm=i64(wx.perm[t + s:t + s + n]) - s,
                inv=i64(wx.invperm[t + s:t + s + n]) - s,
                lab=i64(wx.labels[t + s:t + s + n]) - c0,
                cent=f(wx.centroids[r + c0:r + c0 + m]), vsum=f(wx.value_sums[r + c0:r + c0 + m]),
                k=f(wx.k_pool[pages, h, rows]), v=f(wx.v_pool[pages, h, rows]))


def check_segment_valid(gs, X, V):
    n, m = len(X), len(gs["off"]) - 1
    off, perm, inv = gs["off"], gs["perm"], gs["inv"]
    assert off[0] == 0 and off[-1] == n and np.all(np.diff(off) >= 0)
    assert np.array_equal(np.sort(perm), np.arange(n))
    assert np.array_equal(inv[perm], np.arange(n))
    cl = np.repeat(np.arange(m), np.diff(off))
    same = cl[1:] == cl[:-1]
    assert np.all(perm[1:][same] > perm[:-1][same])
    assert np.array_equal(gs["lab"][perm], cl)
    np.testing.assert_array_equal(gs["k"], X[perm])
    np.testing.assert_array_equal(gs["v"], V[perm])
    cnt = np.diff(off)
    nz = cnt > 0
    ks = np.zeros((m, X.shape[1]))
    vs = np.zeros((m, X.shape[1]))
    np.add.at(ks, cl, X[perm])
    np.add.at(vs, cl, V[perm])
    mean = ks[nz] / cnt[nz, None]
    assert np.all(np.abs(gs["cent"][nz] - mean) <= ulp(mean, 8) + 1e-30)
    assert np.all(np.abs(gs["vsum"] - vs) <= ulp(vs, 8) + 1e-30)
    assert np.all(gs["vsum"][~nz] == 0)
    return cl


def assert_near_ties(X, C, got, ref):
    """Tokens assigned differently must be near-ties: the GPU's centroid lies
    within 1e-5 relative of the best fp64 distance."""
    bad = np.nonzero(got != ref)[0]
    if len(bad):
        D = O.kmeans_distances(X[bad], C)
        dg = D[np.arange(len(bad)), got[bad]]
        dr = D[np.arange(len(bad)), ref[bad]]
        assert np.all(dg <= dr * (1 + 1e-5)), "assignment differs beyond near-ties"
    return len(bad)


@pytest.mark.parametrize("cfg", [2, 4])
def test_fullsize_build_sampled_segments(cfg):
    wl = WI.config(cfg, device=DEV)
    kv = H.paged_kv(wl, DEV)
    S, cs = wl.seg_len, wl.cluster_size
    picks = PICKS[cfg]
    rows = {p: segment_rows(wl, *p) for p in picks}
    wx = W.build_index(kv, S, cs, 1)
    ws = wx._build_ws
    torch.cuda.synchronize()
    assert W.read_device_status(ws) == 0

    # ---- one round from the initial centroids equals the oracle's segment
    for (h, g), (s, n, X, V) in rows.items():
        gs = gpu_segment(wx, h, g, s, n)
        cl = check_segment_valid(gs, X, V)
        lab_o, C1, _ = O.kmeans_segment(X, cs, 1)
        lab_g = np.empty(n, dtype=np.int64)
        lab_g[gs["perm"]] = cl
        moved = assert_near_ties(X, O.kmeans_init(X, cs), lab_g, lab_o)
        if moved == 0:
            ref = O.build_unit(X, V, S, cs, 1, "bf16")
            assert np.array_equal(gs["off"], ref.offsets)
            assert np.array_equal(gs["perm"], ref.perm)
            assert np.all(np.abs(gs["cent"] - ref.centroids) <= ulp(ref.centroids, 8))
            assert np.all(np.abs(gs["vsum"] - ref.value_sums) <= ulp(ref.value_sums, 8))

    # ---- round by round: update and the next assignment from the same centroids
    for r in (1, 5, 9):
        W.build_index(kv, S, cs, r, out=wx, ws=ws)
        cent, asg = W.build_state(kv, wx)
        cent = cent.clone()
        nxt = W.kmeans_assign(kv, S, cs, cent)
        torch.cuda.synchronize()
        assert W.read_device_status(ws) == 0
        cent_h = cent.cpu().numpy()
        asg_h, nxt_h = asg.cpu().numpy(), nxt.cpu().numpy()
        for (h, g), (s, n, X, V) in rows.items():
            m = O.clusters_in_segment(n, cs)
            c0 = wx.cl_row(0, h) + g * (S // cs)
            t0 = wx.tok_row(0, h) + s
            C = cent_h[c0:c0 + m].astype(np.float64)
            lab_r = asg_h[t0:t0 + n].astype(np.int64)
            assert lab_r.min() >= 0 and lab_r.max() < m
            cnt = np.bincount(lab_r, minlength=m)
            sums = np.zeros((m, X.shape[1]))
            np.add.at(sums, lab_r, X)
            nz = cnt > 0
            mean = (sums[nz] / cnt[nz, None]).astype(np.float32).astype(np.float64)
            assert np.all(np.abs(C[nz] - mean) <= ulp(mean, 24)), f"round {r} update"
            got = nxt_h[t0:t0 + n].astype(np.int64)
            assert_near_ties(X, C, got, O.kmeans_assign(X, C))

    # ---- the full ten rounds: a valid index on the sampled segments
    W.build_index(kv, S, cs, wl.iters, out=wx, ws=ws)
    torch.cuda.synchronize()
    assert W.read_device_status(ws) == 0
    for (h, g), (s, n, X, V) in rows.items():
        check_segment_valid(gpu_segment(wx, h, g, s, n), X, V)
