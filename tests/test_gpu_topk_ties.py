"""Top-k edge cases on the GPU: exact ties at the k-th score and a crowded
threshold (Vortex summary, section 2.C Top-K; reading R-6: equal scores go
to the lower cluster id).

The index is a block index (position blocks, perm the identity) of keys
that are multiples a_j * u of one vector u, the group's first query head,
the same for every token of block j, so block j's centroid is a_j * u too:
every query head of the group scores cluster j as a_j * (q_g . u) / sqrt(d),
so clusters with the same a_j score exactly alike, in fp32 on the GPU as in
fp64 in the oracle, and a larger a_j always scores higher.  Each case places
the k-th score inside a run of exactly equal scores; the retrieved set must
then equal the oracle's exactly, with no near-tie slack.  The clusters whose
members all lie in the steady window get the highest a_j of all: they are
not candidates and must not be retrieved.

The last test overwrites the centroids of such an index with values that are
not their members' means: the decode takes its estimation zone as "every
cluster minus what the zone leaves out", which stays precise only while a
cluster's estimated mass is bounded by its members' exact mass (Jensen, true
of every built index), and must report the violation in its status word.
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


def tied_index(n_top, n_tied, seed, consistent=True):
    """One sequence of 65536 tokens, 2 KV heads, G = 4, d = 128, blocks of 16
    (4096 clusters per head).  n_top clusters (spread over the ids) get
    distinct high scores, n_tied others one shared score, the rest a low one.
    consistent: the keys of block j are all a_j * u (so its centroid is the
    mean of its keys); otherwise only the centroids are a_j * u."""
    wl = WI.mixture_workload("ties", seq_lens=[65536], n_q_heads=8, n_kv_heads=2, head_dim=128,
                             n_centers=64, seg_len=1024, cluster_size=16, iters=1,
                             topk_clusters=148, seed=seed, device=DEV)
    keys, vals = H.host_rows(wl)
    qh = H.q_host(wl)
    wx = H.empty_index(wl, DEV)
    rng = np.random.default_rng(seed)
    units = {}
    for h in range(2):
        NC = 65536 // wl.cluster_size
        u = qh[0, 4 * h]                              # bf16 values of the group's first head
        assert np.max(qh[0, 4 * h:4 * h + 4] @ u) > 0
        ids = rng.permutation(NC - 4)                 # the last 4 blocks are all steady
        a = np.full(NC, 0.25)
        a[ids[:n_top]] = 2.0 + np.arange(n_top) / 64.0    # above the tied run
        a[ids[n_top:n_top + n_tied]] = 1.0
        a[NC - 4:] = 4.0                              # best scores, but not candidates
        cent = O.round_bf16(a[:, None] * u[None, :])
        K = np.repeat(cent, wl.cluster_size, axis=0) if consistent else keys[0][h]
        ix = O.build_blocks_unit(K, vals[0][h], wl.seg_len, wl.cluster_size, "bf16")
        if consistent:
            assert np.array_equal(ix.centroids, cent)
        else:
            ix.centroids = cent
        units[(0, h)] = ix
    H.upload_index(wx, units)
    return wl, wx, units


@pytest.mark.parametrize("n_top,n_tied", [(100, 60), (100, 2000), (0, 4000)])
def test_ties_at_the_kth_score_go_to_the_lower_id(n_top, n_tied):
    wl, wx, units = tied_index(n_top, n_tied, seed=17 + n_tied)
    p = H.params_of(wl)
    ws = W.decode_workspace(wx, p)
    out, lse = W.decode(wl.q.to(DEV), wx, p, ws=ws)
    torch.cuda.synchronize()
    assert W.read_device_status(ws) == 0
    lay = W.decode_layout(wx, p)
    info = W.unit_info(ws, lay, 2).cpu().numpy()
    qh = H.q_host(wl)
    for h in range(2):
        ix = units[(0, h)]
        tr = O.decode_unit(qh[0, 4 * h:4 * h + 4], ix, wl.n_sink, wl.window, 148)
        ties = np.count_nonzero(tr.sel_score[tr.selected] == tr.sel_score[tr.selected].min())
        assert 0 < 148 - n_top <= ties or n_top >= 148
        got = W.selected_clusters(ws, lay, wx, 0, h, int(info[h, 0])).cpu().numpy()
        assert np.array_equal(got, tr.selected), (h, np.setxor1d(got, tr.selected))
        og = out[0, 4 * h:4 * h + 4].cpu().numpy().astype(np.float64)
        assert H.rel_err(og, tr.out, wl.dtype) <= 2e-4
        np.testing.assert_allclose(lse[0, 4 * h:4 * h + 4].cpu().numpy(), tr.lse, rtol=2e-6,
                                   atol=2e-5)


def test_centroids_far_from_their_members_are_reported():
    wl, wx, units = tied_index(100, 60, seed=5, consistent=False)
    p = H.params_of(wl)
    ws = W.decode_workspace(wx, p)
    W.decode(wl.q.to(DEV), wx, p, ws=ws)
    flags = W.read_device_status(ws)
    assert flags & W.WI_DEV_CANCELLATION
    assert not flags & ~W.WI_DEV_CANCELLATION
