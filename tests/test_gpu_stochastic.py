"""The sampled top-k on the GPU (Vortex summary, section 2.C: stochastic
radix top-k, early termination by sampling the threshold bin; reading R-16).

The selection keys are the GPU's own fp32 group-max scores (returned through
scores_out), so both sides rank the same keys: the GPU's retrieved set must
then equal the oracle's select_topk_stochastic bit for bit for the same seed
(every candidate above the threshold bin, and the threshold bin's members
with the smallest SplitMix64 draws).  The decode output must match the
oracle's decode on that set, and the sampled set must keep most of the exact
top-k (recall).
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


def small_wl(seed=61, seq_lens=(9000, 5000)):
    return WI.mixture_workload("sampled", seq_lens=list(seq_lens), n_q_heads=8, n_kv_heads=2,
                               head_dim=128, n_centers=24, seg_len=1024, cluster_size=16,
                               iters=3, topk_fraction=0.05, seed=seed, device=DEV)


@pytest.mark.parametrize("seed", [0, 7, 123456789])
def test_sampled_selection_equals_the_oracle(seed):
    wl = small_wl()
    units = H.oracle_build(wl)
    wx = H.empty_index(wl, DEV)
    H.upload_index(wx, units)
    p = H.params_of(wl, sampled=True, seed=seed)
    p.scores_out = W.scores_buffer(wx, wl.n_q_heads)
    ws = W.decode_workspace(wx, p)
    out, lse = W.decode(wl.q.to(DEV), wx, p, ws=ws)
    torch.cuda.synchronize()
    assert W.read_device_status(ws) == 0
    lay = W.decode_layout(wx, p)
    info = W.unit_info(ws, lay, wl.batch * wl.n_kv_heads).cpu().numpy()
    qh = H.q_host(wl)
    G = wl.n_q_heads // wl.n_kv_heads
    sampled_somewhere = False
    for (b, h), ix in sorted(units.items()):
        u = b * wl.n_kv_heads + h
        NC = len(ix.centroids)
        k = O.k_for(NC, p.topk_clusters, p.topk_fraction)
        qg = qh[b, h * G:(h + 1) * G]
        tr = O.decode_unit(qg, ix, wl.n_sink, wl.window, k)
        a32 = W.centroid_scores(p.scores_out, wx, b, h).cpu().numpy().max(1)   # fp32 group max
        want = O.select_topk_stochastic(a32.astype(np.float64), tr.candidate, k, seed)
        got = W.selected_clusters(ws, lay, wx, b, h, int(info[u, 0])).cpu().numpy()
        assert np.array_equal(got, want), (b, h, np.setxor1d(got, want))
        sampled_somewhere |= bool(info[u, 12] == 1)
        ref = O.decode_unit(qg, ix, wl.n_sink, wl.window, k, selected=got)
        og = out[b, h * G:(h + 1) * G].cpu().numpy().astype(np.float64)
        assert H.rel_err(og, ref.out, wl.dtype) <= 2e-4
        np.testing.assert_allclose(lse[b, h * G:(h + 1) * G].cpu().numpy(), ref.lse, rtol=2e-6,
                                   atol=2e-5)
    assert sampled_somewhere   # some unit's threshold bin was actually sampled


def test_sampled_recall_against_the_exact_selection():
    """Over several seeds, the recall of the GPU's sampled sets against its
    exact sets equals the oracle's recall on the same fp32 keys, and the
    sampled sets keep the larger part of the exact top-k."""
    wl = small_wl(seed=62, seq_lens=(16384,))
    kv = H.paged_kv(wl, DEV)
    wx = W.build_index(kv, wl.seg_len, wl.cluster_size, wl.iters)
    pe = H.params_of(wl)
    pe.scores_out = W.scores_buffer(wx, wl.n_q_heads)
    wse = W.decode_workspace(wx, pe)
    W.decode(wl.q.to(DEV), wx, pe, ws=wse)
    torch.cuda.synchronize()
    lay = W.decode_layout(wx, pe)
    info = W.unit_info(wse, lay, 2).cpu().numpy()
    exact = {h: W.selected_clusters(wse, lay, wx, 0, h, int(info[h, 0])).cpu().numpy()
             for h in range(2)}
    keys = {h: W.centroid_scores(pe.scores_out, wx, 0, h).cpu().numpy().max(1).astype(np.float64)
            for h in range(2)}
    cand = {h: W.selection_keys(wse, lay, wx, 0, h).cpu().numpy() != 0 for h in range(2)}
    rec = []
    for seed in range(8):
        ps = H.params_of(wl, sampled=True, seed=seed)
        wss = W.decode_workspace(wx, ps)
        W.decode(wl.q.to(DEV), wx, ps, ws=wss)
        torch.cuda.synchronize()
        lays = W.decode_layout(wx, ps)
        infs = W.unit_info(wss, lays, 2).cpu().numpy()
        for h in range(2):
            got = W.selected_clusters(wss, lays, wx, 0, h, int(infs[h, 0])).cpu().numpy()
            k = len(exact[h])
            assert len(got) == k
            ref_exact = O.select_topk(keys[h], cand[h], k)
            ref_samp = O.select_topk_stochastic(keys[h], cand[h], k, seed)
            assert np.array_equal(exact[h], ref_exact)   # same fp32 keys, same tie rule
            r = O.recall(got, exact[h])
            assert r == O.recall(ref_samp, exact[h])
            rec.append(r)
    assert np.mean(rec) >= 0.5, rec
