"""Pins for the fp64 oracle against what the pages and the mathematics fix.

Every pin here is independent of the oracle's own formulas: library routines
(torch scaled_dot_product_attention, scikit-learn Lloyd k-means, scipy vq and
logsumexp, numpy stable argsort, torch's bfloat16 rounding), closed forms
derived by hand (tests/golden/), invariants the definitions imply, and a
brute-force per-token enumeration written separately below.

Sources: RetroInfer technical summary, section 2.A (Steady, Retrieval and
Estimation zones; Segmented Clustering); Vortex summary, section 2.A
(forward_cache / forward_indexer; Top-K primitive).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def mixture(rng, T, d, n_centers=8, noise=0.3, scale=None):
    centers = rng.standard_normal((n_centers, d))
    ids = rng.integers(0, n_centers, size=T)
    k = centers[ids] + noise * rng.standard_normal((T, d))
    if scale is not None:
        k = k * scale
    return k, rng.standard_normal((T, d)), centers


def sdpa(q, K, V):
    """Library dense attention (torch, fp64, CPU) with GQA head mapping."""
    qt = torch.from_numpy(np.ascontiguousarray(q))[None, :, None, :]
    Kt = torch.from_numpy(np.ascontiguousarray(K))[None, None]
    Vt = torch.from_numpy(np.ascontiguousarray(V))[None, None]
    G = q.shape[0]
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, Kt.expand(1, G, -1, -1), Vt.expand(1, G, -1, -1))
    return out[0, :, 0].numpy()


# ---------------------------------------------------------------- rounding

def test_round_bf16_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    x = np.concatenate([x, np.float32([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3e38, 1e-39])])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_round_bf16_halfway_goes_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: even mantissa is 1.0
    assert O.round_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    # 1 + 3*2^-8 lies halfway between 1+2^-7 (odd) and 1+2^-6 (even)
    assert O.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    # fp64 value just above a halfway point rounds up (no double rounding)
    assert O.round_bf16(np.array([1 + 2 ** -8 + 2 ** -40]))[0] == 1 + 2 ** -7


# ------------------------------------------------------- segmentation, k-means

def test_segment_and_cluster_counts():
    # 4196 = 4*1024 + 100: four full segments of 64 clusters, then ceil(100/16) = 7
    spans = O.segment_spans(4196, 1024)
    assert spans == [(0, 1024), (1024, 1024), (2048, 1024), (3072, 1024), (4096, 100)]
    assert O.n_clusters(4196, 1024, 16) == 4 * 64 + 7
    assert O.n_clusters(131072, 8192, 16) == 8192
    assert O.n_clusters(1048576, 8192, 16) == 65536


def test_topk_fraction_rule():
    # 1.8% of the clusters, rounded up
    assert O.k_for(8192, -1, 0.018) == 148
    assert O.k_for(2048, -1, 0.018) == 37
    assert O.k_for(65536, -1, 0.018) == 1180
    assert O.k_for(8192, 16, 0.5) == 16


def test_assign_matches_scipy_vq():
    from scipy.cluster.vq import vq
    rng = np.random.default_rng(1)
    X, _, _ = mixture(rng, 3000, 16)
    C = rng.standard_normal((70, 16))
    lab, _ = vq(X, C)
    assert np.array_equal(O.kmeans_assign(X, C), lab)


def test_distances_match_scipy_cdist_and_a_direct_loop():
    """kmeans_distances decides which GPU assignment flips count as near-ties,
    so it is pinned to scipy's squared Euclidean distance and to the direct
    per-pair sum of squared differences."""
    from scipy.spatial.distance import cdist
    rng = np.random.default_rng(11)
    X, _, _ = mixture(rng, 400, 24, scale=np.exp(0.5 * rng.standard_normal(24)))
    C = 2.0 * rng.standard_normal((37, 24))
    got = O.kmeans_distances(X, C)
    np.testing.assert_allclose(got, cdist(X, C, "sqeuclidean"), rtol=1e-12, atol=1e-9)
    for i in (0, 123, 399):
        for j in (0, 17, 36):
            direct = sum((X[i, e] - C[j, e]) ** 2 for e in range(24))
            assert abs(got[i, j] - direct) <= 1e-10 * direct
    # a point on a centroid is at distance zero from it
    assert abs(O.kmeans_distances(C[5:6], C)[0, 5]) <= 1e-12 * float((C[5] ** 2).sum())


def test_assign_ties_go_to_lower_index():
    X = np.array([[0.0, 0.0], [0.0, 0.0], [2.0, 0.0]])
    C = np.array([[0.0, 1.0], [1.0, 0.0], [-1.0, 0.0], [1.0, 0.0]])
    # token 0,1: distance 1 to every centroid -> 0; token 2: centroids 1 and 3 tie -> 1
    assert list(O.kmeans_assign(X, C)) == [0, 0, 1]


def test_lloyd_matches_sklearn():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(2)
    X, _, _ = mixture(rng, 1024, 8, n_centers=6, noise=0.5)
    C0 = O.kmeans_init(X, 16)
    iters = 7
    labels, C, _ = O.kmeans_segment(X, 16, iters)
    assert np.all(np.bincount(labels, minlength=len(C)) > 0), "pick data without empty clusters"
    km = KMeans(n_clusters=len(C0), init=C0, n_init=1, max_iter=iters, tol=0.0,
                algorithm="lloyd").fit(X)
    np.testing.assert_allclose(C, km.cluster_centers_, rtol=0, atol=1e-12)


def test_kmeans_init_positions_and_empty_cluster_keeps_centroid():
    X = np.array([[0.0], [0.1], [5.0], [5.1], [0.2], [0.05]])
    # cs=2 -> 3 centroids from positions 0, 2, 4: (0), (5), (0.2)
    np.testing.assert_array_equal(O.kmeans_init(X, 2), [[0.0], [5.0], [0.2]])
    lab = np.array([0, 0, 1, 1, 0, 0])
    C = O.kmeans_update(X, lab, np.array([[0.0], [5.0], [0.2]]))
    np.testing.assert_allclose(C, [[0.0875], [5.05], [0.2]])


def test_kmeans_objective_non_increasing():
    rng = np.random.default_rng(3)
    for T, cs in [(2048, 16), (1000, 7), (333, 1)]:
        X, _, _ = mixture(rng, T, 12, n_centers=20, noise=0.4)
        _, _, hist = O.kmeans_segment(X, cs, 10)
        for a, b in zip(hist, hist[1:]):
            assert b <= a * (1 + 1e-12) + 1e-12


# ------------------------------------------------------------- index layout

def test_build_layout_invariants():
    rng = np.random.default_rng(4)
    K, V, _ = mixture(rng, 1500, 8, n_centers=12)
    ix = O.build_unit(K, V, seg_len=512, cluster_size=16, iters=4, store="f32")
    T = len(K)
    NC = O.n_clusters(T, 512, 16)
    assert len(ix.centroids) == NC and len(ix.offsets) == NC + 1
    assert ix.offsets[0] == 0 and ix.offsets[-1] == T and np.all(np.diff(ix.offsets) >= 0)
    assert sorted(ix.perm.tolist()) == list(range(T))
    assert np.array_equal(ix.invperm[ix.perm], np.arange(T))
    for c in range(NC):
        members = ix.perm[ix.offsets[c]:ix.offsets[c + 1]]
        assert np.all(np.diff(members) > 0)
        assert np.all(ix.labels[members] == c)
    # clusters never cross a segment: each segment keeps its own slot range
    for s, (start, n) in enumerate(O.segment_spans(T, 512)):
        assert set(ix.perm[start:start + n].tolist()) == set(range(start, start + n))
    np.testing.assert_array_equal(ix.k_perm, K[ix.perm])
    np.testing.assert_array_equal(ix.v_perm, V[ix.perm])
    cnt = np.diff(ix.offsets)
    for c in np.nonzero(cnt)[0]:
        members = ix.perm[ix.offsets[c]:ix.offsets[c + 1]]
        np.testing.assert_allclose(ix.centroids_exact[c], K[members].mean(0), atol=1e-13)
        np.testing.assert_allclose(ix.value_sums_exact[c], V[members].sum(0), atol=1e-12)


@pytest.mark.parametrize("T_old,T_new", [(1500, 2900), (1024, 2048), (700, 700), (2048, 2048),
                                         (1, 1030)])
def test_extension_equals_build_of_the_longer_sequence(T_old, T_new):
    """Segments are clustered independently ([RI] 2.A, Segmented Clustering),
    so growing the index of the first T_old tokens to T_new tokens equals
    building it for T_new tokens: every field, exactly."""
    rng = np.random.default_rng(11)
    K, V, _ = mixture(rng, T_new, 8, n_centers=12)
    for store in ("f32", "bf16"):
        old = O.build_unit(K[:T_old], V[:T_old], seg_len=512, cluster_size=16, iters=3, store=store)
        ext = O.extend_unit(old, K, V, seg_len=512, cluster_size=16, iters=3, store=store)
        ref = O.build_unit(K, V, seg_len=512, cluster_size=16, iters=3, store=store)
        for f in ("centroids", "value_sums", "offsets", "perm", "invperm", "labels", "k_perm",
                  "v_perm", "centroids_exact"):
            np.testing.assert_array_equal(getattr(ext, f), getattr(ref, f), err_msg=f)
        # exact value sums agree to summation order (the kept ones are copied)
        np.testing.assert_allclose(ext.value_sums_exact, ref.value_sums_exact, atol=1e-12)


def test_block_index_is_positional():
    """Block top-k index ([VX] 2.A block centroids): block j of a segment is
    positions j*B .. (j+1)*B-1, its summary the mean key; perm is the identity."""
    rng = np.random.default_rng(12)
    K, V, _ = mixture(rng, 1300, 8, n_centers=12)
    ix = O.build_blocks_unit(K, V, seg_len=512, block_size=16, store="f32")
    assert np.array_equal(ix.perm, np.arange(1300)) and np.array_equal(ix.invperm, ix.perm)
    spans = O.segment_spans(1300, 512)
    assert len(ix.centroids) == sum(O.clusters_in_segment(n, 16) for _, n in spans)
    c = 0
    for start, n in spans:
        for j in range(0, n, 16):
            lo, hi = start + j, start + min(j + 16, n)
            assert ix.offsets[c] == lo and ix.offsets[c + 1] == hi
            assert np.all(ix.labels[lo:hi] == c)
            np.testing.assert_allclose(ix.centroids[c], K[lo:hi].mean(0), atol=1e-13)
            np.testing.assert_allclose(ix.value_sums[c], V[lo:hi].sum(0), atol=1e-12)
            c += 1


@pytest.mark.parametrize("n_sink,window", [(4, 64), (0, 0)])
def test_exact_only_with_every_block_is_dense(n_sink, window):
    """Without the estimation zone, retrieving every block is full attention."""
    rng = np.random.default_rng(13)
    K, V, C = mixture(rng, 900, 16, n_centers=10)
    q = C[:4] + 0.3 * rng.standard_normal((4, 16))
    ix = O.build_blocks_unit(K, V, seg_len=256, block_size=16, store="f32")
    tr = O.decode_unit(q, ix, n_sink, window, k=10 ** 6, estimate=False)
    out, lse = O.dense_attention(q, K, V)
    np.testing.assert_allclose(tr.out, out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(tr.lse, lse, rtol=1e-12, atol=1e-12)


def test_exact_only_with_no_block_is_steady_attention():
    """k = 0 and no estimation leaves attention over the sink and window
    tokens alone."""
    rng = np.random.default_rng(14)
    K, V, C = mixture(rng, 700, 16, n_centers=10)
    q = C[:2] + 0.3 * rng.standard_normal((2, 16))
    ix = O.build_blocks_unit(K, V, seg_len=256, block_size=16, store="f32")
    tr = O.decode_unit(q, ix, 4, 32, k=0, estimate=False)
    st = np.r_[0:4, 700 - 32:700]
    out, lse = O.dense_attention(q, K[st], V[st])
    np.testing.assert_allclose(tr.out, out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(tr.lse, lse, rtol=1e-12, atol=1e-12)


def test_exact_only_brute_force():
    """Exact-only decode equals softmax over the retrieved blocks' tokens
    (minus steady ones, counted once) plus the steady tokens, by brute force."""
    rng = np.random.default_rng(15)
    K, V, C = mixture(rng, 300, 8, n_centers=6)
    q = C[:2] + 0.3 * rng.standard_normal((2, 8))
    ix = O.build_blocks_unit(K, V, seg_len=128, block_size=8, store="f32")
    tr = O.decode_unit(q, ix, 2, 16, k=5, estimate=False)
    keep = set(range(2)) | set(range(300 - 16, 300))
    for c in tr.selected:
        keep |= set(range(ix.offsets[c], ix.offsets[c + 1]))
    keep = np.array(sorted(keep))
    out, lse = O.dense_attention(q, K[keep], V[keep])
    np.testing.assert_allclose(tr.out, out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(tr.lse, lse, rtol=1e-12, atol=1e-12)


# ------------------------------------------------ stochastic radix top-k pins

def test_splitmix64_published_outputs():
    """The first three SplitMix64 outputs from state 0 (the generator's
    published known answers: Steele, Lea and Flood 2014, and the reference
    splitmix64.c seeded with 0); the state advances by the golden-ratio
    increment between outputs."""
    gamma = 0x9E3779B97F4A7C15
    got = [O.splitmix64((i * gamma) & ((1 << 64) - 1)) for i in range(3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_ordered_key_preserves_float_order():
    rng = np.random.default_rng(21)
    x = np.concatenate([rng.standard_normal(500) * 10.0 ** rng.integers(-30, 30, 500),
                        [-np.inf, np.inf, -0.0, 0.0, 1e-45, -1e-45]]).astype(np.float32)
    keys = O.ordered_key32(x)
    xs = x.astype(np.float64)
    for i in range(0, len(x), 7):
        for j in range(0, len(x), 11):
            if xs[i] < xs[j]:
                assert keys[i] < keys[j]
            elif xs[i] > xs[j]:
                assert keys[i] > keys[j]


def stochastic_case(seed, n=400):
    rng = np.random.default_rng(seed)
    a = np.round(rng.standard_normal(n), 2)          # duplicates and shared bins
    cand = rng.random(n) > 0.1
    return a, cand


@pytest.mark.parametrize("k", [0, 1, 17, 100, 359, 10 ** 6])
def test_stochastic_topk_invariants(k):
    """k picks (clamped), all candidates; every candidate of a bin above the
    threshold bin is taken, none below it; the rest come from the bin."""
    a, cand = stochastic_case(3)
    sel = O.select_topk_stochastic(a, cand, k, seed=5)
    n_c = int(cand.sum())
    assert len(sel) == min(k, n_c) and len(set(sel.tolist())) == len(sel)
    assert np.all(cand[sel]) and np.all(np.diff(sel) > 0)
    if 0 < k < n_c:
        bins = O.ordered_key32(a.astype(np.float32)) >> 21
        b_star = np.sort(bins[cand])[::-1][k - 1]
        chosen = np.zeros(len(a), dtype=bool)
        chosen[sel] = True
        assert np.all(chosen[cand & (bins > b_star)])
        assert not np.any(chosen[cand & (bins < b_star)])


def test_stochastic_topk_is_exact_when_bins_decide():
    """Scores whose bins are all distinct leave nothing to sample: the
    selection is the exact top-k, whatever the seed."""
    a = 2.0 ** np.arange(-40, 40, 0.5)[::-1]
    rng = np.random.default_rng(4)
    rng.shuffle(a)
    cand = np.ones(len(a), dtype=bool)
    for k in (1, 5, 33, 100):
        exact = O.select_topk(a, cand, k)
        for seed in (0, 1, 99):
            sel = O.select_topk_stochastic(a, cand, k, seed)
            assert np.array_equal(sel, exact)
            assert O.recall(sel, exact) == 1.0


def test_stochastic_topk_samples_the_threshold_bin_uniformly():
    """Ten clear winners and twenty members of one bin: with k = 15 five of
    the twenty are drawn; over 4000 seeds each is drawn with frequency 1/4
    (binomial, five sigma), and a fixed seed repeats its draw."""
    a = np.concatenate([np.arange(10, 20, dtype=np.float64), np.full(20, 1.0)])
    cand = np.ones(30, dtype=bool)
    counts = np.zeros(30)
    for seed in range(4000):
        sel = O.select_topk_stochastic(a, cand, 15, seed)
        assert set(range(10)) <= set(sel.tolist())
        counts[sel] += 1
    f = counts[10:] / 4000
    assert np.all(np.abs(f - 0.25) <= 5 * np.sqrt(0.25 * 0.75 / 4000))
    assert np.array_equal(O.select_topk_stochastic(a, cand, 15, 77),
                          O.select_topk_stochastic(a, cand, 15, 77))


def test_recall_bounds():
    a, cand = stochastic_case(6)
    for k in (0, 10, 60):
        exact = O.select_topk(a, cand, k)
        sel = O.select_topk_stochastic(a, cand, k, seed=3)
        r = O.recall(sel, exact)
        assert 0.0 <= r <= 1.0 and O.recall(exact, exact) == 1.0
        if k:
            bins = O.ordered_key32(a.astype(np.float32)) >> 21
            b_star = np.sort(bins[cand])[::-1][k - 1]
            m = int((cand & (bins == b_star)).sum())
            assert r >= (k - m) / k          # only the threshold bin is sampled


# --------------------------------------------------------------- decode pins

def test_steady_positions():
    assert list(O.steady_positions(100, 4, 64)) == list(range(4)) + list(range(36, 100))
    assert list(O.steady_positions(10, 4, 8)) == list(range(10))
    assert list(O.steady_positions(10, 0, 0)) == []
    assert list(O.steady_positions(3, 4, 64)) == [0, 1, 2]


def test_topk_matches_stable_argsort_and_ties():
    rng = np.random.default_rng(5)
    a = np.round(rng.standard_normal(500), 1)          # many exact ties
    cand = rng.random(500) > 0.2
    for k in [0, 1, 7, 40, 399, 500]:
        idx = np.nonzero(cand)[0]
        order = idx[np.argsort(-a[idx], kind="stable")]
        assert np.array_equal(O.select_topk(a, cand, k), np.sort(order[:k]))
    assert list(O.select_topk(np.array([1.0, 3, 3, 2, 3]), np.ones(5, bool), 2)) == [1, 2]
    assert list(O.select_topk(np.array([1.0, 3, 3, 2, 3]), np.ones(5, bool), 4)) == [1, 2, 3, 4]


def test_lse_merge_matches_logsumexp():
    from scipy.special import logsumexp
    rng = np.random.default_rng(6)
    s = rng.standard_normal((3, 40)) * 4
    v = rng.standard_normal((40, 5))
    parts = [O.zone_stats(s[:, a:b], np.ones(b - a), v[a:b]) for a, b in [(0, 13), (13, 14), (14, 40)]]
    parts.append(O.zone_stats(s[:, :0], np.ones(0), v[:0]))   # an empty part
    out, lse = O.lse_merge(parts)
    np.testing.assert_allclose(lse, logsumexp(s, axis=1), rtol=1e-13)
    w = np.exp(s - logsumexp(s, axis=1)[:, None])
    np.testing.assert_allclose(out, w @ v, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("G,n_sink,window", [(1, 4, 64), (4, 4, 64), (4, 0, 0), (2, 30, 7)])
def test_all_clusters_retrieved_equals_dense_sdpa(G, n_sink, window):
    """P1: retrieving every candidate cluster leaves nothing to estimate, so the
    result is full softmax attention (library routine)."""
    rng = np.random.default_rng(7 + G)
    T, d = 1200, 16
    K, V, centers = mixture(rng, T, d, n_centers=10)
    ix = O.build_unit(K, V, seg_len=256, cluster_size=8, iters=3, store="f32")
    q = centers[rng.integers(0, 10, G)] + 0.3 * rng.standard_normal((G, d))
    NC = len(ix.centroids)
    tr = O.decode_unit(q, ix, n_sink, window, k=NC)
    ref = sdpa(q, K, V)
    assert np.max(np.abs(tr.out - ref)) <= 1e-6 * np.max(np.abs(ref))
    assert np.max(np.abs(tr.out - ref)) <= 1e-12
    _, lse_ref = O.dense_attention(q, K, V)
    np.testing.assert_allclose(tr.lse, lse_ref, rtol=1e-12)


@pytest.mark.parametrize("k,n_sink,window", [(0, 0, 0), (3, 4, 16), (50, 1, 1), (0, 8, 100)])
def test_one_token_per_cluster_estimation_is_exact(k, n_sink, window):
    """P2: with cluster size 1 a centroid is its key, so the estimate of every
    cluster is exact and any retrieval budget gives full attention."""
    rng = np.random.default_rng(11 + k)
    T, d, G = 300, 8, 4
    K, V, centers = mixture(rng, T, d)
    # f32-representable inputs, so the stored centroid of a 1-token cluster is its key
    K = K.astype(np.float32).astype(np.float64)
    V = V.astype(np.float32).astype(np.float64)
    ix = O.build_unit(K, V, seg_len=64, cluster_size=1, iters=2, store="f32")
    q = centers[rng.integers(0, 8, G)] + 0.3 * rng.standard_normal((G, d))
    tr = O.decode_unit(q, ix, n_sink, window, k=k)
    ref = sdpa(q, K, V)
    np.testing.assert_allclose(tr.out, ref, rtol=1e-10, atol=1e-12)


def brute_force(q, K, V, labels, centroids, value_sums, n_sink, window, k):
    """Independent per-token statement of the wave-index decode (no max
    subtraction, tiny inputs): zones assigned token by token."""
    T, d = len(K), len(q)
    steady = [p < n_sink or p >= T - window for p in range(T)]
    NC = len(centroids)
    members = [[p for p in range(T) if labels[p] == c] for c in range(NC)]
    live = [[p for p in members[c] if not steady[p]] for c in range(NC)]
    score = [sum(q[j] * centroids[c][j] for j in range(d)) / math.sqrt(d) for c in range(NC)]
    cands = [c for c in range(NC) if live[c]]
    ranked = sorted(cands, key=lambda c: (-score[c], c))
    chosen = set(ranked[:k])
    num = [0.0] * len(V[0])
    den = 0.0
    for p in range(T):
        if steady[p] or labels[p] in chosen:
            w = math.exp(sum(q[j] * K[p][j] for j in range(d)) / math.sqrt(d))
            den += w
            for j in range(len(num)):
                num[j] += w * V[p][j]
    for c in cands:
        if c in chosen:
            continue
        w = math.exp(score[c])
        vs = list(value_sums[c])
        for p in members[c]:
            if steady[p]:
                vs = [a - b for a, b in zip(vs, V[p])]
        den += w * len(live[c])
        for j in range(len(num)):
            num[j] += w * vs[j]
    return [x / den for x in num], math.log(den), sorted(chosen)


@pytest.mark.parametrize("T,cs,k,n_sink,window", [(64, 4, 3, 2, 5), (50, 5, 0, 0, 0),
                                                  (40, 3, 20, 1, 3), (64, 8, 2, 0, 20),
                                                  (33, 2, 5, 33, 0)])
def test_brute_force_tiny(T, cs, k, n_sink, window):
    """P3: the oracle equals a direct per-token enumeration of the zones."""
    rng = np.random.default_rng(T * 7 + k)
    d = 6
    K, V, centers = mixture(rng, T, d, n_centers=4, noise=0.5)
    ix = O.build_unit(K, V, seg_len=24, cluster_size=cs, iters=3, store="f32")
    q = centers[0] + 0.3 * rng.standard_normal(d)
    out_b, lse_b, chosen = brute_force(q.tolist(), K.tolist(), V.tolist(), ix.labels.tolist(),
                                       ix.centroids.tolist(), ix.value_sums.tolist(),
                                       n_sink, window, k)
    tr = O.decode_unit(q[None], ix, n_sink, window, k)
    assert list(tr.selected) == chosen
    np.testing.assert_allclose(tr.out[0], out_b, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(tr.lse[0], lse_b, rtol=1e-12)


def test_jensen_estimate_never_exceeds_exact_mass():
    """P5: for each cluster cnt * e^(q.kbar/sqrt d) <= sum_i e^(q.k_i/sqrt d)
    (convexity of exp), so estimated mass is a lower bound."""
    rng = np.random.default_rng(13)
    K, V, centers = mixture(rng, 800, 8)
    ix = O.build_unit(K, V, 200, 16, 4, store="f32")
    q = centers[1] + 0.3 * rng.standard_normal(8)
    for c in range(len(ix.offsets) - 1):
        members = ix.perm[ix.offsets[c]:ix.offsets[c + 1]]
        if len(members) == 0:
            continue
        est = len(members) * math.exp(q @ ix.centroids_exact[c] / math.sqrt(8))
        exact = np.exp(K[members] @ q / math.sqrt(8)).sum()
        assert est <= exact * (1 + 1e-12)


def test_all_steady_is_dense():
    """P7a: a steady zone covering the whole sequence is full attention."""
    rng = np.random.default_rng(17)
    K, V, centers = mixture(rng, 200, 8)
    ix = O.build_unit(K, V, 64, 8, 2, store="f32")
    q = centers[:3] + 0.2 * rng.standard_normal((3, 8))
    for ns, w in [(200, 0), (0, 200), (150, 60), (1000, 1000)]:
        tr = O.decode_unit(q, ix, ns, w, k=5)
        assert len(tr.selected) == 0 and not tr.candidate.any()
        np.testing.assert_allclose(tr.out, sdpa(q, K, V), rtol=1e-11, atol=1e-13)


def test_pure_estimate_golden_two_clusters():
    """P7b: hand-derived two-cluster example (tests/golden)."""
    g = json.load(open(os.path.join(GOLDEN, "pure_estimate_two_clusters.json")))
    K = np.array(g["keys"])
    V = np.array(g["values"])
    ix = O.build_unit(K, V, g["seg_len"], g["cluster_size"], g["iters"], store="f32")
    assert list(ix.offsets) == g["expected_offsets"]
    assert list(ix.perm) == g["expected_perm"]
    np.testing.assert_array_equal(ix.value_sums, g["expected_value_sums"])
    tr = O.decode_unit(np.array([g["q"]]), ix, 0, 0, k=0)
    np.testing.assert_allclose(tr.out[0], g["expected_out"], rtol=1e-14)
    np.testing.assert_allclose(tr.lse[0], g["expected_lse"], rtol=1e-14)
    # retrieving cluster 0 instead: exact part is keys 0,1, estimate is cluster 1
    tr1 = O.decode_unit(np.array([g["q"]]), ix, 0, 0, k=1)
    assert list(tr1.selected) == [0]
    qv = np.array(g["q"])
    w = np.exp(K @ qv / math.sqrt(2))
    est_w = math.exp(qv @ np.array([-1.0, np.float32(-0.1)]) / math.sqrt(2))
    num = w[0] * V[0] + w[1] * V[1] + est_w * np.array([2.0, 2.0])
    den = w[0] + w[1] + 2 * est_w
    np.testing.assert_allclose(tr1.out[0], num / den, rtol=1e-13)


def test_gqa_group_uses_its_own_kv_head():
    """R-4: q head h reads KV head floor(h/G).  Two KV heads with disjoint
    content: each group's output equals dense attention over its own head."""
    rng = np.random.default_rng(19)
    Hkv, G, T, d = 2, 3, 300, 8
    keys, vals, qs = [], [], []
    for h in range(Hkv):
        K, V, centers = mixture(rng, T, d)
        keys.append(K + 3 * h)
        vals.append(V + 5 * h)
        qs.append(centers[rng.integers(0, 8, G)])
    q = np.concatenate(qs)[None]                  # [1][Hq][d]
    index = O.build_all([np.stack(keys)], [np.stack(vals)], 100, 4, 2, "f32")
    NC = len(index[0][0].centroids)
    out, _, _ = O.decode_all(q, index, 0, 0, NC, 0.0)
    for h in range(Hkv):
        np.testing.assert_allclose(out[0, h * G:(h + 1) * G], sdpa(q[0, h * G:(h + 1) * G],
                                                                  keys[h], vals[h]), atol=1e-12)


def test_group_selection_uses_max_over_heads():
    """R-4: with several q heads per KV head the selection score of a cluster is
    its best score over the group (checked by a direct loop)."""
    rng = np.random.default_rng(23)
    T, d, G = 600, 8, 3
    K, V, centers = mixture(rng, T, d, n_centers=12)
    ix = O.build_unit(K, V, 200, 8, 2, store="f32")
    q = centers[[0, 5, 9]] + 0.2 * rng.standard_normal((G, d))
    k = 9
    tr = O.decode_unit(q, ix, 0, 0, k)
    best = []
    for c in range(len(ix.centroids)):
        if ix.offsets[c + 1] == ix.offsets[c]:
            continue
        sc = max(sum(q[h][j] * ix.centroids[c][j] for j in range(d)) for h in range(G))
        best.append((-sc, c))
    assert list(tr.selected) == sorted(c for _, c in sorted(best)[:k])
