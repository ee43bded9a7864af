"""Randomised properties of the oracle (CPU, hypothesis): the segment
structure of the index ([RI] 2.A, Segmented Clustering), the block index and
the exact-only decode ([VX] 2.A block top-k), on small random shapes.

Each property follows from the definitions alone, so a failing example is a
mistake in the oracle, not a tolerance question.
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle as O

SET = settings(max_examples=25, deadline=None)


def data(seed, T, d):
    rng = np.random.default_rng(seed)
    centers = rng.standard_normal((6, d))
    K = centers[rng.integers(0, 6, size=T)] + 0.3 * rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    q = centers[:2] + 0.3 * rng.standard_normal((2, d))
    return K, V, q


@SET
@given(seed=st.integers(0, 10 ** 6), T_new=st.integers(1, 700), frac=st.floats(0.0, 1.0),
       seg_blocks=st.integers(1, 6), cs=st.sampled_from([4, 8, 16]))
def test_extension_equals_build(seed, T_new, frac, seg_blocks, cs):
    """Growing the index of any prefix equals building the whole sequence."""
    S = seg_blocks * cs * 4
    T_old = max(1, int(frac * T_new))
    K, V, _ = data(seed, T_new, 4)
    old = O.build_unit(K[:T_old], V[:T_old], S, cs, 2, "bf16")
    ext = O.extend_unit(old, K, V, S, cs, 2, "bf16")
    ref = O.build_unit(K, V, S, cs, 2, "bf16")
    for f in ("centroids", "value_sums", "offsets", "perm", "invperm", "labels"):
        assert np.array_equal(getattr(ext, f), getattr(ref, f)), f


@SET
@given(seed=st.integers(0, 10 ** 6), T=st.integers(1, 600), seg_blocks=st.integers(1, 5),
       B=st.sampled_from([1, 4, 16]))
def test_block_index_definition(seed, T, seg_blocks, B):
    """Blocks never cross a segment, cover every position once in order, and
    hold the mean key and summed values of their positions."""
    S = seg_blocks * B * 2
    K, V, _ = data(seed, T, 4)
    ix = O.build_blocks_unit(K, V, S, B, "f32")
    assert np.array_equal(ix.perm, np.arange(T))
    assert ix.offsets[0] == 0 and ix.offsets[-1] == T and np.all(np.diff(ix.offsets) >= 1)
    assert np.all(np.diff(ix.offsets) <= B)
    for c in range(len(ix.centroids)):
        lo, hi = ix.offsets[c], ix.offsets[c + 1]
        assert lo // S == (hi - 1) // S                  # inside one segment
        np.testing.assert_allclose(ix.centroids_exact[c], K[lo:hi].mean(0), atol=1e-12)
        np.testing.assert_allclose(ix.value_sums_exact[c], V[lo:hi].sum(0), atol=1e-12)


@SET
@given(seed=st.integers(0, 10 ** 6), T=st.integers(20, 400), k=st.integers(0, 40),
       n_sink=st.integers(0, 8), window=st.integers(0, 40), B=st.sampled_from([4, 8]))
def test_exact_only_is_attention_over_the_kept_tokens(seed, T, k, n_sink, window, B):
    """Without the estimation zone the output is plain softmax attention over
    the retrieved blocks' tokens and the steady tokens, each once."""
    K, V, q = data(seed, T, 8)
    ix = O.build_blocks_unit(K, V, 64, B, "f32")
    tr = O.decode_unit(q, ix, n_sink, window, k, estimate=False)
    keep = set(O.steady_positions(T, n_sink, window).tolist())
    for c in tr.selected:
        keep |= set(range(ix.offsets[c], ix.offsets[c + 1]))
    if not keep:
        assert np.all(tr.out == 0) and np.all(np.isneginf(tr.lse))
        return
    keep = np.array(sorted(keep))
    out, lse = O.dense_attention(q, K[keep], V[keep])
    np.testing.assert_allclose(tr.out, out, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(tr.lse, lse, rtol=1e-11, atol=1e-12)


@SET
@given(seed=st.integers(0, 10 ** 6), T=st.integers(20, 400), n_sink=st.integers(0, 8),
       window=st.integers(0, 40))
def test_retrieving_everything_is_dense_with_or_without_estimation(seed, T, n_sink, window):
    """With every cluster retrieved the estimation zone is empty, so both
    decodes are full attention."""
    K, V, q = data(seed, T, 8)
    ix = O.build_unit(K, V, 128, 8, 2, "f32")
    dense, dlse = O.dense_attention(q, K, V)
    for est in (True, False):
        tr = O.decode_unit(q, ix, n_sink, window, 10 ** 6, estimate=est)
        np.testing.assert_allclose(tr.out, dense, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(tr.lse, dlse, rtol=1e-11, atol=1e-12)
