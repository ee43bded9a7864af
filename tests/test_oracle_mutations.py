"""Plant plausible mistakes in a copy of the oracle (CPU only) and check that
at least one pin catches each.  This guards the pins themselves: a pin set
that a dropped term, a wrong sign or an off-by-one slips through is too weak.
"""
import itertools
import os
import sys
import types

import pytest

import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "wave_oracle.py")

MUTATIONS = {
    "scale 1/d": ("scale = 1.0 / math.sqrt(d)", "scale = 1.0 / d"),
    "no steady value correction": ("vsum_p = ix.value_sums - dv", "vsum_p = ix.value_sums"),
    "no steady count correction": ("cnt_p = cnt - dcnt", "cnt_p = cnt"),
    "group mean instead of max": ("a = s.max(0) if NC", "a = s.mean(0) if NC"),
    "top-k ties to higher index": ("idx.sort(key=lambda c: (-a[c], c))",
                                   "idx.sort(key=lambda c: (-a[c], -c))"),
    "window off by one": ("range(max(T - window, 0), T)", "range(max(T - window - 1, 0), T)"),
    "init at consecutive keys": ("X[np.arange(m) * cluster_size]", "X[np.arange(m)]"),
    "empty cluster reset": ("C = np.array(C_prev, dtype=np.float64, copy=True)",
                            "C = np.zeros_like(C_prev, dtype=np.float64)"),
    "assign sign flip": ("dist = (X * X).sum(1)[:, None] - 2.0", "dist = (X * X).sum(1)[:, None] + 2.0"),
    "distance sign flip": ("    return (X * X).sum(1)[:, None] - 2.0 * (X @ C.T)",
                           "    return (X * X).sum(1)[:, None] + 2.0 * (X @ C.T)"),
    "distance drops the centroid norm": ("- 2.0 * (X @ C.T) + (C * C).sum(1)[None, :]\n\n\ndef kmeans_update",
                                         "- 2.0 * (X @ C.T)\n\n\ndef kmeans_update"),
    "merge drops rescale": ("num += f[:, None] * oi", "num += oi"),
    "steady counted twice": ("if not is_steady_pos[ix.perm[slot]]:", "if True:"),
    "estimate ignores counts": ("cnt_p[X].astype(np.float64)", "np.ones(len(X))"),
    "bf16 truncation": ("np.rint(x[nz] / quantum)", "np.trunc(x[nz] / quantum)"),
    "value sum not mean": ("C[nz] = sums[nz] / counts[nz, None]", "C[nz] = sums[nz]"),
    "extension offsets not rebased": ("offsets[nc0 + 1:] = s0 + np.cumsum(counts)",
                                      "offsets[nc0 + 1:] = np.cumsum(counts)"),
    "extension keeps a partial segment": (
        "s0 = (T_old // seg_len) * seg_len                       # first position clustered anew",
        "s0 = -(-T_old // seg_len) * seg_len"),
    "block summary is the key sum": ("C = ksum / np.maximum(counts, 1)[:, None]", "C = ksum"),
    "stochastic draws ignore the seed": ("splitmix64(((seed & 0xFFFFFFFF) << 32) | int(c))",
                                         "splitmix64(int(c))"),
    "splitmix64 without its last xor-shift": ("    return z ^ (z >> 31)", "    return z"),
    "exact-only keeps the estimate": (
        "X = np.nonzero(candidate & ~is_sel)[0] if estimate else np.zeros(0, dtype=np.int64)",
        "X = np.nonzero(candidate & ~is_sel)[0]"),
}

PINS = [
    lambda: pins.test_round_bf16_matches_torch_on_fp32_inputs(),
    lambda: pins.test_assign_matches_scipy_vq(),
    lambda: pins.test_distances_match_scipy_cdist_and_a_direct_loop(),
    lambda: pins.test_lloyd_matches_sklearn(),
    lambda: pins.test_kmeans_init_positions_and_empty_cluster_keeps_centroid(),
    lambda: pins.test_steady_positions(),
    lambda: pins.test_topk_matches_stable_argsort_and_ties(),
    lambda: pins.test_lse_merge_matches_logsumexp(),
    lambda: pins.test_all_clusters_retrieved_equals_dense_sdpa(4, 4, 64),
    lambda: pins.test_one_token_per_cluster_estimation_is_exact(3, 4, 16),
    lambda: pins.test_brute_force_tiny(64, 4, 3, 2, 5),
    lambda: pins.test_pure_estimate_golden_two_clusters(),
    lambda: pins.test_group_selection_uses_max_over_heads(),
    lambda: pins.test_extension_equals_build_of_the_longer_sequence(1500, 2900),
    lambda: pins.test_block_index_is_positional(),
    lambda: pins.test_exact_only_with_no_block_is_steady_attention(),
    lambda: pins.test_exact_only_brute_force(),
    lambda: pins.test_splitmix64_published_outputs(),
    lambda: pins.test_stochastic_topk_samples_the_threshold_bin_uniformly(),
]


def mutated_oracle(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    name = f"oracle_mutant_{next(_COUNTER)}"
    mod = types.ModuleType(name)
    sys.modules[name] = mod          # dataclasses look their module up by name
    exec(compile(src.replace(old, new), SRC, "exec"), mod.__dict__)
    return mod


_COUNTER = itertools.count()


def test_unmutated_oracle_passes_the_pin_subset(monkeypatch):
    monkeypatch.setattr(pins, "O", mutated_oracle("import math", "import math"))
    for pin in PINS:
        pin()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    old, new = MUTATIONS[name]
    monkeypatch.setattr(pins, "O", mutated_oracle(old, new))
    caught = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake {name!r}"
