"""Wave-index oracle: a plain, slow, fp64 restatement of the method.

TEST INFRASTRUCTURE ONLY.  Only tests/, the package-level smoke check and the
bench's CPU-baseline leg may import this module.  It shares no code with the
CUDA path (no kernels, helpers, tables or pre/post-processing) and imports
nothing from it.

Sources (page title, section):
  [RI]  "RetroInfer: A Vector Storage Engine for Scalable Long-Context LLM
        Inference" (technical summary), section 2.A "Wave Index": item 1
        Steady Zone, item 2 Retrieval Zone, item 3 Estimation Zone, and the
        Segmented Clustering paragraph.
  [VX]  "Vortex - Servizio di Attention Sparsa Efficiente e Programmabile per
        Agenti AI", section 2.A (two-phase forward_cache / forward_indexer;
        primitives GeMM, Softmax, Top-K, Gather) and 2.B (vTensor layout).
  [IC]  "IceCache: Memory-Efficient KV-cache Management for Long-Sequence
        LLMs" (catalog summary): attention sinks and the decoded tail stay
        resident; pages are filled by similarity, not position.

Readings where the pages are silent or leave a step open:
  R-1 k-means distance is squared Euclidean on the raw keys.
  R-2 a segment of n tokens gets ceil(n/cs) centroids, centroid j starts as the
      key at segment position j*cs; `iters` rounds of (assign, update); an
      empty cluster keeps its centroid; the stored centroid is the mean of the
      final assignment.
  R-3 every token is counted once: steady tokens are removed from the clusters
      they belong to, both when a cluster is retrieved (they are skipped) and
      when it is estimated (count and value sum are reduced); clusters left
      with no non-steady token are neither candidates nor estimated.
  R-4 GQA: q head h reads KV head floor(h/G); a cluster's selection score for a
      KV head is the max over the group's q heads; each q head estimates with
      its own score.
  R-5 k per (sequence, KV head) = topk_clusters, or ceil(fraction * NC).
  R-6 ties (top-k and argmin) go to the lower index.
  R-7 centroids and value sums are stored in the KV dtype (round to nearest
      even from the exact mean / sum); decode reads the stored values.
  R-8 softmax scale 1/sqrt(d); no causal mask at decode.
  R-14 an index grows segment by segment: the whole segments of the old index
      are kept, a partial last one is clustered again with its new tokens.
  R-15 a block of the block top-k workload is block_size consecutive
      positions inside a segment; its summary is the mean key; blocks are
      scored and selected like clusters; the workload has no estimation zone.
  R-16 the stochastic top-k ranks by the top 11 bits of the fp32 score's
      order-preserving key and samples the threshold bin without replacement
      by a SplitMix64 draw per cluster id.

Parity pins for every function here live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Tuple

import numpy as np


# ---------------------------------------------------------------------------
# Rounding to the stored dtype (reading R-7)
# ---------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (ties to even), returned as fp64.

    bfloat16 keeps 8 significant bits and fp32's exponent range; below 2^-126
    the spacing stays 2^-133 (subnormals).  Overflow goes to +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    _, e = np.frexp(x[nz])                       # x = m * 2^e, 0.5 <= |m| < 1
    quantum = np.ldexp(1.0, np.maximum(e - 1, -126) - 7)
    out[nz] = np.rint(x[nz] / quantum) * quantum  # np.rint rounds half to even
    out[~nz] = x[~nz]
    big = np.abs(out) > 3.3895313892515355e38     # largest finite bfloat16
    out[big] = np.sign(out[big]) * np.inf
    return out


def round_stored(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round to the KV storage dtype ('bf16' or 'f32'), kept as fp64 values."""
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# Segmented clustering ([RI] 2.A, Segmented Clustering paragraph)
# ---------------------------------------------------------------------------

def segment_spans(T: int, seg_len: int) -> List[Tuple[int, int]]:
    """The sequence is cut into consecutive segments of seg_len tokens; the last
    one may be shorter.  Returns (start, length) pairs."""
    return [(s, min(seg_len, T - s)) for s in range(0, T, seg_len)]


def clusters_in_segment(length: int, cluster_size: int) -> int:
    """R-2: ceil(length / cluster_size) centroids per segment."""
    return -(-length // cluster_size)


def n_clusters(T: int, seg_len: int, cluster_size: int) -> int:
    return sum(clusters_in_segment(n, cluster_size) for _, n in segment_spans(T, seg_len))


def kmeans_init(X: np.ndarray, cluster_size: int) -> np.ndarray:
    """R-2: centroid j starts as the key at segment position j*cluster_size."""
    m = clusters_in_segment(len(X), cluster_size)
    return X[np.arange(m) * cluster_size].astype(np.float64).copy()


def kmeans_assign(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    """Assignment step: each key goes to argmin_j ||x - c_j||^2 (R-1), the
    lowest j on ties (R-6).  The squared distance is expanded as
    ||x||^2 - 2 x.c + ||c||^2 and evaluated with an fp64 matrix product."""
    X = np.asarray(X, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    dist = (X * X).sum(1)[:, None] - 2.0 * (X @ C.T) + (C * C).sum(1)[None, :]
    return np.argmin(dist, axis=1)               # argmin returns the first minimum


def kmeans_distances(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    """||x_i - c_j||^2 for all pairs (fp64), used by near-tie checks."""
    X = np.asarray(X, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    return (X * X).sum(1)[:, None] - 2.0 * (X @ C.T) + (C * C).sum(1)[None, :]


def kmeans_update(X: np.ndarray, labels: np.ndarray, C_prev: np.ndarray) -> np.ndarray:
    """Update step: each centroid becomes the mean of its members; a centroid
    with no member keeps its previous value (R-2)."""
    X = np.asarray(X, dtype=np.float64)
    m = len(C_prev)
    counts = np.bincount(labels, minlength=m)
    sums = np.zeros_like(C_prev, dtype=np.float64)
    np.add.at(sums, labels, X)
    C = np.array(C_prev, dtype=np.float64, copy=True)
    nz = counts > 0
    C[nz] = sums[nz] / counts[nz, None]
    return C


def kmeans_objective(X: np.ndarray, labels: np.ndarray, C: np.ndarray) -> float:
    """Sum of squared distances of each key to its assigned centroid."""
    diff = np.asarray(X, dtype=np.float64) - np.asarray(C, dtype=np.float64)[labels]
    return float((diff * diff).sum())


def kmeans_segment(X: np.ndarray, cluster_size: int, iters: int, C0: Optional[np.ndarray] = None):
    """Lloyd iterations on one segment: `iters` rounds of (assign, update).

    Returns (labels of the last assignment, centroids = means of that
    assignment, objective after every assign and every update)."""
    if iters < 1:
        raise ValueError("iters must be >= 1")
    C = kmeans_init(X, cluster_size) if C0 is None else np.array(C0, dtype=np.float64)
    history = []
    labels = None
    for _ in range(iters):
        labels = kmeans_assign(X, C)
        history.append(kmeans_objective(X, labels, C))
        C = kmeans_update(X, labels, C)
        history.append(kmeans_objective(X, labels, C))
    return labels, C, history


@dataclass
class UnitIndex:
    """The wave index of one (sequence, KV head): the query-independent phase
    ([VX] 2.A forward_cache) of the method."""
    centroids: np.ndarray      # [NC][d] stored dtype values (fp64 array)
    value_sums: np.ndarray     # [NC][d] stored dtype values
    offsets: np.ndarray        # [NC+1] int64, slot range of each cluster
    perm: np.ndarray           # [T] slot -> original position
    invperm: np.ndarray        # [T] original position -> slot
    k_perm: np.ndarray         # [T][d] keys in slot order
    v_perm: np.ndarray         # [T][d] values in slot order
    labels: np.ndarray         # [T] global cluster id of each original position
    centroids_exact: np.ndarray  # [NC][d] fp64 means before rounding
    value_sums_exact: np.ndarray  # [NC][d] fp64 sums before rounding


def build_unit(K: np.ndarray, V: np.ndarray, seg_len: int, cluster_size: int, iters: int,
               store: str, kmeans_iters_hook=None) -> UnitIndex:
    """Index build for one (sequence, KV head): segmented k-means ([RI] 2.A),
    then the cluster-permuted layout the retrieval zone reads.

    Cluster ids are global: the clusters of segment s follow those of s-1.
    Slots are cluster-major; inside a cluster, members keep ascending original
    position.  Because clusters never cross a segment, segment s occupies the
    same slot range as its position range.
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    T, d = K.shape
    labels = np.empty(T, dtype=np.int64)
    cents = []
    base = 0
    for start, n in segment_spans(T, seg_len):
        lab, C, _ = kmeans_segment(K[start:start + n], cluster_size, iters)
        labels[start:start + n] = lab + base
        cents.append(C)
        base += len(C)
    NC = base
    C = np.concatenate(cents, 0) if cents else np.zeros((0, d))
    counts = np.bincount(labels, minlength=NC)
    offsets = np.zeros(NC + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(labels, kind="stable")     # cluster-major, positions ascending
    invperm = np.empty(T, dtype=np.int64)
    invperm[perm] = np.arange(T)
    vsum = np.zeros((NC, d))
    np.add.at(vsum, labels, V)
    return UnitIndex(centroids=round_stored(C, store), value_sums=round_stored(vsum, store),
                     offsets=offsets, perm=perm, invperm=invperm, k_perm=K[perm], v_perm=V[perm],
                     labels=labels, centroids_exact=C, value_sums_exact=vsum)


def build_blocks_unit(K: np.ndarray, V: np.ndarray, seg_len: int, block_size: int,
                      store: str) -> UnitIndex:
    """Index of position-contiguous blocks for one (sequence, KV head): inside
    each segment, block j holds positions j*block_size .. (j+1)*block_size - 1
    (the last one may be shorter); its summary is the block's mean key (the
    block centroid of [VX] 2.A forward_cache), its value sum the sum of its
    values.  Blocks keep position order, so perm is the identity."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    T, d = K.shape
    labels = np.empty(T, dtype=np.int64)
    base = 0
    for start, n in segment_spans(T, seg_len):
        labels[start:start + n] = base + np.arange(n) // block_size
        base += clusters_in_segment(n, block_size)
    NC = base
    counts = np.bincount(labels, minlength=NC)
    offsets = np.zeros(NC + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    ksum = np.zeros((NC, d))
    vsum = np.zeros((NC, d))
    np.add.at(ksum, labels, K)
    np.add.at(vsum, labels, V)
    C = ksum / np.maximum(counts, 1)[:, None]
    perm = np.arange(T, dtype=np.int64)
    return UnitIndex(centroids=round_stored(C, store), value_sums=round_stored(vsum, store),
                     offsets=offsets, perm=perm, invperm=perm.copy(), k_perm=K.copy(),
                     v_perm=V.copy(), labels=labels, centroids_exact=C, value_sums_exact=vsum)


def extend_unit(old: UnitIndex, K: np.ndarray, V: np.ndarray, seg_len: int, cluster_size: int,
                iters: int, store: str) -> UnitIndex:
    """Grow the index `old` of a sequence's first T_old tokens to the longer
    sequence K, V ([RI] 2.A, Segmented Clustering: segments are clustered
    independently).  The segments of `old` that are whole are kept as they
    are (their centroids, value sums, offsets, slots and labels); from the
    first position they do not cover on, segments are clustered anew, a
    partial last segment of `old` together with its new tokens."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    T, d = K.shape
    T_old = len(old.perm)
    assert T_old <= T
    s0 = (T_old // seg_len) * seg_len                       # first position clustered anew
    nc0 = (T_old // seg_len) * clusters_in_segment(seg_len, cluster_size)
    labels = np.empty(T, dtype=np.int64)
    labels[:s0] = old.labels[:s0]
    cents, base = [], nc0
    for start, n in segment_spans(T, seg_len):
        if start < s0:
            continue
        lab, C, _ = kmeans_segment(K[start:start + n], cluster_size, iters)
        labels[start:start + n] = lab + base
        cents.append(C)
        base += len(C)
    NC = base
    C_new = np.concatenate(cents, 0) if cents else np.zeros((0, d))
    counts = np.bincount(labels[s0:] - nc0, minlength=NC - nc0)
    offsets = np.zeros(NC + 1, dtype=np.int64)
    offsets[:nc0 + 1] = old.offsets[:nc0 + 1]
    offsets[nc0 + 1:] = s0 + np.cumsum(counts)
    perm = np.concatenate([old.perm[:s0], s0 + np.argsort(labels[s0:], kind="stable")])
    invperm = np.empty(T, dtype=np.int64)
    invperm[perm] = np.arange(T)
    vsum_new = np.zeros((NC - nc0, d))
    np.add.at(vsum_new, labels[s0:] - nc0, V[s0:])
    exact_c = exact_v = None
    if old.centroids_exact is not None and old.value_sums_exact is not None:
        exact_c = np.concatenate([old.centroids_exact[:nc0], C_new], 0)
        exact_v = np.concatenate([old.value_sums_exact[:nc0], vsum_new], 0)
    return UnitIndex(centroids=np.concatenate([old.centroids[:nc0], round_stored(C_new, store)], 0),
                     value_sums=np.concatenate([old.value_sums[:nc0],
                                                round_stored(vsum_new, store)], 0),
                     offsets=offsets, perm=perm, invperm=invperm, k_perm=K[perm], v_perm=V[perm],
                     labels=labels, centroids_exact=exact_c, value_sums_exact=exact_v)


# ---------------------------------------------------------------------------
# Decode: steady, retrieval and estimation zones ([RI] 2.A items 1-3)
# ---------------------------------------------------------------------------

def steady_positions(T: int, n_sink: int, window: int) -> np.ndarray:
    """Steady zone ([RI] 2.A item 1; [IC] sinks and tail resident): the first
    n_sink positions and the last `window` positions, each counted once."""
    pos = set(range(min(n_sink, T))) | set(range(max(T - window, 0), T))
    return np.array(sorted(pos), dtype=np.int64)


def k_for(NC: int, topk_clusters: int, topk_fraction: float) -> int:
    """R-5: a fixed k, or ceil(fraction * NC) computed in double precision."""
    if topk_clusters >= 0:
        return int(topk_clusters)
    return int(math.ceil(float(topk_fraction) * NC))


def select_topk(a: np.ndarray, candidate: np.ndarray, k: int) -> np.ndarray:
    """Retrieval zone selection ([RI] 2.A item 2; [VX] 2.A Top-K): the k
    candidates with the largest score, lower index first on equal scores
    (R-6).  k is clamped to the number of candidates.  Returned ascending."""
    idx = [c for c in range(len(a)) if candidate[c]]
    idx.sort(key=lambda c: (-a[c], c))
    return np.array(sorted(idx[:k]), dtype=np.int64)


# ---------------------------------------------------------------------------
# Stochastic radix top-k ([VX] 2.C): a speed variant of the selection that
# trades exactness for fewer refinement passes
# ---------------------------------------------------------------------------

_M64 = (1 << 64) - 1


def splitmix64(x: int) -> int:
    """One output of the SplitMix64 generator from state x (Steele, Lea and
    Flood, "Fast splittable pseudorandom number generators", 2014): advance
    the state by the golden-ratio increment, then two xor-shift-multiply
    rounds and a final xor-shift."""
    z = (x + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def ordered_key32(x: np.ndarray) -> np.ndarray:
    """Order-preserving uint32 key of float32 values: a negative value has all
    its bits inverted, a non-negative one its sign bit set, so unsigned key
    order is the numeric order."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    return np.where(b & np.uint32(0x80000000), ~b, b | np.uint32(0x80000000)).astype(np.uint32)


def select_topk_stochastic(a: np.ndarray, candidate: np.ndarray, k: int, seed: int,
                           digit_bits: int = 11) -> np.ndarray:
    """Stochastic radix top-k ([VX] 2.C: stop early by sampling from the
    threshold bin once the high-confidence candidates are known).

    The selection scores are ranked by the top `digit_bits` bits of their
    order-preserving key, taken in fp32 as the kernel computes them.  Every
    candidate in a bin above the bin holding the k-th largest key is taken;
    the k - (that many) remaining picks are drawn without replacement from
    the threshold bin: member c draws u_c = splitmix64(seed * 2^32 + c) and
    the smallest (u_c, c) win.  k is clamped to the candidate count.
    Returned ascending."""
    idx = np.nonzero(np.asarray(candidate, dtype=bool))[0].astype(np.int64)
    k = min(max(int(k), 0), len(idx))
    if k == 0:
        return np.zeros(0, dtype=np.int64)
    if k == len(idx):
        return idx
    bins = ordered_key32(np.asarray(a, dtype=np.float64)[idx].astype(np.float32)) >> (32 - digit_bits)
    b_star = np.sort(bins)[::-1][k - 1]
    above = idx[bins > b_star]
    members = idx[bins == b_star]
    krem = k - len(above)
    u = np.array([splitmix64(((seed & 0xFFFFFFFF) << 32) | int(c)) for c in members],
                 dtype=np.uint64)
    picked = members[np.lexsort((members, u))[:krem]]
    return np.sort(np.concatenate([above, picked]))


def recall(selected: np.ndarray, exact: np.ndarray) -> float:
    """Fraction of the exact top-k that a selection retrieves (1 when k = 0)."""
    if len(exact) == 0:
        return 1.0
    return len(np.intersect1d(selected, exact)) / len(exact)


def zone_stats(scores: np.ndarray, weights: np.ndarray, values: np.ndarray):
    """One softmax part: m = max score, l = sum_i w_i e^(s_i - m),
    o = sum_i e^(s_i - m) value_i.  An empty part is (-inf, 0, 0)."""
    G = scores.shape[0]
    d = values.shape[1]
    if scores.shape[1] == 0:
        return np.full(G, -np.inf), np.zeros(G), np.zeros((G, d))
    m = scores.max(1)
    e = np.exp(scores - m[:, None])
    return m, (e * weights[None, :]).sum(1), e @ values


def lse_merge(parts):
    """Log-sum-exp combine of softmax parts (m_i, l_i, o_i): with m = max m_i,
    out = sum e^(m_i-m) o_i / sum e^(m_i-m) l_i and lse = m + ln(denominator)."""
    ms = np.stack([p[0] for p in parts])         # [P][G]
    m = ms.max(0)
    G = m.shape[0]
    d = parts[0][2].shape[1]
    num = np.zeros((G, d))
    den = np.zeros(G)
    for (mi, li, oi) in parts:
        f = np.where(np.isfinite(mi), np.exp(mi - np.where(np.isfinite(m), m, 0.0)), 0.0)
        num += f[:, None] * oi
        den += f * li
    with np.errstate(divide="ignore", invalid="ignore"):
        out = np.where(den[:, None] > 0, num / np.where(den > 0, den, 1.0)[:, None], 0.0)
        lse = np.where(den > 0, m + np.log(np.where(den > 0, den, 1.0)), -np.inf)
    return out, lse


@dataclass
class DecodeTrace:
    out: np.ndarray          # [G][d]
    lse: np.ndarray          # [G]
    selected: np.ndarray     # ascending cluster ids
    scores: np.ndarray       # [G][NC] q.kbar / sqrt(d)
    sel_score: np.ndarray    # [NC] max over the group
    candidate: np.ndarray    # [NC] bool
    k: int
    exact: tuple             # (m, l, o) of the exact part
    estimate: tuple          # (m, l, o) of the estimation part


def decode_unit(q: np.ndarray, ix: UnitIndex, n_sink: int, window: int, k: int,
                selected: Optional[np.ndarray] = None, estimate: bool = True) -> DecodeTrace:
    """One decode step of one KV head's query group ([VX] 2.A forward_indexer).

    q: [G][d] query heads of the group (values as fed to the kernel).
    (a) score every centroid: s[h,c] = q_h . kbar_c / sqrt(d);
    (b) select the top-k clusters on max_h s[h,c] among candidates (R-3, R-4);
    (c) exact attention over the steady zone plus the non-steady members of the
        selected clusters ([RI] item 1 and item 2);
    (d) every other candidate cluster c contributes cnt'_c * e^(s[h,c]) with
        value sum Vsum'_c ([RI] item 3: the cluster counted |C| times at its
        centroid score, times its mean value);
    (e) the two parts are combined by log-sum-exp.
    `selected` overrides step (b) (used to compare downstream steps on a given set).
    estimate=False leaves step (d) out: attention over the retrieved blocks and
    the steady zone only, the block top-k workload ([VX] 2.A: forward_cache
    builds block centroids, forward_indexer selects the top-k blocks and
    attends; [VX] results: "block top-k").
    """
    q = np.asarray(q, dtype=np.float64)
    G, d = q.shape
    T = len(ix.perm)
    NC = len(ix.centroids)
    scale = 1.0 / math.sqrt(d)

    steady_pos = steady_positions(T, n_sink, window)
    is_steady_pos = np.zeros(T, dtype=bool)
    is_steady_pos[steady_pos] = True
    steady_slots = ix.invperm[steady_pos]
    cl_of_slot = np.searchsorted(ix.offsets, steady_slots, side="right") - 1
    dcnt = np.bincount(cl_of_slot, minlength=NC) if NC else np.zeros(0, dtype=np.int64)
    dv = np.zeros((NC, d))
    np.add.at(dv, cl_of_slot, ix.v_perm[steady_slots])
    cnt = np.diff(ix.offsets)
    cnt_p = cnt - dcnt
    vsum_p = ix.value_sums - dv
    candidate = cnt_p > 0

    s = (q @ ix.centroids.T) * scale             # [G][NC]
    a = s.max(0) if NC else np.zeros(0)
    if selected is None:
        sel = select_topk(a, candidate, k)
    else:
        sel = np.asarray(selected, dtype=np.int64)
    is_sel = np.zeros(NC, dtype=bool)
    is_sel[sel] = True

    # exact part: selected clusters' non-steady slots, then the steady slots
    ex = []
    for c in sel:
        for slot in range(ix.offsets[c], ix.offsets[c + 1]):
            if not is_steady_pos[ix.perm[slot]]:
                ex.append(slot)
    ex = np.array(ex + list(steady_slots), dtype=np.int64)
    s_ex = (q @ ix.k_perm[ex].T) * scale
    exact = zone_stats(s_ex, np.ones(len(ex)), ix.v_perm[ex])

    # estimation part: candidates not selected
    X = np.nonzero(candidate & ~is_sel)[0] if estimate else np.zeros(0, dtype=np.int64)
    est = zone_stats(s[:, X], cnt_p[X].astype(np.float64), vsum_p[X])

    out, lse = lse_merge([exact, est])
    return DecodeTrace(out=out, lse=lse, selected=sel, scores=s, sel_score=a,
                       candidate=candidate, k=k, exact=exact, estimate=est)


def dense_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray):
    """Full softmax attention of q [G][d] over all T tokens (no mask)."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    s = (q @ K.T) / math.sqrt(q.shape[1])
    m = s.max(1)
    e = np.exp(s - m[:, None])
    l = e.sum(1)
    return (e @ V) / l[:, None], m + np.log(l)


# ---------------------------------------------------------------------------
# Batched helpers: (sequence, KV head) units of a workload
# ---------------------------------------------------------------------------

def build_all(keys, values, seg_len, cluster_size, iters, store) -> List[List[UnitIndex]]:
    """keys[b], values[b]: [Hkv][T_b][d].  Returns index[b][hkv]."""
    return [[build_unit(kb[h], vb[h], seg_len, cluster_size, iters, store)
             for h in range(kb.shape[0])] for kb, vb in zip(keys, values)]


def decode_all(q: np.ndarray, index, n_sink, window, topk_clusters, topk_fraction):
    """q: [B][Hq][d].  Returns out [B][Hq][d], lse [B][Hq], traces[b][hkv]."""
    B, Hq, d = q.shape
    Hkv = len(index[0])
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    traces = []
    for b in range(B):
        tb = []
        for h in range(Hkv):
            ix = index[b][h]
            k = k_for(len(ix.centroids), topk_clusters, topk_fraction)
            tr = decode_unit(q[b, h * G:(h + 1) * G], ix, n_sink, window, k)
            out[b, h * G:(h + 1) * G] = tr.out
            lse[b, h * G:(h + 1) * G] = tr.lse
            tb.append(tr)
        traces.append(tb)
    return out, lse, traces
