"""Recall of the stochastic radix top-k on one KV head of the 131072-token
workload (Llama-3-8B-shaped layer, bf16), computed with the oracle alone.

Test infrastructure, like the rest of oracle/: it builds the oracle index of
(sequence 0, KV head 0), scores 20 drifting queries, and compares the sampled
selection (5 seeds each) with the exact top-k.  Run from the repository root:

    python -m oracle.stochastic_recall
"""
import numpy as np
import torch

import wave_inputs as WI

from . import wave_oracle as O


def main(steps: int = 20, seeds: int = 5):
    wl = WI.config(2, device="cpu")
    K = wl.keys[0][0].to(torch.float64).numpy()
    V = wl.values[0][0].to(torch.float64).numpy()
    ix = O.build_unit(K, V, wl.seg_len, wl.cluster_size, wl.iters, "bf16")
    G = wl.n_q_heads // wl.n_kv_heads
    gen = torch.Generator(device="cpu")
    gen.manual_seed(3)
    rec, bins = [], []
    for _ in range(steps):
        q = wl.q[0, :G].to(torch.float64).numpy()
        a = ((q @ ix.centroids.T) / np.sqrt(q.shape[1])).max(0)
        cand = np.ones(len(a), dtype=bool)
        k = O.k_for(len(a), -1, wl.topk_fraction)
        exact = O.select_topk(a, cand, k)
        rec += [O.recall(O.select_topk_stochastic(a, cand, k, s), exact) for s in range(seeds)]
        keys = O.ordered_key32(a.astype(np.float32)) >> 21
        bins.append(int((keys == np.sort(keys)[::-1][k - 1]).sum()))
        WI.drift_queries(wl, gen, sigma=0.05)
    print(f"k={k} recall mean {np.mean(rec):.4f} min {np.min(rec):.4f} "
          f"threshold-bin members median {np.median(bins):.0f}")


if __name__ == "__main__":
    main()
