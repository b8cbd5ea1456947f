"""Host-side helpers of bench.py on CPU: the exact top-p counts behind the overshoot statistic
agree with the oracle's sort-based top-p (O2)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from head_wise_sparse_retrieval_b200 import workloads as W  # noqa: E402


def test_exact_top_p_counts_match_the_oracle():
    import bench
    seqs = [3000, 700, 1]
    p = W.custom(batch=3, num_q_heads=8, num_kv_heads=2, seq_lens=seqs, max_ctx=3000,
                 retrieval=[1, 1], kinds=[[W.KIND_DIFFUSE, W.KIND_CONC]] * 3,
                 n_needles=[[0, 3]] * 3, seed=21)
    li = W.make_layer(p, 0, "cpu")
    got = bench.exact_top_p_counts(p, [li], 0.9)
    want = []
    for b in range(3):
        for h in range(2):
            s = oracle.indexer_scores(li.q_idx[b, h].numpy(), li.k_idx[b, h, :seqs[b]].numpy())
            want.append(oracle.exact_topp(s, 0.9).size)
    assert len(got) == len(want) == 6
    # fp32 scores against fp64: a tie at the cut may move the count by one token
    assert all(abs(g - w) <= 1 for g, w in zip(got, want)), (got, want)
    assert sum(g == w for g, w in zip(got, want)) >= 5
    assert got[4] == got[5] == 1  # N = 1
