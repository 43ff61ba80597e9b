"""The budget sweep's synthetic target (bench.plant_targets), on CPU.

Each live row of depth d < L gets its argmax at a token drawn from the
drafter's marginal q_{d+1}, so the greedy walk accepts a path with the
probability the factorised draft gives it, and the mean accepted length
converges to the tree's surrogate (DDTree page, 理論基礎, Proposition 1).
"""
import os
import sys

import numpy as np
import torch
from scipy import stats

import oracle

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_planted_rows_and_their_distribution():
    g = torch.Generator().manual_seed(3)
    b, L, V, n_max = 2, 3, 12, 9
    probs = torch.softmax(torch.randn(b, L, V, generator=g), -1)
    depth = torch.tensor([[0, 1, 1, 2, 3, 2, 0, 0, 0], [0, 1, 2, 3, 0, 0, 0, 0, 0]])
    n_nodes = torch.tensor([6, 4])
    counts = np.zeros((L, V))
    for r in range(3000):
        base = torch.randn(b, n_max, V, generator=g)
        tgt = base.clone()
        tok = bench.plant_targets(tgt, probs, depth, n_nodes, L, g)
        live = (torch.arange(n_max)[None] < n_nodes[:, None]) & (depth < L)
        assert torch.equal(tok >= 0, live)
        assert torch.equal(tgt.argmax(-1)[live], tok[live])
        assert torch.equal(tgt[~live], base[~live])
        for x in range(n_max):
            if live[0, x]:
                counts[int(depth[0, x]), int(tok[0, x])] += 1
    for d in range(L):
        n = counts[d].sum()
        p = probs[0, d].double().numpy()
        assert stats.chisquare(counts[d], p / p.sum() * n).pvalue > 1e-4


def test_mean_acceptance_is_the_surrogate():
    """Oracle tree + oracle greedy walk over planted targets."""
    rng = np.random.default_rng(5)
    L, V, k, B = 4, 10, 3, 12
    z = rng.standard_normal((1, L, V)).astype(np.float32) * 1.5
    ids, zk, logp, lse = oracle.topk(z, k, 1.0)
    tree = oracle.build_tree(ids, zk, lse, B, 1.0)
    n = int(tree["n_nodes"][0])
    probs = torch.softmax(torch.from_numpy(z).double(), -1)
    depth = torch.from_numpy(tree["depth"]).long()
    g = torch.Generator().manual_seed(11)
    acc = []
    for r in range(4000):
        tgt = torch.randn(1, tree["tok"].shape[1], V, generator=g, dtype=torch.float64)
        bench.plant_targets(tgt, probs, depth, torch.tensor([n]), L, g)
        res = oracle.tree_walk(tgt.float().numpy(), tree["tok"], tree["parent"], tree["depth"],
                               tree["n_nodes"], L)
        acc.append(int(res["acc_len"][0]))
    acc = np.array(acc, np.float64)
    se = acc.std() / np.sqrt(len(acc))
    assert abs(acc.mean() - tree["surrogate"][0]) < 5 * se
