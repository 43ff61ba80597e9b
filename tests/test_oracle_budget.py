"""Pins of the oracle's node-budget plan across a batch.

The DDTree page (results and trade-offs) has acceptance grow with the node
budget while the verifier's cost grows too; Proposition 1 makes a tree's
expected acceptance the sum of its nodes' prefix probabilities.  The plan
ranks the nodes of every sequence's largest tree by probability and takes
the best n.  These tests tie it to things other than itself:

* brute force over every split of n nodes between the sequences, each
  sequence's tree rebuilt by the oracle's tree builder with its share: the
  best split's summed surrogate equals the plan's expected acceptance, for
  every n;
* the cost model: brute force over n of (batch + best acceptance(n)) /
  (c0 + c1 * n) picks the plan's n;
* each sequence's expected tokens equal 1 + the surrogate of its tree rebuilt
  with the planned budget (Proposition 1 through the tree builder);
* a hand-worked batch of two sequences (tests/golden/budget_two_seqs.json):
  caps and two cost models, worked out on paper.
"""
import itertools

import numpy as np
import pytest

import oracle

from helpers import f32_up


def _case(seed, batch, L, V, k, B, invT=1.0):
    g = np.random.default_rng(seed)
    z = (g.standard_normal((batch, L, V)) * 1.5).astype(np.float32)
    for b in range(batch):  # sequences of different confidence
        z[b] *= 0.5 + b
    ids, zk, logp, lse = oracle.topk(z, k, invT)
    lse = f32_up(lse).astype(np.float64)
    tree = oracle.build_tree(ids, zk, lse, B, invT, n_max=B + 1)
    return ids, zk, lse, tree


def _surrogate(ids, zk, lse, b, Bb, invT, n_max):
    t = oracle.build_tree(ids[b:b + 1], zk[b:b + 1], lse[b:b + 1], Bb, invT, n_max=n_max)
    return float(t["surrogate"][0])


@pytest.mark.parametrize("seed", [1, 2])
def test_best_split_for_every_total(seed):
    batch, L, V, k, B, invT = 3, 3, 12, 3, 6, 1.0
    ids, zk, lse, tree = _case(seed, batch, L, V, k, B, invT)
    avail = [int(n) - 1 for n in tree["n_nodes"]]
    sur = [[_surrogate(ids, zk, lse, b, x, invT, B + 1) for x in range(avail[b] + 1)]
           for b in range(batch)]
    for n in range(sum(avail) + 1):
        best = max(sum(sur[b][x[b]] for b in range(batch))
                   for x in itertools.product(*[range(a + 1) for a in avail]) if sum(x) == n)
        budget, exp_tok, taken = oracle.plan_budget(ids, zk, lse, tree, L, invT, total_budget=n)
        assert taken == n and budget.sum() == n
        assert np.all(budget <= avail)
        assert (exp_tok - 1).sum() == pytest.approx(best, rel=1e-12, abs=1e-15)
        for b in range(batch):  # Proposition 1 through the tree builder
            assert exp_tok[b] - 1 == pytest.approx(sur[b][budget[b]], rel=1e-12, abs=1e-15)


@pytest.mark.parametrize("c0,c1", [(10.0, 1.0), (3.0, 0.2), (50.0, 0.01), (1.0, 5.0)])
def test_cost_model_picks_the_best_total(c0, c1):
    batch, L, V, k, B, invT = 3, 3, 12, 3, 6, 1.0
    ids, zk, lse, tree = _case(7, batch, L, V, k, B, invT)
    avail = [int(n) - 1 for n in tree["n_nodes"]]
    rate = []
    for n in range(sum(avail) + 1):
        _, exp_tok, _ = oracle.plan_budget(ids, zk, lse, tree, L, invT, total_budget=n)
        rate.append(exp_tok.sum() / (c0 + c1 * n))
    budget, exp_tok, taken = oracle.plan_budget(ids, zk, lse, tree, L, invT, cost_fixed=c0,
                                                cost_per_node=c1)
    assert taken == int(np.argmax(rate))
    assert budget.sum() == taken


def test_no_cost_takes_everything_up_to_the_cap():
    ids, zk, lse, tree = _case(3, 4, 4, 20, 4, 12)
    total = int((tree["n_nodes"] - 1).sum())
    budget, exp_tok, taken = oracle.plan_budget(ids, zk, lse, tree, 4, 1.0)
    assert taken == total and np.array_equal(budget, tree["n_nodes"] - 1)
    np.testing.assert_allclose(exp_tok - 1, tree["surrogate"], rtol=1e-12)
    budget, _, taken = oracle.plan_budget(ids, zk, lse, tree, 4, 1.0, total_budget=5)
    assert taken == 5 and budget.sum() == 5


def test_confident_sequences_get_more_nodes():
    """A sequence whose drafter is sharper has likelier prefixes, so it gets
    a larger share of a shared budget (the page's adaptive-budget reading)."""
    ids, zk, lse, tree = _case(5, 2, 4, 30, 4, 20)  # sequence 1's logits are 3x sequence 0's
    budget, _, _ = oracle.plan_budget(ids, zk, lse, tree, 4, 1.0, total_budget=20)
    assert budget[1] > budget[0]


def test_golden_two_sequences():
    """The hand-worked budgets of tests/golden/budget_two_seqs.json (its
    derivation is in the file): caps and two cost models over a batch of two
    sequences of different confidence."""
    import json
    import os
    d = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "budget_two_seqs.json")))
    z = np.log(np.asarray(d["q"], np.float64)).astype(np.float32)
    invT = d["inv_temperature"]
    ids, zk, logp, lse = oracle.topk(z, d["k"], invT)
    tree = oracle.build_tree(ids, zk, lse, d["B"], invT, n_max=d["B"] + 1)
    assert list(tree["n_nodes"]) == [d["B"] + 1] * 2
    for c in d["cases"]:
        budget, exp_tok, taken = oracle.plan_budget(ids, zk, lse, tree, d["L"], invT,
                                                    total_budget=c["total_budget"],
                                                    cost_fixed=c["cost_fixed"],
                                                    cost_per_node=c["cost_per_node"])
        assert taken == c["taken"], c
        assert list(budget) == c["budget"], c
        np.testing.assert_allclose(exp_tok, c["expected_tokens"], rtol=0, atol=1e-6)
