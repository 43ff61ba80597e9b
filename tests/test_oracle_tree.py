"""Pins for the oracle's step 2 (best-B prefixes) and its compilation.

DDTree page: section 核心創新 (best-first selection under a node budget B),
運作流程 steps 2-3, 理論基礎 Propositions 1-2.  Pins:

* brute force -- every prefix of the k-ary, depth-L candidate trie enumerated
  and sorted by the total order, on tiny inputs with and without ties;
* Proposition 2 -- the selected set is prefix-closed and no other tree of
  size B has a larger surrogate (all trees enumerated on tiny inputs);
* Proposition 1 -- the surrogate equals an independent recursion over the
  compiled tree and a Monte-Carlo estimate of the accepted length when
  target tokens are drawn from the factorised draft;
* hand-worked fixtures in tests/golden/;
* compile invariants (breadth-first order, parent/depth/position, ancestor
  masks from the OR recurrence) and the single-path (k=1) special case.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _topk_inputs(seed, L, V, k, ties=False, inv_t=1.0):
    g = np.random.default_rng(seed)
    if ties:
        z = g.integers(-2, 3, size=(1, L, V)).astype(np.float32)
    else:
        z = g.standard_normal((1, L, V), dtype=np.float32) * 2
    ids, zk, logp, lse = oracle.topk(z, k, inv_t)
    return z, ids, zk, logp, lse


def _paths(tree, b=0):
    """token path (root excluded) of every row of a compiled tree."""
    n = int(tree["n_nodes"][b])
    par, tok = tree["parent"][b], tree["tok"][b]
    out = []
    for j in range(n):
        p, x = [], j
        while x > 0:
            p.append(int(tok[x]))
            x = int(par[x])
        out.append(tuple(reversed(p)))
    return out


def brute_force(ids, zk, lse, B, inv_t, k=None):
    """All prefixes of the candidate trie, sorted by the total order."""
    L, kmax = ids.shape
    k = kmax if k is None else k
    it = float(np.float32(inv_t))
    S = [0.0]
    for t in range(L):
        S.append(S[-1] + float(lse[t]))
    keys = []
    for t in range(1, L + 1):
        for ranks in itertools.product(range(k), repeat=t):
            sz = 0.0
            for i, r in enumerate(ranks):
                sz += float(zk[i, r])
            score = it * sz - S[t]
            toks = tuple(int(ids[i, r]) for i, r in enumerate(ranks))
            keys.append(((-score, t, -sz, tuple(reversed(toks))), toks, score))
    keys.sort(key=lambda e: e[0])
    return keys[:B]


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("ties", [False, True])
def test_selection_equals_brute_force(seed, ties):
    g = np.random.default_rng(100 + seed)
    L = int(g.integers(1, 5))
    k = int(g.integers(1, 5))
    V = int(g.integers(max(k, 3), 9))
    inv_t = [1.0, 0.5, 2.0][seed % 3]
    z, ids, zk, logp, lse = _topk_inputs(seed, L, V, k, ties, inv_t)
    total = sum(k ** t for t in range(1, L + 1))
    for B in sorted({0, 1, 2, min(5, total), total // 2, total}):
        tree = oracle.build_tree(ids, zk, lse, B, inv_t)
        got = set(_paths(tree)[1:])
        ref = brute_force(ids[0], zk[0], lse[0], B, inv_t)
        assert got == {e[1] for e in ref}, (L, k, B)
        np.testing.assert_allclose(tree["surrogate"][0], sum(np.exp(e[2]) for e in ref),
                                   rtol=1e-12, atol=0)


def _check_compiled(tree, ids, L, ctx_len, b=0):
    n = int(tree["n_nodes"][b])
    tok, par, dep, pos, mask = (tree[x][b] for x in ("tok", "parent", "depth", "pos", "mask"))
    assert par[0] == -1 and dep[0] == 0 and pos[0] == ctx_len
    ranks = [0]
    for j in range(1, n):
        assert 0 <= par[j] < j
        assert dep[j] == dep[par[j]] + 1 <= L
        assert pos[j] == ctx_len + dep[j]
        lst = list(ids[b, dep[j] - 1])
        ranks.append(lst.index(tok[j]))
    keys = [(int(dep[j]), int(par[j]), ranks[j]) for j in range(1, n)]
    assert keys == sorted(keys), "rows are not in breadth-first order"
    # siblings form a prefix of the candidate list (a down-set)
    for j in range(1, n):
        if ranks[j] > 0:
            assert any(par[i] == par[j] and ranks[i] == ranks[j] - 1 for i in range(1, n))
    # ancestor masks by the OR recurrence (the oracle walks parent pointers)
    W = mask.shape[-1]
    ref = np.zeros((n, W), np.uint32)
    for j in range(n):
        if j > 0:
            ref[j] = ref[par[j]]
        ref[j, j // 32] |= np.uint32(1 << (j % 32))
    np.testing.assert_array_equal(mask[:n], ref)
    assert np.all(mask[n:] == 0) and np.all(tok[n:] == -1) and np.all(par[n:] == -1)
    assert np.all(dep[n:] == -1) and np.all(pos[n:] == -1)


@pytest.mark.parametrize("L,k,B,V", [(16, 8, 64, 500), (16, 16, 256, 600), (32, 16, 512, 300),
                                     (5, 3, 40, 20), (3, 2, 14, 5)])
def test_compiled_tree_invariants(L, k, B, V):
    z, ids, zk, logp, lse = _topk_inputs(L * 31 + B, L, V, k)
    tree = oracle.build_tree(ids, zk, lse, B, 1.0, root_token=7, ctx_len=1234)
    assert tree["n_nodes"][0] == B + 1
    assert tree["tok"][0, 0] == 7
    _check_compiled(tree, ids, L, 1234)


def _all_trees(L, k, B):
    nodes = [r for t in range(1, L + 1) for r in itertools.product(range(k), repeat=t)]
    for sub in itertools.combinations(nodes, B):
        s = set(sub)
        if all(len(p) == 1 or p[:-1] in s for p in sub):
            yield sub


@pytest.mark.parametrize("seed", range(6))
def test_optimal_among_all_trees(seed):
    L, k, V = 2, 3, 6
    z, ids, zk, logp, lse = _topk_inputs(900 + seed, L, V, k, ties=(seed % 2 == 1))
    for B in (1, 3, 5, 7):
        tree = oracle.build_tree(ids, zk, lse, B, 1.0)
        best = max(sum(np.exp(sum(logp[0, i, r] for i, r in enumerate(p))) for p in t)
                   for t in _all_trees(L, k, B))
        np.testing.assert_allclose(tree["surrogate"][0], best, rtol=1e-12)


def _node_logq(tree, ids, logp, b=0):
    n = int(tree["n_nodes"][b])
    out = np.zeros(n)
    for j in range(1, n):
        d = int(tree["depth"][b, j])
        r = list(ids[b, d - 1]).index(tree["tok"][b, j])
        out[j] = logp[b, d - 1, r]
    return out


@pytest.mark.parametrize("L,k,B", [(3, 3, 6), (4, 2, 9), (6, 4, 30)])
def test_surrogate_equals_recursion(L, k, B):
    z, ids, zk, logp, lse = _topk_inputs(L * 7 + k, L, 12, k)
    tree = oracle.build_tree(ids, zk, lse, B, 1.0)
    lq = _node_logq(tree, ids, logp)
    n = int(tree["n_nodes"][0])
    par = tree["parent"][0]
    E = np.zeros(n)
    for j in range(n - 1, 0, -1):  # children after parents: sweep backwards
        E[par[j]] += np.exp(lq[j]) * (1.0 + E[j])
    np.testing.assert_allclose(E[0], tree["surrogate"][0], rtol=1e-12)


def test_surrogate_is_expected_acceptance_monte_carlo():
    L, k, B, V = 3, 3, 6, 8
    z, ids, zk, logp, lse = _topk_inputs(4242, L, V, k)
    tree = oracle.build_tree(ids, zk, lse, B, 1.0)
    zf = z[0].astype(np.float64)
    q = np.exp(zf - zf.max(-1, keepdims=True))
    q /= q.sum(-1, keepdims=True)
    g = np.random.default_rng(7)
    M = 200_000
    draws = np.stack([g.choice(V, size=M, p=q[i]) for i in range(L)], 1)
    n = int(tree["n_nodes"][0])
    child = {}
    for j in range(1, n):
        child[(int(tree["parent"][0, j]), int(tree["tok"][0, j]))] = j
    acc = np.zeros(M)
    for m in range(M):
        x, a = 0, 0
        for i in range(L):
            x = child.get((x, int(draws[m, i])), -1)
            if x < 0:
                break
            a += 1
        acc[m] = a
    se = acc.std() / np.sqrt(M)
    assert abs(acc.mean() - tree["surrogate"][0]) < 5 * se + 1e-9


def test_single_path_is_argmax_chain():
    L, V = 7, 50
    z, ids, zk, logp, lse = _topk_inputs(3, L, V, 1)
    tree = oracle.build_tree(ids, zk, lse, L, 1.0, root_token=9)
    assert tree["n_nodes"][0] == L + 1
    np.testing.assert_array_equal(tree["parent"][0], np.arange(-1, L))
    np.testing.assert_array_equal(tree["tok"][0, 1:], z[0].argmax(-1))
    # a chain's surrogate is the sum of cumulative products of the marginals
    cp = np.cumsum(logp[0, :, 0])
    np.testing.assert_allclose(tree["surrogate"][0], np.exp(cp).sum(), rtol=1e-12)


def test_budget_larger_than_trie():
    z, ids, zk, logp, lse = _topk_inputs(1, 2, 5, 2)
    tree = oracle.build_tree(ids, zk, lse, 6, 1.0, n_max=10)
    assert tree["n_nodes"][0] == 7


@pytest.mark.parametrize("fixture", ["tree_b5.json", "tree_temp2.json"])
def test_golden_trees(fixture):
    d = json.load(open(os.path.join(GOLDEN, fixture)))
    z = np.log(np.asarray(d["q"], np.float64)).astype(np.float32)[None]
    ids, zk, logp, lse = oracle.topk(z, d["k"], d["inv_temperature"])
    for case in d["cases"]:
        tree = oracle.build_tree(ids, zk, lse, case["B"], d["inv_temperature"],
                                 root_token=d["root_token"], ctx_len=d["ctx_len"])
        n = int(tree["n_nodes"][0])
        assert n == case["B"] + 1
        assert list(tree["tok"][0, :n]) == case["tok"]
        assert list(tree["parent"][0, :n]) == case["parent"]
        assert list(tree["depth"][0, :n]) == case["depth"]
        np.testing.assert_allclose(tree["surrogate"][0], case["surrogate"], atol=2e-6)
