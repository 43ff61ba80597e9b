"""Pins of the oracle's KV commit (the step after the walk).

The round forwards the root (the previous round's bonus token) and the tree;
after the walk, the root and the accepted rows join the committed context at
positions ctx_len + depth, and ctx_len grows by acc_len + 1.  The pins:

* placement, against numpy fancy indexing of the dense cache and of the page
  pool through the page table; nothing else in the cache changes;
* capacity: a position past the cache is reported and not written;
* meaning, against the attention oracle: after the commit, attention over
  the longer context reproduces the tree attention of the last accepted row
  (the same keys, once in the tree and once in the cache).
"""
import numpy as np
import pytest

import oracle


def _bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _case(rng, batch, n_max, hkv, d, L):
    kt = rng.integers(0, 1 << 16, (batch, n_max, hkv, d), dtype=np.uint16)
    vt = rng.integers(0, 1 << 16, (batch, n_max, hkv, d), dtype=np.uint16)
    acc_len = rng.integers(0, L + 1, batch).astype(np.int32)
    acc_nodes = np.full((batch, L), -1, np.int32)
    for b in range(batch):
        rows = np.sort(rng.choice(np.arange(1, n_max), acc_len[b], replace=False))
        acc_nodes[b, :acc_len[b]] = rows
    return kt, vt, acc_len, acc_nodes


def test_dense_placement():
    rng = np.random.default_rng(1)
    batch, n_max, hkv, d, L, t_max = 5, 20, 2, 8, 6, 40
    kt, vt, acc_len, acc_nodes = _case(rng, batch, n_max, hkv, d, L)
    kc = rng.integers(0, 1 << 16, (batch, t_max, hkv, d), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, (batch, t_max, hkv, d), dtype=np.uint16)
    ctx = rng.integers(0, t_max - L - 1, batch).astype(np.int32)
    k2, v2, c2, ok = oracle.kv_commit(kt, vt, acc_len, acc_nodes, ctx, kc, vc)
    assert ok.all()
    np.testing.assert_array_equal(c2, ctx + acc_len + 1)
    for b in range(batch):
        rows = np.concatenate([[0], acc_nodes[b, :acc_len[b]]])
        pos = ctx[b] + np.arange(acc_len[b] + 1)
        np.testing.assert_array_equal(k2[b, pos], kt[b, rows])
        np.testing.assert_array_equal(v2[b, pos], vt[b, rows])
        rest = np.setdiff1d(np.arange(t_max), pos)
        np.testing.assert_array_equal(k2[b, rest], kc[b, rest])
        np.testing.assert_array_equal(v2[b, rest], vc[b, rest])


def test_paged_placement():
    rng = np.random.default_rng(2)
    batch, n_max, hkv, d, L, ps, maxp = 4, 12, 1, 16, 5, 4, 6
    kt, vt, acc_len, acc_nodes = _case(rng, batch, n_max, hkv, d, L)
    pool = batch * maxp
    table = rng.permutation(pool).astype(np.int32).reshape(batch, maxp)
    kc = rng.integers(0, 1 << 16, (pool, ps, hkv, d), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, (pool, ps, hkv, d), dtype=np.uint16)
    ctx = rng.integers(0, maxp * ps - L - 1, batch).astype(np.int32)
    k2, v2, c2, ok = oracle.kv_commit(kt, vt, acc_len, acc_nodes, ctx, kc, vc, page_table=table,
                                      page_size=ps, num_pages=pool)
    assert ok.all()
    np.testing.assert_array_equal(c2, ctx + acc_len + 1)
    touched = np.zeros((pool, ps), bool)
    for b in range(batch):
        rows = np.concatenate([[0], acc_nodes[b, :acc_len[b]]])
        pos = ctx[b] + np.arange(acc_len[b] + 1)
        pg, sl = table[b, pos // ps], pos % ps
        np.testing.assert_array_equal(k2[pg, sl], kt[b, rows])
        np.testing.assert_array_equal(v2[pg, sl], vt[b, rows])
        touched[pg, sl] = True
    np.testing.assert_array_equal(k2[~touched], kc[~touched])
    np.testing.assert_array_equal(v2[~touched], vc[~touched])


def test_capacity_is_reported():
    rng = np.random.default_rng(3)
    kt, vt, _, _ = _case(rng, 1, 8, 1, 4, 4)
    acc_len = np.array([3], np.int32)
    acc_nodes = np.array([[1, 2, 3, -1]], np.int32)
    kc = np.zeros((1, 10, 1, 4), np.uint16)
    vc = np.zeros((1, 10, 1, 4), np.uint16)
    k2, _, c2, ok = oracle.kv_commit(kt, vt, acc_len, acc_nodes, [8], kc, vc)
    assert not ok[0] and c2[0] == 12
    np.testing.assert_array_equal(k2[0, 8:10], kt[0, [0, 1]])  # what fits is written


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_commit_then_attend_equals_tree_attention(seed):
    """Row x_a (last accepted) attends to ctx[0, c) and its path {0, x_1..x_a};
    after the commit the same keys are cache positions [0, c + a]."""
    rng = np.random.default_rng(seed)
    n_max, hq, hkv, d, L, c = 9, 4, 2, 16, 4, 37
    # a tree: root 0; chain 0 -> 1 -> 3 -> 6 -> 8 plus side rows
    parent = np.array([-1, 0, 0, 1, 1, 2, 3, 3, 6], np.int32)
    path = [1, 3, 6, 8]
    a = int(rng.integers(1, L + 1))
    x = path[a - 1]
    W = 1
    mask = np.zeros((1, n_max, W), np.uint32)
    for j in range(n_max):
        m, y = 0, j
        while y >= 0:
            m |= 1 << y
            y = parent[y]
        mask[0, j, 0] = m
    t_max = c + L + 1
    q = _bits(rng.standard_normal((1, n_max, hq, d)))
    kt = _bits(rng.standard_normal((1, n_max, hkv, d)))
    vt = _bits(rng.standard_normal((1, n_max, hkv, d)))
    kc = _bits(rng.standard_normal((1, t_max, hkv, d)))
    vc = _bits(rng.standard_normal((1, t_max, hkv, d)))
    items = [(0, x, h) for h in range(hq)]
    o1, l1 = oracle.tree_attn(items, q, kc, vc, np.array([c], np.int32), kt, vt, mask,
                              np.array([n_max], np.int32), 0.25)
    acc_nodes = np.array([path[:a] + [-1] * (L - a)], np.int32)
    k2, v2, c2, ok = oracle.kv_commit(kt, vt, [a], acc_nodes, [c], kc, vc)
    assert ok[0] and c2[0] == c + a + 1
    # the committed row of x (position c + a) plays the one-row tree; the
    # context ends just before it
    q1 = np.ascontiguousarray(q[:, [x]])
    kt1 = np.ascontiguousarray(k2[:, [c + a]])
    vt1 = np.ascontiguousarray(v2[:, [c + a]])
    o2, l2 = oracle.tree_attn([(0, 0, h) for h in range(hq)], q1, k2, v2,
                              np.array([c + a], np.int32), kt1, vt1,
                              np.ones((1, 1, 1), np.uint32), np.array([1], np.int32), 0.25)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)
