"""Pins for the oracle's tree attention (step 3) and greedy walk (step 4).

DDTree page: 核心創新 third bullet (ancestor-only mask, one target pass,
lossless), 運作流程 steps 3-4.  Pins:

* a single-path tree is causal attention over context + block: the library
  routine ``torch.nn.functional.scaled_dot_product_attention`` in fp64;
* a root-only tree is plain decode attention (same library routine);
* a paged cache gives the same result as the dense cache it was cut from;
* rows that are not ancestors do not influence a row;
* losslessness: with a deterministic toy target, the walk emits exactly the
  tokens that token-by-token greedy decoding emits, computed without a tree;
* the hand-worked walk in tests/golden/tree_b5.json;
* a hand-worked tree attention (tests/golden/attn_hand_tree.json): every
  row and head of a four-row tree, as sums of powers of e.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from block_draft_tree_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(bits):
    return torch.tensor(synth.bf16_bits_to_f32(bits).astype(np.float64))


def _chain_tree(L, n_max, root=0):
    n = L + 1
    tok = np.full((1, n_max), -1, np.int32)
    par = np.full((1, n_max), -1, np.int32)
    dep = np.full((1, n_max), -1, np.int32)
    tok[0, :n] = np.arange(n) + root
    par[0, 1:n] = np.arange(L)
    dep[0, :n] = np.arange(n)
    W = (n_max + 31) // 32
    mask = np.zeros((1, n_max, W), np.uint32)
    for j in range(n):
        for a in range(j + 1):
            mask[0, j, a // 32] |= np.uint32(1 << (a % 32))
    return tok, par, dep, mask, np.array([n], np.int32)


def _attn_inputs(T, n_max, hq, hkv, d, seed):
    g = np.random.default_rng(seed)
    mk = lambda *s: synth.to_bf16_bits(g.standard_normal(s, dtype=np.float32))
    return mk(1, n_max, hq, d), mk(1, T, hkv, d), mk(1, T, hkv, d), mk(1, n_max, hkv, d), mk(1, n_max, hkv, d)


@pytest.mark.parametrize("T,L,hq,hkv,d", [(50, 6, 4, 1, 64), (130, 9, 8, 2, 128), (0, 4, 2, 2, 32)])
def test_chain_is_causal_attention(T, L, hq, hkv, d):
    n_max = L + 3
    q, kc, vc, kt, vt = _attn_inputs(T, n_max, hq, hkv, d, T + L)
    tok, par, dep, mask, nn = _chain_tree(L, n_max)
    n = L + 1
    items = [(0, j, h) for j in range(n) for h in range(hq)]
    scale = 1.0 / np.sqrt(d)
    out, lse = oracle.tree_attn(items, q, kc, vc, np.array([T], np.int32), kt, vt, mask, nn, scale)
    g = hq // hkv
    K = torch.cat([_f64(kc[0]), _f64(kt[0, :n])], 0).permute(1, 0, 2).repeat_interleave(g, 0)
    Vv = torch.cat([_f64(vc[0]), _f64(vt[0, :n])], 0).permute(1, 0, 2).repeat_interleave(g, 0)
    Q = _f64(q[0, :n]).permute(1, 0, 2)
    allow = torch.ones(n, T + n, dtype=torch.bool)
    allow[:, T:] = torch.tril(torch.ones(n, n, dtype=torch.bool))
    ref = F.scaled_dot_product_attention(Q, K, Vv, attn_mask=allow, scale=scale)  # [hq, n, d]
    got = torch.tensor(out).reshape(n, hq, d).permute(1, 0, 2)
    torch.testing.assert_close(got, ref, rtol=1e-12, atol=1e-12)
    s = (Q @ K.transpose(1, 2)) * scale
    s = s.masked_fill(~allow, float("-inf"))
    ref_lse = torch.logsumexp(s, -1)
    torch.testing.assert_close(torch.tensor(lse).reshape(n, hq).T, ref_lse, rtol=1e-12, atol=1e-12)


def test_root_only_is_decode_attention():
    T, hq, hkv, d = 77, 6, 3, 64
    q, kc, vc, kt, vt = _attn_inputs(T, 4, hq, hkv, d, 5)
    tok, par, dep, mask, nn = _chain_tree(0, 4)
    out, _ = oracle.tree_attn([(0, 0, h) for h in range(hq)], q, kc, vc, np.array([T], np.int32),
                              kt, vt, mask, nn, 0.125)
    g = hq // hkv
    K = torch.cat([_f64(kc[0]), _f64(kt[0, :1])], 0).permute(1, 0, 2).repeat_interleave(g, 0)
    Vv = torch.cat([_f64(vc[0]), _f64(vt[0, :1])], 0).permute(1, 0, 2).repeat_interleave(g, 0)
    Q = _f64(q[0, :1]).permute(1, 0, 2)
    ref = F.scaled_dot_product_attention(Q, K, Vv, scale=0.125)[:, 0]
    torch.testing.assert_close(torch.tensor(out), ref, rtol=1e-12, atol=1e-12)


def test_paged_equals_dense():
    w = synth.WORKLOADS["paged128"].scaled(batch=3, B=10, ctx=300, ctx_min=65, hq=4, hkv=2, d=32)
    a = synth.attention_inputs(w)
    T = a["ctx_len"]
    ps = a["page_size"]
    dense_k = np.zeros((3, int(T.max()), 2, 32), np.uint16)
    dense_v = np.zeros_like(dense_k)
    for b in range(3):
        for t in range(T[b]):
            p = a["page_table"][b, t // ps]
            dense_k[b, t] = a["k_cache"][p, t % ps]
            dense_v[b, t] = a["v_cache"][p, t % ps]
    n_max = w.n_max
    W = (n_max + 31) // 32
    g = np.random.default_rng(0)
    mask = g.integers(0, 2**32, size=(3, n_max, W), dtype=np.uint64).astype(np.uint32)
    nn = np.array([n_max, 5, 1], np.int32)
    items = [(b, j, h) for b in range(3) for j in range(nn[b]) for h in range(4)]
    o1, l1 = oracle.tree_attn(items, a["q"], a["k_cache"], a["v_cache"], T, a["k_tree"],
                              a["v_tree"], mask, nn, 0.2, page_table=a["page_table"], page_size=ps)
    o2, l2 = oracle.tree_attn(items, a["q"], dense_k, dense_v, T, a["k_tree"], a["v_tree"], mask,
                              nn, 0.2)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_non_ancestors_do_not_leak():
    T, L, hq, hkv, d = 20, 5, 2, 1, 16
    q, kc, vc, kt, vt = _attn_inputs(T, 8, hq, hkv, d, 9)
    # root with two branches: rows 1,2 under 0; row 3 under 1; row 4 under 2
    n = 5
    par = [-1, 0, 0, 1, 2]
    mask = np.zeros((1, 8, 1), np.uint32)
    for j in range(n):
        x = j
        while x >= 0:
            mask[0, j, 0] |= np.uint32(1 << x)
            x = par[x]
    nn = np.array([n], np.int32)
    items = [(0, 3, 0), (0, 3, 1)]
    o1, _ = oracle.tree_attn(items, q, kc, vc, np.array([T], np.int32), kt, vt, mask, nn, 0.25)
    kt2, vt2 = kt.copy(), vt.copy()
    kt2[0, 2] ^= np.uint16(0x1234)
    vt2[0, 4] ^= np.uint16(0x0F0F)
    o2, _ = oracle.tree_attn(items, q, kc, vc, np.array([T], np.int32), kt2, vt2, mask, nn, 0.25)
    np.testing.assert_array_equal(o1, o2)
    kt2 = kt.copy()
    kt2[0, 1] ^= np.uint16(0x1234)  # an ancestor of row 3: must matter
    o3, _ = oracle.tree_attn(items, q, kc, vc, np.array([T], np.int32), kt2, vt, mask, nn, 0.25)
    assert not np.array_equal(o1, o3)


def _toy_target(history, V):
    h = 1469598103934665603
    for t in history:
        h = ((h ^ (int(t) + 1)) * 1099511628211) & 0xFFFFFFFFFFFFFFFF
    return h % V


@pytest.mark.parametrize("seed", range(8))
def test_walk_is_lossless(seed):
    g = np.random.default_rng(seed)
    L, k, V, B = 5, 3, 7, 25
    z = g.standard_normal((1, L, V), dtype=np.float32)
    ids, zk, logp, lse = oracle.topk(z, k, 1.0)
    root = int(g.integers(0, V))
    tree = oracle.build_tree(ids, zk, lse, B, 1.0, root_token=root)
    n = int(tree["n_nodes"][0])
    ctx = tuple(int(x) for x in g.integers(0, V, size=4))
    logits = g.standard_normal((1, B + 1, V), dtype=np.float32)
    for j in range(n):
        path, x = [], j
        while x > 0:
            path.append(int(tree["tok"][0, x]))
            x = int(tree["parent"][0, x])
        hist = ctx + (root,) + tuple(reversed(path))
        logits[0, j, _toy_target(hist, V)] = 10.0
    res = oracle.tree_walk(logits, tree["tok"], tree["parent"], tree["depth"], tree["n_nodes"], L)
    a = int(res["acc_len"][0])
    emitted = list(res["acc_tok"][0, :a]) + [int(res["bonus"][0])]
    # greedy decoding one token at a time, no tree
    hist = list(ctx) + [root]
    ref = []
    for _ in range(a + 1):
        t = _toy_target(tuple(hist), V)
        ref.append(t)
        hist.append(t)
    assert emitted == ref
    # the walk stopped because the next greedy token is not in the tree (or depth L)
    paths = set()
    for j in range(1, n):
        path, x = [], j
        while x > 0:
            path.append(int(tree["tok"][0, x]))
            x = int(tree["parent"][0, x])
        paths.add(tuple(reversed(path)))
    assert a == L or tuple(ref[:a + 1]) not in paths
    assert all(res["acc_nodes"][0, a:] == -1) and all(res["acc_tok"][0, a:] == -1)


@pytest.mark.parametrize("m", [0, 1, 3, 6])
def test_chain_walk_is_longest_match(m):
    L, V = 6, 20
    n_max = L + 1
    tok, par, dep, mask, nn = _chain_tree(L, n_max, root=2)
    g = np.random.default_rng(m)
    logits = g.standard_normal((1, n_max, V), dtype=np.float32)
    for j in range(L + 1):
        nxt = int(tok[0, j + 1]) if j < L else 0
        want = nxt if j < m else (nxt + 1) % V
        logits[0, j, want] = 50.0
    res = oracle.tree_walk(logits, tok, par, dep, nn, L)
    assert res["acc_len"][0] == m
    assert list(res["acc_nodes"][0, :m]) == list(range(1, m + 1))
    expect_bonus = ((int(tok[0, m + 1]) if m < L else 0) + 1) % V
    assert res["bonus"][0] == expect_bonus


def test_walk_ties_take_lowest_id():
    tok = np.array([[5, 3, 1]], np.int32)
    par = np.array([[-1, 0, 0]], np.int32)
    dep = np.array([[0, 1, 1]], np.int32)
    logits = np.zeros((1, 3, 8), np.float32)
    logits[0, 0, [1, 3]] = 4.0  # tie between the two children's tokens
    res = oracle.tree_walk(logits, tok, par, dep, np.array([3], np.int32), 1)
    assert res["acc_len"][0] == 1 and res["acc_nodes"][0, 0] == 2 and res["bonus"][0] == 0


def test_golden_walk():
    d = json.load(open(os.path.join(GOLDEN, "tree_b5.json")))
    case = [c for c in d["cases"] if c["B"] == d["walk"]["B"]][0]
    n = len(case["tok"])
    V = d["V"]
    logits = np.zeros((1, n, V), np.float32)
    for j, t in enumerate(d["walk"]["argmax_per_row"]):
        logits[0, j, t] = 1.0
    res = oracle.tree_walk(logits, np.array([case["tok"]], np.int32),
                           np.array([case["parent"]], np.int32),
                           np.array([case["depth"]], np.int32), np.array([n], np.int32), d["L"])
    w = d["walk"]
    assert res["acc_len"][0] == w["acc_len"]
    assert list(res["acc_nodes"][0, :w["acc_len"]]) == w["acc_nodes"]
    assert list(res["acc_tok"][0, :w["acc_len"]]) == w["acc_tok"]
    assert res["bonus"][0] == w["bonus"]


def test_attention_golden_hand_tree():
    """tests/golden/attn_hand_tree.json: every row and head of a four-row
    tree over a two-token context, worked out by hand (sums of powers of e;
    the derivation is in the file), including siblings that must not see
    each other and a grouped-query pair of heads."""
    d = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "attn_hand_tree.json")))
    D, n, T = d["d"], len(d["parent"]), d["ctx_len"]

    def bits(rows, shape):
        a = np.zeros(shape, np.float32)
        a.reshape(-1, D)[:len(rows), :2] = np.asarray(rows, np.float32)
        return (a.view(np.uint32) >> 16).astype(np.uint16)

    q = np.zeros((1, n, 2, D), np.float32)
    for h, qh in enumerate(d["q_heads"]):
        q[0, :, h, :2] = qh
    q = (q.view(np.uint32) >> 16).astype(np.uint16)
    kc, vc = bits(d["k_ctx"], (1, T, 1, D)), bits(d["v_ctx"], (1, T, 1, D))
    kt, vt = bits(d["k_tree"], (1, n, 1, D)), bits(d["v_tree"], (1, n, 1, D))
    mask = np.asarray(d["mask"], np.uint32).reshape(1, n, 1)
    items = np.array([(0, e["row"], e["head"]) for e in d["expected"]], np.int32)
    out, lse = oracle.tree_attn(items, q, kc, vc, np.array([T], np.int32), kt, vt, mask,
                                np.array([n], np.int32), d["scale"])
    for i, e in enumerate(d["expected"]):
        np.testing.assert_allclose(out[i, :2], e["out"], rtol=1e-13, atol=0, err_msg=str(e))
        assert np.all(out[i, 2:] == 0.0)
        assert lse[i] == pytest.approx(e["lse"], rel=1e-13)
