"""Parity of ddt_kv_commit (CUDA, through the C ABI) with the oracle's
commit: the whole cache and ctx_len are bit-exact, dense and paged, at the
workloads' head shapes, including a commit that runs out of cache (reported
in dev_status) and one fed by a full round on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api, synth

from helpers import bf16_tensor, i32

pytestmark = pytest.mark.gpu


def _case(rng, batch, n_max, hkv, d, L):
    kt = rng.integers(0, 1 << 16, (batch, n_max, hkv, d), dtype=np.uint16)
    vt = rng.integers(0, 1 << 16, (batch, n_max, hkv, d), dtype=np.uint16)
    acc_len = rng.integers(0, L + 1, batch).astype(np.int32)
    acc_nodes = np.full((batch, L), -1, np.int32)
    for b in range(batch):
        rows = np.sort(rng.choice(np.arange(1, n_max), acc_len[b], replace=False))
        acc_nodes[b, :acc_len[b]] = rows
    return kt, vt, acc_len, acc_nodes


def _run(kt, vt, acc_len, acc_nodes, ctx, kc, vc, table=None, ps=64):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    k = bf16_tensor(kc)
    v = bf16_tensor(vc)
    cl = i32(ctx)
    api.kv_commit(bf16_tensor(kt), bf16_tensor(vt), i32(acc_len), i32(acc_nodes), cl, k, v,
                  page_table=None if table is None else i32(table), page_size=ps, dev_status=st)
    torch.cuda.synchronize()
    bits = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    return bits(k), bits(v), cl.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("name", ["b64", "b256", "long512"])
def test_dense(name):
    w = synth.WORKLOADS[name]
    rng = np.random.default_rng(w.index)
    batch, t_max = min(w.batch, 4), 256
    kt, vt, acc_len, acc_nodes = _case(rng, batch, w.n_max, w.hkv, w.d, w.L)
    kc = rng.integers(0, 1 << 16, (batch, t_max, w.hkv, w.d), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, (batch, t_max, w.hkv, w.d), dtype=np.uint16)
    ctx = rng.integers(0, t_max - w.L - 1, batch).astype(np.int32)
    k2, v2, c2, ok = oracle.kv_commit(kt, vt, acc_len, acc_nodes, ctx, kc, vc)
    gk, gv, gc, st = _run(kt, vt, acc_len, acc_nodes, ctx, kc, vc)
    assert ok.all() and st == 0
    np.testing.assert_array_equal(gc, c2)
    np.testing.assert_array_equal(gk, k2)
    np.testing.assert_array_equal(gv, v2)


def test_paged():
    w = synth.WORKLOADS["paged128"]
    rng = np.random.default_rng(7)
    batch, ps, maxp = 16, w.page_size, 5
    kt, vt, acc_len, acc_nodes = _case(rng, batch, w.n_max, w.hkv, w.d, w.L)
    pool = batch * maxp
    table = rng.permutation(pool).astype(np.int32).reshape(batch, maxp)
    kc = rng.integers(0, 1 << 16, (pool, ps, w.hkv, w.d), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, (pool, ps, w.hkv, w.d), dtype=np.uint16)
    ctx = rng.integers(0, maxp * ps - w.L - 1, batch).astype(np.int32)
    ctx[0] = ps - 3  # the committed rows cross a page boundary
    k2, v2, c2, ok = oracle.kv_commit(kt, vt, acc_len, acc_nodes, ctx, kc, vc, page_table=table,
                                      page_size=ps, num_pages=pool)
    gk, gv, gc, st = _run(kt, vt, acc_len, acc_nodes, ctx, kc, vc, table, ps)
    assert ok.all() and st == 0
    np.testing.assert_array_equal(gc, c2)
    np.testing.assert_array_equal(gk, k2)
    np.testing.assert_array_equal(gv, v2)


def test_out_of_cache_is_reported():
    rng = np.random.default_rng(9)
    kt, vt, _, _ = _case(rng, 2, 10, 2, 64, 4)
    acc_len = np.array([4, 1], np.int32)
    acc_nodes = np.array([[1, 3, 5, 7], [2, -1, -1, -1]], np.int32)
    kc = rng.integers(0, 1 << 16, (2, 12, 2, 64), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, (2, 12, 2, 64), dtype=np.uint16)
    ctx = np.array([9, 0], np.int32)  # sequence 0 fits 3 of its 5 rows
    k2, v2, c2, ok = oracle.kv_commit(kt, vt, acc_len, acc_nodes, ctx, kc, vc)
    gk, gv, gc, st = _run(kt, vt, acc_len, acc_nodes, ctx, kc, vc)
    assert not ok[0] and ok[1] and st == 1
    np.testing.assert_array_equal(gc, c2)
    np.testing.assert_array_equal(gk, k2)
    np.testing.assert_array_equal(gv, v2)


def test_after_a_round_on_the_gpu():
    """The commit consumes the GPU walk's outputs directly."""
    w = synth.WORKLOADS["b64"]
    rng = np.random.default_rng(11)
    n_max, L = w.n_max, w.L
    kt = rng.integers(0, 1 << 16, (1, n_max, w.hkv, w.d), dtype=np.uint16)
    vt = rng.integers(0, 1 << 16, (1, n_max, w.hkv, w.d), dtype=np.uint16)
    # a chain tree walked by a target that agrees on the first 5 tokens
    tok = np.full((1, n_max), -1, np.int32)
    par = np.full((1, n_max), -1, np.int32)
    dep = np.zeros((1, n_max), np.int32)
    n = L + 1
    tok[0, :n] = np.arange(n) + 10
    par[0, 1:n] = np.arange(n - 1)
    dep[0, :n] = np.arange(n)
    logits = rng.standard_normal((1, n_max, 500)).astype(np.float32)
    for j in range(5):
        logits[0, j, tok[0, j + 1]] = 50.0
    walk = api.tree_walk(torch.from_numpy(logits).cuda(), i32(tok), i32(par), i32(dep),
                         i32([n]), L)
    t_max = 64
    kc = rng.integers(0, 1 << 16, (1, t_max, w.hkv, w.d), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, (1, t_max, w.hkv, w.d), dtype=np.uint16)
    k = bf16_tensor(kc)
    v = bf16_tensor(vc)
    cl = i32([20])
    api.kv_commit(bf16_tensor(kt), bf16_tensor(vt), walk["acc_len"], walk["acc_nodes"], cl, k, v)
    torch.cuda.synchronize()
    a = int(walk["acc_len"].item())
    assert a == 5
    k2, v2, c2, ok = oracle.kv_commit(kt, vt, [a], walk["acc_nodes"].cpu().numpy(), [20], kc, vc)
    assert ok[0] and int(cl.item()) == c2[0] == 26
    np.testing.assert_array_equal(k.view(torch.int16).cpu().numpy().view(np.uint16), k2)
    np.testing.assert_array_equal(v.view(torch.int16).cpu().numpy().view(np.uint16), v2)
