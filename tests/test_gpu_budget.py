"""Parity of ddt_plan_budget (CUDA, through the C ABI) with the oracle's
node-budget plan: every sequence's share of the batch's nodes, bit for bit,
and its expected tokens to fp64 summation order.

Both sides rank the same fp64 scores (same formula, same summation order)
by the same total order, so the ranking is identical; the prefix sums of
probabilities are summed in different orders, so under the cost model the
chosen total may only differ where two totals give rates within 1e-12 of
each other (the test then checks that the two rates are that close)."""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api, synth

from helpers import f32_up, i32

pytestmark = pytest.mark.gpu


def _inputs(seed, batch, L, V, k, B, scale=1.5):
    g = np.random.default_rng(seed)
    z = (g.standard_normal((batch, L, V)) * scale).astype(np.float32)
    for b in range(batch):
        z[b] *= 0.4 + 0.3 * (b % 5)
    ids, zk, logp, lse = oracle.topk(z, k, 1.0)
    lse = f32_up(lse)
    tree = oracle.build_tree(ids, zk, lse.astype(np.float64), B, 1.0, n_max=B + 1)
    return ids, zk, lse, tree


def _rate(ids, zk, lse, tree, L, n, c0, c1):
    _, e, _ = oracle.plan_budget(ids, zk, lse.astype(np.float64), tree, L, 1.0, total_budget=n)
    return e.sum() / (c0 + c1 * n)


def _compare(ids, zk, lse, tree, L, total=-1, c0=0.0, c1=0.0):
    ref_b, ref_e, ref_n = oracle.plan_budget(ids, zk, lse.astype(np.float64), tree, L, 1.0,
                                             total_budget=total, cost_fixed=c0, cost_per_node=c1)
    t = {k_: i32(tree[k_]) for k_ in ("tok", "parent", "depth", "n_nodes")}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gb, ge = api.plan_budget(t, i32(ids), torch.from_numpy(zk.astype(np.float32)).cuda(),
                             torch.from_numpy(lse.astype(np.float32)).cuda(), 1.0, total, c0, c1,
                             dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    gb, ge = gb.cpu().numpy(), ge.cpu().numpy()
    if int(gb.sum()) != ref_n:  # only a near-tie of the rate may move the total
        assert c1 > 0
        r_gpu = _rate(ids, zk, lse, tree, L, int(gb.sum()), c0, c1)
        r_ref = _rate(ids, zk, lse, tree, L, ref_n, c0, c1)
        assert abs(r_gpu - r_ref) <= 1e-12 * r_ref
        return gb, ge
    np.testing.assert_array_equal(gb, ref_b)
    np.testing.assert_allclose(ge, ref_e, rtol=1e-12)
    return gb, ge


@pytest.mark.parametrize("seed,batch,L,V,k,B", [(1, 3, 4, 500, 4, 20), (2, 8, 16, 3000, 8, 64),
                                                (3, 5, 6, 200, 3, 30), (4, 1, 8, 1000, 6, 100)])
def test_random_batches(seed, batch, L, V, k, B):
    ids, zk, lse, tree = _inputs(seed, batch, L, V, k, B)
    total = int((tree["n_nodes"] - 1).sum())
    _compare(ids, zk, lse, tree, L)                              # every node
    for cap in (0, 1, total // 3, total - 1):
        _compare(ids, zk, lse, tree, L, total=cap)              # a shared cap
    for c0, c1 in ((20.0, 1.0), (5.0, 0.05), (100.0, 3.0)):
        _compare(ids, zk, lse, tree, L, c0=c0, c1=c1)           # the cost model


@pytest.mark.parametrize("name", ["b256", "paged128", "long512"])
def test_workloads(name):
    w = synth.WORKLOADS[name]
    z = synth.draft_logits(w)
    ids, zk, logp, lse = oracle.topk(z, w.k, w.inv_temperature)
    lse = f32_up(lse)
    tree = oracle.build_tree(ids, zk, lse.astype(np.float64), w.budget_per_seq(),
                             w.inv_temperature, k_per_seq=w.k_per_seq(), n_max=w.n_max)
    ref = oracle.plan_budget(ids, zk, lse.astype(np.float64), tree, w.L, w.inv_temperature,
                             total_budget=w.batch * w.B // 2)
    t = {k_: i32(tree[k_]) for k_ in ("tok", "parent", "depth", "n_nodes")}
    gb, ge = api.plan_budget(t, i32(ids), torch.from_numpy(zk.astype(np.float32)).cuda(),
                             torch.from_numpy(lse).cuda(), w.inv_temperature,
                             w.batch * w.B // 2)
    np.testing.assert_array_equal(gb.cpu().numpy(), ref[0])
    np.testing.assert_allclose(ge.cpu().numpy(), ref[1], rtol=1e-12)


def test_budgets_rebuild_the_surrogate():
    """Feeding the plan to the tree builder: each sequence's rebuilt tree has
    the planned node count and a surrogate of expected_tokens - 1."""
    ids, zk, lse, tree = _inputs(9, 6, 8, 2000, 6, 48)
    t = {k_: i32(tree[k_]) for k_ in ("tok", "parent", "depth", "n_nodes")}
    g_ids, g_zk, g_lse = i32(ids), torch.from_numpy(zk.astype(np.float32)).cuda(), \
        torch.from_numpy(lse).cuda()
    budget, exp_tok = api.plan_budget(t, g_ids, g_zk, g_lse, 1.0, total_budget=100)
    rebuilt = api.build_tree(g_ids, g_zk, g_lse, 48, i32(np.arange(6) + 1), 1.0, budget=budget)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(rebuilt["n_nodes"].cpu().numpy(), budget.cpu().numpy() + 1)
    np.testing.assert_allclose(rebuilt["surrogate"].cpu().numpy(), exp_tok.cpu().numpy() - 1,
                               rtol=1e-12)
