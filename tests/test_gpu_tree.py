"""Parity of ddt_build_tree (CUDA, through the C ABI) with the oracle's
steps 2-3.

Both sides receive the same candidates (the oracle's top-k, lse rounded to
f32) and so compute identical fp64 keys: the compiled tree (tokens, parents,
depths, positions, masks, node count) must match bit for bit and the
surrogate to fp64 summation-order error."""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api, synth

from helpers import f32_up, i32, oracle_tree_inputs

pytestmark = pytest.mark.gpu


def _run(ids, zk, lse, B_max, inv_t, k_per_seq=None, budget=None, root=None, ctx=None):
    b = ids.shape[0]
    root = np.arange(b, dtype=np.int32) + 3 if root is None else root
    ctx = np.full(b, 100, np.int32) if ctx is None else ctx
    kref = None if k_per_seq is None else k_per_seq
    bref = B_max if budget is None else budget
    ref = oracle.build_tree(ids, zk, lse.astype(np.float64), bref, inv_t, root_token=root,
                            ctx_len=ctx, k_per_seq=kref, n_max=B_max + 1)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = api.build_tree(i32(ids), torch.from_numpy(zk.astype(np.float32)).cuda(),
                         torch.from_numpy(lse.astype(np.float32)).cuda(), B_max, i32(root),
                         inv_t, k_per_seq=None if k_per_seq is None else i32(k_per_seq),
                         budget=None if budget is None else i32(budget), ctx_len=i32(ctx),
                         dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    for key in ("tok", "parent", "depth", "pos", "n_nodes"):
        np.testing.assert_array_equal(got[key].cpu().numpy(), ref[key], err_msg=key)
    np.testing.assert_array_equal(got["mask"].cpu().numpy().view(np.uint32), ref["mask"])
    np.testing.assert_allclose(got["surrogate"].cpu().numpy(), ref["surrogate"], rtol=1e-12)
    return got, ref


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_workload_trees(name):
    w = synth.WORKLOADS[name]
    ids, zk, lse = oracle_tree_inputs(w, synth.draft_logits(w))
    _run(ids, zk, lse, w.B, w.inv_temperature, k_per_seq=w.k_per_seq(),
         budget=w.budget_per_seq(), root=synth.root_tokens(w), ctx=synth.context_lengths(w))


def _random_inputs(seed, b, L, V, k, ties=False, inv_t=1.0):
    g = np.random.default_rng(seed)
    if ties:
        z = g.integers(-2, 3, size=(b, L, V)).astype(np.float32)
    else:
        z = g.standard_normal((b, L, V), dtype=np.float32) * 2
    ids, zk, logp, lse = oracle.topk(z, k, inv_t)
    return ids, zk, f32_up(lse)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("ties", [False, True])
def test_random_small(seed, ties):
    g = np.random.default_rng(seed)
    L = int(g.integers(1, 7))
    k = int(g.integers(1, 6))
    inv_t = [1.0, 0.5, 3.0][seed % 3]
    ids, zk, lse = _random_inputs(seed, 4, L, 12, k, ties, inv_t)
    total = sum(k ** t for t in range(1, L + 1))
    for B in sorted({0, 1, 3, min(total, 20), min(total + 5, 60)}):
        _run(ids, zk, lse, B, inv_t)


def test_per_sequence_budget_and_width():
    ids, zk, lse = _random_inputs(11, 5, 8, 40, 6)
    _run(ids, zk, lse, 50, 1.0, k_per_seq=np.array([1, 6, 3, 2, 6], np.int32),
         budget=np.array([8, 50, 0, 17, 1], np.int32))


def test_largest_shapes():
    ids, zk, lse = _random_inputs(12, 2, 64, 40, 32)
    _run(ids, zk, lse, 1023, 1.0)
    ids, zk, lse = _random_inputs(13, 2, 32, 300, 16)
    _run(ids, zk, lse, 512, 1.0)


def test_all_equal_logits():
    # every candidate ties: the order falls to depth and token ids throughout
    z = np.zeros((2, 6, 50), np.float32)
    ids, zk, logp, lse = oracle.topk(z, 8, 1.0)
    for B in (5, 40, 300):
        _run(ids, zk, f32_up(lse), B, 1.0)


def test_confident_draft_chain_rounds():
    # one dominant token per position: the selection grows deep chains, one
    # node per round at first
    g = np.random.default_rng(5)
    z = g.standard_normal((2, 16, 300), dtype=np.float32)
    z[:, :, 7] += 20.0
    ids, zk, logp, lse = oracle.topk(z, 4, 1.0)
    _run(ids, zk, f32_up(lse), 64, 1.0)


def test_device_values_out_of_range_are_flagged():
    ids, zk, lse = _random_inputs(14, 2, 4, 20, 4)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.build_tree(i32(ids), torch.from_numpy(zk.astype(np.float32)).cuda(),
                   torch.from_numpy(lse).cuda(), 10, i32([1, 2]), 1.0,
                   budget=i32([5, 99]), dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 1


@pytest.mark.parametrize("L,k,B", [(16, 8, 256), (16, 8, 200), (16, 4, 384), (32, 8, 160),
                                   (8, 16, 256)])
def test_shared_memory_between_static_and_opt_in(L, k, B):
    """Shapes whose dynamic shared memory fits in 48 KB only without the
    builder's static scratch: the launch must still opt in."""
    ids, zk, lse = _random_inputs(L * 100 + k + B, 2, L, 400, k)
    _run(ids, zk, lse, B, 1.0)


def _extreme_inputs(seed, b, L, V, k, small):
    """f32 drafts whose candidates mix magnitudes: 3.0 and 2.5 beside 0, -0
    and +-`small` (the eight largest logits of every row)."""
    g = np.random.default_rng(seed)
    z = np.full((b, L, V), -50.0, np.float32)
    for bb in range(b):
        for i in range(L):
            picks = g.choice(V, 8, replace=False)
            vals = np.array([3.0, small, 0.0, -0.0, small / 2, -small / 2, -small, 2.5], np.float32)
            z[bb, i, picks] = vals
    ids, zk, logp, lse = oracle.topk(z, k, 1.0)
    return ids, zk, f32_up(lse)


def _run_or_flag(ids, zk, lse, B_max):
    """The GPU tree equals the oracle's, or the builder flags the input as
    outside what it supports (DDT_ERR_UNSUPPORTED in the status word)."""
    b = ids.shape[0]
    root = np.arange(b, dtype=np.int32) + 3
    ctx = np.full(b, 100, np.int32)
    ref = oracle.build_tree(ids, zk, lse.astype(np.float64), B_max, 1.0, root_token=root,
                            ctx_len=ctx, n_max=B_max + 1)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = api.build_tree(i32(ids), torch.from_numpy(zk.astype(np.float32)).cuda(),
                         torch.from_numpy(lse.astype(np.float32)).cuda(), B_max, i32(root), 1.0,
                         ctx_len=i32(ctx), dev_status=st)
    torch.cuda.synchronize()
    if st.item() == 2:
        return "flagged"
    assert st.item() == 0
    for key in ("tok", "parent", "depth", "pos", "n_nodes"):
        np.testing.assert_array_equal(got[key].cpu().numpy(), ref[key], err_msg=key)
    np.testing.assert_array_equal(got["mask"].cpu().numpy().view(np.uint32), ref["mask"])
    return "exact"


def test_candidates_of_mixed_magnitude():
    """The builder takes siblings in candidate order, which is the order K as
    long as path sums of logits are exact in fp64.  Zeros (of either sign)
    keep them exact and must give the oracle's tree; candidates 2^-20 beside
    3.0 (sums that still fit) must too; subnormals or 1e-30 beside 3.0 can
    round a path sum, and the builder must then flag the input."""
    L, V, k, B = 6, 64, 8, 40
    assert _run_or_flag(*_extreme_inputs(1, 4, L, V, k, small=0.0), B) == "exact"
    assert _run_or_flag(*_extreme_inputs(2, 4, L, V, k, small=2.0 ** -20), B) == "exact"
    assert _run_or_flag(*_extreme_inputs(3, 4, L, V, k, small=1e-30), B) == "flagged"
    assert _run_or_flag(*_extreme_inputs(4, 4, L, V, k, small=2e-42), B) == "flagged"  # subnormal
