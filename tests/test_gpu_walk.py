"""Parity of ddt_tree_walk (CUDA, through the C ABI) with the oracle's greedy
walk: accepted length, accepted rows and tokens, and the bonus token are
bit-exact, in each of the walk's modes (every row scanned, only the visited
rows, and the library's choice).  Target logits are planted on the oracle's
tree for every workload, plus ties, bf16 logits, single-row trees, walks down
to depth L and ragged vocabularies."""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api, synth

from helpers import i32, logits_tensor, oracle_tree_inputs

pytestmark = pytest.mark.gpu


def _tree(w):
    ids, zk, lse = oracle_tree_inputs(w, synth.draft_logits(w))
    return oracle.build_tree(ids, zk, lse.astype(np.float64), w.budget_per_seq(),
                             w.inv_temperature, root_token=synth.root_tokens(w),
                             k_per_seq=w.k_per_seq(), n_max=w.n_max)


MODES = (api.WALK_ALL_ROWS, api.WALK_LAZY, api.WALK_AUTO)


def _compare(logits, tree, L, modes=MODES):
    ref = oracle.tree_walk(logits, tree["tok"], tree["parent"], tree["depth"], tree["n_nodes"], L)
    t = logits_tensor(logits)
    for mode in modes:
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = api.tree_walk(t, i32(tree["tok"]), i32(tree["parent"]), i32(tree["depth"]),
                            i32(tree["n_nodes"]), L, dev_status=st, mode=mode)
        torch.cuda.synchronize()
        assert st.item() == 0
        for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
            np.testing.assert_array_equal(got[key].cpu().numpy(), ref[key],
                                          err_msg="%s (mode %d)" % (key, mode))
    return ref


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_workload_walks(name):
    w = synth.WORKLOADS[name]
    tree = _tree(w)
    logits = synth.target_logits(w, tree["tok"], tree["parent"], tree["depth"], tree["n_nodes"])
    _compare(logits, tree, w.L)


def test_bf16_logits_and_ties():
    w = synth.WORKLOADS["tiny"].scaled(batch=6, L=6, V=3000, k=4, B=40)
    tree = _tree(w)
    g = np.random.default_rng(0)
    logits = g.integers(-4, 5, size=(w.batch, w.n_max, w.V)).astype(np.float32)
    _compare(logits, tree, w.L)                         # many exact ties
    _compare(synth.to_bf16_bits(logits + 0.25), tree, w.L)


def test_single_row_and_full_depth():
    w = synth.WORKLOADS["tiny"].scaled(batch=3, L=3, V=20000, k=1, B=3)
    tree = _tree(w)
    logits = np.random.default_rng(1).standard_normal((3, 4, w.V), dtype=np.float32)
    # sequence 0: accept the whole chain, sequence 1: reject at the root
    for j in range(3):
        logits[0, j, tree["tok"][0, j + 1]] = 9.0
    logits[1, 0, :] = 0.0
    logits[1, 0, 5] = 1.0
    _compare(logits, tree, w.L)
    tree0 = {k: v.copy() for k, v in tree.items()}
    tree0["n_nodes"][:] = 1
    _compare(logits, tree0, w.L)


@pytest.mark.parametrize("V", [1, 100, 8192, 8193, 50001])
def test_ragged_vocab(V):
    w = synth.WORKLOADS["tiny"].scaled(batch=2, L=4, V=max(V, 4), k=2, B=10)
    tree = _tree(w)
    logits = np.random.default_rng(V).standard_normal((2, w.n_max, V), dtype=np.float32)
    tree = {k: v.copy() for k, v in tree.items()}
    tree["tok"] = np.where(tree["tok"] >= 0, tree["tok"] % V, -1).astype(np.int32)
    _compare(logits, tree, w.L)


def test_repeated_calls_reuse_workspace():
    w = synth.WORKLOADS["b64"]
    tree = _tree(w)
    logits = synth.target_logits(w, tree["tok"], tree["parent"], tree["depth"], tree["n_nodes"])
    for _ in range(3):
        _compare(logits, tree, w.L)


def test_deep_walks_every_mode():
    """Walks that accept down to depth L (the path-only walk's longest chain of
    dependent steps): sequence 0 drafts a single path of L tokens, the others
    full trees; the target agrees with every first child.  f32 and bf16."""
    w = synth.WORKLOADS["long512"].scaled(batch=3, V=40000)
    ids, zk, lse = oracle_tree_inputs(w, synth.draft_logits(w))
    tree = oracle.build_tree(ids, zk, lse.astype(np.float64), [w.L, w.B, w.B], w.inv_temperature,
                             root_token=synth.root_tokens(w), k_per_seq=[1, w.k, w.k],
                             n_max=w.n_max)
    g = np.random.default_rng(11)
    logits = g.standard_normal((w.batch, w.n_max, w.V), dtype=np.float32)
    for b in range(w.batch):
        n = int(tree["n_nodes"][b])
        par = tree["parent"][b][:n]
        x = 0
        while True:  # plant the first child of every row along the first-child path
            kids = np.nonzero(par == x)[0]
            if len(kids) == 0:
                break
            c = int(kids[0])
            logits[b, x, tree["tok"][b][c]] = 50.0
            x = c
    ref = _compare(logits, tree, w.L)
    assert ref["acc_len"][0] == w.L
    _compare(synth.to_bf16_bits(logits), tree, w.L)


def test_auto_mode_resolves():
    for name in synth.WORKLOADS:
        w = synth.WORKLOADS[name]
        m = api.tree_walk_resolve_mode(api.WALK_AUTO, torch.float32, w.batch, w.n_max, w.V, w.L)
        assert m in (api.WALK_ALL_ROWS, api.WALK_LAZY), (name, m)
    assert api.tree_walk_resolve_mode(api.WALK_LAZY, torch.float32, 1, 9, 100, 4) == api.WALK_LAZY
    assert api.tree_walk_resolve_mode(api.WALK_ALL_ROWS, torch.float32, 1, 9, 100, 4) == 0
    assert api.tree_walk_resolve_mode(7, torch.float32, 1, 9, 100, 4) == -1
