"""Parity of ddt_tree_walk (CUDA, through the C ABI) with the oracle's greedy
walk: accepted length, accepted rows and tokens, and the bonus token are
bit-exact.  Target logits are planted on the oracle's tree for every
workload, plus ties, bf16 logits, single-row trees and ragged vocabularies."""
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


def _compare(logits, tree, L):
    ref = oracle.tree_walk(logits, tree["tok"], tree["parent"], tree["depth"], tree["n_nodes"], L)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = api.tree_walk(logits_tensor(logits), i32(tree["tok"]), i32(tree["parent"]),
                        i32(tree["depth"]), i32(tree["n_nodes"]), L, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
        np.testing.assert_array_equal(got[key].cpu().numpy(), ref[key], err_msg=key)
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
