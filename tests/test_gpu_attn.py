"""Parity of ddt_tree_attn (CUDA, through the C ABI) with the oracle's fp64
masked attention.

Tolerance: bf16 output with fp32 accumulation against fp64, max-abs 2e-2 and
max-abs / max|ref| <= 1e-2 per case.  Small workloads compare every row; the
large ones compare a seeded sample of (sequence, row, head) items, always
including the root, the deepest rows and the last sequence."""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api, synth

from helpers import assert_attn_close, bf16_tensor, i32, oracle_tree_inputs

pytestmark = pytest.mark.gpu


def _tree_for(w):
    ids, zk, lse = oracle_tree_inputs(w, synth.draft_logits(w))
    return oracle.build_tree(ids, zk, lse.astype(np.float64), w.budget_per_seq(),
                             w.inv_temperature, root_token=synth.root_tokens(w),
                             ctx_len=synth.context_lengths(w), k_per_seq=w.k_per_seq(),
                             n_max=w.n_max)


def _gpu_attn(a, tree, w, want_lse=True):
    kc = bf16_tensor(a["k_cache"])
    vc = bf16_tensor(a["v_cache"])
    pt = i32(a["page_table"]) if "page_table" in a else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = api.tree_attn(bf16_tensor(a["q"]), kc, vc, bf16_tensor(a["k_tree"]),
                             bf16_tensor(a["v_tree"]),
                             torch.from_numpy(tree["mask"].view(np.int32)).cuda(),
                             i32(tree["n_nodes"]), i32(a["ctx_len"]), int(a["ctx_len"].max()),
                             page_table=pt, want_lse=True, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _oracle_attn(a, tree, w, items):
    return oracle.tree_attn(items, a["q"], a["k_cache"], a["v_cache"], a["ctx_len"], a["k_tree"],
                            a["v_tree"], tree["mask"], tree["n_nodes"], 1.0 / np.sqrt(w.d),
                            page_table=a.get("page_table"), page_size=a.get("page_size", 64))


def _items(w, tree, sample, seed):
    all_items = [(b, j, h) for b in range(w.batch) for j in range(int(tree["n_nodes"][b]))
                 for h in range(w.hq)]
    if sample is None or sample >= len(all_items):
        return np.array(all_items, np.int32)
    g = np.random.default_rng(seed)
    pick = set(map(tuple, np.array(all_items)[g.choice(len(all_items), sample, replace=False)]))
    for b in (0, w.batch - 1):
        n = int(tree["n_nodes"][b])
        pick |= {(b, 0, 0), (b, n - 1, w.hq - 1)}
    return np.array(sorted(pick), np.int32)


def _check(w, sample=None, seed=0):
    tree = _tree_for(w)
    a = synth.attention_inputs(w)
    out, lse = _gpu_attn(a, tree, w)
    items = _items(w, tree, sample, seed)
    ref, ref_lse = _oracle_attn(a, tree, w, items)
    got = out[items[:, 0], items[:, 1], items[:, 2]]
    assert_attn_close(got, ref, w.name)
    np.testing.assert_allclose(lse[items[:, 0], items[:, 1], items[:, 2]], ref_lse, atol=2e-3)
    # padding rows are written as zero
    for b in range(w.batch):
        n = int(tree["n_nodes"][b])
        assert np.all(out[b, n:] == 0)
        assert np.all(np.isneginf(lse[b, n:]))


def test_tiny_all_rows():
    _check(synth.WORKLOADS["tiny"])


def test_b64_all_rows():
    _check(synth.WORKLOADS["b64"])


@pytest.mark.parametrize("name,sample", [("b256", 96), ("paged128", 96), ("long512", 40)])
def test_large_sampled(name, sample):
    _check(synth.WORKLOADS[name], sample=sample, seed=len(name))


@pytest.mark.parametrize("kw", [
    dict(ctx=0, hq=4, hkv=1, d=64),
    dict(ctx=1, hq=8, hkv=2, d=128),
    dict(ctx=63, hq=2, hkv=2, d=64),
    dict(ctx=1000, hq=16, hkv=1, d=128),
    dict(ctx=777, hq=32, hkv=8, d=128, B=40),
])
def test_small_shapes(kw):
    w = synth.WORKLOADS["tiny"].scaled(batch=2, L=5, V=50, k=3, B=kw.pop("B", 12), **kw)
    _check(w)


def test_paged_ragged_small():
    w = synth.WORKLOADS["paged128"].scaled(batch=5, L=4, V=300, k=3, B=20, ctx=700, ctx_min=1,
                                           hq=8, hkv=2, d=64)
    _check(w)
