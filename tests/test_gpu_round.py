"""A whole verification round on the GPU (the four C-ABI calls chained, each
consuming the previous call's device outputs) against the oracle's round
computed on the CPU from the same seeded inputs.

The GPU's lse is fp32, the oracle's fp64, so tree membership can differ only
where a selected and an unselected prefix at different depths score within
the margin; the oracle reports that gap.  Above the margin the compiled tree,
the masks, the accepted prefix and the bonus token must be bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api, synth

from helpers import TREE_MARGIN, assert_attn_close, bf16_tensor, i32, logits_tensor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_round(name):
    w = synth.WORKLOADS[name]
    z = synth.draft_logits(w)
    root = synth.root_tokens(w)
    a = synth.attention_inputs(w)
    ctx = a["ctx_len"]
    # oracle round
    ids, zk, logp, lse = oracle.topk(z, w.k, w.inv_temperature)
    tree = oracle.build_tree(ids, zk, lse, w.budget_per_seq(), w.inv_temperature, root_token=root,
                             ctx_len=ctx, k_per_seq=w.k_per_seq(), n_max=w.n_max)
    tgt = synth.target_logits(w, tree["tok"], tree["parent"], tree["depth"], tree["n_nodes"])
    walk = oracle.tree_walk(tgt, tree["tok"], tree["parent"], tree["depth"], tree["n_nodes"], w.L)
    # GPU round
    g_ids, g_zk, _, g_lse = api.topk(logits_tensor(z), w.k, w.inv_temperature)
    g_tree = api.build_tree(g_ids, g_zk, g_lse, w.B, i32(root), w.inv_temperature,
                            k_per_seq=i32(w.k_per_seq()), budget=i32(w.budget_per_seq()),
                            ctx_len=i32(ctx))
    pt = i32(a["page_table"]) if "page_table" in a else None
    out = api.tree_attn(bf16_tensor(a["q"]), bf16_tensor(a["k_cache"]), bf16_tensor(a["v_cache"]),
                        bf16_tensor(a["k_tree"]), bf16_tensor(a["v_tree"]), g_tree["mask"],
                        g_tree["n_nodes"], i32(ctx), int(ctx.max()), page_table=pt)
    g_walk = api.tree_walk(logits_tensor(tgt), g_tree["tok"], g_tree["parent"], g_tree["depth"],
                           g_tree["n_nodes"], w.L)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(g_ids.cpu().numpy(), ids)
    exact = tree["delta_min"] >= TREE_MARGIN
    for b in range(w.batch):
        if not exact[b]:
            continue
        for key in ("tok", "parent", "depth", "pos"):
            np.testing.assert_array_equal(g_tree[key][b].cpu().numpy(), tree[key][b])
        np.testing.assert_array_equal(g_tree["mask"][b].cpu().numpy().view(np.uint32), tree["mask"][b])
        for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
            np.testing.assert_array_equal(g_walk[key][b].cpu().numpy(), walk[key][b])
    # the cross-depth margin of the synthetic workloads is far above fp32 lse error
    assert exact.all(), "tie-ambiguous sequences: %s" % np.nonzero(~exact)[0]
    # attention of a sample of rows (all rows for the small workloads)
    g = np.random.default_rng(7)
    items = []
    for b in range(w.batch):
        n = int(tree["n_nodes"][b])
        js = np.arange(n) if n * w.hq <= 256 else np.unique(np.r_[0, n - 1, g.integers(0, n, 6)])
        hs = np.arange(w.hq) if n * w.hq <= 256 else g.integers(0, w.hq, len(js))
        for j, h in (zip(js, hs) if n * w.hq > 256 else [(j, h) for j in js for h in hs]):
            items.append((b, int(j), int(h)))
        if len(items) > 400:
            break
    items = np.array(items, np.int32)
    ref, _ = oracle.tree_attn(items, a["q"], a["k_cache"], a["v_cache"], ctx, a["k_tree"],
                              a["v_tree"], tree["mask"], tree["n_nodes"], 1.0 / np.sqrt(w.d),
                              page_table=a.get("page_table"), page_size=a.get("page_size", 64))
    got = out.float().cpu().numpy()[items[:, 0], items[:, 1], items[:, 2]]
    assert_attn_close(got, ref, name)
