"""The round driver (VerifyRound) with the target's other decoding rules and
the commit, on the GPU, against the oracle composed on the CPU:

* decode="sample" captured once into a CUDA graph and replayed: replay i
  draws with step i (the device step counter), so consecutive replays are
  fresh draws, each equal to the oracle's sampled walk of that step;
* decode="lm_head" with commit: the walk from hidden states and the LM head,
  then the root's and the accepted rows' K/V appended and ctx_len advanced.
The tree itself is the GPU's (its parity is pinned elsewhere); these tests
cover what the driver adds on top.
"""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import synth
from block_draft_tree_b200.round import VerifyRound

from helpers import bf16_tensor, check_sampled_walk, i32, logits_tensor

pytestmark = pytest.mark.gpu


def _inputs(w, extra_ctx=0):
    z = synth.draft_logits(w)
    a = synth.attention_inputs(w)
    x = {"draft": logits_tensor(z), "root": i32(synth.root_tokens(w)), "ctx_len": i32(a["ctx_len"]),
         "q": bf16_tensor(a["q"]), "k_tree": bf16_tensor(a["k_tree"]),
         "v_tree": bf16_tensor(a["v_tree"])}
    kc, vc = a["k_cache"], a["v_cache"]
    if extra_ctx:  # room after the context for committed rows
        pad = lambda c: np.concatenate([c, np.zeros((c.shape[0], extra_ctx) + c.shape[2:], c.dtype)], 1)
        kc, vc = pad(kc), pad(vc)
    x["k_cache"], x["v_cache"] = bf16_tensor(kc), bf16_tensor(vc)
    return x, a, kc, vc


def _round(w, **kw):
    return VerifyRound(batch=w.batch, L=w.L, V=w.V, k=w.k, B_max=w.B, hq=w.hq, hkv=w.hkv, d=w.d,
                       max_ctx=w.ctx, draft_dtype=torch.float32 if w.draft_dtype == "f32" else torch.bfloat16,
                       target_dtype=torch.float32, inv_temperature=w.inv_temperature, **kw)


def _tree(o):
    return {k: o[k].cpu().numpy() for k in ("tok", "parent", "depth", "n_nodes")}


def test_sampled_round_replays_draw_fresh_steps():
    w = synth.WORKLOADS["tiny"].scaled(batch=3, L=4, V=3000, k=4, B=12)
    x, a, _, _ = _inputs(w)
    rnd = _round(w, decode="sample", sample_inv_temperature=1.0, seed=9)
    rng = np.random.default_rng(3)
    tgt = rng.standard_normal((w.batch, w.n_max, w.V)).astype(np.float32)
    x["target"] = torch.from_numpy(tgt).cuda()
    rnd.bind(x)
    rnd.launch()  # eager warm-up: step 0
    torch.cuda.synchronize()
    tree = _tree(rnd.out)
    # make the tree's children likely under the target, then re-bind the same buffer
    for b in range(w.batch):
        n = int(tree["n_nodes"][b])
        for c in range(1, n):
            tgt[b, tree["parent"][b][c], tree["tok"][b][c]] += 9.0
    x["target"].copy_(torch.from_numpy(tgt))
    rnd.step_counter.zero_()
    g = rnd.capture()
    draws = []
    for i in range(3):
        g.replay()
        torch.cuda.synchronize()
        draws.append({k: rnd.out[k].cpu().numpy().copy() for k in ("acc_len", "acc_nodes", "acc_tok", "bonus")})
    assert int(rnd.step_counter.item()) == 3
    assert int(rnd.out["status"].item()) == 0
    for i, got in enumerate(draws):  # replay i draws the oracle's walk of step i
        check_sampled_walk(tgt, tree, w.L, 1.0, 9, i, got)
    # fresh draws: the three replays do not all agree
    assert any(not np.array_equal(draws[0][k], draws[i][k]) for i in (1, 2) for k in draws[0])


def test_lm_head_round_with_commit():
    w = synth.WORKLOADS["tiny"].scaled(batch=2, L=4, V=3000, k=4, B=12)
    x, a, kc, vc = _inputs(w, extra_ctx=w.L + 1)
    K = 128
    rng = np.random.default_rng(5)
    head = (rng.standard_normal((w.V, K)) / np.sqrt(K)).astype(np.float32)
    hid = (rng.standard_normal((w.batch, w.n_max, K)) * 0.5).astype(np.float32)
    tob = lambda v: (v.view(np.uint32) >> 16).astype(np.uint16)
    x["head"] = bf16_tensor(tob(head))
    x["hidden"] = bf16_tensor(tob(hid))
    rnd = _round(w, decode="lm_head", commit=True)
    rnd.bind(x)
    # plant: every row points at its first child, so that the walk descends
    rnd_tree = _round(w)
    x_tree = dict(x)
    x_tree["target"] = torch.zeros((w.batch, w.n_max, w.V), device="cuda")
    x_tree["ctx_len"] = x["ctx_len"].clone()
    rnd_tree.bind(x_tree)
    rnd_tree.launch()
    torch.cuda.synchronize()
    tree = _tree(rnd_tree.out)
    for b in range(w.batch):
        n = int(tree["n_nodes"][b])
        for xr in range(n):
            kids = [c for c in range(n) if tree["parent"][b][c] == xr]
            t = int(tree["tok"][b][kids[0]]) if kids else 11
            hid[b, xr] = 8.0 * head[t] / float(head[t] @ head[t])
    x["hidden"].copy_(bf16_tensor(tob(hid)))
    ctx0 = a["ctx_len"].copy()
    rnd.launch()
    torch.cuda.synchronize()
    assert int(rnd.out["status"].item()) == 0
    rt, _, gap = oracle.lm_head_argmax(tob(hid).reshape(-1, K), tob(head))
    assert (gap.reshape(w.batch, w.n_max)[:, :int(tree["n_nodes"].min())] > 1.0).all()
    walk = oracle.walk_row_tokens(rt.reshape(w.batch, w.n_max), tree["tok"], tree["parent"],
                                  tree["depth"], tree["n_nodes"], w.L)
    for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
        np.testing.assert_array_equal(rnd.out[key].cpu().numpy(), walk[key])
    assert walk["acc_len"].min() >= 1
    k2, v2, c2, ok = oracle.kv_commit(a["k_tree"], a["v_tree"], walk["acc_len"], walk["acc_nodes"],
                                      ctx0, kc, vc)
    assert ok.all()
    np.testing.assert_array_equal(x["ctx_len"].cpu().numpy(), c2)
    bits = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(bits(x["k_cache"]), k2)
    np.testing.assert_array_equal(bits(x["v_cache"]), v2)
