"""The bounded waits of the tensor-core kernels, made to run out on purpose.

Every wait of the tensor-core attention and of the LM-head walk on an on-chip
barrier gives up after a bound (about one second by default).  A wait that
gives up raises DDT_ERR_TIMEOUT in the call's status word; the kernel then
lets the copies and MMAs it has in flight complete, frees its tensor memory
and returns.  These tests shorten the bound to a few clock cycles through the
library's test hook (ddt_debug_set_wait_limit), so that the waits run out on
an ordinary input, check the status, then restore the default and check that
the next call on the same stream is correct (the context, the tensor memory
and the workspace are all still usable).  No fault is involved: the kernel's
own bound ends the wait.
"""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api, synth

from helpers import ATTN_PATH_SHAPES, assert_attn_close, bf16_tensor, i32, oracle_tree_inputs

pytestmark = pytest.mark.gpu

DDT_ERR_TIMEOUT = 5
SHORT = 4  # clock cycles: every wait that is not already satisfied runs out


class _ShortWaits:
    def __enter__(self):
        self.prev = api.set_wait_limit(SHORT)
        return self

    def __exit__(self, *exc):
        api.set_wait_limit(self.prev)
        return False


def _attn_case(kw):
    w = synth.WORKLOADS["b64"].scaled(L=6, V=400, k=4, hq=32, hkv=8, d=128, **kw)
    ids, zk, lse = oracle_tree_inputs(w, synth.draft_logits(w))
    tree = oracle.build_tree(ids, zk, lse.astype(np.float64), w.budget_per_seq(),
                             w.inv_temperature, root_token=synth.root_tokens(w),
                             ctx_len=synth.context_lengths(w), n_max=w.n_max)
    a = synth.attention_inputs(w)
    args = (bf16_tensor(a["q"]), bf16_tensor(a["k_cache"]), bf16_tensor(a["v_cache"]),
            bf16_tensor(a["k_tree"]), bf16_tensor(a["v_tree"]),
            torch.from_numpy(tree["mask"].view(np.int32)).cuda(), i32(tree["n_nodes"]),
            i32(a["ctx_len"]), int(a["ctx_len"].max()))
    return w, tree, a, args


@pytest.mark.parametrize("path", ["TC", "TC_CLUSTER", "TC_PAIRS", "TC_PAIRS_COMBINE"],
                         ids=["one-pass", "cluster-splits", "pairs", "pairs-combined"])
def test_attention_wait_runs_out_then_recovers(path):
    for kw in ATTN_PATH_SHAPES[path]:
        w, tree, a, args = _attn_case(kw)
        if api.tree_attn_plan(*args)[0] == getattr(api, "ATTN_PATH_" + path):
            break
    else:
        pytest.fail("no candidate shape takes path " + path)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with _ShortWaits():
        api.tree_attn(*args, dev_status=st)
        torch.cuda.synchronize()
    assert st.item() == DDT_ERR_TIMEOUT
    # the default bound again: the next call on the same stream is exact
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = api.tree_attn(*args, dev_status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    seqs = [0, w.batch - 1]
    items = np.array([(b, j, h) for b in sorted(set(seqs)) for j in range(int(tree["n_nodes"][b]))
                      for h in range(0, w.hq, 3)], np.int32)
    ref, _ = oracle.tree_attn(items, a["q"], a["k_cache"], a["v_cache"], a["ctx_len"], a["k_tree"],
                              a["v_tree"], tree["mask"], tree["n_nodes"], 1.0 / np.sqrt(w.d))
    got = out.float().cpu().numpy()[items[:, 0], items[:, 1], items[:, 2]]
    assert_attn_close(got, ref, "attention after a timeout")


def test_lm_head_wait_runs_out_then_recovers():
    rng = np.random.default_rng(4)
    bsz, n, K, V, L = 2, 9, 256, 3000, 4
    tob = lambda v: (v.view(np.uint32) >> 16).astype(np.uint16)
    head = tob((rng.standard_normal((V, K)) / np.sqrt(K)).astype(np.float32))
    hid = tob(rng.standard_normal((bsz, n, K)).astype(np.float32))
    # a chain tree per sequence: root -> 1 -> 2 -> 3 -> ... (tokens 5, 6, ...)
    tok = np.tile(np.array([0] + [5 + i for i in range(n - 1)], np.int32), (bsz, 1))
    parent = np.tile(np.arange(-1, n - 1, dtype=np.int32), (bsz, 1))
    depth = np.tile(np.minimum(np.arange(n, dtype=np.int32), L), (bsz, 1))
    parent[:, L + 1:] = -1
    nn = np.full(bsz, L + 1, np.int32)
    targs = (bf16_tensor(hid), bf16_tensor(head), i32(tok), i32(parent), i32(depth), i32(nn), L)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with _ShortWaits():
        api.lm_head_walk(*targs, dev_status=st)
        torch.cuda.synchronize()
    assert st.item() == DDT_ERR_TIMEOUT
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        got = api.lm_head_walk(*targs, want_row_token=True, dev_status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    rt, _, gap = oracle.lm_head_argmax(hid.reshape(-1, K), head)
    rt = rt.reshape(bsz, n)
    close = gap.reshape(bsz, n) < 1e-3  # rows whose argmax rounding may decide either way
    g_rt = got["row_token"].cpu().numpy()
    assert np.all((g_rt == rt) | close)
    walk = oracle.walk_row_tokens(g_rt, tok, parent, depth, nn, L)
    for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
        np.testing.assert_array_equal(got[key].cpu().numpy(), walk[key], err_msg=key)


def test_default_bound_is_restored():
    assert api.set_wait_limit(0) == 0
