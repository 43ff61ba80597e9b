"""Parity of ddt_lm_head_walk (tcgen05 LM head + argmax + walk, through the
C ABI) with the oracle: fp64 logits H W^T, lowest-id argmax, walk over the row
tokens.

The kernel accumulates in fp32 on the tensor cores, so a row's argmax is
compared exactly when the oracle's top-2 gap is at least LOGIT_MARGIN; a
closer row may take either of its near-equal tokens (the check is then that
the kernel's token is one of them).  A walk is compared bit for bit when
every row it visits clears the margin.

Margin: logits here are sums of K products of bf16 values (exact in fp32);
accumulating K of them in fp32 is within K * 2^-24 * sum|h_k w_k| of exact.
For the unplanted rows of these inputs sum|h w| is about 20 at K = 4096, so
the bound is about 5e-3 (the observed error is far smaller: the roundings
of a long sum mostly cancel).  Planted rows lead by about 8.
"""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api

from helpers import bf16_tensor, i32

pytestmark = pytest.mark.gpu

LOGIT_MARGIN = 5e-3


def _bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _tree(rng, n_max, L, V, n):
    """A random breadth-first tree of n rows (root 0) with depth <= L."""
    tok = np.full(n_max, -1, np.int32)
    par = np.full(n_max, -1, np.int32)
    dep = np.zeros(n_max, np.int32)
    tok[0] = int(rng.integers(0, V))
    for j in range(1, n):
        while True:
            p = int(rng.integers(0, j))
            if dep[p] < L:
                break
        par[j], dep[j], tok[j] = p, dep[p] + 1, int(rng.integers(0, V))
    order = np.argsort(dep[:n], kind="stable")  # breadth first
    remap = np.empty(n, np.int64)
    remap[order] = np.arange(n)
    tok2, par2, dep2 = tok.copy(), par.copy(), dep.copy()
    tok2[:n], dep2[:n] = tok[order], dep[order]
    par2[:n] = [remap[par[o]] if par[o] >= 0 else -1 for o in order]
    return tok2, par2, dep2


def _case(seed, batch, n_max, L, K, V, plant=0.7):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((V, K)) / np.sqrt(K)).astype(np.float32)
    h = rng.standard_normal((batch, n_max, K)).astype(np.float32) * 0.5
    toks, pars, deps, ns = [], [], [], []
    for b in range(batch):
        n = int(rng.integers(max(1, n_max // 2), n_max + 1))
        tok, par, dep = _tree(rng, n_max, L, V, n)
        # plant: with probability `plant` row x points at one of its children
        # (a leaf at a random token) with a logit of 8, far above the rest
        for x in range(n):
            if rng.random() >= plant:
                continue
            kids = [c for c in range(n) if par[c] == x]
            t = tok[kids[int(rng.integers(0, len(kids)))]] if kids else int(rng.integers(0, V))
            h[b, x] = 8.0 * w[t] / float(w[t] @ w[t])
        toks.append(tok)
        pars.append(par)
        deps.append(dep)
        ns.append(n)
    return (_bits(h), _bits(w), np.stack(toks), np.stack(pars), np.stack(deps),
            np.array(ns, np.int32))


def _compare(h, w, tok, par, dep, n, L, block=None):
    batch, n_max, K = h.shape
    rt, top, gap = oracle.lm_head_argmax(h.reshape(-1, K), w, block=block)
    rt = rt.reshape(batch, n_max)
    gap = gap.reshape(batch, n_max)
    ref = oracle.walk_row_tokens(rt, tok, par, dep, n, L)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = api.lm_head_walk(bf16_tensor(h), bf16_tensor(w), i32(tok), i32(par), i32(dep), i32(n), L,
                           want_row_token=True, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    g = {k: v.cpu().numpy() for k, v in got.items()}
    clear = gap >= LOGIT_MARGIN
    np.testing.assert_array_equal(g["row_token"][clear], rt[clear])
    if (~clear).any():  # a near tie: the kernel's token must be one of the near-equal ones
        hf = (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        wf = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        for b, j in zip(*np.nonzero(~clear)):
            lg = wf @ hf[b, j]
            assert lg[g["row_token"][b, j]] >= lg.max() - LOGIT_MARGIN
    exact = 0
    for b in range(batch):
        rows = [0] + list(ref["acc_nodes"][b][:ref["acc_len"][b]])
        if all(clear[b, x] for x in rows):
            exact += 1
            for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
                np.testing.assert_array_equal(g[key][b], ref[key][b], err_msg="%s[%d]" % (key, b))
    return ref, g, exact


@pytest.mark.parametrize("batch,n_max,L,K,V", [
    (1, 9, 4, 128, 1000),        # one tile of rows, a ragged vocabulary tile
    (3, 40, 6, 520, 3001),       # K not a multiple of 64, rows across sequences
    (4, 65, 16, 256, 20000),     # 260 rows: three row tiles
    (2, 129, 8, 1024, 8192),     # exact vocabulary tiles
])
def test_small_shapes(batch, n_max, L, K, V):
    h, w, tok, par, dep, n = _case(batch * 1000 + K, batch, n_max, L, K, V)
    ref, got, exact = _compare(h, w, tok, par, dep, n, L)
    assert exact >= (batch + 1) // 2
    assert ref["acc_len"].sum() > 0  # the planted rows make the walks descend


def test_b64_shape_full_vocabulary():
    """One sequence of 65 rows against a 151936 x 4096 LM head (1.2 GB)."""
    h, w, tok, par, dep, n = _case(64, 1, 65, 16, 4096, 151936, plant=1.0)
    ref, got, exact = _compare(h, w, tok, par, dep, n, 16, block=16384)
    assert exact == 1


def test_repeated_calls_reuse_the_workspace():
    h, w, tok, par, dep, n = _case(7, 2, 33, 8, 256, 5000)
    first = None
    for _ in range(3):
        _, got, _ = _compare(h, w, tok, par, dep, n, 8)
        if first is None:
            first = got
        for k in first:
            np.testing.assert_array_equal(got[k], first[k])


def test_b256_rows_sampled_at_full_size():
    """2056 rows (8 trees of 257) against the 151936 x 4096 head: the row
    tokens of 64 sampled rows against the oracle's, row by row, and every
    walk checked as a walk over the kernel's own row tokens."""
    batch, n_max, L, K, V = 8, 257, 16, 4096, 151936
    rng = np.random.default_rng(256)
    w = _bits((rng.standard_normal((V, K)) / np.sqrt(K)).astype(np.float32))
    hf = rng.standard_normal((batch, n_max, K)).astype(np.float32) * 0.5
    toks, pars, deps = [], [], []
    wf = (w.astype(np.uint32) << 16).view(np.float32)
    for b in range(batch):
        tok, par, dep = _tree(rng, n_max, L, V, n_max)
        for x in range(n_max):  # plant every inner row on its first child
            kids = np.nonzero(par[:n_max] == x)[0]
            if len(kids):
                t = int(tok[kids[0]])
                hf[b, x] = 8.0 * wf[t] / float(wf[t] @ wf[t])
        toks.append(tok)
        pars.append(par)
        deps.append(dep)
    h = _bits(hf)
    tok, par, dep = np.stack(toks), np.stack(pars), np.stack(deps)
    n = np.full(batch, n_max, np.int32)
    got = api.lm_head_walk(bf16_tensor(h), bf16_tensor(w), i32(tok), i32(par), i32(dep), i32(n), L,
                           want_row_token=True)
    torch.cuda.synchronize()
    g = {k: v.cpu().numpy() for k, v in got.items()}
    rows = rng.choice(batch * n_max, 64, replace=False)
    rt, _, gap = oracle.lm_head_argmax(h.reshape(-1, K)[rows], w, block=16384)
    clear = gap >= LOGIT_MARGIN
    np.testing.assert_array_equal(g["row_token"].reshape(-1)[rows][clear], rt[clear])
    assert clear.sum() >= 48
    ref = oracle.walk_row_tokens(g["row_token"], tok, par, dep, n, L)
    for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
        np.testing.assert_array_equal(g[key], ref[key])
    assert ref["acc_len"].min() >= 1  # the planted first children are accepted
