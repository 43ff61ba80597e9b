"""Parity of ddt_tree_attn (CUDA, through the C ABI) with the oracle's fp64
masked attention.

Tolerance: bf16 output with fp32 accumulation against fp64, max-abs 2e-2 and
max-abs / max|ref| <= 1e-2 per case.  Small workloads compare every row; the
large ones compare a seeded sample of (sequence, row, head) items, always
including the root, the deepest rows and the last sequence, and, for every
head, the rows that open and close each 128-row query tile (the partial last
tile included), at the shortest context and at partial last pages and KV
tiles.  Each path of the kernel (CUDA cores; tensor cores with one KV pass,
with cluster-merged KV splits, with workspace-combined KV splits) runs on a
shape that ddt_tree_attn_plan says takes it."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api, synth

from helpers import ATTN_PATH_SHAPES, assert_attn_close, bf16_tensor, i32, oracle_tree_inputs

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


# ---------------------------------------------------------------------------
# Every row that opens or closes a query tile, the deepest rows, and the
# context edges (shortest context, partial last page / KV tile), all heads.
# ---------------------------------------------------------------------------
def _tile_edge_rows(w, n, tiles=None):
    """Tree rows holding the first or the last query row of a 128-row query
    tile of a kv head (query row = tree row * g + head in group), including
    the partial last tile; ``tiles`` restricts to some tile indices."""
    g = w.hq // w.hkv
    R = w.n_max * g
    nt = (R + 127) // 128
    rows = set()
    for t in (range(nt) if tiles is None else [t % nt for t in tiles]):
        for qr in (128 * t, min(128 * t + 127, R - 1)):
            if qr // g < n:
                rows.add(qr // g)
    return rows


def _edge_items(w, tree, seqs, tiles=None):
    items = []
    for b in seqs:
        n = int(tree["n_nodes"][b])
        dep = tree["depth"][b][:n]
        rows = _tile_edge_rows(w, n, tiles) | set(np.nonzero(dep == dep.max())[0][:2].tolist())
        rows.add(n - 1)
        items += [(b, j, h) for j in sorted(rows) for h in range(w.hq)]
    return np.array(items, np.int32)


def _paged_edge_seqs(ctx):
    """The shortest context, the longest, and contexts whose last page (64)
    and last KV tile (128) are partial or exactly full."""
    pick = {int(np.argmin(ctx)), int(np.argmax(ctx))}
    for cond in (lambda c: 0 < c % 64 < 32, lambda c: 64 < c % 128, lambda c: c % 64 == 0):
        hit = [b for b in range(len(ctx)) if cond(int(ctx[b]))]
        if hit:
            pick.add(hit[0])
    return sorted(pick)


@pytest.mark.parametrize("name", ["b64", "b256", "paged128", "long512"])
def test_large_edge_rows(name):
    w = synth.WORKLOADS[name]
    tree = _tree_for(w)
    a = synth.attention_inputs(w)
    out, lse = _gpu_attn(a, tree, w)
    if name == "paged128":
        seqs = _paged_edge_seqs(a["ctx_len"])
        assert any(0 < int(a["ctx_len"][b]) % 64 for b in seqs)
        tiles = None
    elif name == "long512":
        seqs, tiles = [w.batch - 1], [0, 1, 31, 32, -2, -1]
    else:
        seqs, tiles = ([0, 1] if w.batch > 1 else [0]), None
    items = _edge_items(w, tree, seqs, tiles)
    ref, ref_lse = _oracle_attn(a, tree, w, items)
    got = out[items[:, 0], items[:, 1], items[:, 2]]
    assert_attn_close(got, ref, name + " tile edges")
    np.testing.assert_allclose(lse[items[:, 0], items[:, 1], items[:, 2]], ref_lse, atol=2e-3)


# ---------------------------------------------------------------------------
# Each path of ddt_tree_attn, asserted through ddt_tree_attn_plan
# ---------------------------------------------------------------------------
def _plan(w, max_ctx):
    """ddt_tree_attn_plan for a workload's sizes (pointers are placeholders:
    the plan reads sizes only)."""
    lib = api.load_library()
    a = api.AttnArgs()
    fake = 1 << 20
    for f in ("q", "k_cache", "v_cache", "k_tree", "v_tree", "mask", "n_nodes", "ctx_len", "out"):
        setattr(a, f, fake)
    if w.page_size:
        a.page_table, a.page_size = fake, w.page_size
        a.max_pages = (max_ctx + w.page_size - 1) // w.page_size
        a.num_pages = a.max_pages * w.batch
    else:
        a.page_table, a.page_size, a.max_pages, a.num_pages = None, 0, 0, 0
        a.t_max = max_ctx
    a.max_ctx = max_ctx
    a.batch, a.n_max, a.hq, a.hkv, a.d = w.batch, w.n_max, w.hq, w.hkv, w.d
    a.scale = 1.0 / np.sqrt(w.d)
    path, splits = ctypes.c_int(), ctypes.c_int()
    assert lib.ddt_tree_attn_plan(ctypes.byref(a), ctypes.byref(path), ctypes.byref(splits)) == 0
    return path.value, splits.value


# candidate shapes per path; the test takes the first whose plan is that path
_PATH_CANDIDATES = {getattr(api, "ATTN_PATH_" + k): v for k, v in ATTN_PATH_SHAPES.items()}


@pytest.mark.parametrize("path", sorted(_PATH_CANDIDATES))
def test_each_attention_path(path):
    base = synth.WORKLOADS["b64"].scaled(L=6, V=400, k=4, hq=32, hkv=8, d=128)
    for kw in _PATH_CANDIDATES[path]:
        w = base.scaled(**kw)
        got_path, splits = _plan(w, w.ctx)
        if got_path == path:
            break
    else:
        pytest.fail("no candidate shape takes path %d" % path)
    if path in (api.ATTN_PATH_TC_CLUSTER, api.ATTN_PATH_TC_COMBINE, api.ATTN_PATH_TC_PAIRS_COMBINE):
        assert splits > 1
    tree = _tree_for(w)
    a = synth.attention_inputs(w)
    kw_t = dict(ctx_len=i32(a["ctx_len"]), max_ctx=int(a["ctx_len"].max()))
    args = (bf16_tensor(a["q"]), bf16_tensor(a["k_cache"]), bf16_tensor(a["v_cache"]),
            bf16_tensor(a["k_tree"]), bf16_tensor(a["v_tree"]),
            torch.from_numpy(tree["mask"].view(np.int32)).cuda(), i32(tree["n_nodes"]))
    assert api.tree_attn_plan(*args, kw_t["ctx_len"], kw_t["max_ctx"]) == (got_path, splits)
    nb = api.tree_attn_workspace_size(*args, kw_t["ctx_len"], kw_t["max_ctx"])
    assert (nb > 0) == (path in (api.ATTN_PATH_TC_COMBINE, api.ATTN_PATH_TC_PAIRS_COMBINE) or
                        (path == api.ATTN_PATH_SIMT and splits > 1))
    out, lse = _gpu_attn(a, tree, w)
    seqs = [0, w.batch - 1] if w.batch > 1 else [0]
    items = np.array([(b, j, h) for b in seqs for j in range(int(tree["n_nodes"][b]))
                      for h in range(w.hq)], np.int32)
    ref, ref_lse = _oracle_attn(a, tree, w, items)
    assert_attn_close(out[items[:, 0], items[:, 1], items[:, 2]], ref, "path %d" % path)
    np.testing.assert_allclose(lse[items[:, 0], items[:, 1], items[:, 2]], ref_lse, atol=2e-3)


@pytest.mark.parametrize("name,path", [("b64", api.ATTN_PATH_TC_CLUSTER), ("tiny", api.ATTN_PATH_SIMT)])
def test_workload_paths(name, path):
    """The path each named workload takes (the large ones: any tensor-core path)."""
    w = synth.WORKLOADS[name]
    assert _plan(w, w.ctx)[0] == path
    for big in ("b256", "paged128", "long512"):
        assert _plan(synth.WORKLOADS[big], synth.WORKLOADS[big].ctx)[0] != api.ATTN_PATH_SIMT


@pytest.mark.parametrize("paged", [False, True], ids=["dense", "paged"])
@pytest.mark.parametrize("kernel", ["ONE_TILE", "PAIRS"])
def test_each_kernel_family(kernel, paged):
    """Both tensor-core kernels, chosen through the library's override, on the
    same inputs: a dense cache and a paged one (ragged contexts, partial last
    pages), with two query tiles per kv head, match the oracle; the planner's
    own choice is restored afterwards."""
    base = synth.WORKLOADS["paged128" if paged else "b64"]
    w = base.scaled(batch=3, L=6, V=400, k=4, B=63, ctx=1500, hq=32, hkv=8, d=128,
                    **(dict(ctx_min=200) if paged else {}))
    prev = api.set_attn_kernel(getattr(api, "ATTN_KERNEL_" + kernel))
    try:
        got_path, _ = _plan(w, int(synth.context_lengths(w).max()))
        if kernel == "PAIRS":
            assert got_path in (api.ATTN_PATH_TC_PAIRS, api.ATTN_PATH_TC_PAIRS_COMBINE)
        else:
            assert got_path in (api.ATTN_PATH_TC, api.ATTN_PATH_TC_CLUSTER, api.ATTN_PATH_TC_COMBINE)
        _check(w, sample=400, seed=3)
    finally:
        api.set_attn_kernel(prev)


@pytest.mark.parametrize("path", ["TC_COMBINE", "TC_PAIRS_COMBINE", "TC_CLUSTER", "TC_PAIRS"])
def test_small_budgets_leave_dead_tiles(path):
    """Per-sequence budgets far below B_max (an adaptive split of the nodes):
    whole query tiles and pairs hold no tree row, and split partials exist
    only for the tree's rows.  Rows of the tree match the oracle; rows past
    n_nodes are zero with lse = -inf, on every path that splits or pairs."""
    base = synth.WORKLOADS["b64"].scaled(L=6, V=400, k=4, hq=32, hkv=8, d=128)
    want = getattr(api, "ATTN_PATH_" + path)
    for kw in ATTN_PATH_SHAPES[path]:
        w = base.scaled(**kw)
        if _plan(w, w.ctx)[0] == want:
            break
    else:
        pytest.fail("no candidate shape takes path " + path)
    ids, zk, lse = oracle_tree_inputs(w, synth.draft_logits(w))
    budgets = np.array([[w.B, 0, 3, max(1, w.B // 3)][b % 4] for b in range(w.batch)], np.int32)
    tree = oracle.build_tree(ids, zk, lse.astype(np.float64), budgets, w.inv_temperature,
                             root_token=synth.root_tokens(w), ctx_len=synth.context_lengths(w),
                             k_per_seq=w.k_per_seq(), n_max=w.n_max)
    a = synth.attention_inputs(w)
    out, lse_g = _gpu_attn(a, tree, w)
    seqs = sorted({0, 1, 2, 3, w.batch - 1} & set(range(w.batch)))
    items = np.array([(b, j, h) for b in seqs for j in range(int(tree["n_nodes"][b]))
                      for h in range(0, w.hq, 5)], np.int32)
    ref, ref_lse = _oracle_attn(a, tree, w, items)
    assert_attn_close(out[items[:, 0], items[:, 1], items[:, 2]], ref, "path %s, small budgets" % path)
    np.testing.assert_allclose(lse_g[items[:, 0], items[:, 1], items[:, 2]], ref_lse, atol=2e-3)
    for b in range(w.batch):
        n = int(tree["n_nodes"][b])
        assert np.all(out[b, n:] == 0) and np.all(np.isneginf(lse_g[b, n:]))
