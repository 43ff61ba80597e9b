"""The C ABI without a GPU: libddt.so builds, loads, exports every function
include/ddt.h declares, and rejects bad arguments on the host before any
launch (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from block_draft_tree_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(ddt_[a-z0-9_]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load_library()


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert {"ddt_topk", "ddt_build_tree", "ddt_tree_attn", "ddt_tree_walk"} <= declared
    raw = ctypes.CDLL(api.library_path())
    for name in sorted(declared):
        assert hasattr(raw, name), name
    assert set(api.EXPORTED) <= declared


def test_status_strings(lib):
    for code in range(6):
        assert lib.ddt_status_string(code).startswith(b"DDT_")
    assert lib.ddt_mask_words(513) == 17 and lib.ddt_mask_words(32) == 1


def test_topk_rejects_bad_arguments(lib):
    f = lib.ddt_topk
    dummy = ctypes.c_void_p(16)
    args = dict(logits=dummy, dt=0, b=1, L=4, V=64, stride=64, k=4, it=1.0)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["logits"], a["dt"], a["b"], a["L"], a["V"], a["stride"], a["k"], a["it"],
                 dummy, dummy, dummy, dummy, None, 0, None)

    assert call(k=33) == 2           # above DDT_TOPK_K_MAX
    assert call(k=65) in (1, 2)      # k > V
    assert call(stride=10) == 1      # row stride < V
    assert call(it=0.0) == 1 and call(it=-1.0) == 1 and call(it=float("inf")) == 1
    assert call(dt=7) == 2
    assert call(logits=None) == 1
    assert call(V=200000, stride=200000) == 3  # needs a workspace, none given
    assert call(b=100, L=1000) == 2  # more rows than the grid holds


def test_build_tree_rejects_bad_arguments(lib):
    f = lib.ddt_build_tree
    d = ctypes.c_void_p(16)

    def call(b=1, L=4, k=4, B=8, it=1.0, ids=d):
        return f(ids, d, d, b, L, k, it, None, None, B, d, None, d, d, d, d, d, d, None, None, None)

    assert call(L=65) == 2 and call(k=33) == 2 and call(B=1024) == 2
    assert call(L=0) == 1 and call(B=-1) == 1 and call(it=0.0) == 1
    assert call(ids=None) == 1


def test_attn_rejects_bad_arguments(lib):
    a = api.AttnArgs()
    a.q = a.k_cache = a.v_cache = a.k_tree = a.v_tree = a.mask = a.n_nodes = a.ctx_len = a.out = 256
    a.batch, a.n_max, a.hq, a.hkv, a.d, a.max_ctx, a.t_max = 1, 9, 4, 1, 64, 128, 128
    a.scale = 0.125
    f = lib.ddt_tree_attn
    base = dict((n, getattr(a, n)) for n, _ in api.AttnArgs._fields_)

    def call(**kw):
        b = api.AttnArgs(**dict(base, **kw))
        return f(ctypes.byref(b), None, 0, None)

    assert call(d=96) == 2
    assert call(hq=6, hkv=4) == 1
    assert call(n_max=1025) == 2
    assert call(q=None) == 1
    assert call(q=258) == 1              # misaligned
    assert call(t_max=100) == 1          # dense cache shorter than max_ctx
    assert call(page_table=512, page_size=10, max_pages=20) == 2
    assert call(page_table=512, page_size=16, max_pages=2) == 1
    assert call(scale=0.0) == 1
    assert f(None, None, 0, None) == 1


def test_walk_rejects_bad_arguments(lib):
    f = lib.ddt_tree_walk
    d = ctypes.c_void_p(16)

    def call(b=1, n=9, V=64, stride=64, L=4, dt=1, logits=d, mode=0):
        return f(logits, dt, b, n, V, stride, d, d, d, d, L, mode, d, d, d, d, None, 0, None, None)

    assert call(stride=3) == 1 and call(dt=5) == 2 and call(n=2000) == 2 and call(L=65) == 2
    assert call(mode=-1) == 1 and call(mode=3) == 1
    assert call(logits=None) == 1
    assert call(V=10 ** 6, stride=10 ** 6) == 3  # workspace required


def test_walk_sample_rejects_bad_arguments(lib):
    f = lib.ddt_tree_walk_sample
    d = ctypes.c_void_p(16)

    def call(b=1, n=9, V=64, stride=64, L=4, dt=1, it=1.0, logits=d):
        return f(logits, dt, b, n, V, stride, d, d, d, d, L, it, 7, 0, None, d, d, d, d, None, 0,
                 None, None)

    assert call(it=0.0) == 1 and call(it=-0.5) == 1 and call(it=float("nan")) == 1
    assert call(it=float("inf")) == 1 and call(it=3e38) == 1  # 1/T * log2(e) overflows
    assert call(stride=3) == 1 and call(dt=5) == 2 and call(n=2000) == 2 and call(L=65) == 2
    assert call(logits=None) == 1
    assert call(V=10 ** 6, stride=10 ** 6) == 3  # workspace required
    assert f(d, 1, 1, 9, 64, 64, d, d, d, d, 4, 1.0, 7, 0, ctypes.c_void_p(20), d, d, d, d, None,
             0, None, None) == 1                 # a step counter must be 8-byte aligned


def test_kv_commit_rejects_bad_arguments(lib):
    d = 4096  # any 16-byte aligned non-null address: nothing is launched

    def call(**kw):
        a = api.KVCommitArgs()
        a.k_tree = a.v_tree = a.acc_len = a.acc_nodes = a.ctx_len = a.k_cache = a.v_cache = d
        a.page_table, a.page_size, a.max_pages, a.num_pages, a.t_max = None, 0, 0, 0, 64
        a.batch, a.n_max, a.hkv, a.d, a.L, a.dev_status = 1, 9, 8, 128, 4, None
        for k, v in kw.items():
            setattr(a, k, v)
        return lib.ddt_kv_commit(ctypes.byref(a), None)

    assert lib.ddt_kv_commit(None, None) == 1
    assert call(n_max=0) == 1 and call(hkv=0) == 1 and call(L=-1) == 1
    assert call(L=65) == 2 and call(hkv=1, d=3) == 2    # L above the limit; hkv*d % 8 != 0
    assert call(k_tree=None) == 1 and call(k_cache=4100) == 1  # null; misaligned
    assert call(t_max=0) == 1                           # dense cache without capacity
    assert call(page_table=d, page_size=0, max_pages=4) == 1
    assert call(batch=0, k_tree=None) == 0              # nothing to do


def test_lm_head_walk_rejects_bad_arguments(lib):
    d = 4096  # any 16-byte aligned non-null address: nothing is launched
    assert lib.ddt_lm_head_max_rows() >= 30000

    def call(ws=None, nb=0, **kw):
        a = api.LmHeadWalkArgs()
        a.hidden = a.weight = a.tok = a.parent = a.depth = a.n_nodes = d
        a.acc_len = a.acc_nodes = a.acc_tok = a.bonus = d
        a.K, a.V, a.batch, a.n_max, a.L = 4096, 151936, 1, 65, 16
        a.row_token = a.dev_status = None
        for k, v in kw.items():
            setattr(a, k, v)
        return lib.ddt_lm_head_walk(ctypes.byref(a), ws, nb, None)

    assert lib.ddt_lm_head_walk(None, None, 0, None) == 1
    assert call(K=0) == 1 and call(V=0) == 1 and call(n_max=0) == 1 and call(L=-1) == 1
    assert call(K=100) == 2                          # K not a multiple of 8
    assert call(batch=1000, n_max=513) == 2          # more rows than the counter region holds
    assert call(L=65) == 2 and call(n_max=1025) == 2
    assert call(hidden=None) == 1 and call(weight=4100) == 1
    assert call() == 3                               # workspace required
    assert call(batch=0, hidden=None) == 0


def test_binding_refuses_cpu_tensors(lib):
    import torch
    with pytest.raises(api.DDTError):
        api.topk(torch.zeros(1, 2, 64), 4)


def test_round_driver_rejects_an_unknown_decoding_rule():
    from block_draft_tree_b200.round import VerifyRound
    with pytest.raises(ValueError):
        VerifyRound(batch=1, L=4, V=64, k=4, B_max=8, hq=4, hkv=1, d=64, max_ctx=128, decode="beam")


def test_noalloc_topk_rejects_like_topk(lib):
    """ddt_topk_noalloc checks its arguments exactly as ddt_topk does, and
    before it touches its scratch array (no CUDA call is made here)."""
    f = lib.ddt_topk_noalloc
    f.restype = ctypes.c_int
    vp = ctypes.c_void_p
    f.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                  ctypes.c_int, ctypes.c_float, vp, vp, vp, vp, vp]
    dummy = ctypes.c_void_p(16)
    base = dict(logits=dummy, dt=0, b=1, L=4, V=64, stride=64, k=4, it=1.0)
    cases = [dict(k=33), dict(k=65), dict(stride=10), dict(it=0.0), dict(it=float("inf")),
             dict(dt=7), dict(b=-1), dict(logits=None), dict(b=4096, L=17)]
    for kw in cases:
        a = dict(base, **kw)
        ref = lib.ddt_topk(a["logits"], a["dt"], a["b"], a["L"], a["V"], a["stride"], a["k"],
                           a["it"], dummy, dummy, dummy, dummy, None, 0, None)
        got = f(a["logits"], a["dt"], a["b"], a["L"], a["V"], a["stride"], a["k"], a["it"],
                dummy, dummy, dummy, dummy, None)
        assert ref != 0 and got == ref, (kw, ref, got)


def test_walk_rejects_an_unknown_mode(lib):
    dummy = ctypes.c_void_p(256)
    rc = lib.ddt_tree_walk(dummy, 1, 1, 9, 100, 100, dummy, dummy, dummy, dummy, 4, 7,
                           dummy, dummy, dummy, dummy, None, 0, None, None)
    assert rc == 1
    assert lib.ddt_tree_walk_resolve_mode(7, 1, 1, 9, 100, 4) == -1


def test_attention_kernel_override_is_a_setting(lib):
    prev = api.set_attn_kernel(api.ATTN_KERNEL_PAIRS)
    try:
        assert api.set_attn_kernel(api.ATTN_KERNEL_ONE_TILE) == api.ATTN_KERNEL_PAIRS
        assert api.set_attn_kernel(3) == -1 and api.set_attn_kernel(-1) == -1
        assert api.set_attn_kernel(api.ATTN_KERNEL_AUTO) == api.ATTN_KERNEL_ONE_TILE
    finally:
        api.set_attn_kernel(prev)


def test_plan_budget_rejects_bad_arguments(lib):
    d = ctypes.c_void_p(256)  # any non-null address: nothing is launched

    def call(batch=4, L=16, k=8, n_max=65, inv_t=1.0, total=128, c0=1.0, c1=0.01, **ptrs):
        p = dict(tok=d, parent=d, depth=d, n_nodes=d, ids=d, zk=d, lse=d, budget=d)
        p.update(ptrs)
        return lib.ddt_plan_budget(p["tok"], p["parent"], p["depth"], p["n_nodes"], p["ids"],
                                   p["zk"], p["lse"], batch, L, k, n_max, inv_t, total, c0, c1,
                                   p["budget"], None, None, None)

    assert call(batch=-1) == 1 and call(L=0) == 1 and call(k=0) == 1 and call(n_max=0) == 1
    assert call(L=65) == 2 and call(k=33) == 2 and call(n_max=1025) == 2
    assert call(batch=129, n_max=65) == 2            # 129 * 64 nodes > 8192
    assert call(inv_t=0.0) == 1 and call(inv_t=float("inf")) == 1 and call(inv_t=float("nan")) == 1
    assert call(c0=-1.0) == 1 and call(c0=float("inf")) == 1
    assert call(c1=float("nan")) == 1 and call(c1=float("inf")) == 1
    assert call(c0=0.0, c1=0.5) == 1                  # a per-node cost needs a fixed cost
    for name in ("tok", "parent", "depth", "n_nodes", "ids", "zk", "lse", "budget"):
        assert call(**{name: None}) == 1, name


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without libddt.so every call raises: there is no other implementation
    to fall back to."""
    import torch
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "_LIB_PATH", str(tmp_path / "libddt.so"))
    with pytest.raises(api.DDTError, match="not built"):
        api.load_library()
    with pytest.raises(api.DDTError):
        api.topk(torch.zeros(1, 2, 64), 4)


def test_binding_checks_tree_tensor_types(lib):
    """The walk and budget bindings refuse tree tensors the kernels would
    misread (int64, float, non-contiguous) before anything else."""
    import torch
    logits = torch.zeros(1, 3, 16)
    ok = [torch.zeros(1, 3, dtype=torch.int32) for _ in range(3)] + [torch.ones(1, dtype=torch.int32)]
    bad64 = [t.long() for t in ok]
    strided = torch.zeros(1, 6, dtype=torch.int32)[:, ::2]
    for fn, extra in ((api.tree_walk, ()), (api.tree_walk_sample, (1.0, 1, 0))):
        with pytest.raises(api.DDTError, match="contiguous"):
            fn(logits, *bad64, 2, *extra)
        with pytest.raises(api.DDTError, match="contiguous"):
            fn(logits, strided, *ok[1:], 2, *extra)
        with pytest.raises(api.DDTError, match="CUDA tensors only"):
            fn(logits, *ok, 2, *extra)
    tree = dict(zip(("tok", "parent", "depth", "n_nodes"), ok))
    ids = torch.zeros(1, 2, 2, dtype=torch.int32)
    zk, lse = torch.zeros(1, 2, 2), torch.zeros(1, 2)
    with pytest.raises(api.DDTError, match="contiguous"):
        api.plan_budget(tree, ids, zk.double(), lse)
    with pytest.raises(api.DDTError, match="contiguous"):
        api.plan_budget(dict(tree, parent=bad64[1]), ids, zk, lse)
    with pytest.raises(api.DDTError, match="CUDA tensors only"):
        api.plan_budget(tree, ids, zk, lse)


def test_binding_checks_tree_tensor_shapes(lib):
    """Tree tensors whose extents differ from the logits' [batch, n_max] (or
    the candidates' batch) are refused before anything is launched."""
    import torch
    i32 = lambda *s: torch.zeros(*s, dtype=torch.int32)
    logits = torch.zeros(2, 3, 16)
    for fn, extra in ((api.tree_walk, ()), (api.tree_walk_sample, (1.0, 1, 0))):
        with pytest.raises(api.DDTError, match=r"\[2, 3\]"):
            fn(logits, i32(2, 2), i32(2, 3), i32(2, 3), i32(2), 2, *extra)
        with pytest.raises(api.DDTError, match=r"n_nodes must be \[2\]"):
            fn(logits, i32(2, 3), i32(2, 3), i32(2, 3), i32(1), 2, *extra)
    tree = {"tok": i32(2, 3), "parent": i32(2, 3), "depth": i32(1, 3), "n_nodes": i32(2)}
    ids, zk, lse = i32(2, 4, 2), torch.zeros(2, 4, 2), torch.zeros(2, 4)
    with pytest.raises(api.DDTError, match=r"\[2, 3\]"):
        api.plan_budget(tree, ids, zk, lse)
    with pytest.raises(api.DDTError, match="lse"):
        api.plan_budget(dict(tree, depth=i32(2, 3)), ids, zk, torch.zeros(2, 3))


def test_binding_checks_attention_and_commit_extents(lib):
    """tree_attn and kv_commit refuse K/V, caches, masks and per-sequence
    arrays whose extents disagree with q / the tree K/V, before any launch."""
    import torch
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    i32 = lambda *s: torch.zeros(*s, dtype=torch.int32)
    b, n, hq, hkv, d, T = 2, 5, 4, 2, 64, 16
    good = dict(q=bf(b, n, hq, d), k_cache=bf(b, T, hkv, d), v_cache=bf(b, T, hkv, d),
                k_tree=bf(b, n, hkv, d), v_tree=bf(b, n, hkv, d), mask=i32(b, n, 1),
                n_nodes=i32(b), ctx_len=i32(b), max_ctx=T)

    def attn(**kw):
        return api.tree_attn(**dict(good, **kw))

    with pytest.raises(api.DDTError, match="CUDA tensors only"):
        attn()
    for kw, msg in ((dict(k_tree=bf(b, n + 1, hkv, d)), "tree K"),
                    (dict(v_tree=bf(b, n, hkv, d + 64)), "tree V"),
                    (dict(k_cache=bf(b + 1, T, hkv, d), v_cache=bf(b + 1, T, hkv, d)), "dense"),
                    (dict(v_cache=bf(b, T - 1, hkv, d)), "V cache"),
                    (dict(k_cache=bf(b, T, 1, d), v_cache=bf(b, T, 1, d)), "caches"),
                    (dict(mask=i32(b, n, 2)), "mask"),
                    (dict(n_nodes=i32(b + 1)), "n_nodes"),
                    (dict(k_cache=bf(9, 16, hkv, d), v_cache=bf(9, 16, hkv, d),
                          page_table=i32(b + 1, 3)), "page_table")):
        with pytest.raises(api.DDTError, match=msg):
            attn(**kw)

    kt, acc_len, acc_nodes, cl = bf(b, n, hkv, d), i32(b), i32(b, 3), i32(b)
    with pytest.raises(api.DDTError, match="CUDA tensors only"):
        api.kv_commit(kt, kt.clone(), acc_len, acc_nodes, cl, bf(b, T, hkv, d), bf(b, T, hkv, d))
    with pytest.raises(api.DDTError, match="dense"):
        api.kv_commit(kt, kt.clone(), acc_len, acc_nodes, cl, bf(1, T, hkv, d), bf(1, T, hkv, d))
    with pytest.raises(api.DDTError, match="page_size"):
        api.kv_commit(kt, kt.clone(), acc_len, acc_nodes, cl, bf(8, 32, hkv, d), bf(8, 32, hkv, d),
                      page_table=i32(b, 4), page_size=64)
    with pytest.raises(api.DDTError, match="acc_nodes"):
        api.kv_commit(kt, kt.clone(), acc_len, i32(b), cl, bf(b, T, hkv, d), bf(b, T, hkv, d))
    with pytest.raises(api.DDTError, match="acc_len"):
        api.kv_commit(kt, kt.clone(), i32(b + 1), acc_nodes, cl, bf(b, T, hkv, d), bf(b, T, hkv, d))


def test_binding_checks_tree_builder_extents(lib):
    import torch
    i32 = lambda *s: torch.zeros(*s, dtype=torch.int32)
    ids, zk, lse = i32(2, 3, 4), torch.zeros(2, 3, 4), torch.zeros(2, 3)
    with pytest.raises(api.DDTError, match="CUDA tensors only"):
        api.build_tree(ids, zk, lse, 8, i32(2))
    with pytest.raises(api.DDTError, match="lse"):
        api.build_tree(ids, zk, torch.zeros(2, 4), 8, i32(2))
    with pytest.raises(api.DDTError, match="root_token"):
        api.build_tree(ids, zk, lse, 8, i32(3))
    with pytest.raises(api.DDTError, match="budget"):
        api.build_tree(ids, zk, lse, 8, i32(2), budget=i32(1))


def test_binding_checks_lm_head_extents(lib):
    import torch
    i32 = lambda *s: torch.zeros(*s, dtype=torch.int32)
    h, wt = torch.zeros(2, 5, 64, dtype=torch.bfloat16), torch.zeros(100, 64, dtype=torch.bfloat16)
    tree = (i32(2, 5), i32(2, 5), i32(2, 5), i32(2))
    with pytest.raises(api.DDTError, match="CUDA tensors only"):
        api.lm_head_walk(h, wt, *tree, 4)
    with pytest.raises(api.DDTError, match=r"\[2, 5\]"):
        api.lm_head_walk(h, wt, i32(2, 4), *tree[1:], 4)
    with pytest.raises(api.DDTError, match="weight"):
        api.lm_head_walk(h, wt.reshape(-1), *tree, 4)


def test_round_driver_checks_bound_inputs():
    """VerifyRound.bind refuses inputs that disagree with the round's sizes
    (shape, dtype, row layout), before any pointer reaches the library."""
    import torch
    from block_draft_tree_b200.round import VerifyRound
    b, L, V, k, B, hq, hkv, d, T = 2, 4, 64, 4, 8, 4, 1, 64, 32
    n = B + 1
    rnd = VerifyRound(batch=b, L=L, V=V, k=k, B_max=B, hq=hq, hkv=hkv, d=d, max_ctx=T,
                      draft_dtype=torch.float32, device="cpu")
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    i32 = lambda *s: torch.zeros(*s, dtype=torch.int32)
    good = {"draft": torch.zeros(b, L, V), "root": i32(b), "ctx_len": i32(b),
            "q": bf(b, n, hq, d), "k_tree": bf(b, n, hkv, d), "v_tree": bf(b, n, hkv, d),
            "k_cache": bf(b, T, hkv, d), "v_cache": bf(b, T, hkv, d),
            "target": torch.zeros(b, n, V)}
    rnd._check_inputs(good)   # consistent inputs pass
    bad = [(dict(draft=torch.zeros(b, L, V, dtype=torch.bfloat16)), "draft"),
           (dict(draft=torch.zeros(b, L + 1, V)), "draft"),
           (dict(draft=torch.zeros(b, L, 2 * V)[:, :, ::2]), "row stride"),
           (dict(root=i32(b + 1)), "root"),
           (dict(ctx_len=torch.zeros(b, dtype=torch.int64)), "ctx_len"),
           (dict(q=bf(b, n, hq, 128)), "'q'"),
           (dict(k_tree=bf(b, n - 1, hkv, d)), "k_tree"),
           (dict(k_cache=bf(b + 1, T, hkv, d), v_cache=bf(b + 1, T, hkv, d)), "dense"),
           (dict(target=torch.zeros(b, n - 1, V)), "target"),
           (dict(budget=i32(b + 1)), "budget")]
    for kw, msg in bad:
        with pytest.raises(api.DDTError, match=msg):
            rnd.bind(dict(good, **kw))
    lm = VerifyRound(batch=b, L=L, V=V, k=k, B_max=B, hq=hq, hkv=hkv, d=d, max_ctx=T,
                     draft_dtype=torch.float32, decode="lm_head", device="cpu")
    with pytest.raises(api.DDTError, match="hidden"):
        lm.bind(good)
    with pytest.raises(api.DDTError, match="head"):
        lm.bind(dict(good, hidden=bf(b, n, 128), head=bf(V, 64)))
