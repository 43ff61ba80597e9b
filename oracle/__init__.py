"""CPU oracle for the DDTree verification round (fp64, plain C + ctypes).

TEST INFRASTRUCTURE ONLY.  The test-suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers.  The product library (``block_draft_tree_b200``) never imports this
package, and this package never imports the product: the two share no code.

Each function restates one step of the DDTree page (Diffusion Draft Tree,
curated summary of the authors' announcement), section "運作流程"
(workflow):

* :func:`topk`       -- step 1, per-position marginals q_i: log-sum-exp and
  the top-k candidate tokens of each position;
* :func:`build_tree` -- step 2 (best B prefixes of the factorised draft,
  "核心創新" / "理論基礎" Propositions 1-2) and step 3's compilation into
  token / parent / depth / position / ancestor-mask tensors;
* :func:`tree_attn`  -- step 3, ancestor-only masked attention of each
  tree row against the context KV cache and the tree's own KV;
* :func:`tree_walk`  -- step 4, the greedy walk that accepts matching
  children and returns the bonus token;
* :func:`lm_head_argmax`, :func:`walk_row_tokens` -- step 4 from the target's
  hidden states and LM-head weights: each row's logits as an fp64 matmul,
  its argmax (lowest id on ties), and the walk over those row tokens;
* :func:`kv_commit`  -- after step 4: the root and the accepted rows' K/V
  appended to the committed context, which grows by acc_len + 1;
* :func:`plan_budget` -- after step 2: the node budget of every sequence of
  a batch that maximises the round's expected emitted tokens per unit of
  cost ("實驗結果與權衡": acceptance grows with B, so does the verifier's
  cost; Proposition 1);
* :func:`tree_walk_sample` -- step 4 under a sampling decoding rule
  (temperature > 0): each visited row draws its token from softmax(z / T)
  by inversion with a Philox4x64-10 uniform (:func:`philox4x64_10`,
  :func:`row_uniform`, :func:`sample_row`).

Parity pins for every function live in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ddt_oracle.c")
_LIB = os.path.join(_HERE, "libddt_oracle.so")
_lib = None

i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
u32p = np.ctypeslib.ndpointer(dtype=np.uint32, flags="C_CONTIGUOUS")
f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction, plain -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.ddto_topk.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int64, ctypes.c_int, ctypes.c_double,
                                  i32p, f64p, f64p, f64p]
        lib.ddto_build_tree.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_double, i32p, f64p, f64p, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_int, ctypes.c_int,
                                        i32p, i32p, i32p, i32p, u32p,
                                        ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_double),
                                        ctypes.POINTER(ctypes.c_double)]
        lib.ddto_tree_attn.argtypes = [ctypes.c_int, i32p, ctypes.c_void_p, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                       ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                       i32p, ctypes.c_void_p, ctypes.c_void_p, u32p,
                                       ctypes.c_int, i32p, ctypes.c_double, f64p, f64p]
        lib.ddto_tree_walk.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                       ctypes.c_int, i32p, i32p, i32p, ctypes.c_int,
                                       ctypes.c_int, ctypes.POINTER(ctypes.c_int32),
                                       i32p, i32p, ctypes.POINTER(ctypes.c_int32)]
        u64p = np.ctypeslib.ndpointer(dtype=np.uint64, flags="C_CONTIGUOUS")
        lib.ddto_philox4x64_10.argtypes = [u64p, u64p, u64p]
        lib.ddto_philox4x64_10.restype = None
        lib.ddto_word_to_uniform.argtypes = [ctypes.c_uint64]
        lib.ddto_word_to_uniform.restype = ctypes.c_double
        lib.ddto_row_uniform.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int,
                                         ctypes.c_int]
        lib.ddto_row_uniform.restype = ctypes.c_double
        lib.ddto_sample_row.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                        ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                        ctypes.POINTER(ctypes.c_double)]
        lib.ddto_sampler_row_weights.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_double, f64p]
        lib.ddto_sampler_row_weights.restype = ctypes.c_int
        lib.ddto_tree_walk_sample.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                              ctypes.c_int, i32p, i32p, i32p, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_double, ctypes.c_uint64,
                                              ctypes.c_uint64, ctypes.c_int,
                                              ctypes.POINTER(ctypes.c_int32), i32p, i32p,
                                              ctypes.POINTER(ctypes.c_int32),
                                              ctypes.POINTER(ctypes.c_double)]
        lib.ddto_kv_commit.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32),
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                       ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.ddto_kv_commit.restype = ctypes.c_int
        lib.ddto_walk_row_tokens.argtypes = [i32p, i32p, i32p, i32p, ctypes.c_int, ctypes.c_int,
                                             ctypes.POINTER(ctypes.c_int32), i32p, i32p,
                                             ctypes.POINTER(ctypes.c_int32)]
        lib.ddto_walk_row_tokens.restype = ctypes.c_int
        lib.ddto_plan_budget.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_double, i32p, f64p, f64p, i32p, i32p, i32p,
                                         i32p, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                         i32p, f64p, ctypes.POINTER(ctypes.c_int32)]
        lib.ddto_plan_budget.restype = ctypes.c_int
        for f in (lib.ddto_topk, lib.ddto_build_tree, lib.ddto_tree_attn, lib.ddto_tree_walk,
                  lib.ddto_sample_row, lib.ddto_tree_walk_sample):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _raw(x: np.ndarray):
    """(pointer, is_bf16) for a bf16 (stored as uint16 bits) or float32 array."""
    if x.dtype == np.uint16:
        return x.ctypes.data_as(ctypes.c_void_p), 1
    if x.dtype == np.float32:
        return x.ctypes.data_as(ctypes.c_void_p), 0
    raise TypeError("logits must be bf16 bits (uint16) or float32, got %s" % x.dtype)


def topk(z: np.ndarray, k: int, inv_temperature: float = 1.0):
    """Step 1 for every row of ``z`` (shape [..., V], bf16 bits or f32).

    Returns ``ids`` int32 [..., k], ``zk`` f64 [..., k] (the raw logits of the
    candidates), ``logp`` f64 [..., k] = invT*z - lse and ``lse`` f64 [...].
    The order is logit descending, token id ascending.
    """
    z = np.ascontiguousarray(z)
    lead = z.shape[:-1]
    V = z.shape[-1]
    rows = int(np.prod(lead)) if lead else 1
    ids = np.empty(rows * k, np.int32)
    zk = np.empty(rows * k, np.float64)
    logp = np.empty(rows * k, np.float64)
    lse = np.empty(rows, np.float64)
    p, is_bf16 = _raw(z)
    rc = _load().ddto_topk(p, is_bf16, rows, V, V, k, float(np.float32(inv_temperature)),
                           ids, zk, logp, lse)
    if rc != 0:
        raise ValueError("ddto_topk failed (%d)" % rc)
    return (ids.reshape(*lead, k), zk.reshape(*lead, k), logp.reshape(*lead, k),
            lse.reshape(lead))


def mask_words(n_max: int) -> int:
    return (n_max + 31) // 32


def build_tree(ids, zk, lse, budget, inv_temperature=1.0, root_token=None, ctx_len=None,
               k_per_seq=None, n_max=None):
    """Steps 2-3 for a batch.

    ``ids``/``zk``: [batch, L, k] top-k ids and raw logits; ``lse``: [batch, L];
    ``budget``: int or [batch] draft-node budgets; ``k_per_seq``: optional
    [batch] number of candidates used per position (<= k).
    Returns a dict of numpy arrays: tok, parent, depth, pos [batch, Nmax],
    mask [batch, Nmax, W] uint32, n_nodes [batch], surrogate [batch],
    delta_min [batch].
    """
    ids = np.ascontiguousarray(ids, np.int32)
    zk = np.ascontiguousarray(zk, np.float64)
    lse = np.ascontiguousarray(lse, np.float64)
    bsz, L, kmax = ids.shape
    budget = np.broadcast_to(np.asarray(budget, np.int64), (bsz,))
    if k_per_seq is None:
        k_per_seq = np.full(bsz, kmax, np.int64)
    k_per_seq = np.broadcast_to(np.asarray(k_per_seq, np.int64), (bsz,))
    root_token = np.zeros(bsz, np.int64) if root_token is None else np.broadcast_to(
        np.asarray(root_token, np.int64), (bsz,))
    ctx_len = np.zeros(bsz, np.int64) if ctx_len is None else np.broadcast_to(
        np.asarray(ctx_len, np.int64), (bsz,))
    if n_max is None:
        n_max = int(budget.max()) + 1
    W = mask_words(n_max)
    out = {k_: np.empty((bsz, n_max), np.int32) for k_ in ("tok", "parent", "depth", "pos")}
    out["mask"] = np.empty((bsz, n_max, W), np.uint32)
    out["n_nodes"] = np.empty(bsz, np.int32)
    out["surrogate"] = np.empty(bsz, np.float64)
    out["delta_min"] = np.empty(bsz, np.float64)
    lib = _load()
    for b in range(bsz):
        t, p, dp, ps = (np.empty(n_max, np.int32) for _ in range(4))
        m = np.empty(n_max * W, np.uint32)
        nn = ctypes.c_int32()
        sg = ctypes.c_double()
        dm = ctypes.c_double()
        rc = lib.ddto_build_tree(L, int(k_per_seq[b]), kmax, int(budget[b]),
                                 float(np.float32(inv_temperature)),
                                 np.ascontiguousarray(ids[b]), np.ascontiguousarray(zk[b]),
                                 np.ascontiguousarray(lse[b]), int(root_token[b]),
                                 int(ctx_len[b]), n_max, W, t, p, dp, ps, m,
                                 ctypes.byref(nn), ctypes.byref(sg), ctypes.byref(dm))
        if rc != 0:
            raise ValueError("ddto_build_tree failed (%d) for sequence %d" % (rc, b))
        out["tok"][b], out["parent"][b], out["depth"][b], out["pos"][b] = t, p, dp, ps
        out["mask"][b] = m.reshape(n_max, W)
        out["n_nodes"][b] = nn.value
        out["surrogate"][b] = sg.value
        out["delta_min"][b] = dm.value
    return out


def tree_attn(items, q, k_cache, v_cache, ctx_len, k_tree, v_tree, mask, n_nodes, scale,
              page_table=None, page_size=64):
    """Step 3's attention for the listed (b, j, h) items.

    ``q`` [batch, Nmax, Hq, d], ``k_tree``/``v_tree`` [batch, Nmax, Hkv, d] and the
    cache are bf16 bits (uint16).  Dense cache: [batch, Tmax, Hkv, d]; paged
    cache: [pages, page_size, Hkv, d] with ``page_table`` [batch, max_pages].
    Returns (out f64 [n, d], lse f64 [n]).
    """
    items = np.ascontiguousarray(np.asarray(items, np.int32).reshape(-1, 3))
    for a in (q, k_cache, v_cache, k_tree, v_tree):
        if a.dtype != np.uint16 or not a.flags.c_contiguous:
            raise TypeError("attention operands must be C-contiguous bf16 bits (uint16)")
    bsz, n_max, hq, d = q.shape
    hkv = k_tree.shape[2]
    if page_table is None:
        tmax = k_cache.shape[1]
        pt = None
        maxp = 0
    else:
        tmax = 0
        pt = np.ascontiguousarray(page_table, np.int32)
        maxp = pt.shape[1]
    n = items.shape[0]
    out = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    W = mask.shape[-1]
    rc = _load().ddto_tree_attn(
        n, items, q.ctypes.data_as(ctypes.c_void_p), n_max, hq, hkv, d,
        k_cache.ctypes.data_as(ctypes.c_void_p), v_cache.ctypes.data_as(ctypes.c_void_p),
        tmax, None if pt is None else pt.ctypes.data_as(ctypes.c_void_p), page_size, maxp,
        np.ascontiguousarray(ctx_len, np.int32), k_tree.ctypes.data_as(ctypes.c_void_p),
        v_tree.ctypes.data_as(ctypes.c_void_p), np.ascontiguousarray(mask, np.uint32), W,
        np.ascontiguousarray(n_nodes, np.int32), float(scale), out, lse)
    if rc != 0:
        raise ValueError("ddto_tree_attn failed (%d)" % rc)
    return out, lse


def tree_walk(logits, tok, parent, depth, n_nodes, L):
    """Step 4 for a batch.  ``logits`` [batch, Nmax, V] f32 or bf16 bits.

    Returns a dict: acc_len [batch], acc_nodes/acc_tok [batch, L], bonus [batch].
    """
    logits = np.ascontiguousarray(logits)
    bsz, n_max, V = logits.shape
    res = {"acc_len": np.empty(bsz, np.int32), "acc_nodes": np.empty((bsz, L), np.int32),
           "acc_tok": np.empty((bsz, L), np.int32), "bonus": np.empty(bsz, np.int32)}
    lib = _load()
    for b in range(bsz):
        row = np.ascontiguousarray(logits[b])
        p, is_bf16 = _raw(row)
        al = ctypes.c_int32()
        bo = ctypes.c_int32()
        an = np.empty(max(L, 1), np.int32)
        at = np.empty(max(L, 1), np.int32)
        rc = lib.ddto_tree_walk(p, is_bf16, V, V, np.ascontiguousarray(tok[b], np.int32),
                                np.ascontiguousarray(parent[b], np.int32),
                                np.ascontiguousarray(depth[b], np.int32), int(n_nodes[b]), L,
                                ctypes.byref(al), an, at, ctypes.byref(bo))
        if rc != 0:
            raise ValueError("ddto_tree_walk failed (%d)" % rc)
        res["acc_len"][b] = al.value
        res["acc_nodes"][b] = an[:L]
        res["acc_tok"][b] = at[:L]
        res["bonus"][b] = bo.value
    return res


def philox4x64_10(ctr, key) -> np.ndarray:
    """Philox4x64-10 block at counter ``ctr`` (4 words) under ``key`` (2 words)."""
    out = np.zeros(4, np.uint64)
    _load().ddto_philox4x64_10(np.ascontiguousarray(ctr, np.uint64),
                               np.ascontiguousarray(key, np.uint64), out)
    return out


def word_to_uniform(w: int) -> float:
    """A 64-bit word to a uniform in (0, 1) (top 53 bits, centred)."""
    return float(_load().ddto_word_to_uniform(int(w)))


def row_uniform(seed: int, step: int, b: int, j: int) -> float:
    """The uniform that tree row ``j`` of sequence ``b`` draws in round ``step``."""
    return float(_load().ddto_row_uniform(int(seed), int(step), int(b), int(j)))


def _f32(x: float) -> float:
    """The fp32 value of a temperature argument (the C ABI takes a float)."""
    return float(np.float32(x))


def sampler_row_weights(row: np.ndarray, inv_temperature: float) -> np.ndarray:
    """The draw's weights of one row: w_v = exp(invT * z_v - max_u invT * z_u)
    in fp64 (0 for -inf logits), invT being the fp32 value of the argument."""
    row = np.ascontiguousarray(row)
    p, is_bf16 = _raw(row)
    w = np.empty(row.shape[-1], np.float64)
    rc = _load().ddto_sampler_row_weights(p, is_bf16, row.shape[-1], _f32(inv_temperature), w)
    if rc != 0:
        raise ValueError("ddto_sampler_row_weights failed (%d)" % rc)
    return w


def sample_row(row: np.ndarray, inv_temperature: float, u: float):
    """One inverse-CDF draw from softmax(inv_temperature * row) (fp64 weights
    of :func:`sampler_row_weights`).  Returns (token, margin), margin =
    distance of u*S from the chosen interval's nearer end over S."""
    row = np.ascontiguousarray(row)
    p, is_bf16 = _raw(row)
    mg = ctypes.c_double()
    t = _load().ddto_sample_row(p, is_bf16, 0, row.shape[-1], _f32(inv_temperature), float(u),
                                ctypes.byref(mg))
    return int(t), float(mg.value)


def tree_walk_sample(logits, tok, parent, depth, n_nodes, L, inv_temperature, seed, step):
    """Step 4 under sampling for a batch.  Same outputs as :func:`tree_walk`
    plus ``min_margin`` [batch], the smallest draw margin along each walk."""
    logits = np.ascontiguousarray(logits)
    bsz, n_max, V = logits.shape
    res = {"acc_len": np.empty(bsz, np.int32), "acc_nodes": np.empty((bsz, L), np.int32),
           "acc_tok": np.empty((bsz, L), np.int32), "bonus": np.empty(bsz, np.int32),
           "min_margin": np.empty(bsz, np.float64)}
    lib = _load()
    for b in range(bsz):
        row = np.ascontiguousarray(logits[b])
        p, is_bf16 = _raw(row)
        al = ctypes.c_int32()
        bo = ctypes.c_int32()
        mm = ctypes.c_double()
        an = np.empty(max(L, 1), np.int32)
        at = np.empty(max(L, 1), np.int32)
        rc = lib.ddto_tree_walk_sample(p, is_bf16, V, V, np.ascontiguousarray(tok[b], np.int32),
                                       np.ascontiguousarray(parent[b], np.int32),
                                       np.ascontiguousarray(depth[b], np.int32), int(n_nodes[b]),
                                       L, _f32(inv_temperature), int(seed), int(step), b,
                                       ctypes.byref(al), an, at, ctypes.byref(bo),
                                       ctypes.byref(mm))
        if rc != 0:
            raise ValueError("ddto_tree_walk_sample failed (%d)" % rc)
        res["acc_len"][b] = al.value
        res["acc_nodes"][b] = an[:L]
        res["acc_tok"][b] = at[:L]
        res["bonus"][b] = bo.value
        res["min_margin"][b] = mm.value
    return res


def kv_commit(k_tree, v_tree, acc_len, acc_nodes, ctx_len, k_cache, v_cache, page_table=None,
              page_size=64, num_pages=0):
    """Append each sequence's root and accepted rows of the tree K/V to the
    cache (in place on copies) and advance ctx_len by acc_len + 1.

    ``k_tree``/``v_tree`` bf16 bits (uint16) [batch, n_max, hkv, d]; the
    cache is dense [batch, t_max, hkv, d] (``page_table`` None) or a page pool
    [pages, page_size, hkv, d].  Returns (k_cache, v_cache, ctx_len, ok) with
    ok[b] False where a position fell outside the cache.
    """
    kt = np.ascontiguousarray(k_tree, np.uint16)
    vt = np.ascontiguousarray(v_tree, np.uint16)
    kc = np.array(k_cache, np.uint16, copy=True, order="C")
    vc = np.array(v_cache, np.uint16, copy=True, order="C")
    bsz, n_max, hkv, d = kt.shape
    cl = np.array(ctx_len, np.int32, copy=True)
    ok = np.ones(bsz, bool)
    lib = _load()
    for b in range(bsz):
        a = int(acc_len[b])
        nodes = np.ascontiguousarray(np.asarray(acc_nodes[b], np.int32)[:max(a, 1)])
        c = ctypes.c_int32(int(cl[b]))
        if page_table is None:
            kb, vb = kc[b], vc[b]
            t_max, pages, maxp = kb.shape[0], None, 0
        else:
            kb, vb = kc, vc
            t_max = 0
            pages = np.ascontiguousarray(page_table[b], np.int32)
            maxp = pages.shape[0]
        rc = lib.ddto_kv_commit(kt[b].ctypes.data_as(ctypes.c_void_p),
                                vt[b].ctypes.data_as(ctypes.c_void_p), n_max, hkv, d, a,
                                nodes.ctypes.data_as(ctypes.c_void_p), ctypes.byref(c),
                                kb.ctypes.data_as(ctypes.c_void_p),
                                vb.ctypes.data_as(ctypes.c_void_p), t_max,
                                None if pages is None else pages.ctypes.data_as(ctypes.c_void_p),
                                page_size, maxp, num_pages)
        ok[b] = rc == 0
        cl[b] = c.value
    return kc, vc, cl, ok


def _bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def lm_head_argmax(hidden, weight, block=None):
    """The target's decision at each row: logits = H W^T with every product
    and sum in fp64 (the products of bf16 values are exact), argmax with the
    lowest token id on ties.

    ``hidden`` bf16 bits [rows, K], ``weight`` bf16 bits [V, K].  Returns
    (token [rows] int32, top [rows] f64, gap [rows] f64): gap = top logit
    minus the largest logit of any other token (0 on a tie).  ``block``
    bounds the vocabulary rows widened to fp64 at a time (memory only: every
    logit is its own dot product, and the running top two keep the first
    occurrence)."""
    h = _bf16_to_f64(hidden)
    rows, V = h.shape[0], weight.shape[0]
    block = V if block is None else block
    top = np.full(rows, -np.inf)
    second = np.full(rows, -np.inf)
    tok = np.zeros(rows, np.int32)
    for v0 in range(0, V, block):
        logits = h @ _bf16_to_f64(weight[v0:v0 + block]).T
        bt = np.argmax(logits, axis=1)  # first occurrence: lowest id within the block
        bv = logits[np.arange(rows), bt]
        rest = logits.copy()
        rest[np.arange(rows), bt] = -np.inf
        b2 = rest.max(axis=1) if logits.shape[1] > 1 else np.full(rows, -np.inf)
        new = bv > top  # strictly larger: an earlier block keeps its equal maximum
        second = np.where(new, np.maximum(top, b2), np.maximum(second, bv))
        top = np.where(new, bv, top)
        tok = np.where(new, bt + v0, tok).astype(np.int32)
    gap = top - second
    return tok, top, gap


def walk_row_tokens(row_tok, tok, parent, depth, n_nodes, L):
    """Step 4 over given row tokens [batch, n_max]; outputs as :func:`tree_walk`."""
    row_tok = np.ascontiguousarray(row_tok, np.int32)
    bsz = row_tok.shape[0]
    res = {"acc_len": np.empty(bsz, np.int32), "acc_nodes": np.empty((bsz, L), np.int32),
           "acc_tok": np.empty((bsz, L), np.int32), "bonus": np.empty(bsz, np.int32)}
    lib = _load()
    for b in range(bsz):
        al = ctypes.c_int32()
        bo = ctypes.c_int32()
        an = np.empty(max(L, 1), np.int32)
        at = np.empty(max(L, 1), np.int32)
        rc = lib.ddto_walk_row_tokens(np.ascontiguousarray(row_tok[b]),
                                      np.ascontiguousarray(tok[b], np.int32),
                                      np.ascontiguousarray(parent[b], np.int32),
                                      np.ascontiguousarray(depth[b], np.int32), int(n_nodes[b]), L,
                                      ctypes.byref(al), an, at, ctypes.byref(bo))
        if rc != 0:
            raise ValueError("ddto_walk_row_tokens failed (%d)" % rc)
        res["acc_len"][b] = al.value
        res["acc_nodes"][b] = an[:L]
        res["acc_tok"][b] = at[:L]
        res["bonus"][b] = bo.value
    return res


def plan_budget(ids, zk, lse, tree, L, inv_temperature, total_budget=-1, cost_fixed=0.0,
                cost_per_node=0.0):
    """Node budgets across a batch from trees built with each sequence's
    largest budget (``tree``: dict with tok, parent, depth, n_nodes);
    ``total_budget`` < 0: no cap on the nodes taken.
    ``ids``/``zk`` [batch, L, k], ``lse`` [batch, L].  Returns (budget int32
    [batch], expected_tokens f64 [batch], n_taken)."""
    ids = np.ascontiguousarray(ids, np.int32)
    zk = np.ascontiguousarray(zk, np.float64)
    lse = np.ascontiguousarray(lse, np.float64)
    bsz, Lx, kk = ids.shape
    n_max = tree["tok"].shape[1]
    budget = np.empty(bsz, np.int32)
    exp_tok = np.empty(bsz, np.float64)
    taken = ctypes.c_int32()
    rc = _load().ddto_plan_budget(bsz, L, kk, n_max, _f32(inv_temperature), ids, zk, lse,
                                  np.ascontiguousarray(tree["tok"], np.int32),
                                  np.ascontiguousarray(tree["parent"], np.int32),
                                  np.ascontiguousarray(tree["depth"], np.int32),
                                  np.ascontiguousarray(tree["n_nodes"], np.int32),
                                  int(total_budget), float(cost_fixed), float(cost_per_node),
                                  budget, exp_tok, ctypes.byref(taken))
    if rc != 0:
        raise ValueError("ddto_plan_budget failed (%d)" % rc)
    return budget, exp_tok, int(taken.value)
