"""ctypes binding of libddt.so (argument marshalling only).

Every function here checks shapes and dtypes, allocates the output tensors
with torch on the input's device, and calls the matching C entry point of
``include/ddt.h`` on the current torch stream.  All arithmetic happens in the
library's CUDA kernels; if ``libddt.so`` is missing or fails to load, every
call raises :class:`DDTError` -- there is no other implementation.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libddt.so")
_lib = None
_lock = threading.Lock()

DDT_BF16, DDT_F32 = 0, 1
DDT_TOPK_K_MAX = 32
DDT_TREE_L_MAX = 64
DDT_TREE_B_MAX = 1023

EXPORTED = ("ddt_status_string", "ddt_mask_words", "ddt_topk_workspace_size", "ddt_topk",
            "ddt_build_tree", "ddt_tree_attn_workspace_size", "ddt_tree_attn",
            "ddt_tree_walk_workspace_size", "ddt_tree_walk", "ddt_tree_walk_sample",
            "ddt_kv_commit", "ddt_lm_head_max_rows", "ddt_lm_head_walk_workspace_size",
            "ddt_lm_head_walk", "ddt_tree_attn_plan", "ddt_debug_set_wait_limit",
            "ddt_topk_noalloc", "ddt_tree_walk_resolve_mode", "ddt_plan_budget",
            "ddt_debug_set_attn_kernel")

# ddt_tree_walk's modes
WALK_ALL_ROWS, WALK_LAZY, WALK_AUTO = 0, 1, 2

# ddt_tree_attn_plan's paths
ATTN_PATH_SIMT, ATTN_PATH_TC, ATTN_PATH_TC_CLUSTER, ATTN_PATH_TC_COMBINE = 0, 1, 2, 3
ATTN_PATH_TC_PAIRS, ATTN_PATH_TC_PAIRS_COMBINE = 4, 5


class KVCommitArgs(ctypes.Structure):
    """Mirror of ``ddt_kv_commit_args`` (field order and types as in ddt.h)."""
    _fields_ = [("k_tree", ctypes.c_void_p), ("v_tree", ctypes.c_void_p),
                ("acc_len", ctypes.c_void_p), ("acc_nodes", ctypes.c_void_p),
                ("ctx_len", ctypes.c_void_p), ("k_cache", ctypes.c_void_p),
                ("v_cache", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
                ("page_size", ctypes.c_int), ("max_pages", ctypes.c_int),
                ("num_pages", ctypes.c_int), ("t_max", ctypes.c_int64),
                ("batch", ctypes.c_int), ("n_max", ctypes.c_int), ("hkv", ctypes.c_int),
                ("d", ctypes.c_int), ("L", ctypes.c_int), ("dev_status", ctypes.c_void_p)]


class LmHeadWalkArgs(ctypes.Structure):
    """Mirror of ``ddt_lm_head_walk_args`` (field order and types as in ddt.h)."""
    _fields_ = [("hidden", ctypes.c_void_p), ("weight", ctypes.c_void_p), ("K", ctypes.c_int),
                ("V", ctypes.c_int), ("tok", ctypes.c_void_p), ("parent", ctypes.c_void_p),
                ("depth", ctypes.c_void_p), ("n_nodes", ctypes.c_void_p), ("batch", ctypes.c_int),
                ("n_max", ctypes.c_int), ("L", ctypes.c_int), ("acc_len", ctypes.c_void_p),
                ("acc_nodes", ctypes.c_void_p), ("acc_tok", ctypes.c_void_p),
                ("bonus", ctypes.c_void_p), ("row_token", ctypes.c_void_p),
                ("dev_status", ctypes.c_void_p)]


class DDTError(RuntimeError):
    """A libddt call returned an error status (or the library is unavailable)."""


class AttnArgs(ctypes.Structure):
    """Mirror of ``ddt_attn_args`` (field order and types as in ddt.h)."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p), ("page_size", ctypes.c_int), ("max_pages", ctypes.c_int),
        ("num_pages", ctypes.c_int),
        ("t_max", ctypes.c_int64), ("ctx_len", ctypes.c_void_p), ("max_ctx", ctypes.c_int),
        ("k_tree", ctypes.c_void_p), ("v_tree", ctypes.c_void_p), ("mask", ctypes.c_void_p),
        ("n_nodes", ctypes.c_void_p), ("batch", ctypes.c_int), ("n_max", ctypes.c_int),
        ("hq", ctypes.c_int), ("hkv", ctypes.c_int), ("d", ctypes.c_int),
        ("scale", ctypes.c_float), ("out", ctypes.c_void_p), ("lse_out", ctypes.c_void_p),
        ("dev_status", ctypes.c_void_p),
    ]


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libddt.so (once).  Raises DDTError if it is missing or broken."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise DDTError("libddt.so is not built (python -m block_draft_tree_b200.build)")
        try:
            lib = ctypes.CDLL(_LIB_PATH)
        except OSError as e:  # pragma: no cover - depends on the machine
            raise DDTError("cannot load %s: %s" % (_LIB_PATH, e)) from e
        vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                                 ctypes.c_size_t)
        lib.ddt_status_string.restype = ctypes.c_char_p
        lib.ddt_status_string.argtypes = [i32]
        lib.ddt_mask_words.restype = i32
        lib.ddt_mask_words.argtypes = [i32]
        lib.ddt_topk_workspace_size.restype = sz
        lib.ddt_topk_workspace_size.argtypes = [i32, i32, i32, i32]
        lib.ddt_topk.restype = i32
        lib.ddt_topk.argtypes = [vp, i32, i32, i32, i32, i64, i32, f32, vp, vp, vp, vp, vp, sz, vp]
        lib.ddt_build_tree.restype = i32
        lib.ddt_build_tree.argtypes = [vp, vp, vp, i32, i32, i32, f32, vp, vp, i32, vp, vp,
                                       vp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.ddt_tree_attn_workspace_size.restype = sz
        lib.ddt_tree_attn_workspace_size.argtypes = [ctypes.POINTER(AttnArgs)]
        lib.ddt_tree_attn.restype = i32
        lib.ddt_tree_attn.argtypes = [ctypes.POINTER(AttnArgs), vp, sz, vp]
        lib.ddt_tree_attn_plan.restype = i32
        lib.ddt_tree_attn_plan.argtypes = [ctypes.POINTER(AttnArgs), ctypes.POINTER(i32),
                                           ctypes.POINTER(i32)]
        lib.ddt_debug_set_wait_limit.restype = ctypes.c_longlong
        lib.ddt_debug_set_wait_limit.argtypes = [ctypes.c_longlong]
        lib.ddt_debug_set_attn_kernel.restype = ctypes.c_int
        lib.ddt_debug_set_attn_kernel.argtypes = [ctypes.c_int]
        lib.ddt_tree_walk_workspace_size.restype = sz
        lib.ddt_tree_walk_workspace_size.argtypes = [i32, i32, i32]
        lib.ddt_tree_walk.restype = i32
        lib.ddt_tree_walk.argtypes = [vp, i32, i32, i32, i32, i64, vp, vp, vp, vp, i32, i32,
                                      vp, vp, vp, vp, vp, sz, vp, vp]
        lib.ddt_plan_budget.restype = i32
        lib.ddt_plan_budget.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32,
                                        ctypes.c_double, ctypes.c_double, vp, vp, vp, vp]
        lib.ddt_tree_walk_resolve_mode.restype = i32
        lib.ddt_tree_walk_resolve_mode.argtypes = [i32, i32, i32, i32, i32, i32]
        lib.ddt_lm_head_max_rows.restype = i32
        lib.ddt_lm_head_max_rows.argtypes = []
        lib.ddt_lm_head_walk_workspace_size.restype = sz
        lib.ddt_lm_head_walk_workspace_size.argtypes = [ctypes.POINTER(LmHeadWalkArgs)]
        lib.ddt_lm_head_walk.restype = i32
        lib.ddt_lm_head_walk.argtypes = [ctypes.POINTER(LmHeadWalkArgs), vp, sz, vp]
        lib.ddt_kv_commit.restype = i32
        lib.ddt_kv_commit.argtypes = [ctypes.POINTER(KVCommitArgs), vp]
        u64 = ctypes.c_uint64
        lib.ddt_tree_walk_sample.restype = i32
        lib.ddt_tree_walk_sample.argtypes = [vp, i32, i32, i32, i32, i64, vp, vp, vp, vp, i32,
                                             f32, u64, u64, vp, vp, vp, vp, vp, vp, sz, vp, vp]
        _lib = lib
        return lib


def _check(rc: int, what: str):
    if rc != 0:
        msg = load_library().ddt_status_string(rc).decode()
        raise DDTError("%s failed: %s" % (what, msg))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need_cuda(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise DDTError("libddt works on CUDA tensors only (got a %s tensor)" % t.device)
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise DDTError("all tensors must be on one device")
    return dev


def _check_types(fn: str, *pairs):
    """Raise unless every given tensor (None skipped) is contiguous with its
    dtype: the kernels read plain int32 / float32 arrays."""
    for t, dt in pairs:
        if t is not None and (t.dtype != dt or not t.is_contiguous()):
            raise DDTError("%s: expected contiguous %s tensors, got %s" % (fn, dt, t.dtype))


def _check_tree_shapes(fn: str, b: int, n_max: int, tok, parent, depth, n_nodes):
    """Raise unless tok/parent/depth are [b, n_max] and n_nodes is [b]: the
    kernels index them with those extents."""
    for t in (tok, parent, depth):
        if tuple(t.shape) != (b, n_max):
            raise DDTError("%s: tree tensors must be [%d, %d], got %s"
                           % (fn, b, n_max, tuple(t.shape)))
    if tuple(n_nodes.shape) != (b,):
        raise DDTError("%s: n_nodes must be [%d], got %s" % (fn, b, tuple(n_nodes.shape)))


def _check_kv_shapes(fn: str, b: int, n_max: int, d: int, k_tree, v_tree, k_cache, v_cache,
                     page_table, page_size=None):
    """Raise unless the tree K/V are [b, n_max, hkv, d] and a non-empty cache
    is dense [b, t_max, hkv, d] or, with ``page_table`` [b, max_pages], a page
    pool [pages, page_size, hkv, d]: the kernels index them with those
    extents.  Returns hkv."""
    if k_tree.dim() != 4 or tuple(k_tree.shape[:2]) != (b, n_max) or k_tree.shape[3] != d:
        raise DDTError("%s: tree K must be [%d, %d, hkv, %d], got %s"
                       % (fn, b, n_max, d, tuple(k_tree.shape)))
    if v_tree.shape != k_tree.shape:
        raise DDTError("%s: tree V must have tree K's shape" % fn)
    hkv = k_tree.shape[2]
    if k_cache is not None and k_cache.numel():
        if v_cache is None or v_cache.shape != k_cache.shape:
            raise DDTError("%s: the V cache must have the K cache's shape" % fn)
        if k_cache.dim() != 4 or tuple(k_cache.shape[2:]) != (hkv, d):
            raise DDTError("%s: caches must be [.., .., %d, %d], got %s"
                           % (fn, hkv, d, tuple(k_cache.shape)))
        if page_table is None and k_cache.shape[0] != b:
            raise DDTError("%s: a dense cache must have %d sequences" % (fn, b))
        if page_table is not None:
            if page_table.dim() != 2 or page_table.shape[0] != b:
                raise DDTError("%s: page_table must be [%d, max_pages]" % (fn, b))
            if page_size is not None and k_cache.shape[1] != page_size:
                raise DDTError("%s: the page pool's pages hold %d tokens, page_size is %d"
                               % (fn, k_cache.shape[1], page_size))
    return hkv


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DDT_BF16
    if t.dtype == torch.float32:
        return DDT_F32
    raise DDTError("logits must be bfloat16 or float32, got %s" % t.dtype)


class _Workspaces:
    """Zero-filled scratch per (device, stream, stage); grown on demand.

    The kernels return every counter they use to zero, so a workspace stays
    valid across calls that do not overlap on the GPU (same stream)."""

    def __init__(self):
        self._bufs = {}

    def get(self, dev: torch.device, tag: str, nbytes: int) -> Optional[torch.Tensor]:
        if nbytes == 0:
            return None
        key = (dev, torch.cuda.current_stream(dev).cuda_stream, tag)
        buf = self._bufs.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
            self._bufs[key] = buf
        return buf


workspaces = _Workspaces()


def topk_workspace_size(batch: int, L: int, V: int, k: int) -> int:
    return int(load_library().ddt_topk_workspace_size(batch, L, V, k))


def topk(logits: torch.Tensor, k: int, inv_temperature: float = 1.0, want_logp: bool = True):
    """Stage 1.  ``logits`` [batch, L, V] bf16/f32 with unit stride on V and a
    uniform row stride.  Returns (ids int32, zk f32, logp f32 or None) [batch, L, k]
    and lse f32 [batch, L]."""
    lib = load_library()
    dev = _need_cuda(logits)
    if logits.dim() != 3 or logits.stride(2) != 1 or logits.stride(0) != logits.stride(1) * logits.shape[1]:
        raise DDTError("logits must be [batch, L, V] with contiguous rows and a uniform row stride")
    b, L, V = logits.shape
    ids = torch.empty((b, L, k), dtype=torch.int32, device=dev)
    zk = torch.empty((b, L, k), dtype=torch.float32, device=dev)
    logp = torch.empty((b, L, k), dtype=torch.float32, device=dev) if want_logp else None
    lse = torch.empty((b, L), dtype=torch.float32, device=dev)
    nb = int(lib.ddt_topk_workspace_size(b, L, V, k))
    ws = workspaces.get(dev, "topk", nb)
    with torch.cuda.device(dev):
        rc = lib.ddt_topk(_ptr(logits), _dtype_code(logits), b, L, V, logits.stride(1), k,
                          float(inv_temperature), _ptr(ids), _ptr(zk), _ptr(logp), _ptr(lse),
                          _ptr(ws), nb, _stream(dev))
    _check(rc, "ddt_topk")
    return ids, zk, logp, lse


def mask_words(n_max: int) -> int:
    return (n_max + 31) // 32


def build_tree(ids: torch.Tensor, zk: torch.Tensor, lse: torch.Tensor, B_max: int,
               root_token: torch.Tensor, inv_temperature: float = 1.0,
               k_per_seq: Optional[torch.Tensor] = None, budget: Optional[torch.Tensor] = None,
               ctx_len: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None):
    """Stages 2-3 (selection and compilation).  Returns a dict of tensors:
    tok, parent, depth, pos [batch, B_max+1] int32, mask [batch, B_max+1, W]
    int32 (bit pattern of the uint32 words), n_nodes [batch] int32,
    surrogate [batch] float64."""
    lib = load_library()
    if ids.dim() != 3 or zk.shape != ids.shape or lse.shape != ids.shape[:2]:
        raise DDTError("build_tree: ids/zk must be [batch, L, k] and lse [batch, L]")
    for t in (root_token, k_per_seq, budget, ctx_len):
        if t is not None and tuple(t.shape) != (ids.shape[0],):
            raise DDTError("build_tree: root_token / k_per_seq / budget / ctx_len must be [%d]"
                           % ids.shape[0])
    dev = _need_cuda(ids, zk, lse, root_token, k_per_seq, budget, ctx_len, dev_status)
    for t, dt in ((ids, torch.int32), (zk, torch.float32), (lse, torch.float32),
                  (root_token, torch.int32), (k_per_seq, torch.int32), (budget, torch.int32),
                  (ctx_len, torch.int32), (dev_status, torch.int32)):
        if t is not None and (t.dtype != dt or not t.is_contiguous()):
            raise DDTError("build_tree: expected contiguous %s tensors" % dt)
    b, L, k = ids.shape
    n_max = B_max + 1
    W = mask_words(n_max)
    out = {n: torch.empty((b, n_max), dtype=torch.int32, device=dev)
           for n in ("tok", "parent", "depth", "pos")}
    out["mask"] = torch.empty((b, n_max, W), dtype=torch.int32, device=dev)
    out["n_nodes"] = torch.empty(b, dtype=torch.int32, device=dev)
    out["surrogate"] = torch.empty(b, dtype=torch.float64, device=dev)
    with torch.cuda.device(dev):
        rc = lib.ddt_build_tree(_ptr(ids), _ptr(zk), _ptr(lse), b, L, k, float(inv_temperature),
                                _ptr(k_per_seq), _ptr(budget), B_max, _ptr(root_token),
                                _ptr(ctx_len), _ptr(out["tok"]), _ptr(out["parent"]),
                                _ptr(out["depth"]), _ptr(out["pos"]), _ptr(out["mask"]),
                                _ptr(out["n_nodes"]), _ptr(out["surrogate"]), _ptr(dev_status),
                                _stream(dev))
    _check(rc, "ddt_build_tree")
    return out


def plan_budget(tree: dict, ids: torch.Tensor, zk: torch.Tensor, lse: torch.Tensor,
                inv_temperature: float = 1.0, total_budget: int = -1, cost_fixed: float = 0.0,
                cost_per_node: float = 0.0, dev_status: Optional[torch.Tensor] = None):
    """``ddt_plan_budget``: each sequence's share of the batch's node budget,
    from ``tree`` (tok, parent, depth, n_nodes of a build with the largest
    budgets) and the candidates ``ids``/``zk`` [batch, L, k], ``lse`` [batch, L]
    it was built from.  Returns (budget int32 [batch], expected_tokens f64
    [batch]); pass ``budget`` to :func:`build_tree` as its per-sequence budget."""
    lib = load_library()
    _check_types("plan_budget", *[(tree[n], torch.int32) for n in ("tok", "parent", "depth",
                                                                   "n_nodes")],
                 (ids, torch.int32), (zk, torch.float32), (lse, torch.float32),
                 (dev_status, torch.int32))
    if ids.dim() != 3 or zk.shape != ids.shape or lse.shape != ids.shape[:2] or tree["tok"].dim() != 2:
        raise DDTError("plan_budget: ids/zk must be [batch, L, k], lse [batch, L], tree [batch, n_max]")
    b, L, k = ids.shape
    n_max = tree["tok"].shape[1]
    _check_tree_shapes("plan_budget", b, n_max, tree["tok"], tree["parent"], tree["depth"],
                       tree["n_nodes"])
    dev = _need_cuda(ids, zk, lse, tree["tok"], tree["parent"], tree["depth"], tree["n_nodes"],
                     dev_status)
    budget = torch.empty(b, dtype=torch.int32, device=dev)
    exp_tok = torch.empty(b, dtype=torch.float64, device=dev)
    with torch.cuda.device(dev):
        rc = lib.ddt_plan_budget(_ptr(tree["tok"]), _ptr(tree["parent"]), _ptr(tree["depth"]),
                                 _ptr(tree["n_nodes"]), _ptr(ids), _ptr(zk), _ptr(lse), b, L, k,
                                 n_max, float(inv_temperature), int(total_budget),
                                 float(cost_fixed), float(cost_per_node), _ptr(budget),
                                 _ptr(exp_tok), _ptr(dev_status), _stream(dev))
    _check(rc, "ddt_plan_budget")
    return budget, exp_tok


def _attn_args(q, k_cache, v_cache, k_tree, v_tree, mask, n_nodes, ctx_len, max_ctx, scale,
               page_table, out, lse_out, dev_status) -> AttnArgs:
    b, n_max, hq, d = q.shape
    hkv = k_tree.shape[2]
    a = AttnArgs()
    a.q = q.data_ptr()
    a.k_cache = k_cache.data_ptr() if k_cache is not None and k_cache.numel() else None
    a.v_cache = v_cache.data_ptr() if v_cache is not None and v_cache.numel() else None
    if page_table is not None:
        a.page_table = page_table.data_ptr()
        a.page_size = k_cache.shape[1]
        a.max_pages = page_table.shape[1]
        a.num_pages = k_cache.shape[0]
        a.t_max = 0
    else:
        a.page_table = None
        a.page_size = 0
        a.max_pages = 0
        a.num_pages = 0
        a.t_max = k_cache.shape[1] if k_cache is not None else 0
    a.ctx_len = ctx_len.data_ptr()
    a.max_ctx = int(max_ctx)
    a.k_tree = k_tree.data_ptr()
    a.v_tree = v_tree.data_ptr()
    a.mask = mask.data_ptr()
    a.n_nodes = n_nodes.data_ptr()
    a.batch, a.n_max, a.hq, a.hkv, a.d = b, n_max, hq, hkv, d
    a.scale = float(scale)
    a.out = out.data_ptr() if out is not None else None
    a.lse_out = lse_out.data_ptr() if lse_out is not None else None
    a.dev_status = dev_status.data_ptr() if dev_status is not None else None
    return a


def tree_attn_workspace_size(q, k_cache, v_cache, k_tree, v_tree, mask, n_nodes, ctx_len,
                             max_ctx, scale=None, page_table=None) -> int:
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    # the output pointer only has to be valid for the argument check: q stands in
    a = _attn_args(q, k_cache, v_cache, k_tree, v_tree, mask, n_nodes, ctx_len, max_ctx, scale,
                   page_table, q, None, None)
    return int(load_library().ddt_tree_attn_workspace_size(ctypes.byref(a)))


def tree_attn_plan(q, k_cache, v_cache, k_tree, v_tree, mask, n_nodes, ctx_len, max_ctx,
                   scale=None, page_table=None):
    """``ddt_tree_attn_plan``: (path, kv_splits) that :func:`tree_attn` would
    use for these arguments on the current device (one of the ATTN_PATH_*)."""
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    a = _attn_args(q, k_cache, v_cache, k_tree, v_tree, mask, n_nodes, ctx_len, max_ctx, scale,
                   page_table, q, None, None)
    path, splits = ctypes.c_int(), ctypes.c_int()
    with torch.cuda.device(q.device):
        rc = load_library().ddt_tree_attn_plan(ctypes.byref(a), ctypes.byref(path),
                                               ctypes.byref(splits))
    _check(rc, "ddt_tree_attn_plan")
    return path.value, splits.value


def set_wait_limit(cycles: int) -> int:
    """``ddt_debug_set_wait_limit``: bound (clock cycles) of the tensor-core
    kernels' on-chip waits for later launches; <= 0 restores the default of
    about one second.  Returns the previous setting.  A test hook."""
    return int(load_library().ddt_debug_set_wait_limit(int(cycles)))


# ddt_debug_set_attn_kernel's choices
ATTN_KERNEL_AUTO, ATTN_KERNEL_ONE_TILE, ATTN_KERNEL_PAIRS = 0, 1, 2


def set_attn_kernel(which: int) -> int:
    """``ddt_debug_set_attn_kernel``: the tensor-core attention kernel later
    calls use (ATTN_KERNEL_AUTO, _ONE_TILE or _PAIRS).  Returns the previous
    choice (-1 for a value out of range, which changes nothing).  A tuning and
    test hook."""
    return int(load_library().ddt_debug_set_attn_kernel(int(which)))


def tree_attn(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              k_tree: torch.Tensor, v_tree: torch.Tensor, mask: torch.Tensor,
              n_nodes: torch.Tensor, ctx_len: torch.Tensor, max_ctx: int,
              scale: Optional[float] = None, page_table: Optional[torch.Tensor] = None,
              want_lse: bool = False, dev_status: Optional[torch.Tensor] = None):
    """Stage 3.  q [batch, n_max, hq, d] bf16; dense cache [batch, T_max, hkv, d]
    or paged cache [pages, page_size, hkv, d] + page_table [batch, max_pages];
    tree K/V [batch, n_max, hkv, d]; mask [batch, n_max, W].  Returns out bf16
    [batch, n_max, hq, d] (and lse f32 [batch, n_max, hq] when asked)."""
    lib = load_library()
    if q.dim() != 4:
        raise DDTError("tree_attn: q must be [batch, n_max, hq, d]")
    bq, nq, _, dq = q.shape
    _check_kv_shapes("tree_attn", bq, nq, dq, k_tree, v_tree, k_cache, v_cache, page_table)
    if tuple(mask.shape) != (bq, nq, mask_words(nq)):
        raise DDTError("tree_attn: mask must be [%d, %d, %d], got %s"
                       % (bq, nq, mask_words(nq), tuple(mask.shape)))
    if tuple(n_nodes.shape) != (bq,) or tuple(ctx_len.shape) != (bq,):
        raise DDTError("tree_attn: n_nodes and ctx_len must be [%d]" % bq)
    dev = _need_cuda(q, k_cache, v_cache, k_tree, v_tree, mask, n_nodes, ctx_len, page_table,
                     dev_status)
    for t in (q, k_cache, v_cache, k_tree, v_tree):
        if t is not None and (t.dtype != torch.bfloat16 or not t.is_contiguous()):
            raise DDTError("tree_attn: q / caches / tree K,V must be contiguous bfloat16")
    for t in (mask, n_nodes, ctx_len, page_table):
        if t is not None and (t.dtype != torch.int32 or not t.is_contiguous()):
            raise DDTError("tree_attn: mask / n_nodes / ctx_len / page_table must be contiguous int32")
    b, n_max, hq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = torch.empty_like(q)
    lse = torch.empty((b, n_max, hq), dtype=torch.float32, device=dev) if want_lse else None
    a = _attn_args(q, k_cache, v_cache, k_tree, v_tree, mask, n_nodes, ctx_len, max_ctx, scale,
                   page_table, out, lse, dev_status)
    nb = int(lib.ddt_tree_attn_workspace_size(ctypes.byref(a)))
    ws = workspaces.get(dev, "attn", nb)
    with torch.cuda.device(dev):
        rc = lib.ddt_tree_attn(ctypes.byref(a), _ptr(ws), nb, _stream(dev))
    _check(rc, "ddt_tree_attn")
    return (out, lse) if want_lse else out


def tree_walk_workspace_size(batch: int, n_max: int, V: int) -> int:
    return int(load_library().ddt_tree_walk_workspace_size(batch, n_max, V))


def tree_walk_resolve_mode(mode: int, dtype: torch.dtype, batch: int, n_max: int, V: int,
                           L: int) -> int:
    """``ddt_tree_walk_resolve_mode``: WALK_ALL_ROWS or WALK_LAZY, the walk that
    ``mode`` runs for these sizes on the current device."""
    code = _dtype_code(torch.empty(0, dtype=dtype))
    return int(load_library().ddt_tree_walk_resolve_mode(mode, code, batch, n_max, V, L))


def tree_walk(logits: torch.Tensor, tok: torch.Tensor, parent: torch.Tensor,
              depth: torch.Tensor, n_nodes: torch.Tensor, L: int,
              dev_status: Optional[torch.Tensor] = None, mode: int = WALK_AUTO):
    """Stage 4.  ``logits`` [batch, n_max, V] f32/bf16 (rows contiguous, uniform
    stride); ``mode`` one of WALK_ALL_ROWS, WALK_LAZY, WALK_AUTO.  Returns dict
    acc_len [batch], acc_nodes/acc_tok [batch, L], bonus [batch]."""
    lib = load_library()
    _check_types("tree_walk", (tok, torch.int32), (parent, torch.int32), (depth, torch.int32),
                 (n_nodes, torch.int32), (dev_status, torch.int32))
    if logits.dim() != 3 or logits.stride(2) != 1 or logits.stride(0) != logits.stride(1) * logits.shape[1]:
        raise DDTError("logits must be [batch, n_max, V] with contiguous rows and a uniform row stride")
    b, n_max, V = logits.shape
    _check_tree_shapes("tree_walk", b, n_max, tok, parent, depth, n_nodes)
    dev = _need_cuda(logits, tok, parent, depth, n_nodes, dev_status)
    res = {"acc_len": torch.empty(b, dtype=torch.int32, device=dev),
           "acc_nodes": torch.empty((b, L), dtype=torch.int32, device=dev),
           "acc_tok": torch.empty((b, L), dtype=torch.int32, device=dev),
           "bonus": torch.empty(b, dtype=torch.int32, device=dev)}
    nb = int(lib.ddt_tree_walk_workspace_size(b, n_max, V))
    ws = workspaces.get(dev, "walk", nb)
    with torch.cuda.device(dev):
        rc = lib.ddt_tree_walk(_ptr(logits), _dtype_code(logits), b, n_max, V, logits.stride(1),
                               _ptr(tok), _ptr(parent), _ptr(depth), _ptr(n_nodes), L, int(mode),
                               _ptr(res["acc_len"]), _ptr(res["acc_nodes"]), _ptr(res["acc_tok"]),
                               _ptr(res["bonus"]), _ptr(ws), nb, _ptr(dev_status), _stream(dev))
    _check(rc, "ddt_tree_walk")
    return res


def tree_walk_sample(logits: torch.Tensor, tok: torch.Tensor, parent: torch.Tensor,
                     depth: torch.Tensor, n_nodes: torch.Tensor, L: int, inv_temperature: float,
                     seed: int, step: int, dev_status: Optional[torch.Tensor] = None,
                     step_counter: Optional[torch.Tensor] = None):
    """Stage 4 under temperature sampling (``ddt_tree_walk_sample``): row j of
    sequence b draws its token from softmax(inv_temperature * z) with the
    Philox4x64-10 uniform of counter (j, b, 0, 0) and key (seed, step).
    ``step_counter`` (optional int64 [1] on the device) is added to ``step``
    and advanced by one per call, for replays of a captured graph.
    Arguments and outputs otherwise as :func:`tree_walk`."""
    lib = load_library()
    _check_types("tree_walk_sample", (tok, torch.int32), (parent, torch.int32),
                 (depth, torch.int32), (n_nodes, torch.int32), (dev_status, torch.int32))
    if step_counter is not None and (step_counter.dtype != torch.int64 or step_counter.numel() != 1):
        raise DDTError("step_counter must be a one-element int64 tensor")
    if logits.dim() != 3 or logits.stride(2) != 1 or logits.stride(0) != logits.stride(1) * logits.shape[1]:
        raise DDTError("logits must be [batch, n_max, V] with contiguous rows and a uniform row stride")
    b, n_max, V = logits.shape
    _check_tree_shapes("tree_walk_sample", b, n_max, tok, parent, depth, n_nodes)
    dev = _need_cuda(logits, tok, parent, depth, n_nodes, dev_status, step_counter)
    res = {"acc_len": torch.empty(b, dtype=torch.int32, device=dev),
           "acc_nodes": torch.empty((b, L), dtype=torch.int32, device=dev),
           "acc_tok": torch.empty((b, L), dtype=torch.int32, device=dev),
           "bonus": torch.empty(b, dtype=torch.int32, device=dev)}
    nb = int(lib.ddt_tree_walk_workspace_size(b, n_max, V))
    ws = workspaces.get(dev, "walk", nb)
    mask64 = (1 << 64) - 1
    with torch.cuda.device(dev):
        rc = lib.ddt_tree_walk_sample(_ptr(logits), _dtype_code(logits), b, n_max, V,
                                      logits.stride(1), _ptr(tok), _ptr(parent), _ptr(depth),
                                      _ptr(n_nodes), L, float(inv_temperature), int(seed) & mask64,
                                      int(step) & mask64, _ptr(step_counter), _ptr(res["acc_len"]),
                                      _ptr(res["acc_nodes"]), _ptr(res["acc_tok"]),
                                      _ptr(res["bonus"]), _ptr(ws), nb, _ptr(dev_status),
                                      _stream(dev))
    _check(rc, "ddt_tree_walk_sample")
    return res


def kv_commit(k_tree: torch.Tensor, v_tree: torch.Tensor, acc_len: torch.Tensor,
              acc_nodes: torch.Tensor, ctx_len: torch.Tensor, k_cache: torch.Tensor,
              v_cache: torch.Tensor, page_table: Optional[torch.Tensor] = None,
              page_size: int = 64, dev_status: Optional[torch.Tensor] = None):
    """``ddt_kv_commit``: append each sequence's root and accepted rows of the
    tree K/V ([batch, n_max, hkv, d] bf16) to the cache (dense [batch, t_max,
    hkv, d] or a page pool [pages, page_size, hkv, d] with ``page_table``) and
    advance ``ctx_len`` (int32, in place) by acc_len + 1."""
    lib = load_library()
    if k_tree.dim() != 4:
        raise DDTError("kv_commit: tree K must be [batch, n_max, hkv, d]")
    bk, nk, _, dk = k_tree.shape
    _check_kv_shapes("kv_commit", bk, nk, dk, k_tree, v_tree, k_cache, v_cache, page_table,
                     page_size)
    if tuple(acc_len.shape) != (bk,) or tuple(ctx_len.shape) != (bk,):
        raise DDTError("kv_commit: acc_len and ctx_len must be [%d]" % bk)
    if acc_nodes.dim() != 2 or acc_nodes.shape[0] != bk:
        raise DDTError("kv_commit: acc_nodes must be [%d, L]" % bk)
    dev = _need_cuda(k_tree, v_tree, acc_len, acc_nodes, ctx_len, k_cache, v_cache, page_table,
                     dev_status)
    for t in (k_tree, v_tree, k_cache, v_cache):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise DDTError("kv_commit: tree K/V and caches must be contiguous bfloat16")
    for t in (acc_len, acc_nodes, ctx_len, page_table):
        if t is not None and (t.dtype != torch.int32 or not t.is_contiguous()):
            raise DDTError("kv_commit: acc_len / acc_nodes / ctx_len / page_table must be "
                           "contiguous int32")
    b, n_max, hkv, d = k_tree.shape

    def addr(t):
        return None if t is None else t.data_ptr()

    a = KVCommitArgs()
    a.k_tree, a.v_tree = addr(k_tree), addr(v_tree)
    a.acc_len, a.acc_nodes, a.ctx_len = addr(acc_len), addr(acc_nodes), addr(ctx_len)
    a.k_cache, a.v_cache = addr(k_cache), addr(v_cache)
    if page_table is None:
        a.page_table, a.page_size, a.max_pages, a.num_pages = None, 0, 0, 0
        a.t_max = k_cache.shape[1]
    else:
        a.page_table, a.page_size = addr(page_table), page_size
        a.max_pages, a.num_pages, a.t_max = page_table.shape[1], k_cache.shape[0], 0
    a.batch, a.n_max, a.hkv, a.d = b, n_max, hkv, d
    a.L = acc_nodes.shape[1]
    a.dev_status = addr(dev_status)
    with torch.cuda.device(dev):
        rc = lib.ddt_kv_commit(ctypes.byref(a), _stream(dev))
    _check(rc, "ddt_kv_commit")


def lm_head_walk(hidden: torch.Tensor, weight: torch.Tensor, tok: torch.Tensor,
                 parent: torch.Tensor, depth: torch.Tensor, n_nodes: torch.Tensor, L: int,
                 want_row_token: bool = False, dev_status: Optional[torch.Tensor] = None):
    """``ddt_lm_head_walk``: the greedy walk straight from the target's hidden
    states ([batch, n_max, K] bf16) and LM head ([V, K] bf16).  Returns the
    walk outputs of :func:`tree_walk` (plus ``row_token`` [batch, n_max] when
    asked)."""
    lib = load_library()
    if hidden.dim() != 3 or weight.dim() != 2:
        raise DDTError("lm_head_walk: hidden must be [batch, n_max, K] and weight [V, K]")
    _check_tree_shapes("lm_head_walk", hidden.shape[0], hidden.shape[1], tok, parent, depth,
                       n_nodes)
    dev = _need_cuda(hidden, weight, tok, parent, depth, n_nodes, dev_status)
    for t in (hidden, weight):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise DDTError("lm_head_walk: hidden and weight must be contiguous bfloat16")
    for t in (tok, parent, depth, n_nodes):
        if t.dtype != torch.int32 or not t.is_contiguous():
            raise DDTError("lm_head_walk: tree tensors must be contiguous int32")
    b, n_max, K = hidden.shape
    V = weight.shape[0]
    if weight.shape[1] != K:
        raise DDTError("lm_head_walk: weight must be [V, K] with the hidden size K")
    res = {"acc_len": torch.empty(b, dtype=torch.int32, device=dev),
           "acc_nodes": torch.empty((b, L), dtype=torch.int32, device=dev),
           "acc_tok": torch.empty((b, L), dtype=torch.int32, device=dev),
           "bonus": torch.empty(b, dtype=torch.int32, device=dev)}
    if want_row_token:
        res["row_token"] = torch.empty((b, n_max), dtype=torch.int32, device=dev)
    a = LmHeadWalkArgs()
    a.hidden, a.weight, a.K, a.V = hidden.data_ptr(), weight.data_ptr(), K, V
    a.tok, a.parent, a.depth, a.n_nodes = (tok.data_ptr(), parent.data_ptr(), depth.data_ptr(),
                                           n_nodes.data_ptr())
    a.batch, a.n_max, a.L = b, n_max, L
    a.acc_len, a.acc_nodes = res["acc_len"].data_ptr(), res["acc_nodes"].data_ptr()
    a.acc_tok, a.bonus = res["acc_tok"].data_ptr(), res["bonus"].data_ptr()
    a.row_token = res["row_token"].data_ptr() if want_row_token else None
    a.dev_status = None if dev_status is None else dev_status.data_ptr()
    nb = int(lib.ddt_lm_head_walk_workspace_size(ctypes.byref(a)))
    ws = workspaces.get(dev, "lm_head", nb)
    with torch.cuda.device(dev):
        rc = lib.ddt_lm_head_walk(ctypes.byref(a), _ptr(ws), nb, _stream(dev))
    _check(rc, "ddt_lm_head_walk")
    return res
