"""One verification round = the four C-ABI calls on preallocated buffers.

:class:`VerifyRound` owns every output and workspace for one shape, so the
round allocates nothing per call and can be captured once into a CUDA graph
and replayed.  Inputs are bound by pointer (:meth:`bind`); the four calls
read them in place.  Marshalling only -- all arithmetic is in libddt.so.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from . import api


class VerifyRound:
    """One verification round on fixed shapes.

    ``decode`` is the target's decoding rule in stage 4: ``"greedy"``
    (``ddt_tree_walk`` over the bound target logits, in ``walk_mode``), ``"sample"``
    (``ddt_tree_walk_sample`` at ``sample_inv_temperature`` with a device step
    counter, so that every replay of a captured round draws fresh uniforms) or
    ``"lm_head"`` (``ddt_lm_head_walk`` from the bound hidden states and LM
    head; no logits are stored).  With ``commit`` the round ends with
    ``ddt_kv_commit``: the root's and the accepted rows' K/V join the bound
    cache and ``ctx_len`` advances in place.

    With ``adaptive_budget`` (a dict of ``total``, ``cost_fixed``,
    ``cost_per_node``) stage 2 builds every sequence's tree with its largest
    budget, splits the batch's nodes with ``ddt_plan_budget`` under that cost
    model, and builds the trees again with those budgets; ``out["budget"]``
    and ``out["expected_tokens"]`` hold the split.
    """

    def __init__(self, *, batch: int, L: int, V: int, k: int, B_max: int, hq: int, hkv: int,
                 d: int, max_ctx: int, draft_dtype: torch.dtype = torch.bfloat16,
                 target_dtype: torch.dtype = torch.float32, inv_temperature: float = 1.0,
                 paged: bool = False, page_size: int = 64, max_pages: int = 0,
                 decode: str = "greedy", sample_inv_temperature: float = 1.0, seed: int = 0,
                 commit: bool = False, walk_mode: int = api.WALK_AUTO,
                 adaptive_budget: Optional[dict] = None, device: str = "cuda"):
        if decode not in ("greedy", "sample", "lm_head"):
            raise ValueError("decode must be 'greedy', 'sample' or 'lm_head'")
        self.decode, self.commit, self.walk_mode = decode, commit, int(walk_mode)
        self.adaptive = dict(adaptive_budget) if adaptive_budget else None
        self.sample_inv_t, self.seed = float(sample_inv_temperature), int(seed)
        self.lib = api.load_library()
        self.dev = torch.device(device)
        self.batch, self.L, self.V, self.k, self.B_max = batch, L, V, k, B_max
        self.n_max = B_max + 1
        self.hq, self.hkv, self.d, self.max_ctx = hq, hkv, d, max_ctx
        self.inv_t = float(inv_temperature)
        self.paged, self.page_size, self.max_pages = paged, page_size, max_pages
        self.draft_code = api._dtype_code(torch.empty(0, dtype=draft_dtype))
        self.target_code = api._dtype_code(torch.empty(0, dtype=target_dtype))
        dev = self.dev
        e = lambda *s, dt=torch.int32: torch.empty(s, dtype=dt, device=dev)
        W = api.mask_words(self.n_max)
        self.out = {
            "ids": e(batch, L, k), "zk": e(batch, L, k, dt=torch.float32),
            "lse": e(batch, L, dt=torch.float32),
            "tok": e(batch, self.n_max), "parent": e(batch, self.n_max),
            "depth": e(batch, self.n_max), "pos": e(batch, self.n_max),
            "mask": e(batch, self.n_max, W), "n_nodes": e(batch),
            "surrogate": e(batch, dt=torch.float64),
            "attn": e(batch, self.n_max, hq, d, dt=torch.bfloat16),
            "acc_len": e(batch), "acc_nodes": e(batch, L), "acc_tok": e(batch, L), "bonus": e(batch),
            "status": torch.zeros(1, dtype=torch.int32, device=dev),
            "budget": e(batch), "expected_tokens": e(batch, dt=torch.float64),
        }
        self.ws_topk_n = int(self.lib.ddt_topk_workspace_size(batch, L, V, k))
        self.ws_walk_n = int(self.lib.ddt_tree_walk_workspace_size(batch, self.n_max, V))
        self.ws_topk = torch.zeros(max(self.ws_topk_n, 256), dtype=torch.uint8, device=dev)
        self.ws_walk = torch.zeros(max(self.ws_walk_n, 256), dtype=torch.uint8, device=dev)
        self.ws_attn = None
        self.attn_args = None
        self.inputs = None
        # stage 4 under sampling: the step that replays advance on the device
        self.step_counter = torch.zeros(1, dtype=torch.int64, device=dev)
        self.lm_args = None
        self.ws_lm = None
        self.commit_args = None

    # ------------------------------------------------------------------
    def bind(self, inputs: dict):
        """Bind device input tensors: draft [b,L,V], root [b], ctx_len [b],
        q [b,n,hq,d], k_cache/v_cache, optional page_table, k_tree/v_tree
        [b,n,hkv,d], target [b,n,V]; optional k_per_seq / budget [b]."""
        self._check_inputs(inputs)
        self.inputs = inputs
        o = self.out
        a = api._attn_args(inputs["q"], inputs["k_cache"], inputs["v_cache"], inputs["k_tree"],
                           inputs["v_tree"], o["mask"], o["n_nodes"], inputs["ctx_len"],
                           self.max_ctx, 1.0 / math.sqrt(self.d), inputs.get("page_table"),
                           o["attn"], None, o["status"])
        self.attn_args = a
        n = int(self.lib.ddt_tree_attn_workspace_size(ctypes.byref(a)))
        if self.ws_attn is None or self.ws_attn.numel() < n:
            self.ws_attn = torch.zeros(max(n, 256), dtype=torch.uint8, device=self.dev)
        self.ws_attn_n = n
        if self.decode == "lm_head":
            hid, head = inputs["hidden"], inputs["head"]
            la = api.LmHeadWalkArgs()
            la.hidden, la.weight = hid.data_ptr(), head.data_ptr()
            la.K, la.V = hid.shape[-1], head.shape[0]
            la.tok, la.parent = o["tok"].data_ptr(), o["parent"].data_ptr()
            la.depth, la.n_nodes = o["depth"].data_ptr(), o["n_nodes"].data_ptr()
            la.batch, la.n_max, la.L = self.batch, self.n_max, self.L
            la.acc_len, la.acc_nodes = o["acc_len"].data_ptr(), o["acc_nodes"].data_ptr()
            la.acc_tok, la.bonus = o["acc_tok"].data_ptr(), o["bonus"].data_ptr()
            la.row_token, la.dev_status = None, o["status"].data_ptr()
            self.lm_args = la
            nl = int(self.lib.ddt_lm_head_walk_workspace_size(ctypes.byref(la)))
            if self.ws_lm is None or self.ws_lm.numel() < nl:
                self.ws_lm = torch.zeros(max(nl, 256), dtype=torch.uint8, device=self.dev)
            self.ws_lm_n = nl
        if self.commit:
            ca = api.KVCommitArgs()
            ca.k_tree, ca.v_tree = inputs["k_tree"].data_ptr(), inputs["v_tree"].data_ptr()
            ca.acc_len, ca.acc_nodes = o["acc_len"].data_ptr(), o["acc_nodes"].data_ptr()
            ca.ctx_len = inputs["ctx_len"].data_ptr()
            ca.k_cache, ca.v_cache = inputs["k_cache"].data_ptr(), inputs["v_cache"].data_ptr()
            pt = inputs.get("page_table")
            if pt is None:
                ca.page_table, ca.page_size, ca.max_pages, ca.num_pages = None, 0, 0, 0
                ca.t_max = inputs["k_cache"].shape[1]
            else:
                ca.page_table, ca.page_size = pt.data_ptr(), self.page_size
                ca.max_pages, ca.num_pages = pt.shape[1], inputs["k_cache"].shape[0]
                ca.t_max = 0
            ca.batch, ca.n_max, ca.hkv, ca.d, ca.L = self.batch, self.n_max, self.hkv, self.d, self.L
            ca.dev_status = o["status"].data_ptr()
            self.commit_args = ca

    def _check_inputs(self, x: dict):
        """Refuse inputs whose shapes, dtypes or layouts differ from this
        round's sizes: the calls index the bound memory with those sizes."""
        b, L, V, n = self.batch, self.L, self.V, self.n_max

        def need(name, shape, dtype):
            t = x.get(name)
            if t is None:
                raise api.DDTError("bind: input %r is missing" % name)
            if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
                raise api.DDTError("bind: %r must be %s %s, got %s %s"
                                   % (name, tuple(shape), dtype, tuple(t.shape), t.dtype))
            return t

        def rows(name, t, r):  # [b, r, V] with contiguous rows and a uniform row stride
            if t.stride(2) != 1 or t.stride(0) != t.stride(1) * r:
                raise api.DDTError("bind: %r needs contiguous rows and a uniform row stride" % name)

        rows("draft", need("draft", (b, L, V), torch.bfloat16 if self.draft_code == api.DDT_BF16
                           else torch.float32), L)
        need("root", (b,), torch.int32)
        need("ctx_len", (b,), torch.int32)
        for name in ("k_per_seq", "budget"):
            if x.get(name) is not None:
                need(name, (b,), torch.int32)
        for name, shape in (("q", (b, n, self.hq, self.d)), ("k_tree", (b, n, self.hkv, self.d)),
                            ("v_tree", (b, n, self.hkv, self.d))):
            if not need(name, shape, torch.bfloat16).is_contiguous():
                raise api.DDTError("bind: %r must be contiguous" % name)
        api._check_types("bind", (x.get("k_cache"), torch.bfloat16),
                         (x.get("v_cache"), torch.bfloat16), (x.get("page_table"), torch.int32))
        pt = x.get("page_table")
        api._check_kv_shapes("bind", b, n, self.d, x["k_tree"], x["v_tree"], x.get("k_cache"),
                             x.get("v_cache"), pt,
                             self.page_size if self.commit and pt is not None else None)
        if self.decode == "lm_head":
            hid, head = x.get("hidden"), x.get("head")
            if hid is None or head is None:
                raise api.DDTError("bind: decode='lm_head' needs 'hidden' and 'head'")
            need("hidden", (b, n, hid.shape[-1]), torch.bfloat16)
            need("head", (V, hid.shape[-1]), torch.bfloat16)
            api._check_types("bind", (hid, torch.bfloat16), (head, torch.bfloat16))
        else:
            rows("target", need("target", (b, n, V), torch.bfloat16
                                if self.target_code == api.DDT_BF16 else torch.float32), n)

    def launch(self, stream: Optional[torch.cuda.Stream] = None, marks=None):
        """Enqueue the four stages (and the commit) on ``stream``.  ``marks(i)``
        is called before stage i and after the last (i = 0..4, and 5 after
        the commit), e.g. to record events."""
        n = 5 if self.commit else 4
        for i in range(n):
            if marks:
                marks(i)
            self.launch_stage(i, stream)
        if marks:
            marks(n)

    def launch_stage(self, i: int, stream: Optional[torch.cuda.Stream] = None):
        """Enqueue stage i alone: 0 top-k, 1 tree, 2 attention, 3 walk, 4 commit."""
        lib, o, x = self.lib, self.out, self.inputs
        s = ctypes.c_void_p((stream or torch.cuda.current_stream(self.dev)).cuda_stream)
        P = api._ptr
        if i == 0:
            rc = lib.ddt_topk(P(x["draft"]), self.draft_code, self.batch, self.L, self.V,
                              x["draft"].stride(1), self.k, self.inv_t, P(o["ids"]), P(o["zk"]),
                              None, P(o["lse"]), P(self.ws_topk), self.ws_topk_n, s)
            api._check(rc, "ddt_topk")
        elif i == 1:
            def build(budget):
                rc = lib.ddt_build_tree(P(o["ids"]), P(o["zk"]), P(o["lse"]), self.batch, self.L,
                                        self.k, self.inv_t, P(x.get("k_per_seq")), P(budget),
                                        self.B_max, P(x["root"]), P(x["ctx_len"]), P(o["tok"]),
                                        P(o["parent"]), P(o["depth"]), P(o["pos"]), P(o["mask"]),
                                        P(o["n_nodes"]), P(o["surrogate"]), P(o["status"]), s)
                api._check(rc, "ddt_build_tree")

            build(x.get("budget"))
            if self.adaptive:
                a = self.adaptive
                rc = lib.ddt_plan_budget(P(o["tok"]), P(o["parent"]), P(o["depth"]),
                                         P(o["n_nodes"]), P(o["ids"]), P(o["zk"]), P(o["lse"]),
                                         self.batch, self.L, self.k, self.n_max, self.inv_t,
                                         int(a.get("total", -1)), float(a.get("cost_fixed", 0.0)),
                                         float(a.get("cost_per_node", 0.0)), P(o["budget"]),
                                         P(o["expected_tokens"]), P(o["status"]), s)
                api._check(rc, "ddt_plan_budget")
                build(o["budget"])
        elif i == 2:
            rc = lib.ddt_tree_attn(ctypes.byref(self.attn_args), P(self.ws_attn), self.ws_attn_n, s)
            api._check(rc, "ddt_tree_attn")
        elif i == 3:
            if self.decode == "greedy":
                rc = lib.ddt_tree_walk(P(x["target"]), self.target_code, self.batch, self.n_max,
                                       self.V, x["target"].stride(1), P(o["tok"]), P(o["parent"]),
                                       P(o["depth"]), P(o["n_nodes"]), self.L, self.walk_mode,
                                       P(o["acc_len"]),
                                       P(o["acc_nodes"]), P(o["acc_tok"]), P(o["bonus"]),
                                       P(self.ws_walk), self.ws_walk_n, P(o["status"]), s)
                api._check(rc, "ddt_tree_walk")
            elif self.decode == "sample":
                rc = lib.ddt_tree_walk_sample(P(x["target"]), self.target_code, self.batch,
                                              self.n_max, self.V, x["target"].stride(1),
                                              P(o["tok"]), P(o["parent"]), P(o["depth"]),
                                              P(o["n_nodes"]), self.L, self.sample_inv_t,
                                              self.seed, 0, P(self.step_counter), P(o["acc_len"]),
                                              P(o["acc_nodes"]), P(o["acc_tok"]), P(o["bonus"]),
                                              P(self.ws_walk), self.ws_walk_n, P(o["status"]), s)
                api._check(rc, "ddt_tree_walk_sample")
            else:
                rc = lib.ddt_lm_head_walk(ctypes.byref(self.lm_args), P(self.ws_lm), self.ws_lm_n,
                                          s)
                api._check(rc, "ddt_lm_head_walk")
        elif i == 4 and self.commit:
            rc = lib.ddt_kv_commit(ctypes.byref(self.commit_args), s)
            api._check(rc, "ddt_kv_commit")
        else:
            raise ValueError("no stage %d in this round" % i)

    def capture(self, marks=None) -> torch.cuda.CUDAGraph:
        """Capture one round (with its current bindings) into a CUDA graph."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.launch(torch.cuda.current_stream(self.dev), marks)
        return g
