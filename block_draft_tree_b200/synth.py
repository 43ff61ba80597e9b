"""Seeded synthetic inputs for the verification round.

This module draws random numbers and lays them out; it holds none of the
round's arithmetic (no softmax, no top-k, no tree, no attention, no walk).
It is the one piece of code that both the CUDA path and the CPU oracle are
fed from.

Workloads (the five named shapes of the verification round):

* ``tiny``      batch 1, L=4, V=64, k=4, B=8; fp32 draft logits; ctx 128;
  4 q heads / 1 kv head, d=64; planted agreement 0.7.
* ``b64``       batch 1, L=16, V=151936, k=8, B=64; bf16 draft logits with
  spikes; ctx 4096; GQA 32/8, d=128; agreement 0.8 decaying 0.03/depth.
* ``b256``      batch 8, L=16, V=151936, k=16, B=256; ctx 8192; GQA 64/8;
  sequence 0 is forced to a chain (k=1, B=16: single-path drafting).
* ``paged128``  batch 32, ragged ctx U{1024..32768}, L=16, V=129280, k=8,
  B=128; Zipf(1.1) draft logits over a seeded permutation, temperature 0.7;
  GQA 32/8; KV in 64-token pages in a seeded random order.
* ``long512``   batch 4, ctx 131072, L=32, V=151936, k=16, B=512; MQA 16/1;
  agreement 0.9 decaying 0.02/depth.

Drafts and K/V are N(0,1); spikes add +6/+4/+3 at distinct seeded tokens of
each position (+6/+4 for ``tiny``).  Every tensor has its own numpy PCG64
stream derived from ``SeedSequence([seed, tensor_tag])``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    L: int
    V: int
    k: int
    B: int
    ctx: int                 # context length (upper end when ragged)
    hq: int
    hkv: int
    d: int
    draft: str               # "spikes" | "zipf"
    draft_dtype: str         # "f32" | "bf16"
    spikes: tuple = (6.0, 4.0, 3.0)
    inv_temperature: float = 1.0
    plant_p0: float = 0.8
    plant_decay: float = 0.03
    ctx_min: Optional[int] = None   # ragged contexts when set
    page_size: int = 0              # paged KV when > 0
    chain_seq0: bool = False        # sequence 0 drafted as a single path (k=1, B=L)
    index: int = 0

    @property
    def n_max(self) -> int:
        return self.B + 1

    @property
    def seed(self) -> int:
        return 0xDD7 + self.index

    def k_per_seq(self) -> np.ndarray:
        k = np.full(self.batch, self.k, np.int32)
        if self.chain_seq0:
            k[0] = 1
        return k

    def budget_per_seq(self) -> np.ndarray:
        b = np.full(self.batch, self.B, np.int32)
        if self.chain_seq0:
            b[0] = self.L
        return b

    def scaled(self, **kw) -> "Workload":
        """A copy with some fields replaced (smaller test shapes)."""
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 64, 4, 8, 128, 4, 1, 64, "spikes", "f32",
                     spikes=(6.0, 4.0), plant_p0=0.7, plant_decay=0.0, index=0),
    "b64": Workload("b64", 1, 16, 151936, 8, 64, 4096, 32, 8, 128, "spikes", "bf16",
                    plant_p0=0.8, plant_decay=0.03, index=1),
    "b256": Workload("b256", 8, 16, 151936, 16, 256, 8192, 64, 8, 128, "spikes", "bf16",
                     plant_p0=0.8, plant_decay=0.03, chain_seq0=True, index=2),
    "paged128": Workload("paged128", 32, 16, 129280, 8, 128, 32768, 32, 8, 128, "zipf", "bf16",
                         inv_temperature=1.0 / 0.7, plant_p0=0.8, plant_decay=0.03,
                         ctx_min=1024, page_size=64, index=3),
    "long512": Workload("long512", 4, 32, 151936, 16, 512, 131072, 16, 1, 128, "spikes", "bf16",
                        plant_p0=0.9, plant_decay=0.02, index=4),
}

_TAGS = {"draft": 1, "root": 2, "ctx": 3, "q": 4, "kc": 5, "vc": 6, "kt": 7, "vt": 8,
         "pages": 9, "target": 10, "plant": 11}


def rng(w: Workload, tag: str, seed: Optional[int] = None) -> np.random.Generator:
    s = w.seed if seed is None else seed
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([s, _TAGS[tag]])))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(g: np.random.Generator, shape) -> np.ndarray:
    return g.standard_normal(shape, dtype=np.float32)


def draft_logits(w: Workload, seed: Optional[int] = None) -> np.ndarray:
    """[batch, L, V] draft logits: float32, or bf16 bits (uint16)."""
    g = rng(w, "draft", seed)
    shape = (w.batch, w.L, w.V)
    if w.draft == "spikes":
        z = _normal(g, shape)
        ns = len(w.spikes)
        for b in range(w.batch):
            for i in range(w.L):
                toks = g.choice(w.V, size=ns, replace=False)
                for t, s in zip(toks, w.spikes):
                    z[b, i, t] += np.float32(s)
    elif w.draft == "zipf":
        ranks = np.arange(1, w.V + 1, dtype=np.float64)
        zipf = (-1.1 * np.log(ranks)).astype(np.float32)
        z = np.empty(shape, np.float32)
        for b in range(w.batch):
            for i in range(w.L):
                z[b, i, g.permutation(w.V)] = zipf
    else:
        raise ValueError(w.draft)
    return z if w.draft_dtype == "f32" else to_bf16_bits(z)


def root_tokens(w: Workload, seed: Optional[int] = None) -> np.ndarray:
    return rng(w, "root", seed).integers(0, w.V, size=w.batch).astype(np.int32)


def context_lengths(w: Workload, seed: Optional[int] = None) -> np.ndarray:
    if w.ctx_min is None:
        return np.full(w.batch, w.ctx, np.int32)
    return rng(w, "ctx", seed).integers(w.ctx_min, w.ctx + 1, size=w.batch).astype(np.int32)


def attention_inputs(w: Workload, seed: Optional[int] = None, ctx_len=None) -> dict:
    """Query rows, the context KV cache (dense or paged) and the tree KV.

    Dense cache: ``k_cache``/``v_cache`` [batch, Tmax, Hkv, d].
    Paged cache: ``k_cache``/``v_cache`` [pages, page_size, Hkv, d] and
    ``page_table`` [batch, max_pages] holding a seeded random placement.
    All bf16 bits (uint16).
    """
    if ctx_len is None:
        ctx_len = context_lengths(w, seed)
    ctx_len = np.asarray(ctx_len, np.int32)
    out = {"ctx_len": ctx_len}
    n = w.n_max
    out["q"] = to_bf16_bits(_normal(rng(w, "q", seed), (w.batch, n, w.hq, w.d)))
    out["k_tree"] = to_bf16_bits(_normal(rng(w, "kt", seed), (w.batch, n, w.hkv, w.d)))
    out["v_tree"] = to_bf16_bits(_normal(rng(w, "vt", seed), (w.batch, n, w.hkv, w.d)))
    if w.page_size > 0:
        ps = w.page_size
        npg = (ctx_len.astype(np.int64) + ps - 1) // ps
        total = int(npg.sum())
        max_pages = int(npg.max()) if w.batch else 0
        perm = rng(w, "pages", seed).permutation(total).astype(np.int32)
        pt = np.full((w.batch, max(max_pages, 1)), -1, np.int32)
        off = 0
        for b in range(w.batch):
            pt[b, :npg[b]] = perm[off:off + npg[b]]
            off += int(npg[b])
        out["page_table"] = pt
        out["page_size"] = ps
        shape = (total, ps, w.hkv, w.d)
    else:
        shape = (w.batch, int(ctx_len.max()) if w.batch else 0, w.hkv, w.d)
    out["k_cache"] = to_bf16_bits(_normal(rng(w, "kc", seed), shape))
    out["v_cache"] = to_bf16_bits(_normal(rng(w, "vc", seed), shape))
    return out


def target_logits(w: Workload, tok, parent, depth, n_nodes, seed: Optional[int] = None,
                  n_max: Optional[int] = None) -> np.ndarray:
    """[batch, Nmax, V] float32 target logits, N(0,1), with planted agreement.

    For every tree row x that has children, with probability
    max(0, p0 - decay*depth(x)) one child is chosen uniformly and its token's
    logit in row x is set to (row maximum + 2), so that the target's greedy
    choice at x agrees with the draft.  The tree (tok/parent/depth/n_nodes)
    is an input here; rows beyond n_nodes stay random.
    """
    n_max = w.n_max if n_max is None else n_max
    g = rng(w, "target", seed)
    gp = rng(w, "plant", seed)
    out = _normal(g, (w.batch, n_max, w.V))
    for b in range(w.batch):
        n = int(n_nodes[b])
        par = np.asarray(parent[b][:n])
        for x in range(n):
            kids = np.nonzero(par == x)[0]
            p = max(0.0, w.plant_p0 - w.plant_decay * float(depth[b][x]))
            u = gp.random()
            c = gp.integers(0, max(len(kids), 1))
            if len(kids) == 0 or u >= p:
                continue
            t = int(tok[b][kids[c]])
            row = out[b, x]
            row[t] = row.max() + np.float32(2.0)
    return out
