"""Shared helpers for the parity tests: seeded inputs for a workload, tensor
conversion, and the comparisons the tests apply.

Inputs come from block_draft_tree_b200.synth (random numbers only) and, where
a stage needs the previous stage's result as input, from the CPU oracle --
never from the CUDA path.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from block_draft_tree_b200 import synth

# fp32 log-sum-exp over bf16 logits: each term's base-2 exponent carries
# ~|z*c|*2^-24 + ~1 ulp of ex2 (~2^-22 relative); per-thread sums of 32 terms
# and the merges add < 2e-6 relative.  1e-5 absolute on lse covers that with
# margin; logp = invT*z - lse adds one fp32 rounding of a value below 64.
LSE_ATOL = 1e-5
LOGP_ATOL = 2e-5
# bf16 output of an fp32-accumulated attention against fp64:
# max-abs 2e-2 and max-abs / max|ref| <= 1e-2.
ATTN_ABS = 2e-2
ATTN_REL = 1e-2
# the tree is bit-exact when every cross-depth score gap between a selected
# node and an unselected child exceeds this margin
TREE_MARGIN = 1e-4


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def logits_tensor(z: np.ndarray, device="cuda") -> torch.Tensor:
    return bf16_tensor(z, device) if z.dtype == np.uint16 else torch.from_numpy(z).to(device)


def i32(x, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(device)


def f32_up(x: np.ndarray) -> np.ndarray:
    """fp64 -> f32 rounded towards +inf (the library stores lse this way, so
    that no candidate's log-probability turns positive when widened back)."""
    y = np.asarray(x, np.float64).astype(np.float32)
    low = y.astype(np.float64) < x
    y[low] = np.nextafter(y[low], np.float32(np.inf))
    return y


def oracle_tree_inputs(w: synth.Workload, z: np.ndarray):
    """Oracle top-k of the draft with lse rounded up to f32, as both sides receive it."""
    ids, zk, logp, lse = oracle.topk(z, w.k, w.inv_temperature)
    return ids, zk, f32_up(lse)


def paths(tok, parent, n):
    out = []
    for j in range(n):
        p, x = [], j
        while x > 0:
            p.append(int(tok[x]))
            x = int(parent[x])
        out.append(tuple(reversed(p)))
    return out


def assert_attn_close(got: np.ndarray, ref: np.ndarray, what: str):
    err = np.abs(got.astype(np.float64) - ref)
    mx = float(err.max()) if err.size else 0.0
    scale = float(np.abs(ref).max()) if ref.size else 1.0
    assert mx <= ATTN_ABS, "%s: max abs error %.3g > %.3g" % (what, mx, ATTN_ABS)
    assert mx <= ATTN_REL * max(scale, 1e-30), "%s: max abs error %.3g > %.3g * max|ref| %.3g" % (
        what, mx, ATTN_REL, scale)
    return mx, scale
