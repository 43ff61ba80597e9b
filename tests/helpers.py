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


# ---------------------------------------------------------------------------
# The sampled walk: which tokens the kernel's fp32 draw may return
# ---------------------------------------------------------------------------
LOG2E = 1.4426950408889634074
POLY_REL = 2.0 ** -22
SUM_SLACK = 1e-10


def _values(row: np.ndarray) -> np.ndarray:
    if row.dtype == np.uint16:
        return (row.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return row.astype(np.float64)


def allowed_tokens(row: np.ndarray, invT: float, u: float, with_width: bool = False):
    """Tokens that ddt_tree_walk_sample may draw from ``row`` with uniform
    ``u``, against the oracle's exact draw (fp64 weights w_v = exp(invT*z_v - m),
    inversion over ids in increasing order).

    The kernel evaluates each weight in fp32 by its stated arithmetic; its
    error against w_v, relative, with A = fl32(invT) * log2(e):
      * the exponent: t = fl32(a*z) with a = fl32(A), plus the part of A*z
        that t lost, e = fma(a_lo, z, fma(a, z, -t)) with a_lo = fl32(A - a),
        applied as P * (1 + ln2 * e).  The residual fma(a, z, -t) is exact;
        the rest leaves |A*z - t - e| <= 2^-40 * (|A*z| + 1), and the linear
        form of 2^e is off by at most (ln2 * e)^2 / 2 with |e| <= 2^-23 |A*z|;
      * 2^r on |r| <= 1/2 by the fp32 Horner form of its degree-7 Taylor
        polynomial: fp32 coefficients below 0.6 ulp of 2^r, seven fused
        roundings below 1.8 ulp, truncation below 0.13 ulp; 2^-22 bounds
        the sum (ulp = 2^-24 relative);
      * the correction's own fp32 rounding: 2^-24;
      * the power-of-two scaling of weights against a common reference is
        exact; weights below 2^-120 of the largest are dropped (absolute
        error below V * 2^-119 of the largest weight, inside the slack);
      * sums: double-float per thread (2^-40 relative), fp64 beyond
        (V * 2^-53 relative); a slack of 1e-10 * S covers both.
    So the cumulative sum C_j is within E_j = sum_{i<=j} theta_i w_i +
    1e-10 * S of the exact one, theta_i being the product of these factors
    minus one.  The allowed tokens are those whose interval [C_{v-1}, C_v)
    meets u*S for some sums within these bounds; exact-zero weights (-inf
    logits) are never drawn.  A one-element set means the draw is decided
    beyond rounding.  With ``with_width`` it also returns the probability mass
    of the allowed tokens between the first and the last, and the band's
    width (relative to S): the first can never exceed the second."""
    w = oracle.sampler_row_weights(row, invT)
    S = float(w.sum())
    if not S > 0.0:  # no finite logit: token 0
        return (np.array([0]), 0.0, 0.0) if with_width else np.array([0])
    z = _values(row)
    zf = np.where(np.isfinite(z), z, 0.0)
    tz = np.abs(np.float64(np.float32(invT)) * LOG2E * zf)
    delta = 2.0 ** -40 * (tz + 1.0)
    lin = (np.log(2.0) * 2.0 ** -23 * tz) ** 2 / 2
    theta = np.exp2(delta) * (1.0 + lin) * (1.0 + POLY_REL) * (1.0 + 2.0 ** -24) - 1.0
    C = np.cumsum(w)
    E = np.cumsum(theta * w) + SUM_SLACK * S
    ES = float(E[-1])
    C_prev = np.concatenate([[0.0], C[:-1]])
    E_prev = np.concatenate([[0.0], E[:-1]])
    ok = (C_prev - E_prev <= u * (S + ES)) & (C + E > u * (S - ES)) & (w > 0.0)
    allowed = np.nonzero(ok)[0]
    if with_width:
        # probability mass of the allowed tokens strictly between the first
        # and the last one, against the width of the band they come from
        inner = float(C[allowed[-1] - 1] - C[allowed[0]]) / S if len(allowed) > 2 else 0.0
        return allowed, inner, 2.0 * (float(E[allowed[-1]]) + ES) / S
    return allowed


class DrawCount:
    """Draws checked, and draws whose allowed set held more than one token."""

    def __init__(self):
        self.draws = 0
        self.ambiguous = 0

    def add(self, allowed):
        self.draws += 1
        self.ambiguous += len(allowed) > 1


def check_sampled_walk(logits, tree, L, invT, seed, step, got, count=None):
    """Check a sampled walk ``got`` (numpy outputs of ddt_tree_walk_sample)
    decision by decision: every visited row's token is allowed by the error
    bound (and so is the oracle's exact draw), the walk descends to the child
    carrying it or stops there; a walk whose draws were all decided beyond
    rounding equals the oracle's walk exactly.  Returns the oracle's walk."""
    ref = oracle.tree_walk_sample(logits, tree["tok"], tree["parent"], tree["depth"],
                                  tree["n_nodes"], L, invT, seed, step)
    count = DrawCount() if count is None else count
    for b in range(logits.shape[0]):
        a = int(got["acc_len"][b])
        n = int(tree["n_nodes"][b])
        x = 0
        exact = True
        for i in range(a + 1):
            tk = int(got["acc_tok"][b][i]) if i < a else int(got["bonus"][b])
            u = oracle.row_uniform(seed, step, b, x)
            allowed, inner, width = allowed_tokens(logits[b, x], invT, u, with_width=True)
            t_ref, _ = oracle.sample_row(logits[b, x], invT, u)
            assert t_ref in allowed, (b, x, t_ref, allowed)
            assert tk in allowed, (b, x, tk, allowed)
            assert inner <= width, (b, x, inner, width)  # the set spans no more than the band
            count.add(allowed)
            exact = exact and len(allowed) == 1
            kids = [c for c in range(n) if tree["parent"][b][c] == x and tree["tok"][b][c] == tk]
            if i < a:
                assert kids and int(got["acc_nodes"][b][i]) == kids[0]
                x = kids[0]
            else:
                assert not kids or tree["depth"][b][x] >= L or a >= L
        if exact:
            for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
                np.testing.assert_array_equal(got[key][b], ref[key][b], err_msg="%s[%d]" % (key, b))
    return ref


# Shapes (batch, budget, context; b64 heads, L=6, V=400, k=4) that take each
# attention path on a B200; the plan depends on the device (SM count,
# co-resident clusters), so a test takes the first shape whose plan matches.
# Keys: the suffix of the binding's ATTN_PATH_* constant.
ATTN_PATH_SHAPES = {
    "TC_CLUSTER": [dict(batch=1, B=64, ctx=4096), dict(batch=1, B=40, ctx=2000),
                   dict(batch=2, B=30, ctx=3000)],
    "TC_COMBINE": [dict(batch=b, B=31, ctx=8192) for b in (20, 24, 30, 12)] +
                  [dict(batch=5, B=20, ctx=16384)],
    "TC": [dict(batch=37, B=31, ctx=500), dict(batch=74, B=20, ctx=300)],
    "TC_PAIRS": [dict(batch=37, B=63, ctx=500), dict(batch=37, B=127, ctx=500)],
    "TC_PAIRS_COMBINE": [dict(batch=2, B=63, ctx=16384), dict(batch=3, B=100, ctx=8192),
                         dict(batch=8, B=256, ctx=1000), dict(batch=16, B=63, ctx=16384)],
    "SIMT": [dict(batch=3, B=8, ctx=900)],
}
