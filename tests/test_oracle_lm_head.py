"""Pins of the oracle's LM-head decision and the walk over row tokens.

* logits: brute-force fp64 dot products (pure Python) on small shapes, and
  exactness: products of bf16 values are exact in fp64, so integer-valued
  inputs give integer logits exactly;
* argmax: constructed ties take the lowest id; the reported gap is the top
  logit minus the runner-up;
* walk: over the argmax tokens of one-hot logits it equals the pinned greedy
  walk (oracle.tree_walk) on those logits.
"""
import numpy as np

import oracle


def _bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_logits_are_exact_dot_products():
    rng = np.random.default_rng(0)
    h = _bits(rng.standard_normal((5, 24)))
    w = _bits(rng.standard_normal((17, 24)))
    tok, top, gap = oracle.lm_head_argmax(h, w)
    hf, wf = _f(h), _f(w)
    for r in range(5):
        logits = [sum(hf[r, k] * wf[v, k] for k in range(24)) for v in range(17)]
        best = max(range(17), key=lambda v: (logits[v], -v))
        assert tok[r] == best
        assert abs(top[r] - logits[best]) < 1e-12
        second = max(logits[v] for v in range(17) if v != best)
        assert abs(gap[r] - (logits[best] - second)) < 1e-12


def test_integer_inputs_give_exact_integer_logits_and_ties():
    h = _bits([[1, 2, 0, -1], [0, 0, 0, 0]])
    w = _bits([[3, 0, 1, 1], [1, 1, 0, 0], [2, 1, 5, 3], [0, 1, 1, -2]])
    tok, top, gap = oracle.lm_head_argmax(h, w)
    # row 0: logits 2, 3, 1, 4 -> token 3, gap 1; row 1: all zero -> token 0, gap 0
    assert list(tok) == [3, 0] and list(top) == [4.0, 0.0] and list(gap) == [1.0, 0.0]


def test_walk_over_row_tokens_equals_the_greedy_walk():
    rng = np.random.default_rng(4)
    V, L = 30, 4
    tok = np.array([[0, 5, 7, 2, 9, 4, 4, -1]], np.int32)
    parent = np.array([[-1, 0, 0, 1, 1, 2, 3, -1]], np.int32)
    depth = np.array([[0, 1, 1, 2, 2, 2, 3, 0]], np.int32)
    n = np.array([7], np.int32)
    for trial in range(30):
        row_tok = rng.integers(0, V, (1, 8)).astype(np.int32)
        if trial % 3 == 0:
            row_tok[0, 0], row_tok[0, 1], row_tok[0, 3] = 5, 2, 4  # a path to depth 3
        logits = np.full((1, 8, V), -1.0, np.float32)
        logits[0, np.arange(8), row_tok[0]] = 1.0
        a = oracle.walk_row_tokens(row_tok, tok, parent, depth, n, L)
        b = oracle.tree_walk(logits, tok, parent, depth, n, L)
        for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
            np.testing.assert_array_equal(a[key], b[key])


def test_vocabulary_blocks_change_nothing():
    """Blocking the vocabulary (for memory) gives the same tokens, tops and
    gaps, ties across block boundaries included."""
    rng = np.random.default_rng(2)
    h = _bits(rng.standard_normal((9, 40)))
    w = _bits(rng.standard_normal((700, 40)))
    w[650] = w[13]  # an exact tie across blocks: the lower id must win
    h[4] = _bits(np.ones(40))
    whole = oracle.lm_head_argmax(h, w)
    for block in (1, 64, 97, 700):
        part = oracle.lm_head_argmax(h, w, block=block)
        for x, y in zip(whole, part):
            np.testing.assert_array_equal(x, y)
