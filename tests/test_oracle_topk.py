"""Pins for the oracle's step 1 (softmax + per-position top-k).

DDTree page, section 運作流程 step 1: one marginal q_i per position.  The
candidate list is the top-k of q_i by (logit desc, token id asc); lse is the
log normaliser of the tempered softmax.  The pins: a library sort
(numpy.lexsort), a library log-sum-exp (torch.logsumexp in fp64), and the
closed form of a constant row.
"""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import synth


def _as_f64(z):
    return synth.bf16_bits_to_f32(z).astype(np.float64) if z.dtype == np.uint16 else z.astype(np.float64)


def _inputs(seed, rows, V, ties, bf16):
    g = np.random.default_rng(seed)
    if ties:
        z = g.integers(-3, 4, size=(rows, V)).astype(np.float32)
    else:
        z = g.standard_normal((rows, V), dtype=np.float32) * 3
    return synth.to_bf16_bits(z) if bf16 else z


@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("V,k", [(64, 4), (1000, 16), (4099, 32), (40, 40)])
def test_ids_match_library_sort(ties, bf16, V, k):
    z = _inputs(V * 7 + k, 6, V, ties, bf16)
    ids, zk, logp, lse = oracle.topk(z, k, 1.0)
    zf = _as_f64(z)
    for r in range(z.shape[0]):
        order = np.lexsort((np.arange(V), -zf[r]))  # primary: -z, secondary: id
        np.testing.assert_array_equal(ids[r], order[:k])
        np.testing.assert_array_equal(zk[r], zf[r, order[:k]])


@pytest.mark.parametrize("inv_t", [1.0, 1.0 / 0.7, 0.25, 3.0])
def test_lse_and_logp_match_library_logsumexp(inv_t):
    z = _inputs(11, 5, 3001, False, True)
    ids, zk, logp, lse = oracle.topk(z, 8, inv_t)
    it = float(np.float32(inv_t))
    u = torch.tensor(_as_f64(z) * it, dtype=torch.float64)
    ref = torch.logsumexp(u, dim=-1).numpy()
    np.testing.assert_allclose(lse, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(logp, zk * it - lse[:, None], rtol=0, atol=1e-12)
    # the candidates' probabilities are the library softmax at those ids
    sm = torch.softmax(u, dim=-1).numpy()
    np.testing.assert_allclose(np.exp(logp), np.take_along_axis(sm, ids.astype(np.int64), 1),
                               rtol=1e-12, atol=0)


def test_temperature_does_not_reorder():
    z = _inputs(5, 4, 777, True, True)
    a = oracle.topk(z, 12, 1.0)[0]
    b = oracle.topk(z, 12, 0.3)[0]
    c = oracle.topk(z, 12, 5.0)[0]
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(a, c)


@pytest.mark.parametrize("c", [0.0, -7.5, 3.25])
def test_constant_row_closed_form(c):
    V, k = 300, 10
    z = np.full((2, V), c, np.float32)
    ids, zk, logp, lse = oracle.topk(z, k, 2.0)
    np.testing.assert_array_equal(ids, np.tile(np.arange(k), (2, 1)))
    np.testing.assert_allclose(lse, 2.0 * c + np.log(V), atol=1e-12)
    np.testing.assert_allclose(logp, -np.log(V), atol=1e-12)


def test_single_spike_probability():
    # one token at +s over V-1 zeros: q = e^s / (e^s + V - 1)
    V, s = 1000, 6.0
    z = np.zeros((1, V), np.float32)
    z[0, 123] = s
    ids, zk, logp, lse = oracle.topk(z, 3, 1.0)
    assert ids[0, 0] == 123 and list(ids[0, 1:]) == [0, 1]
    np.testing.assert_allclose(np.exp(logp[0, 0]), np.exp(s) / (np.exp(s) + V - 1), rtol=1e-12)
