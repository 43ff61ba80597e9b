"""Parity of ddt_topk (CUDA, through the C ABI) with the oracle's step 1.

Bit-exact: candidate ids and their raw logits.  Within the fp32 bound in
helpers.py: lse and logp.  Full-size draft logits of every workload, plus
ragged and degenerate rows (ties, constant rows, -inf entries, padded and
unaligned row strides)."""
import numpy as np
import pytest
import torch

import oracle
from block_draft_tree_b200 import api, synth

from helpers import LOGP_ATOL, LSE_ATOL, logits_tensor

pytestmark = pytest.mark.gpu


def _compare(z_np, k, inv_t, z_dev=None):
    ids, zk, logp, lse = oracle.topk(z_np, k, inv_t)
    t = logits_tensor(z_np) if z_dev is None else z_dev
    g_ids, g_zk, g_logp, g_lse = api.topk(t, k, inv_t)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(g_ids.cpu().numpy(), ids)
    np.testing.assert_array_equal(g_zk.cpu().numpy().astype(np.float64), zk)
    fin = np.isfinite(lse)
    np.testing.assert_allclose(g_lse.cpu().numpy()[fin], lse[fin], rtol=0, atol=LSE_ATOL)
    lp = logp[np.isfinite(logp)]
    np.testing.assert_allclose(g_logp.cpu().numpy()[np.isfinite(logp)], lp, rtol=0, atol=LOGP_ATOL)


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_workload_full_size(name):
    w = synth.WORKLOADS[name]
    z = synth.draft_logits(w)
    _compare(z, w.k, w.inv_temperature)


@pytest.mark.parametrize("V", [1, 7, 64, 1000, 8191, 8192, 8193, 20000, 65537])
@pytest.mark.parametrize("bf16", [True, False])
def test_ragged_vocab(V, bf16):
    g = np.random.default_rng(V)
    z = g.standard_normal((3, 5, V), dtype=np.float32) * 2
    z = synth.to_bf16_bits(z) if bf16 else z
    for k in sorted({1, min(8, V), min(32, V)}):
        _compare(z, k, 1.0)


@pytest.mark.parametrize("bf16", [True, False])
def test_ties_and_temperature(bf16):
    g = np.random.default_rng(1)
    z = g.integers(-3, 4, size=(2, 6, 30011)).astype(np.float32)
    z = synth.to_bf16_bits(z) if bf16 else z
    for it in (1.0, 0.7, 2.5):
        _compare(z, 32, it)


def test_constant_rows_take_the_fallback():
    z = np.full((1, 3, 50000), 1.5, np.float32)
    _compare(synth.to_bf16_bits(z), 16, 1.0)
    _compare(z, 32, 1.0)


def test_neg_inf_entries():
    g = np.random.default_rng(2)
    z = g.standard_normal((1, 4, 9000), dtype=np.float32)
    z[0, 0, :] = -np.inf
    z[0, 0, 17] = 0.5
    z[0, 1, 100:] = -np.inf
    _compare(z, 8, 1.0)


def test_padded_and_unaligned_rows():
    g = np.random.default_rng(3)
    V = 12345
    full = synth.to_bf16_bits(g.standard_normal((2, 3, V + 11), dtype=np.float32))
    dev = logits_tensor(full)[:, :, :V]  # row stride V+11: not 16-byte aligned
    _compare(np.ascontiguousarray(full[:, :, :V]), 8, 1.0, z_dev=dev)
    full32 = g.standard_normal((2, 3, V + 3), dtype=np.float32)
    dev32 = torch.from_numpy(full32).cuda()[:, :, :V]
    _compare(np.ascontiguousarray(full32[:, :, :V]), 8, 1.0, z_dev=dev32)


def test_repeated_calls_reuse_workspace():
    w = synth.WORKLOADS["b64"]
    z = synth.draft_logits(w)
    t = logits_tensor(z)
    first = api.topk(t, w.k)
    for _ in range(3):
        again = api.topk(t, w.k)
        torch.cuda.synchronize()
        assert torch.equal(first[0], again[0]) and torch.equal(first[3], again[3])
