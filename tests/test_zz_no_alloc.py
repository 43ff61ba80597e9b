"""ddt_topk_noalloc: the top-k entry point for callers that cannot allocate
device memory (code running under a memory manager that owns the whole heap,
an embedded runtime with a fixed memory plan, a plug-in whose host forbids
cudaMalloc).  Its scratch is a fixed device array inside libddt.so.

Checked through the C ABI against ddt_topk (the entry point that takes a
caller workspace) on two calls in a row with different shapes, within the
tolerances the other top-k tests use.  This file runs last so that a failure
here leaves every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_draft_tree_b200 import api, synth

from helpers import LOGP_ATOL, LSE_ATOL, logits_tensor

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20
DDT_ERR_WORKSPACE = 3


def _entry():
    lib = api.load_library()
    f = lib.ddt_topk_noalloc
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                  ctypes.c_int, ctypes.c_float, vp, vp, vp, vp, vp]
    return f


def _noalloc(t, k, inv_t):
    b, L, V = t.shape
    ids = torch.empty((b, L, k), dtype=torch.int32, device=t.device)
    zk = torch.empty((b, L, k), dtype=torch.float32, device=t.device)
    logp = torch.empty((b, L, k), dtype=torch.float32, device=t.device)
    lse = torch.empty((b, L), dtype=torch.float32, device=t.device)
    code = 0 if t.dtype == torch.bfloat16 else 1
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _entry()(ctypes.c_void_p(t.data_ptr()), code, b, L, V, t.stride(1), k, float(inv_t),
                  ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(zk.data_ptr()),
                  ctypes.c_void_p(logp.data_ptr()), ctypes.c_void_p(lse.data_ptr()), stream)
    assert rc == 0, api.load_library().ddt_status_string(rc)
    return ids, zk, logp, lse


def _same(a, b):
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0])
    assert torch.equal(a[1], b[1])
    assert (a[2] - b[2]).abs().max().item() <= LOGP_ATOL
    assert (a[3] - b[3]).abs().max().item() <= LSE_ATOL


def test_matches_workspace_entry_point_on_two_calls():
    w1 = synth.WORKLOADS["b64"]
    w2 = synth.WORKLOADS["paged128"].scaled(batch=6)  # another shape, Zipf rows, temperature
    t1 = logits_tensor(synth.draft_logits(w1))
    t2 = logits_tensor(synth.draft_logits(w2))
    n1 = _noalloc(t1, w1.k, w1.inv_temperature)
    n2 = _noalloc(t2, w2.k, w2.inv_temperature)
    _same(n1, api.topk(t1, w1.k, w1.inv_temperature))
    _same(n2, api.topk(t2, w2.k, w2.inv_temperature))


def test_rejects_shapes_beyond_the_scratch():
    lib = api.load_library()
    b, L, V, k = 4095, 16, 151936, 32  # 65520 rows of partials
    assert lib.ddt_topk_workspace_size(b, L, V, k) > SCRATCH_BYTES
    dummy = ctypes.c_void_p(256)
    rc = _entry()(dummy, 0, b, L, V, V, k, 1.0, dummy, dummy, dummy, dummy, None)
    assert rc == DDT_ERR_WORKSPACE
