"""The seeded input generators (CPU): they draw and lay out random numbers
only, and every recipe property that the parity tests and the bench rely on
holds -- determinism, one independent stream per tensor, bf16 rounding to
nearest even, valid page placements, the ragged-context range, the spikes
and the Zipf profile of the drafts, and the planted agreement of the target."""
import numpy as np
import pytest
import torch

from block_draft_tree_b200 import synth

W = synth.WORKLOADS


def test_same_seed_same_inputs_other_seed_other_inputs():
    w = W["tiny"]
    a, b = synth.draft_logits(w), synth.draft_logits(w)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, synth.draft_logits(w, seed=w.seed + 1))
    x, y = synth.attention_inputs(w), synth.attention_inputs(w)
    for k in ("q", "k_cache", "v_cache", "k_tree", "v_tree", "ctx_len"):
        assert np.array_equal(x[k], y[k]), k


def test_each_tensor_has_its_own_stream():
    """A tensor's values do not depend on which other tensors were drawn, or
    in which order: q drawn alone equals q drawn after everything else."""
    w = W["tiny"].scaled(batch=2)
    alone = synth.to_bf16_bits(synth._normal(synth.rng(w, "q"), (w.batch, w.n_max, w.hq, w.d)))
    synth.draft_logits(w)
    synth.root_tokens(w)
    full = synth.attention_inputs(w)
    assert np.array_equal(full["q"], alone)
    assert not np.array_equal(full["k_tree"].ravel()[:64], full["v_tree"].ravel()[:64])


def test_bf16_rounding_is_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 100,
                        np.float32([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40, np.inf, -np.inf])])
    # halfway cases: the low 16 bits exactly 0x8000, with even and odd kept bits
    half = (np.array([0x3F808000, 0x3F818000, 0xBF808000, 0xBF818000], np.uint32)).view(np.float32)
    x = np.concatenate([x, half])
    got = synth.to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    assert np.array_equal(synth.bf16_bits_to_f32(got),
                          torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_paged_placement_uses_every_page_once():
    w = W["paged128"].scaled(batch=6, ctx=3000, ctx_min=65, L=4, B=8, hq=4, hkv=1, d=64)
    x = synth.attention_inputs(w)
    ctx, pt, ps = x["ctx_len"], x["page_table"], x["page_size"]
    assert ps == 64 and np.all(ctx >= 65) and np.all(ctx <= 3000)
    npg = (ctx + ps - 1) // ps
    assert pt.shape == (w.batch, npg.max())
    used = np.concatenate([pt[b, :npg[b]] for b in range(w.batch)])
    assert np.array_equal(np.sort(used), np.arange(npg.sum()))     # a permutation of the pool
    for b in range(w.batch):
        assert np.all(pt[b, npg[b]:] == -1)
    assert x["k_cache"].shape == (npg.sum(), ps, w.hkv, w.d) == x["v_cache"].shape


def test_ragged_contexts_span_their_range():
    w = W["paged128"]
    c = synth.context_lengths(w)
    assert c.shape == (32,) and c.dtype == np.int32
    assert np.all((c >= 1024) & (c <= 32768)) and len(np.unique(c)) > 16
    assert np.all(synth.context_lengths(W["b64"]) == 4096)


def test_spiked_drafts_have_their_spikes_at_distinct_tokens():
    w = W["tiny"].scaled(batch=3, L=5, V=512)
    z = synth.draft_logits(w)
    g = synth.rng(w, "draft")
    base = synth._normal(g, (w.batch, w.L, w.V))
    for b in range(w.batch):
        for i in range(w.L):
            toks = g.choice(w.V, size=2, replace=False)
            assert toks[0] != toks[1]
            diff = z[b, i] - base[b, i]
            assert np.flatnonzero(diff).tolist() == sorted(toks.tolist())
            assert diff[toks[0]] == pytest.approx(6.0) and diff[toks[1]] == pytest.approx(4.0)


def test_zipf_drafts_are_a_permuted_profile():
    w = W["paged128"].scaled(batch=2, L=3, V=1000, draft_dtype="f32")
    z = synth.draft_logits(w)
    prof = (-1.1 * np.log(np.arange(1, 1001, dtype=np.float64))).astype(np.float32)
    for row in z.reshape(-1, w.V):
        assert np.array_equal(np.sort(row)[::-1], prof)
    assert not np.array_equal(z[0, 0], z[0, 1])


def test_planted_target_agrees_with_one_child():
    """A planted row's maximum is one of its children's tokens, at least 2
    above the rest of the row; with agreement 1 and no decay every row with
    children is planted, with agreement 0 none is."""
    w = W["tiny"].scaled(batch=1, V=300, plant_p0=1.0, plant_decay=0.0)
    tok = np.array([[7, 11, 12, 13, 21, 22, 0, 0, 0]], np.int32)
    parent = np.array([[-1, 0, 0, 0, 1, 1, 0, 0, 0]], np.int32)
    depth = np.array([[0, 1, 1, 1, 2, 2, 0, 0, 0]], np.int32)
    n = np.array([6], np.int32)
    t = synth.target_logits(w, tok, parent, depth, n)
    assert t.shape == (1, w.n_max, w.V)
    for x, kids in ((0, [11, 12, 13]), (1, [21, 22])):
        row = t[0, x]
        top = int(np.argmax(row))
        assert top in kids
        rest = np.delete(row, top)
        assert row[top] >= np.float32(rest.max() + np.float32(2.0))
    t0 = synth.target_logits(w.scaled(plant_p0=0.0), tok, parent, depth, n)
    assert np.abs(t0[0, :2]).max() < 7.0   # plain N(0,1) noise in 300 draws per row
