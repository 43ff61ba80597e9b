"""Pins of the oracle's sampled walk (target temperature > 0).

The DDTree page (workflow, step 4) has the walk follow the target's decoding
rule and stresses that the output distribution is preserved; under sampling
that rule draws each token from softmax(z / T).  The oracle draws by
inversion with one Philox4x64-10 uniform per (sequence, tree row).  These
tests tie each piece to something other than the oracle itself:

* the generator to numpy's independent Philox4x64-10 bit generator;
* the draw's fp64 weights to scipy's softmax, and the draw to closed forms
  (equal logits, two tokens) and to numpy's
  cumulative sum + searchsorted over scipy's softmax;
* the walk to the greedy walk in the zero-temperature limit and, by Monte
  Carlo, to the target's own autoregressive sampling (losslessness).
"""
import math

import numpy as np
import pytest
from scipy import special, stats

import oracle

U64 = (1 << 64) - 1


def _numpy_block(ctr, key):
    """numpy's Philox advances its 256-bit counter before each block, so the
    block at counter c comes from a generator started at c - 1."""
    c = [int(x) for x in ctr]
    for i in range(4):  # subtract one with borrow
        if c[i] > 0:
            c[i] -= 1
            break
        c[i] = U64
    return np.random.Philox(counter=np.array(c, np.uint64),
                            key=np.array([int(k) for k in key], np.uint64)).random_raw(4)


def test_philox_matches_numpy():
    rng = np.random.default_rng(11)
    cases = [([0, 0, 0, 0], [0, 0]), ([1, 0, 0, 0], [0, 0]), ([U64] * 4, [U64, U64]),
             ([0, 1, 0, 0], [5, 9])]
    for _ in range(16):
        cases.append((rng.integers(0, 1 << 63, 4, dtype=np.uint64) * 2 + 1,
                      rng.integers(0, 1 << 63, 2, dtype=np.uint64)))
    for ctr, key in cases:
        assert np.array_equal(oracle.philox4x64_10(ctr, key), _numpy_block(ctr, key)), (ctr, key)


def test_word_to_uniform_range_and_order():
    assert oracle.word_to_uniform(0) == 2.0 ** -53
    assert oracle.word_to_uniform(U64) == 1.0 - 2.0 ** -53 < 1.0
    ws = sorted(np.random.default_rng(2).integers(0, 1 << 63, 50, dtype=np.uint64).tolist())
    us = [oracle.word_to_uniform(w * 2) for w in ws]
    assert all(0.0 < a <= b < 1.0 for a, b in zip(us, us[1:]))


@pytest.mark.parametrize("seed,step,b,j", [(0, 0, 0, 0), (7, 3, 2, 5), (2**63 + 1, 2**40, 31, 512)])
def test_row_uniform_is_word0_of_the_row_counter(seed, step, b, j):
    w = int(_numpy_block([j, b, 0, 0], [seed, step])[0])
    assert oracle.row_uniform(seed, step, b, j) == ((w >> 12) + 0.5) * 2.0 ** -52
    # every argument reaches the counter or the key
    others = {oracle.row_uniform(seed + 1, step, b, j), oracle.row_uniform(seed, step + 1, b, j),
              oracle.row_uniform(seed, step, b + 1, j), oracle.row_uniform(seed, step, b, j + 1)}
    assert oracle.row_uniform(seed, step, b, j) not in others and len(others) == 4


@pytest.mark.parametrize("V,z,invT", [(1000, 0.37, 1.0), (151936, -2.5, 1 / 0.7), (7, 0.0, 3.0)])
def test_equal_logits_draw_floor_uV(V, z, invT):
    """Equal logits: every weight is exactly 1, so C_v = v + 1 and the draw is floor(u*V)."""
    row = np.full(V, z, np.float32)
    for u in np.random.default_rng(V).random(40).tolist() + [2.0 ** -53, 1 - 2.0 ** -53]:
        t, mg = oracle.sample_row(row, invT, u)
        assert t == math.floor(u * V)
        assert mg == pytest.approx(min(u * V - t, t + 1 - u * V) / V, abs=1e-15)


@pytest.mark.parametrize("invT", [1.0, 1 / 0.7, 4.0])
def test_sampler_weights_are_the_softmax(invT):
    """Normalised, the draw's weights are scipy's softmax of invT * z (invT
    rounded to fp32, as the C ABI takes it), to fp64 rounding; -inf logits
    weigh 0 and the largest logit weighs exactly 1."""
    rng = np.random.default_rng(3)
    z = (rng.standard_normal(5000) * 3).astype(np.float32)
    z[::97] = -np.inf
    w = oracle.sampler_row_weights(z, invT)
    fin = np.isfinite(z)
    assert np.all(w[~fin] == 0.0) and np.all(w[fin] > 0.0)
    assert w[np.argmax(np.where(fin, z, -np.inf))] == 1.0
    ref = special.softmax(np.float64(np.float32(invT)) * z[fin].astype(np.float64))
    np.testing.assert_allclose(w[fin] / w.sum(), ref, rtol=1e-12, atol=0)


def test_two_tokens_closed_form():
    row = np.array([0.0, 1.5], np.float32)
    for invT in (1.0, 0.5, 2.0):
        p0 = 1.0 / (1.0 + math.exp(1.5 * invT))
        assert oracle.sample_row(row, invT, p0 - 1e-9)[0] == 0
        assert oracle.sample_row(row, invT, p0 + 1e-9)[0] == 1
        assert oracle.sample_row(row, invT, 1e-12)[0] == 0
        assert oracle.sample_row(row, invT, 1 - 1e-12)[0] == 1


@pytest.mark.parametrize("dtype", [np.float32, "bf16"])
def test_draw_is_inverse_cdf_of_softmax(dtype):
    rng = np.random.default_rng(5)
    V = 300
    zf = (rng.standard_normal(V) * 2).astype(np.float32)
    zf[rng.integers(0, V, 3)] += 5.0
    if dtype == "bf16":
        bits = (zf.view(np.uint32) >> 16).astype(np.uint16)
        row, zval = bits, (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    else:
        row, zval = zf, zf.astype(np.float64)
    for invT in (1.0, 1 / 0.7, 0.25):
        cdf = np.cumsum(special.softmax(zval * np.float64(np.float32(invT))))
        for u in rng.random(300):
            t, mg = oracle.sample_row(row, invT, float(u))
            if np.min(np.abs(cdf - u)) < 1e-12:
                continue
            assert t == int(np.searchsorted(cdf, u, side="right"))
            lo = cdf[t - 1] if t > 0 else 0.0
            assert mg == pytest.approx(min(u - lo, cdf[t] - u), abs=1e-12)


def test_masked_tokens_are_never_drawn_and_empty_row():
    row = np.full(64, -np.inf, np.float32)
    row[[3, 40, 41]] = [0.5, 0.5, 2.0]
    for u in np.linspace(1e-9, 1 - 1e-9, 200):
        assert oracle.sample_row(row, 1.0, float(u))[0] in (3, 40, 41)
    t, mg = oracle.sample_row(np.full(8, -np.inf, np.float32), 1.0, 0.5)
    assert t == 0 and mg == math.inf


def _chain_tree(tokens):
    """A chain root -> tokens[0] -> tokens[1] ... in breadth-first layout."""
    n = len(tokens) + 1
    tok = np.array([0] + list(tokens), np.int32)
    parent = np.arange(-1, n - 1, dtype=np.int32)
    depth = np.arange(n, dtype=np.int32)
    return tok, parent, depth


def test_zero_temperature_limit_is_the_greedy_walk():
    rng = np.random.default_rng(9)
    V, L = 50, 6
    for trial in range(20):
        chain = rng.integers(0, V, L).tolist()
        tok, parent, depth = _chain_tree(chain)
        n = L + 1
        logits = rng.standard_normal((1, n, V)).astype(np.float32)
        for j in range(n - 1):  # make the target agree on a random prefix of the chain
            if rng.random() < 0.8:
                logits[0, j, chain[j]] = logits[0, j].max() + 1.0
        g = oracle.tree_walk(logits, tok[None], parent[None], depth[None], [n], L)
        s = oracle.tree_walk_sample(logits, tok[None], parent[None], depth[None], [n], L,
                                    1e5, seed=trial, step=0)
        for key in ("acc_len", "acc_nodes", "acc_tok", "bonus"):
            assert np.array_equal(g[key], s[key]), key


def test_walk_draws_each_visited_row_with_its_own_uniform():
    """Sequence b's walk draws row x with row_uniform(seed, step, b, x): the
    sequences of a batch and the rows of one walk use different uniforms."""
    V, L, B = 5, 3, 4
    tok, parent, depth = _chain_tree([1, 2, 3])
    n = L + 1
    logits = np.zeros((B, n, V), np.float32)  # uniform target: draws are floor(u*V)
    res = oracle.tree_walk_sample(logits, np.tile(tok, (B, 1)), np.tile(parent, (B, 1)),
                                  np.tile(depth, (B, 1)), [n] * B, L, 1.0, seed=77, step=5)
    for b in range(B):
        x, emitted = 0, []
        while True:
            t = math.floor(oracle.row_uniform(77, 5, b, x) * V)
            emitted.append(t)
            if x < L and tok[x + 1] == t:
                x += 1
            else:
                break
        a = int(res["acc_len"][b])
        assert list(res["acc_tok"][b][:a]) + [int(res["bonus"][b])] == emitted


def test_sampled_walk_is_lossless():
    """Monte Carlo: the first two emitted tokens of a round follow the
    target's own two-step sampling, whatever the tree holds."""
    V, T = 3, 0.8
    # target logits depend only on the prefix after the root
    target = {(): np.array([0.2, 1.0, -0.5]), (0,): np.array([1.5, 0.0, 0.3]),
              (1,): np.array([-1.0, 0.7, 0.9]), (2,): np.array([0.0, 0.0, 0.0])}
    # tree: root -> {1, 2}, 1 -> {2}; rows in breadth-first order
    tok = np.array([0, 1, 2, 2], np.int32)
    parent = np.array([-1, 0, 0, 1], np.int32)
    depth = np.array([0, 1, 1, 2], np.int32)
    logits = np.zeros((1, 4, V), np.float32)
    logits[0, 0] = target[()]
    logits[0, 1] = target[(1,)]
    logits[0, 2] = target[(2,)]
    logits[0, 3] = np.array([0.3, -0.2, 0.1])  # row after (1, 2): only its bonus is drawn
    logits = logits.astype(np.float32)
    p1 = special.softmax(target[()].astype(np.float32).astype(np.float64) / T)
    p2 = {t: special.softmax(target[(t,)].astype(np.float32).astype(np.float64) / T) for t in (1, 2)}
    n_draws = 6000
    first = np.zeros(V)
    second = {1: np.zeros(V), 2: np.zeros(V)}
    for s in range(n_draws):
        r = oracle.tree_walk_sample(logits, tok[None], parent[None], depth[None], [4], 2,
                                    1 / T, seed=1234, step=s)
        a = int(r["acc_len"][0])
        em = list(r["acc_tok"][0][:a]) + [int(r["bonus"][0])]
        first[em[0]] += 1
        if em[0] in (1, 2):
            second[em[0]][em[1]] += 1
    assert stats.chisquare(first, p1 * n_draws).pvalue > 1e-4
    for t in (1, 2):
        tot = second[t].sum()
        assert tot > 500
        assert stats.chisquare(second[t], p2[t] * tot).pvalue > 1e-4


def test_draw_bound_is_narrow_and_catches_a_wrong_weight():
    """The bound the GPU parity applies to sampled draws (helpers.allowed_tokens)
    always holds the exact draw, leaves one token for three draws in four over
    a 151936-token row, and rejects draws made from wrong weights: a
    temperature off by 0.1 %, or one 8192-token chunk scaled by 1.001 (as a
    wrong power-of-two merge or a lost term in one chunk would make it)."""
    from helpers import allowed_tokens
    rng = np.random.default_rng(17)
    V = 151936
    z = rng.standard_normal(V).astype(np.float32)
    z[rng.integers(0, V, 3)] += 6.0
    zd = z.astype(np.float64)
    w_scale = np.cumsum(np.exp((1.0 + 1e-3) * (zd - zd.max())))
    w_chunk = np.exp(zd - zd.max())
    w_chunk[5 * 8192:6 * 8192] *= 1.001
    w_chunk = np.cumsum(w_chunk)
    n = 200
    single = caught_scale = caught_chunk = 0
    for u in rng.random(n):
        allowed = allowed_tokens(z, 1.0, float(u))
        t, _ = oracle.sample_row(z, 1.0, float(u))
        assert t in allowed
        single += len(allowed) == 1
        caught_scale += int(np.searchsorted(w_scale, u * w_scale[-1], side="right")) not in allowed
        caught_chunk += int(np.searchsorted(w_chunk, u * w_chunk[-1], side="right")) not in allowed
    assert single >= 0.75 * n
    assert caught_scale >= 0.2 * n and caught_chunk >= 0.5 * n
