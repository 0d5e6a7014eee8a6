"""Property-based checks of the oracle on tiny random shapes (CPU): each
property follows from the definitions, independent of how the oracle
computes them."""
import math

import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
import synth


def bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, np.float32))


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 48), st.integers(1, 20), st.integers(0, 2**31 - 1), st.integers(0, 48))
def test_topk_is_the_stable_sort_prefix(n, k, seed, n_valid):
    """Top-k = the first min(k, n_valid) entries of the sort by (score
    descending, index ascending), emitted in ascending index order, padded
    with -1.  Scores drawn from a few values so that ties are common."""
    n_valid = min(n_valid, n)
    rng = np.random.default_rng(seed)
    s = rng.integers(-3, 4, n).astype(np.float32) / 2
    got = oracle.topk(s[None], [n_valid], k)[0]
    order = sorted(range(n_valid), key=lambda i: (-float(s[i]), i))[:k]
    want = np.full(k, -1, np.int32)
    want[: len(order)] = sorted(order)
    assert np.array_equal(got, want)


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 40), st.integers(1, 6), st.integers(0, 2**31 - 1))
def test_attention_is_invariant_to_selection_order_and_duplicate_padding(S, k, seed):
    """Softmax attention over a set of keys: permuting the selected entries
    or appending -1 padding changes nothing."""
    rng = np.random.default_rng(seed)
    d, Hq, Hkv = 8, 2, 1
    k = min(k, S)
    Q = bf16(rng.standard_normal((1, 1, Hq, d)))
    K = bf16(rng.standard_normal(S * Hkv * d))
    V = bf16(rng.standard_normal(S * Hkv * d))
    sel = rng.choice(S, k, replace=False).astype(np.int32)
    a = oracle.sparse_decode_attn(Q, K, V, [0, S], [S], np.sort(sel)[None], Hkv, 1 / math.sqrt(d))
    perm = rng.permutation(sel)
    padded = np.concatenate([perm, np.full(3, -1, np.int32)])[None]
    b = oracle.sparse_decode_attn(Q, K, V, [0, S], [S], padded, Hkv, 1 / math.sqrt(d))
    assert np.allclose(a, b, rtol=0, atol=1e-12)


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 12), st.integers(64, 700), st.integers(1, 40), st.integers(0, 2**31 - 1))
def test_block_union_covers_exactly_the_selected_blocks(Nq, S, k, seed):
    """The table of every group is the sorted set of blocks holding a
    selected token: every selected token's block is listed (coverage) and
    every listed block holds one (minimality)."""
    rng = np.random.default_rng(seed)
    k = min(k, S)
    idx = np.stack([rng.choice(S, k, replace=False) for _ in range(Nq)]).astype(np.int32)
    idx[rng.random(idx.shape) < 0.1] = -1
    ptr, ind = oracle.block_union(idx, S, 64, 2)
    want = sorted({int(t) // 64 for t in idx.ravel() if t >= 0})
    assert ptr[0] == 0 and ptr[1] - ptr[0] == len(want) and ptr[2] - ptr[1] == len(want)
    assert list(ind[: len(want)]) == want and list(ind[len(want): 2 * len(want)]) == want


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 30), st.integers(1, 4), st.integers(0, 2**31 - 1))
def test_index_score_is_monotone_in_each_head_weight(S, H_I, seed):
    """Raising one head's weight never lowers a score (ReLU terms are >= 0),
    and scaling every weight by 2 doubles every score exactly."""
    rng = np.random.default_rng(seed)
    d_I = 8
    qI = bf16(rng.standard_normal((1, H_I, d_I)) / 4)
    KI = bf16(rng.standard_normal((S, d_I)) / 4)
    w = rng.uniform(0.1, 1.0, (1, H_I)).astype(np.float32)
    base = oracle.index_score(qI, w, KI, [0, S], [0], [S - 1])[0][:S]
    w2 = w.copy()
    w2[0, rng.integers(H_I)] *= 1.5
    up = oracle.index_score(qI, w2, KI, [0, S], [0], [S - 1])[0][:S]
    assert np.all(up >= base)
    dbl = oracle.index_score(qI, 2 * w, KI, [0, S], [0], [S - 1])[0][:S]
    assert np.array_equal(dbl, 2 * base)


@settings(max_examples=60, deadline=None)
@given(st.lists(st.integers(0, 40), min_size=1, max_size=4), st.integers(1, 6), st.integers(1, 12),
       st.integers(0, 2**31 - 1))
def test_slice_candidates_select_the_whole_context_topk(lens, N, k, seed):
    """Context-parallel selection: for any slicing of each context into N
    contiguous pieces, the union of every rank's share of the selection over
    the slices' top-k candidates is the top-k of the whole context (stable
    sort prefix), and each share is ascending then -1."""
    rng = np.random.default_rng(seed)
    B = len(lens)
    full = [rng.integers(-2, 3, n).astype(np.float32) / 2 for n in lens]
    cuts = [np.sort(np.concatenate([[0, n], rng.integers(0, n + 1, N - 1)])) for n in lens]
    cand_s = np.zeros((N, B, k), np.float32)
    cand_i = np.zeros((N, B, k), np.int32)
    for r in range(N):
        w = max(1, max(int(c[r + 1] - c[r]) for c in cuts))
        sc = np.zeros((B, w), np.float32)
        nv = []
        for b in range(B):
            lo, hi = int(cuts[b][r]), int(cuts[b][r + 1])
            sc[b, :hi - lo] = full[b][lo:hi]
            nv.append(hi - lo)
        cand_i[r], cand_s[r] = oracle.topk(sc, nv, k, with_scores=True)
    got = [[] for _ in range(B)]
    for r in range(N):
        share = oracle.cp_select(cand_s, cand_i, r)
        for b in range(B):
            row = [int(t) for t in share[b] if t >= 0]
            assert row == sorted(row) and all(t < 0 for t in share[b][len(row):])
            got[b] += [int(cuts[b][r]) + t for t in row]
    for b in range(B):
        want = sorted(sorted(range(lens[b]), key=lambda t: (-float(full[b][t]), t))[:k])
        assert sorted(got[b]) == want


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 6), st.integers(1, 5), st.integers(0, 2**31 - 1))
def test_combine_is_order_free_and_splits_compose(P, rows, seed):
    """The log-sum-exp merge does not depend on the order of the parts, and
    merging two parts first (a part's (m, l, o) after a merge is (M, L, O*L))
    then the rest gives the same as merging all at once."""
    rng = np.random.default_rng(seed)
    d = 4
    l = rng.uniform(0.5, 4, (P, rows))
    l[rng.random((P, rows)) < 0.2] = 0.0
    m = rng.uniform(-6, 6, (P, rows))
    m[l == 0] = -np.inf
    o = rng.standard_normal((P, rows, d)) * l[..., None]
    ml = np.stack([m, l], -1)
    whole = oracle.combine_partials(o, ml)
    perm = rng.permutation(P)
    np.testing.assert_allclose(oracle.combine_partials(o[perm], ml[perm]), whole, rtol=1e-12, atol=1e-12)
    if P >= 2:
        first = oracle.combine_partials(o[:2], ml[:2])
        M = np.max(np.where(ml[:2, :, 1] > 0, ml[:2, :, 0], -np.inf), axis=0)
        L = np.sum(np.where(ml[:2, :, 1] > 0, np.exp2(ml[:2, :, 0] - np.where(np.isfinite(M), M, 0)) * ml[:2, :, 1],
                            0), axis=0)
        merged_ml = np.stack([np.where(L > 0, M, -np.inf), L], -1)[None]
        merged_o = (first * L[:, None])[None]
        again = oracle.combine_partials(np.concatenate([merged_o, o[2:]]), np.concatenate([merged_ml, ml[2:]]))
        np.testing.assert_allclose(again, whole, rtol=1e-10, atol=1e-12)


def _osk_inputs(rng, Nq, Hq, Hkv, S, d, block):
    q_pos = np.sort(rng.choice(S, Nq, replace=False)).astype(np.int32)
    Q = bf16(rng.standard_normal((Nq, Hq, d)) * 2)
    K = bf16(rng.standard_normal((Hkv, S, d)))
    V = bf16(rng.standard_normal((Hkv, S, d)))
    return q_pos, Q, K, V


@settings(max_examples=30, deadline=None)
@given(st.integers(1, 6), st.sampled_from([(2, 1), (4, 2), (2, 2)]), st.integers(40, 400), st.integers(1, 3),
       st.integers(0, 2**31 - 1))
def test_osk_steps_fall_as_tau_rises_and_the_rule_holds(Nq, heads, S, q_block, seed):
    """Ordered skipping: the step count of every unit is non-increasing in
    tau (the first step below a larger tau comes no later), tau = 0 runs
    every step, and each count satisfies the rule against the unit's
    per-step scores."""
    Hq, Hkv = heads
    block, d, lag = 8, 4, 2
    rng = np.random.default_rng(seed)
    q_pos, Q, K, V = _osk_inputs(rng, Nq, Hq, Hkv, S, d, block)
    nb = (S + block - 1) // block
    n_qb = (Nq + q_block - 1) // q_block
    order = np.stack([rng.permutation(nb) for _ in range(n_qb)]).astype(np.int32)
    n_steps = (nb + 1) // 2
    prev = None
    for tau in (0.0, 0.01, 0.1, 0.3, 0.7, 1.5):
        _, steps, crit = oracle.osk_prefill_attn(Q, q_pos, K, V, block, order, q_block, 0.5, tau, lag=lag)
        if tau == 0.0:
            assert np.all(steps == n_steps)
        for u, N in enumerate(steps):
            below = np.nonzero(crit[u] < tau)[0]
            want = n_steps if below.size == 0 else min(n_steps, int(below[0]) + 1 + lag)
            assert N == want
        if prev is not None:
            assert np.all(steps <= prev)
        prev = steps


@settings(max_examples=25, deadline=None)
@given(st.integers(1, 5), st.integers(30, 300), st.integers(0, 2**31 - 1))
def test_osk_without_skipping_ignores_the_order(Nq, S, seed):
    """tau = 0 runs every step, so any two orders of the same table give the
    same softmax over the same keys."""
    rng = np.random.default_rng(seed)
    block, d, Hq, Hkv, q_block = 8, 4, 2, 1, 2
    q_pos, Q, K, V = _osk_inputs(rng, Nq, Hq, Hkv, S, d, block)
    nb = (S + block - 1) // block
    n_qb = (Nq + q_block - 1) // q_block
    T = np.sort(rng.choice(nb, max(1, nb // 2), replace=False)).astype(np.int32)
    o1 = np.stack([rng.permutation(T) for _ in range(n_qb)]).astype(np.int32)
    o2 = np.stack([rng.permutation(T) for _ in range(n_qb)]).astype(np.int32)
    A, _, _ = oracle.osk_prefill_attn(Q, q_pos, K, V, block, o1, q_block, 0.5, 0.0)
    B, _, _ = oracle.osk_prefill_attn(Q, q_pos, K, V, block, o2, q_block, 0.5, 0.0)
    np.testing.assert_allclose(A, B, rtol=0, atol=1e-12)
