"""Pins for the CPU oracle: each test ties it to something other than itself.

The pages print no worked example, so the pins are closed forms, brute force
on tiny inputs, special cases that reduce to a library routine (torch fp64
softmax attention), exact rational arithmetic, and invariants that the
definitions imply.  Each is chosen so that a plausible slip in the oracle
(dropped ReLU, wrong head weight, transposed operand, wrong GQA map, wrong
tie rule, off-by-one visibility, wrong block map) fails at least one.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import bf16_bits_to_f32, f32_to_bf16_bits


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


# ----------------------------------------------------------------------------
# indexer score
# ----------------------------------------------------------------------------
def test_index_one_hot_closed_form():
    # q_j = e_{a_j}, k_t = 2 e_{t mod 8}: dot_j = 2 [a_j == t mod 8], score = 2 w_j of that head
    d_I, H_I, S = 8, 3, 24
    a = [1, 4, 6]
    qI = np.zeros((1, H_I, d_I), np.float32)
    for j, aj in enumerate(a):
        qI[0, j, aj] = 1.0
    KI = np.zeros((S, d_I), np.float32)
    for t in range(S):
        KI[t, t % 8] = 2.0
    w = np.array([[0.25, 0.5, 0.875]], np.float32)
    s = oracle.index_score(bf(qI), w, bf(KI), [0, S], [0], [S - 1])[0]
    for t in range(S):
        want = 2.0 * w[0, a.index(t % 8)] if (t % 8) in a else 0.0
        assert s[t] == np.float32(want), t


def test_index_relu_sign_and_positive_zero():
    # q_0 = +1, q_1 = -1, q_2 = +0.5 (all coords), k_t = (t-3) (all coords)
    # dot_j = d*s_j*c_t ; score = d*c_t*(w0 + 0.5 w2) for c_t>0, d*|c_t|*w1 for c_t<0, +0 at c_t=0
    d_I, S = 4, 8
    sj = [1.0, -1.0, 0.5]
    qI = np.array([[[v] * d_I for v in sj]], np.float32)
    KI = np.array([[t - 3.0] * d_I for t in range(S)], np.float32)
    w = np.array([[0.5, 0.25, 1.0]], np.float32)
    s = oracle.index_score(bf(qI), w, bf(KI), [0, S], [0], [S - 1])[0]
    for t in range(S):
        c = t - 3
        if c > 0:
            want = d_I * c * (0.5 + 0.5 * 1.0)
        elif c < 0:
            want = d_I * (-c) * 0.25
        else:
            want = 0.0
        assert s[t] == np.float32(want)
    assert np.float32(s[3]).view(np.uint32) == 0, "score must be +0, not -0"


def test_index_visibility_and_sequence_offsets():
    # two packed sequences with constant keys 1 and 3; query b reads only its own
    # sequence and only keys t <= q_pos
    d_I, H_I = 4, 2
    S0, S1 = 5, 7
    KI = np.concatenate([np.full((S0, d_I), 1.0), np.full((S1, d_I), 3.0)]).astype(np.float32)
    qI = np.ones((2, H_I, d_I), np.float32)
    w = np.array([[1.0, 0.5], [0.25, 0.125]], np.float32)
    s = oracle.index_score(bf(qI), w, bf(KI), [0, S0, S0 + S1], [0, 1], [2, 6], ld=8)
    assert np.all(s[0, :3] == np.float32(d_I * 1.0 * 1.5))
    assert np.all(np.isnan(s[0, 3:])), "keys past q_pos must not be written"
    assert np.all(s[1, :7] == np.float32(d_I * 3.0 * 0.375))
    assert np.isnan(s[1, 7])


def test_index_exact_rational_arithmetic():
    # the oracle's fp32 score is the exact real score rounded once (allow one ulp)
    rng = np.random.default_rng(7)
    H_I, d_I, S = 4, 16, 32
    qI = bf(rng.standard_normal((1, H_I, d_I)) / 8)
    KI = bf(rng.standard_normal((S, d_I)) / 8)
    w = rng.uniform(0.1, 1.0, (1, H_I)).astype(np.float32)
    s = oracle.index_score(qI, w, KI, [0, S], [0], [S - 1])[0]
    qf = bf16_bits_to_f32(qI)[0]
    kf = bf16_bits_to_f32(KI)
    for t in range(S):
        exact = Fraction(0)
        for j in range(H_I):
            dot = sum(Fraction(float(qf[j, c])) * Fraction(float(kf[t, c])) for c in range(d_I))
            exact += Fraction(float(w[0, j])) * max(dot, Fraction(0))
        ulp = np.spacing(np.float32(float(exact)))
        assert abs(Fraction(float(s[t])) - exact) <= Fraction(float(ulp)), t


def test_index_weight_scaling_and_head_permutation():
    rng = np.random.default_rng(3)
    H_I, d_I, S = 5, 32, 40
    qI = bf(rng.standard_normal((1, H_I, d_I)) / 8)
    KI = bf(rng.standard_normal((S, d_I)) / 8)
    w = rng.uniform(0.1, 1.0, (1, H_I)).astype(np.float32)
    base = oracle.index_score(qI, w, KI, [0, S], [0], [S - 1])[0]
    doubled = oracle.index_score(qI, 2 * w, KI, [0, S], [0], [S - 1])[0]
    assert np.array_equal(doubled, 2 * base)
    perm = rng.permutation(H_I)
    permuted = oracle.index_score(qI[:, perm], w[:, perm], KI, [0, S], [0], [S - 1])[0]
    np.testing.assert_allclose(permuted, base, rtol=2 ** -23, atol=0)
    # a head with a zero weight contributes nothing
    w0 = w.copy()
    w0[0, 2] = 0
    drop = oracle.index_score(np.delete(qI, 2, axis=1), np.delete(w, 2, axis=1), KI, [0, S], [0], [S - 1])[0]
    np.testing.assert_allclose(oracle.index_score(qI, w0, KI, [0, S], [0], [S - 1])[0], drop,
                               rtol=2 ** -23)


# ----------------------------------------------------------------------------
# top-k
# ----------------------------------------------------------------------------
def _brute_force_topk(s, k):
    """Unique subset whose members all beat all non-members under
    (score desc, index asc), found by enumeration."""
    n = len(s)
    good = []
    for sub in itertools.combinations(range(n), k):
        inside = set(sub)
        ok = all((s[i] > s[j]) or (s[i] == s[j] and i < j)
                 for i in inside for j in range(n) if j not in inside)
        if ok:
            good.append(sub)
    assert len(good) == 1
    return list(good[0])


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(11)
    for trial in range(40):
        n = int(rng.integers(1, 10))
        s = rng.choice(np.array([0.0, 0.5, 1.0, 1.5], np.float32), size=n)
        for k in range(1, n + 1):
            got = oracle.topk(s[None, :], [n], k)[0]
            assert list(got) == _brute_force_topk(list(s), k)


def test_topk_all_equal_takes_lowest_indices():
    s = np.full((2, 100), 0.75, np.float32)
    got = oracle.topk(s, [100, 60], 16)
    assert list(got[0]) == list(range(16))
    assert list(got[1]) == list(range(16))


def test_topk_short_rows_pad_with_minus_one():
    s = np.array([[3.0, 1.0, 2.0, 9.0]], np.float32)
    got, ts = oracle.topk(s, [3], 5, with_scores=True)
    assert list(got[0]) == [0, 1, 2, -1, -1]
    assert list(ts[0]) == [3.0, 1.0, 2.0, 0.0, 0.0]
    assert list(oracle.topk(s, [0], 3)[0]) == [-1, -1, -1]


def test_topk_distinct_scores_match_argsort():
    rng = np.random.default_rng(5)
    s = rng.permutation(5000).astype(np.float32)[None, :] * np.float32(0.001)
    got = oracle.topk(s, [5000], 300)[0]
    want = np.sort(np.argsort(-s[0], kind="stable")[:300])
    assert np.array_equal(got, want)


def test_topk_signed_zero_ties_by_index():
    s = np.array([[-0.0, 0.0, -0.0, 0.0, -1.0]], np.float32)
    assert list(oracle.topk(s, [5], 3)[0]) == [0, 1, 2]


# ----------------------------------------------------------------------------
# sparse decode attention
# ----------------------------------------------------------------------------
def _dense_attention_torch(Q, K, V, scale):
    """Library routine: softmax(scale*Q K^T) V in fp64 (torch CPU)."""
    q = torch.from_numpy(bf16_bits_to_f32(Q).astype(np.float64))
    k = torch.from_numpy(bf16_bits_to_f32(K).astype(np.float64))
    v = torch.from_numpy(bf16_bits_to_f32(V).astype(np.float64))
    return (torch.softmax(scale * q @ k.T, dim=-1) @ v).numpy()


def _tiny_decode(rng, B=2, S=(9, 13), Hq=4, Hkv=2, d=16, L=2):
    seq_off = np.concatenate([[0], np.cumsum(S)]).astype(np.int64)
    T = int(seq_off[-1])
    Q = bf(rng.standard_normal((L, B, Hq, d)))
    K = bf(rng.standard_normal(T * Hkv * d))
    V = bf(rng.standard_normal(T * Hkv * d))
    return seq_off, np.array(S, np.int32), Q, K, V


def _kv(K, seq_off, S, Hkv, d, b, g):
    base = seq_off[b] * Hkv * d + g * S[b] * d
    return K[base: base + S[b] * d].reshape(S[b], d)


def test_attn_full_selection_equals_dense_attention():
    rng = np.random.default_rng(1)
    seq_off, S, Q, K, V = _tiny_decode(rng)
    L, B, Hq, d = Q.shape
    Hkv, k = 2, int(S.max())
    idx = np.full((B, k), -1, np.int32)
    for b in range(B):
        idx[b, :S[b]] = np.arange(S[b])
    scale = 1 / math.sqrt(d)
    got = oracle.sparse_decode_attn(Q, K, V, seq_off, S, idx, Hkv, scale)
    for l, b, h in itertools.product(range(L), range(B), range(Hq)):
        g = h // (Hq // Hkv)
        want = _dense_attention_torch(Q[l, b, h][None], _kv(K, seq_off, S, Hkv, d, b, g),
                                      _kv(V, seq_off, S, Hkv, d, b, g), scale)[0]
        np.testing.assert_allclose(got[l, b, h], want, rtol=0, atol=1e-12)


def test_attn_sparse_equals_masked_dense():
    rng = np.random.default_rng(2)
    seq_off, S, Q, K, V = _tiny_decode(rng)
    L, B, Hq, d = Q.shape
    Hkv, k = 2, 5
    idx = np.stack([np.sort(rng.choice(S[b], k, replace=False)) for b in range(B)]).astype(np.int32)
    scale = 1 / math.sqrt(d)
    got = oracle.sparse_decode_attn(Q, K, V, seq_off, S, idx, Hkv, scale)
    for l, b, h in itertools.product(range(L), range(B), range(Hq)):
        g = h // (Hq // Hkv)
        Kb = _kv(K, seq_off, S, Hkv, d, b, g)
        Vb = _kv(V, seq_off, S, Hkv, d, b, g)
        q = torch.from_numpy(bf16_bits_to_f32(Q[l, b, h]).astype(np.float64))
        z = scale * torch.from_numpy(bf16_bits_to_f32(Kb).astype(np.float64)) @ q
        mask = torch.full_like(z, -math.inf)
        mask[torch.from_numpy(idx[b].astype(np.int64))] = 0.0
        want = torch.softmax(z + mask, 0) @ torch.from_numpy(bf16_bits_to_f32(Vb).astype(np.float64))
        np.testing.assert_allclose(got[l, b, h], want.numpy(), rtol=0, atol=1e-12)


def test_attn_single_token_returns_its_value_row():
    rng = np.random.default_rng(4)
    seq_off, S, Q, K, V = _tiny_decode(rng)
    L, B, Hq, d = Q.shape
    idx = np.array([[-1, 3, -1], [-1, -1, 12]], np.int32)
    got = oracle.sparse_decode_attn(Q, K, V, seq_off, S, idx, 2, 0.25)
    for l, b, h in itertools.product(range(L), range(B), range(Hq)):
        t = idx[b][idx[b] >= 0][0]
        want = bf16_bits_to_f32(_kv(V, seq_off, S, 2, d, b, h // 2)[t])
        assert np.array_equal(got[l, b, h], want.astype(np.float64))


def test_attn_two_tokens_closed_form():
    # q = (1,..,1), K rows = 1 and 2 (all coords) -> logits scale*d*1, scale*d*2
    d = 8
    Q = bf(np.ones((1, 1, 1, d)))
    K = bf(np.concatenate([np.full(d, 1.0), np.full(d, 2.0)]))
    V = bf(np.concatenate([np.full(d, 3.0), np.full(d, -1.0)]))
    scale = 0.125
    got = oracle.sparse_decode_attn(Q, K, V, [0, 2], [2], np.array([[0, 1]], np.int32), 1, scale)
    z1, z2 = scale * d * 1.0, scale * d * 2.0
    want = (math.exp(z1) * 3.0 + math.exp(z2) * -1.0) / (math.exp(z1) + math.exp(z2))
    np.testing.assert_allclose(got[0, 0, 0], np.full(d, want), rtol=0, atol=1e-14)


def test_attn_common_key_shift_changes_nothing():
    # adding a vector e to every key adds q.e to every logit of that query
    rng = np.random.default_rng(8)
    d, S = 16, 12
    Q = bf(rng.integers(-2, 3, (1, 1, 1, d)))
    Kf = rng.integers(-2, 3, (S, d)).astype(np.float32)
    e = rng.integers(-2, 3, d).astype(np.float32)
    V = bf(rng.standard_normal(S * d))
    idx = np.array([[0, 2, 3, 7, 11]], np.int32)
    a = oracle.sparse_decode_attn(Q, bf(Kf.ravel()), V, [0, S], [S], idx, 1, 0.1)
    b = oracle.sparse_decode_attn(Q, bf((Kf + e).ravel()), V, [0, S], [S], idx, 1, 0.1)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_attn_padding_and_index_order_do_not_matter():
    rng = np.random.default_rng(9)
    seq_off, S, Q, K, V = _tiny_decode(rng)
    idx = np.array([[1, 4, 6, -1], [0, 2, 11, 12]], np.int32)
    shuffled = np.array([[-1, 6, 1, 4], [12, 0, 11, 2]], np.int32)
    a = oracle.sparse_decode_attn(Q, K, V, seq_off, S, idx, 2, 0.3)
    b = oracle.sparse_decode_attn(Q, K, V, seq_off, S, shuffled, 2, 0.3)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_attn_gqa_head_to_kv_head_map():
    # KV head 0 has V = +1 everywhere, KV head 1 has V = -1: heads 0,1 -> +1, heads 2,3 -> -1
    d, S, Hq, Hkv = 8, 6, 4, 2
    rng = np.random.default_rng(10)
    Q = bf(rng.standard_normal((1, 1, Hq, d)))
    K = bf(rng.standard_normal(Hkv * S * d))
    V = bf(np.concatenate([np.ones(S * d), -np.ones(S * d)]))
    got = oracle.sparse_decode_attn(Q, K, V, [0, S], [S], np.array([[0, 1, 5]], np.int32), Hkv, 0.5)
    np.testing.assert_allclose(got[0, 0, :2], 1.0, atol=1e-15)
    np.testing.assert_allclose(got[0, 0, 2:], -1.0, atol=1e-15)


def test_attn_no_valid_key_gives_zero():
    Q = bf(np.ones((1, 1, 1, 4)))
    out = oracle.sparse_decode_attn(Q, bf(np.ones(8)), bf(np.ones(8)), [0, 2], [2],
                                    np.array([[-1, -1]], np.int32), 1, 1.0)
    assert np.all(out == 0)


# ----------------------------------------------------------------------------
# index reuse across layers (F/S pattern)
# ----------------------------------------------------------------------------
def _decode_inputs(rng, L, same_indexer):
    B, S, H_I, d_I, Hq, Hkv, d = 2, (20, 31), 2, 8, 4, 2, 8
    seq_off = np.concatenate([[0], np.cumsum(S)]).astype(np.int64)
    T = int(seq_off[-1])
    mk = lambda: (bf(rng.standard_normal((B, H_I, d_I)) / 8),
                  rng.uniform(0.1, 1, (B, H_I)).astype(np.float32),
                  bf(rng.standard_normal((T, d_I)) / 8))
    ix = [mk()] * L if same_indexer else [mk() for _ in range(L)]
    Q = bf(rng.standard_normal((L, B, Hq, d)))
    K = bf(rng.standard_normal(T * Hkv * d))
    V = bf(rng.standard_normal(T * Hkv * d))
    return ix, seq_off, np.array(S), Q, K, V, Hkv


def test_reuse_FFFF_with_identical_indexers_equals_FSSS():
    rng = np.random.default_rng(12)
    ix, seq_off, S, Q, K, V, Hkv = _decode_inputs(rng, 4, True)
    args = ([a[0] for a in ix], [a[1] for a in ix], [a[2] for a in ix], seq_off, S, 6, Q, [K] * 4,
            [V] * 4, Hkv, 0.35)
    o1, used1 = oracle.decode_step("FFFF", *args)
    o2, used2 = oracle.decode_step("FSSS", *args)
    assert np.array_equal(o1, o2)
    for a, b in zip(used1, used2):
        assert np.array_equal(a, b)


def test_reuse_takes_nearest_upstream_full_layer():
    rng = np.random.default_rng(13)
    ix, seq_off, S, Q, K, V, Hkv = _decode_inputs(rng, 4, False)
    o, used = oracle.decode_step("FSFS", [a[0] for a in ix], [a[1] for a in ix], [a[2] for a in ix],
                                 seq_off, S, 6, Q, [K] * 4, [V] * 4, Hkv, 0.35)
    assert used[1] is used[0] and used[3] is used[2]
    assert not np.array_equal(used[0], used[2])
    # the index of layer 2 is its own indexer's top-k
    s2 = oracle.index_score(ix[2][0], ix[2][1], ix[2][2], seq_off, [0, 1], S - 1)
    assert np.array_equal(used[2], oracle.topk(s2, S, 6))


def test_pattern_must_start_with_full_layer():
    with pytest.raises(ValueError):
        oracle.decode_step("SFSS", [None] * 4, [None] * 4, [None] * 4, [0, 1], [1], 1, None, [], [], 1, 1.0)


# ----------------------------------------------------------------------------
# block union + paged causal attention
# ----------------------------------------------------------------------------
def test_union_matches_set_union_coverage_and_minimality():
    rng = np.random.default_rng(14)
    S, block, Hkv, Nq, k = 1000, 64, 3, 7, 20
    idx = np.stack([rng.choice(S, k, replace=False) for _ in range(Nq)]).astype(np.int32)
    idx[2, 5:] = -1
    indptr, indices = oracle.block_union(idx, S, block, Hkv)
    want = sorted({int(t) // block for t in idx.ravel() if t >= 0})
    assert list(indptr) == [g * len(want) for g in range(Hkv + 1)]
    for g in range(Hkv):
        T = list(indices[indptr[g]:indptr[g + 1]])
        assert T == want
        covered = {t for t in idx.ravel() if t >= 0}
        assert all(t // block in T for t in covered)                      # coverage
        assert all(any(bl * block <= t < (bl + 1) * block for t in covered) for bl in T)  # minimal


def test_dense_selection_gives_dense_causal_attention():
    rng = np.random.default_rng(15)
    S, block, Hq, Hkv, d, Nq = 200, 64, 4, 2, 16, 6
    q_pos = np.arange(S - Nq, S, dtype=np.int32)
    idx = np.stack([np.concatenate([np.arange(p + 1), -np.ones(S - p - 1)]) for p in q_pos]).astype(np.int32)
    indptr, indices = oracle.block_union(idx, S, block, Hkv)
    assert list(indices[:indptr[1]]) == list(range((S + block - 1) // block))  # partial last block kept
    Q = bf(rng.standard_normal((Nq, Hq, d)))
    K = bf(rng.standard_normal((Hkv, S, d)))
    V = bf(rng.standard_normal((Hkv, S, d)))
    scale = 1 / math.sqrt(d)
    got = oracle.paged_prefill_attn(Q, q_pos, K, V, block, indptr, indices, scale)
    for i, h in itertools.product(range(Nq), range(Hq)):
        g = h // (Hq // Hkv)
        p = q_pos[i]
        want = _dense_attention_torch(Q[i, h][None], K[g, :p + 1], V[g, :p + 1], scale)[0]
        np.testing.assert_allclose(got[i, h], want, rtol=0, atol=1e-12)


def test_paged_attention_only_reads_listed_blocks_and_is_causal():
    # table {1}; query at position 70 sees keys 64..70 of block 1 only
    rng = np.random.default_rng(16)
    S, block, d = 256, 64, 8
    Q = bf(rng.standard_normal((1, 1, d)))
    K = bf(rng.standard_normal((1, S, d)))
    V = bf(rng.standard_normal((1, S, d)))
    got = oracle.paged_prefill_attn(Q, [70], K, V, block, [0, 1], [1], 0.5)
    want = _dense_attention_torch(Q[0, 0][None], K[0, 64:71], V[0, 64:71], 0.5)[0]
    np.testing.assert_allclose(got[0, 0], want, rtol=0, atol=1e-12)
    # a query before the listed block sees nothing -> zero output
    assert np.all(oracle.paged_prefill_attn(Q, [10], K, V, block, [0, 1], [1], 0.5) == 0)


# ----------------------------------------------------------------------------
# the synthetic workloads: planted needles are found
# ----------------------------------------------------------------------------
def test_c1_needles_are_selected():
    cfg = synth.workload("c1")
    g = 0
    s = oracle.index_score(cfg.qI(g), cfg.w(g), cfg.KI_full(g), cfg.seq_off, [0], [cfg.S_max - 1])
    idx = oracle.topk(s, cfg.seq_lens, cfg.k)[0]
    needles = [t for (b, t, _, kr) in cfg.planted(g) if kr is not None]
    assert len(needles) == 8
    kth = np.sort(s[0])[::-1][cfg.k - 1]
    for t in needles:
        assert s[0, t] > kth and t in set(idx.tolist())


def test_kv_append_writes_only_the_new_token_rows():
    """The appended caches differ from the old ones exactly at each
    sequence's last position (every KV head), where they hold the new rows."""
    rng = np.random.default_rng(3)
    lens, Hkv, d, d_I = [5, 3], 2, 4, 3
    seq_off = np.array([0, 5, 8])
    KI = rng.integers(0, 1000, (8, d_I)).astype(np.uint16)
    K = rng.integers(0, 1000, 8 * Hkv * d).astype(np.uint16)
    V = rng.integers(0, 1000, 8 * Hkv * d).astype(np.uint16)
    nKI = np.full((2, d_I), 7, np.uint16)
    nK = np.arange(2 * Hkv * d, dtype=np.uint16).reshape(2, Hkv, d) + 2000
    nV = nK + 1000
    KIa, Ka, Va = oracle.kv_append(KI, K, V, seq_off, lens, nKI, nK, nV, Hkv, d)
    assert np.array_equal(KIa[[4, 7]], nKI) and np.array_equal(np.delete(KIa, [4, 7], 0), np.delete(KI, [4, 7], 0))
    # sequence 0: heads at element rows 0*2+h*5+4; sequence 1: 5*2 + h*3 + 2
    rows = [4, 9, 12, 15]
    want = [nK[0, 0], nK[0, 1], nK[1, 0], nK[1, 1]]
    K3, Ka3 = K.reshape(-1, d), Ka.reshape(-1, d)
    for r, wv in zip(rows, want):
        assert np.array_equal(Ka3[r], wv)
    assert np.array_equal(np.delete(Ka3, rows, 0), np.delete(K3, rows, 0))
    assert np.array_equal(Va.reshape(-1, d)[rows], np.stack([nV[0, 0], nV[0, 1], nV[1, 0], nV[1, 1]]))


# ----------------------------------------------------------------------------
# CLSA indexer layer read as full attention whose weights route the index
# ----------------------------------------------------------------------------
def _torch_weights(q, Kb, scale):
    """Library routine: the softmax attention weights of one query row (fp64)."""
    qq = torch.from_numpy(bf16_bits_to_f32(q).astype(np.float64))
    kk = torch.from_numpy(bf16_bits_to_f32(Kb).astype(np.float64))
    return torch.softmax(scale * kk @ qq, dim=0).numpy()


def test_indexer_layer_output_is_dense_attention():
    rng = np.random.default_rng(11)
    seq_off, S, Q, K, V = _tiny_decode(rng)
    _, B, Hq, d = Q.shape
    Hkv, scale = 2, 1 / math.sqrt(d)
    O, _ = oracle.indexer_layer_attn(Q[0], K, V, seq_off, S, Hkv, scale)
    for b, h in itertools.product(range(B), range(Hq)):
        g = h // (Hq // Hkv)
        want = _dense_attention_torch(Q[0, b, h][None], _kv(K, seq_off, S, Hkv, d, b, g),
                                      _kv(V, seq_off, S, Hkv, d, b, g), scale)[0]
        np.testing.assert_allclose(O[b, h], want, rtol=0, atol=1e-12)


def test_indexer_layer_route_is_the_head_sum_of_attention_weights():
    rng = np.random.default_rng(12)
    seq_off, S, Q, K, V = _tiny_decode(rng, Hq=8, Hkv=2)
    _, B, Hq, d = Q.shape
    Hkv, scale = 2, 1 / math.sqrt(d)
    _, route = oracle.indexer_layer_attn(Q[0], K, V, seq_off, S, Hkv, scale, ld=16)
    for b in range(B):
        want = sum(_torch_weights(Q[0, b, h], _kv(K, seq_off, S, Hkv, d, b, h // (Hq // Hkv)), scale)
                   for h in range(Hq))
        np.testing.assert_allclose(route[b, :S[b]], want, rtol=2e-7, atol=0)
        assert np.all(np.isnan(route[b, S[b]:]))  # nothing written past the sequence
        # each head's weights sum to one, so the routing scores sum to Hq
        assert abs(float(route[b, :S[b]].astype(np.float64).sum()) - Hq) < 1e-5


def test_indexer_layer_single_head_routes_by_logit():
    # one head, integer-valued q and k: the logits are exact integers, and the
    # softmax is monotone, so the top-k of the routing scores is the top-k of
    # the logits under the tie rule (brute force), ties included
    rng = np.random.default_rng(13)
    S, d, k = 40, 8, 9
    q = rng.integers(-2, 3, (1, 1, d)).astype(np.float32)
    Kt = rng.integers(-2, 3, (S, d)).astype(np.float32)
    V = rng.standard_normal(S * d).astype(np.float32)
    _, route = oracle.indexer_layer_attn(bf(q), bf(Kt.ravel()), bf(V), [0, S], [S], 1, 0.5)
    logits = Kt @ q[0, 0]
    order = sorted(range(S), key=lambda t: (-logits[t], t))[:k]
    assert list(oracle.topk(route, [S], k)[0]) == sorted(order)
    for a, b2 in itertools.combinations(range(S), 2):
        if logits[a] == logits[b2]:
            assert route[0, a] == route[0, b2]


def test_indexer_layer_identical_keys_route_uniformly():
    S, d, Hq = 24, 8, 4
    Q = bf(np.random.default_rng(14).standard_normal((1, Hq, d)))
    K = bf(np.tile(np.linspace(-1, 1, d), S))
    V = bf(np.arange(S * d, dtype=np.float32) / 64)
    O, route = oracle.indexer_layer_attn(Q, K, V, [0, S], [S], 1, 0.3)
    np.testing.assert_allclose(route[0], np.float32(Hq / S), rtol=1e-7, atol=0)
    assert list(oracle.topk(route, [S], 5)[0]) == [0, 1, 2, 3, 4]  # all tied: lowest indices
    # uniform weights: the output is the mean value row
    np.testing.assert_allclose(O[0, 0], bf16_bits_to_f32(V).reshape(S, d).mean(0), rtol=0, atol=1e-12)


def test_indexer_layer_reads_each_head_group_cache():
    # heads 0,1 (KV head 0) and heads 2,3 (KV head 1): a key aligned with the
    # group's queries sits at token 3 in KV head 0 and at token 7 in KV head
    # 1, so the routing score peaks at both with about 2 (two heads each)
    S, d, Hq, Hkv = 12, 8, 4, 2
    Q = np.zeros((1, Hq, d), np.float32)
    Q[0, :2, 0] = 4.0
    Q[0, 2:, 1] = 4.0
    K = np.zeros((Hkv, S, d), np.float32)
    K[0, 3, 0] = 4.0
    K[1, 7, 1] = 4.0
    V = np.zeros(Hkv * S * d, np.float32)
    _, route = oracle.indexer_layer_attn(bf(Q), bf(K.ravel()), bf(V), [0, S], [S], Hkv, 1.0)
    assert set(oracle.topk(route, [S], 2)[0]) == {3, 7}
    assert route[0, 3] > 1.99 and route[0, 7] > 1.99


def test_attn_route_step_with_every_token_selected_is_dense():
    # k = S: every later layer attends to every token, i.e. dense attention
    rng = np.random.default_rng(15)
    seq_off, S, Q, K, V = _tiny_decode(rng, L=3)
    L, B, Hq, d = Q.shape
    Hkv, scale = 2, 1 / math.sqrt(d)
    O, idx, _ = oracle.decode_step_attn_route(Q, K, V, seq_off, S, int(S.max()), Hkv, scale)
    for b in range(B):
        assert list(idx[b, :S[b]]) == list(range(S[b]))
    for l, b, h in itertools.product(range(L), range(B), range(Hq)):
        g = h // (Hq // Hkv)
        want = _dense_attention_torch(Q[l, b, h][None], _kv(K, seq_off, S, Hkv, d, b, g),
                                      _kv(V, seq_off, S, Hkv, d, b, g), scale)[0]
        np.testing.assert_allclose(O[l, b, h], want, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# context-parallel decode: partial attention, log-sum-exp combine, selection
# ----------------------------------------------------------------------------
def test_cp_partial_is_the_unnormalised_softmax():
    # library routine: torch fp64 logsumexp / softmax over the selected keys
    rng = np.random.default_rng(40)
    seq_off, S, Q, K, V = _tiny_decode(rng)
    L, B, Hq, d = Q.shape
    Hkv, k = 2, 6
    idx = np.stack([np.sort(rng.choice(S[b], 5, replace=False)) for b in range(B)]).astype(np.int32)
    idx = np.concatenate([idx, np.full((B, 1), -1, np.int32)], axis=1)
    scale = 0.3
    o, ml = oracle.sparse_decode_attn_partial(Q, K, V, seq_off, S, idx, Hkv, scale)
    for l, b, h in itertools.product(range(L), range(B), range(Hq)):
        g = h // (Hq // Hkv)
        sel = torch.from_numpy(idx[b][idx[b] >= 0].astype(np.int64))
        Kb = torch.from_numpy(bf16_bits_to_f32(_kv(K, seq_off, S, Hkv, d, b, g)).astype(np.float64))[sel]
        Vb = torch.from_numpy(bf16_bits_to_f32(_kv(V, seq_off, S, Hkv, d, b, g)).astype(np.float64))[sel]
        q = torch.from_numpy(bf16_bits_to_f32(Q[l, b, h]).astype(np.float64))
        z = scale * (Kb @ q)
        m = float(z.max())
        assert ml[l, b, h, 0] == pytest.approx(m / math.log(2), rel=0, abs=1e-12)
        assert ml[l, b, h, 1] == pytest.approx(math.exp(float(torch.logsumexp(z, 0)) - m), rel=1e-12)
        np.testing.assert_allclose(o[l, b, h] / ml[l, b, h, 1], (torch.softmax(z, 0) @ Vb).numpy(), rtol=0,
                                   atol=1e-12)


def test_cp_partial_of_an_empty_selection():
    rng = np.random.default_rng(41)
    seq_off, S, Q, K, V = _tiny_decode(rng)
    idx = np.full((2, 4), -1, np.int32)
    o, ml = oracle.sparse_decode_attn_partial(Q, K, V, seq_off, S, idx, 2, 0.3)
    assert np.all(o == 0) and np.all(ml[..., 1] == 0) and np.all(np.isneginf(ml[..., 0]))


def test_cp_combine_closed_form():
    # part 0: m = 0, l = 1, o = u; part 1: m = 1, l = 3, o = v  ->  (u + 2 v) / (1 + 6)
    u = np.arange(4, dtype=np.float64)[None]
    v = np.full((1, 4), 7.0)
    ml = np.array([[[0.0, 1.0]], [[1.0, 3.0]]])
    got = oracle.combine_partials(np.stack([u, v]), ml)
    np.testing.assert_allclose(got[0], (u[0] + 2 * v[0]) / 7.0, rtol=0, atol=1e-15)
    # a part with l = 0 is ignored, whatever its m; all-empty rows give 0
    ml2 = np.array([[[0.0, 1.0], [5.0, 0.0]], [[50.0, 0.0], [-np.inf, 0.0]]])
    parts = np.stack([np.stack([u[0], v[0]]), np.stack([v[0], u[0]])])
    got = oracle.combine_partials(parts, ml2)
    np.testing.assert_allclose(got[0], u[0], rtol=0, atol=0)
    assert np.all(got[1] == 0)


def test_cp_combine_of_a_key_split_equals_attention_over_the_union():
    # the selected keys of each sequence split into 3 disjoint parts (one of
    # them empty for sequence 0): the merge equals the one-part attention
    rng = np.random.default_rng(42)
    seq_off, S, Q, K, V = _tiny_decode(rng)
    L, B, Hq, d = Q.shape
    k, Hkv, scale = 8, 2, 0.4
    idx = np.stack([np.sort(rng.choice(S[b], k, replace=False)) for b in range(B)]).astype(np.int32)
    owner = rng.integers(0, 3, (B, k))
    owner[0][owner[0] == 2] = 1
    parts, mls = [], []
    for p in range(3):
        ip = np.where(owner == p, idx, -1).astype(np.int32)
        o, ml = oracle.sparse_decode_attn_partial(Q, K, V, seq_off, S, ip, Hkv, scale)
        parts.append(o.reshape(-1, d))
        mls.append(ml.reshape(-1, 2))
    got = oracle.combine_partials(np.stack(parts), np.stack(mls)).reshape(L, B, Hq, d)
    want = oracle.sparse_decode_attn(Q, K, V, seq_off, S, idx, Hkv, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def _python_topk(row, k):
    order = sorted(range(len(row)), key=lambda t: (-float(row[t]), t))
    return sorted(order[:k])


def test_cp_select_over_slices_is_the_global_topk():
    for N in (1, 2, 3, 5):
        _cp_select_case(N)


def _cp_select_case(N):
    # scores drawn from a few values (many ties), one sequence shorter than
    # k, one shorter than N (empty slices); brute force on the whole context
    rng = np.random.default_rng(43 + N)
    lens = [40, 7, 3, 64]
    k = 9
    B = len(lens)
    full = [rng.integers(0, 6, n).astype(np.float32) * np.float32(0.5) for n in lens]
    bounds = [[(r * n // N, (r + 1) * n // N) for n in lens] for r in range(N)]
    cand_s = np.zeros((N, B, k), np.float32)
    cand_i = np.zeros((N, B, k), np.int32)
    for r in range(N):
        lo_hi = bounds[r]
        width = max(1, max(hi - lo for lo, hi in lo_hi))
        sc = np.zeros((B, width), np.float32)
        for b, (lo, hi) in enumerate(lo_hi):
            sc[b, : hi - lo] = full[b][lo:hi]
        cand_i[r], cand_s[r] = oracle.topk(sc, [hi - lo for lo, hi in lo_hi], k, with_scores=True)
    got = [set() for _ in range(B)]
    for r in range(N):
        loc = oracle.cp_select(cand_s, cand_i, r)
        for b in range(B):
            row = [int(t) for t in loc[b] if t >= 0]
            assert row == sorted(row) and all(t < 0 for t in loc[b][len(row):])
            got[b] |= {bounds[r][b][0] + t for t in row}
    for b in range(B):
        assert sorted(got[b]) == _python_topk(full[b], k), b


# --------------------------------------------------------------------------
# Dynamic k by routing mass [CLSA news article, "Le cout : limites de
# compatibilite": k could be set per query; the rule here is a reading]:
# the smallest m, in the top-k order, whose running score reaches tau of
# the row's total, at most k_max.
def _dynamic_brute(row, n, k_max, tau):
    """Exact rational arithmetic, sorting by (score desc, index asc)."""
    vals = [Fraction(float(x)) for x in row[:n]]
    total = sum(vals, Fraction(0))
    order = sorted(range(n), key=lambda t: (-vals[t], t))
    target = Fraction(tau) * total
    m, run = n, Fraction(0)
    for j, t in enumerate(order):
        run += vals[t]
        if run >= target:
            m = j + 1
            break
    m = min(m, k_max)
    return sorted(order[:m]), m


def test_dynamic_k_brute_force_exact_rationals():
    rng = np.random.default_rng(41)
    for trial in range(40):
        n = int(rng.integers(1, 60))
        # dyadic scores with ties: every sum is exact in fp64
        row = (rng.integers(0, 12, n) / 8.0).astype(np.float32)
        k_max = int(rng.integers(1, 70))
        tau = float(rng.choice([0.125, 0.25, 0.5, 0.75, 0.875, 1.0]))
        idx, counts = oracle.topk_dynamic(row[None], [n], k_max, tau)
        want, m = _dynamic_brute(row, n, k_max, tau)
        assert counts[0] == m, (trial, counts[0], m)
        assert list(idx[0, :m]) == want and np.all(idx[0, m:] == -1), trial


def test_dynamic_k_uniform_scores_closed_form():
    # n equal scores: the running sum after j tokens is j/n of the total, so
    # m = ceil(tau * n), the lowest indices
    n, k_max = 1000, 2048
    row = np.full((1, n), 0.25, np.float32)
    for tau, m in ((0.375, 375), (0.5, 500), (0.0625, 63), (1.0, 1000)):
        idx, counts = oracle.topk_dynamic(row, [n], k_max, tau)
        assert counts[0] == m, (tau, counts[0])
        assert np.array_equal(idx[0, :m], np.arange(m)) and np.all(idx[0, m:] == -1)


def test_dynamic_k_cap_dominant_token_and_zero_tail():
    row = np.zeros((1, 300), np.float32)
    row[0, 7] = 100.0
    row[0, 50:60] = 1.0
    # the dominant token alone carries 100/110 of the mass
    idx, counts = oracle.topk_dynamic(row, [300], 64, 0.9)
    assert counts[0] == 1 and idx[0, 0] == 7 and np.all(idx[0, 1:] == -1)
    # the whole mass needs the 11 positive tokens, not the zero tail
    idx, counts = oracle.topk_dynamic(row, [300], 64, 1.0)
    assert counts[0] == 11 and list(idx[0, :11]) == [7] + list(range(50, 60))
    # capped at k_max
    idx, counts = oracle.topk_dynamic(row, [300], 5, 1.0)
    assert counts[0] == 5 and list(idx[0, :5]) == [7, 50, 51, 52, 53]
    # an empty row keeps nothing
    idx, counts = oracle.topk_dynamic(row, [0], 5, 0.5)
    assert counts[0] == 0 and np.all(idx[0] == -1)


def test_dynamic_k_total_is_over_the_whole_row():
    # the top-2 carry 2/3 of their own mass but only 2/8 of the row's
    row = np.array([[1, 1, 1, 1, 1, 1, 1, 1]], np.float32)
    row[0, 3] = 2.0
    row[0, 6] = 2.0  # total 10
    idx, counts = oracle.topk_dynamic(row, [8], 8, 0.5)  # target 5: 2 + 2 + 1
    assert counts[0] == 3 and list(idx[0, :3]) == [0, 3, 6]


# ----------------------------------------------------------------------------
# CoSA: the proxy's priority list and the ordered-skipping kernel (reading in
# oracle/sa_oracle.c: hit counts order the union table per query block; the
# kernel runs two blocks per step and stops `lag` steps after the first step
# whose largest row share of the running softmax mass is below tau)
# ----------------------------------------------------------------------------
def _kap_brute(idx, S, block, q_block, T):
    out = []
    Nq = len(idx)
    for i in range(0, Nq, q_block):
        hits = {int(b): 0 for b in T}
        for p in range(i, min(Nq, i + q_block)):
            for t in idx[p]:
                t = int(t)
                if 0 <= t < S and t // block in hits:
                    hits[t // block] += 1
        out.append(sorted(hits, key=lambda b: (-hits[b], b)))
    return out


def test_kap_order_hand_example():
    # S = 512, 64-token blocks; query block 0 = queries 0, 1; block 1 = query 2
    idx = np.array([[5, 70, 71, 300],      # blocks 0, 1, 1, 4
                    [72, 301, -1, 600],    # blocks 1, 4; -1 and 600 >= S not counted
                    [130, 131, 450, 0]],   # blocks 2, 2, 7, 0
                   np.int32)
    T = [0, 1, 2, 4, 7]
    order = oracle.kap_order(idx, 512, 64, 2, T)
    # block 0: hits 0:1, 1:3, 2:0, 4:2, 7:0; block 1: 0:1, 1:0, 2:2, 4:0, 7:1
    assert order.tolist() == [[1, 4, 0, 2, 7], [2, 0, 7, 1, 4]]


def test_kap_order_brute_force():
    rng = np.random.default_rng(51)
    for trial in range(20):
        S = int(rng.integers(64, 2000))
        block = int(rng.choice([16, 64]))
        Nq, k, q_block = int(rng.integers(1, 12)), int(rng.integers(1, 40)), int(rng.integers(1, 5))
        idx = rng.integers(-3, S + 40, (Nq, k)).astype(np.int32)      # padding, past-S entries, duplicates
        nb = (S + block - 1) // block
        T = sorted(set(rng.choice(nb, int(rng.integers(0, nb + 1)), replace=False).tolist()) |
                   {int(t) // block for t in idx.ravel() if 0 <= t < S})
        got = oracle.kap_order(idx, S, block, q_block, T)
        want = _kap_brute(idx, S, block, q_block, T)
        assert got.tolist() == want, trial
        assert all(sorted(r) == T for r in got.tolist())


def _osk_case(seed, Nq=6, Hq=4, Hkv=2, S=700, d=16, block=64, chunk_end=True):
    rng = np.random.default_rng(seed)
    q_pos = (np.arange(S - Nq, S) if chunk_end else np.sort(rng.choice(S, Nq, replace=False))).astype(np.int32)
    Q = bf(rng.standard_normal((Nq, Hq, d)))
    K = bf(rng.standard_normal((Hkv, S, d)))
    V = bf(rng.standard_normal((Hkv, S, d)))
    idx = np.full((Nq, 40), -1, np.int32)
    for i, p in enumerate(q_pos):
        n = min(40, int(p) + 1)
        idx[i, :n] = rng.choice(int(p) + 1, n, replace=False)
    return rng, q_pos, Q, K, V, idx


def test_osk_without_skipping_is_the_paged_attention():
    # tau = 0: no share is below it, every unit runs every step, and the
    # order of the blocks does not change a softmax over the same keys
    for seed, chunk_end in ((52, True), (53, False)):
        rng, q_pos, Q, K, V, idx = _osk_case(seed, chunk_end=chunk_end)
        S, block, Hkv, q_block = K.shape[1], 64, K.shape[0], 2
        indptr, indices = oracle.block_union(idx, S, block, Hkv)
        T = indices[:indptr[1]]
        order = oracle.kap_order(idx, S, block, q_block, T)
        O, steps, crit = oracle.osk_prefill_attn(Q, q_pos, K, V, block, order, q_block, 0.25, tau=0.0)
        want = oracle.paged_prefill_attn(Q, q_pos, K, V, block, indptr, indices, 0.25)
        np.testing.assert_allclose(O, want, rtol=0, atol=1e-12)
        assert np.all(steps == (len(T) + 1) // 2)
        assert np.all((crit >= 0) & ((crit <= 1 + 1e-12) | np.isinf(crit)))  # 0: a step no row sees


def test_osk_stopping_at_once_reads_the_first_blocks_only():
    # tau > 1: every step's share is at most 1, so each unit stops after
    # step 0 and runs 1 + lag steps: attention over its first 2 (1 + lag)
    # blocks of the order, the paged attention over that table
    rng, q_pos, Q, K, V, idx = _osk_case(54)
    S, block, Hkv, G, q_block = K.shape[1], 64, K.shape[0], 2, 3
    T = list(range((S + block - 1) // block))
    order = np.stack([rng.permutation(T) for _ in range(2)]).astype(np.int32)
    for lag in (0, 1, 2):
        O, steps, _ = oracle.osk_prefill_attn(Q, q_pos, K, V, block, order, q_block, 0.25, tau=1.5, lag=lag)
        assert np.all(steps == 1 + lag)
        for i in range(2):
            sub = np.sort(order[i, :2 * (1 + lag)]).astype(np.int32)
            want = oracle.paged_prefill_attn(Q, q_pos, K, V, block, [g * len(sub) for g in range(Hkv + 1)],
                                             np.tile(sub, Hkv), 0.25)
            rows = slice(i * q_block, (i + 1) * q_block)
            np.testing.assert_allclose(O[rows], want[rows], rtol=0, atol=1e-12)


def _osk_pow2_case():
    # one query (position 15, sees every key), two heads of one KV group,
    # 2-token blocks run in the order 3 1 6 0 2 7 4 5: steps (3,1) (6,0) (2,7) (4,5).
    # scale = ln 2 and integer dots make every weight a power of two:
    #   head 0 dots 3, 1, 0, -1 per step -> masses 32, 8, 4, 2
    #   head 1 dots 0, 1, 0, -2 per step -> masses 4, 8, 4, 1
    # shares per step: head 0  1, 8/40, 4/44, 2/46;  head 1  1, 8/12, 4/16, 1/17
    # largest share c = 1, 2/3, 1/4, 1/17
    order = np.array([[3, 1, 6, 0, 2, 7, 4, 5]], np.int32)
    step_of = {}
    for n in range(4):
        for b in order[0, 2 * n:2 * n + 2]:
            step_of[2 * int(b)] = n
            step_of[2 * int(b) + 1] = n
    dots = {0: (3, 1, 0, -1), 1: (0, 1, 0, -2)}
    K = np.zeros((1, 16, 2), np.float32)
    V = np.zeros((1, 16, 2), np.float32)
    for t in range(16):
        K[0, t] = (dots[0][step_of[t]], dots[1][step_of[t]])
        V[0, t] = (step_of[t], 1.0)
    Q = np.array([[[1.0, 0.0], [0.0, 1.0]]], np.float32)
    return bf(Q), bf(K), bf(V), order


def test_osk_powers_of_two_closed_form():
    Q, K, V, order = _osk_pow2_case()
    mass = {0: (32, 8, 4, 2), 1: (4, 8, 4, 1)}
    for tau, lag, N in ((0.7, 0, 2), (0.7, 1, 3), (0.7, 2, 4), (0.3, 0, 3), (0.3, 1, 4), (0.1, 0, 4),
                        (0.05, 0, 4), (1.5, 0, 1)):
        O, steps, crit = oracle.osk_prefill_attn(Q, [15], K, V, 2, order, 1, math.log(2.0), tau=tau, lag=lag)
        np.testing.assert_allclose(crit[0], [1.0, 2 / 3, 1 / 4, 1 / 17], rtol=1e-13)
        assert steps[0] == N, (tau, lag)
        for h in range(2):
            w = [Fraction(4 * 0 + m) for m in mass[h][:N]]
            want = float(sum(n * w[n] for n in range(N)) / sum(w))
            np.testing.assert_allclose(O[0, h], [want, 1.0], rtol=0, atol=1e-13)


def test_osk_equal_logits_strict_threshold():
    # K = 0: every logit is 0 and every weight exp(0) = 1 exactly, so after
    # step n (4 keys per step) the share is exactly 4 / (4 (n + 1)).
    # tau = 1/4: step 3's share equals tau and does not stop (strict), step 4's does.
    d, S = 4, 48
    Q = bf(np.ones((1, 1, d)))
    K = bf(np.zeros((1, S, d)))
    V = bf(np.arange(S * d, dtype=np.float32).reshape(1, S, d) % 7)
    order = np.arange(12, dtype=np.int32)[None]
    for tau, N in ((0.25, 5), (0.2, 6), (0.5, 3), (0.49, 3)):
        O, steps, crit = oracle.osk_prefill_attn(Q, [S - 1], K, V, 4, order, 1, 1.0, tau=tau, lag=0)
        assert crit[0].tolist() == [1 / (n + 1) for n in range(6)]
        assert steps[0] == N, tau
        want = bf16_bits_to_f32(V[0, :8 * N]).astype(np.float64).mean(axis=0)
        np.testing.assert_allclose(O[0, 0], want, rtol=0, atol=1e-12)


def test_osk_a_row_with_nothing_visible_keeps_the_unit_running():
    # query 0 (position 3) sees only block 0, which comes last in the order;
    # query 1 (position 47) sees everything.  With tau = 0.9 query 1 alone
    # would stop after step 1, but query 0 has seen no key until the last
    # step (share +inf), so the unit runs all of them.
    d, S = 4, 48
    Q = bf(np.ones((2, 1, d)))
    K = bf(np.zeros((1, S, d)))
    V = bf(np.arange(S * d, dtype=np.float32).reshape(1, S, d) % 5)
    order = np.array([[11, 10, 9, 8, 7, 6, 5, 4, 3, 2, 1, 0]], np.int32)
    O, steps, crit = oracle.osk_prefill_attn(Q, [3, 47], K, V, 4, order, 2, 1.0, tau=0.9, lag=0)
    assert steps[0] == 6 and np.all(np.isinf(crit[0, :5])) and crit[0, 5] == 1.0
    # the same query 1 in a unit of its own stops after step 1 (share 1/2)
    O1, steps1, _ = oracle.osk_prefill_attn(Q[1:], [47], K, V, 4, order, 1, 1.0, tau=0.9, lag=0)
    assert steps1[0] == 2
    np.testing.assert_allclose(O1[0, 0], bf16_bits_to_f32(V[0, 32:48]).astype(np.float64).mean(axis=0),
                               rtol=0, atol=1e-12)


def test_osk_given_steps_is_the_attention_over_that_prefix():
    # steps_in fixes N per unit: the output is the paged attention over the
    # first 2N blocks of the unit's order, whatever tau says
    rng, q_pos, Q, K, V, idx = _osk_case(55)
    S, block, Hkv, q_block = K.shape[1], 64, K.shape[0], 3
    T = list(range((S + block - 1) // block))
    order = np.stack([rng.permutation(T) for _ in range(2)]).astype(np.int32)
    steps_in = np.array([2, 0, 5, 1], np.int32)   # unit u = g * 2 + i
    O, steps, _ = oracle.osk_prefill_attn(Q, q_pos, K, V, block, order, q_block, 0.25, tau=0.5, steps_in=steps_in)
    assert steps.tolist() == [2, 0, 5, 1]
    G = Q.shape[1] // Hkv
    for u, N in enumerate(steps_in):
        g, i = divmod(u, 2)
        sub = np.sort(order[i, :2 * N]).astype(np.int32)
        want = oracle.paged_prefill_attn(Q, q_pos, K, V, block, [j * len(sub) for j in range(Hkv + 1)],
                                         np.tile(sub, Hkv), 0.25)
        rows = slice(i * q_block, (i + 1) * q_block)
        heads = slice(g * G, (g + 1) * G)
        np.testing.assert_allclose(O[rows, heads], want[rows, heads], rtol=0, atol=1e-12)


def _osk_brute(Q, q_pos, K, V, block, order, q_block, scale, tau, lag):
    """The ordered-skipping rule written out directly on tiny inputs: after
    each step the shares are recomputed from every logit seen so far (no
    running update), then the output over the steps run."""
    Qf, Kf, Vf = (bf16_bits_to_f32(x).astype(np.float64) for x in (Q, K, V))
    Nq, Hq, d = Qf.shape
    Hkv, S, _ = Kf.shape
    G = Hq // Hkv
    n_qb, nT = order.shape
    n_steps = (nT + 1) // 2
    O = np.zeros((Nq, Hq, d))
    steps = np.zeros(n_qb * Hkv, np.int64)
    crit = np.zeros((n_qb * Hkv, n_steps))
    for g in range(Hkv):
        for i in range(n_qb):
            rows = [(p, g * G + h) for p in range(i * q_block, min(Nq, (i + 1) * q_block)) for h in range(G)]
            step_keys = []
            for n in range(n_steps):
                ks = []
                for b in order[i, 2 * n:2 * n + 2]:
                    ks += [t for t in range(int(b) * block, int(b) * block + block) if t < S]
                step_keys.append(ks)
            N = n_steps
            for n in range(n_steps):
                c = -math.inf
                for (p, h) in rows:
                    seen = [t for m in range(n + 1) for t in step_keys[m] if t <= q_pos[p]]
                    if not seen:
                        share = math.inf
                    else:
                        z = {t: scale * float(Qf[p, h] @ Kf[g, t]) for t in seen}
                        M = max(z.values())
                        L = sum(math.exp(v - M) for v in z.values())
                        a = sum(math.exp(z[t] - M) for t in step_keys[n] if t <= q_pos[p])
                        share = a / L
                    c = max(c, share)
                crit[g * n_qb + i, n] = c
                if c < tau and N == n_steps:
                    N = min(n_steps, n + 1 + lag)
            steps[g * n_qb + i] = N
            for (p, h) in rows:
                ks = [t for m in range(N) for t in step_keys[m] if t <= q_pos[p]]
                if ks:
                    z = np.array([scale * float(Qf[p, h] @ Kf[g, t]) for t in ks])
                    w = np.exp(z - z.max())
                    O[p, h] = (w[:, None] * Vf[g, ks]).sum(0) / w.sum()
    return O, steps, crit


def test_osk_brute_force_on_tiny_chunks():
    rng = np.random.default_rng(57)
    for trial in range(8):
        Nq = int(rng.integers(1, 5))
        Hkv = int(rng.choice([1, 2]))
        G = int(rng.choice([1, 2, 3]))
        S = int(rng.integers(10, 48))
        block = int(rng.choice([3, 4, 8]))
        d = 4
        q_block = int(rng.integers(1, 4))
        q_pos = np.sort(rng.choice(S, Nq, replace=False)).astype(np.int32)
        Q = bf(rng.standard_normal((Nq, Hkv * G, d)) * 1.5)
        K = bf(rng.standard_normal((Hkv, S, d)))
        V = bf(rng.standard_normal((Hkv, S, d)))
        nb = (S + block - 1) // block
        T = np.sort(rng.choice(nb, int(rng.integers(1, nb + 1)), replace=False))
        n_qb = (Nq + q_block - 1) // q_block
        order = np.stack([rng.permutation(T) for _ in range(n_qb)]).astype(np.int32)
        tau = float(rng.choice([0.0, 0.05, 0.2, 0.5]))
        lag = int(rng.integers(0, 3))
        O, steps, crit = oracle.osk_prefill_attn(Q, q_pos, K, V, block, order, q_block, 0.7, tau, lag=lag)
        Ob, sb, cb = _osk_brute(Q, q_pos, K, V, block, order, q_block, 0.7, tau, lag)
        finite = np.isfinite(cb)
        assert np.array_equal(np.isfinite(crit), finite), trial
        np.testing.assert_allclose(crit[finite], cb[finite], rtol=1e-12, atol=0)
        assert np.array_equal(steps, sb), (trial, steps, sb)
        np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
