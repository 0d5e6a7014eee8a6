"""Hand-worked examples in tests/golden/worked_examples.json against the oracle."""
import json
import os

import numpy as np

import oracle
from synth import f32_to_bf16_bits

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, np.float32))


def test_golden_index_score():
    c = G["index_score"]
    n = len(c["KI"])
    s = oracle.index_score(bf(c["qI"]), np.array(c["w"], np.float32), bf(c["KI"]), [0, n], [0], [n - 1])
    assert s[0].tolist() == c["expected"]


def test_golden_topk():
    c = G["topk"]
    s = np.array([c["scores"]], np.float32)
    for case in c["cases"]:
        assert oracle.topk(s, [case["n_valid"]], case["k"])[0].tolist() == case["expected"]


def test_golden_sparse_attention():
    c = G["sparse_attention"]
    K, V = np.array(c["K"], np.float32), np.array(c["V"], np.float32)
    n, d = K.shape
    out = oracle.sparse_decode_attn(bf(np.array(c["q"])[None, None, None]), bf(K.ravel()), bf(V.ravel()),
                                    [0, n], [n], np.array([c["idx"]], np.int32), 1, c["scale"])
    np.testing.assert_allclose(out[0, 0, 0], c["expected"], rtol=0, atol=1e-15)


def test_golden_block_union():
    c = G["block_union"]
    indptr, indices = oracle.block_union(np.array(c["idx"], np.int32), c["S"], c["block"], c["Hkv"])
    assert indptr.tolist() == c["expected_indptr"] and indices.tolist() == c["expected_indices"]


def test_golden_cp_select():
    c = G["cp_select"]
    s = np.array(c["scores"], np.float32)
    k = c["k"]
    N = len(c["slices"])
    cand_s = np.zeros((N, 1, k), np.float32)
    cand_i = np.zeros((N, 1, k), np.int32)
    for r, (lo, hi) in enumerate(c["slices"]):
        cand_i[r], cand_s[r] = oracle.topk(s[None, lo:hi], [hi - lo], k, with_scores=True)
    for r in range(N):
        assert oracle.cp_select(cand_s, cand_i, r)[0].tolist() == c["expected_local"][r]


def test_golden_combine_partials():
    c = G["combine_partials"]
    o = np.array([[p["o"]] for p in c["parts"]], np.float64)
    ml = np.array([[[p["m"], p["l"]]] for p in c["parts"]], np.float64)
    np.testing.assert_allclose(oracle.combine_partials(o, ml)[0], c["expected"], rtol=0, atol=1e-15)


def test_golden_sparse_attention_partial():
    c = G["sparse_attention_partial"]
    K, V = np.array(c["K"], np.float32), np.array(c["V"], np.float32)
    n = K.shape[0]
    o, ml = oracle.sparse_decode_attn_partial(bf(np.array(c["q"])[None, None, None]), bf(K.ravel()), bf(V.ravel()),
                                              [0, n], [n], np.array([c["idx"]], np.int32), 1, c["scale"])
    assert abs(ml[0, 0, 0, 0] - c["expected_m"]) <= 1e-15
    assert abs(ml[0, 0, 0, 1] - c["expected_l"]) <= 1e-15
    np.testing.assert_allclose(o[0, 0, 0], c["expected_o"], rtol=0, atol=1e-15)


def test_golden_ordered_skipping():
    c = G["ordered_skipping"]
    idx = np.array(c["idx"], np.int32)
    order = oracle.kap_order(idx, c["S"], c["block"], c["q_block"], c["table"])
    assert order.tolist() == c["expected_order"]
    S = c["S"]
    K = np.array([[[x, 0.0] for x in c["K_x"]]], np.float32)
    V = np.array([[[float(t), 1.0] for t in range(S)]], np.float32)
    Q = np.array([[c["q"]]], np.float32)
    for case in c["cases"]:
        O, steps, crit = oracle.osk_prefill_attn(bf(Q), c["q_pos"], bf(K), bf(V), c["block"], order, c["q_block"],
                                                 float(np.log(2.0)), case["tau"], lag=case["lag"])
        np.testing.assert_allclose(crit[0], c["expected_crit"], rtol=1e-13)
        assert steps[0] == case["expected_steps"], case
        np.testing.assert_allclose(O[0, 0], case["expected_o"], rtol=0, atol=1e-13)
