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
