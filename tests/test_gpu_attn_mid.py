"""The warp-level MMA attention for 9 to 128 query rows per (sequence, KV
head) on few units (a short batch with few KV heads: the shapes where
sa_sparse_decode_attn takes it) against the oracle, through the C ABI.
Cases span 9 to 128 rows (the last warp's rows partly real), one and many
key slices, a k that is not a whole number of 16-entry passes, padding, a
row with no valid entry, both output types, and a reported out-of-range
entry."""
import math

import numpy as np
import pytest
import torch

import cross_layer_shared_b200 as sa
import oracle
import synth
from synth import gpu as sgpu
from tests import parity
from tests.test_gpu_parity import _attn_case, assert_status_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    from cross_layer_shared_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda")


def _pick(k):
    return lambda rng, b, S: np.sort(rng.choice(S, k, replace=False))


def _padded(k):
    def f(rng, b, S):
        r = rng.choice(S, k, replace=False)
        r[rng.random(k) < 0.3] = -1
        return r if b else np.full(k, -1)  # sequence 0: nothing valid
    return f


# name: (L, Hq, Hkv, lens, k, index rows, out dtype); R = L * Hq / Hkv rows
CASES = {
    "r9_one_warp": (9, 1, 1, [3000], 2048, _pick(2048), torch.float32),
    "r16_two_units": (2, 8, 1, [2500, 4000], 700, _pick(700), torch.float32),
    "r17_partial_second_warp": (17, 1, 1, [5000], 1000, _pick(1000), torch.float32),
    "r32_c1_shape": (4, 8, 1, [4096], 256, _pick(256), torch.float32),
    "r64_k_ragged": (8, 8, 1, [6000], 333, _pick(333), torch.float32),
    "r96_group_bf16": (24, 4, 1, [20000], 2048, _pick(2048), torch.bfloat16),
    "r128_eight_warps": (16, 8, 1, [9000], 1000, _pick(1000), torch.float32),
    "r24_padding_and_empty_row": (3, 8, 1, [900, 400], 256, _padded(256), torch.float32),
    "r32_one_slice": (4, 8, 1, [100], 16, _pick(16), torch.bfloat16),
}


@pytest.mark.parametrize("name", list(CASES))
def test_mid_rows_match_oracle(name, dev):
    L, Hq, Hkv, lens, k, fn, dt = CASES[name]
    assert 8 < L * (Hq // Hkv) <= 128
    err, ws = _attn_case(dev, L, len(lens), Hq, Hkv, lens, k, fn, seed=100 + list(CASES).index(name), out_dtype=dt)
    assert_status_ok(ws)
    assert err <= (parity.ATOL_BF16 if dt == torch.bfloat16 else parity.ATOL_F32), err


def test_mid_rows_report_an_out_of_range_entry(dev):
    """An entry at or past its sequence's length is reported (kernel id 3,
    the entry, its value) and skipped: the output matches the oracle over
    the other entries."""
    rng = np.random.default_rng(9)
    d, S, L, Hq = 128, 300, 4, 8
    Q = synth.f32_to_bf16_bits(rng.standard_normal((L, 1, Hq, d)).astype(np.float32))
    K = synth.f32_to_bf16_bits(rng.standard_normal(S * d).astype(np.float32))
    V = synth.f32_to_bf16_bits(rng.standard_normal(S * d).astype(np.float32))
    idx = np.arange(64, dtype=np.int32)
    idx[5] = S + 7
    ws = sa.workspace(sa.sparse_decode_attn_workspace_size(L, 1, Hq, 1, d, 64), dev)
    O = sa.sparse_decode_attn(sgpu.to_dev_bf16(Q, dev), sgpu.to_dev_bf16(K, dev), sgpu.to_dev_bf16(V, dev),
                              torch.tensor([0, S], device=dev), torch.tensor([S], dtype=torch.int32, device=dev),
                              torch.from_numpy(idx[None]).to(dev), 1, 1 / math.sqrt(d), out_dtype=torch.float32,
                              ws=ws)
    code, det = sa.read_status(ws)
    assert code == sa.SA_ERR_DEVICE and det[0] == 3 and det[1] == 5 and det[2] == S + 7
    keep = idx.copy()
    keep[5] = -1
    want = oracle.sparse_decode_attn(Q, K, V, [0, S], [S], keep[None], 1, 1 / math.sqrt(d))
    assert np.abs(O.cpu().numpy() - want).max() <= parity.ATOL_F32
