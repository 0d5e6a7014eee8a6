"""The CUDA-core sparse decode attention (at most 8 query rows per sequence
and KV head: the per-layer decode mode) against the oracle, through the C
ABI.  Cases span every row-count instantiation (1, 2, 4, 8 rows, and 3, 5, 6
rows run on the next larger one), every cluster size of the key split (1, 2,
4, 8 CTAs), a k that is not a multiple of a warp's 16-entry pass, padding,
a row with no valid entry, bf16 output, and the full-size per-layer step."""
import math

import numpy as np
import pytest
import torch

import cross_layer_shared_b200 as sa
import oracle
import synth
from synth import gpu as sgpu
from tests import parity
from tests.test_gpu_parity import _attn_case, _plan_inputs, assert_status_ok, check_group

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
    "r1_one_pass": (1, 4, 4, [300, 50], 16, _pick(16), torch.float32),
    "r2_ragged_k": (2, 8, 8, [700, 900], 100, _pick(100), torch.float32),
    "r3_gqa3_two_ctas": (1, 6, 2, [1000], 129, _pick(129), torch.float32),
    "r4_four_ctas": (1, 32, 8, [5000, 3000, 4000], 300, _pick(300), torch.float32),
    "r5_eight_ctas": (5, 4, 4, [2000], 1000, _pick(1000), torch.float32),
    "r6_k2048": (3, 4, 2, [3000, 2500], 2048, _pick(2048), torch.float32),
    "r8_k4096": (2, 8, 2, [9000], 4096, _pick(4096), torch.float32),
    "r4_padding_and_empty_row": (1, 8, 2, [900, 400], 256, _padded(256), torch.float32),
    "r4_bf16_out": (1, 32, 8, [4000, 4000], 2048, _pick(2048), torch.bfloat16),
}


@pytest.mark.parametrize("name", list(CASES))
def test_small_rows_match_oracle(name, dev):
    L, Hq, Hkv, lens, k, fn, dt = CASES[name]
    assert L * (Hq // Hkv) <= 8
    err, ws = _attn_case(dev, L, len(lens), Hq, Hkv, lens, k, fn, seed=list(CASES).index(name), out_dtype=dt)
    assert_status_ok(ws)
    assert err <= (parity.ATOL_BF16 if dt == torch.bfloat16 else parity.ATOL_F32), err


def test_small_rows_empty_row_is_zero(dev):
    """A sequence whose index row holds no valid entry gets zero rows."""
    rng = np.random.default_rng(3)
    d, S = 128, 64
    Q = sgpu.to_dev_bf16(synth.f32_to_bf16_bits(rng.standard_normal((1, 1, 4, d)).astype(np.float32)), dev)
    K = sgpu.to_dev_bf16(synth.f32_to_bf16_bits(rng.standard_normal(S * d).astype(np.float32)), dev)
    idx = torch.full((1, 48), -1, dtype=torch.int32, device=dev)
    O = sa.sparse_decode_attn(Q, K, K, torch.tensor([0, S], device=dev), torch.tensor([S], dtype=torch.int32, device=dev),
                              idx, 1, 1 / math.sqrt(d), out_dtype=torch.float32)
    assert torch.count_nonzero(O).item() == 0


def test_small_rows_entry_order_does_not_matter(dev):
    """One (sequence, KV head) over 2048 entries (a cluster of 8 key slices):
    the same selection given sorted and reversed lands in other slices and
    passes, yet gives outputs equal within fp32 rounding, both matching the
    oracle."""
    rng = np.random.default_rng(11)
    d, S, k = 128, 20000, 2048
    Qb = synth.f32_to_bf16_bits(rng.standard_normal((1, 1, 4, d)).astype(np.float32))
    Kb = synth.f32_to_bf16_bits(rng.standard_normal(S * d).astype(np.float32))
    Vb = synth.f32_to_bf16_bits(rng.standard_normal(S * d).astype(np.float32))
    sel = np.sort(rng.choice(S, k, replace=False)).astype(np.int32)
    Q, K, V = (sgpu.to_dev_bf16(x, dev) for x in (Qb, Kb, Vb))
    off, ln = torch.tensor([0, S], device=dev), torch.tensor([S], dtype=torch.int32, device=dev)
    outs = []
    for s in (sel, sel[::-1].copy()):
        outs.append(sa.sparse_decode_attn(Q, K, V, off, ln, torch.from_numpy(s[None]).to(dev), 1, 1 / math.sqrt(d),
                                          out_dtype=torch.float32))
    assert (outs[0] - outs[1]).abs().max().item() <= parity.ATOL_F32
    want = oracle.sparse_decode_attn(Qb, Kb, Vb, [0, S], [S], sel[None], 1, 1 / math.sqrt(d))
    assert np.abs(outs[0].cpu().numpy() - want).max() <= parity.ATOL_F32


def test_per_layer_step_c3_matches_oracle(dev):
    """c3 (4 x 131072 tokens, 24 layers, 32 query / 8 KV heads, top-2048) as
    a decoder runs it: one attention launch per layer, 4 rows per (sequence,
    KV head).  Every sequence, every layer, against the oracle over the
    step's index; and against the fused step's output."""
    cfg = synth.workload("c3")
    wl = sgpu.decode_workload(cfg, dev)
    qI, w, KI, K, V = _plan_inputs(cfg, wl)
    scores = torch.empty((cfg.B, cfg.S_max), dtype=torch.float32, device=dev)
    args = (cfg.pattern, qI, w, KI, K, V, wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k, wl["Q"], cfg.Hkv, cfg.scale)
    O, idx = sa.decode_step(*args, out_dtype=torch.float32, scores=scores, per_layer=True)
    torch.cuda.synchronize()
    check_group(cfg, 0, list(range(cfg.B)), scores.cpu().numpy(), idx.cpu().numpy(),
                {torch.float32: O.cpu().numpy()})
    O_fused, idx_fused = sa.decode_step(*args, out_dtype=torch.float32)
    assert torch.equal(idx_fused, idx)
    assert (O_fused - O).abs().max().item() <= parity.ATOL_F32
