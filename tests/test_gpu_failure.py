"""Failure detection on the GPU without faulting it: a bounded wait is made to
run out (an mbarrier that nothing ever arrives on, a limit of 2 ms instead of
the kernels' 1 s), the give-up is reported through the status block with the
kernel id and the limit, and the context stays usable -- a normal call right
after runs and matches the oracle."""
import math
import time

import numpy as np
import pytest
import torch

import cross_layer_shared_b200 as sa
import oracle
import synth
from cross_layer_shared_b200 import build
from synth import gpu as sgpu
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda")


def test_bounded_wait_gives_up_and_the_context_stays_usable(dev):
    ws = sa.workspace(sa.WS_HEADER_BYTES, dev)
    limit = 2_000_000
    t0 = time.perf_counter()
    sa.wait_probe(ws, limit)
    code, det = sa.read_status(ws)  # synchronises
    elapsed = time.perf_counter() - t0
    assert code == sa.SA_ERR_TIMEOUT, (code, det)
    assert det[0] == 8 and det[3] == limit, det
    assert elapsed < 0.5, elapsed  # the wait gave up after ~limit, not after the kernels' 1 s
    # the status is sticky until cleared, then a second probe reports again
    sa.clear_status(ws)
    assert sa.read_status(ws)[0] == 0
    sa.wait_probe(ws, 50_000)
    assert sa.read_status(ws)[0] == sa.SA_ERR_TIMEOUT
    # a normal call on the same context right after: sparse attention of a
    # small group against the oracle, with a clear status
    rng = np.random.default_rng(9)
    d, L, B, Hq, Hkv, k, lens = 128, 3, 2, 8, 2, 256, [700, 1200]
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(seq_off[-1])
    Q = synth.f32_to_bf16_bits(rng.standard_normal((L, B, Hq, d)).astype(np.float32))
    K = synth.f32_to_bf16_bits(rng.standard_normal(T * Hkv * d).astype(np.float32))
    V = synth.f32_to_bf16_bits(rng.standard_normal(T * Hkv * d).astype(np.float32))
    idx = np.stack([np.sort(rng.choice(s, k, replace=False)) for s in lens]).astype(np.int32)
    aws = sa.workspace(sa.sparse_decode_attn_workspace_size(L, B, Hq, Hkv, d, k), dev)
    O = sa.sparse_decode_attn(sgpu.to_dev_bf16(Q, dev), sgpu.to_dev_bf16(K, dev), sgpu.to_dev_bf16(V, dev),
                              torch.from_numpy(seq_off).to(dev), torch.tensor(lens, dtype=torch.int32, device=dev),
                              torch.from_numpy(idx).to(dev), Hkv, 1 / math.sqrt(d), out_dtype=torch.float32, ws=aws)
    code, det = sa.read_status(aws)
    assert code == 0, (code, det)
    want = oracle.sparse_decode_attn(Q, K, V, seq_off, lens, idx, Hkv, 1 / math.sqrt(d))
    assert np.abs(O.cpu().numpy() - want).max() <= parity.ATOL_F32
