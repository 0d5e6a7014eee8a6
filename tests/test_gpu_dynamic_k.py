"""Dynamic k by routing mass (CLSA, k chosen per query; the rule is a
reading): the GPU against the oracle on the same scores.

m, the count a row keeps, is decided by fp64 sums taken in different orders
on the two sides.  A GPU count is accepted when it is a valid answer within
that rounding: its running sum (sequential fp64, top-k order) reaches the
target up to 1e-12 relative, and one token fewer does not.  Given m, the kept
set is unique (the m first tokens of the top-k order), so the index must then
equal the oracle's top-m bit for bit."""
import math

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

REL = 1e-12


@pytest.fixture(scope="module")
def dev():
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda")


def check_row(row, n, k_max, tau, got_idx, got_m, what=""):
    s = np.asarray(row[:n], np.float32)
    if n == 0:
        assert got_m == 0 and np.all(got_idx == -1), what
        return
    order = np.lexsort((np.arange(n), -s.astype(np.float64)))  # score desc, index asc
    run = np.cumsum(s[order].astype(np.float64))
    target = tau * float(np.sum(s.astype(np.float64)))
    _, (m_ora,) = oracle.topk_dynamic(s[None], [n], k_max, tau)
    if got_m != m_ora:  # a different count is accepted only inside the rounding band
        assert 1 <= got_m <= min(n, k_max), what
        reaches = run[got_m - 1] >= target * (1 - REL) or got_m == min(n, k_max)
        fewer_short = got_m == 1 or run[got_m - 2] < target * (1 + REL)
        assert reaches and fewer_short, f"{what}: m {got_m} vs oracle {m_ora}"
    want = np.full(k_max, -1, np.int32)
    want[:got_m] = np.sort(order[:got_m])
    assert np.array_equal(got_idx, want), what


def _rows(rng, n):
    rows, nval = [], []
    rows.append(np.exp(3 * rng.standard_normal(n)).astype(np.float32)); nval.append(n)      # heavy tail
    rows.append((rng.integers(0, 5, n) / 4).astype(np.float32)); nval.append(n)             # heavy ties
    z = np.zeros(n, np.float32); z[rng.choice(n, 40, replace=False)] = 1.0
    rows.append(z); nval.append(n)                                                          # zero tail
    rows.append(rng.random(n).astype(np.float32)); nval.append(min(n, 1500))                # n_valid < k_max
    rows.append(rng.random(n).astype(np.float32)); nval.append(0)                           # empty row
    rows.append(np.full(n, 0.5, np.float32)); nval.append(n)                                # all equal
    return rows, nval


@pytest.mark.parametrize("n,replicas", [(100_000, 1), (9001, 10)])
@pytest.mark.parametrize("tau", [0.3, 0.9, 1.0])
def test_topk_dynamic_matches_oracle(dev, n, replicas, tau):
    rng = np.random.default_rng(int(tau * 100) + n)
    rows, nval = _rows(rng, n)
    S = np.concatenate([np.stack(rows)] * replicas)
    nv = np.array(nval * replicas, np.int32)
    for k_max in (2048, 64):
        ws = sa.workspace(sa.lib().sa_topk_dynamic_workspace_size(len(S), n, k_max), dev)
        idx, counts = sa.topk_dynamic(torch.from_numpy(S).to(dev), torch.from_numpy(nv).to(dev), n, k_max, tau,
                                      ws=ws)
        code, det = sa.read_status(ws)
        assert code == 0, (code, det)
        got, cnt = idx.cpu().numpy(), counts.cpu().numpy()
        for r in range(len(S)):
            check_row(S[r], int(nv[r]), k_max, tau, got[r], int(cnt[r]), f"row {r} k_max={k_max} tau={tau}")


def test_attn_route_dynamic_k_c3_full_size_sampled(dev):
    """The c3 group under the attention-routing reading with a dynamic k
    (tau = 0.9 of each sequence's routing mass, at most 2048): the index
    against the oracle's dynamic k on the GPU's routing scores, and the 23
    sparse layers against the oracle over that index (sequences 0 and 3)."""
    cfg = synth.workload("c3")
    wl = sgpu.decode_workload(cfg, dev, groups=[0])
    gr = wl["groups"][0]
    ws = sa.workspace(sa.decode_step_attn_route_workspace_size(cfg.B, cfg.S_max, cfg.Hq, cfg.Hkv, cfg.d, cfg.k,
                                                               cfg.L), dev)
    scores = torch.empty((cfg.B, cfg.S_max), dtype=torch.float32, device=dev)
    O, idx, counts = sa.decode_step_attn_route(wl["Q"], gr["K"], gr["V"], wl["seq_off"], wl["seq_len"], cfg.S_max,
                                               cfg.k, cfg.Hkv, cfg.scale, out_dtype=torch.float32, ws=ws,
                                               scores=scores, tau=0.9)
    code, det = sa.read_status(ws)
    assert code == 0, (code, det)
    sc, idx_h, cnt, O_h = scores.cpu().numpy(), idx.cpu().numpy(), counts.cpu().numpy(), O.cpu().numpy()
    Q = cfg.Q()
    for b in range(cfg.B):
        S = cfg.seq_lens[b]
        check_row(sc[b], S, cfg.k, 0.9, idx_h[b], int(cnt[b]), f"c3 b={b}")
    for b in (0, 3):
        m = int(cnt[b])
        Kc, remap, mm = parity.compact_selected(lambda h, r: cfg.KV_rows(0, b, h, r, "K"), idx_h[b, :m], cfg.Hkv,
                                                cfg.d)
        Vc, _, _ = parity.compact_selected(lambda h, r: cfg.KV_rows(0, b, h, r, "V"), idx_h[b, :m], cfg.Hkv, cfg.d)
        want = oracle.sparse_decode_attn(Q[1:, b:b + 1], Kc.ravel(), Vc.ravel(), [0, mm], [mm], remap[None], cfg.Hkv,
                                         cfg.scale)[:, 0]
        assert np.abs(O_h[1:, b] - want).max() <= parity.ATOL_F32, b
