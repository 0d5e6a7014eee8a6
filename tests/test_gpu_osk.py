"""CoSA's priority-ordered block execution with early skipping, through the C
ABI, against the oracle: the union table and each query block's priority
list bit for bit, the number of steps each unit ran checked against the
oracle's progressive score (every share computed in fp64; the kernel's
decision may differ only where a share lies within 0.1 % of tau), and the
output against the oracle's attention over exactly the steps the unit ran.

Cases span the GQA ratios whose query blocks fill a 128-row tile (G = 1, 2,
4, 8), ragged query blocks and a ragged last KV block, a table of fewer
than three steps (no vote is ever read), an odd table (a last step of one
block), queries spread through the context (rows that see nothing in the
first steps), tau = 0 (never stops: the plain union attention), tau above
1 (stops at once), both output types, and the 2048-query chunk at full
size with the attention drawn to its hot regions (sampled units)."""
import math

import numpy as np
import pytest
import torch

import cross_layer_shared_b200 as sa
import oracle
import synth
from synth import gpu as sgpu
from tests import parity
from tests.test_gpu_parity import assert_status_ok

pytestmark = pytest.mark.gpu

LAG = 2       # steps already in flight when a unit decides to stop
BAND = 1e-3   # relative band around tau inside which either decision is accepted


@pytest.fixture(scope="module")
def dev():
    from cross_layer_shared_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda")


def bf16_dev(bits, dev):
    return sgpu.to_dev_bf16(bits, dev)


def assert_steps_valid(steps, crit, tau, n_steps, what=""):
    """steps[u] (tiles the GPU ran) is a valid outcome of the rule for the
    oracle's per-step scores crit[u]: the stop step clears tau and no earlier
    step did, each up to the band."""
    lo, hi = tau * (1 - BAND), tau * (1 + BAND)
    for u, N in enumerate(steps):
        c = crit[u]
        if N < n_steps:
            ns = N - 1 - LAG
            assert ns >= 0, (what, u, N)
            assert c[ns] < hi, (what, u, N, c[ns], tau)
            assert np.all(c[:ns] >= lo), (what, u, N, np.min(c[:ns]) if ns else None)
        else:
            assert N == n_steps, (what, u, N, n_steps)
            assert np.all(c[:max(0, n_steps - 1 - LAG)] >= lo), (what, u)


def _make_case(seed, Nq, Hq, Hkv, S, k, spread=False, concentrated=True, d=128):
    """Seeded chunk: 6 hot regions of 128 tokens whose K rows lie along a
    per-group direction that the (optionally biased) queries share; each
    query's index holds hot tokens and random visible ones (-1 padded)."""
    rng = np.random.default_rng(seed)
    G = Hq // Hkv
    q_pos = (np.sort(rng.choice(S, Nq, replace=False)) if spread else np.arange(S - Nq, S)).astype(np.int32)
    dirs = rng.standard_normal((Hkv, d))
    dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
    slots = max(1, (S - 128) // 64)
    hot_start = np.sort(rng.choice(slots, min(6, slots), replace=False)) * 64
    hot = np.concatenate([np.arange(s, min(S, s + 128)) for s in hot_start])
    K = rng.standard_normal((Hkv, S, d))
    V = rng.standard_normal((Hkv, S, d))
    Q = rng.standard_normal((Nq, Hq, d))
    if concentrated:
        for g in range(Hkv):
            K[g, hot] += 8.0 * dirs[g]
            Q[:, g * G:(g + 1) * G] += 16.0 * dirs[g]
    idx = np.full((Nq, k), -1, np.int32)
    for i, p in enumerate(q_pos):
        vis_hot = hot[hot <= p]
        nh = min(len(vis_hot), k // 2)
        a = rng.choice(vis_hot, nh, replace=False) if nh else np.zeros(0, np.int64)
        rest = rng.permutation(np.setdiff1d(np.unique(rng.integers(0, p + 1, k)), a))[: k - nh - (i % 3)]
        row = np.sort(np.concatenate([a, rest]))
        idx[i, :len(row)] = row
    f = synth.f32_to_bf16_bits
    return (q_pos, f(Q.astype(np.float32)), f(K.astype(np.float32)), f(V.astype(np.float32)), idx)


def _run(dev, q_pos, Q, K, V, idx, tau, out_dtype):
    Nq, Hq, d = Q.shape
    Hkv, S, _ = K.shape
    scale = 1 / math.sqrt(d)
    ws = sa.workspace(sa.osk_prefill_workspace_size(S, Nq, Hq, Hkv, d, idx.shape[1], 64), dev)
    indptr, indices, order, steps, O = sa.osk_prefill(
        torch.from_numpy(idx).to(dev), torch.from_numpy(q_pos).to(dev), bf16_dev(Q, dev), bf16_dev(K, dev),
        bf16_dev(V, dev), 64, scale, tau, out_dtype=out_dtype, ws=ws)
    torch.cuda.synchronize()
    assert_status_ok(ws)
    return (indptr.cpu().numpy(), indices.cpu().numpy(), order.cpu().numpy(), steps.cpu().numpy(),
            O.float().cpu().numpy(), scale)


# name: (seed, Nq, Hq, Hkv, S, k, tau, spread, concentrated, out dtype)
CASES = {
    "g4_concentrated_ragged": (61, 100, 8, 2, 20000, 256, 1e-3, False, True, torch.float32),
    "g1_tau0_is_the_union_attention": (62, 200, 2, 2, 9000, 128, 0.0, False, True, torch.float32),
    "g8_stops_at_once": (63, 40, 16, 2, 12000, 128, 2.0, False, False, torch.float32),
    "g2_spread_positions_bf16": (64, 150, 4, 2, 16000, 256, 1e-2, True, True, torch.bfloat16),
    "g4_odd_table": (65, 64, 8, 2, 448, 64, 0.05, False, False, torch.float32),
    "g4_short_table": (66, 40, 8, 2, 150, 32, 0.5, False, False, torch.float32),
    "g4_isotropic_no_skip": (67, 96, 8, 2, 30000, 512, 1e-3, False, False, torch.float32),
}


@pytest.mark.parametrize("name", list(CASES))
def test_osk_matches_oracle(name, dev):
    seed, Nq, Hq, Hkv, S, k, tau, spread, conc, dt = CASES[name]
    q_pos, Q, K, V, idx = _make_case(seed, Nq, Hq, Hkv, S, k, spread=spread, concentrated=conc)
    indptr, indices, order, steps, O, scale = _run(dev, q_pos, Q, K, V, idx, tau, dt)
    # the union table, bit for bit
    ip_o, ind_o = oracle.block_union(idx, S, 64, Hkv)
    assert np.array_equal(indptr, ip_o) and np.array_equal(indices[:indptr[-1]], ind_o)
    nT = int(indptr[1])
    # the priority lists, bit for bit
    G = Hq // Hkv
    q_block = 128 // G
    ord_o = oracle.kap_order(idx, S, 64, q_block, ind_o[:nT])
    assert np.array_equal(order[:, :nT], ord_o)
    # the steps each unit ran, against the oracle's progressive score
    n_steps = (nT + 1) // 2
    _, steps_o, crit = oracle.osk_prefill_attn(Q, q_pos, K, V, 64, ord_o, q_block, scale, tau, lag=LAG)
    assert_steps_valid(steps, crit, tau, n_steps, name)
    # the output over exactly those steps
    O_o, _, _ = oracle.osk_prefill_attn(Q, q_pos, K, V, 64, ord_o, q_block, scale, tau, lag=LAG, steps_in=steps)
    tol = parity.ATOL_F32 if dt == torch.float32 else parity.ATOL_BF16
    assert np.abs(O - O_o).max() <= tol, np.abs(O - O_o).max()
    if tau == 0.0:
        assert np.all(steps == n_steps)
        want = oracle.paged_prefill_attn(Q, q_pos, K, V, 64, ip_o, ind_o, scale)
        assert np.abs(O - want).max() <= tol
    if tau > 1.0:
        assert np.all(steps == min(n_steps, 1 + LAG))
    if name == "g4_concentrated_ragged":
        assert steps.min() < n_steps, "the hot blocks come first and the rest is skipped"
    if name == "g4_short_table":
        assert n_steps <= 2 and np.all(steps == n_steps)


def test_kap_order_alone_matches_oracle(dev):
    """sa_kap_order on its own: several query-block sizes, padding and
    entries past S (not counted), a table of every block."""
    rng = np.random.default_rng(68)
    S, Nq, k = 5000, 77, 96
    nb = (S + 63) // 64
    idx = rng.integers(-5, S + 300, (Nq, k)).astype(np.int32)
    T = np.arange(nb, dtype=np.int32)
    indptr = torch.tensor([0, nb], dtype=torch.int32, device=dev)
    indices = torch.from_numpy(T).to(dev)
    ws = sa.workspace(sa.kap_order_workspace_size(), dev)
    for q_block in (1, 7, 32, 128):
        order = sa.kap_order(torch.from_numpy(idx).to(dev), S, 64, q_block, indptr, indices, ws=ws)
        torch.cuda.synchronize()
        assert_status_ok(ws)
        want = oracle.kap_order(idx, S, 64, q_block, T)
        assert np.array_equal(order.cpu().numpy(), want), q_block


def _host_idx_c4(cfg, seed):
    """A seeded stand-in for the chunk's per-query selection: about half of
    each row from the hot regions, the rest random visible tokens."""
    rng = np.random.default_rng(seed)
    hot = np.array([p + i for p in cfg.regions() for i in range(cfg.region_len)], dtype=np.int64)
    idx = np.full((cfg.chunk, cfg.k), -1, np.int32)
    for i, p in enumerate(cfg.q_pos):
        a = rng.choice(hot, cfg.k // 2, replace=False)
        rest = rng.permutation(np.setdiff1d(np.unique(rng.integers(0, p + 1, cfg.k)), a))[: cfg.k - len(a)]
        row = np.sort(np.concatenate([a, rest]))
        idx[i, :len(row)] = row
    return idx


def test_osk_c4_concentrated_full_size_sampled(dev):
    """The 2048-query chunk over 131072 tokens with the attention drawn to
    the hot regions, at full size: union and every priority list bit for
    bit; steps and outputs of sampled units (each checked over its whole
    KV group's cache)."""
    cfg = synth.workload("c4-concentrated")
    wl = sgpu.prefill_workload(cfg, dev)
    idx = _host_idx_c4(cfg, 69)
    tau = 2.0 ** -10
    G = cfg.Hq // cfg.Hkv
    q_block = 128 // G
    ws = sa.workspace(sa.osk_prefill_workspace_size(cfg.S, cfg.chunk, cfg.Hq, cfg.Hkv, cfg.d, cfg.k, cfg.block), dev)
    indptr, indices, order, steps, O = sa.osk_prefill(torch.from_numpy(idx).to(dev), wl["q_pos"], wl["Q"], wl["K"],
                                                      wl["V"], cfg.block, cfg.scale, tau, out_dtype=torch.float32,
                                                      ws=ws)
    torch.cuda.synchronize()
    assert_status_ok(ws)
    indptr, indices, order, steps = (t.cpu().numpy() for t in (indptr, indices, order, steps))
    ip_o, ind_o = oracle.block_union(idx, cfg.S, cfg.block, cfg.Hkv)
    assert np.array_equal(indptr, ip_o) and np.array_equal(indices[:indptr[-1]], ind_o)
    nT = int(indptr[1])
    ord_o = oracle.kap_order(idx, cfg.S, cfg.block, q_block, ind_o[:nT])
    assert np.array_equal(order[:, :nT], ord_o)
    n_steps = (nT + 1) // 2
    n_qb = ord_o.shape[0]
    assert steps.max() < n_steps // 4, "most of the table is skipped on this chunk"
    Q = cfg.Q()
    O_h = O.cpu().numpy()
    for g, i in ((0, 0), (5, 37), (7, n_qb - 1)):
        Kg = cfg.KV_rows(g, np.arange(cfg.S), "K")[None]
        Vg = cfg.KV_rows(g, np.arange(cfg.S), "V")[None]
        Qg = Q[:, g * G:(g + 1) * G]
        u = g * n_qb + i
        _, s_o, crit = oracle.osk_prefill_attn(Qg, cfg.q_pos, Kg, Vg, cfg.block, ord_o, q_block, cfg.scale, tau,
                                               lag=LAG, units=[i])
        assert_steps_valid(steps[u:u + 1], crit[i:i + 1], tau, n_steps, f"unit {g},{i}")
        O_o, _, _ = oracle.osk_prefill_attn(Qg, cfg.q_pos, Kg, Vg, cfg.block, ord_o, q_block, cfg.scale, tau,
                                            lag=LAG, units=[i], steps_in=np.full(n_qb, steps[u], np.int32))
        rows = slice(i * q_block, min(cfg.chunk, (i + 1) * q_block))
        err = np.abs(O_h[rows, g * G:(g + 1) * G] - O_o[rows]).max()
        assert err <= parity.ATOL_F32, (g, i, err)
