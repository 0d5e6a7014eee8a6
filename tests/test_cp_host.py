"""Host logic of context-parallel decode on CPU: the slicing of the caches, the
packed exchange buffers, and a two-rank step over a gloo group whose per-rank
arithmetic is the oracle's, which must equal the one-device oracle step."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from cross_layer_shared_b200 import cp
from synth import f32_to_bf16_bits


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_bounds_partition_every_sequence():
    lens = [0, 1, 5, 64, 1000, 13]
    for N in (1, 2, 3, 8):
        b = cp.shard_bounds(lens, N)
        assert b.shape == (N, len(lens), 2)
        for j, S in enumerate(lens):
            assert b[0, j, 0] == 0 and b[N - 1, j, 1] == S
            assert all(b[r, j, 1] == b[r + 1, j, 0] for r in range(N - 1))
            widths = b[:, j, 1] - b[:, j, 0]
            assert widths.min() >= 0 and widths.max() - widths.min() <= 1


def test_shard_cache_takes_each_head_group_slice():
    # row value = 1000*b + 100*g + t: the slice of (b, g) must be t in [lo, hi)
    lens, G, dim = [5, 3, 7], 2, 4
    rows = []
    for b, S in enumerate(lens):
        for g in range(G):
            for t in range(S):
                rows.append([1000 * b + 100 * g + t] * dim)
    cache = torch.tensor(rows, dtype=torch.float32).reshape(-1)
    lo, hi = [1, 0, 7], [4, 3, 7]
    out = cp.shard_cache(cache, lens, G, dim, lo, hi)
    want = [1000 * b + 100 * g + t for b in range(3) for g in range(G) for t in range(lo[b], hi[b])]
    assert out.shape == (len(want), dim)
    assert out[:, 0].tolist() == want and bool((out == out[:, :1]).all())


def test_packed_views():
    buf = torch.arange(2 * 2 * 3 * 4, dtype=torch.int32).view(2, 2, 3, 4)
    s, i = cp.cand_views(buf)
    assert s.dtype == torch.float32 and s.shape == (2, 3, 4) and s.stride(0) == 24
    assert torch.equal(i, buf[:, 1])
    rows, d = 3, 4
    n = cp.part_floats(rows, d)
    assert n % 4 == 0 and n >= rows * (d + 2)
    parts = torch.arange(2 * n, dtype=torch.float32).view(2, n)
    o, ml = cp.part_views(parts, rows, d)
    assert o.shape == (2, rows, d) and ml.shape == (2, rows, 2)
    assert o[1, 0, 0] == n and ml[1, 0, 0] == n + rows * d


def test_rank_state_rejects_empty_slices_and_bad_ranks():
    x = torch.zeros(0)
    with pytest.raises(ValueError, match="no token"):
        cp.CPRank(8, 7, x, x, x, [0, 0], 16, 4, 64, 8, 2, 128, 2, 0.1)
    with pytest.raises(ValueError, match="outside"):
        cp.CPRank(2, 2, x, x, x, [5, 5], 16, 4, 64, 8, 2, 128, 2, 0.1)


# ---------------------------------------------------------------- two ranks over gloo
def _order_keys(sc):
    """fp32 scores -> the 32-bit keys the kernels order them by (-0 == +0)."""
    u = np.ascontiguousarray(sc, dtype=np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def _threshold(g, prefix, need, all_, bits):
    """The previous level's threshold digit from every rank's histograms g
    [N, bins]: where the keys above, summed over the ranks, first reach
    `need`.  Returns (prefix, need, all, digit)."""
    if all_:
        return prefix, need, True, -1
    tot = g.sum(0)
    above = 0
    for dgt in range(len(tot) - 1, -1, -1):
        if above + int(tot[dgt]) >= need:
            return (prefix << bits) | dgt, need - above, False, dgt
        above += int(tot[dgt])
    return prefix, need, True, -1


class OracleRank:
    """A rank whose arithmetic runs on the CPU (the oracle's scores and
    attention; the exchange's histograms and thresholds in numpy), with
    CPRank's interface and exchange layouts."""

    def __init__(self, N, rank, KI, K, V, local_len, k, Hkv, d, L_g, Hq, scale):
        self.N, self.rank, self.k = N, rank, k
        self.KI, self.K, self.V = KI, K, V
        self.len = np.asarray(local_len, np.int32)
        self.off = np.concatenate([[0], np.cumsum(self.len)]).astype(np.int64)
        self.Hkv, self.d, self.L_g, self.Hq, self.scale = Hkv, d, L_g, Hq, scale
        self.B = len(local_len)
        self.rows = L_g * self.B * Hq

    def scores_local(self, qI, w, stream=None):
        self.sc = oracle.index_score(qI, w, self.KI, self.off, np.arange(self.B), self.len - 1,
                                     ld=max(int(self.len.max()), 1))
        return self.sc

    def radix_level(self, level, gathered=None, stream=None):
        bins = (4096, 4096, 256)[level]
        if level == 0:
            self.state = [(0, self.k, False)] * self.B
        else:
            g = gathered.numpy()
            self.state = [_threshold(g[:, b], *self.state[b], 12)[:3] for b in range(self.B)]
        hist = np.zeros((self.B, bins), np.int32)
        for b in range(self.B):
            prefix, need, all_ = self.state[b]
            if all_:
                continue
            key = _order_keys(self.sc[b, :self.len[b]])
            if level == 0:
                dg = key >> 20
            elif level == 1:
                dg = (key[key >> 20 == prefix] >> 8) & 0xFFF
            else:
                dg = key[key >> 8 == prefix] & 0xFF
            hist[b] = np.bincount(dg.astype(np.int64), minlength=bins)
        return torch.from_numpy(hist)

    def radix_select(self, gathered, stream=None):
        g = gathered.numpy()
        self.local_idx = np.full((self.B, self.k), -1, np.int32)
        for b in range(self.B):
            T, need, all_, dgt = _threshold(g[:, b], *self.state[b], 8)
            key = _order_keys(self.sc[b, :self.len[b]])
            if all_:
                keep = np.ones(len(key), bool)
            else:
                before = int(g[:self.rank, b, dgt].sum())
                take = min(max(need - before, 0), int(g[self.rank, b, dgt]))
                eq = key == T
                keep = (key > T) | (eq & (np.cumsum(eq) - 1 < take))
            sel = np.nonzero(keep)[0]
            self.local_idx[b, :len(sel)] = sel
        return self.local_idx

    def partial(self, Q, stream=None):
        o, ml = oracle.sparse_decode_attn_partial(Q, self.K, self.V, self.off, self.len, self.local_idx,
                                                  self.Hkv, self.scale)
        buf = torch.zeros(cp.part_floats(self.rows, self.d), dtype=torch.float32)
        bo, bml = cp.part_views(buf, self.rows, self.d)
        bo.copy_(torch.from_numpy(o.reshape(self.rows, self.d)))
        bml.copy_(torch.from_numpy(ml.reshape(self.rows, 2)))
        return buf

    def combine(self, gathered, O=None, out_dtype=None, stream=None):
        o, ml = cp.part_views(gathered, self.rows, self.d)
        out = oracle.combine_partials(o.double().numpy(), ml.double().numpy())
        return torch.from_numpy(out).view(self.L_g, self.B, self.Hq, self.d)


def _inputs():
    rng = np.random.default_rng(7)
    lens, H_I, d_I, Hq, Hkv, d, L_g, k = [37, 12, 50], 4, 16, 4, 2, 8, 3, 10
    T = sum(lens)
    qI = f32_to_bf16_bits(rng.standard_normal((len(lens), H_I, d_I)).astype(np.float32))
    w = rng.uniform(0.1, 1.0, (len(lens), H_I)).astype(np.float32)
    # indexer keys from a few values: ties across the slice boundaries
    KI = f32_to_bf16_bits((rng.integers(-2, 3, (T, d_I)) * 0.25).astype(np.float32))
    K = f32_to_bf16_bits(rng.standard_normal(T * Hkv * d).astype(np.float32))
    V = f32_to_bf16_bits(rng.standard_normal(T * Hkv * d).astype(np.float32))
    Q = f32_to_bf16_bits(rng.standard_normal((L_g, len(lens), Hq, d)).astype(np.float32))
    return lens, H_I, d_I, Hq, Hkv, d, L_g, k, qI, w, KI, K, V, Q


def _one_device():
    lens, H_I, d_I, Hq, Hkv, d, L_g, k, qI, w, KI, K, V, Q = _inputs()
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    L = np.asarray(lens, np.int32)
    sc = oracle.index_score(qI, w, KI, off, np.arange(len(lens)), L - 1)
    idx = oracle.topk(sc, L, k)
    return oracle.sparse_decode_attn(Q, K, V, off, L, idx, Hkv, 0.3), idx


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lens, H_I, d_I, Hq, Hkv, d, L_g, k, qI, w, KI, K, V, Q = _inputs()
        bnd = cp.shard_bounds(lens, world)[rank]
        lo, hi = bnd[:, 0], bnd[:, 1]
        sl = lambda c, G, dim: cp.shard_cache(torch.from_numpy(c.astype(np.int32)), lens, G, dim, lo, hi).numpy()
        KI_l = sl(KI.reshape(-1), 1, d_I).astype(np.uint16)
        K_l = sl(K, Hkv, d).astype(np.uint16).reshape(-1)
        V_l = sl(V, Hkv, d).astype(np.uint16).reshape(-1)
        me = OracleRank(world, rank, KI_l, K_l, V_l, hi - lo, k, Hkv, d, L_g, Hq, 0.3)
        O = cp.step(me, cp.nccl_exchange(world), qI, w, Q)
        results[rank] = (O.numpy(), [list(lo[b] + t for t in me.local_idx[b] if t >= 0) for b in range(len(lens))])
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_step_equals_the_one_device_step(world):
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, free_port(), results), nprocs=world, start_method="spawn",
                       join=True)
    want_O, want_idx = _one_device()
    for r in range(world):
        np.testing.assert_allclose(results[r][0], want_O, rtol=0, atol=1e-5)
    for b in range(want_idx.shape[0]):
        got = sorted(t for r in range(world) for t in results[r][1][b])
        assert got == [int(t) for t in want_idx[b] if t >= 0], b


def _oracle_ranks(world):
    lens, H_I, d_I, Hq, Hkv, d, L_g, k, qI, w, KI, K, V, Q = _inputs()
    bnd = cp.shard_bounds(lens, world)
    ranks = []
    for r in range(world):
        lo, hi = bnd[r, :, 0], bnd[r, :, 1]
        sl = lambda c, G, dim: cp.shard_cache(torch.from_numpy(c.astype(np.int32)), lens, G, dim, lo, hi).numpy()
        ranks.append(OracleRank(world, r, sl(KI.reshape(-1), 1, d_I).astype(np.uint16),
                                sl(K, Hkv, d).astype(np.uint16).reshape(-1), sl(V, Hkv, d).astype(np.uint16).reshape(-1),
                                hi - lo, k, Hkv, d, L_g, Hq, 0.3))
    return ranks, qI, w, Q


@pytest.mark.parametrize("order", ["rank-major", "reversed"])
def test_the_exchange_order_matters(order):
    """All ranks in one process, phase by phase: rank-major gathers give the
    one-device result; gathering in reverse rank order (a plausible layout
    slip) breaks the selection's tie rule: the ties at the threshold go to
    the wrong ranks."""
    world = 3
    ranks, qI, w, Q = _oracle_ranks(world)
    flip = (lambda t: t.flip(0)) if order == "reversed" else (lambda t: t)
    for r in ranks:
        r.scores_local(qI, w)
    h = flip(torch.stack([r.radix_level(0) for r in ranks]))
    h = flip(torch.stack([r.radix_level(1, h) for r in ranks]))
    h = flip(torch.stack([r.radix_level(2, h) for r in ranks]))
    for r in ranks:
        r.radix_select(h)
    parts = torch.stack([r.partial(Q) for r in ranks])
    O = ranks[0].combine(parts).numpy()
    want_O, _ = _one_device()
    same = np.abs(O - want_O).max() <= 1e-5
    assert same == (order == "rank-major")
