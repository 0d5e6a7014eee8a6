"""Context-parallel decode on the GPU against the oracle: the unnormalised
attention, the log-sum-exp combine, the global selection (by histogram
exchange, and over gathered candidates), and whole sharded steps (all ranks
emulated on one device, phase by phase) against the one-device step.  Every
call goes through the C ABI."""
import math

import numpy as np
import pytest
import torch

import cross_layer_shared_b200 as sa
import oracle
import synth
from cross_layer_shared_b200 import build, cp
from synth import gpu as sgpu
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda")


def assert_status_ok(ws):
    code, det = sa.read_status(ws)
    assert code == 0, f"device status {code} detail {det}"


def bf16_dev(bits, dev):
    return sgpu.to_dev_bf16(np.asarray(bits, np.uint16), dev)


def bits(rng, shape, s=1.0):
    return synth.f32_to_bf16_bits((rng.standard_normal(shape) * s).astype(np.float32))


# --------------------------------------------------------------------------
@pytest.mark.parametrize("L,B,Hq,Hkv,lens,k,empty_row", [
    (4, 3, 16, 4, [900, 333, 1500], 300, True),   # many units: one CTA per (sequence, KV head)
    (6, 1, 16, 1, [5000], 1024, False),           # one unit: keys split over a cluster
    (2, 2, 32, 8, [2000, 64], 512, True),         # a sequence shorter than k
])
def test_partial_attention_matches_the_oracle(dev, L, B, Hq, Hkv, lens, k, empty_row):
    rng = np.random.default_rng(sum(lens) + k)
    d = 128
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(seq_off[-1])
    Q, K, V = bits(rng, (L, B, Hq, d)), bits(rng, T * Hkv * d), bits(rng, T * Hkv * d)
    idx = np.full((B, k), -1, np.int32)
    for b in range(B):
        m = min(k, lens[b])
        idx[b, :m] = np.sort(rng.choice(lens[b], m, replace=False))
    if empty_row:
        idx[-1] = -1
    scale = 1 / math.sqrt(d)
    ws = sa.workspace(sa.sparse_decode_attn_workspace_size(L, B, Hq, Hkv, d, k), dev)
    args = (bf16_dev(Q, dev), bf16_dev(K, dev), bf16_dev(V, dev), torch.from_numpy(seq_off).to(dev),
            torch.tensor(lens, dtype=torch.int32, device=dev), torch.from_numpy(idx).to(dev), Hkv, scale)
    o, ml = sa.sparse_decode_attn_partial(*args, ws=ws)
    full = sa.sparse_decode_attn(*args, out_dtype=torch.float32, ws=ws)
    one = sa.combine_partials(o.view(1, -1, d), ml.view(1, -1, 2), out_dtype=torch.float32)
    assert_status_ok(ws)
    o, ml = o.cpu().numpy().astype(np.float64), ml.cpu().numpy().astype(np.float64)
    o_ora, ml_ora = oracle.sparse_decode_attn_partial(Q, K, V, seq_off, lens, idx, Hkv, scale)
    live = ml_ora[..., 1] > 0
    assert np.all(ml[~live][:, 1] == 0) and np.all(o[~live] == 0)
    # m is the kernel's reference logit (within 8 of the max); the row's
    # log-sum-exp m + log2(l) is what is defined
    assert np.all(ml[live][:, 0] <= ml_ora[live][:, 0] + 1e-4)
    assert np.all(ml[live][:, 0] >= ml_ora[live][:, 0] - 8 - 1e-4)
    lse = ml[live][:, 0] + np.log2(ml[live][:, 1])
    lse_ora = ml_ora[live][:, 0] + np.log2(ml_ora[live][:, 1])
    assert np.abs(lse - lse_ora).max() <= 1e-4
    norm = o[live] / ml[live][:, 1:2]
    assert np.abs(norm - o_ora[live] / ml_ora[live][:, 1:2]).max() <= parity.ATOL_F32
    # one part merged alone is the normalised output (within fp32 rounding:
    # with few units the full call takes the warp-level MMA kernel)
    assert (one.view_as(full) - full).abs().max().item() <= parity.ATOL_F32


@pytest.mark.parametrize("B,lens,k,counts", [
    (3, [900, 333, 1500], 1024, [0, 100, 1024]),   # many units
    (1, [5000], 2048, [300]),                      # one unit over a cluster: splits of the 300 real entries
    (2, [4000, 64], 2048, [2048, 64]),
])
def test_partial_attention_reads_only_the_counted_entries(dev, B, lens, k, counts):
    """Entries past idx_count[b] are ignored even when they hold valid
    indices: the result is the oracle's over the counted prefix."""
    rng = np.random.default_rng(k + B)
    L, Hq, Hkv, d = 3, 16, 4, 128
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(seq_off[-1])
    Q, K, V = bits(rng, (L, B, Hq, d)), bits(rng, T * Hkv * d), bits(rng, T * Hkv * d)
    idx = np.full((B, k), -1, np.int32)
    for b in range(B):
        m = min(k, lens[b])
        idx[b, :m] = np.sort(rng.choice(lens[b], m, replace=False))
    scale = 1 / math.sqrt(d)
    ws = sa.workspace(sa.sparse_decode_attn_workspace_size(L, B, Hq, Hkv, d, k), dev)
    o, ml = sa.sparse_decode_attn_partial(bf16_dev(Q, dev), bf16_dev(K, dev), bf16_dev(V, dev),
                                          torch.from_numpy(seq_off).to(dev),
                                          torch.tensor(lens, dtype=torch.int32, device=dev),
                                          torch.from_numpy(idx).to(dev), Hkv, scale,
                                          idx_count=torch.tensor(counts, dtype=torch.int32, device=dev), ws=ws)
    got = sa.combine_partials(o.view(1, -1, d), ml.view(1, -1, 2), out_dtype=torch.float32).cpu().numpy()
    assert_status_ok(ws)
    cut = idx.copy()
    for b in range(B):
        cut[b, counts[b]:] = -1
    want = oracle.sparse_decode_attn(Q, K, V, seq_off, lens, cut, Hkv, scale).reshape(-1, d)
    assert np.abs(got - want).max() <= parity.ATOL_F32


@pytest.mark.parametrize("P", [1, 3, 8])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_combine_partials_matches_the_oracle(dev, P, out_dtype):
    rng = np.random.default_rng(100 + P)
    rows, d = 1003, 128
    l = rng.uniform(0.5, 50.0, (P, rows))
    l[rng.random((P, rows)) < 0.25] = 0.0
    l[:, 7] = 0.0  # a row no part reached
    m = rng.uniform(-20, 20, (P, rows))
    m[l == 0] = -np.inf
    o = (0.25 * rng.standard_normal((P, rows, d)) * l[..., None]).astype(np.float32)
    ml = np.stack([m, l], -1).astype(np.float32)
    n = cp.part_floats(rows, d)
    buf = torch.zeros((P, n), dtype=torch.float32, device=dev)
    bo, bml = cp.part_views(buf, rows, d)
    bo.copy_(torch.from_numpy(o))
    bml.copy_(torch.from_numpy(ml))
    got = sa.combine_partials(bo, bml, out_dtype=out_dtype).float().cpu().numpy()
    want = oracle.combine_partials(o.astype(np.float64), ml.astype(np.float64))
    tol = parity.ATOL_F32 if out_dtype == torch.float32 else parity.ATOL_BF16
    assert np.abs(got - want).max() <= tol
    assert np.all(got[7] == 0)


def _slice_candidates(rng, lens, N, k, levels):
    """Per-rank top-k (with scores) of each slice of random scores drawn from
    `levels` values (many ties); returns the packed [N, 2, B, k] block."""
    B = len(lens)
    full = [(rng.integers(0, levels, S) * 0.125).astype(np.float32) for S in lens]
    bnd = cp.shard_bounds(lens, N)
    cand = np.zeros((N, 2, B, k), np.int32)
    for r in range(N):
        w = max(1, int((bnd[r, :, 1] - bnd[r, :, 0]).max()))
        sc = np.zeros((B, w), np.float32)
        for b in range(B):
            lo, hi = bnd[r, b]
            sc[b, :hi - lo] = full[b][lo:hi]
        idx, ts = oracle.topk(sc, bnd[r, :, 1] - bnd[r, :, 0], k, with_scores=True)
        cand[r, 0] = ts.view(np.int32)
        cand[r, 1] = idx
    return cand


@pytest.mark.parametrize("N,lens,k,levels", [
    (1, [3000, 100], 256, 50),
    (2, [20000, 5000, 300, 9000], 2048, 1000),
    (8, [131072, 4000], 2048, 300),
    (8, [7, 5000, 64], 64, 4),
])
def test_cp_select_is_bit_exact(dev, N, lens, k, levels):
    rng = np.random.default_rng(N * 7 + k)
    cand = _slice_candidates(rng, lens, N, k, levels)
    g = torch.from_numpy(cand).to(dev)
    s, i = cp.cand_views(g)
    ws = sa.workspace(sa.cp_select_workspace_size(N, len(lens), k), dev)
    cnt = torch.empty(len(lens), dtype=torch.int32, device=dev)
    for r in range(N):
        got = sa.cp_select(s, i, r, local_count=cnt, ws=ws).cpu().numpy()
        want = oracle.cp_select(cand[:, 0].view(np.float32), cand[:, 1], r)
        assert np.array_equal(got, want), f"rank {r}"
        assert np.array_equal(cnt.cpu().numpy(), (want >= 0).sum(1)), f"rank {r} counts"
    assert_status_ok(ws)


def _radix_exchange(dev, full, lens, N, k):
    """Every rank's share of the global top-k by the histogram exchange, all
    ranks on this device: [N] local index arrays [B, k] and counts [B]."""
    B = len(lens)
    bnd = cp.shard_bounds(lens, N)
    ranks = []
    for r in range(N):
        n = (bnd[r, :, 1] - bnd[r, :, 0]).astype(np.int32)
        sc = np.zeros((B, max(1, int(n.max()))), np.float32)
        for b in range(B):
            sc[b, :n[b]] = full[b][bnd[r, b, 0]:bnd[r, b, 1]]
        ranks.append((torch.from_numpy(sc).to(dev), torch.from_numpy(n).to(dev),
                      sa.workspace(sa.cp_radix_workspace_size(B), dev)))
    h = torch.stack([sa.cp_radix_level(sc, n, k, N, 0, ws=ws) for sc, n, ws in ranks])
    h = torch.stack([sa.cp_radix_level(sc, n, k, N, 1, h, ws=ws) for sc, n, ws in ranks])
    h = torch.stack([sa.cp_radix_level(sc, n, k, N, 2, h, ws=ws) for sc, n, ws in ranks])
    out = []
    for r, (sc, n, ws) in enumerate(ranks):
        cnt = torch.empty(B, dtype=torch.int32, device=dev)
        idx = sa.cp_radix_select(sc, n, k, N, r, h, local_count=cnt, ws=ws)
        assert_status_ok(ws)
        out.append((idx.cpu().numpy(), cnt.cpu().numpy()))
    return out, bnd


@pytest.mark.parametrize("N,lens,k,kind", [
    (1, [3000, 100], 256, "levels"),            # one rank: the plain top-k
    (2, [20000, 5000, 300, 9000], 2048, "levels"),
    (3, [4096, 50, 7000], 512, "normal"),       # distinct scores, ragged slices
    (8, [131072, 4000], 2048, "levels"),        # c3's sharding
    (8, [7, 5000, 64], 64, "levels"),           # empty slices (7 tokens over 8 ranks), k above a sequence
    (4, [6000, 6000], 700, "one_value"),        # every score equal: ties decided by index alone
    (4, [3000, 3000], 300, "signed"),           # negative scores, -0 and +0
    (5, [40, 30], 128, "normal"),               # fewer tokens than k in all: every one selected
])
def test_radix_exchange_selects_the_global_top_k(dev, N, lens, k, kind):
    """The union of the ranks' shares, in global positions, is the oracle's
    top-k of the whole row (the lower index first among ties); each share
    is ascending, -1 padded, and counted."""
    rng = np.random.default_rng(N * 31 + k)
    if kind == "levels":      # few distinct values: ties across slice edges
        full = [(rng.integers(0, 300, S) * 0.125).astype(np.float32) for S in lens]
    elif kind == "one_value":
        full = [np.full(S, 0.5, np.float32) for S in lens]
    elif kind == "signed":
        full = [(rng.integers(-40, 40, S) * 0.25).astype(np.float32) for S in lens]
        for f in full:
            f[rng.random(len(f)) < 0.1] = -0.0
    else:
        full = [rng.standard_normal(S).astype(np.float32) for S in lens]
    shares, bnd = _radix_exchange(dev, full, lens, N, k)
    W = max(lens)
    rows = np.zeros((len(lens), W), np.float32)
    for b, f in enumerate(full):
        rows[b, :len(f)] = f
    want = oracle.topk(rows, lens, k)
    for b in range(len(lens)):
        got = []
        for r in range(N):
            idx, cnt = shares[r]
            row = idx[b]
            assert np.all(row[:cnt[b]] >= 0) and np.all(row[cnt[b]:] == -1), f"rank {r} b={b} padding"
            assert np.all(np.diff(row[:cnt[b]]) > 0), f"rank {r} b={b} order"
            assert np.all(row[:cnt[b]] < bnd[r, b, 1] - bnd[r, b, 0]), f"rank {r} b={b} range"
            got += [int(bnd[r, b, 0] + t) for t in row[:cnt[b]]]
        assert sorted(got) == [int(t) for t in want[b] if t >= 0], f"b={b}"


def test_radix_exchange_reports_a_negative_length(dev):
    sc = torch.zeros((2, 8), dtype=torch.float32, device=dev)
    n = torch.tensor([8, -3], dtype=torch.int32, device=dev)
    ws = sa.workspace(sa.cp_radix_workspace_size(2), dev)
    h = sa.cp_radix_level(sc, n, 4, 1, 0, ws=ws)
    code, det = sa.read_status(ws)
    assert code == sa.SA_ERR_DEVICE and det[0] == 9 and det[1] == 1 and det[2] == -3
    assert int(h[1].sum()) == 0 and int(h[0].sum()) == 8


# --------------------------------------------------------------------------
def _step_inputs(seed, lens, H_I=32, d_I=128, Hq=32, Hkv=8, d=128, L_g=3):
    rng = np.random.default_rng(seed)
    B, T = len(lens), sum(lens)
    return dict(qI=bits(rng, (B, H_I, d_I), 0.25), w=rng.uniform(0.05, 1.0, (B, H_I)).astype(np.float32),
                KI=bits(rng, (T, d_I), 0.25), K=bits(rng, T * Hkv * d), V=bits(rng, T * Hkv * d),
                Q=bits(rng, (L_g, B, Hq, d)), H_I=H_I, d_I=d_I, Hq=Hq, Hkv=Hkv, d=d, L_g=L_g)


@pytest.mark.parametrize("N,lens,k", [(2, [6000, 2500, 777], 512), (4, [6000, 2500, 3], 512), (8, [20000], 2048)])
def test_emulated_context_parallel_step_matches_one_device(dev, N, lens, k):
    x = _step_inputs(N + k, lens)
    B, d, Hkv, L_g, Hq = len(lens), x["d"], x["Hkv"], x["L_g"], x["Hq"]
    scale = 1 / math.sqrt(d)
    KI, K, V = bf16_dev(x["KI"], dev).view(-1, x["d_I"]), bf16_dev(x["K"], dev), bf16_dev(x["V"], dev)
    qI, w, Q = bf16_dev(x["qI"], dev), torch.from_numpy(x["w"]).to(dev), bf16_dev(x["Q"], dev)
    bnd = cp.shard_bounds(lens, N)
    ranks = []
    for r in range(N):
        lo, hi = bnd[r, :, 0], bnd[r, :, 1]
        ranks.append(cp.CPRank(N, r, cp.shard_cache(KI, lens, 1, x["d_I"], lo, hi),
                               cp.shard_cache(K, lens, Hkv, d, lo, hi).view(-1),
                               cp.shard_cache(V, lens, Hkv, d, lo, hi).view(-1), hi - lo, k, x["H_I"], x["d_I"], Hq,
                               Hkv, d, L_g, scale))
    O_cp, local = cp.emulate_step(ranks, qI, w, Q, out_dtype=torch.float32)
    for r in ranks:
        for ws in (r.ws_index, r.ws_radix, r.ws_attn):
            assert_status_ok(ws)
    # the one-device step on the whole context
    seq_off, seq_len = cp.seq_tables(lens, dev)
    S_max = max(lens)
    scores = sa.index_score(qI, w, KI, seq_off, seq_len, S_max)
    idx1 = sa.topk(scores, seq_len, S_max, k)
    O1 = sa.sparse_decode_attn(Q, K, V, seq_off, seq_len, idx1, Hkv, scale, out_dtype=torch.float32)
    idx1 = idx1.cpu().numpy()
    # the same index: the union of the ranks' shares, in global positions
    for b in range(B):
        got = sorted(int(bnd[r, b, 0] + t) for r in range(N) for t in local[r][b].cpu().numpy() if t >= 0)
        assert got == [int(t) for t in idx1[b] if t >= 0], f"b={b}"
    # the same output as one device, and as the oracle on that index
    assert (O_cp - O1).abs().max().item() <= parity.ATOL_F32
    off_h = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    want = oracle.sparse_decode_attn(x["Q"], x["K"], x["V"], off_h, lens, idx1, Hkv, scale)
    assert np.abs(O_cp.cpu().numpy() - want).max() <= parity.ATOL_F32
    # and the index against the oracle's scores (exact outside the tie band)
    sc = scores.cpu().numpy()
    for b in range(B):
        S = lens[b]
        ora = oracle.index_score(x["qI"][b:b + 1], x["w"][b:b + 1], x["KI"][off_h[b]:off_h[b + 1]], [0, S], [0],
                                 [S - 1])[0]
        parity.assert_topk_band(idx1[b], ora, S, k, f"b={b}")
        assert np.array_equal(idx1[b], oracle.topk(sc[b:b + 1, :S], [S], k)[0])


def test_emulated_step_bf16_output(dev):
    N, lens, k = 2, [3000, 1200], 256
    x = _step_inputs(5, lens)
    d, Hkv = x["d"], x["Hkv"]
    KI, K, V = bf16_dev(x["KI"], dev).view(-1, x["d_I"]), bf16_dev(x["K"], dev), bf16_dev(x["V"], dev)
    bnd = cp.shard_bounds(lens, N)
    ranks = [cp.CPRank(N, r, cp.shard_cache(KI, lens, 1, x["d_I"], bnd[r, :, 0], bnd[r, :, 1]),
                       cp.shard_cache(K, lens, Hkv, d, bnd[r, :, 0], bnd[r, :, 1]).view(-1),
                       cp.shard_cache(V, lens, Hkv, d, bnd[r, :, 0], bnd[r, :, 1]).view(-1),
                       bnd[r, :, 1] - bnd[r, :, 0], k, x["H_I"], x["d_I"], x["Hq"], Hkv, d, x["L_g"], 0.1)
             for r in range(N)]
    O, local = cp.emulate_step(ranks, bf16_dev(x["qI"], dev), torch.from_numpy(x["w"]).to(dev),
                               bf16_dev(x["Q"], dev), out_dtype=torch.bfloat16)
    assert O.dtype == torch.bfloat16
    idx = np.full((len(lens), k), -1, np.int32)
    for b in range(len(lens)):
        g = sorted(int(bnd[r, b, 0] + t) for r in range(N) for t in local[r][b].cpu().numpy() if t >= 0)
        idx[b, :len(g)] = g
    off_h = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    want = oracle.sparse_decode_attn(x["Q"], x["K"], x["V"], off_h, lens, idx, Hkv, 0.1)
    assert np.abs(O.float().cpu().numpy() - want).max() <= parity.ATOL_BF16
