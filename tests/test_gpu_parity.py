"""CUDA path vs the CPU oracle, stage by stage and end to end, on the seeded
workloads (full size, sampled sequences where the oracle would be slow) and
on edge cases.  Every call goes through the C ABI (libsa.so)."""
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


# --------------------------------------------------------------------------
def test_generator_twin_is_bit_exact(dev):
    rng = np.random.default_rng(0)
    for seed, tid, scale, n in ((1237, 2, 0.125, 1 << 20), (1239, 5 + 64 * 3, 1.0, (1 << 20) + 13)):
        t = sgpu.normal_bf16_gpu(n, seed, tid, scale, dev)
        pick = np.unique(np.concatenate([rng.integers(0, n, 4096), [0, n - 1, n - 2]]))
        got = t.view(torch.int16).cpu().numpy().view(np.uint16)[pick]
        want = synth.normal_bf16_at(seed, tid, pick.astype(np.uint64), scale)
        assert np.array_equal(got, want)
    # offset form (the fill of a slice far into a stream)
    off = 3_000_000_017
    t = sgpu.normal_bf16_gpu(1000, 5, 9, 1.0, dev, offset=off)
    want = synth.normal_bf16_at(5, 9, np.arange(off, off + 1000, dtype=np.uint64), 1.0)
    assert np.array_equal(t.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c5"])
def test_decode_workload_tensors_match_host_rows(dev, name):
    """Every device tensor of the decode workloads (first group; planted rows
    included) equals the host generator's rows bit for bit, on sampled rows
    of every sequence and KV head."""
    cfg = synth.workload(name)
    wl = sgpu.decode_workload(cfg, dev, groups=[0])
    gr = wl["groups"][0]
    rng = np.random.default_rng(11)

    def bits(t):
        return t.view(torch.int16).cpu().numpy().view(np.uint16)

    planted = {(b, t) for (b, t, _, _) in cfg.planted(0)}
    for b in range(0, cfg.B, max(1, cfg.B // 4)):
        S = cfg.seq_lens[b]
        rows = np.unique(np.concatenate([rng.integers(0, S, 64), [0, S - 1],
                                         [t for (bb, t) in planted if bb == b][:8]])).astype(np.int64)
        got = bits(gr["KI"][torch.from_numpy(cfg.seq_off[b] + rows).to(dev)])
        assert np.array_equal(got, cfg.KI_rows(0, b, rows)), f"KI b={b}"
        K3 = gr["K"].view(-1, cfg.d)
        V3 = gr["V"].view(-1, cfg.d)
        for h in (0, cfg.Hkv - 1):
            flat = torch.from_numpy(cfg.seq_off[b] * cfg.Hkv + h * S + rows).to(dev)
            assert np.array_equal(bits(K3[flat]), cfg.KV_rows(0, b, h, rows, "K")), f"K b={b} h={h}"
            assert np.array_equal(bits(V3[flat]), cfg.KV_rows(0, b, h, rows, "V")), f"V b={b} h={h}"
    assert np.array_equal(bits(wl["Q"]), cfg.Q())
    assert np.array_equal(bits(gr["qI"]), cfg.qI(0))


def test_prefill_workload_tensors_match_host_rows(dev):
    cfg = synth.workload("c4")
    wl = sgpu.prefill_workload(cfg, dev)
    rng = np.random.default_rng(12)
    rows = np.unique(np.concatenate([rng.integers(0, cfg.S, 256), cfg.hot_ki_rows()[0][:16], [cfg.S - 1]]))
    KI = cfg.KI_full()
    got = wl["KI"][torch.from_numpy(rows).to(dev)].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, KI[rows])
    for h in (0, cfg.Hkv - 1):
        for which in ("K", "V"):
            got = wl[which][h][torch.from_numpy(rows).to(dev)].view(torch.int16).cpu().numpy().view(np.uint16)
            assert np.array_equal(got, cfg.KV_rows(h, rows, which)), f"{which} h={h}"


def test_key_split_count_does_not_change_the_output(dev):
    """One (sequence, KV head) alone is split over 8 CTAs of a cluster; the
    same data inside a batch of 148 units runs unsplit: same output within
    the fp32 tolerance (only the merge order differs)."""
    rng = np.random.default_rng(21)
    d, k, S, Hq, L = 128, 1024, 5000, 4, 6
    K = synth.f32_to_bf16_bits(rng.standard_normal(S * d).astype(np.float32))
    V = synth.f32_to_bf16_bits(rng.standard_normal(S * d).astype(np.float32))
    Q = synth.f32_to_bf16_bits(rng.standard_normal((L, 1, Hq, d)).astype(np.float32))
    sel = np.sort(rng.choice(S, k, replace=False)).astype(np.int32)
    one = sa.sparse_decode_attn(bf16_dev(Q, dev), bf16_dev(K, dev), bf16_dev(V, dev),
                                torch.tensor([0, S], device=dev), torch.tensor([S], dtype=torch.int32, device=dev),
                                torch.from_numpy(sel[None]).to(dev), 1, 1 / math.sqrt(d), out_dtype=torch.float32)
    B = 148  # as many units as SMs: no room to split
    Kb = bf16_dev(np.tile(K, B), dev)
    Vb = bf16_dev(np.tile(V, B), dev)
    Qb = bf16_dev(np.repeat(Q, B, axis=1), dev)
    offs = torch.arange(0, (B + 1) * S, S, device=dev)
    many = sa.sparse_decode_attn(Qb, Kb, Vb, offs, torch.full((B,), S, dtype=torch.int32, device=dev),
                                 torch.from_numpy(np.tile(sel, (B, 1))).to(dev), 1, 1 / math.sqrt(d),
                                 out_dtype=torch.float32)
    err = (many - one.expand(-1, B, -1, -1)).abs().max().item()
    assert err <= parity.ATOL_F32, err


# --------------------------------------------------------------------------
def decode_group_parity(cfg, g, seqs, dev, out_dtypes=(torch.bfloat16, torch.float32)):
    wl = sgpu.decode_workload(cfg, dev, groups=[g])
    gr = wl["groups"][g]
    ws = sa.workspace(max(sa.lib().sa_topk_workspace_size(cfg.B, cfg.S_max, cfg.k),
                          sa.lib().sa_index_score_workspace_size(cfg.B)), dev)
    scores = sa.index_score(gr["qI"], gr["w"], gr["KI"], wl["seq_off"], wl["seq_len"], cfg.S_max, ws=ws)
    idx = sa.topk(scores, wl["seq_len"], cfg.S_max, cfg.k, ws=ws)
    layers = list(cfg.groups[g])
    Qg = wl["Q"][layers[0]:layers[-1] + 1].contiguous()
    outs = {}
    for dt in out_dtypes:
        aws = sa.workspace(sa.sparse_decode_attn_workspace_size(len(layers), cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.k), dev)
        outs[dt] = sa.sparse_decode_attn(Qg, gr["K"], gr["V"], wl["seq_off"], wl["seq_len"], idx, cfg.Hkv, cfg.scale,
                                         out_dtype=dt, ws=aws)
        assert_status_ok(aws)
    assert_status_ok(ws)
    scores_h = scores.cpu().numpy()
    idx_h = idx.cpu().numpy()
    outs_h = {dt: o.float().cpu().numpy() for dt, o in outs.items()}
    check_group(cfg, g, seqs, scores_h, idx_h, outs_h)
    return idx_h, scores_h


def check_group(cfg, g, seqs, scores_h, idx_h, outs_h):
    """Stage by stage against the oracle for the sequences `seqs` of group g:
    scores within the fp32 bound; the index bit-exact against the oracle's
    top-k of the GPU's scores and exact outside the tie band against the
    oracle's own scores; every layer's output within the dtype's tolerance
    of the oracle's attention over the GPU's index.  outs_h maps an output
    dtype to the group's output rows [L_g, B, Hq, d]."""
    layers = list(cfg.groups[g])
    qI, w, Q = cfg.qI(g), cfg.w(g), cfg.Q()
    for b in seqs:
        S = cfg.seq_lens[b]
        KI = cfg.KI_rows(g, b, np.arange(S))
        ora = oracle.index_score(qI[b:b + 1], w[b:b + 1], KI, [0, S], [0], [S - 1])[0]
        parity.assert_scores_close(scores_h[b, :S], ora, parity.index_error_bound(qI[b], w[b], KI), f"{cfg.name} b={b}")
        exact = oracle.topk(scores_h[b:b + 1, :S], [S], cfg.k)[0]
        assert np.array_equal(idx_h[b], exact), f"{cfg.name} b={b}: top-k differs on identical scores"
        parity.assert_topk_band(idx_h[b], ora, S, cfg.k, f"{cfg.name} b={b}")
        Kc, remap, m = parity.compact_selected(lambda h, r: cfg.KV_rows(g, b, h, r, "K"), idx_h[b], cfg.Hkv, cfg.d)
        Vc, _, _ = parity.compact_selected(lambda h, r: cfg.KV_rows(g, b, h, r, "V"), idx_h[b], cfg.Hkv, cfg.d)
        O_ora = oracle.sparse_decode_attn(Q[layers][:, b:b + 1], Kc.ravel(), Vc.ravel(), [0, m], [m], remap[None],
                                          cfg.Hkv, cfg.scale)[:, 0]
        for dt, O in outs_h.items():
            tol = parity.ATOL_F32 if dt == torch.float32 else parity.ATOL_BF16
            err = np.abs(O[:, b] - O_ora).max()
            assert err <= tol, f"{cfg.name} b={b} {dt}: max-abs {err} > {tol}"


def test_c1_decode_group_with_needles(dev):
    cfg = synth.workload("c1")
    idx_h, _ = decode_group_parity(cfg, 0, [0], dev)
    needles = [t for (_, t, _, kr) in cfg.planted(0) if kr is not None]
    assert set(needles) <= set(idx_h[0].tolist())


@pytest.mark.parametrize("name,group", [("c2", 0), ("c2", 1), ("c2", 2), ("c3", 0)])
def test_full_size_decode_group(name, group, dev):
    """Every sequence of every F group of c2 (8 x 32768 tokens, three groups)
    and of the c3 group (4 x 131072 tokens, 24 layers): scores, index and
    both output dtypes against the oracle."""
    cfg = synth.workload(name)
    decode_group_parity(cfg, group, list(range(cfg.B)), dev)


@pytest.mark.parametrize("group", [0, 11])
def test_c5_ragged_group_sampled(dev, group):
    cfg = synth.workload("c5")
    lens = np.array(cfg.seq_lens)
    seqs = [int(np.argmin(lens)), int(np.argmax(lens)), 7]
    decode_group_parity(cfg, group, seqs, dev, out_dtypes=(torch.bfloat16,))


# --------------------------------------------------------------------------
# 8 rows: many CTAs per row; 80 rows: one CTA per row.  Rows of at most
# 16384 keys (n = 16384, and a ragged 9001): shorter rows, split over fewer CTAs.
@pytest.mark.parametrize("n", [100_000, 16384, 9001])
@pytest.mark.parametrize("replicas", [1, 10])
def test_topk_edge_cases(dev, replicas, n):
    rng = np.random.default_rng(3)
    rows, nval, ks = [], [], []
    rows.append(np.full(n, 0.75, np.float32)); nval.append(5000)                           # all equal
    rows.append((rng.integers(0, 20, n) / 4).astype(np.float32)); nval.append(n)           # heavy ties at threshold
    rows.append(rng.standard_normal(n).astype(np.float32)); nval.append(n)                 # negative scores
    z = np.zeros(n, np.float32); z[::2] = -0.0; z[5::7] = 1.0; rows.append(z); nval.append(n)  # signed zeros
    rows.append(rng.random(n).astype(np.float32)); nval.append(1500)                       # n_valid < k
    rows.append(rng.random(n).astype(np.float32)); nval.append(0)                          # empty row
    big = (1.0 + np.arange(n, dtype=np.float64) * 2 ** -23).astype(np.float32)            # one huge bucket
    rows.append(rng.permutation(big)); nval.append(n)
    rows.append(rng.random(n).astype(np.float32)); nval.append(2048)                       # n_valid == k
    nval = [min(v, n) for v in nval]
    S = np.concatenate([np.stack(rows)] * replicas)
    nv = np.array(nval * replicas, np.int32)
    rows = rows * replicas
    for k in (1, 2048, 3000):
        d_scores = torch.from_numpy(S).to(dev)
        ws = sa.workspace(sa.lib().sa_topk_workspace_size(len(rows), n, k), dev)
        idx, ts = sa.topk(d_scores, torch.from_numpy(nv).to(dev), n, k, want_scores=True, ws=ws)
        assert_status_ok(ws)
        want, want_s = oracle.topk(S, nv, k, with_scores=True)
        got = idx.cpu().numpy()
        for r in range(len(rows)):
            assert np.array_equal(got[r], want[r]), f"row {r} k={k}"
        assert np.array_equal(ts.cpu().numpy().view(np.uint32), want_s.view(np.uint32)) or \
            np.array_equal(ts.cpu().numpy(), want_s)


def test_topk_reports_bad_n_valid(dev):
    s = torch.rand(2, 1000, device=dev)
    ws = sa.workspace(256, dev)
    idx = sa.topk(s, torch.tensor([1000, 5000], dtype=torch.int32, device=dev), 1000, 10, ws=ws)
    code, det = sa.read_status(ws)
    assert code == sa.SA_ERR_DEVICE and det[0] == 2 and det[2] == 5000
    parity.assert_valid_index_row(idx[1].cpu().numpy(), 1000, 10)


# --------------------------------------------------------------------------
def _attn_case(dev, L, B, Hq, Hkv, lens, k, idx_fn, seed=0, out_dtype=torch.float32):
    rng = np.random.default_rng(seed)
    d = 128
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(seq_off[-1])
    Q = synth.f32_to_bf16_bits(rng.standard_normal((L, B, Hq, d)).astype(np.float32))
    K = synth.f32_to_bf16_bits(rng.standard_normal(T * Hkv * d).astype(np.float32))
    V = synth.f32_to_bf16_bits(rng.standard_normal(T * Hkv * d).astype(np.float32))
    idx = np.stack([idx_fn(rng, b, lens[b]) for b in range(B)]).astype(np.int32)
    ws = sa.workspace(sa.sparse_decode_attn_workspace_size(L, B, Hq, Hkv, d, k), dev)
    O = sa.sparse_decode_attn(bf16_dev(Q, dev), bf16_dev(K, dev), bf16_dev(V, dev), torch.from_numpy(seq_off).to(dev),
                              torch.tensor(lens, dtype=torch.int32, device=dev), torch.from_numpy(idx).to(dev), Hkv,
                              1 / math.sqrt(d), out_dtype=out_dtype, ws=ws)
    want = oracle.sparse_decode_attn(Q, K, V, seq_off, lens, idx, Hkv, 1 / math.sqrt(d))
    err = np.abs(O.float().cpu().numpy() - want).max()
    return err, ws


@pytest.mark.parametrize("case", ["full_selection", "padding", "ragged_k", "two_mtiles", "mha", "mqa"])
def test_attention_edge_cases(case, dev):
    def pick(k):
        return lambda rng, b, S: np.sort(rng.choice(S, k, replace=False))
    if case == "full_selection":  # k = S: dense attention
        err, ws = _attn_case(dev, 2, 2, 8, 2, [700, 700], 700, lambda rng, b, S: np.arange(S))
    elif case == "padding":       # -1 entries anywhere, and one row with none valid
        def f(rng, b, S):
            r = rng.choice(S, 256, replace=False)
            r[rng.random(256) < 0.3] = -1
            return r if b else np.full(256, -1)
        err, ws = _attn_case(dev, 3, 2, 8, 1, [900, 400], 256, f)
    elif case == "ragged_k":      # k not a multiple of the 128-key tile
        err, ws = _attn_case(dev, 4, 3, 16, 4, [500, 333, 1200], 300, pick(300))
    elif case == "two_mtiles":    # L*G = 200 query rows > one 128-row tile
        err, ws = _attn_case(dev, 25, 1, 32, 4, [3000], 512, pick(512))
    elif case == "mha":
        err, ws = _attn_case(dev, 2, 2, 8, 8, [1000, 800], 384, pick(384))
    else:
        err, ws = _attn_case(dev, 6, 1, 16, 1, [5000], 1024, pick(1024), out_dtype=torch.bfloat16)
    assert_status_ok(ws)
    assert err <= (parity.ATOL_BF16 if case == "mqa" else parity.ATOL_F32), err


def test_attention_reports_out_of_range_index(dev):
    def f(rng, b, S):
        r = np.arange(64)
        r[3] = S + 5
        return r
    err, ws = _attn_case(dev, 1, 1, 4, 1, [100], 64, lambda rng, b, S: np.where(np.arange(64) == 3, -1, np.arange(64)))
    assert err <= parity.ATOL_F32
    rng = np.random.default_rng(1)
    d = 128
    Q = bf16_dev(synth.f32_to_bf16_bits(rng.standard_normal((1, 1, 4, d)).astype(np.float32)), dev)
    K = bf16_dev(synth.f32_to_bf16_bits(rng.standard_normal(100 * d).astype(np.float32)), dev)
    idx = torch.from_numpy(f(None, 0, 100).astype(np.int32)[None]).to(dev)
    ws = sa.workspace(1 << 20, dev)
    sa.sparse_decode_attn(Q, K, K, torch.tensor([0, 100], device=dev), torch.tensor([100], dtype=torch.int32, device=dev),
                          idx, 1, 0.0884, ws=ws)
    code, det = sa.read_status(ws)
    assert code == sa.SA_ERR_DEVICE and det[0] == 3 and det[2] == 105


# --------------------------------------------------------------------------
def test_decode_step_c1_matches_oracle_walk(dev):
    cfg = synth.workload("c1")
    wl = sgpu.decode_workload(cfg, dev)
    gr = wl["groups"][0]
    n = cfg.L
    O, idx = sa.decode_step(cfg.pattern, [gr["qI"]] + [None] * (n - 1), [gr["w"]] + [None] * (n - 1),
                            [gr["KI"]] + [None] * (n - 1), [gr["K"]] * n, [gr["V"]] * n, wl["seq_off"],
                            wl["seq_len"], cfg.S_max, cfg.k, wl["Q"], cfg.Hkv, cfg.scale, out_dtype=torch.float32)
    KI = cfg.KI_full(0)
    K, V = cfg.KV_full(0, "K"), cfg.KV_full(0, "V")
    O_ora, used = oracle.decode_step(cfg.pattern, [cfg.qI(0)] * n, [cfg.w(0)] * n, [KI] * n, cfg.seq_off, cfg.seq_lens,
                                     cfg.k, cfg.Q(), [K] * n, [V] * n, cfg.Hkv, cfg.scale)
    got_idx = idx.cpu().numpy()
    parity.assert_topk_band(got_idx[0], oracle.index_score(cfg.qI(0), cfg.w(0), KI, cfg.seq_off, [0],
                                                           [cfg.S_max - 1])[0], cfg.S_max, cfg.k)
    # every layer of the F,S,S,S walk reads the F layer's index
    assert all(np.array_equal(u, used[0]) for u in used)
    # the output, always: the oracle's attention over the GPU's (validated) index
    O_gpu_idx = oracle.sparse_decode_attn(cfg.Q(), K, V, cfg.seq_off, cfg.seq_lens, got_idx, cfg.Hkv, cfg.scale)
    assert np.abs(O.cpu().numpy() - O_gpu_idx).max() <= parity.ATOL_F32
    if np.array_equal(got_idx, used[0]):  # no tie inside the band moved the selection: the oracle's own walk too
        assert np.abs(O.cpu().numpy() - O_ora).max() <= parity.ATOL_F32


def test_decode_step_plan_c3_matches_oracle(dev):
    """The call the benchmark times: c3 (4 x 131072 tokens; one indexer pass
    and top-2048 shared by 24 cross-decoder layers over one KV cache; bf16
    outputs) through a DecodeStepPlan built as the benchmark builds it, every
    sequence checked stage by stage against the oracle: the scores the step
    left behind, its index, and all 24 layers' outputs."""
    cfg = synth.workload("c3")
    wl = sgpu.decode_workload(cfg, dev)
    n = cfg.L
    grs = wl["groups"]
    starts = [gr[0] for gr in cfg.groups]
    qI = [grs[starts.index(l)]["qI"] if l in starts else None for l in range(n)]
    w = [grs[starts.index(l)]["w"] if l in starts else None for l in range(n)]
    KI = [grs[starts.index(l)]["KI"] if l in starts else None for l in range(n)]
    gi = [max(i for i, s0 in enumerate(starts) if s0 <= l) for l in range(n)]
    K = [grs[gi[l]]["K"] for l in range(n)]
    V = [grs[gi[l]]["V"] for l in range(n)]
    plan = sa.DecodeStepPlan(cfg.pattern, qI, w, KI, K, V, wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k, wl["Q"],
                             cfg.Hkv, cfg.scale, out_dtype=torch.bfloat16)
    O, idx = plan.run()
    torch.cuda.synchronize()
    assert_status_ok(plan.ws)
    check_group(cfg, 0, list(range(cfg.B)), plan.scores.cpu().numpy(), idx.cpu().numpy(),
                {torch.bfloat16: O.float().cpu().numpy()})
    # a second run of the same plan gives the same bits
    O2, idx2 = plan.run()
    torch.cuda.synchronize()
    assert torch.equal(idx2, idx) and torch.equal(O2.view(torch.int16), O.view(torch.int16))


def _plan_inputs(cfg, wl):
    """Per-layer lists of a whole-pattern step, as the benchmark builds them."""
    n = cfg.L
    grs = wl["groups"]
    starts = [gr[0] for gr in cfg.groups]
    qI = [grs[starts.index(l)]["qI"] if l in starts else None for l in range(n)]
    w = [grs[starts.index(l)]["w"] if l in starts else None for l in range(n)]
    KI = [grs[starts.index(l)]["KI"] if l in starts else None for l in range(n)]
    gi = [max(i for i, s0 in enumerate(starts) if s0 <= l) for l in range(n)]
    K = [grs[gi[l]]["K"] for l in range(n)]
    V = [grs[gi[l]]["V"] for l in range(n)]
    return qI, w, KI, K, V


def test_decode_step_plan_c2_matches_oracle(dev):
    """c2 through a DecodeStepPlan (three F groups of F,S,S,S, B = 8, S =
    32768), as the benchmark would time it.  Every group's outputs, every
    sequence, against the oracle over that group's index; the last group's
    index and scores are also bit-equal to the standalone index-score and
    top-k calls on the same inputs."""
    cfg = synth.workload("c2")
    wl = sgpu.decode_workload(cfg, dev)
    qI, w, KI, K, V = _plan_inputs(cfg, wl)
    plan = sa.DecodeStepPlan(cfg.pattern, qI, w, KI, K, V, wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k, wl["Q"],
                             cfg.Hkv, cfg.scale, out_dtype=torch.float32)
    plan.run()
    O, idx = plan.run()  # a second run on the same workspace
    torch.cuda.synchronize()
    assert_status_ok(plan.ws)
    O_h = O.cpu().numpy()
    ws = sa.workspace(max(sa.lib().sa_topk_workspace_size(cfg.B, cfg.S_max, cfg.k),
                          sa.lib().sa_index_score_workspace_size(cfg.B)), dev)
    for g, layers in enumerate(cfg.groups):
        gr = wl["groups"][g]
        scores = sa.index_score(gr["qI"], gr["w"], gr["KI"], wl["seq_off"], wl["seq_len"], cfg.S_max, ws=ws)
        idx_g = sa.topk(scores, wl["seq_len"], cfg.S_max, cfg.k, ws=ws)
        if g == len(cfg.groups) - 1:
            assert torch.equal(idx_g, idx), "the step's index differs from the standalone top-k's"
            assert torch.equal(scores, plan.scores[:, :cfg.S_max])
        check_group(cfg, g, list(range(cfg.B)), scores.cpu().numpy(), idx_g.cpu().numpy(),
                    {torch.float32: O_h[layers[0]:layers[-1] + 1]})
    assert_status_ok(ws)


def test_decode_step_c5_group_matches_oracle(dev):
    """One c5 group (B = 32, ragged 8192..131072, F,S,S,S) through the step.
    Sampled sequences (shortest, longest, one more) against the oracle."""
    cfg = synth.workload("c5")
    wl = sgpu.decode_workload(cfg, dev, groups=[0])
    gr = wl["groups"][0]
    layers = list(cfg.groups[0])
    n = len(layers)
    Q = wl["Q"][layers[0]:layers[-1] + 1].contiguous()
    plan = sa.DecodeStepPlan("F" + "S" * (n - 1), [gr["qI"]] + [None] * (n - 1), [gr["w"]] + [None] * (n - 1),
                             [gr["KI"]] + [None] * (n - 1), [gr["K"]] * n, [gr["V"]] * n, wl["seq_off"],
                             wl["seq_len"], cfg.S_max, cfg.k, Q, cfg.Hkv, cfg.scale, out_dtype=torch.bfloat16)
    plan.run()
    O, idx = plan.run()
    torch.cuda.synchronize()
    assert_status_ok(plan.ws)
    lens = np.array(cfg.seq_lens)
    seqs = [int(np.argmin(lens)), int(np.argmax(lens)), 7]
    check_group(cfg, 0, seqs, plan.scores.cpu().numpy(), idx.cpu().numpy(), {torch.bfloat16: O.float().cpu().numpy()})


def test_decode_step_does_not_depend_on_workspace_contents(dev):
    """The workspace is scratch: a step on a workspace full of garbage (status
    block clear) gives the same index and outputs, bit for bit, as on a
    zeroed one, and as the general index-score and top-k calls."""
    rng = np.random.default_rng(17)
    lens, H_I, d_I, Hq, Hkv, d, k, pattern = [20000, 9000, 33000], 16, 128, 8, 2, 128, 512, "FSS"
    B, L = len(lens), len(pattern)
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(seq_off[-1])

    def bf(shape, sd=1.0):
        return bf16_dev(synth.f32_to_bf16_bits((rng.standard_normal(shape) * sd).astype(np.float32)), dev)

    qI, KI, K, V, Q = bf((B, H_I, d_I), 1 / 8), bf((T, d_I), 1 / 8), bf(T * Hkv * d), bf(T * Hkv * d), bf((L, B, Hq, d))
    w = torch.from_numpy(rng.uniform(0.1, 1.0, (B, H_I)).astype(np.float32)).to(dev)
    d_off = torch.from_numpy(seq_off).to(dev)
    d_len = torch.tensor(lens, dtype=torch.int32, device=dev)
    S_max = max(lens)
    none = [None] * (L - 1)
    args = (pattern, [qI] + none, [w] + none, [KI] + none, [K] * L, [V] * L, d_off, d_len, S_max, k, Q, Hkv,
            1 / math.sqrt(d))
    gws = sa.workspace(max(sa.lib().sa_topk_workspace_size(B, S_max, k), sa.lib().sa_index_score_workspace_size(B)),
                       dev)
    want = sa.topk(sa.index_score(qI, w, KI, d_off, d_len, S_max, ws=gws), d_len, S_max, k, ws=gws)
    nbytes = sa.decode_step_workspace_size(L, B, S_max, Hq, Hkv, d, k)
    O0, idx0 = sa.decode_step(*args, out_dtype=torch.float32, ws=sa.workspace(nbytes, dev))
    ws = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device=dev)
    ws[:sa.WS_HEADER_BYTES] = 0  # a clear header (status block, counters), garbage everywhere else
    for trial in range(2):
        O, idx = sa.decode_step(*args, out_dtype=torch.float32, ws=ws)
        torch.cuda.synchronize()
        assert_status_ok(ws)
        assert torch.equal(idx, want) and torch.equal(idx, idx0), f"trial {trial}: index differs"
        assert torch.equal(O, O0), f"trial {trial}: outputs differ"


def test_decode_step_append_and_per_layer(dev):
    """The new token's rows land in the caches bit-exactly (nothing else
    changes), the step over the appended caches matches the oracle on them,
    and one attention launch per layer gives the fused group's output bit for
    bit."""
    rng = np.random.default_rng(5)
    lens, H_I, d_I, Hq, Hkv, d, k, pattern = [3000, 1500], 4, 64, 8, 2, 128, 128, "FSSS"
    B, L = len(lens), len(pattern)
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(seq_off[-1])
    scale = 1.0 / math.sqrt(d)

    def bf(shape, sd=1.0):
        return synth.f32_to_bf16_bits((rng.standard_normal(shape) * sd).astype(np.float32))

    qI, KI, K, V, Q = bf((B, H_I, d_I), 1 / 8), bf((T, d_I), 1 / 8), bf(T * Hkv * d), bf(T * Hkv * d), bf((L, B, Hq, d))
    w = rng.uniform(0.1, 1.0, (B, H_I)).astype(np.float32)
    nKI, nK, nV = bf((B, d_I), 1 / 8), bf((B, Hkv, d)), bf((B, Hkv, d))
    KIa, Ka, Va = oracle.kv_append(KI, K, V, seq_off, lens, nKI, nK, nV, Hkv, d)
    dKI, dK, dV = bf16_dev(KI, dev), bf16_dev(K, dev), bf16_dev(V, dev)
    dqI, dw, dQ = bf16_dev(qI, dev), torch.from_numpy(w).to(dev), bf16_dev(Q, dev)
    d_off = torch.from_numpy(seq_off).to(dev)
    d_len = torch.tensor(lens, dtype=torch.int32, device=dev)
    none = [None] * (L - 1)
    common = ([dK] * L, [dV] * L, d_off, d_len, max(lens), k, dQ, Hkv, scale)
    O, idx = sa.decode_step(pattern, [dqI] + none, [dw] + none, [dKI] + none, *common, out_dtype=torch.float32,
                            new_KI=[bf16_dev(nKI, dev)] + none, new_K=[bf16_dev(nK, dev)] + none,
                            new_V=[bf16_dev(nV, dev)] + none)
    assert np.array_equal(dKI.cpu().view(torch.int16).numpy().view(np.uint16), KIa)
    assert np.array_equal(dK.cpu().view(torch.int16).numpy().view(np.uint16), Ka)
    assert np.array_equal(dV.cpu().view(torch.int16).numpy().view(np.uint16), Va)
    O_ora, used = oracle.decode_step(pattern, [qI] * L, [w] * L, [KIa] * L, seq_off, lens, k, Q, [Ka] * L, [Va] * L,
                                     Hkv, scale)
    got_idx = idx.cpu().numpy()
    for b in range(B):
        ora = oracle.index_score(qI[b:b + 1], w[b:b + 1], KIa, seq_off, [b], [lens[b] - 1])[0][:lens[b]]
        parity.assert_topk_band(got_idx[b], ora, lens[b], k, f"b={b}")
    # the output, always: the oracle's attention on the appended caches over the GPU's (validated) index
    O_gpu_idx = oracle.sparse_decode_attn(Q, Ka, Va, seq_off, lens, got_idx, Hkv, scale)
    assert np.abs(O.cpu().numpy() - O_gpu_idx).max() <= parity.ATOL_F32
    if np.array_equal(got_idx, used[0]):  # no tie inside the band moved the selection: the oracle's own walk too
        assert np.abs(O.cpu().numpy() - O_ora).max() <= parity.ATOL_F32
    # the caches now hold the new token: per-layer launches (R = G = 4 rows per
    # (b, g): the CUDA-core kernel) against the fused group (R = 16: the
    # tensor-core kernel) and against the oracle over the same index
    args = (pattern, [dqI] + none, [dw] + none, [dKI] + none, *common)
    O_fused, i_fused = sa.decode_step(*args, out_dtype=torch.float32)
    O_layer, i_layer = sa.decode_step(*args, out_dtype=torch.float32, per_layer=True)
    assert torch.equal(i_fused, i_layer)
    assert (O_fused - O_layer).abs().max().item() <= parity.ATOL_F32
    assert np.abs(O_layer.cpu().numpy() - O_gpu_idx).max() <= parity.ATOL_F32


def test_shared_index_equals_per_layer_recompute(dev):
    """F,F,F,F with identical indexer inputs gives what F,S,S,S gives."""
    cfg = synth.workload("c1")
    wl = sgpu.decode_workload(cfg, dev)
    gr = wl["groups"][0]
    n = 4
    common = ([gr["K"]] * n, [gr["V"]] * n, wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k, wl["Q"], cfg.Hkv, cfg.scale)
    O1, i1 = sa.decode_step("FFFF", [gr["qI"]] * n, [gr["w"]] * n, [gr["KI"]] * n, *common, out_dtype=torch.float32)
    O2, i2 = sa.decode_step("FSSS", [gr["qI"]] * n, [gr["w"]] * n, [gr["KI"]] * n, *common, out_dtype=torch.float32)
    assert torch.equal(i1, i2)
    # FFFF runs one layer per launch (8 rows per (b, g): the CUDA-core kernel),
    # FSSS one launch of 32 rows (the tensor-core kernel)
    assert (O1 - O2).abs().max().item() <= parity.ATOL_F32


def test_step_is_deterministic(dev):
    cfg = synth.workload("c1")
    wl = sgpu.decode_workload(cfg, dev)
    gr = wl["groups"][0]
    n = cfg.L
    args = ([gr["qI"]] + [None] * (n - 1), [gr["w"]] + [None] * (n - 1), [gr["KI"]] + [None] * (n - 1),
            [gr["K"]] * n, [gr["V"]] * n, wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k, wl["Q"], cfg.Hkv, cfg.scale)
    a = sa.decode_step(cfg.pattern, *args)
    b = sa.decode_step(cfg.pattern, *args)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16)) and torch.equal(a[1], b[1])


# --------------------------------------------------------------------------
def prefill_parity(cfg, dev, q_sample=None, heads=None):
    wl = sgpu.prefill_workload(cfg, dev)
    ws = sa.workspace(max(sa.lib().sa_index_score_prefill_workspace_size(cfg.chunk),
                          sa.lib().sa_topk_workspace_size(cfg.chunk, cfg.S, cfg.k)), dev)
    scores = sa.index_score_prefill(wl["qI"], wl["w"], wl["KI"], wl["q_pos"], cfg.S - 1, ws=ws)
    n_valid = (wl["q_pos"] + 1).to(torch.int32)
    idx = sa.topk(scores, n_valid, cfg.S, cfg.k, ws=ws)
    uws = sa.workspace(sa.lib().sa_block_union_prefill_workspace_size(cfg.S, cfg.chunk, cfg.Hq, cfg.Hkv, cfg.d,
                                                                       cfg.k, cfg.block), dev)
    indptr, indices, O = sa.block_union_prefill(idx, wl["q_pos"], wl["Q"], wl["K"], wl["V"], cfg.block, cfg.scale,
                                                out_dtype=torch.float32, ws=uws)
    assert_status_ok(ws)
    assert_status_ok(uws)
    idx_h = idx.cpu().numpy()
    q_pos = cfg.q_pos
    sample = range(cfg.chunk) if q_sample is None else q_sample
    KI = cfg.KI_full()
    qI, w = cfg.qI(), cfg.w()
    scores_h = scores.cpu().numpy() if q_sample is None else scores[torch.tensor(list(sample), device=dev)].cpu().numpy()
    for i, p in enumerate(sample):
        n = int(q_pos[p]) + 1
        ora = oracle.index_score(qI[p:p + 1], w[p:p + 1], KI, [0, cfg.S], [0], [n - 1])[0][:n]
        parity.assert_scores_close(scores_h[i, :n], ora, parity.index_error_bound(qI[p], w[p], KI[:n]), f"p={p}")
        assert np.array_equal(idx_h[p], oracle.topk(scores_h[i:i + 1, :n], [n], cfg.k)[0])
        parity.assert_topk_band(idx_h[p], ora, n, cfg.k, f"p={p}")
    # the union of the GPU's index, exactly
    want_ptr, want_ind = oracle.block_union(idx_h, cfg.S, cfg.block, cfg.Hkv)
    got_ptr = indptr.cpu().numpy()
    assert np.array_equal(got_ptr, want_ptr)
    assert np.array_equal(indices.cpu().numpy()[:got_ptr[-1]], want_ind)
    # paged causal attention over the union, sampled rows of the chosen heads
    heads = range(cfg.Hq) if heads is None else heads
    G = cfg.Hq // cfg.Hkv
    O_h = O.cpu().numpy()
    Qh = cfg.Q()
    for h in heads:
        g = h // G
        Kg = cfg.KV_rows(g, np.arange(cfg.S), "K")[None]
        Vg = cfg.KV_rows(g, np.arange(cfg.S), "V")[None]
        rows = list(sample)
        Qs = Qh[rows][:, h:h + 1]
        ptr1 = np.array([0, want_ptr[1]], np.int32)
        want = oracle.paged_prefill_attn(Qs, q_pos[rows], Kg, Vg, cfg.block, ptr1, want_ind[:want_ptr[1]], cfg.scale)
        err = np.abs(O_h[rows, h] - want[:, 0]).max()
        assert err <= parity.ATOL_F32, f"head {h}: {err}"


@pytest.mark.parametrize("H_I,d_I,Nq,S", [
    (16, 128, 300, 5000),   # blocks of 16 queries, ragged last block
    (4, 64, 100, 3000),     # blocks of 64 queries
    (64, 128, 37, 2500),    # blocks of 4 queries
    (2, 128, 257, 1500),    # blocks of 128 queries
    (12, 64, 50, 2000),     # not a power of two: the one-query-per-row path
])
def test_prefill_indexer_shapes(dev, H_I, d_I, Nq, S):
    """Every query's scores over its causal prefix, against the oracle, for
    the block-of-queries kernel (several block sizes) and the general path."""
    rng = np.random.default_rng(H_I * 1000 + Nq)
    qI = synth.f32_to_bf16_bits((rng.standard_normal((Nq, H_I, d_I)) / 8).astype(np.float32))
    KI = synth.f32_to_bf16_bits((rng.standard_normal((S, d_I)) / 8).astype(np.float32))
    w = rng.uniform(0.1, 1.0, (Nq, H_I)).astype(np.float32)
    q_pos = (S - Nq + np.arange(Nq)).astype(np.int32)
    q_pos[::7] = rng.integers(0, S - Nq, len(q_pos[::7]))  # some queries see a short prefix
    ws = sa.workspace(sa.lib().sa_index_score_prefill_workspace_size(Nq), dev)
    scores = sa.index_score_prefill(bf16_dev(qI, dev), torch.from_numpy(w).to(dev), bf16_dev(KI, dev),
                                    torch.from_numpy(q_pos).to(dev), S - 1, ws=ws)
    assert_status_ok(ws)
    got = scores.cpu().numpy()
    for p in range(Nq):
        n = int(q_pos[p]) + 1
        ora = oracle.index_score(qI[p:p + 1], w[p:p + 1], KI, [0, S], [0], [n - 1])[0][:n]
        parity.assert_scores_close(got[p, :n], ora, parity.index_error_bound(qI[p], w[p], KI[:n]), f"p={p}")


@pytest.mark.parametrize("H_I,d_I,Nq,S,k,rows", [
    (16, 128, 300, 6000, 256, 37),    # tensor-core indexer; blocks of 37 queries, a ragged last block
    (16, 128, 64, 3000, 128, 0),      # one block (the default block size)
    (12, 64, 50, 2000, 64, 16),       # the one-query-per-row indexer path
    (16, 128, 129, 131072, 2048, 64), # the c4 context: two full blocks and a one-query block
])
def test_index_topk_prefill_blocked(dev, H_I, d_I, Nq, S, k, rows):
    """The blocked indexer + top-k selects exactly what the indexer over the
    whole chunk followed by the top-k selects (the same kernels, the same
    scores), and that index holds against the oracle's scores outside the
    tie band."""
    rng = np.random.default_rng(Nq + S)
    qI = synth.f32_to_bf16_bits((rng.standard_normal((Nq, H_I, d_I)) / 8).astype(np.float32))
    KI = synth.f32_to_bf16_bits((rng.standard_normal((S, d_I)) / 8).astype(np.float32))
    w = rng.uniform(0.1, 1.0, (Nq, H_I)).astype(np.float32)
    q_pos = (S - Nq + np.arange(Nq)).astype(np.int32)
    q_pos[::5] = rng.integers(0, S - Nq, len(q_pos[::5]))  # some queries see a short prefix
    q_pos[3] = 10  # a prefix shorter than k
    dq, dw, dK, dp = bf16_dev(qI, dev), torch.from_numpy(w).to(dev), bf16_dev(KI, dev), torch.from_numpy(q_pos).to(dev)
    ws = sa.workspace(sa.index_topk_prefill_workspace_size(Nq, S, S - 1, k, rows), dev)
    idx = sa.index_topk_prefill(dq, dw, dK, dp, S - 1, k, rows_per_block=rows, ws=ws)
    assert_status_ok(ws)
    scores = sa.index_score_prefill(dq, dw, dK, dp, S - 1)
    want = sa.topk(scores, dp + 1, S, k)
    assert torch.equal(idx, want)
    got = idx.cpu().numpy()
    for p in list(range(0, Nq, max(1, Nq // 6))) + [3]:
        n = int(q_pos[p]) + 1
        ora = oracle.index_score(qI[p:p + 1], w[p:p + 1], KI, [0, S], [0], [n - 1])[0][:n]
        parity.assert_topk_band(got[p], ora, n, k, f"p={p}")


def test_prefill_ragged_last_block(dev):
    """A context that is not a whole number of 64-token blocks: the last
    block is partial (its tile load reaches past the head's keys), every
    query of the chunk sees it, and G = 2 query heads per KV head."""
    cfg = synth.PrefillConfig("ragged", S=4000, chunk=160, H_I=16, d_I=128, k=512, block=64, Hq=4, Hkv=2, d=128,
                              seed=78, hot_regions=3, region_len=128)
    prefill_parity(cfg, dev)


def test_prefill_small_full_oracle(dev):
    cfg = synth.PrefillConfig("small", S=4096, chunk=256, H_I=16, d_I=128, k=256, block=64, Hq=8, Hkv=2, d=128,
                              seed=77, hot_regions=4, region_len=128)
    prefill_parity(cfg, dev)


def test_prefill_c4_full_size_sampled(dev):
    cfg = synth.workload("c4")
    prefill_parity(cfg, dev, q_sample=[0, 1, 1000, 2047], heads=[0, 13, 31])


# --------------------------------------------------------------------------
# CLSA indexer layer read as full attention whose weights route the index
def _route_case(dev, B, Hq, Hkv, lens, k, seed, out_dtype=torch.float32):
    rng = np.random.default_rng(seed)
    d = 128
    lens = list(lens)
    seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T = int(seq_off[-1])
    S_max = max(max(lens), 1)
    Q = synth.f32_to_bf16_bits(rng.standard_normal((2, B, Hq, d)).astype(np.float32))
    K = synth.f32_to_bf16_bits(rng.standard_normal(max(T, 1) * Hkv * d).astype(np.float32))
    V = synth.f32_to_bf16_bits(rng.standard_normal(max(T, 1) * Hkv * d).astype(np.float32))
    scale = 1 / math.sqrt(d)
    ws = sa.workspace(sa.decode_step_attn_route_workspace_size(B, S_max, Hq, Hkv, d, k, 2), dev)
    scores = torch.full((B, S_max + 5), float("nan"), dtype=torch.float32, device=dev)
    O, idx = sa.decode_step_attn_route(bf16_dev(Q, dev), bf16_dev(K, dev), bf16_dev(V, dev),
                                       torch.from_numpy(seq_off).to(dev), torch.tensor(lens, dtype=torch.int32, device=dev),
                                       S_max, k, Hkv, scale, out_dtype=out_dtype, scores=scores, ws=ws)
    assert_status_ok(ws)
    O_ora, route = oracle.indexer_layer_attn(Q[0], K, V, seq_off, lens, Hkv, scale)
    sc, idx_h, O_h = scores.cpu().numpy(), idx.cpu().numpy(), O.float().cpu().numpy()
    tol = parity.ATOL_F32 if out_dtype == torch.float32 else parity.ATOL_BF16
    assert np.abs(O_h[0] - O_ora).max() <= tol
    for b in range(B):
        S = lens[b]
        assert np.all(np.isnan(sc[b, S:])), "nothing is written past the sequence"
        if S:
            Kb = K[seq_off[b] * Hkv * d:(seq_off[b] + S) * Hkv * d].reshape(Hkv, S, d)
            rtol = parity.route_rtol(Q[0, b], Kb, scale)
            err = np.abs(sc[b, :S].astype(np.float64) - route[b, :S]) / np.maximum(route[b, :S], 1e-30)
            assert err.max() <= rtol, (b, float(err.max()), rtol)
        assert np.array_equal(idx_h[b], oracle.topk(sc[b:b + 1, :S], [S], k)[0]) if S else np.all(idx_h[b] == -1)
        if S:
            parity.assert_topk_band(idx_h[b], route[b], S, k, f"route b={b}")
    # layer 1 reads the GPU's index: dense-routed sparse attention
    O1 = oracle.sparse_decode_attn(Q[1:], K, V, seq_off, lens, idx_h, Hkv, scale)
    assert np.abs(O_h[1:] - O1).max() <= tol


@pytest.mark.parametrize("B,Hq,Hkv,lens,k", [
    (2, 32, 8, [5000, 2048], 256),          # G = 4, several 2048-key chunks, exact chunk edge
    (3, 16, 2, [77, 4099, 31], 64),          # G = 8, ragged tiles, a sequence shorter than k
    (2, 4, 4, [1000, 0], 128),               # G = 1 and an empty sequence
    (1, 8, 4, [300], 300),                   # G = 2, k = S: every token routed
])
def test_indexer_layer_routing_small(dev, B, Hq, Hkv, lens, k):
    _route_case(dev, B, Hq, Hkv, lens, k, seed=B * 100 + Hq)


def test_indexer_layer_routing_bf16_output(dev):
    _route_case(dev, 2, 32, 8, [3000, 1500], 512, seed=7, out_dtype=torch.bfloat16)


def test_attn_route_step_c3_full_size_sampled(dev):
    """The c3 group (4 x 131072 tokens, 32 / 8 heads, 24 layers) under the
    attention-routing reading: layer 0 dense with its routing scores, top-2048,
    23 sparse layers; sequences 0 and 3 against the oracle."""
    cfg = synth.workload("c3")
    wl = sgpu.decode_workload(cfg, dev, groups=[0])
    gr = wl["groups"][0]
    ws = sa.workspace(sa.decode_step_attn_route_workspace_size(cfg.B, cfg.S_max, cfg.Hq, cfg.Hkv, cfg.d, cfg.k,
                                                               cfg.L), dev)
    O, idx = sa.decode_step_attn_route(wl["Q"], gr["K"], gr["V"], wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k,
                                       cfg.Hkv, cfg.scale, out_dtype=torch.float32, ws=ws)
    assert_status_ok(ws)
    O_h, idx_h = O.cpu().numpy(), idx.cpu().numpy()
    Q = cfg.Q()
    for b in (0, 3):
        S = cfg.seq_lens[b]
        rows = np.arange(S)
        K = np.stack([cfg.KV_rows(0, b, h, rows, "K") for h in range(cfg.Hkv)])
        V = np.stack([cfg.KV_rows(0, b, h, rows, "V") for h in range(cfg.Hkv)])
        O0, route = oracle.indexer_layer_attn(Q[0, b:b + 1], K.ravel(), V.ravel(), [0, S], [S], cfg.Hkv, cfg.scale)
        assert np.abs(O_h[0, b] - O0[0]).max() <= parity.ATOL_F32
        parity.assert_topk_band(idx_h[b], route[0], S, cfg.k, f"c3 route b={b}")
        O_rest = oracle.sparse_decode_attn(Q[1:, b:b + 1], K.ravel(), V.ravel(), [0, S], [S], idx_h[b:b + 1],
                                           cfg.Hkv, cfg.scale)[:, 0]
        assert np.abs(O_h[1:, b] - O_rest).max() <= parity.ATOL_F32


def test_indexer_layer_reports_bad_length(dev):
    """A sequence length above S_max is reported (kernel id 7) and the
    sequence is treated as empty: zero output, nothing routed; the other
    sequence is unaffected."""
    rng = np.random.default_rng(5)
    d, Hq, Hkv, S_max = 128, 8, 2, 300
    lens_real = [300, 200]
    seq_off = np.array([0, 300, 500], np.int64)
    Q = synth.f32_to_bf16_bits(rng.standard_normal((2, Hq, d)).astype(np.float32))
    K = synth.f32_to_bf16_bits(rng.standard_normal(500 * Hkv * d).astype(np.float32))
    V = synth.f32_to_bf16_bits(rng.standard_normal(500 * Hkv * d).astype(np.float32))
    ws = sa.workspace(sa.indexer_layer_attn_workspace_size(2, S_max, Hq, Hkv, d), dev)
    bad = torch.tensor([300, S_max + 5], dtype=torch.int32, device=dev)
    O, sc = sa.indexer_layer_attn(bf16_dev(Q, dev), bf16_dev(K, dev), bf16_dev(V, dev),
                                  torch.from_numpy(seq_off).to(dev), bad, S_max, Hkv, 1 / math.sqrt(d),
                                  out_dtype=torch.float32, ws=ws)
    code, det = sa.read_status(ws)
    assert code == sa.SA_ERR_DEVICE and det[0] == 7 and det[1] == 1 and det[2] == S_max + 5
    O_h = O.cpu().numpy()
    assert np.all(O_h[1] == 0)
    O_ora, _ = oracle.indexer_layer_attn(Q[:1], K[:300 * Hkv * d], V[:300 * Hkv * d], seq_off[:2], lens_real[:1],
                                         Hkv, 1 / math.sqrt(d))
    assert np.abs(O_h[0] - O_ora[0]).max() <= parity.ATOL_F32


def test_binding_rejects_outputs_of_the_wrong_shape(dev):
    """Caller-supplied outputs and sequence tables are checked before any
    launch: a kernel would otherwise write past a smaller tensor."""
    d, B, Hq, Hkv, L, k, S = 128, 2, 8, 2, 2, 64, 300
    Q = torch.zeros((L, B, Hq, d), dtype=torch.bfloat16, device=dev)
    K = torch.zeros((B * S * Hkv * d,), dtype=torch.bfloat16, device=dev)
    seq_off = torch.tensor([0, S, 2 * S], device=dev)
    seq_len = torch.tensor([S, S], dtype=torch.int32, device=dev)
    idx = torch.zeros((B, k), dtype=torch.int32, device=dev)
    with pytest.raises(ValueError, match="O must have shape"):
        sa.sparse_decode_attn(Q, K, K, seq_off, seq_len, idx, Hkv, 0.088,
                              O=torch.empty((L, B, Hq, d - 1), dtype=torch.bfloat16, device=dev))
    with pytest.raises(ValueError, match="seq_off"):
        sa.sparse_decode_attn(Q, K, K, seq_off.to(torch.int32), seq_len, idx, Hkv, 0.088)
    with pytest.raises(ValueError, match="scores must be"):
        sa.indexer_layer_attn(Q[0], K, K, seq_off, seq_len, S, Hkv, 0.088,
                              scores=torch.empty((B, S - 1), dtype=torch.float32, device=dev))
    with pytest.raises(ValueError, match="idx must have shape"):
        sa.topk(torch.zeros((B, S), device=dev), seq_len, S, k, idx=torch.empty((B, k - 1), dtype=torch.int32,
                                                                                 device=dev))


def test_decode_step_plan_matches_decode_step(dev):
    """A DecodeStepPlan (arguments checked and marshalled once) runs the same
    step as decode_step, bit for bit, also after its input buffers are
    refilled in place (c2: three F layers)."""
    cfg = synth.workload("c2")
    wl = sgpu.decode_workload(cfg, dev)
    n = cfg.L
    gi = [max(i for i, g in enumerate(cfg.groups) if g[0] <= l) for l in range(n)]  # each layer's group
    grs = wl["groups"]
    qI = [grs[gi[l]]["qI"] if cfg.pattern[l] == "F" else None for l in range(n)]
    w = [grs[gi[l]]["w"] if cfg.pattern[l] == "F" else None for l in range(n)]
    KI = [grs[gi[l]]["KI"] if cfg.pattern[l] == "F" else None for l in range(n)]
    K = [grs[gi[l]]["K"] for l in range(n)]
    V = [grs[gi[l]]["V"] for l in range(n)]
    O0, idx0 = sa.decode_step(cfg.pattern, qI, w, KI, K, V, wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k, wl["Q"],
                              cfg.Hkv, cfg.scale)
    Q = wl["Q"].clone()
    plan = sa.DecodeStepPlan(cfg.pattern, qI, w, KI, K, V, wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k, Q, cfg.Hkv,
                             cfg.scale)
    O1, idx1 = plan.run()
    torch.cuda.synchronize()
    assert torch.equal(O1, O0) and torch.equal(idx1, idx0)
    Q.copy_(torch.flip(wl["Q"], dims=[1]))  # new queries in the same buffer
    O2, _ = plan.run()
    O3, _ = sa.decode_step(cfg.pattern, qI, w, KI, K, V, wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k, Q, cfg.Hkv,
                           cfg.scale)
    assert torch.equal(O2, O3)
    assert_status_ok(plan.ws)
