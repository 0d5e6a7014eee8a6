#!/usr/bin/env python
"""Decode-step throughput of cross-layer shared sparse attention on B200.

One step = the whole hot path for one batch: the indexer scores every cached
key of every sequence, the top-k picks 2048 tokens per sequence, and every
layer of the group runs sparse attention over them (the index computed once,
shared by all layers reading the one KV cache).  Default workload: decode,
batch 4, 131072-token contexts, indexer 16 heads x 128, top-2048 shared by 24
cross-decoder layers, 32 query / 8 KV heads, d=128, bf16 (seeded synthetic).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs N independent replicas (one per GPU, launched by torchrun): the
path shards by sequence with no data-path collective, so scaling is weak and
`value` is the aggregate over all ranks; the elapsed time is the max over ranks.
`--impl reference` times the CPU oracle (plain C, fp64) on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode steps/s and achieved HBM GB/s (% of roofline) at 128K ctx, 1×B200"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
PROFILE = os.path.join(ROOT, "profiles", "indexer_decode_c3.md")
L2_BYTES = 126 * 1024 * 1024  # B200 L2
INDEXER_SRC = os.path.join(ROOT, "cross_layer_shared_b200", "csrc", "indexer.cu")
CSRC_DIR = os.path.join(ROOT, "cross_layer_shared_b200", "csrc")
STEP_PROFILE = os.path.join(ROOT, "profiles", "step_traffic_c3.md")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="c3", choices=["c1", "c2", "c3", "c4", "c5"],
                   help="c4 times one chunked-prefill chunk instead of a decode step")
    p.add_argument("--sets", type=int, default=0,
                   help="rotating input sets (cold L2 between steps); 0 = two if they fit in device memory, else one")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline sample budget")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--out-f32", action="store_true", help="fp32 attention output instead of bf16")
    p.add_argument("--no-others", action="store_true",
                   help="skip the one-GPU timings of the other workloads (c1, c2, c5 decode; c4 prefill)")
    p.add_argument("--osk-only", action="store_true",
                   help="with --workload c4: time only the ordered-skipping prefill path against the full one")
    p.add_argument("--cp-ranks", type=int, default=8,
                   help="ranks of the emulated context-parallel step (single-group workloads, N=1; 0 = skip)")
    return p.parse_args()


# ---------------------------------------------------------------- ranks
def rank_workload(name: str, rank: int):
    """The workload one rank decodes: the named configuration, its seed offset
    by the rank so that every rank serves sequences of its own (weak scaling:
    the per-GPU work stays fixed as the number of GPUs grows)."""
    cfg = synth.workload(name)
    if rank:
        cfg = dataclasses.replace(cfg, seed=cfg.seed + 7919 * rank)
    return cfg


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's elapsed time (every rank gets it)."""
    if world == 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time."""
    return world * units_per_rank / (ms / 1e3)


# ---------------------------------------------------------------- accounting
def algorithmic_bytes(cfg: synth.DecodeConfig, out_bytes: int = 2) -> dict:
    """Strict HBM bytes one step must move (each selected K/V row once per
    sequence, KV head and cache; every indexer-key row once per F layer)."""
    n_f = len(cfg.groups)
    ki = n_f * cfg.T * cfg.d_I * 2
    sel = sum(min(cfg.k, s) for s in cfg.seq_lens)
    kv = n_f * sel * cfg.Hkv * cfg.d * 2 * 2
    q = cfg.L * cfg.B * cfg.Hq * cfg.d * 2
    o = cfg.L * cfg.B * cfg.Hq * cfg.d * out_bytes
    small = n_f * (cfg.B * cfg.k * 4 + cfg.B * cfg.H_I * cfg.d_I * 2 + cfg.B * cfg.H_I * 4)
    return {"KI": ki, "KV": kv, "Q": q, "O": o, "small": small, "total": ki + kv + q + o + small}


def attn_route_bytes(cfg: synth.DecodeConfig, out_bytes: int = 2) -> dict:
    """Strict HBM bytes of one step under the attention-routing reading
    (layer 0 attends densely; its summed attention weights route the index
    of layers 1..L-1): every K and V row of the cache once, each selected
    row once more for the sparse layers, Q and O of every layer."""
    dense = cfg.T * cfg.Hkv * cfg.d * 2 * 2
    sel = sum(min(cfg.k, s) for s in cfg.seq_lens) * cfg.Hkv * cfg.d * 2 * 2
    q = cfg.L * cfg.B * cfg.Hq * cfg.d * 2
    o = cfg.L * cfg.B * cfg.Hq * cfg.d * out_bytes
    return {"dense_KV": dense, "selected_KV": sel, "Q": q, "O": o, "total": dense + sel + q + o}


def indexer_launch_bytes(cfg: synth.DecodeConfig) -> int:
    """Bytes one indexer launch must move: each visible key row (d_I bf16) read
    once, the query/weights read, one fp32 score per key written."""
    return cfg.T * (cfg.d_I * 2 + 4) + cfg.B * cfg.H_I * (cfg.d_I * 2 + 4)


def measured_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profile_traffic(workload: str):
    """ncu DRAM bytes per indexer launch recorded in profiles/, if the kernel
    source still matches the one profiled and the workload is the one it
    was taken on."""
    try:
        text = open(PROFILE).read()
        if re.search(r"workload:\s*(\w+)", text).group(1) != workload:
            return None
        sha = re.search(r"indexer_source_sha256:\s*([0-9a-f]+)", text).group(1)
        traffic = float(re.search(r"traffic_bytes_per_launch_full:\s*([0-9.eE+]+)", text).group(1))
        cur = hashlib.sha256(open(INDEXER_SRC, "rb").read()).hexdigest()
        return traffic if cur == sha else None
    except Exception:
        return None


def step_traffic(workload: str, launches: int):
    """ncu DRAM bytes (read + write) of one whole step, summed over its
    launches, recorded in profiles/ for this workload while every kernel
    source still matches the one profiled; None otherwise."""
    try:
        text = open(STEP_PROFILE).read()
        if re.search(r"workload:\s*(\w+)", text).group(1) != workload:
            return None
        if int(re.search(r"launches_per_step:\s*(\d+)", text).group(1)) != launches:
            return None
        for name, sha in re.findall(r"source_sha256\[([\w.]+)\]:\s*([0-9a-f]+)", text):
            cur = hashlib.sha256(open(os.path.join(CSRC_DIR, name), "rb").read()).hexdigest()
            if cur != sha:
                return None
        return float(re.search(r"traffic_bytes_per_step:\s*([0-9.eE+]+)", text).group(1))
    except Exception:
        return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """NVML samples of SM clock and throttle reasons while the timed region runs."""

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _sample(self):
        nv = self.nv
        mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        self.samples.append((mhz, reasons))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.ok or not self.samples:
            return None
        nv = self.nv
        names = {
            "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1),
            "applications_clocks_setting": getattr(nv, "nvmlClocksEventReasonApplicationsClocksSetting", 0x2),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sync_boost": getattr(nv, "nvmlClocksEventReasonSyncBoost", 0x10),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        seen = 0
        for _, r in self.samples:
            seen |= r
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for n, bit in names.items() if seen & bit and n != "gpu_idle"),
                "samples": len(self.samples)}


# ---------------------------------------------------------------- CPU oracle
def oracle_sample_inputs(cfg: synth.DecodeConfig, b: int):
    """Host inputs of one sequence of the workload (generation is not timed)."""
    g = 0
    S = cfg.seq_lens[b]
    return {"b": b, "S": S, "qI": cfg.qI(g)[b:b + 1], "w": cfg.w(g)[b:b + 1], "KI": cfg.KI_rows(g, b, np.arange(S)),
            "Q": cfg.Q()[:, b:b + 1], "Kf": lambda h, r: cfg.KV_rows(g, b, h, r, "K"),
            "Vf": lambda h, r: cfg.KV_rows(g, b, h, r, "V")}


def oracle_sequence_step(cfg, inp, kv_cache):
    """The oracle's hot path for one sequence: score, top-k, every layer's attention."""
    import oracle
    S = inp["S"]
    s = oracle.index_score(inp["qI"], inp["w"], inp["KI"], [0, S], [0], [S - 1])
    idx = oracle.topk(s, [S], cfg.k)
    key = idx.tobytes()
    if key not in kv_cache:  # gather the selected rows' bits (input plumbing, untimed below)
        kv_cache.clear()
        kv_cache[key] = (synth.gather_selected_rows(inp["Kf"], idx[0], cfg.Hkv, cfg.d),
                         synth.gather_selected_rows(inp["Vf"], idx[0], cfg.Hkv, cfg.d)[0])
    return idx, kv_cache[key]


def run_oracle_sample(cfg, budget_s: float, min_reps: int = 1):
    """Times oracle steps over whole sequences until `budget_s` of CPU work;
    returns (steps/s equivalent, seconds, sequences timed, threads)."""
    import oracle
    oracle.build()
    inputs = [oracle_sample_inputs(cfg, b) for b in range(cfg.B)]
    cache = {}
    # untimed: one pass to materialise the selected rows of every sequence
    sel = {}
    for inp in inputs:
        idx, ((Kc, remap, m), Vc) = oracle_sequence_step(cfg, inp, cache)
        sel[inp["b"]] = (Kc, Vc, remap, m)
    t_total = 0.0
    n_seq = 0
    reps = 0
    while (t_total < budget_s and reps < 1000) or reps < min_reps:
        for inp in inputs:
            Kc, Vc, remap, m = sel[inp["b"]]
            S = inp["S"]
            t0 = time.perf_counter()
            s = oracle.index_score(inp["qI"], inp["w"], inp["KI"], [0, S], [0], [S - 1])
            oracle.topk(s, [S], cfg.k)
            oracle.sparse_decode_attn(inp["Q"], Kc.ravel(), Vc.ravel(), [0, m], [m], remap[None], cfg.Hkv, cfg.scale)
            t_total += time.perf_counter() - t0
            n_seq += 1
        reps += 1
    steps = n_seq / cfg.B
    return steps / t_total, t_total, n_seq, oracle.num_threads()


# ---------------------------------------------------------------- chunked prefill (c4)
PREFILL_METRIC = ("prefill chunk latency at 128K ctx: 2048 queries, indexer + per-query top-2048 + block union "
                  "+ zero-copy paged causal attention, 1xB200")


def prefill_attention_flops(cfg: synth.PrefillConfig, kv_indptr, kv_indices) -> int:
    """Tensor-core flops of the paged causal attention: for every query p and
    head, QK^T and PV over each key of the union blocks at or before p
    (2 d multiply-adds each way = 4 d flops per (row, key))."""
    blocks = np.asarray(kv_indices[: int(kv_indptr[1])], np.int64)  # every group's table is the same set
    starts = blocks * cfg.block
    ends = np.minimum(starts + cfg.block, cfg.S)
    qp = np.asarray(cfg.q_pos, np.int64)[:, None]
    visible = np.clip(np.minimum(ends[None, :], qp + 1) - starts[None, :], 0, None).sum()
    return int(4 * cfg.d * cfg.Hq * visible)


def prefill_indexer_flops(cfg: synth.PrefillConfig) -> int:
    return int(2 * cfg.H_I * cfg.d_I * (np.asarray(cfg.q_pos, np.int64) + 1).sum())


def prefill_oracle_sample(cfg: synth.PrefillConfig, budget_s: float):
    """The oracle on a bounded sample of the chunk: per sampled query its
    indexer scores over the whole causal prefix, its top-k, and every head's
    paged attention over the union table (the union itself is built once from
    the sampled rows' index, untimed).  Returns (estimated ms per chunk,
    seconds timed, queries timed, threads)."""
    import oracle
    oracle.build()
    KI = cfg.KI_full()
    qI, w, Q = cfg.qI(), cfg.w(), cfg.Q()
    K = np.stack([cfg.KV_rows(h, np.arange(cfg.S), "K") for h in range(cfg.Hkv)])
    V = np.stack([cfg.KV_rows(h, np.arange(cfg.S), "V") for h in range(cfg.Hkv)])
    rng = np.random.default_rng(cfg.seed)
    order = rng.permutation(cfg.chunk)
    t_total, n = 0.0, 0
    for p in order:
        pos = int(cfg.q_pos[p])
        t0 = time.perf_counter()
        s = oracle.index_score(qI[p:p + 1], w[p:p + 1], KI, [0, cfg.S], [0], [pos])[:, : pos + 1]
        idx = oracle.topk(s, [pos + 1], cfg.k)
        ptr, ind = oracle.block_union(idx, cfg.S, cfg.block, cfg.Hkv)
        oracle.paged_prefill_attn(Q[p:p + 1], cfg.q_pos[p:p + 1], K, V, cfg.block, ptr, ind, cfg.scale)
        t_total += time.perf_counter() - t0
        n += 1
        if t_total >= budget_s:
            break
    return 1e3 * t_total / n * cfg.chunk, t_total, n, oracle.num_threads()


def prefill_device_timing(args, dev, cap):
    """One c4 chunk (indexer, per-query top-k, block union + paged attention)
    replayed from CUDA graphs: chunk and per-stage device times, FLOPs and
    the tensors and calls the end-to-end leg reuses."""
    import torch

    import cross_layer_shared_b200 as sa
    from synth import gpu as sgpu

    cfg = synth.workload("c4")
    wl = sgpu.prefill_workload(cfg, dev)
    out_dtype = torch.float32 if args.out_f32 else torch.bfloat16
    ws = sa.workspace(max(sa.lib().sa_index_score_prefill_workspace_size(cfg.chunk),
                          sa.lib().sa_topk_workspace_size(cfg.chunk, cfg.S, cfg.k)), dev)
    uws = sa.workspace(sa.lib().sa_block_union_prefill_workspace_size(cfg.S, cfg.chunk, cfg.Hq, cfg.Hkv, cfg.d,
                                                                        cfg.k, cfg.block), dev)
    scores = torch.empty((cfg.chunk, cfg.S), dtype=torch.float32, device=dev)
    idx = torch.empty((cfg.chunk, cfg.k), dtype=torch.int32, device=dev)
    n_valid = (wl["q_pos"] + 1).to(torch.int32)
    nb = (cfg.S + cfg.block - 1) // cfg.block
    kv_indptr = torch.empty(cfg.Hkv + 1, dtype=torch.int32, device=dev)
    kv_indices = torch.empty(cfg.Hkv * nb, dtype=torch.int32, device=dev)
    O = torch.empty((cfg.chunk, cfg.Hq, cfg.d), dtype=out_dtype, device=dev)

    def run_index(qI=wl["qI"], w=wl["w"]):
        sa.index_score_prefill(qI, w, wl["KI"], wl["q_pos"], cfg.S - 1, scores=scores, ld=cfg.S, ws=ws)

    def run_topk():
        sa.topk(scores, n_valid, cfg.S, cfg.k, idx=idx, ws=ws)

    def run_attn(Q=wl["Q"]):
        sa.block_union_prefill(idx, wl["q_pos"], Q, wl["K"], wl["V"], cfg.block, cfg.scale, O=O,
                               kv_indptr=kv_indptr, kv_indices=kv_indices, ws=uws)

    def chunk():
        run_index(); run_topk(); run_attn()

    chunk()
    torch.cuda.synchronize()
    for w_ in (ws, uws):
        code, det = sa.read_status(w_)
        if code != 0:
            raise RuntimeError(f"device status {code} {det}")
    graphs = {}
    for name, fn in (("chunk", chunk), ("indexer", run_index), ("topk", run_topk), ("attention", run_attn)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            fn()
        graphs[name] = g

    def timed(g, count):
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(count):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / count

    steps = max(1, min(args.steps, 50))
    warm = max(3, min(args.warmup, 10))
    for _ in range(warm):
        graphs["chunk"].replay()
    with ClockSampler(dev.index or 0) as clocks:
        ms = timed(graphs["chunk"], steps)
    stage_ms = {name: timed(graphs[name], steps) for name in ("indexer", "topk", "attention")}
    ptr_h, ind_h = kv_indptr.cpu().numpy(), kv_indices.cpu().numpy()
    attn_flops = prefill_attention_flops(cfg, ptr_h, ind_h)
    idx_flops = prefill_indexer_flops(cfg)
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        peak, peak_kind = float(pk["bf16_tflops"]), "measured (burst cuBLAS bf16)"
    except Exception:
        peak, peak_kind = 1590.0, "fallback"
    attn_tf = attn_flops / (stage_ms["attention"] / 1e3) / 1e12

    return {"cfg": cfg, "wl": wl, "O": O, "idx": idx, "run_index": run_index, "run_topk": run_topk,
            "run_attn": run_attn,
            "ms": ms, "stage_ms": stage_ms, "attn_flops": attn_flops, "idx_flops": idx_flops, "peak": peak,
            "peak_kind": peak_kind, "attn_tf": attn_tf, "clocks": clocks, "union_blocks": int(ptr_h[1]),
            "steps": steps, "warm": warm, "graphs": graphs}


OSK_TAU = 2.0 ** -10


def osk_device_timing(args, dev, cap, idx, tau: float = OSK_TAU, names=("c4-concentrated", "c4")) -> dict:
    """Priority-ordered block execution with early skipping on the c4 chunk's
    own selection (idx from its indexer and top-k): sa_osk_prefill (union,
    priority lists, ordered-skipping attention) against sa_block_union_prefill
    (union, attention over every union block), both replayed from CUDA graphs,
    on the plain chunk and on the chunk whose attention is drawn to the hot
    regions.  Times are taken with bf16 outputs (the chunk's own); the
    share of tiles run and how far the skipped output is from the full one
    come from one untimed call of each with fp32 outputs."""
    import torch

    import cross_layer_shared_b200 as sa
    from synth import gpu as sgpu

    out = {"tau": tau}
    steps = max(1, min(args.steps, 50))
    for name in names:
        cfg = synth.workload(name)
        wl = sgpu.prefill_workload(cfg, dev)
        G = cfg.Hq // cfg.Hkv
        n_qb = (cfg.chunk * G + 127) // 128
        nb = (cfg.S + cfg.block - 1) // cfg.block
        ws = sa.workspace(sa.osk_prefill_workspace_size(cfg.S, cfg.chunk, cfg.Hq, cfg.Hkv, cfg.d, cfg.k, cfg.block),
                          dev)
        uws = sa.workspace(sa.lib().sa_block_union_prefill_workspace_size(cfg.S, cfg.chunk, cfg.Hq, cfg.Hkv, cfg.d,
                                                                            cfg.k, cfg.block), dev)
        kws = sa.workspace(sa.kap_order_workspace_size(), dev)
        ptr = torch.empty(cfg.Hkv + 1, dtype=torch.int32, device=dev)
        ind = torch.empty(cfg.Hkv * nb, dtype=torch.int32, device=dev)
        order = torch.empty((n_qb, nb), dtype=torch.int32, device=dev)
        st = torch.empty(cfg.Hkv * n_qb, dtype=torch.int32, device=dev)
        O_osk = torch.empty((cfg.chunk, cfg.Hq, cfg.d), dtype=torch.float32, device=dev)
        O_full = torch.empty_like(O_osk)
        O_b16 = torch.empty((cfg.chunk, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=dev)

        def run_osk(O=O_b16):
            sa.osk_prefill(idx, wl["q_pos"], wl["Q"], wl["K"], wl["V"], cfg.block, cfg.scale, tau, O=O,
                           kv_indptr=ptr, kv_indices=ind, order=order, steps=st, ws=ws)

        def run_full(O=O_b16):
            sa.block_union_prefill(idx, wl["q_pos"], wl["Q"], wl["K"], wl["V"], cfg.block, cfg.scale, O=O,
                                   kv_indptr=ptr, kv_indices=ind, ws=uws)

        def run_order():
            sa.kap_order(idx, cfg.S, cfg.block, 128 // G, ptr, ind, order=order, ws=kws)

        run_full(O_full)
        run_osk(O_osk)
        torch.cuda.synchronize()
        for w_ in (ws, uws, kws):
            code, det = sa.read_status(w_)
            if code != 0:
                raise RuntimeError(f"device status {code} {det}")
        res = {}
        for key, fn in (("osk", run_osk), ("full", run_full), ("order", run_order)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                fn()
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            res[key] = e0.elapsed_time(e1) / steps
            del g
        n_t = int(ptr[1].item())
        n_steps = (n_t + 1) // 2
        st_h = st.cpu().numpy()
        diff = (O_osk - O_full).abs()
        out[name] = {"osk_ms": res["osk"], "full_ms": res["full"], "order_ms": res["order"],
                     "speedup": res["full"] / res["osk"], "union_blocks": n_t,
                     "tiles_run_frac": float(st_h.sum()) / (len(st_h) * max(1, n_steps)),
                     "tiles_per_unit_min_max": [int(st_h.min()), int(st_h.max())],
                     "max_abs_diff_vs_full": float(diff.max().item()),
                     "mean_abs_diff_vs_full": float(diff.mean().item()),
                     "workload": name + ": " + synth.DESCRIPTIONS.get(name, synth.DESCRIPTIONS["c4"])}
        del wl, O_osk, O_full, O_b16, ws, uws, kws
        torch.cuda.empty_cache()
    return out


def run_prefill(args):
    import torch

    import cross_layer_shared_b200 as sa
    from cross_layer_shared_b200 import build
    from synth import gpu as sgpu

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        print(json.dumps({"workload": "c4", "error": "the prefill chunk runs on one GPU"}), flush=True)
        return 0
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    build.build()
    sa.lib()
    cap = torch.cuda.Stream()
    pt = prefill_device_timing(args, dev, cap)
    cfg, wl, O = pt["cfg"], pt["wl"], pt["O"]
    run_index, run_topk, run_attn = pt["run_index"], pt["run_topk"], pt["run_attn"]
    ms, stage_ms, steps, warm = pt["ms"], pt["stage_ms"], pt["steps"], pt["warm"]
    attn_flops, idx_flops, peak, peak_kind, attn_tf = (pt["attn_flops"], pt["idx_flops"], pt["peak"],
                                                        pt["peak_kind"], pt["attn_tf"])
    clocks = pt["clocks"]

    # end to end through the public API: host Q, qI, w in, host O out
    Q_h, qI_h, w_h = (wl["Q"].cpu().pin_memory(), wl["qI"].cpu().pin_memory(), wl["w"].cpu().pin_memory())
    O_h = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    Qd, qId, wd = torch.empty_like(wl["Q"]), torch.empty_like(wl["qI"]), torch.empty_like(wl["w"])

    def e2e():
        Qd.copy_(Q_h, non_blocking=True); qId.copy_(qI_h, non_blocking=True); wd.copy_(w_h, non_blocking=True)
        run_index(qId, wd); run_topk(); run_attn(Qd)
        O_h.copy_(O, non_blocking=True)

    e2e()
    torch.cuda.synchronize()
    n_e2e = max(3, min(steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        e2e()
    e1.record()
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / n_e2e
    h2d = Q_h.numel() * 2 + qI_h.numel() * 2 + w_h.numel() * 4
    d2h = O_h.numel() * O_h.element_size()

    cpu = None
    if not args.no_cpu_baseline:
        v, secs, nq, threads = prefill_oracle_sample(cfg, args.cpu_seconds)
        cpu = {"value": v, "unit": "ms", "cores": threads, "kind": "oracle",
               "sample": f"{nq} queries of the chunk ({secs:.1f} s of CPU work: indexer over the whole causal prefix, "
                         f"top-{cfg.k}, block union and all {cfg.Hq} heads of paged attention per query), "
                         f"scaled to {cfg.chunk} queries"}
    line = {
        "metric": PREFILL_METRIC, "value": ms, "unit": "ms", "n_gpus": 1, "steps": steps, "warmup": warm,
        "ms_per_step": ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-based generator, random init)",
        "config": {"workload": "c4: " + synth.DESCRIPTIONS["c4"], "queries": cfg.chunk, "context": cfg.S,
                   "top_k": cfg.k, "block": cfg.block, "heads": f"{cfg.Hq}q/{cfg.Hkv}kv", "head_dim": cfg.d,
                   "union_blocks": pt["union_blocks"], "l2": "scores (1.07 GB) and K/V (537 MB) exceed L2",
                   "parallelism": "single"},
        "roofline": {"kernel": "sparse_attn_kernel (paged prefill, with the block-union kernels)", "bound": "tensor",
                     "achieved": attn_tf, "peak": peak, "unit": "TFLOP/s", "frac": attn_tf / peak, "traffic": None,
                     "flops_per_launch": attn_flops, "launch_ms": stage_ms["attention"], "peak_kind": peak_kind},
        "stages_ms": stage_ms,
        "indexer_tflops": idx_flops / (stage_ms["indexer"] / 1e3) / 1e12,
        "cpu_baseline": cpu,
        "e2e": {"value": ms_e2e, "unit": "ms", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 6 * steps,  # per chunk: prefill rows, indexer, top-k rows, union mark, union compact, attention
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_osk_only(args):
    """--workload c4 --osk-only: the chunk's selection (indexer and top-k,
    untimed), then only the ordered-skipping comparison, on the chunk whose
    attention is drawn to its hot regions.  Prints one JSON line."""
    import torch

    import cross_layer_shared_b200 as sa
    from cross_layer_shared_b200 import build
    from synth import gpu as sgpu

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        print(json.dumps({"workload": "c4", "error": "the prefill chunk runs on one GPU"}), flush=True)
        return 0
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    build.build()
    sa.lib()
    cap = torch.cuda.Stream()
    cfg = synth.workload("c4")
    wl = sgpu.prefill_workload(cfg, dev)
    ws = sa.workspace(max(sa.lib().sa_index_score_prefill_workspace_size(cfg.chunk),
                          sa.lib().sa_topk_workspace_size(cfg.chunk, cfg.S, cfg.k)), dev)
    scores = torch.empty((cfg.chunk, cfg.S), dtype=torch.float32, device=dev)
    idx = torch.empty((cfg.chunk, cfg.k), dtype=torch.int32, device=dev)
    sa.index_score_prefill(wl["qI"], wl["w"], wl["KI"], wl["q_pos"], cfg.S - 1, scores=scores, ld=cfg.S, ws=ws)
    sa.topk(scores, (wl["q_pos"] + 1).to(torch.int32), cfg.S, cfg.k, idx=idx, ws=ws)
    torch.cuda.synchronize()
    code, det = sa.read_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} {det}")
    del scores, wl
    torch.cuda.empty_cache()
    res = osk_device_timing(args, dev, cap, idx, names=("c4-concentrated",))
    r = res["c4-concentrated"]
    print(json.dumps({"metric": "ordered-skipping prefill chunk (union + priority lists + attention), 1xB200",
                      "value": r["osk_ms"], "unit": "ms per chunk", "higher_is_better": False,
                      "config": {"workload": r["workload"], "tau": res["tau"]}, "ordered_skipping": res}),
          flush=True)
    return 0


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = synth.workload(args.workload)
    import oracle
    oracle.build()
    per_step = []
    inputs = [oracle_sample_inputs(cfg, b) for b in range(cfg.B)]
    cache = {}
    sel = {}
    for inp in inputs:
        idx, ((Kc, remap, m), Vc) = oracle_sequence_step(cfg, inp, cache)
        sel[inp["b"]] = (Kc, Vc, remap, m)
    # each step: one sequence of the batch (a bounded sample of the step)
    for i in range(args.warmup + args.steps):
        inp = inputs[i % cfg.B]
        Kc, Vc, remap, m = sel[inp["b"]]
        S = inp["S"]
        t0 = time.perf_counter()
        s = oracle.index_score(inp["qI"], inp["w"], inp["KI"], [0, S], [0], [S - 1])
        oracle.topk(s, [S], cfg.k)
        oracle.sparse_decode_attn(inp["Q"], Kc.ravel(), Vc.ravel(), [0, m], [m], remap[None], cfg.Hkv, cfg.scale)
        if i >= args.warmup:
            per_step.append(time.perf_counter() - t0)
    t = sum(per_step)
    value = (len(per_step) / cfg.B) / t
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / (len(per_step) / cfg.B),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, args),
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"each timed step is one of the {cfg.B} sequences of the batch (index score over "
                                   f"all its keys, top-{cfg.k}, attention of all {cfg.L} layers); steps/s = "
                                   f"sequences/{cfg.B}/s; {cores} host cores visible"},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def build_decode_sets(cfg, dev, n_sets: int, out_dtype):
    """n_sets independent device copies of a decode workload, each with the
    per-layer lists a step takes and its own outputs and workspace."""
    import torch

    import cross_layer_shared_b200 as sa
    from synth import gpu as sgpu

    n = cfg.L
    sets = []
    for _ in range(n_sets):
        wl = sgpu.decode_workload(cfg, dev)
        grs = wl["groups"]
        starts = [gr[0] for gr in cfg.groups]
        qI = [grs[starts.index(l)]["qI"] if l in starts else None for l in range(n)]
        w = [grs[starts.index(l)]["w"] if l in starts else None for l in range(n)]
        KI = [grs[starts.index(l)]["KI"] if l in starts else None for l in range(n)]
        gi = [max(i for i, s0 in enumerate(starts) if s0 <= l) for l in range(n)]
        K = [grs[gi[l]]["K"] for l in range(n)]
        V = [grs[gi[l]]["V"] for l in range(n)]
        sets.append({"wl": wl, "qI": qI, "w": w, "KI": KI, "K": K, "V": V,
                     "O": torch.empty((n, cfg.B, cfg.Hq, cfg.d), dtype=out_dtype, device=dev),
                     "idx": torch.empty((cfg.B, cfg.k), dtype=torch.int32, device=dev),
                     "scores": torch.empty((cfg.B, cfg.S_max), dtype=torch.float32, device=dev),
                     "ws": sa.workspace(sa.decode_step_workspace_size(n, cfg.B, cfg.S_max, cfg.Hq, cfg.Hkv, cfg.d,
                                                                      cfg.k), dev)})
    return sets


def decode_step_fn(cfg):
    import cross_layer_shared_b200 as sa

    def step(st, stream=None):
        sa.decode_step(cfg.pattern, st["qI"], st["w"], st["KI"], st["K"], st["V"], st["wl"]["seq_off"],
                       st["wl"]["seq_len"], cfg.S_max, cfg.k, st["wl"]["Q"], cfg.Hkv, cfg.scale, O=st["O"],
                       idx=st["idx"], scores=st["scores"], ws=st["ws"], stream=stream)
    return step


def time_decode_workload(name: str, args, dev, cap, peak: float) -> dict:
    """Device time of whole decode steps of another workload (one GPU):
    CUDA graphs of 8 steps over alternating input sets, after warm-up."""
    import torch

    import cross_layer_shared_b200 as sa

    cfg = synth.workload(name)
    out_dtype = torch.float32 if args.out_f32 else torch.bfloat16
    n_sets = 2 if 2 * set_bytes(cfg) < 0.5 * torch.cuda.mem_get_info()[0] else 1
    sets = build_decode_sets(cfg, dev, n_sets, out_dtype)
    step = decode_step_fn(cfg)
    for st in sets:
        step(st)
    torch.cuda.synchronize()
    for st in sets:
        code, det = sa.read_status(st["ws"])
        if code != 0:
            raise RuntimeError(f"{name}: device status {code} {det}")
    per_graph = 8
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for j in range(per_graph):
            step(sets[j % len(sets)])
    for _ in range(max(1, args.warmup // per_graph)):
        g.replay()
    torch.cuda.synchronize()
    n_rep = max(3, min(200, args.steps // (4 * per_graph)))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_rep):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (n_rep * per_graph)
    nb = algorithmic_bytes(cfg, 4 if args.out_f32 else 2)
    gbs = nb["total"] / (ms / 1e3) / 1e9
    del g
    out = {"value": 1e3 / ms, "unit": "steps/s", "ms_per_step": ms, "hbm_gbs": gbs, "hbm_frac": gbs / peak,
           "algorithmic_bytes_per_step": nb["total"], "steps_timed": n_rep * per_graph, "input_sets": n_sets,
           "workload": name + ": " + synth.DESCRIPTIONS[name]}
    sets.clear()
    torch.cuda.empty_cache()
    return out


def set_bytes(cfg) -> int:
    """Device bytes of one input set: the indexer keys and K/V caches of every group."""
    per_group = cfg.T * (cfg.d_I * 2 + 2 * cfg.Hkv * cfg.d * 2)
    return len(cfg.groups) * per_group


def input_sets(cfg, args) -> int:
    """Rotating input sets: as asked, else two when they fit in 80 % of the
    device's free memory (the full 180 GB when no device is visible), else one."""
    if args.sets > 0:
        return args.sets
    free = 180e9
    try:
        import torch
        if torch.cuda.is_available():
            free, _ = torch.cuda.mem_get_info()
    except Exception:
        pass
    return 2 if 2 * set_bytes(cfg) < 0.8 * free else 1


def workload_config(cfg, args):
    return {"workload": f"{cfg.name}: {synth.DESCRIPTIONS[cfg.name]}", "batch": cfg.B, "context": cfg.S_max,
            "layers": cfg.L, "pattern": cfg.pattern if len(cfg.pattern) <= 8 else f"{cfg.pattern[:4]}... ({cfg.L})",
            "top_k": cfg.k, "indexer": f"{cfg.H_I}x{cfg.d_I}", "heads": f"{cfg.Hq}q/{cfg.Hkv}kv", "head_dim": cfg.d,
            "l2": (f"{input_sets(cfg, args)} rotating input set(s) of {set_bytes(cfg) / 1e9:.1f} GB each, larger than L2"
                   if set_bytes(cfg) > L2_BYTES else
                   f"{input_sets(cfg, args)} input set(s) of {set_bytes(cfg) / 1e6:.1f} MB: resident in L2 "
                   f"(warm-cache figure)"),
            "parallelism": "replicas" if args.gpus > 1 else "single"}


# ---------------------------------------------------------------- our arm
def context_parallel_section(cfg, st, N, cap, dev, reps: int = 16, iters: int = 20) -> dict:
    """Per-rank device time of a context-parallel step of `cfg`'s one layer
    group with N ranks, all emulated on this GPU (phases of every rank run in
    turn; each rank's chain then replayed from a CUDA graph on the gathered
    buffers of that step)."""
    import torch

    import cross_layer_shared_b200 as sa
    from cross_layer_shared_b200 import cp

    lens = [int(x) for x in cfg.seq_lens]
    bnd = cp.shard_bounds(lens, N)
    KI, K, V = st["KI"][0].view(-1, cfg.d_I), st["K"][0], st["V"][0]
    qI, w, Q = st["qI"][0], st["w"][0], st["wl"]["Q"]
    ranks = []
    for r in range(N):
        lo, hi = bnd[r, :, 0], bnd[r, :, 1]
        ranks.append(cp.CPRank(N, r, cp.shard_cache(KI, lens, 1, cfg.d_I, lo, hi),
                               cp.shard_cache(K, lens, cfg.Hkv, cfg.d, lo, hi).view(-1),
                               cp.shard_cache(V, lens, cfg.Hkv, cfg.d, lo, hi).view(-1), hi - lo, cfg.k, cfg.H_I,
                               cfg.d_I, cfg.Hq, cfg.Hkv, cfg.d, cfg.L, cfg.scale))
    O_cp, local = cp.emulate_step(ranks, qI, w, Q)
    # the one-device step on the same inputs, for the record
    scores = sa.index_score(qI, w, KI, st["wl"]["seq_off"], st["wl"]["seq_len"], cfg.S_max)
    idx = sa.topk(scores, st["wl"]["seq_len"], cfg.S_max, cfg.k)
    O1 = sa.sparse_decode_attn(Q, K, V, st["wl"]["seq_off"], st["wl"]["seq_len"], idx, cfg.Hkv, cfg.scale)
    same_idx = True
    idx_h = idx.cpu().numpy()
    for b in range(len(lens)):
        got = sorted(int(bnd[r, b, 0] + t) for r in range(N) for t in local[r][b].cpu().numpy() if t >= 0)
        same_idx &= got == [int(t) for t in idx_h[b] if t >= 0]
    max_abs = (O_cp.float() - O1.float()).abs().max().item()
    for r in ranks:
        for ws in (r.ws_index, r.ws_radix, r.ws_attn):
            code, det = sa.read_status(ws)
            if code != 0:
                raise RuntimeError(f"context-parallel device status {code} {det}")
    # every rank's histograms of each exchange level, and its partials, as
    # the all-gathers of that step delivered them
    for r in ranks:
        r.scores_local(qI, w)
    gathered = [torch.stack([r.radix_level(0) for r in ranks])]
    gathered.append(torch.stack([r.radix_level(1, gathered[0]) for r in ranks]))
    gathered.append(torch.stack([r.radix_level(2, gathered[1]) for r in ranks]))
    for r in ranks:
        r.radix_select(gathered[2])
    parts = torch.stack([r.part for r in ranks])
    O = torch.empty_like(O1)

    def graph_ms(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (iters * reps)

    def select(r):
        r.radix_level(0)
        r.radix_level(1, gathered[0])
        r.radix_level(2, gathered[1])
        r.radix_select(gathered[2])

    def chain(r):
        r.scores_local(qI, w)
        select(r)
        r.partial(Q)
        r.combine(parts, O)

    per_rank = [graph_ms(lambda r=r: chain(r)) for r in ranks]
    slow = ranks[max(range(N), key=lambda i: per_rank[i])]
    phases = {"scores": graph_ms(lambda: slow.scores_local(qI, w)), "select": graph_ms(lambda: select(slow)),
              "partial_attention": graph_ms(lambda: slow.partial(Q)),
              "combine": graph_ms(lambda: slow.combine(parts, O))}
    hist_b = sum(h.numel() * 4 for h in ranks[0].hist)
    part_b = ranks[0].part.numel() * 4
    return {"ranks": N, "context_per_rank": [int(x) for x in (bnd[:, :, 1] - bnd[:, :, 0]).max(1)],
            "ms_per_rank_step_max": max(per_rank), "ms_per_rank_step": per_rank, "phases_ms_slowest_rank": phases,
            "selected_per_rank": [int((x >= 0).sum().item()) for x in local],
            "allgather_bytes_per_rank": {"histograms": hist_b, "partials": part_b},
            "allgather_bytes_received_per_rank": (N - 1) * (hist_b + part_b),
            "launches_per_rank_step": 7, "collectives_per_rank_step": 4, "same_index_as_one_device": bool(same_idx),
            "max_abs_vs_one_device": max_abs,
            "note": "every rank emulated on one GPU; the four all-gathers (three histogram levels, the partials) "
                    "are not timed (one GPU): add their NVLink time for the received bytes; one group of all "
                    "layers shares the index"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import cross_layer_shared_b200 as sa
    from cross_layer_shared_b200 import build
    from synth import gpu as sgpu

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    sa.lib()

    cfg = rank_workload(args.workload, rank)
    out_dtype = torch.float32 if args.out_f32 else torch.bfloat16
    n = cfg.L
    nb = algorithmic_bytes(cfg, 4 if args.out_f32 else 2)

    args.sets = input_sets(cfg, args)
    sets = build_decode_sets(cfg, dev, args.sets, out_dtype)
    step = decode_step_fn(cfg)

    # eager run first (sets kernel attributes, checks status), then capture
    for st in sets:
        step(st)
    torch.cuda.synchronize()
    for st in sets:
        code, det = sa.read_status(st["ws"])
        if code != 0:
            raise RuntimeError(f"device status {code} {det}")

    # the timed loop replays graphs of STEPS_PER_GRAPH whole steps (input sets
    # alternating, so every step reads inputs another step evicted from L2);
    # single-step graphs cover a remainder
    STEPS_PER_GRAPH = 8
    cap = torch.cuda.Stream()
    multi = torch.cuda.CUDAGraph()
    with torch.cuda.graph(multi, stream=cap):
        for j in range(STEPS_PER_GRAPH):
            step(sets[j % len(sets)])
    graphs = []
    for st in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            step(st)
        graphs.append(g)

    def run_steps(count):
        for _ in range(count // STEPS_PER_GRAPH):
            multi.replay()
        for i in range(count % STEPS_PER_GRAPH):
            graphs[i % len(graphs)].replay()

    # kernels of ours inside one step: per F layer the indexer and the top-k,
    # per fused group one attention launch
    launches_per_step = 0
    l = 0
    while l < n:
        if cfg.pattern[l] == "F":
            launches_per_step += 2
        m = l
        while m + 1 < n and cfg.pattern[m + 1] == "S" and sets[0]["K"][m + 1] is sets[0]["K"][l]:
            m += 1
        launches_per_step += 1
        l = m + 1

    run_steps(args.warmup)
    torch.cuda.synchronize()

    def timed(fn, count):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(count):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        if world > 1:
            dist.barrier()
        return ms

    with ClockSampler(local) as clocks:
        ms = timed(lambda i: run_steps(args.steps), 1)
    ms_per_step = ms / args.steps
    value = aggregate_rate(args.steps, world, ms)

    # ---- the same step as a real decoder runs it: the new token appended to
    # the caches first, then one attention launch per layer ----
    gen = torch.Generator(device="cpu").manual_seed(cfg.seed)
    rows = {"KI": (torch.randn((cfg.B, cfg.d_I), generator=gen) / 8).to(torch.bfloat16).to(dev),
            "K": torch.randn((cfg.B, cfg.Hkv, cfg.d), generator=gen).to(torch.bfloat16).to(dev),
            "V": torch.randn((cfg.B, cfg.Hkv, cfg.d), generator=gen).to(torch.bfloat16).to(dev)}

    def step_seq(st):
        new_KI = [rows["KI"] if t is not None else None for t in st["qI"]]
        new_K = [rows["K"] if t is not None else None for t in st["qI"]]
        new_V = [rows["V"] if t is not None else None for t in st["qI"]]
        sa.decode_step(cfg.pattern, st["qI"], st["w"], st["KI"], st["K"], st["V"], st["wl"]["seq_off"],
                       st["wl"]["seq_len"], cfg.S_max, cfg.k, st["wl"]["Q"], cfg.Hkv, cfg.scale, O=st["O"],
                       idx=st["idx"], scores=st["scores"], ws=st["ws"], new_KI=new_KI, new_K=new_K, new_V=new_V,
                       per_layer=True)

    for st in sets:
        step_seq(st)
    torch.cuda.synchronize()
    g_seq = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_seq, stream=cap):
        for j in range(STEPS_PER_GRAPH):
            step_seq(sets[j % len(sets)])
    g_seq.replay()
    n_seq = max(2, min(250, args.steps // STEPS_PER_GRAPH))
    ms_seq = timed(lambda i: g_seq.replay(), n_seq) / (n_seq * STEPS_PER_GRAPH)
    seq_launches = 0
    for l in range(cfg.L):
        seq_launches += (2 if cfg.pattern[l] == "F" else 0) + 1

    # ---- the attention-routing reading of the indexer layer (one group only):
    # layer 0 attends densely and its summed attention weights are the
    # routing scores; their top-k serves layers 1..L-1 ----
    route = None
    if len(cfg.groups) == 1 and cfg.L > 1:
        rws = [sa.workspace(sa.decode_step_attn_route_workspace_size(cfg.B, cfg.S_max, cfg.Hq, cfg.Hkv, cfg.d, cfg.k,
                                                                     cfg.L), dev) for _ in sets]

        def step_route(j):
            st = sets[j % len(sets)]
            sa.decode_step_attn_route(st["wl"]["Q"], st["K"][0], st["V"][0], st["wl"]["seq_off"], st["wl"]["seq_len"],
                                      cfg.S_max, cfg.k, cfg.Hkv, cfg.scale, O=st["O"], idx=st["idx"],
                                      scores=st["scores"], ws=rws[j % len(sets)])

        for j in range(len(sets)):
            step_route(j)
        torch.cuda.synchronize()
        for w in rws:
            code, det = sa.read_status(w)
            if code != 0:
                raise RuntimeError(f"device status {code} {det}")
        g_route = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_route, stream=cap):
            for j in range(STEPS_PER_GRAPH):
                step_route(j)
        g_route.replay()
        n_route = max(3, min(50, args.steps // (4 * STEPS_PER_GRAPH)))
        ms_route = timed(lambda i: g_route.replay(), n_route) / (n_route * STEPS_PER_GRAPH)
        rb = attn_route_bytes(cfg, 4 if args.out_f32 else 2)
        route = {"value": aggregate_rate(1, world, ms_route), "unit": "steps/s", "ms_per_step": ms_route,
                 "hbm_gbs": rb["total"] / (ms_route / 1e3) / 1e9 * world, "algorithmic_bytes_per_step": rb,
                 "launches_per_step": 4,
                 "note": "CLSA read as routing from the indexer layer's own attention weights: layer 0 attends "
                         "densely over every cached token, the sum over its query heads of each token's weight "
                         "is the routing score, its top-k is the index of layers 1..L-1"}
        del g_route

    # ---- context-parallel decode, every rank emulated on this GPU: each
    # sequence's context sharded over cp_ranks ranks; a rank's step is its
    # indexer over its slice, the global selection by three histogram
    # levels, attention over its share, and the merge of all partials.
    # The four all-gathers between the phases are not run (one GPU): their
    # bytes per rank are reported instead ----
    cpar = None
    if world == 1 and len(cfg.groups) == 1 and args.cp_ranks > 1:
        cpar = context_parallel_section(cfg, sets[0], args.cp_ranks, cap, dev)

    # ---- per-kernel device time: each graph holds REP back-to-back launches
    # (alternating input sets, so consecutive launches read different data),
    # which keeps the host's replay cost out of the figure ----
    REP = 16

    def rep_graph(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for r in range(REP):
                fn(sets[r % len(sets)])
        return g

    l0 = cfg.groups[0]

    def run_index(st):
        sa.index_score(st["qI"][0], st["w"][0], st["KI"][0], st["wl"]["seq_off"], st["wl"]["seq_len"], cfg.S_max,
                       scores=st["scores"], ws=st["ws"])

    def run_topk(st):
        sa.topk(st["scores"], st["wl"]["seq_len"], cfg.S_max, cfg.k, idx=st["idx"], ws=st["ws"])

    def run_attn(st):
        sa.sparse_decode_attn(st["wl"]["Q"][l0[0]:l0[-1] + 1], st["K"][0], st["V"][0], st["wl"]["seq_off"],
                              st["wl"]["seq_len"], st["idx"], cfg.Hkv, cfg.scale, O=st["O"][l0[0]:l0[-1] + 1],
                              ws=st["ws"])

    g_idx, g_topk, g_attn = rep_graph(run_index), rep_graph(run_topk), rep_graph(run_attn)
    for g in (g_idx, g_topk, g_attn):
        g.replay()
    n_rep = max(20, min(250, args.steps // REP))
    ms_idx = timed(lambda i: g_idx.replay(), n_rep) / (n_rep * REP)
    ms_topk = timed(lambda i: g_topk.replay(), n_rep) / (n_rep * REP)
    ms_attn = timed(lambda i: g_attn.replay(), n_rep) / (n_rep * REP)

    # ---- end to end through the public API: pinned host in, host out ---------
    # Every step copies its inputs in from pinned host memory (the queries of
    # every layer and the indexer queries and head weights of every F layer,
    # packed in one buffer: one copy), runs through a DecodeStepPlan (the
    # call prepared once for these buffers), and copies its outputs back out.
    # Copies run on their own streams with two device buffer sets, so step
    # i+1's inputs travel while step i computes; the steps themselves stay in
    # order on one stream.
    nbuf = len(sets)
    e2e = []
    for st in sets:
        parts = [st["wl"]["Q"]] + [t for t in st["qI"] if t is not None] + [t for t in st["w"] if t is not None]
        offs, total = [], 0
        for t in parts:
            offs.append(total)
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        dbuf = torch.empty(total, dtype=torch.uint8, device=dev)
        views = [dbuf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(parts, offs)]
        for v, t in zip(views, parts):
            v.copy_(t)
        rest = iter(views[1:])
        qIv = [next(rest) if t is not None else None for t in st["qI"]]
        wv = [next(rest) if t is not None else None for t in st["w"]]
        plan = sa.DecodeStepPlan(cfg.pattern, qIv, wv, st["KI"], st["K"], st["V"], st["wl"]["seq_off"],
                                 st["wl"]["seq_len"], cfg.S_max, cfg.k, views[0], cfg.Hkv, cfg.scale, O=st["O"],
                                 idx=st["idx"], scores=st["scores"], ws=st["ws"])
        e2e.append({"dbuf": dbuf, "hbuf": dbuf.cpu().pin_memory(), "plan": plan, "O": st["O"],
                    "O_host": torch.empty(st["O"].shape, dtype=st["O"].dtype).pin_memory()})
    h2d = e2e[0]["hbuf"].numel()
    d2h = e2e[0]["O_host"].numel() * e2e[0]["O_host"].element_size()
    cs, hs, ds = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    h2d_ev = [torch.cuda.Event() for _ in range(nbuf)]
    comp_ev = [torch.cuda.Event() for _ in range(nbuf)]
    d2h_ev = [torch.cuda.Event() for _ in range(nbuf)]

    def e2e_h2d(i):
        b = i % nbuf
        e = e2e[b]
        if i >= nbuf:
            hs.wait_event(comp_ev[b])  # the step that last read this buffer set is done
        with torch.cuda.stream(hs):
            e["dbuf"].copy_(e["hbuf"], non_blocking=True)
        h2d_ev[b].record(hs)

    def e2e_step_out(i):
        b = i % nbuf
        e = e2e[b]
        cs.wait_event(h2d_ev[b])
        if i >= nbuf:
            cs.wait_event(d2h_ev[b])  # O of this buffer set has been copied out
        e["plan"].run(cs)
        comp_ev[b].record(cs)
        ds.wait_event(comp_ev[b])
        with torch.cuda.stream(ds):
            e["O_host"].copy_(e["O"], non_blocking=True)
        d2h_ev[b].record(ds)

    def e2e_run(n):
        e2e_h2d(0)
        for i in range(n):
            if i + 1 < n:
                e2e_h2d(i + 1)
            e2e_step_out(i)

    e2e_run(4)
    torch.cuda.synchronize()
    n_e2e = max(50, min(2000, args.steps))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(hs)
    cs.wait_event(e0)
    ds.wait_event(e0)
    e2e_run(n_e2e)
    e1.record(ds)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = aggregate_rate(n_e2e, world, ms_e2e)
    for st in sets:
        code, det = sa.read_status(st["ws"])
        if code != 0:
            raise RuntimeError(f"device status {code} {det}")

    # ---- CPU baseline: the oracle on this host (rank 0, N = 1 only) ----------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, secs, nseq, threads = run_oracle_sample(cfg, args.cpu_seconds)
        cpu = {"value": v, "unit": "steps/s", "cores": threads, "kind": "oracle",
               "sample": f"{nseq} whole sequences of this workload ({secs:.1f} s of CPU work: index score over every "
                         f"key, top-{cfg.k}, attention of all {cfg.L} layers); steps/s = sequences/{cfg.B}/s"}

    peak, peak_kind = measured_peaks()
    # ---- the other workloads on this GPU (N = 1): each decode workload's
    # whole step and the c4 prefill chunk, device-timed from CUDA graphs ----
    others = None
    if world == 1 and not args.no_others:
        e2e.clear()
        graphs.clear()
        sets.clear()
        del multi, g_idx, g_topk, g_attn, g_seq
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        others = {}
        for name in ("c1", "c2", "c5"):
            if name != cfg.name:
                others[name] = time_decode_workload(name, args, dev, cap, peak)
        pt = prefill_device_timing(args, dev, cap)
        others["c4"] = {"value": pt["ms"], "unit": "ms per chunk", "stage_ms": pt["stage_ms"],
                        "attention_tflops": pt["attn_tf"], "attention_frac": pt["attn_tf"] / pt["peak"],
                        "indexer_tflops": pt["idx_flops"] / (pt["stage_ms"]["indexer"] / 1e3) / 1e12,
                        "peak_tflops": pt["peak"], "peak_kind": pt["peak_kind"],
                        "workload": "c4: " + synth.DESCRIPTIONS["c4"]}
        others["c4_ordered_skipping"] = osk_device_timing(args, dev, cap, pt["idx"])
        del pt
        torch.cuda.empty_cache()

    if world > 1:
        graphs.clear()
        del multi, g_idx, g_topk, g_attn, g_seq
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    if route is not None:
        route["hbm_frac"] = route["hbm_gbs"] / world / peak
    step_gbs = nb["total"] / (ms_per_step / 1e3) / 1e9
    idx_bytes = indexer_launch_bytes(cfg)
    idx_gbs = idx_bytes / (ms_idx / 1e3) / 1e9
    traffic = profile_traffic(cfg.name)
    cs = clocks.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based generator, random init)",
        "config": workload_config(cfg, args),
        "hbm_gbs": step_gbs * world, "hbm_frac": step_gbs / peak, "hbm_peak_gbs": peak, "hbm_peak_kind": peak_kind,
        "algorithmic_bytes_per_step": nb,
        # the metric's own roofline: one whole step (indexer, top-k and the
        # group's attention, replayed from CUDA graphs) against the measured
        # copy peak; the dominant HBM kernel's own figure sits beside it
        "roofline": {"kernel": "decode step (indexer + top-k + one attention launch per fused group)",
                     "bound": "hbm", "achieved": step_gbs, "peak": peak, "unit": "GB/s", "frac": step_gbs / peak,
                     "traffic": step_traffic(cfg.name, launches_per_step),
                     "algorithmic_bytes_per_launch": nb["total"], "launch_ms": ms_per_step,
                     "peak_kind": f"{peak_kind} (burst copy)",
                     "indexer": {"kernel": "indexer_decode_kernel", "bound": "hbm", "achieved": idx_gbs,
                                 "peak": peak, "unit": "GB/s", "frac": idx_gbs / peak, "traffic": traffic,
                                 "algorithmic_bytes_per_launch": idx_bytes, "launch_ms": ms_idx}},
        "kernels_ms": {"indexer": ms_idx, "topk": ms_topk, "attention_group": ms_attn},
        "per_layer_with_append": {"value": aggregate_rate(1, world, ms_seq), "unit": "steps/s", "ms_per_step": ms_seq,
                                  "launches_per_step": seq_launches,
                                  "note": "the new token's rows appended to the caches by the indexer, then one "
                                          "attention launch per layer (no fusion of the group's layers), as a "
                                          "decoder that computes layer l+1's queries from layer l runs it"},
        "attn_route": route,
        "context_parallel": cpar,
        "other_workloads": others,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "per step: one pinned host -> device copy of that step's queries, indexer queries and "
                        "head weights (packed); the step through the public API (a DecodeStepPlan prepared once "
                        "for these buffers); device -> pinned host copy of the outputs; copies on their own "
                        "streams with two buffer sets (step i+1's inputs travel while step i computes; steps run "
                        "in order on one stream); the KV and indexer-key caches stay resident"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": cs,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.workload == "c4":
        if args.impl == "reference":
            if int(os.environ.get("RANK", "0")) != 0:
                return 0
            v, secs, nq, threads = prefill_oracle_sample(synth.workload("c4"), args.cpu_seconds)
            print(json.dumps({"impl": "reference", "metric": PREFILL_METRIC, "value": v, "unit": "ms",
                              "n_gpus": args.gpus, "steps": nq, "warmup": 0, "ms_per_step": v,
                              "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                              "data": "synthetic", "config": {"workload": "c4: " + synth.DESCRIPTIONS["c4"]},
                              "cpu_baseline": {"value": v, "unit": "ms", "cores": threads, "kind": "oracle",
                                               "sample": f"{nq} queries, scaled to the chunk"},
                              "e2e": {"value": v, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
                  flush=True)
            return 0
        if args.osk_only:
            return run_osk_only(args)
        return run_prefill(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
