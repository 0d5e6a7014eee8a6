"""Host logic of bench.py for N > 1 ranks, run as a world-size-2 gloo group on
CPU: every rank gets its own sequences, the elapsed time is the slowest
rank's, and the aggregate rate counts every rank's units over that time."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "took" 10 + 5r ms: everyone must see the slowest, 15 ms
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        cfg = bench.rank_workload("c3", rank)
        results[rank] = (ms, cfg.seed, bench.aggregate_rate(300, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_workload_split():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, free_port(), results), nprocs=world, start_method="spawn", join=True)
    (ms0, seed0, v0), (ms1, seed1, v1) = results[0], results[1]
    assert ms0 == ms1 == 15.0
    assert seed0 == synth.workload("c3").seed and seed1 != seed0
    assert v0 == v1 == pytest.approx(2 * 300 / 0.015)


def test_single_rank_is_unchanged():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.rank_workload("c3", 0) == synth.workload("c3")
    assert bench.aggregate_rate(10, 1, 1000.0) == pytest.approx(10.0)


def test_rank_workloads_differ_only_in_seed():
    a, b = bench.rank_workload("c5", 0), bench.rank_workload("c5", 3)
    assert a.seed != b.seed
    assert (a.seq_lens, a.k, a.pattern, a.Hq, a.Hkv, a.d) == (b.seq_lens, b.k, b.pattern, b.Hq, b.Hkv, b.d)


def test_byte_counts_and_profile_lookup():
    cfg = synth.workload("c3")
    rb = bench.attn_route_bytes(cfg)
    # the routing step reads every K and V row once (4 x 131072 tokens x 8 heads x 256 B x 2)
    assert rb["dense_KV"] == 4 * 131072 * 8 * 256 * 2
    assert rb["selected_KV"] == 4 * 2048 * 8 * 256 * 2
    assert rb["total"] == sum(v for k, v in rb.items() if k != "total")
    nb = bench.algorithmic_bytes(cfg)
    assert nb["KI"] == 4 * 131072 * 256 and nb["KV"] == rb["selected_KV"]
    # one input set: the indexer keys and both caches of each group
    assert bench.set_bytes(cfg) == 4 * 131072 * (256 + 2 * 8 * 256)
    assert bench.set_bytes(synth.workload("c1")) < bench.L2_BYTES < bench.set_bytes(cfg)
    # ncu traffic is reported only for the workload it was captured on
    assert bench.profile_traffic("c1") is None


def test_prefill_flop_counts_match_a_brute_force_count():
    """The prefill roofline's flops: 4 d flops per (query, head, visible key
    of the union blocks); the indexer's 2 H_I d_I per (query, key <= its
    position).  Checked on a small chunk by counting pairs one by one."""
    import numpy as np
    cfg = synth.PrefillConfig("t", 300, 7, 2, 8, 5, 64, 4, 2, 16, seed=5)
    ind = np.array([0, 2, 4], np.int32)     # blocks 0, 2 and the partial last block 4 (256..299)
    ptr = np.array([0, 3, 6], np.int32)
    visible = sum(1 for p in cfg.q_pos for b in ind for t in range(b * 64, b * 64 + 64) if t < cfg.S and t <= p)
    assert bench.prefill_attention_flops(cfg, ptr, np.concatenate([ind, ind])) == 4 * cfg.d * cfg.Hq * visible
    pairs = sum(int(p) + 1 for p in cfg.q_pos)
    assert bench.prefill_indexer_flops(cfg) == 2 * cfg.H_I * cfg.d_I * pairs
