"""Context-parallel decode: every sequence's context sharded over N ranks.

The pages leave contexts past one GPU open (CLSA news article, section "Ce
que cela signifie pour l'inference sur longs contextes").  This is the
plainest sharding that gives the one-GPU result: rank r keeps the contiguous
slice [lo_r(b), hi_r(b)) of every sequence b in its own packed caches, and a
decode step over one layer group (one index shared by the group's layers)
takes four all-gathers:

1. indexer scores over the local slice;
2. the global top-k by a radix select whose histograms are summed over the
   ranks: three levels (key bits [31:20], [19:8], [7:0]), each this rank's
   histogram of the level's digit (sa_cp_radix_level) all-gathered, the
   next level finding the previous threshold from the gathered histograms;
   sa_cp_radix_select then keeps this rank's share as local indices;
3. sparse attention over the local selected rows, left unnormalised (o, m, l);
4. all-gather of the partials; sa_combine_partials (log-sum-exp merge).

A histogram exchange carries 16 KB per sequence and level (1 KB at the last
level) whatever k is; sa_cp_select (still exported) is the earlier design:
every rank's top-k candidates gathered and selected again.

Every rank ends with the whole output.  The arithmetic runs in libsa's
kernels; this module holds the slicing, the buffer layout and the order of
the exchanges.  `exchange` is any all-gather: `nccl_exchange()` over
torch.distributed, or the single-device emulation in `emulate_step`.

One process per GPU (e.g. under torchrun), each holding its slices:

    dist.init_process_group("nccl", device_id=dev)
    lo, hi = shard_bounds(seq_lens, N)[rank].T
    me = CPRank(N, rank, KI_slice, K_slice, V_slice, hi - lo, k, H_I, d_I, Hq, Hkv, d, L_g, scale)
    O = step(me, nccl_exchange(N), qI, w, Q)      # the same O on every rank

Every rank makes the same four collectives in the same order each step.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist

from . import (RADIX_BINS, combine_partials, cp_radix_level, cp_radix_select, cp_radix_workspace_size, index_score,
               sparse_decode_attn_partial, sparse_decode_attn_workspace_size, workspace)
from . import lib


def shard_bounds(seq_len: Sequence[int], N: int) -> np.ndarray:
    """[N, B, 2] (lo, hi) of each rank's slice: lo_r = floor(r*S/N)."""
    S = np.asarray(seq_len, dtype=np.int64)
    r = np.arange(N + 1, dtype=np.int64)[:, None]
    edges = r * S[None, :] // N
    return np.stack([edges[:-1], edges[1:]], axis=-1)


def shard_cache(cache: torch.Tensor, seq_len: Sequence[int], groups: int, dim: int, lo: Sequence[int],
                hi: Sequence[int]) -> torch.Tensor:
    """The slice [lo_b, hi_b) of every sequence of a packed cache.

    The cache holds sequence b at row sum(seq_len[:b])*groups, laid out
    [groups, seq_len[b], dim] (the K/V caches with groups = Hkv, the indexer
    keys with groups = 1); the slice has the same layout over hi_b - lo_b
    tokens, as [rows, dim].  A one-time re-layout (a gather of rows on the
    cache's device), not part of a step."""
    rows: List[np.ndarray] = []
    base = 0
    for b, S in enumerate(seq_len):
        for g in range(groups):
            rows.append(base + g * S + np.arange(lo[b], hi[b], dtype=np.int64))
        base += S * groups
    ridx = torch.from_numpy(np.concatenate(rows) if rows else np.zeros(0, np.int64)).to(cache.device)
    return cache.reshape(-1, dim).index_select(0, ridx)


def seq_tables(lengths: Sequence[int], device) -> Tuple[torch.Tensor, torch.Tensor]:
    """seq_off int64 [B+1] and seq_len int32 [B] on `device`."""
    L = np.asarray(lengths, dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(L)]).astype(np.int64)
    return torch.from_numpy(off).to(device), torch.from_numpy(L.astype(np.int32)).to(device)


def part_floats(rows: int, d: int) -> int:
    """Floats of one rank's packed partial block: O_part [rows, d] then (m, l)
    [rows, 2], padded to 16 bytes so every rank's block stays aligned."""
    return (rows * (d + 2) + 3) // 4 * 4


def part_views(buf: torch.Tensor, rows: int, d: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """(O_part [..., rows, d], ml [..., rows, 2]) views of packed partial blocks
    buf [..., part_floats(rows, d)]."""
    lead = tuple(buf.shape[:-1])
    return (buf[..., : rows * d].view(lead + (rows, d)), buf[..., rows * d: rows * (d + 2)].view(lead + (rows, 2)))


def cand_views(buf: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """(scores fp32, idx int32) views of packed candidate blocks buf int32
    [..., 2, B, k] (sa_cp_select's input): the scores are bit-cast in
    [..., 0, :, :]."""
    return buf[..., 0, :, :].view(torch.float32), buf[..., 1, :, :]


class CPRank:
    """One rank's state: its slices of the caches, their tables, buffers and
    workspaces, for one layer group of L_g layers sharing one index."""

    def __init__(self, N: int, rank: int, KI: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                 local_len: Sequence[int], k: int, H_I: int, d_I: int, Hq: int, Hkv: int, d: int, L_g: int,
                 scale: float):
        if not 0 <= rank < N:
            raise ValueError(f"rank {rank} outside [0, {N})")
        if sum(int(x) for x in local_len) == 0:
            # the attention's tensor maps need at least one cached row
            raise ValueError(f"rank {rank} holds no token of any sequence: use at most as many ranks as the "
                             "longest sequence has tokens")
        self.N, self.rank, self.k = N, rank, k
        self.KI, self.K, self.V = KI, K, V
        self.B = len(local_len)
        self.H_I, self.d_I, self.Hq, self.Hkv, self.d, self.L_g = H_I, d_I, Hq, Hkv, d, L_g
        self.scale = float(scale)
        dev = K.device
        self.S_max = int(max(local_len)) if self.B else 0
        self.seq_off, self.seq_len = seq_tables(local_len, dev)
        B = self.B
        self.scores = torch.empty((B, max(self.S_max, 1)), dtype=torch.float32, device=dev)
        # this rank's histogram of each exchange level, all-gathered as is
        self.hist = [torch.empty((B, bins), dtype=torch.int32, device=dev) for bins in RADIX_BINS]
        self.rows = L_g * B * Hq
        self.part_floats = part_floats(self.rows, d)
        self.part = torch.empty(self.part_floats, dtype=torch.float32, device=dev)
        self.local_idx = torch.empty((B, k), dtype=torch.int32, device=dev)
        self.local_count = torch.empty(B, dtype=torch.int32, device=dev)
        self.ws_index = workspace(int(lib().sa_index_score_workspace_size(B)), dev)
        self.ws_radix = workspace(cp_radix_workspace_size(B), dev)
        self.ws_attn = workspace(sparse_decode_attn_workspace_size(L_g, B, Hq, Hkv, d, k), dev)

    def scores_local(self, qI: torch.Tensor, w: torch.Tensor, stream=None) -> torch.Tensor:
        """Indexer scores over the local slice, into self.scores."""
        if self.S_max > 0:
            index_score(qI, w, self.KI, self.seq_off, self.seq_len, self.S_max, scores=self.scores,
                        ws=self.ws_index, stream=stream)
        return self.scores

    def radix_level(self, level: int, gathered: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Exchange level 0, 1 or 2: the previous level's threshold from every
        rank's histograms `gathered` int32 [N, B, bins] (levels 1, 2), then
        this rank's histogram of the level, into self.hist[level]."""
        return cp_radix_level(self.scores, self.seq_len, self.k, self.N, level, gathered, hist_out=self.hist[level],
                              ws=self.ws_radix, stream=stream)

    def radix_select(self, gathered: torch.Tensor, stream=None) -> torch.Tensor:
        """gathered int32 [N, B, 256] (level 2) -> this rank's share of the
        global top-k, into self.local_idx and self.local_count."""
        return cp_radix_select(self.scores, self.seq_len, self.k, self.N, self.rank, gathered,
                               local_idx=self.local_idx, local_count=self.local_count, ws=self.ws_radix,
                               stream=stream)

    def partial(self, Q: torch.Tensor, stream=None) -> torch.Tensor:
        """Unnormalised attention over the local selected rows, into self.part."""
        o, ml = part_views(self.part, self.rows, self.d)
        sparse_decode_attn_partial(Q, self.K, self.V, self.seq_off, self.seq_len, self.local_idx, self.Hkv,
                                   self.scale, O_part=o.view(self.L_g, self.B, self.Hq, self.d),
                                   ml=ml.view(self.L_g, self.B, self.Hq, 2), idx_count=self.local_count,
                                   ws=self.ws_attn, stream=stream)
        return self.part

    def combine(self, gathered: torch.Tensor, O: Optional[torch.Tensor] = None, out_dtype=torch.bfloat16,
                stream=None) -> torch.Tensor:
        """gathered fp32 [N, part_floats] -> O [L_g, B, Hq, d]."""
        o, ml = part_views(gathered, self.rows, self.d)
        out = None if O is None else O.view(self.rows, self.d)
        out = combine_partials(o, ml, O=out, out_dtype=out_dtype, stream=stream)
        return out.view(self.L_g, self.B, self.Hq, self.d)


Exchange = Callable[[torch.Tensor], torch.Tensor]


def nccl_exchange(N: int, group=None) -> Exchange:
    """All-gather over torch.distributed: t -> [N, *t.shape] in rank order."""

    def exchange(t: torch.Tensor) -> torch.Tensor:
        out = torch.empty(N * t.numel(), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous().view(-1), group=group)
        return out.view((N,) + tuple(t.shape))

    return exchange


def select(rank_state: CPRank, exchange: Exchange, stream=None) -> torch.Tensor:
    """This rank's share of the global top-k from its scores: three histogram
    levels, each all-gathered, then the selection."""
    h = rank_state.radix_level(0, None, stream)
    h = rank_state.radix_level(1, exchange(h), stream)
    h = rank_state.radix_level(2, exchange(h), stream)
    return rank_state.radix_select(exchange(h), stream)


def step(rank_state: CPRank, exchange: Exchange, qI: torch.Tensor, w: torch.Tensor, Q: torch.Tensor,
         O: Optional[torch.Tensor] = None, out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    """One context-parallel decode step of a layer group on this rank.

    qI bf16 [B, H_I, d_I], w fp32 [B, H_I]: the group's indexer query (the
    same on every rank); Q bf16 [L_g, B, Hq, d]: the group's queries.  Every
    rank returns the whole O [L_g, B, Hq, d]."""
    rank_state.scores_local(qI, w, stream)
    select(rank_state, exchange, stream)
    part = rank_state.partial(Q, stream)
    return rank_state.combine(exchange(part), O, out_dtype, stream)


def emulate_step(ranks: Sequence[CPRank], qI: torch.Tensor, w: torch.Tensor, Q: torch.Tensor,
                 out_dtype=torch.bfloat16, stream=None) -> Tuple[torch.Tensor, List[torch.Tensor]]:
    """All N ranks of a step on one device, phase by phase (no kernel waits on
    another rank's): returns rank 0's O and every rank's local index."""
    for r in ranks:
        r.scores_local(qI, w, stream)
    h = torch.stack([r.radix_level(0, None, stream) for r in ranks])
    h = torch.stack([r.radix_level(1, h, stream) for r in ranks])
    h = torch.stack([r.radix_level(2, h, stream) for r in ranks])
    for r in ranks:
        r.radix_select(h, stream)
    parts = torch.stack([r.partial(Q, stream) for r in ranks])
    return ranks[0].combine(parts, None, out_dtype, stream), [r.local_idx for r in ranks]


def main(argv=None) -> int:
    """Run emulated context-parallel decode steps on one GPU (seeded random
    inputs of the given shape; defaults: 4 sequences of 128K tokens, a 16x128
    indexer, k = 2048, one group of 24 layers with 32q/8kv heads of 128)."""
    import argparse
    import math

    p = argparse.ArgumentParser(prog="python -m cross_layer_shared_b200.cp")
    p.add_argument("--ranks", type=int, default=8)
    p.add_argument("--steps", type=int, default=2)
    p.add_argument("--batch", type=int, default=4)
    p.add_argument("--context", type=int, default=131072)
    p.add_argument("--k", type=int, default=2048)
    p.add_argument("--layers", type=int, default=24)
    p.add_argument("--seed", type=int, default=1)
    a = p.parse_args(argv)
    H_I, d_I, Hq, Hkv, d = 16, 128, 32, 8, 128
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(a.seed)

    def rnd(*shape, s=1.0):
        return (torch.randn(*shape, device=dev, generator=g) * s).to(torch.bfloat16)

    qI, w = rnd(a.batch, H_I, d_I, s=0.25), torch.rand(a.batch, H_I, device=dev, generator=g)
    Q = rnd(a.layers, a.batch, Hq, d)
    bnd = shard_bounds([a.context] * a.batch, a.ranks)
    ranks = []
    for r in range(a.ranks):
        n = [int(x) for x in bnd[r, :, 1] - bnd[r, :, 0]]
        T = sum(n)
        ranks.append(CPRank(a.ranks, r, rnd(T, d_I, s=0.25), rnd(T * Hkv * d), rnd(T * Hkv * d), n, a.k, H_I, d_I, Hq,
                            Hkv, d, a.layers, 1 / math.sqrt(d)))
    for _ in range(a.steps):
        O, local = emulate_step(ranks, qI, w, Q)
    torch.cuda.synchronize()
    print(f"{a.steps} emulated steps over {a.ranks} ranks; selected per rank "
          f"{[int((x >= 0).sum().item()) for x in local]}; |O| max {O.float().abs().max().item():.4f}")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
