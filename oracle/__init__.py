"""CPU oracle for cross-layer shared sparse attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares no code with the CUDA path in
``cross_layer_shared_b200``: the arithmetic is the plain C in
``oracle/sa_oracle.c`` (fp64, naive loops, OpenMP over independent
outputs), loaded here through ctypes; the only Python logic is the layer
pattern walk of ``decode_step`` (IndexCache's F/S rule) and argument
marshalling.  The context-parallel pieces (``sparse_decode_attn_partial``,
``combine_partials``, ``cp_select``) have no oracle of a whole sharded step:
a sharded step must equal the one-device ``decode_step``, which is the
oracle for it.

Parity pins: tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.c")
_LIB = os.path.join(_HERE, "libsa_oracle.so")
CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def load(path: str):
    """Load a compiled oracle library and declare its signatures."""
    lb = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    I64 = ctypes.c_int64
    D = ctypes.c_double
    lb.oracle_index_score.argtypes = [P, P, P, P, P, P, I, I, I, P, I64]
    lb.oracle_topk.argtypes = [P, I64, P, I, I, P, P]
    lb.oracle_sparse_decode_attn.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, D, P]
    lb.oracle_block_union.argtypes = [P, I, I, I, I, I, P, P]
    lb.oracle_block_union.restype = I
    lb.oracle_paged_prefill_attn.argtypes = [P, P, P, P, I, I, I, I, I, I, P, P, D, P]
    lb.oracle_indexer_layer_attn.argtypes = [P, P, P, P, P, I, I, I, I, I, D, P, P, I64, P]
    lb.oracle_sparse_decode_attn_partial.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, D, P, P]
    lb.oracle_combine_partials.argtypes = [P, P, I, I64, I, P]
    lb.oracle_cp_select.argtypes = [P, P, I, I, I, I, P]
    lb.oracle_topk_dynamic.argtypes = [P, I64, P, I, I, D, P, P]
    lb.oracle_kap_order.argtypes = [P, I, I, I, I, I, P, I, P, I64]
    lb.oracle_osk_prefill_attn.argtypes = [P, P, P, P, I, I, I, I, I, I, P, I64, I, I, D, D, I, P, I, P, P, P, P, I64]
    lb.oracle_num_threads.restype = I
    return lb


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def index_score(qI, w, KI, seq_off, q_seq, q_pos, ld: Optional[int] = None) -> np.ndarray:
    """scores [Nq, ld] fp32; entries past q_pos are NaN (never written)."""
    qI = _c(qI, np.uint16)
    Nq, H_I, d_I = qI.shape
    w = _c(w, np.float32)
    KI = _c(KI, np.uint16)
    seq_off = _c(seq_off, np.int64)
    q_seq = _c(q_seq, np.int32)
    q_pos = _c(q_pos, np.int32)
    ld = int(ld if ld is not None else q_pos.max() + 1)
    out = np.full((Nq, ld), np.nan, dtype=np.float32)
    lib().oracle_index_score(_p(qI), _p(w), _p(KI), _p(seq_off), _p(q_seq), _p(q_pos), Nq, H_I, d_I,
                             _p(out), ld)
    return out


def topk(scores, n_valid, k: int, with_scores: bool = False):
    scores = _c(scores, np.float32)
    Nq, ld = scores.shape
    n_valid = _c(n_valid, np.int32)
    idx = np.empty((Nq, k), dtype=np.int32)
    ts = np.empty((Nq, k), dtype=np.float32) if with_scores else None
    lib().oracle_topk(_p(scores), ld, _p(n_valid), Nq, k, _p(idx), _p(ts))
    return (idx, ts) if with_scores else idx


def topk_dynamic(scores, n_valid, k_max: int, tau: float):
    """Dynamic k by routing mass (see oracle_topk_dynamic): (idx [Nq, k_max]
    ascending then -1, counts [Nq])."""
    scores = _c(scores, np.float32)
    Nq, ld = scores.shape
    n_valid = _c(n_valid, np.int32)
    idx = np.empty((Nq, k_max), dtype=np.int32)
    counts = np.empty(Nq, dtype=np.int32)
    lib().oracle_topk_dynamic(_p(scores), ld, _p(n_valid), Nq, k_max, float(tau), _p(idx), _p(counts))
    return idx, counts


def sparse_decode_attn(Q, K, V, seq_off, seq_len, idx, Hkv: int, scale: float) -> np.ndarray:
    Q = _c(Q, np.uint16)
    L, B, Hq, d = Q.shape
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    idx = _c(idx, np.int32)
    k = idx.shape[1]
    out = np.empty((L, B, Hq, d), dtype=np.float64)
    lib().oracle_sparse_decode_attn(_p(Q), _p(K), _p(V), _p(_c(seq_off, np.int64)),
                                    _p(_c(seq_len, np.int32)), _p(idx), L, B, Hq, Hkv, d, k,
                                    float(scale), _p(out))
    return out


def sparse_decode_attn_partial(Q, K, V, seq_off, seq_len, idx, Hkv: int, scale: float):
    """One rank's share of a context-parallel step: (O_part [L,B,Hq,d],
    ml [L,B,Hq,2]) fp64, the attention rows before the division, with the
    row max in log2 units and the sum of weights."""
    Q = _c(Q, np.uint16)
    L, B, Hq, d = Q.shape
    idx = _c(idx, np.int32)
    k = idx.shape[1]
    O = np.empty((L, B, Hq, d), dtype=np.float64)
    ml = np.empty((L, B, Hq, 2), dtype=np.float64)
    lib().oracle_sparse_decode_attn_partial(_p(Q), _p(_c(K, np.uint16)), _p(_c(V, np.uint16)),
                                            _p(_c(seq_off, np.int64)), _p(_c(seq_len, np.int32)), _p(idx), L,
                                            B, Hq, Hkv, d, k, float(scale), _p(O), _p(ml))
    return O, ml


def combine_partials(O_part, ml) -> np.ndarray:
    """Log-sum-exp merge of P partials: O_part [P, rows, d], ml [P, rows, 2]."""
    O_part = _c(O_part, np.float64)
    ml = _c(ml, np.float64)
    P, rows, d = O_part.shape
    out = np.empty((rows, d), dtype=np.float64)
    lib().oracle_combine_partials(_p(O_part), _p(ml), P, rows, d, _p(out))
    return out


def cp_select(cand_scores, cand_idx, rank: int) -> np.ndarray:
    """Global top-k of N ranks' candidates [N, B, k]; rank's local indices [B, k]."""
    cand_scores = _c(cand_scores, np.float32)
    cand_idx = _c(cand_idx, np.int32)
    N, B, k = cand_idx.shape
    out = np.empty((B, k), dtype=np.int32)
    lib().oracle_cp_select(_p(cand_scores), _p(cand_idx), N, B, k, int(rank), _p(out))
    return out


def indexer_layer_attn(Q, K, V, seq_off, seq_len, Hkv: int, scale: float, ld: Optional[int] = None):
    """The CLSA indexer layer as a full attention layer whose weights route
    the shared index: (O [B,Hq,d] fp64 dense output, route [B, ld] fp32 with
    route[b,t] = sum over heads of the attention weight of token t; entries
    past seq_len[b] are NaN)."""
    Q = _c(Q, np.uint16)
    B, Hq, d = Q.shape
    seq_len = _c(seq_len, np.int32)
    S_max = int(seq_len.max()) if B else 0
    ld = int(ld if ld is not None else max(S_max, 1))
    O = np.empty((B, Hq, d), dtype=np.float64)
    route = np.full((B, ld), np.nan, dtype=np.float32)
    P = np.empty((B, Hq, max(S_max, 1)), dtype=np.float64)
    lib().oracle_indexer_layer_attn(_p(Q), _p(_c(K, np.uint16)), _p(_c(V, np.uint16)), _p(_c(seq_off, np.int64)),
                                    _p(seq_len), B, Hq, Hkv, d, max(S_max, 1), float(scale), _p(O), _p(route), ld,
                                    _p(P))
    return O, route


def decode_step_attn_route(Q, K, V, seq_off, seq_len, k: int, Hkv: int, scale: float):
    """One decode step of a cross-decoder group under the CLSA reading in
    which layer 0 is the indexer layer: it attends densely, the top-k of its
    summed attention weights is the index, and layers 1..L-1 reuse that index
    over the same cache.  Returns (O [L,B,Hq,d] fp64, idx [B,k], route)."""
    Q = np.asarray(Q)
    O0, route = indexer_layer_attn(Q[0], K, V, seq_off, seq_len, Hkv, scale)
    idx = topk(route, seq_len, k)
    out = [O0]
    if Q.shape[0] > 1:
        out.extend(sparse_decode_attn(Q[1:], K, V, seq_off, seq_len, idx, Hkv, scale))
    return np.stack(out), idx, route


def block_union(idx, S: int, block: int, Hkv: int):
    idx = _c(idx, np.int32)
    Nq, k = idx.shape
    nb = (S + block - 1) // block
    indptr = np.zeros(Hkv + 1, dtype=np.int32)
    indices = np.zeros(max(1, Hkv * nb), dtype=np.int32)
    n = lib().oracle_block_union(_p(idx), Nq, k, S, block, Hkv, _p(indptr), _p(indices))
    return indptr, indices[: Hkv * n].copy()


def paged_prefill_attn(Q, q_pos, K, V, block: int, kv_indptr, kv_indices, scale: float) -> np.ndarray:
    Q = _c(Q, np.uint16)
    Nq, Hq, d = Q.shape
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    Hkv, S, _ = K.shape
    out = np.empty((Nq, Hq, d), dtype=np.float64)
    ind = _c(kv_indices, np.int32)
    if ind.size == 0:
        ind = np.zeros(1, np.int32)
    lib().oracle_paged_prefill_attn(_p(Q), _p(_c(q_pos, np.int32)), _p(K), _p(V), S, Nq, Hq, Hkv, d,
                                    block, _p(_c(kv_indptr, np.int32)), _p(ind), float(scale),
                                    _p(out))
    return out


def kap_order(idx, S: int, block: int, q_block: int, T) -> np.ndarray:
    """CoSA's proxy read as a priority list per query block of q_block
    queries: the union table T ordered by hit count (entries of the block's
    index rows falling in each table block), larger first, ties by
    ascending block id.  Returns int32 [ceil(Nq/q_block), len(T)]."""
    idx = _c(idx, np.int32)
    Nq, k = idx.shape
    T = _c(T, np.int32)
    nT = int(T.size)
    n_qb = (Nq + q_block - 1) // q_block
    order = np.zeros((n_qb, max(1, nT)), dtype=np.int32)
    lib().oracle_kap_order(_p(idx), Nq, k, S, block, q_block, _p(T if nT else np.zeros(1, np.int32)), nT,
                           _p(order), order.shape[1])
    return order[:, :nT].copy()


def osk_prefill_attn(Q, q_pos, K, V, block: int, order, q_block: int, scale: float, tau: float,
                     lag: int = 2, units=None, steps_in=None):
    """CoSA's ordered-skipping kernel under the reading in oracle/sa_oracle.c:
    unit (query block i, KV group g) runs the blocks of order[i] two per
    step and stops lag steps after the first step whose largest row share
    of the running softmax mass is below tau.  Returns (O [Nq,Hq,d] fp64,
    NaN outside the computed units; steps [n_units] int32, -1 where not
    computed; crit [n_units, n_steps] fp64, NaN where not computed).  With
    steps_in [n_units], unit u runs steps_in[u] steps instead (the attention
    over a given prefix of its order; crit is still the rule's)."""
    Q = _c(Q, np.uint16)
    Nq, Hq, d = Q.shape
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    Hkv, S, _ = K.shape
    order = _c(order, np.int32)
    n_qb, nT = order.shape
    assert n_qb == (Nq + q_block - 1) // q_block
    n_steps = (nT + 1) // 2
    O = np.full((Nq, Hq, d), np.nan, dtype=np.float64)
    steps = np.full(n_qb * Hkv, -1, dtype=np.int32)
    crit = np.full((n_qb * Hkv, max(1, n_steps)), np.nan, dtype=np.float64)
    u = None if units is None else _c(units, np.int32)
    ordp = order if order.size else np.zeros(1, np.int32)
    lib().oracle_osk_prefill_attn(_p(Q), _p(_c(q_pos, np.int32)), _p(K), _p(V), S, Nq, Hq, Hkv, d, block,
                                  _p(ordp), max(1, nT), nT, q_block, float(scale), float(tau), int(lag),
                                  _p(u), 0 if u is None else int(u.size),
                                  _p(None if steps_in is None else _c(steps_in, np.int32)), _p(O), _p(steps), _p(crit),
                                  crit.shape[1])
    return O, steps, crit[:, :n_steps]


def kv_append(KI, K, V, seq_off, seq_len, new_KI, new_K, new_V, Hkv: int, d: int):
    """The caches after the new token of every sequence is written at
    position seq_len[b] - 1 (the length counts the new token): row
    seq_off[b] + seq_len[b] - 1 of KI gets new_KI[b]; in sequence b's KV
    region ([Hkv, seq_len[b], d] from element seq_off[b]*Hkv*d) the row of
    every head at that position gets new_K[b, h] / new_V[b, h].  Plain
    copies; returns (KI, K, V) as new arrays."""
    KI = np.array(KI, copy=True)
    K = np.array(K, copy=True).reshape(-1)
    V = np.array(V, copy=True).reshape(-1)
    new_K = np.asarray(new_K).reshape(len(seq_len), Hkv, d)
    new_V = np.asarray(new_V).reshape(len(seq_len), Hkv, d)
    for b, n in enumerate(seq_len):
        t = int(n) - 1
        KI[int(seq_off[b]) + t] = new_KI[b]
        for h in range(Hkv):
            row = (int(seq_off[b]) * Hkv + h * int(n) + t) * d
            K[row:row + d] = new_K[b, h]
            V[row:row + d] = new_V[b, h]
    return KI, K, V


def decode_step(pattern: str, qI: Sequence, w: Sequence, KI: Sequence, seq_off, seq_len, k: int,
                Q, K: Sequence, V: Sequence, Hkv: int, scale: float):
    """One decode step over the layers of `pattern` [IndexCache, technical
    summary section 2: an F layer runs its indexer and overwrites the cached
    top-k index; an S layer reuses the index of the nearest upstream F
    layer].  qI/w/KI/K/V are per-layer lists (entries of S layers' indexer
    inputs are ignored).  Returns (O [L,B,Hq,d] fp64, list of the index used
    by each layer)."""
    if not pattern or pattern[0] != "F":
        raise ValueError("a layer pattern must start with F: an S layer needs an upstream F layer")
    L = len(pattern)
    B = len(seq_len)
    seq_len = np.asarray(seq_len, dtype=np.int32)
    out = []
    used = []
    idx = None
    for layer in range(L):
        if pattern[layer] == "F":
            s = index_score(qI[layer], w[layer], KI[layer], seq_off, np.arange(B), seq_len - 1)
            idx = topk(s, seq_len, k)
        elif pattern[layer] != "S":
            raise ValueError("pattern letters are F or S")
        used.append(idx)
        out.append(sparse_decode_attn(np.asarray(Q)[layer:layer + 1], K[layer], V[layer], seq_off,
                                      seq_len, idx, Hkv, scale)[0])
    return np.stack(out), used
