"""Seeded synthetic inputs for the cross-layer shared sparse-attention path.

This module is shared by both sides of every parity check: the CPU oracle
(``oracle/``) and the CUDA path (``cross_layer_shared_b200``) receive the
same tensors from here.  It contains none of the method's arithmetic: no
indexer score, no top-k, no attention.  Only random draws, the workload
shapes, and the planted structure (needles, hot regions) that make the
synthetic data look like the pages' workloads.

Generator (counter based, so any element can be produced on its own):

* ``key = mix64(seed * GAMMA + tid)`` names one tensor stream,
* element ``i`` of the stream is ``h(i) = mix64(key + (i + 1) * GAMMA)``,
  i.e. the i-th output of the published SplitMix64 generator started at
  ``key`` (Steele, Lea, Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; finaliser constants from Stafford's "Mix13").
* "~N(0,1)": Irwin-Hall sum of the four 16-bit fields of ``h(i)``, centred
  and multiplied once in fp32 by sqrt(3)/65536 (variance 1, support
  +-3.46).  Integer operations plus one IEEE multiply, so the CUDA twin in
  ``synth/synth.cu`` produces the same bits.
* "~U(a,b)": ``a + u*(b-a)`` in fp32 with ``u = (h >> 40) * 2**-24``.
* bf16 storage: round-to-nearest-even of the fp32 value.

Large tensors (indexer keys, K, V) are filled on the GPU by the CUDA twin;
small ones (queries, head weights, planted rows) are made here and copied.
The host can also produce any subset of a large tensor by flat index, which
is how full-size parity checks feed the oracle.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1
# fp32 value of sqrt(3)/65536 rounded to nearest (bits 0x37ddb3d7)
IH_SCALE = np.array([0x37DDB3D7], dtype=np.uint32).view(np.float32)[0]

# tensor-stream identifiers; a per-group stream adds 64*group
TID_QI, TID_KI, TID_W, TID_Q, TID_K, TID_V = 1, 2, 3, 4, 5, 6
TID_QEPS, TID_PLANT, TID_SEQLEN, TID_DIR, TID_QPREF = 7, 8, 9, 10, 11


def tid_for(base: int, group: int = 0) -> int:
    return base + 64 * group


# --------------------------------------------------------------------------
# counter-based draws
# --------------------------------------------------------------------------
def _mix64_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tid: int) -> int:
    return _mix64_int(seed * GAMMA + tid)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def hash_at(seed: int, tid: int, idx) -> np.ndarray:
    """h(i) for an array of flat indices (uint64)."""
    key = np.uint64(stream_key(seed, tid))
    i = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + (i + np.uint64(1)) * np.uint64(GAMMA))


def normal_at(seed: int, tid: int, idx) -> np.ndarray:
    h = hash_at(seed, tid, idx)
    m = np.uint64(0xFFFF)
    s = (h & m) + ((h >> np.uint64(16)) & m) + ((h >> np.uint64(32)) & m) + (h >> np.uint64(48))
    c = (s.astype(np.int64) - 131070).astype(np.float32)
    return c * IH_SCALE


def uniform_at(seed: int, tid: int, idx, lo: float, hi: float) -> np.ndarray:
    h = hash_at(seed, tid, idx)
    u = (h >> np.uint64(40)).astype(np.float32) * np.float32(2.0 ** -24)
    return np.float32(lo) + u * (np.float32(hi) - np.float32(lo))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16_at(seed: int, tid: int, idx, scale: float = 1.0) -> np.ndarray:
    return f32_to_bf16_bits(normal_at(seed, tid, idx) * np.float32(scale))


def normal_bf16(seed: int, tid: int, n: int, scale: float = 1.0, offset: int = 0) -> np.ndarray:
    return normal_bf16_at(seed, tid, np.arange(offset, offset + n, dtype=np.uint64), scale)


def distinct_positions(seed: int, tid: int, count: int, lo: int, hi: int, align: int = 1,
                       span: int = 1) -> List[int]:
    """`count` distinct, non-overlapping starts in [lo, hi) (multiples of
    `align`, each covering `span` positions), drawn in stream order."""
    slots = (hi - lo - span) // align + 1
    assert slots >= count * max(1, span // align)
    out: List[int] = []
    i = 0
    while len(out) < count:
        p = lo + int(hash_at(seed, tid, [i])[0] % np.uint64(slots)) * align
        i += 1
        if all(p + span <= q or q + span <= p for q in out):
            out.append(p)
    return out


def gather_selected_rows(rows_fn, idx_row, Hkv: int, d: int):
    """Copy the cache rows a selection uses into a compact [Hkv, m, d] cache
    and remap the index to it (-1 entries stay -1).  rows_fn(head, rows)
    returns the bf16 rows.  Pure data movement."""
    idx_row = np.asarray(idx_row)
    valid = idx_row[idx_row >= 0]
    m = max(len(valid), 1)
    K = np.zeros((Hkv, m, d), np.uint16)
    for h in range(Hkv):
        if len(valid):
            K[h] = rows_fn(h, valid)
    remap = np.full(len(idx_row), -1, np.int32)
    remap[idx_row >= 0] = np.arange(len(valid), dtype=np.int32)
    return K, remap, m


def _unit(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    return v / np.linalg.norm(v)


# --------------------------------------------------------------------------
# decode workloads
# --------------------------------------------------------------------------
@dataclasses.dataclass
class DecodeConfig:
    """One decode step: for every layer of `pattern` ('F' = the layer runs
    the indexer and overwrites the shared index, 'S' = it reuses it), every
    sequence of the batch.  Each F layer starts a group whose layers read
    one KV cache."""
    name: str
    seq_lens: List[int]
    H_I: int
    d_I: int
    k: int
    pattern: str
    Hq: int
    Hkv: int
    d: int
    seed: int
    needles: int = 0        # planted in the indexer keys and the attention keys
    planted_ki: int = 0     # planted in the indexer keys only
    q_rho: Optional[float] = None  # AR(1) correlation of Q between layers

    @property
    def B(self) -> int:
        return len(self.seq_lens)

    @property
    def L(self) -> int:
        return len(self.pattern)

    @property
    def groups(self) -> List[range]:
        starts = [i for i, c in enumerate(self.pattern) if c == "F"]
        assert starts and starts[0] == 0, "a layer pattern must start with F"
        ends = starts[1:] + [len(self.pattern)]
        return [range(a, b) for a, b in zip(starts, ends)]

    @property
    def seq_off(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seq_lens)]).astype(np.int64)

    @property
    def T(self) -> int:
        return int(sum(self.seq_lens))

    @property
    def S_max(self) -> int:
        return int(max(self.seq_lens))

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.d)))

    # ---- small tensors, made on the host --------------------------------
    def qI(self, g: int) -> np.ndarray:
        n = self.B * self.H_I * self.d_I
        return normal_bf16(self.seed, tid_for(TID_QI, g), n, 0.125).reshape(self.B, self.H_I, self.d_I)

    def w(self, g: int) -> np.ndarray:
        n = self.B * self.H_I
        return uniform_at(self.seed, tid_for(TID_W, g), np.arange(n), 0.1, 1.0).reshape(self.B, self.H_I)

    def Q(self) -> np.ndarray:
        shape = (self.L, self.B, self.Hq, self.d)
        per = self.B * self.Hq * self.d
        if self.q_rho is None:
            return normal_bf16(self.seed, TID_Q, self.L * per).reshape(shape)
        rho = np.float32(self.q_rho)
        c = np.float32(math.sqrt(1.0 - self.q_rho * self.q_rho))
        out = np.empty(shape, dtype=np.uint16)
        prev = normal_at(self.seed, TID_Q, np.arange(per))
        out[0] = f32_to_bf16_bits(prev).reshape(shape[1:])
        for layer in range(1, self.L):
            eps = normal_at(self.seed, TID_QEPS, np.arange(layer * per, (layer + 1) * per))
            prev = rho * prev + c * eps
            out[layer] = f32_to_bf16_bits(prev).reshape(shape[1:])
        return out

    # ---- bulk tensors: stream ids and scales ----------------------------
    def ki_stream(self, g: int):
        return tid_for(TID_KI, g), 0.125

    def k_stream(self, g: int):
        return tid_for(TID_K, g), 1.0

    def v_stream(self, g: int):
        return tid_for(TID_V, g), 1.0

    # ---- planted rows ---------------------------------------------------
    def planted(self, g: int):
        """Planted rows of group g: list of (b, t, ki_row or None,
        k_rows [Hkv,d] or None) as bf16 bit patterns."""
        out = []
        n = self.needles + self.planted_ki
        if n == 0:
            return out
        qI = bf16_bits_to_f32(self.qI(g)).astype(np.float64)
        w = self.w(g).astype(np.float64)
        Q0 = bf16_bits_to_f32(self.Q()[self.groups[g][0]]).astype(np.float64) if self.needles else None
        G = self.Hq // self.Hkv
        for b in range(self.B):
            pos = distinct_positions(self.seed, tid_for(TID_PLANT, g) + 4096 * b, n, 0, self.seq_lens[b])
            u = _unit((w[b][:, None] * qI[b]).sum(axis=0))
            ki = f32_to_bf16_bits((math.sqrt(self.d_I) * u).astype(np.float32))
            krow = None
            if self.needles:
                vs = [_unit(Q0[b, h * G:(h + 1) * G].mean(axis=0)) for h in range(self.Hkv)]
                krow = f32_to_bf16_bits((4.0 * math.sqrt(self.d) * np.stack(vs)).astype(np.float32))
            for i, t in enumerate(pos):
                out.append((b, t, ki, krow if i < self.needles else None))
        return out

    # ---- host materialisation (small configs / sampled rows) ------------
    def KI_rows(self, g: int, b: int, rows) -> np.ndarray:
        """Indexer-key rows t (of sequence b) of group g, planted rows applied."""
        rows = np.asarray(rows, dtype=np.int64)
        tid, sc = self.ki_stream(g)
        base = int(self.seq_off[b]) + rows
        flat = (base[:, None] * self.d_I + np.arange(self.d_I)[None, :]).astype(np.uint64)
        out = normal_bf16_at(self.seed, tid, flat, sc)
        where = {int(t): i for i, t in enumerate(rows)}
        for (bb, t, ki, _) in self.planted(g):
            if bb == b and t in where:
                out[where[t]] = ki
        return out

    def KV_rows(self, g: int, b: int, head: int, rows, which: str) -> np.ndarray:
        rows = np.asarray(rows, dtype=np.int64)
        tid, sc = self.k_stream(g) if which == "K" else self.v_stream(g)
        S = self.seq_lens[b]
        base = int(self.seq_off[b]) * self.Hkv * self.d + (head * S + rows) * self.d
        flat = (base[:, None] + np.arange(self.d)[None, :]).astype(np.uint64)
        out = normal_bf16_at(self.seed, tid, flat, sc)
        if which == "K" and self.needles:
            where = {int(t): i for i, t in enumerate(rows)}
            for (bb, t, _, krow) in self.planted(g):
                if bb == b and krow is not None and t in where:
                    out[where[t]] = krow[head]
        return out

    def KI_full(self, g: int) -> np.ndarray:
        tid, sc = self.ki_stream(g)
        out = normal_bf16(self.seed, tid, self.T * self.d_I, sc).reshape(self.T, self.d_I)
        for (b, t, ki, _) in self.planted(g):
            out[self.seq_off[b] + t] = ki
        return out

    def KV_full(self, g: int, which: str) -> np.ndarray:
        """Packed per-sequence head-major cache: seq b at seq_off[b]*Hkv*d, [Hkv,S_b,d]."""
        tid, sc = self.k_stream(g) if which == "K" else self.v_stream(g)
        out = normal_bf16(self.seed, tid, self.T * self.Hkv * self.d, sc)
        if which == "K" and self.needles:
            for (b, t, _, krow) in self.planted(g):
                if krow is None:
                    continue
                S = self.seq_lens[b]
                for h in range(self.Hkv):
                    o = int(self.seq_off[b]) * self.Hkv * self.d + (h * S + t) * self.d
                    out[o:o + self.d] = krow[h]
        return out


# --------------------------------------------------------------------------
# chunked prefill workload
# --------------------------------------------------------------------------
@dataclasses.dataclass
class PrefillConfig:
    """One chunk of `chunk` queries at positions [S-chunk, S) of one sequence."""
    name: str
    S: int
    chunk: int
    H_I: int
    d_I: int
    k: int
    block: int
    Hq: int
    Hkv: int
    d: int
    seed: int
    hot_regions: int = 16
    region_len: int = 256
    # attention queries drawn toward the hot regions: Q[p,h] gets q_gain * v_hat(h's KV head)
    # added, and the hot K rows carry hot_k_gain * v_hat (0 and 2 in the plain chunk)
    q_gain: float = 0.0
    hot_k_gain: float = 2.0

    @property
    def q_pos(self) -> np.ndarray:
        return np.arange(self.S - self.chunk, self.S, dtype=np.int32)

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.d)))

    def regions(self) -> List[int]:
        if self.hot_regions == 0:
            return []
        return distinct_positions(self.seed, TID_PLANT, self.hot_regions, 0, self.S - self.chunk,
                                  align=self.block, span=self.region_len)

    def u_hat(self) -> np.ndarray:
        return _unit(normal_at(self.seed, TID_DIR, np.arange(self.d_I)))

    def v_hat(self, h: int) -> np.ndarray:
        return _unit(normal_at(self.seed, TID_DIR + 1, np.arange(h * self.d, (h + 1) * self.d)))

    def qI(self) -> np.ndarray:
        n = self.chunk * self.H_I * self.d_I
        base = normal_at(self.seed, TID_QI, np.arange(n)).reshape(self.chunk, self.H_I, self.d_I)
        x = base * np.float32(0.125) + (0.25 * self.u_hat()).astype(np.float32)
        return f32_to_bf16_bits(x.astype(np.float32))

    def w(self) -> np.ndarray:
        n = self.chunk * self.H_I
        return uniform_at(self.seed, TID_W, np.arange(n), 0.1, 1.0).reshape(self.chunk, self.H_I)

    def Q(self) -> np.ndarray:
        n = self.chunk * self.Hq * self.d
        if self.q_gain == 0.0:
            return normal_bf16(self.seed, TID_Q, n).reshape(self.chunk, self.Hq, self.d)
        x = normal_at(self.seed, TID_Q, np.arange(n)).reshape(self.chunk, self.Hq, self.d)
        G = self.Hq // self.Hkv
        for h in range(self.Hq):
            x[:, h, :] += (self.q_gain * self.v_hat(h // G)).astype(np.float32)
        return f32_to_bf16_bits(x.astype(np.float32))

    def ki_stream(self):
        return TID_KI, 0.125

    def k_stream(self):
        return TID_K, 1.0

    def v_stream(self):
        return TID_V, 1.0

    def hot_ki_rows(self):
        """(positions [n], rows [n,d_I] bf16) of the hot regions in the indexer keys."""
        pos = np.array([p + i for p in self.regions() for i in range(self.region_len)], dtype=np.int64)
        if pos.size == 0:
            return pos, np.zeros((0, self.d_I), np.uint16)
        flat = (pos[:, None] * self.d_I + np.arange(self.d_I)[None, :]).astype(np.uint64)
        x = normal_at(self.seed, TID_KI, flat) * np.float32(0.125) + (0.5 * self.u_hat()).astype(np.float32)
        return pos, f32_to_bf16_bits(x.astype(np.float32))

    def hot_k_rows(self, h: int):
        pos = np.array([p + i for p in self.regions() for i in range(self.region_len)], dtype=np.int64)
        if pos.size == 0:
            return pos, np.zeros((0, self.d), np.uint16)
        flat = ((h * self.S + pos)[:, None] * self.d + np.arange(self.d)[None, :]).astype(np.uint64)
        x = normal_at(self.seed, TID_K, flat) + (self.hot_k_gain * self.v_hat(h)).astype(np.float32)
        return pos, f32_to_bf16_bits(x.astype(np.float32))

    def KI_full(self) -> np.ndarray:
        tid, sc = self.ki_stream()
        out = normal_bf16(self.seed, tid, self.S * self.d_I, sc).reshape(self.S, self.d_I)
        pos, rows = self.hot_ki_rows()
        out[pos] = rows
        return out

    def KV_full(self, which: str) -> np.ndarray:
        tid, sc = self.k_stream() if which == "K" else self.v_stream()
        out = normal_bf16(self.seed, tid, self.Hkv * self.S * self.d, sc).reshape(self.Hkv, self.S, self.d)
        if which == "K":
            for h in range(self.Hkv):
                pos, rows = self.hot_k_rows(h)
                out[h, pos] = rows
        return out

    def KV_rows(self, head: int, rows, which: str) -> np.ndarray:
        rows = np.asarray(rows, dtype=np.int64)
        tid, sc = self.k_stream() if which == "K" else self.v_stream()
        flat = ((head * self.S + rows)[:, None] * self.d + np.arange(self.d)[None, :]).astype(np.uint64)
        out = normal_bf16_at(self.seed, tid, flat, sc)
        if which == "K":
            pos, hot = self.hot_k_rows(head)
            where = {int(p): i for i, p in enumerate(pos)}
            for i, t in enumerate(rows):
                j = where.get(int(t))
                if j is not None:
                    out[i] = hot[j]
        return out


# --------------------------------------------------------------------------
# the five workloads (seed = 1234 + workload number)
# --------------------------------------------------------------------------
def c5_seq_lens(seed: int, B: int = 32, lo: int = 8192, hi: int = 131072) -> List[int]:
    h = hash_at(seed, TID_SEQLEN, np.arange(B))
    return [lo + int(x % np.uint64(hi - lo + 1)) for x in h]


def workload(name: str):
    if name == "c1":
        return DecodeConfig("c1", [4096], 4, 64, 256, "FSSS", 8, 1, 128, seed=1235, needles=8)
    if name == "c2":
        return DecodeConfig("c2", [32768] * 8, 16, 128, 2048, "FSSS" * 3, 32, 4, 128, seed=1236,
                            planted_ki=64)
    if name == "c3":
        return DecodeConfig("c3", [131072] * 4, 16, 128, 2048, "F" + "S" * 23, 32, 8, 128, seed=1237,
                            q_rho=0.9)
    if name == "c4":
        return PrefillConfig("c4", 131072, 2048, 16, 128, 2048, 64, 32, 8, 128, seed=1238)
    if name == "c4-concentrated":
        # the c4 chunk with the attention drawn to the hot regions the indexer
        # finds: same indexer inputs, queries biased along each group's
        # direction, hot K rows four times further along it
        return PrefillConfig("c4-concentrated", 131072, 2048, 16, 128, 2048, 64, 32, 8, 128, seed=1238,
                             q_gain=16.0, hot_k_gain=8.0)
    if name == "c5":
        return DecodeConfig("c5", c5_seq_lens(1239), 16, 128, 2048, "FSSS" * 12, 32, 8, 128, seed=1239)
    raise KeyError(name)


WORKLOADS = ("c1", "c2", "c3", "c4", "c5")

DESCRIPTIONS = {
    "c1": "decode B=1 S=4096, indexer 4x64, k=256, 4 layers (1 full + 3 shared), 8q/1kv heads d=128, 8 needles",
    "c2": "decode B=8 S=32768, indexer 16x128, k=2048, 12 layers F,S,S,S, 32q/4kv heads d=128, 64 planted keys",
    "c3": "decode B=4 S=131072, one indexer pass 16x128, k=2048, shared by 24 cross-decoder layers, 32q/8kv d=128",
    "c4": "chunked prefill 2048 queries vs 131072-token cache, indexer 16x128 k=2048, 64-token blocks, 32q/8kv d=128",
    "c5": "decode B=32 ragged S in [8192,131072], indexer 16x128, k=2048, 48 layers F,S,S,S, 32q/8kv d=128",
    "c4-concentrated": "the c4 chunk with its attention queries biased along each KV group's hot-region "
                       "direction (gain 16) and the hot K rows at gain 8 instead of 2",
}
