"""Comparison rules between the CUDA path and the oracle.

* Indexer scores: the GPU accumulates exact bf16 products in fp32 in an
  order of its own; the oracle is the exact value rounded once.  Any fp32
  summation of n terms (ties-to-even or truncating adds) stays within
  gamma_n * sum|terms| with gamma_n = n * 2^-23 / (1 - n * 2^-23), so per key
  |gpu - oracle| <= gamma_{d_I + H_I + 2} * sum_j w_j sum_c |q_jc k_c| + ulp(oracle).
* Top-k: bit-exact against the oracle's top-k of the SAME fp32 scores (the
  decision is integer work on identical inputs); against the oracle's own
  scores, exact outside the ambiguous band A = {t: |s_t - s_(k)| <= 1e-3 |s_(k)|}.
* Attention: max-abs 1e-2 for bf16 outputs, 1e-4 for fp32 outputs, computed
  by the oracle on the GPU's (validated) index.
* Routing scores of the indexer layer (sum over heads of attention weights):
  each GPU logit is an fp32 sum of 16-term chains and a 3-level butterfly,
  so |dz| <= gamma_20 * scale * sum_c |q_c k_c| (natural units).  A weight
  2^(z - M) / L then carries at most |dz| from z, |dz| from M, 2|dz| +
  gamma_n from L, and a few ulp from exp2; the head sum adds gamma_Hq.  The
  relative bound is 4 |dz|_max + gamma_64 + gamma_Hq + 8 ulp.
"""
from __future__ import annotations

import numpy as np

from synth import bf16_bits_to_f32, gather_selected_rows

ATOL_BF16 = 1e-2
ATOL_F32 = 1e-4
BAND = 1e-3


def index_error_bound(qI_bits, w, KI_bits) -> np.ndarray:
    """Per-key bound on |fp32 score - exact score| (see module doc)."""
    H_I, d_I = qI_bits.shape
    q = np.abs(bf16_bits_to_f32(qI_bits).astype(np.float64))
    k = np.abs(bf16_bits_to_f32(KI_bits).astype(np.float64))
    mag = k @ (q.T @ np.asarray(w, np.float64))
    n = d_I + H_I + 2
    u = 2.0 ** -23
    gamma = n * u / (1 - n * u)
    return gamma * mag


def route_rtol(Q_bits, K_bits, scale) -> float:
    """Relative bound on GPU vs oracle routing scores (see module doc).
    Q_bits [Hq, d]; K_bits [Hkv, S, d] of one sequence."""
    Hq, d = Q_bits.shape
    Hkv = K_bits.shape[0]
    G = Hq // Hkv
    q = np.abs(bf16_bits_to_f32(Q_bits).astype(np.float64))
    mag = 0.0
    for g in range(Hkv):
        k = np.abs(bf16_bits_to_f32(K_bits[g]).astype(np.float64))
        mag = max(mag, float((k @ q[g * G:(g + 1) * G].T).max()))
    u = 2.0 ** -23

    def gamma(n):
        return n * u / (1 - n * u)
    return 4 * gamma(20) * scale * mag + gamma(64) + gamma(Hq) + 8 * u


def assert_scores_close(gpu, ora, bound, what=""):
    gpu = np.asarray(gpu, np.float64)
    ora = np.asarray(ora, np.float64)
    tol = bound + np.abs(ora) * 2.0 ** -24 + 1e-30
    err = np.abs(gpu - ora)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, f"{what}: {bad.size} scores outside the fp32 bound, first {bad[:5]} err {err[bad[:5]]} tol {tol[bad[:5]]}"


def assert_valid_index_row(row, n, k):
    """ascending, distinct, in [0, n), then -1 padding; min(k, n) entries."""
    row = np.asarray(row)
    m = min(k, n)
    assert np.all(row[m:] == -1), "padding must be -1"
    sel = row[:m]
    assert np.all(sel >= 0) and np.all(sel < n), "index out of range"
    assert np.all(np.diff(sel) > 0), "indices must be strictly ascending"


def assert_topk_band(gpu_row, ora_scores, n, k, what=""):
    """GPU set vs the oracle's scores with the ambiguous band around the k-th score."""
    s = np.asarray(ora_scores[:n], np.float64)
    m = min(k, n)
    assert_valid_index_row(gpu_row, n, k)
    gset = set(int(t) for t in gpu_row[:m])
    if m == n:
        assert gset == set(range(n))
        return
    order = np.lexsort((np.arange(n), -s))  # score desc, index asc
    ora = set(int(t) for t in order[:m])
    kth = s[order[m - 1]]
    band = set(int(t) for t in np.nonzero(np.abs(s - kth) <= BAND * abs(kth))[0])
    missing = [t for t in ora - gset if t not in band]
    extra = [t for t in gset - ora if t not in band]
    assert not missing and not extra, f"{what}: missing {missing[:5]} extra {extra[:5]} (band {len(band)})"


def compact_selected(K_rows_fn, idx_row, Hkv, d):
    """Compact [Hkv, m, d] copy of the rows a selection uses, remapped index."""
    return gather_selected_rows(K_rows_fn, idx_row, Hkv, d)
