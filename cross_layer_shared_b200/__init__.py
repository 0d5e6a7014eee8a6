"""Cross-layer shared sparse attention on B200 (sm_100a).

Thin Python binding of libsa (include/sa.h): argument marshalling only.
Every step of the path runs in the CUDA kernels of ``csrc/``; PyTorch
provides device memory and streams.  There is no CPU fallback: if the
library is not built, every call raises.

Build:  python -m cross_layer_shared_b200.build
"""
from __future__ import annotations

import array
import ctypes
import os
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsa.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE, SA_ERR_CUDA, SA_ERR_TIMEOUT, SA_ERR_DEVICE = range(7)
SA_BF16, SA_F32 = 0, 1
WS_HEADER_BYTES = 4096

# every symbol include/sa.h declares, with its ctypes signature
_P, _I, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_PP = ctypes.POINTER(ctypes.c_void_p)
SIGNATURES = {
    "sa_status_string": ([_I], ctypes.c_char_p),
    "sa_last_error": ([], ctypes.c_char_p),
    "sa_abi_version": ([], _I),
    "sa_read_device_status": ([_P, _P, ctypes.POINTER(_I), ctypes.POINTER(_I64)], _I),
    "sa_clear_device_status": ([_P, _P], _I),
    "sa_wait_probe": ([_P, _SZ, ctypes.c_ulonglong, _P], _I),
    "sa_index_score_workspace_size": ([_I], _SZ),
    "sa_index_score": ([_P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _P, _I64, _P, _SZ, _P], _I),
    "sa_index_score_prefill_workspace_size": ([_I], _SZ),
    "sa_index_score_prefill": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I64, _P, _SZ, _P], _I),
    "sa_topk_workspace_size": ([_I, _I, _I], _SZ),
    "sa_topk": ([_P, _I64, _P, _I, _I, _I, _P, _P, _P, _SZ, _P], _I),
    "sa_topk_dynamic_workspace_size": ([_I, _I, _I], _SZ),
    "sa_topk_dynamic": ([_P, _I64, _P, _I, _I, _I, ctypes.c_double, _P, _P, _P, _SZ, _P], _I),
    "sa_sparse_decode_attn_workspace_size": ([_I, _I, _I, _I, _I, _I], _SZ),
    "sa_sparse_decode_attn": ([_P, _P, _P, _P, _P, _P, _I, _I, _I64, _I, _I, _I, _I, _F, _P, _I, _P, _SZ, _P], _I),
    "sa_indexer_layer_attn_workspace_size": ([_I, _I, _I, _I, _I], _SZ),
    "sa_indexer_layer_attn": ([_P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _F, _P, _I, _P, _I64, _P, _SZ, _P], _I),
    "sa_decode_step_workspace_size": ([_I, _I, _I, _I, _I, _I, _I], _SZ),
    "sa_decode_step": ([ctypes.c_char_p, _I, _P, _P, _P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _P, _I,
                        _I, _I, _F, _P, _I, _P, _P, _I64, _P, _SZ, _P], _I),
    "sa_decode_step_ex": ([ctypes.c_char_p, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I64, _I, _I,
                           _I, _I, _P, _I, _I, _I, _F, _P, _I, _P, _P, _I64, _I, _P, _SZ, _P], _I),
    "sa_block_union_prefill_workspace_size": ([_I, _I, _I, _I, _I, _I, _I], _SZ),
    "sa_block_union_prefill": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _I, _P, _SZ, _P],
                               _I),
    "sa_block_union_prefill_noalloc": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _I, _P],
                                       _I),
    "sa_sparse_decode_attn_partial": ([_P, _P, _P, _P, _P, _P, _I, _I, _I64, _I, _I, _I, _I, _P, _F, _P, _P, _P,
                                       _SZ, _P], _I),
    "sa_cp_select_workspace_size": ([_I, _I, _I], _SZ),
    "sa_cp_select": ([_P, _P, _I64, _I, _I, _I, _I, _P, _P, _P, _SZ, _P], _I),
    "sa_combine_partials": ([_P, _I64, _P, _I64, _I, _I64, _I, _P, _I, _P], _I),
    "sa_index_topk_prefill_workspace_size": ([_I, _I, _I, _I, _I], _SZ),
    "sa_index_topk_prefill": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P], _I),
    "sa_cp_radix_workspace_size": ([_I], _SZ),
    "sa_cp_radix_level": ([_P, _I64, _P, _I, _I, _I, _I, _P, _I64, _P, _P, _SZ, _P], _I),
    "sa_cp_radix_select": ([_P, _I64, _P, _I, _I, _I, _I, _P, _I64, _P, _P, _P, _SZ, _P], _I),
    "sa_kap_order_workspace_size": ([], _SZ),
    "sa_kap_order": ([_P, _I, _I, _I, _I, _I, _P, _P, _P, _I64, _P, _SZ, _P], _I),
    "sa_osk_prefill_workspace_size": ([_I, _I, _I, _I, _I, _I, _I], _SZ),
    "sa_osk_prefill": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _P, _P, _P, _P, _P, _I, _P, _SZ,
                        _P], _I),
}


class SAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_STATUS_NAMES = {0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_UNSUPPORTED", 3: "SA_ERR_WORKSPACE",
                 4: "SA_ERR_CUDA", 5: "SA_ERR_TIMEOUT", 6: "SA_ERR_DEVICE"}

_lib = None


def lib():
    """The loaded libsa.  Raises if the CUDA library has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m cross_layer_shared_b200.build`"
                               " (there is no fallback path)")
        lb = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lb, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lb
    return _lib


def _check(code: int) -> None:
    if code != SA_OK:
        raise SAError(code, lib().sa_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream) -> int:
    """The cudaStream_t of `stream`, or of the current stream (the raw query
    skips building a Stream object on every call)."""
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None:
        return _raw_stream(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _dev(t: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor of {dtype}")
    return t


def _out(t: torch.Tensor, shape, dtypes, name: str) -> torch.Tensor:
    """A caller-supplied output: contiguous, on the GPU, of an accepted dtype
    and exactly the shape the call writes (a kernel would write past a smaller
    one)."""
    if not (t.is_cuda and t.is_contiguous() and t.dtype in dtypes):
        raise ValueError(f"{name} must be a contiguous CUDA tensor of {' or '.join(str(x) for x in dtypes)}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    return t


def _rows_out(t: torch.Tensor, rows: int, min_cols: int, name: str) -> int:
    """A caller-supplied fp32 score table [rows, ld] with ld >= min_cols; returns ld."""
    if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.float32 and t.dim() == 2):
        raise ValueError(f"{name} must be a contiguous 2-D CUDA tensor of torch.float32")
    if t.shape[0] != rows or t.shape[1] < max(min_cols, 1):
        raise ValueError(f"{name} must be [{rows}, >= {max(min_cols, 1)}], not {tuple(t.shape)}")
    return int(t.shape[1])


def _seqs(seq_off: torch.Tensor, seq_len: torch.Tensor, B: int) -> None:
    _out(seq_off, (B + 1,), (torch.int64,), "seq_off")
    _out(seq_len, (B,), (torch.int32,), "seq_len")


def _ws(ws: torch.Tensor) -> torch.Tensor:
    return _dev(ws, torch.uint8, "ws")


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zeroed workspace (status block included) of at least nbytes."""
    n = max(int(nbytes), WS_HEADER_BYTES)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def read_status(ws: torch.Tensor, stream=None):
    """(code, [kernel, element, value, bound]) of the device status block (synchronises)."""
    code = ctypes.c_int(0)
    det = (ctypes.c_int64 * 4)()
    _check(lib().sa_read_device_status(_ptr(ws), _stream(stream), ctypes.byref(code), det))
    return code.value, list(det)


def wait_probe(ws: torch.Tensor, limit_ns: int, stream=None) -> None:
    """sa_wait_probe: one CTA whose bounded wait must give up after limit_ns
    and record SA_ERR_TIMEOUT in ws (a self-test of the kernels' waits)."""
    _ws(ws)
    _check(lib().sa_wait_probe(ws.data_ptr(), ws.numel(), int(limit_ns), _stream(stream)))


def clear_status(ws: torch.Tensor, stream=None) -> None:
    _check(lib().sa_clear_device_status(_ptr(ws), _stream(stream)))


# ---------------------------------------------------------------------------
def index_score(qI, w, KI, seq_off, seq_len, S_max: int, scores=None, ld: Optional[int] = None, ws=None,
                stream=None) -> torch.Tensor:
    B, H_I, d_I = qI.shape
    _dev(qI, torch.bfloat16, "qI"), _dev(w, torch.float32, "w"), _dev(KI, torch.bfloat16, "KI")
    _seqs(seq_off, seq_len, B)
    if scores is None:
        ld = int(ld if ld is not None else max(S_max, 1))
        scores = torch.empty((B, ld), dtype=torch.float32, device=qI.device)
    else:
        have = _rows_out(scores, B, S_max, "scores")
        if ld is not None and int(ld) != have:
            raise ValueError(f"ld={ld} does not match scores of {have} columns")
        ld = have
    if ws is None:
        ws = workspace(lib().sa_index_score_workspace_size(B), qI.device)
    _ws(ws)
    _check(lib().sa_index_score(_ptr(qI), _ptr(w), _ptr(KI), _ptr(seq_off), _ptr(seq_len), B, KI.shape[0], S_max,
                                H_I, d_I, _ptr(scores), ld, _ptr(ws), ws.numel(), _stream(stream)))
    return scores


def index_score_prefill(qI, w, KI, q_pos, max_pos: int, scores=None, ld: Optional[int] = None, ws=None,
                        stream=None) -> torch.Tensor:
    Nq, H_I, d_I = qI.shape
    _dev(qI, torch.bfloat16, "qI"), _dev(w, torch.float32, "w"), _dev(KI, torch.bfloat16, "KI")
    _out(q_pos, (Nq,), (torch.int32,), "q_pos")
    if scores is None:
        ld = int(ld if ld is not None else max_pos + 1)
        scores = torch.empty((Nq, ld), dtype=torch.float32, device=qI.device)
    else:
        have = _rows_out(scores, Nq, max_pos + 1, "scores")
        if ld is not None and int(ld) != have:
            raise ValueError(f"ld={ld} does not match scores of {have} columns")
        ld = have
    if ws is None:
        ws = workspace(lib().sa_index_score_prefill_workspace_size(Nq), qI.device)
    _ws(ws)
    _check(lib().sa_index_score_prefill(_ptr(qI), _ptr(w), _ptr(KI), _ptr(q_pos), Nq, KI.shape[0], max_pos, H_I,
                                        d_I, _ptr(scores), ld, _ptr(ws), ws.numel(), _stream(stream)))
    return scores


def index_topk_prefill_workspace_size(Nq: int, S: int, max_pos: int, k: int, rows_per_block: int = 0) -> int:
    return int(lib().sa_index_topk_prefill_workspace_size(Nq, S, max_pos, k, rows_per_block))


def index_topk_prefill(qI, w, KI, q_pos, max_pos: int, k: int, idx=None, rows_per_block: int = 0, ws=None,
                       stream=None) -> torch.Tensor:
    """Prefill indexer scores and per-query top-k, block of queries by block
    (no score matrix for the whole chunk): idx int32 [Nq, k]."""
    Nq, H_I, d_I = qI.shape
    _dev(qI, torch.bfloat16, "qI"), _dev(w, torch.float32, "w"), _dev(KI, torch.bfloat16, "KI")
    _out(q_pos, (Nq,), (torch.int32,), "q_pos")
    if idx is None:
        idx = torch.empty((Nq, k), dtype=torch.int32, device=qI.device)
    _out(idx, (Nq, k), (torch.int32,), "idx")
    S = KI.shape[0]
    if ws is None:
        ws = workspace(index_topk_prefill_workspace_size(Nq, S, max_pos, k, rows_per_block), qI.device)
    _ws(ws)
    _check(lib().sa_index_topk_prefill(_ptr(qI), _ptr(w), _ptr(KI), _ptr(q_pos), Nq, S, max_pos, H_I, d_I, k,
                                       int(rows_per_block), _ptr(idx), _ptr(ws), ws.numel(), _stream(stream)))
    return idx


def topk(scores, n_valid, n_max: int, k: int, idx=None, top_scores=None, want_scores=False, ws=None, stream=None):
    Nq, ld = scores.shape
    _rows_out(scores, Nq, n_max, "scores")
    _out(n_valid, (Nq,), (torch.int32,), "n_valid")
    if idx is None:
        idx = torch.empty((Nq, k), dtype=torch.int32, device=scores.device)
    _out(idx, (Nq, k), (torch.int32,), "idx")
    if want_scores and top_scores is None:
        top_scores = torch.empty((Nq, k), dtype=torch.float32, device=scores.device)
    if top_scores is not None:
        _out(top_scores, (Nq, k), (torch.float32,), "top_scores")
    if ws is None:
        ws = workspace(lib().sa_topk_workspace_size(Nq, n_max, k), scores.device)
    _ws(ws)
    _check(lib().sa_topk(_ptr(scores), ld, _ptr(n_valid), Nq, n_max, k, _ptr(idx), _ptr(top_scores), _ptr(ws),
                         ws.numel(), _stream(stream)))
    return (idx, top_scores) if want_scores else idx


def topk_dynamic(scores, n_valid, n_max: int, k_max: int, tau: float, idx=None, counts=None, ws=None,
                 stream=None):
    """sa_topk_dynamic: per row, the fewest tokens in top-k order whose scores
    reach tau of the row's total, at most k_max.  Returns (idx [Nq, k_max]
    ascending then -1, counts [Nq])."""
    Nq, ld = scores.shape
    _rows_out(scores, Nq, n_max, "scores")
    _out(n_valid, (Nq,), (torch.int32,), "n_valid")
    if idx is None:
        idx = torch.empty((Nq, k_max), dtype=torch.int32, device=scores.device)
    _out(idx, (Nq, k_max), (torch.int32,), "idx")
    if counts is None:
        counts = torch.empty((Nq,), dtype=torch.int32, device=scores.device)
    _out(counts, (Nq,), (torch.int32,), "counts")
    if ws is None:
        ws = workspace(lib().sa_topk_dynamic_workspace_size(Nq, n_max, k_max), scores.device)
    _ws(ws)
    _check(lib().sa_topk_dynamic(_ptr(scores), ld, _ptr(n_valid), Nq, n_max, k_max, float(tau), _ptr(idx),
                                 _ptr(counts), _ptr(ws), ws.numel(), _stream(stream)))
    return idx, counts


def sparse_decode_attn_workspace_size(L_g, B, Hq, Hkv, d, k) -> int:
    return int(lib().sa_sparse_decode_attn_workspace_size(L_g, B, Hq, Hkv, d, k))


def sparse_decode_attn(Q, K, V, seq_off, seq_len, idx, Hkv: int, scale: float, out_dtype=torch.bfloat16, O=None,
                       ws=None, stream=None) -> torch.Tensor:
    """K, V: packed caches of n_tokens * Hkv rows of d (n_tokens = sum of seq_len)."""
    L, B, Hq, d = Q.shape
    k = idx.shape[1]
    n_tokens = K.numel() // (Hkv * d)
    _dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), _dev(V, torch.bfloat16, "V")
    _out(idx, (B, k), (torch.int32,), "idx")
    _seqs(seq_off, seq_len, B)
    if O is None:
        O = torch.empty((L, B, Hq, d), dtype=out_dtype, device=Q.device)
    _out(O, (L, B, Hq, d), (torch.bfloat16, torch.float32), "O")
    if ws is None:
        ws = workspace(sparse_decode_attn_workspace_size(L, B, Hq, Hkv, d, k), Q.device)
    _ws(ws)
    code = SA_F32 if O.dtype == torch.float32 else SA_BF16
    _check(lib().sa_sparse_decode_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(seq_off), _ptr(seq_len), _ptr(idx), L, B,
                                       n_tokens, Hq, Hkv, d, k, float(scale), _ptr(O), code, _ptr(ws), ws.numel(),
                                       _stream(stream)))
    return O


def sparse_decode_attn_partial(Q, K, V, seq_off, seq_len, idx, Hkv: int, scale: float, O_part=None, ml=None,
                                idx_count=None, ws=None, stream=None):
    """sparse_decode_attn left unnormalised: O_part fp32 [L, B, Hq, d] and ml
    fp32 [L, B, Hq, 2], (m, l) with m a reference logit in log2 units (within
    8 of the row's max) and l the sum of 2^(logit - m); O_part / l is the
    output.  idx_count int32 [B] (optional): only the first idx_count[b]
    entries of idx row b are real."""
    L, B, Hq, d = Q.shape
    k = idx.shape[1]
    n_tokens = K.numel() // (Hkv * d)
    _dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), _dev(V, torch.bfloat16, "V")
    _out(idx, (B, k), (torch.int32,), "idx")
    if idx_count is not None:
        _out(idx_count, (B,), (torch.int32,), "idx_count")
    _seqs(seq_off, seq_len, B)
    if O_part is None:
        O_part = torch.empty((L, B, Hq, d), dtype=torch.float32, device=Q.device)
    if ml is None:
        ml = torch.empty((L, B, Hq, 2), dtype=torch.float32, device=Q.device)
    _out(O_part, (L, B, Hq, d), (torch.float32,), "O_part")
    _out(ml, (L, B, Hq, 2), (torch.float32,), "ml")
    if ws is None:
        ws = workspace(sparse_decode_attn_workspace_size(L, B, Hq, Hkv, d, k), Q.device)
    _ws(ws)
    _check(lib().sa_sparse_decode_attn_partial(_ptr(Q), _ptr(K), _ptr(V), _ptr(seq_off), _ptr(seq_len), _ptr(idx),
                                               L, B, n_tokens, Hq, Hkv, d, k, _ptr(idx_count), float(scale),
                                               _ptr(O_part), _ptr(ml), _ptr(ws), ws.numel(), _stream(stream)))
    return O_part, ml


def cp_select_workspace_size(N, B, k) -> int:
    return int(lib().sa_cp_select_workspace_size(N, B, k))


def cp_select(cand_scores, cand_idx, rank: int, local_idx=None, local_count=None, ws=None,
              stream=None) -> torch.Tensor:
    """Global top-k of N ranks' candidates, as `rank`'s local indices [B, k]
    (and, into local_count int32 [B] if given, how many there are).

    cand_scores fp32 / cand_idx int32, each [N, B, k] or a view of one
    all-gathered int32 buffer [N, 2, B, k] (scores bit-cast in [:, 0])."""
    N, B, k = cand_idx.shape
    if not (cand_scores.is_cuda and cand_idx.is_cuda and cand_scores.dtype == torch.float32
            and cand_idx.dtype == torch.int32 and tuple(cand_scores.shape) == (N, B, k)):
        raise ValueError("cand_scores fp32 and cand_idx int32 must be CUDA tensors of one shape [N, B, k]")
    stride = cand_idx.stride(0) if N > 1 else B * k
    if (cand_scores.stride(0) != stride and N > 1) or cand_idx.stride()[1:] != (k, 1) \
            or cand_scores.stride()[1:] != (k, 1):
        raise ValueError("cand_scores and cand_idx must be [B, k] blocks of one rank stride")
    if local_idx is None:
        local_idx = torch.empty((B, k), dtype=torch.int32, device=cand_idx.device)
    _out(local_idx, (B, k), (torch.int32,), "local_idx")
    if local_count is not None:
        _out(local_count, (B,), (torch.int32,), "local_count")
    if ws is None:
        ws = workspace(cp_select_workspace_size(N, B, k), cand_idx.device)
    _ws(ws)
    _check(lib().sa_cp_select(_ptr(cand_scores), _ptr(cand_idx), stride, N, B, k, int(rank), _ptr(local_idx),
                              _ptr(local_count), _ptr(ws), ws.numel(), _stream(stream)))
    return local_idx


RADIX_BINS = (4096, 4096, 256)  # histogram bins of the exchange's levels 0, 1, 2


def cp_radix_workspace_size(B: int) -> int:
    return int(lib().sa_cp_radix_workspace_size(B))


def _gathered(gathered, N: int, B: int, bins: int, what: str):
    if gathered is None:
        return None, 0
    if not (gathered.is_cuda and gathered.dtype == torch.int32 and gathered.dim() == 3
            and tuple(gathered.shape) == (N, B, bins) and gathered.stride()[1:] == (bins, 1)):
        raise ValueError(f"{what}: gathered histograms must be int32 CUDA [N, B, {bins}] with [B, {bins}] blocks")
    return gathered, (gathered.stride(0) if N > 1 else B * bins)


def cp_radix_level(scores, n_local, k: int, N: int, level: int, gathered=None, hist_out=None, ws=None,
                   stream=None) -> torch.Tensor:
    """One level of the histogram exchange (levels 0, 1, 2): the previous
    level's threshold from `gathered` (every rank's histograms of it, int32
    [N, B, bins]; None at level 0), then this rank's histogram of the level's
    digit over its scores fp32 [B, ld] (entries [0, n_local[b])).  Returns
    hist_out int32 [B, 4096] (levels 0, 1) or [B, 256] (level 2).  `ws`
    (cp_radix_workspace_size) carries the state across the step's calls."""
    B = n_local.shape[0]
    _rows_out(scores, B, 1, "scores")
    _dev(n_local, torch.int32, "n_local")
    if level not in (0, 1, 2):
        raise ValueError("level must be 0, 1 or 2")
    if (gathered is None) != (level == 0):
        raise ValueError("gathered histograms are needed at levels 1 and 2 only")
    g, stride = _gathered(gathered, N, B, RADIX_BINS[level - 1], "cp_radix_level") if level else (None, 0)
    if hist_out is None:
        hist_out = torch.empty((B, RADIX_BINS[level]), dtype=torch.int32, device=scores.device)
    _out(hist_out, (B, RADIX_BINS[level]), (torch.int32,), "hist_out")
    if ws is None:
        raise ValueError("cp_radix_level needs the step's workspace (it carries the state across levels)")
    _ws(ws)
    _check(lib().sa_cp_radix_level(_ptr(scores), scores.stride(0), _ptr(n_local), B, int(k), int(N), int(level),
                                   _ptr(g), stride, _ptr(hist_out), _ptr(ws), ws.numel(), _stream(stream)))
    return hist_out


def cp_radix_select(scores, n_local, k: int, N: int, rank: int, gathered, local_idx=None, local_count=None, ws=None,
                    stream=None) -> torch.Tensor:
    """The exchange's last call: the level-2 threshold from `gathered`
    (int32 [N, B, 256]), then this rank's entries of the global top-k as
    local indices [B, k] (ascending, -1 padded; their number into
    local_count int32 [B] if given)."""
    B = n_local.shape[0]
    _rows_out(scores, B, 1, "scores")
    _dev(n_local, torch.int32, "n_local")
    g, stride = _gathered(gathered, N, B, RADIX_BINS[2], "cp_radix_select")
    if local_idx is None:
        local_idx = torch.empty((B, k), dtype=torch.int32, device=scores.device)
    _out(local_idx, (B, k), (torch.int32,), "local_idx")
    if local_count is not None:
        _out(local_count, (B,), (torch.int32,), "local_count")
    if ws is None:
        raise ValueError("cp_radix_select needs the step's workspace (it carries the state across levels)")
    _ws(ws)
    _check(lib().sa_cp_radix_select(_ptr(scores), scores.stride(0), _ptr(n_local), B, int(k), int(N), int(rank),
                                    _ptr(g), stride, _ptr(local_idx), _ptr(local_count), _ptr(ws), ws.numel(),
                                    _stream(stream)))
    return local_idx


def combine_partials(O_part, ml, O=None, out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    """Log-sum-exp merge of P partials: O_part fp32 [P, rows, d], ml fp32
    [P, rows, 2] (each part contiguous; the parts may sit at any common
    stride, e.g. views of one all-gathered buffer).  Returns O [rows, d]."""
    P, rows, d = O_part.shape
    if not (O_part.is_cuda and ml.is_cuda and O_part.dtype == torch.float32 and ml.dtype == torch.float32
            and tuple(ml.shape) == (P, rows, 2)):
        raise ValueError("O_part [P, rows, d] and ml [P, rows, 2] must be fp32 CUDA tensors")
    if O_part.stride()[1:] != (d, 1) or ml.stride()[1:] != (2, 1):
        raise ValueError("each part of O_part and ml must be contiguous")
    if O is None:
        O = torch.empty((rows, d), dtype=out_dtype, device=O_part.device)
    _out(O, (rows, d), (torch.bfloat16, torch.float32), "O")
    code = SA_F32 if O.dtype == torch.float32 else SA_BF16
    _check(lib().sa_combine_partials(_ptr(O_part), O_part.stride(0), _ptr(ml), ml.stride(0), P, rows, d, _ptr(O),
                                     code, _stream(stream)))
    return O


def indexer_layer_attn_workspace_size(B, S_max, Hq, Hkv, d) -> int:
    return int(lib().sa_indexer_layer_attn_workspace_size(B, S_max, Hq, Hkv, d))


def indexer_layer_attn(Q, K, V, seq_off, seq_len, S_max: int, Hkv: int, scale: float, out_dtype=torch.bfloat16,
                       O=None, scores=None, ws=None, stream=None):
    """The CLSA indexer layer as full attention whose weights route the index
    (sa_indexer_layer_attn): Q [B, Hq, d] -> (O [B, Hq, d] dense output,
    scores [B, ld] fp32 routing scores, the sum over heads of each token's
    attention weight)."""
    B, Hq, d = Q.shape
    n_tokens = K.numel() // (Hkv * d)
    _dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), _dev(V, torch.bfloat16, "V")
    _seqs(seq_off, seq_len, B)
    if O is None:
        O = torch.empty((B, Hq, d), dtype=out_dtype, device=Q.device)
    _out(O, (B, Hq, d), (torch.bfloat16, torch.float32), "O")
    if scores is None:
        scores = torch.empty((B, max(S_max, 1)), dtype=torch.float32, device=Q.device)
    ld = _rows_out(scores, B, S_max, "scores")
    if ws is None:
        ws = workspace(indexer_layer_attn_workspace_size(B, S_max, Hq, Hkv, d), Q.device)
    _ws(ws)
    code = SA_F32 if O.dtype == torch.float32 else SA_BF16
    _check(lib().sa_indexer_layer_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(seq_off), _ptr(seq_len), B, n_tokens, S_max,
                                       Hq, Hkv, d, float(scale), _ptr(O), code, _ptr(scores), ld,
                                       _ptr(ws), ws.numel(), _stream(stream)))
    return O, scores


def decode_step_attn_route_workspace_size(B, S_max, Hq, Hkv, d, k, L) -> int:
    return max(indexer_layer_attn_workspace_size(B, S_max, Hq, Hkv, d), int(lib().sa_topk_workspace_size(B, S_max, k)),
               int(lib().sa_topk_dynamic_workspace_size(B, S_max, k)),
               sparse_decode_attn_workspace_size(max(L - 1, 1), B, Hq, Hkv, d, k))


def decode_step_attn_route(Q, K, V, seq_off, seq_len, S_max: int, k: int, Hkv: int, scale: float,
                           out_dtype=torch.bfloat16, O=None, idx=None, scores=None, ws=None, stream=None,
                           tau: Optional[float] = None, counts=None):
    """One decode step of a cross-decoder group under the CLSA reading in
    which layer 0 is the indexer layer: it attends densely and its summed
    attention weights give the routing scores; their top-k is the index that
    layers 1..L-1 share over the same cache.  Q [L, B, Hq, d] -> (O, idx).
    With tau, k is dynamic: each sequence keeps the fewest tokens whose
    routing mass reaches tau of its total, at most k (sa_topk_dynamic); the
    index is then -1 padded and (O, idx, counts) is returned."""
    L, B, Hq, d = Q.shape
    if O is None:
        O = torch.empty((L, B, Hq, d), dtype=out_dtype, device=Q.device)
    if ws is None:
        ws = workspace(decode_step_attn_route_workspace_size(B, S_max, Hq, Hkv, d, k, L), Q.device)
    _, scores = indexer_layer_attn(Q[0], K, V, seq_off, seq_len, S_max, Hkv, scale, O=O[0], scores=scores, ws=ws,
                                   stream=stream)
    if tau is None:
        idx = topk(scores, seq_len, S_max, k, idx=idx, ws=ws, stream=stream)
    else:
        idx, counts = topk_dynamic(scores, seq_len, S_max, k, tau, idx=idx, counts=counts, ws=ws, stream=stream)
    if L > 1:
        sparse_decode_attn(Q[1:], K, V, seq_off, seq_len, idx, Hkv, scale, O=O[1:], ws=ws, stream=stream)
    return (O, idx) if tau is None else (O, idx, counts)


def decode_step_workspace_size(n_layers, B, S_max, Hq, Hkv, d, k) -> int:
    return int(lib().sa_decode_step_workspace_size(n_layers, B, S_max, Hq, Hkv, d, k))


def _ptr_arrays(lists: Sequence[Sequence[Optional[torch.Tensor]]]):
    """Host arrays of device pointers (NULL for None), one per list, in one
    buffer: returns the buffer (keep it alive across the call) and the
    address of each array.  A tensor listed many times is asked for its
    address once."""
    memo = {}
    vals = []
    for lst in lists:
        for t in lst:
            if t is None:
                vals.append(0)
            else:
                p = memo.get(id(t))
                if p is None:
                    p = memo[id(t)] = t.data_ptr()
                vals.append(p)
    buf = array.array("Q", vals)
    base = buf.buffer_info()[0]
    addrs = []
    off = 0
    for lst in lists:
        addrs.append(base + 8 * off)
        off += len(lst)
    return buf, addrs


STEP_PER_LAYER = 1


def decode_step(pattern: str, qI: Sequence, w: Sequence, KI: Sequence, K: Sequence, V: Sequence, seq_off, seq_len,
                S_max: int, k: int, Q, Hkv: int, scale: float, out_dtype=torch.bfloat16, O=None, idx=None,
                scores=None, ws=None, stream=None, new_KI: Optional[Sequence] = None,
                new_K: Optional[Sequence] = None, new_V: Optional[Sequence] = None, per_layer: bool = False):
    """One decode step over `pattern` (per-layer lists; entries of S layers'
    indexer inputs may be None).  With new_KI (and new_K / new_V) per layer,
    the new token's rows are written into the caches first (sa_decode_step_ex);
    per_layer runs one attention launch per layer.  Returns (O, idx of the
    last F layer)."""
    L, B, Hq, d = Q.shape
    n = len(pattern)
    assert L == n and len(K) == n and len(V) == n
    f0 = next(t for t in qI if t is not None)
    H_I, d_I = f0.shape[1], f0.shape[2]
    n_tokens = next(t for t in KI if t is not None).shape[0]
    _dev(Q, torch.bfloat16, "Q")
    _seqs(seq_off, seq_len, B)
    if O is None:
        O = torch.empty((L, B, Hq, d), dtype=out_dtype, device=Q.device)
    _out(O, (L, B, Hq, d), (torch.bfloat16, torch.float32), "O")
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=Q.device)
    _out(idx, (B, k), (torch.int32,), "idx")
    if scores is None:
        scores = torch.empty((B, max(S_max, 1)), dtype=torch.float32, device=Q.device)
    _rows_out(scores, B, S_max, "scores")
    if ws is None:
        ws = workspace(decode_step_workspace_size(n, B, S_max, Hq, Hkv, d, k), Q.device)
    _ws(ws)
    code = SA_F32 if O.dtype == torch.float32 else SA_BF16
    if new_KI is None and new_K is None and not per_layer:
        buf, arrays = _ptr_arrays((qI, w, KI, K, V))
        _check(lib().sa_decode_step(pattern.encode(), n, *arrays, seq_off.data_ptr(), seq_len.data_ptr(), B,
                                    n_tokens, S_max, H_I, d_I, k, Q.data_ptr(), Hq, Hkv, d, float(scale),
                                    O.data_ptr(), code, idx.data_ptr(), scores.data_ptr(), scores.shape[1],
                                    ws.data_ptr(), ws.numel(), _stream(stream)))
        return O, idx
    extra_lists = [lst for lst in (new_KI, new_K, new_V) if lst is not None]
    buf, arrays = _ptr_arrays([qI, w, KI, K, V] + extra_lists)
    it = iter(arrays[5:])
    extra = [None if lst is None else next(it) for lst in (new_KI, new_K, new_V)]
    _check(lib().sa_decode_step_ex(pattern.encode(), n, *arrays[:5], *extra, seq_off.data_ptr(), seq_len.data_ptr(),
                                   B, n_tokens, S_max, H_I, d_I, k, Q.data_ptr(), Hq, Hkv, d, float(scale),
                                   O.data_ptr(), code, idx.data_ptr(), scores.data_ptr(), scores.shape[1],
                                   STEP_PER_LAYER if per_layer else 0, ws.data_ptr(), ws.numel(),
                                   _stream(stream)))
    return O, idx


class DecodeStepPlan:
    """sa_decode_step prepared once for tensors a decode loop reuses every
    step (caches, query buffers, outputs, workspace): the arguments are
    checked and marshalled here, and run() makes only the C call.  The plan
    holds the tensors it points to; build a new plan if any of them is
    replaced by another allocation."""

    def __init__(self, pattern: str, qI: Sequence, w: Sequence, KI: Sequence, K: Sequence, V: Sequence, seq_off,
                 seq_len, S_max: int, k: int, Q, Hkv: int, scale: float, out_dtype=torch.bfloat16, O=None, idx=None,
                 scores=None, ws=None):
        L, B, Hq, d = Q.shape
        n = len(pattern)
        if not (L == n and len(qI) == n and len(w) == n and len(KI) == n and len(K) == n and len(V) == n):
            raise ValueError("every per-layer list and Q must have one entry per pattern letter")
        f0 = next(t for t in qI if t is not None)
        H_I, d_I = f0.shape[1], f0.shape[2]
        n_tokens = next(t for t in KI if t is not None).shape[0]
        _dev(Q, torch.bfloat16, "Q")
        _seqs(seq_off, seq_len, B)
        if O is None:
            O = torch.empty((L, B, Hq, d), dtype=out_dtype, device=Q.device)
        _out(O, (L, B, Hq, d), (torch.bfloat16, torch.float32), "O")
        if idx is None:
            idx = torch.empty((B, k), dtype=torch.int32, device=Q.device)
        _out(idx, (B, k), (torch.int32,), "idx")
        if scores is None:
            scores = torch.empty((B, max(S_max, 1)), dtype=torch.float32, device=Q.device)
        _rows_out(scores, B, S_max, "scores")
        if ws is None:
            ws = workspace(decode_step_workspace_size(n, B, S_max, Hq, Hkv, d, k), Q.device)
        _ws(ws)
        self.O, self.idx, self.scores, self.ws = O, idx, scores, ws
        self._hold = (qI, w, KI, K, V, seq_off, seq_len, Q)
        self._buf, arrays = _ptr_arrays((qI, w, KI, K, V))
        code = SA_F32 if O.dtype == torch.float32 else SA_BF16
        self._args = (pattern.encode(), n, *arrays, seq_off.data_ptr(), seq_len.data_ptr(), B, n_tokens, S_max, H_I,
                      d_I, k, Q.data_ptr(), Hq, Hkv, d, float(scale), O.data_ptr(), code, idx.data_ptr(),
                      scores.data_ptr(), scores.shape[1], ws.data_ptr(), ws.numel())
        self._fn = lib().sa_decode_step

    def run(self, stream=None):
        """Enqueue the step on `stream` (default: the current stream); returns (O, idx)."""
        _check(self._fn(*self._args, _stream(stream)))
        return self.O, self.idx


def block_union_prefill(idx, q_pos, Q, K, V, block: int, scale: float, out_dtype=torch.bfloat16, O=None,
                        kv_indptr=None, kv_indices=None, ws=None, stream=None):
    """Returns (kv_indptr [Hkv+1], kv_indices [Hkv*ceil(S/block)], O [Nq,Hq,d])."""
    Nq, Hq, d = Q.shape
    Hkv, S, _ = K.shape
    k = idx.shape[1]
    _out(idx, (Nq, k), (torch.int32,), "idx"), _out(q_pos, (Nq,), (torch.int32,), "q_pos")
    _dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), _dev(V, torch.bfloat16, "V")
    nb = (S + block - 1) // block
    if kv_indptr is None:
        kv_indptr = torch.empty(Hkv + 1, dtype=torch.int32, device=Q.device)
    _out(kv_indptr, (Hkv + 1,), (torch.int32,), "kv_indptr")
    if kv_indices is None:
        kv_indices = torch.empty(Hkv * nb, dtype=torch.int32, device=Q.device)
    _out(kv_indices, (Hkv * nb,), (torch.int32,), "kv_indices")
    if O is None:
        O = torch.empty((Nq, Hq, d), dtype=out_dtype, device=Q.device)
    _out(O, (Nq, Hq, d), (torch.bfloat16, torch.float32), "O")
    if ws is None:
        ws = workspace(lib().sa_block_union_prefill_workspace_size(S, Nq, Hq, Hkv, d, k, block), Q.device)
    _ws(ws)
    code = SA_F32 if O.dtype == torch.float32 else SA_BF16
    _check(lib().sa_block_union_prefill(_ptr(idx), _ptr(q_pos), _ptr(Q), _ptr(K), _ptr(V), S, Nq, Hq, Hkv, d, k,
                                        block, float(scale), _ptr(kv_indptr), _ptr(kv_indices), _ptr(O), code,
                                        _ptr(ws), ws.numel(), _stream(stream)))
    return kv_indptr, kv_indices, O


def kap_order_workspace_size() -> int:
    return int(lib().sa_kap_order_workspace_size())


def osk_prefill_workspace_size(S, Nq, Hq, Hkv, d, k, block) -> int:
    return int(lib().sa_osk_prefill_workspace_size(S, Nq, Hq, Hkv, d, k, block))


def kap_order(idx, S: int, block: int, q_block: int, kv_indptr, kv_indices, order=None, ws=None, stream=None):
    """sa_kap_order: the union table ordered per query block of q_block
    queries by hit count (larger first, ties by ascending block id).
    Returns order [ceil(Nq/q_block), ceil(S/block)] int32; row i's first
    kv_indptr[1] - kv_indptr[0] entries are written."""
    Nq, k = idx.shape
    _out(idx, (Nq, k), (torch.int32,), "idx")
    nb = (S + block - 1) // block
    n_qb = (Nq + q_block - 1) // q_block
    _out(kv_indptr, (kv_indptr.numel(),), (torch.int32,), "kv_indptr")
    _out(kv_indices, (kv_indices.numel(),), (torch.int32,), "kv_indices")
    if order is None:
        order = torch.empty((n_qb, nb), dtype=torch.int32, device=idx.device)
    _out(order, (n_qb, nb), (torch.int32,), "order")
    if ws is None:
        ws = workspace(lib().sa_kap_order_workspace_size(), idx.device)
    _ws(ws)
    _check(lib().sa_kap_order(_ptr(idx), Nq, k, S, block, q_block, _ptr(kv_indptr), _ptr(kv_indices), _ptr(order),
                              nb, _ptr(ws), ws.numel(), _stream(stream)))
    return order


def osk_prefill(idx, q_pos, Q, K, V, block: int, scale: float, tau: float, out_dtype=torch.bfloat16, O=None,
                kv_indptr=None, kv_indices=None, order=None, steps=None, ws=None, stream=None):
    """sa_osk_prefill: block union, priority lists (one per query block of
    128 / (Hq/Hkv) queries) and ordered-skipping attention with threshold
    tau.  Returns (kv_indptr, kv_indices, order [n_qb, ceil(S/block)],
    steps [Hkv * n_qb] (tiles of two blocks run per unit g * n_qb + i),
    O [Nq,Hq,d])."""
    Nq, Hq, d = Q.shape
    Hkv, S, _ = K.shape
    k = idx.shape[1]
    _out(idx, (Nq, k), (torch.int32,), "idx"), _out(q_pos, (Nq,), (torch.int32,), "q_pos")
    _dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), _dev(V, torch.bfloat16, "V")
    nb = (S + block - 1) // block
    G = Hq // Hkv
    n_qb = (Nq * G + 127) // 128
    dev = Q.device
    if kv_indptr is None:
        kv_indptr = torch.empty(Hkv + 1, dtype=torch.int32, device=dev)
    _out(kv_indptr, (Hkv + 1,), (torch.int32,), "kv_indptr")
    if kv_indices is None:
        kv_indices = torch.empty(Hkv * nb, dtype=torch.int32, device=dev)
    _out(kv_indices, (Hkv * nb,), (torch.int32,), "kv_indices")
    if order is None:
        order = torch.empty((n_qb, nb), dtype=torch.int32, device=dev)
    _out(order, (n_qb, nb), (torch.int32,), "order")
    if steps is None:
        steps = torch.empty(Hkv * n_qb, dtype=torch.int32, device=dev)
    _out(steps, (Hkv * n_qb,), (torch.int32,), "steps")
    if O is None:
        O = torch.empty((Nq, Hq, d), dtype=out_dtype, device=dev)
    _out(O, (Nq, Hq, d), (torch.bfloat16, torch.float32), "O")
    if ws is None:
        ws = workspace(lib().sa_osk_prefill_workspace_size(S, Nq, Hq, Hkv, d, k, block), dev)
    _ws(ws)
    code = SA_F32 if O.dtype == torch.float32 else SA_BF16
    _check(lib().sa_osk_prefill(_ptr(idx), _ptr(q_pos), _ptr(Q), _ptr(K), _ptr(V), S, Nq, Hq, Hkv, d, k, block,
                                float(scale), float(tau), _ptr(kv_indptr), _ptr(kv_indices), _ptr(order), _ptr(steps),
                                _ptr(O), code, _ptr(ws), ws.numel(), _stream(stream)))
    return kv_indptr, kv_indices, order, steps, O


def block_union_prefill_noalloc(idx, q_pos, Q, K, V, block: int, scale: float, kv_indptr, kv_indices, O,
                                stream=None):
    """sa_block_union_prefill_noalloc: the same result as block_union_prefill
    without a workspace, for callers that cannot allocate device memory around
    the call (outputs are passed in).  Its scratch is a fixed array inside
    libsa; calls that can overlap on the GPU must not be issued together."""
    Nq, Hq, d = Q.shape
    Hkv, S, _ = K.shape
    k = idx.shape[1]
    _out(idx, (Nq, k), (torch.int32,), "idx"), _out(q_pos, (Nq,), (torch.int32,), "q_pos")
    _dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), _dev(V, torch.bfloat16, "V")
    nb = (S + block - 1) // block
    _out(kv_indptr, (Hkv + 1,), (torch.int32,), "kv_indptr")
    _out(kv_indices, (Hkv * nb,), (torch.int32,), "kv_indices")
    _out(O, (Nq, Hq, d), (torch.bfloat16, torch.float32), "O")
    code = SA_F32 if O.dtype == torch.float32 else SA_BF16
    _check(lib().sa_block_union_prefill_noalloc(_ptr(idx), _ptr(q_pos), _ptr(Q), _ptr(K), _ptr(V), S, Nq, Hq, Hkv,
                                                d, k, block, float(scale), _ptr(kv_indptr), _ptr(kv_indices),
                                                _ptr(O), code, _stream(stream)))
    return kv_indptr, kv_indices, O
