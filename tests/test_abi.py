"""libsa loads on a machine without a GPU, exports every symbol include/sa.h
declares, and rejects bad arguments on the host (no device call needed)."""
import ctypes
import os
import re

import pytest

import cross_layer_shared_b200 as sa
from cross_layer_shared_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sa.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return sa.lib()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_path_entry_points():
    names = declared_symbols()
    for n in ("sa_index_score", "sa_topk", "sa_sparse_decode_attn", "sa_block_union_prefill", "sa_decode_step"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in sa.SIGNATURES, f"binding lacks {name}"


def test_status_strings_and_version(lib):
    assert lib.sa_abi_version() == 1
    assert lib.sa_status_string(0) == b"SA_OK"
    assert lib.sa_status_string(5) == b"SA_ERR_TIMEOUT"


FAKE = ctypes.c_void_p(0x7F0000001000)  # never dereferenced: validation fails first
FAKE_WS = ctypes.c_void_p(0x7F0000002000)


def test_topk_rejects_bad_k_and_missing_workspace(lib):
    rc = lib.sa_topk(FAKE, 100, FAKE, 2, 100, 0, FAKE, None, FAKE_WS, 4096, None)
    assert rc == sa.SA_ERR_INVALID_ARG and b"k=0" in lib.sa_last_error()
    rc = lib.sa_topk(FAKE, 100, FAKE, 2, 100, 8, FAKE, None, None, 0, None)
    assert rc == sa.SA_ERR_WORKSPACE
    rc = lib.sa_topk(FAKE, 100, FAKE, 2, 100, 8, FAKE, None, ctypes.c_void_p(0x7F0000002010), 4096, None)
    assert rc == sa.SA_ERR_WORKSPACE and b"aligned" in lib.sa_last_error()
    rc = lib.sa_topk(FAKE, 50, FAKE, 2, 100, 8, FAKE, None, FAKE_WS, 4096, None)
    assert rc == sa.SA_ERR_INVALID_ARG  # ld below n_max


def test_index_score_rejects_unsupported_shapes(lib):
    rc = lib.sa_index_score(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 100, 100, 65, 128, FAKE, 100, FAKE_WS, 4096, None)
    assert rc == sa.SA_ERR_UNSUPPORTED
    rc = lib.sa_index_score(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 100, 100, 16, 96, FAKE, 100, FAKE_WS, 4096, None)
    assert rc == sa.SA_ERR_UNSUPPORTED
    rc = lib.sa_index_score(ctypes.c_void_p(0x7F0000001002), FAKE, FAKE, FAKE, FAKE, 1, 100, 100, 16, 128, FAKE,
                            100, FAKE_WS, 4096, None)
    assert rc == sa.SA_ERR_INVALID_ARG and b"aligned" in lib.sa_last_error()


def test_attention_rejects_bad_head_counts(lib):
    rc = lib.sa_sparse_decode_attn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 1, 4096, 30, 4, 128, 256, 0.088, FAKE, 0,
                                   FAKE_WS, 1 << 20, None)
    assert rc == sa.SA_ERR_INVALID_ARG and b"multiple" in lib.sa_last_error()
    rc = lib.sa_sparse_decode_attn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 1, 4096, 32, 4, 64, 256, 0.125, FAKE, 0,
                                   FAKE_WS, 1 << 20, None)
    assert rc == sa.SA_ERR_UNSUPPORTED


def test_decode_step_pattern_must_start_with_full_layer(lib):
    arr = (ctypes.c_void_p * 4)(*([0x7F0000001000] * 4))
    pp = ctypes.cast(arr, sa._PP)
    for pat, want in ((b"SFSS", b"first layer must be F"), (b"FSXS", b"F or S")):
        rc = lib.sa_decode_step(pat, 4, pp, pp, pp, pp, pp, FAKE, FAKE, 1, 4096, 4096, 4, 64, 256, FAKE, 8, 1, 128,
                                0.088, FAKE, 0, FAKE, FAKE, 4096, FAKE_WS, 1 << 24, None)
        assert rc == sa.SA_ERR_INVALID_ARG and want in lib.sa_last_error()


def test_block_union_rejects_other_block_sizes(lib):
    rc = lib.sa_block_union_prefill(FAKE, FAKE, FAKE, FAKE, FAKE, 4096, 16, 8, 2, 128, 64, 32, 0.088, FAKE, FAKE,
                                    FAKE, 0, FAKE_WS, 1 << 20, None)
    assert rc == sa.SA_ERR_UNSUPPORTED


def test_workspace_sizes_are_host_computable(lib):
    assert lib.sa_topk_workspace_size(4, 131072, 2048) >= sa.WS_HEADER_BYTES
    w1 = lib.sa_sparse_decode_attn_workspace_size(24, 4, 32, 8, 128, 2048)
    assert w1 >= sa.WS_HEADER_BYTES
    assert lib.sa_decode_step_workspace_size(24, 4, 131072, 32, 8, 128, 2048) >= w1


def test_decode_step_ex_rejects_bad_append_requests(lib):
    arr = (ctypes.c_void_p * 4)(*([0x7F0000001000] * 4))
    pp = ctypes.cast(arr, sa._PP)
    other = (ctypes.c_void_p * 4)(0x7F0000001000, 0x7F0000003000, 0x7F0000001000, 0x7F0000001000)
    po = ctypes.cast(other, sa._PP)

    def call(K, new_KI, new_K, new_V, flags=0):
        return lib.sa_decode_step_ex(b"FSSS", 4, pp, pp, pp, K, pp, new_KI, new_K, new_V, FAKE, FAKE, 1, 4096, 4096, 4,
                                     64, 256, FAKE, 8, 1, 128, 0.088, FAKE, 0, FAKE, FAKE, 4096, flags, FAKE_WS,
                                     1 << 24, None)
    assert call(pp, pp, pp, None) == sa.SA_ERR_INVALID_ARG and b"together" in lib.sa_last_error()
    assert call(pp, None, pp, pp) == sa.SA_ERR_INVALID_ARG and b"new_KI" in lib.sa_last_error()
    assert call(po, pp, pp, pp) == sa.SA_ERR_UNSUPPORTED and b"F layer" in lib.sa_last_error()
    assert call(pp, None, None, None, flags=4) == sa.SA_ERR_INVALID_ARG and b"flags" in lib.sa_last_error()


def test_indexer_layer_attn_rejects_bad_requests(lib):
    need = lib.sa_indexer_layer_attn_workspace_size(4, 131072, 32, 8, 128)
    # logits of every head and token, plus the partial results
    assert need >= sa.WS_HEADER_BYTES + 4 * 32 * 131072 * 4

    def call(Hq=32, Hkv=8, d=128, ld=4096, ws_bytes=1 << 30, S_max=4096, Q=FAKE):
        return lib.sa_indexer_layer_attn(Q, FAKE, FAKE, FAKE, FAKE, 2, 8192, S_max, Hq, Hkv, d, 0.088, FAKE, 0,
                                         FAKE, ld, FAKE_WS, ws_bytes, None)

    assert call(Hq=24, Hkv=8) == sa.SA_ERR_UNSUPPORTED and b"{1, 2, 4, 8}" in lib.sa_last_error()
    assert call(Hq=30, Hkv=8) == sa.SA_ERR_INVALID_ARG
    assert call(d=64) == sa.SA_ERR_UNSUPPORTED
    assert call(ld=100) == sa.SA_ERR_INVALID_ARG and b"ld" in lib.sa_last_error()
    assert call(ws_bytes=1024) == sa.SA_ERR_WORKSPACE
    assert call(Q=ctypes.c_void_p(0x7F0000001008)) == sa.SA_ERR_INVALID_ARG


def test_context_parallel_entry_points_reject_bad_requests(lib):
    B, k = 4, 2048
    need = lib.sa_cp_select_workspace_size(8, B, k)
    # the gathered rows of scores, their counts and the selected positions
    assert need >= sa.WS_HEADER_BYTES + 4 * B * 8 * k + 4 * B + 4 * B * k

    def select(N=2, rank=0, stride=B * k, ws_bytes=1 << 30):
        return lib.sa_cp_select(FAKE, FAKE, stride, N, B, k, rank, FAKE, None, FAKE_WS, ws_bytes, None)

    assert select(rank=2) == sa.SA_ERR_INVALID_ARG and b"rank" in lib.sa_last_error()
    assert select(rank=-1) == sa.SA_ERR_INVALID_ARG
    assert select(N=0) == sa.SA_ERR_INVALID_ARG
    assert select(stride=B * k - 1) == sa.SA_ERR_INVALID_ARG and b"cand_stride" in lib.sa_last_error()
    assert select(ws_bytes=1024) == sa.SA_ERR_WORKSPACE

    rows = 96

    def combine(P=2, d=128, o_stride=rows * 130, ml_stride=rows * 130, ml=FAKE, dtype=sa.SA_BF16, n=rows):
        return lib.sa_combine_partials(FAKE, o_stride, ml, ml_stride, P, n, d, FAKE, dtype, None)

    assert combine(d=64) == sa.SA_ERR_UNSUPPORTED
    assert combine(P=0) == sa.SA_ERR_INVALID_ARG
    assert combine(dtype=7) == sa.SA_ERR_INVALID_ARG
    assert combine(o_stride=rows * 128 - 4) == sa.SA_ERR_INVALID_ARG
    assert combine(o_stride=rows * 130 + 2) == sa.SA_ERR_INVALID_ARG
    assert combine(ml_stride=rows * 130 + 1) == sa.SA_ERR_INVALID_ARG
    assert combine(ml=ctypes.c_void_p(0x7F0000001004)) == sa.SA_ERR_INVALID_ARG
    assert combine(n=0) == sa.SA_OK  # nothing to merge: no launch

    def partial(ml=FAKE, d=128):
        return lib.sa_sparse_decode_attn_partial(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 8192, 32, 8, d, 64, None,
                                                 0.088, FAKE, ml, FAKE_WS, 1 << 30, None)

    assert partial(ml=None) == sa.SA_ERR_INVALID_ARG and b"ml" in lib.sa_last_error()
    assert partial(ml=ctypes.c_void_p(0x7F0000001004)) == sa.SA_ERR_INVALID_ARG
    assert partial(d=64) == sa.SA_ERR_UNSUPPORTED


def test_wait_probe_checks_its_arguments_before_any_launch(lib):
    fake = ctypes.c_void_p(0x7F0000001000)
    assert lib.sa_wait_probe(fake, 256, 10, None) == sa.SA_ERR_INVALID_ARG  # limit below 1 us
    assert lib.sa_wait_probe(fake, 256, 2_000_000_000, None) == sa.SA_ERR_INVALID_ARG  # above 1 s
    assert lib.sa_wait_probe(None, 256, 2_000_000, None) == sa.SA_ERR_WORKSPACE
    assert lib.sa_wait_probe(fake, 64, 2_000_000, None) == sa.SA_ERR_WORKSPACE


def test_ordered_skipping_entry_points_reject_bad_requests(lib):
    """sa_kap_order / sa_osk_prefill check their arguments before any launch."""
    # the proxy: query blocks of at least one query, ld covering every KV block,
    # and at most 16384 KV blocks
    ws = lib.sa_kap_order_workspace_size()
    assert ws == sa.WS_HEADER_BYTES
    assert lib.sa_kap_order(FAKE, 64, 32, 4096, 64, 0, FAKE, FAKE, FAKE, 64, FAKE_WS, ws, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_kap_order(FAKE, 64, 32, 4096, 64, 32, FAKE, FAKE, FAKE, 63, FAKE_WS, ws, None) == sa.SA_ERR_INVALID_ARG
    assert b"ld=63" in lib.sa_last_error()
    assert lib.sa_kap_order(FAKE, 64, 32, 64 * 16385, 64, 32, FAKE, FAKE, FAKE, 16385, FAKE_WS, ws,
                            None) == sa.SA_ERR_UNSUPPORTED
    assert lib.sa_kap_order(FAKE, 64, 32, 4096, 64, 32, None, FAKE, FAKE, 64, FAKE_WS, ws, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_kap_order(FAKE, 64, 32, 4096, 64, 32, FAKE, FAKE, FAKE, 64, None, ws, None) == sa.SA_ERR_WORKSPACE

    wsz = lib.sa_osk_prefill_workspace_size(4096, 64, 32, 8, 128, 32, 64)
    assert wsz == lib.sa_block_union_prefill_workspace_size(4096, 64, 32, 8, 128, 32, 64)

    def osk(S=4096, Hq=32, Hkv=8, d=128, block=64, tau=1e-3, steps=FAKE, ws_=FAKE_WS):
        return lib.sa_osk_prefill(FAKE, FAKE, FAKE, FAKE, FAKE, S, 64, Hq, Hkv, d, 32, block, 0.088, tau, FAKE, FAKE,
                                  FAKE, steps, FAKE, 0, ws_, 1 << 20, None)

    assert osk(d=64) == sa.SA_ERR_UNSUPPORTED
    assert osk(block=32) == sa.SA_ERR_UNSUPPORTED
    assert osk(Hq=24, Hkv=8) == sa.SA_ERR_UNSUPPORTED and b"divide 128" in lib.sa_last_error()  # G = 3
    assert osk(Hq=30, Hkv=8) == sa.SA_ERR_INVALID_ARG  # Hq not a multiple of Hkv
    assert osk(S=64 * 16385) == sa.SA_ERR_UNSUPPORTED
    assert osk(tau=-0.5) == sa.SA_ERR_INVALID_ARG and b"tau" in lib.sa_last_error()
    assert osk(tau=float("nan")) == sa.SA_ERR_INVALID_ARG
    assert osk(tau=float("inf")) == sa.SA_ERR_INVALID_ARG
    assert osk(steps=None) == sa.SA_ERR_INVALID_ARG
    assert osk(ws_=None) == sa.SA_ERR_WORKSPACE
