"""sa_block_union_prefill_noalloc against sa_block_union_prefill.

The no-workspace entry point is for callers that cannot allocate device
memory around the call (inside a CUDA graph capture, or in a runtime that
has no device allocator to hand).  Its scratch is a fixed array inside
libsa, shared by every call, so these tests make two calls in a row with
different selections: each must match the workspace entry point on the same
inputs (block table exactly, outputs within the attention tolerance), which
also shows the second call does not see the first call's leftovers.  One
case makes the first call carry an out-of-range entry (recorded in the
shared array, then skipped) before a valid call; another repeats the two
calls in a fresh Python process, where the first call on the device is also
the one that looks up the array's address.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import cross_layer_shared_b200 as sa
import synth
from cross_layer_shared_b200 import build
from synth import gpu as sgpu
from tests import parity

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _selection(cfg, seed, dev):
    rng = np.random.default_rng(seed)
    idx = np.full((cfg.chunk, cfg.k), -1, np.int32)
    for i, p in enumerate(cfg.q_pos):
        n = min(cfg.k, int(p) + 1)
        idx[i, :n] = np.sort(rng.choice(int(p) + 1, n, replace=False))
    return torch.from_numpy(idx).to(dev)


def two_calls(out_dtype, bad_first=False):
    """Two no-alloc calls in a row, each against the workspace entry point on
    the same inputs.  With bad_first, the first call's selection holds an
    entry past the context (skipped by both entry points)."""
    build.build()
    dev = torch.device("cuda")
    cfg = synth.PrefillConfig("noalloc", S=8192, chunk=256, H_I=16, d_I=128, k=192, block=64, Hq=8, Hkv=2, d=128,
                              seed=91, hot_regions=4, region_len=128)
    wl = sgpu.prefill_workload(cfg, dev)
    nb = (cfg.S + cfg.block - 1) // cfg.block
    tol = parity.ATOL_F32 if out_dtype == torch.float32 else parity.ATOL_BF16
    for call, seed in enumerate((5, 6)):
        idx = _selection(cfg, seed, dev)
        if bad_first and call == 0:
            idx[3, 0] = cfg.S + 100  # out of range: reported into the scratch's status block and skipped
        want_ptr, want_ind, want_O = sa.block_union_prefill(idx, wl["q_pos"], wl["Q"], wl["K"], wl["V"], cfg.block,
                                                            cfg.scale, out_dtype=out_dtype)
        ptr = torch.full((cfg.Hkv + 1,), -7, dtype=torch.int32, device=dev)
        ind = torch.full((cfg.Hkv * nb,), -7, dtype=torch.int32, device=dev)
        O = torch.full((cfg.chunk, cfg.Hq, cfg.d), float("nan"), dtype=out_dtype, device=dev)
        sa.block_union_prefill_noalloc(idx, wl["q_pos"], wl["Q"], wl["K"], wl["V"], cfg.block, cfg.scale, ptr, ind, O)
        torch.cuda.synchronize()
        assert torch.equal(ptr, want_ptr), f"call {call}: kv_indptr differs"
        n = int(want_ptr[-1])
        assert torch.equal(ind[:n], want_ind[:n]), f"call {call}: kv_indices differ"
        err = (O.float() - want_O.float()).abs().max().item()
        assert err <= tol, f"call {call}: outputs differ by {err}"


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_workspace_entry_point_twice(out_dtype):
    two_calls(out_dtype)


def test_noalloc_valid_call_after_one_with_an_out_of_range_entry():
    two_calls(torch.float32, bad_first=True)


def test_noalloc_twice_in_a_fresh_process():
    code = "import torch; from tests.test_zz_no_alloc import two_calls; two_calls(torch.float32); print('ok')"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]


def test_noalloc_rejects_contexts_beyond_its_scratch():
    lib = sa.lib()
    too_long = 32768 * 64 + 1  # one KV block past the static array
    fake = ctypes.c_void_p(0x7F0000001000)
    rc = lib.sa_block_union_prefill_noalloc(fake, fake, fake, fake, fake, too_long, 16, 8, 2, 128, 64, 64, 0.088,
                                            fake, fake, fake, 0, None)
    assert rc == sa.SA_ERR_UNSUPPORTED and b"static scratch" in lib.sa_last_error()
