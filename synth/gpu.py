"""Device-resident synthetic workloads: the bulk tensors are filled on the GPU
by the CUDA twin of the generator (synth/synth.cu), the small ones and the
planted rows are made on the host by synth/__init__.py and copied.  torch is
used for device memory and copies only."""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List

import numpy as np
import torch

import synth

_LIB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsasynth.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB):
            raise RuntimeError(f"{_LIB} missing: run `python -m cross_layer_shared_b200.build`")
        _lib = ctypes.CDLL(_LIB)
        _lib.synth_fill_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint64,
                                                ctypes.c_int64, ctypes.c_float, ctypes.c_void_p]
        _lib.synth_fill_normal_bf16.restype = ctypes.c_int
    return _lib


def fill_normal_bf16(t: torch.Tensor, seed: int, tid: int, scale: float, offset: int = 0) -> torch.Tensor:
    assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    rc = lib().synth_fill_normal_bf16(ctypes.c_void_p(t.data_ptr()), t.numel(), seed, tid, offset, scale,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill_normal_bf16 failed: cudaError {rc}")
    return t


def to_dev_bf16(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def normal_bf16_gpu(n: int, seed: int, tid: int, scale: float, device, offset: int = 0) -> torch.Tensor:
    return fill_normal_bf16(torch.empty(n, dtype=torch.bfloat16, device=device), seed, tid, scale, offset)


def decode_group(cfg: synth.DecodeConfig, g: int, device) -> Dict[str, torch.Tensor]:
    """Indexer inputs and KV cache of group g of a decode workload."""
    tid, sc = cfg.ki_stream(g)
    KI = normal_bf16_gpu(cfg.T * cfg.d_I, cfg.seed, tid, sc, device).view(cfg.T, cfg.d_I)
    tid, sc = cfg.k_stream(g)
    K = normal_bf16_gpu(cfg.T * cfg.Hkv * cfg.d, cfg.seed, tid, sc, device)
    tid, sc = cfg.v_stream(g)
    V = normal_bf16_gpu(cfg.T * cfg.Hkv * cfg.d, cfg.seed, tid, sc, device)
    planted = cfg.planted(g)
    if planted:
        rows = torch.tensor([int(cfg.seq_off[b]) + t for (b, t, _, _) in planted], device=device)
        KI[rows] = to_dev_bf16(np.stack([ki for (_, _, ki, _) in planted]), device)
        for (b, t, _, krow) in planted:
            if krow is None:
                continue
            S = cfg.seq_lens[b]
            for h in range(cfg.Hkv):
                o = int(cfg.seq_off[b]) * cfg.Hkv * cfg.d + (h * S + t) * cfg.d
                K[o:o + cfg.d] = to_dev_bf16(krow[h], device)
    return {
        "KI": KI, "K": K, "V": V,
        "qI": to_dev_bf16(cfg.qI(g), device),
        "w": torch.from_numpy(cfg.w(g)).to(device),
    }


def decode_workload(cfg: synth.DecodeConfig, device="cuda", groups=None) -> Dict:
    groups = range(len(cfg.groups)) if groups is None else groups
    out = {
        "Q": to_dev_bf16(cfg.Q(), device),
        "seq_off": torch.from_numpy(cfg.seq_off).to(device),
        "seq_len": torch.tensor(cfg.seq_lens, dtype=torch.int32, device=device),
        "groups": {g: decode_group(cfg, g, device) for g in groups},
    }
    return out


def prefill_workload(cfg: synth.PrefillConfig, device="cuda") -> Dict[str, torch.Tensor]:
    tid, sc = cfg.ki_stream()
    KI = normal_bf16_gpu(cfg.S * cfg.d_I, cfg.seed, tid, sc, device).view(cfg.S, cfg.d_I)
    tid, sc = cfg.k_stream()
    K = normal_bf16_gpu(cfg.Hkv * cfg.S * cfg.d, cfg.seed, tid, sc, device).view(cfg.Hkv, cfg.S, cfg.d)
    tid, sc = cfg.v_stream()
    V = normal_bf16_gpu(cfg.Hkv * cfg.S * cfg.d, cfg.seed, tid, sc, device).view(cfg.Hkv, cfg.S, cfg.d)
    pos, rows = cfg.hot_ki_rows()
    if pos.size:
        KI[torch.from_numpy(pos).to(device)] = to_dev_bf16(rows, device)
        for h in range(cfg.Hkv):
            p, r = cfg.hot_k_rows(h)
            K[h, torch.from_numpy(p).to(device)] = to_dev_bf16(r, device)
    return {
        "KI": KI, "K": K, "V": V,
        "qI": to_dev_bf16(cfg.qI(), device),
        "w": torch.from_numpy(cfg.w()).to(device),
        "Q": to_dev_bf16(cfg.Q(), device),
        "q_pos": torch.from_numpy(cfg.q_pos).to(device),
    }
