"""Per-phase device timeline of one decode step.

    python -m cross_layer_shared_b200.timeline [workload]              (default c3)
    python -m cross_layer_shared_b200.timeline [workload] --per-layer

The second form runs the step with one attention launch per layer (the
few-rows attention kernel) and reports that kernel's points for the last
layer of the step.

Builds the tracing variant of the library (``-DSA_TIMELINE``: the
``SA_TL`` points of ``csrc/timeline.cuh``, compiled out of ``libsa.so``),
runs the workload's decode step as the benchmark does (CUDA graphs of whole
steps over two input sets, so each traced step follows another), and prints,
for the last step, every point's time across the CTAs of its kernel (min,
median, max, in microseconds from the first indexer CTA's entry).  A point
is stamped by one thread of each CTA: the CTA's entry, the return of
griddepcontrol.wait (the previous kernel complete), phase ends, and exit.

Run it on a machine with a B200; it loads ``libsa_timeline.so`` in place of
``libsa.so`` for this process only.
"""
from __future__ import annotations

import ctypes
import os
import sys

import numpy as np
import torch

from . import build

POINTS = {
    "indexer": {0: "entry", 1: "griddepcontrol.wait returned, tile table built",
                **{2 + b: f"this CTA's last tile of sequence {b}" for b in range(12)},
                14: "this CTA's last tile of sequence >= 12", 15: "exit"},
    "topk": {0: "entry", 1: "griddepcontrol.wait returned", 2: "chunk histogram and bin list built",
             3: "cluster barrier 1", 4: "threshold bin found", 5: "chunk classified, counts pushed",
             6: "cluster barrier 2", 7: "row candidates gathered", 8: "k-th key found (radix refine)",
             9: "offset of this chunk's output", 10: "indices written", 11: "exit"},
    "attention": {0: "entry", 1: "set-up done (barriers, TMEM)", 2: "griddepcontrol.wait returned",
                  **{3 + j: f"tile {j} gathers issued" for j in range(8)},
                  **{12 + j: f"tile {j} scores (QK^T) ready" for j in range(8)},
                  **{20 + j: f"tile {j} softmax done" for j in range(8)},
                  30: "last PV done", 31: "split merge: halves merged, before the cluster wait",
                  32: "split merge: after the cluster wait", 33: "split merge: slices staged and sent",
                  34: "split merge: peers' slices landed", 35: "split merge: rows merged and stored",
                  36: "exit"},
    "attention (few rows)": {0: "entry", 1: "griddepcontrol.wait returned",
                             2: "query staged", 3: "first loads issued",
                             **{4 + p: f"pass {p} scores (S^T) ready" for p in range(4)},
                             **{8 + p: f"pass {p} PV done" for p in range(4)},
                             12: "all warps done", 20: "slice partial written", 13: "slice counted",
                             17: "last slice: fence done", 18: "last slice: partials in shared memory",
                             19: "last slice: row weights", 15: "exit (unsplit, or the last slice after the merge)"},
}
KERNELS = ("indexer", "topk", "attention")


def trace_per_layer(name: str = "c3", steps_per_graph: int = 2):
    """The few-rows attention kernel inside a per-layer step: every point of
    the step's last attention launch (earlier launches write the same slots
    first, so CTAs without a point in the last launch keep an older value:
    only values after the launch's griddepcontrol.wait are that launch's)."""
    import cross_layer_shared_b200 as sa
    import synth
    from synth import gpu as sgpu

    sa.LIB_PATH = build.build_timeline()
    lb = sa.lib()
    setter = lb.sa_timeline_set_attn_small
    setter.argtypes = [ctypes.c_void_p]
    setter.restype = ctypes.c_int
    dev = torch.device("cuda")
    cfg = synth.workload(name)
    n = cfg.L
    wl = sgpu.decode_workload(cfg, dev)
    grs = wl["groups"]
    starts = [gr[0] for gr in cfg.groups]
    qI = [grs[starts.index(l)]["qI"] if l in starts else None for l in range(n)]
    w = [grs[starts.index(l)]["w"] if l in starts else None for l in range(n)]
    KI = [grs[starts.index(l)]["KI"] if l in starts else None for l in range(n)]
    gi = [max(i for i, s0 in enumerate(starts) if s0 <= l) for l in range(n)]
    K = [grs[gi[l]]["K"] for l in range(n)]
    V = [grs[gi[l]]["V"] for l in range(n)]
    O = torch.empty((n, cfg.B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device=dev)
    scores = torch.empty((cfg.B, cfg.S_max), dtype=torch.float32, device=dev)
    ws = sa.workspace(sa.decode_step_workspace_size(n, cfg.B, cfg.S_max, cfg.Hq, cfg.Hkv, cfg.d, cfg.k), dev)

    def step():
        sa.decode_step(cfg.pattern, qI, w, KI, K, V, wl["seq_off"], wl["seq_len"], cfg.S_max, cfg.k, wl["Q"],
                       cfg.Hkv, cfg.scale, O=O, idx=idx, scores=scores, ws=ws, per_layer=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    code, det = sa.read_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} {det}")
    cap = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for _ in range(steps_per_graph):
            step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    buf = torch.zeros(4 * 4096 * 64, dtype=torch.int64, device=dev)
    if setter(buf.data_ptr()) != 0:
        raise RuntimeError("timeline buffer could not be set")
    g.replay()
    torch.cuda.synchronize()
    setter(None)
    T = buf.view(4, 4096, 64)[3].cpu().numpy().astype(np.int64)
    live = T[:, 1] > 0
    t_wait = T[live, 1].min()  # the last launch's griddepcontrol.wait
    rows = T[live]
    stats = []
    for slot, label in POINTS["attention (few rows)"].items():
        v = rows[:, slot]
        # this launch's points: all after its wait, but entries, which may
        # precede it (the launch starts early) by less than a launch's length
        v = v[v >= (t_wait - 30_000 if slot == 0 else t_wait)]
        if v.size:
            v = (v - t_wait) / 1e3
            stats.append((slot, label, float(v.min()), float(np.median(v)), float(v.max()), int(v.size)))
    return cfg, {"attention (few rows)": {"ctas": int(live.sum()), "points": stats}}


def trace(name: str = "c3", steps_per_graph: int = 4):
    import cross_layer_shared_b200 as sa
    import synth
    from synth import gpu as sgpu

    sa.LIB_PATH = build.build_timeline()
    lb = sa.lib()
    setters = []
    for unit in ("indexer", "topk", "attn"):
        f = getattr(lb, f"sa_timeline_set_{unit}")
        f.argtypes = [ctypes.c_void_p]
        f.restype = ctypes.c_int
        setters.append(f)
    dev = torch.device("cuda")
    cfg = synth.workload(name)
    n = cfg.L
    plans = []
    for _ in range(2):
        wl = sgpu.decode_workload(cfg, dev)
        grs = wl["groups"]
        starts = [gr[0] for gr in cfg.groups]
        qI = [grs[starts.index(l)]["qI"] if l in starts else None for l in range(n)]
        w = [grs[starts.index(l)]["w"] if l in starts else None for l in range(n)]
        KI = [grs[starts.index(l)]["KI"] if l in starts else None for l in range(n)]
        gi = [max(i for i, s0 in enumerate(starts) if s0 <= l) for l in range(n)]
        K = [grs[gi[l]]["K"] for l in range(n)]
        V = [grs[gi[l]]["V"] for l in range(n)]
        plans.append((wl, sa.DecodeStepPlan(cfg.pattern, qI, w, KI, K, V, wl["seq_off"], wl["seq_len"], cfg.S_max,
                                            cfg.k, wl["Q"], cfg.Hkv, cfg.scale)))
    for _, p in plans:
        p.run()
    torch.cuda.synchronize()
    for _, p in plans:
        code, det = sa.read_status(p.ws)
        if code != 0:
            raise RuntimeError(f"device status {code} {det}")
    cap = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for j in range(steps_per_graph):
            plans[j % 2][1].run()
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    buf = torch.zeros(3 * 4096 * 64, dtype=torch.int64, device=dev)
    for f in setters:
        if f(buf.data_ptr()) != 0:
            raise RuntimeError("timeline buffer could not be set")
    g.replay()  # every point keeps the last step's time
    torch.cuda.synchronize()
    for f in setters:
        f(None)
    T = buf.view(3, 4096, 64).cpu().numpy().astype(np.int64)
    live0 = T[0, :, 0] > 0
    t0 = T[0, live0, 0].min()
    out = {}
    for kid, kname in enumerate(KERNELS):
        rows = T[kid]
        live = rows[:, 0] > 0
        stats = []
        for slot, label in POINTS[kname].items():
            v = rows[live, slot]
            v = v[v > 0]
            if v.size:
                v = (v - t0) / 1e3
                stats.append((slot, label, float(v.min()), float(np.median(v)), float(v.max()), int(v.size)))
        out[kname] = {"ctas": int(live.sum()), "points": stats}
    return cfg, out


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    per_layer = "--per-layer" in argv
    argv = [x for x in argv if x != "--per-layer"]
    name = argv[0] if argv else "c3"
    if per_layer:
        cfg, out = trace_per_layer(name)
        print(f"per-layer decode step, {name}, last attention launch: microseconds from its "
              f"griddepcontrol.wait (min / median / max over its CTAs)")
    else:
        cfg, out = trace(name)
        print(f"decode step timeline, {name}: microseconds from the first indexer CTA's entry "
              f"(min / median / max over the CTAs of each kernel)")
    for kname in out:
        k = out[kname]
        print(f"== {kname}: {k['ctas']} CTAs")
        for slot, label, lo, med, hi, cnt in k["points"]:
            print(f"  {lo:8.2f} {med:8.2f} {hi:8.2f}  {label}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
