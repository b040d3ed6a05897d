"""Pipeline timeline of the tensor-core attention kernels, from the tracing
build of the library (INFINI_TRACE; include/infini_attn_trace.h).

    python -m compressive_memory_segment_b200.trace_timeline [--kernel tile|paired]
        [--workload profile_64k_bf16] [--calls 3] [--raw events.npz]

Builds libinfini_attn_trace.so if needed, runs the forward on the workload
(warm-up, then one traced call) on the one-tile attention kernel (path TC) or
the paired-query-tile kernel (path TC_PAIRED) and prints, for CTA 0 of the
attention launch, each interval of the pipeline in SM clock cycles: median,
10th / 90th percentile, mean and total, plus a short excerpt of the raw
event stream. Event codes, by kernel and channel:
  one-tile kernel
    0 producer    1 K (or M) tile load issued, 2 V tile load issued, 3 Q tile load issued
    1 MMA         10 waits for the unit's Q tile, 11 Q tile in, 14 QK^T issued, 12 PV begins
                  (waits for P and V), 13 PV issued, 15 retrieval issued
    3/4 softmax   (warps 4 / 8: the two column halves of rows 0-31) 20 waits for S, 21 S ready,
                  22 row max done, 29 max exchange / rescale done, 26 exponentials done,
                  23 P handed to the MMA, 28 row sums handed over (end of the unit)
    5 epilogue    (warp 10) 30 unit starts, 31 den done, 34 last QK^T done, 32 sigma(Q) written,
                  33 row sums in, 24 O and R ready, 25 output row stored
  paired kernel
    0 K producer  1 K tile load issued
    7 V/Q producer 2 V tile load issued, 3/4 Q load of slot 0/1 issued
    1/2 MMA x     10 waits for the next unit's Q tile, 11 its first two QK^Ts issued, 12 PV begins
                  (waits for P), 13 PV issued, 14 next QK^T issued (after waiting for its K tile),
                  15 retrieval issued
    3/4 softmax   20 waits for S, 21 S ready, 22 row max done, 26 exponentials done (P stores issued),
                  23 P handed to the MMA, 28 row sums handed over (end of the slot's unit)
    5/6 retrieval warps (warp 8) of slot 0/1: 30 sigma(Q) starts, 31 sigma(Q) and den done,
                  33 row sums in (c scaling starts), 27 c scaling done, 24 O ready (epilogue starts),
                  25 epilogue stored
  single-pass d = 64 kernel (--kernel fused64, on the HF-reproduction workload)
    0 producer    1 the pair's tiles requested (index t)
    3 attention group (warp 0) 40 pair starts, 41 tiles in, 42 sigma(q) done, 43 S ready,
                  44 P stored, 45 prefix rows in, 46 P V and retrieval issued, 47 O ready,
                  48 output rows stored
    4 state group (warp 4) 50 pair starts, 51 tiles in, 52 sigma(K) done, 53 dM MMA issued,
                  54 dM in registers, 55 prefix rows and z written
  tensor-core backward, dK/dV kernel (--kernel bwd_kv, on the mid-length 8K workload; the
  backward's last launch, so its channels overwrite the statistics pass's)
    0 TMA         1 stage of query tile t requested, 2 G_s requested
    1 MMA         9 first stage in, 10 waits for P^T(t), 11 P^T in (dV, next S^T issued),
                  12 waits for dS^T(t), 13 dS^T in (dK, next dP^T issued), 14 loop's MMAs committed,
                  15 X and Y issued
    3 warp 2      20 waits for S^T(t), 21 S^T ready, 22 P^T stored, 23 dP^T ready, 24 dS^T stored,
                  30 loop done and G_s in, 31 sigma(K), G_s written, 32 X and Y done,
                  34 this thread's dk, dv rows staged, 35 every compute thread's staged,
                  33 dk, dv stored (TMA stores read out)
  tensor-core backward, d = 64 pair kernel (--kernel bwd64_pair, on the HF-reproduction workload)
    0 TMA, MMA    60 start, 61 tiles in (S, dP issued), 62 sigma(Q) in (R issued), 63 P in (O issued),
                  64 dS, dnum in (dQ, dnum M^T, dK, dV, sigma(Q)^T dnum issued), 65 committed
    3 warp 0      70 start, 71 tiles in, 72 sigma(Q) stored, 73 S, dP ready, 74 P stored, 75 R, O ready,
                  76 dS, dnum stored, 79 Gz summed (while the last MMAs run), 77 last MMAs done,
                  78 dq, G staged (their TMA stores issued), dk, dv staged and Gz stored,
                  80 every tile's TMA store read out
This is a profiling tool; it is not used by the library or its tests.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import statistics
import sys

import numpy as np
import torch

from . import build as _build
from . import synth

NAMES = {1: "K load", 2: "V load", 3: "Q(0) load", 4: "Q1 load", 10: "Q wait", 11: "Q in / QK0,1",
         12: "PV begin", 13: "PV issued", 14: "QK issued", 15: "R issued", 20: "S wait", 21: "S ready",
         22: "max done", 23: "P done", 24: "epi O ready", 25: "epi stored", 26: "exp done", 27: "c-scaled",
         28: "l handed", 29: "xchg done", 30: "unit/sigma start", 31: "den/sigma done", 32: "sigma(Q) in",
         33: "l in", 34: "last QK done"}
CHANNELS = ["producer", "mma0", "mma1", "softmax0", "softmax1", "sigma0", "sigma1", "producer_v"]

# Intervals to report: (title, channel, from code, to code).
TILE_INTERVALS = [
    ("softmax, column half %d" % h, "softmax%d" % h, [
        ("S wait (20->21)", 20, 21), ("load + max (21->22)", 21, 22), ("max exchange / rescale (22->29)", 22, 29),
        ("exponentials (29->26)", 29, 26), ("P store wait (26->23)", 26, 23),
        ("unit end -> next S ready (28->21)", 28, 21)]) for h in range(2)] + [
    ("MMA issuer", "mma0", [
        ("wait for the unit's Q (10->11)", 10, 11), ("PV: wait for P and V (12->13)", 12, 13),
        ("QK^T issue (13->14)", 13, 14)]),
    ("epilogue warp", "sigma0", [
        ("den (30->31)", 30, 31), ("wait for the last QK^T (31->34)", 31, 34), ("sigma(Q) (34->32)", 34, 32),
        ("wait for row sums (32->33)", 32, 33), ("wait for O and R (33->24)", 33, 24), ("store (24->25)", 24, 25)]),
]
FUSED64_INTERVALS = [
    ("attention group (warp 0)", "softmax0", [
        ("wait for the pair's tiles (40->41)", 40, 41), ("sigma(q) (41->42)", 41, 42),
        ("wait for QK^T (42->43)", 42, 43), ("softmax, P store (43->44)", 43, 44),
        ("wait for the prefix rows (44->45)", 44, 45), ("den, c sigma(q), barrier, MMA issue (45->46)", 45, 46),
        ("wait for P V + retrieval (46->47)", 46, 47), ("epilogue (47->48)", 47, 48),
        ("to the next pair (48->40)", 48, 40)]),
    ("state group (warp 4)", "softmax1", [
        ("wait for the pair's tiles (50->51)", 50, 51), ("sigma(K) hi / lo, dz partials (51->52)", 51, 52),
        ("barrier, dM MMA issue (52->53)", 52, 53), ("dz, wait for MR free and dM, load dM (53->54)", 53, 54),
        ("prefix rows, z, barriers (54->55)", 54, 55), ("to the next pair (55->50)", 55, 50)]),
]
BWD_KV_INTERVALS = [
    ("MMA warp (channel 1)", "mma0", [
        ("wait for P^T (10->11)", 10, 11),
        ("dV, next S^T issue (11->12)", 11, 12),
        ("wait for dS^T (12->13)", 12, 13),
        ("loop end -> X, Y issued (14->15)", 14, 15)]),
    ("compute warp 2, key rows 64-95, query columns 0-63 (channel 3)", "softmax0", [
        ("wait for S^T (20->21)", 20, 21),
        ("P^T: load, exponentials, store (21->22)", 21, 22),
        ("wait for dP^T (22->23)", 22, 23),
        ("dS^T: load, products, store (23->24)", 23, 24),
        ("tile end -> next tile (24->20)", 24, 20),
        ("last tile -> loop done and G_s in (24->30)", 24, 30),
        ("sigma(K), G_s to bf16 (30->31)", 30, 31),
        ("wait for X, Y (31->32)", 31, 32),
        ("epilogue: dk, dv staged (32->34)", 32, 34),
        ("barrier over the compute warps (34->35)", 34, 35),
        ("TMA stores issued and read out (35->33)", 35, 33)]),
]
BWD_KV_NAMES = {1: "stage req", 2: "G req", 9: "stage0 in", 10: "P wait", 11: "P in", 12: "dS wait", 13: "dS in",
                14: "loop done", 15: "X,Y issued", 20: "S^T wait", 21: "S^T in", 22: "P^T stored",
                23: "dP^T in", 24: "dS^T stored", 30: "tail", 31: "sigma,G", 32: "X,Y in", 33: "stored",
                34: "staged", 35: "all staged"}
BWD64_INTERVALS = [
    ("TMA and MMA warp (channel 0)", "producer", [
        ("start -> tiles in (60->61)", 60, 61),
        ("tiles in -> sigma(Q) in (61->62)", 61, 62),
        ("sigma(Q) in -> P in (62->63)", 62, 63),
        ("P in -> dS in (63->64)", 63, 64),
        ("issue of the last MMAs (64->65)", 64, 65)]),
    ("row warp 0 (channel 3)", "softmax0", [
        ("start -> tiles in (70->71)", 70, 71),
        ("sigma(q), den, stores (71->72)", 71, 72),
        ("wait for S, dP (72->73)", 72, 73),
        ("softmax, P stores (73->74)", 73, 74),
        ("wait for R, O (74->75)", 74, 75),
        ("dnum, dS (75->76)", 75, 76),
        ("Gz sum (76->79)", 76, 79),
        ("wait for the last MMAs (79->77)", 79, 77),
        ("dq, G staged and stored, dk, dv staged (77->78)", 77, 78),
        ("barrier, dk, dv stores, every tile read out (78->80)", 78, 80)]),
]
BWD64_NAMES = {60: "start", 61: "tiles in", 62: "sigQ in", 63: "P in", 64: "dS in", 65: "committed",
               70: "start", 71: "tiles in", 72: "sigQ st", 73: "S in", 74: "P st", 75: "O in", 76: "dS st",
               77: "fin in", 78: "staged", 79: "Gz sum", 80: "stored"}
PAIRED_INTERVALS = []
for _x in range(2):
    PAIRED_INTERVALS += [
        ("slot %d softmax" % _x, "softmax%d" % _x, [
            ("S wait (20->21)", 20, 21), ("load + max (21->22)", 21, 22), ("exponentials (22->26)", 22, 26),
            ("P store wait (26->23)", 26, 23), ("unit end -> next S ready (28->21)", 28, 21)]),
        ("slot %d MMA issuer" % _x, "mma%d" % _x, [
            ("wait for P and V (12->13)", 12, 13), ("wait for K (13->14)", 13, 14),
            ("wait for next Q (10->11)", 10, 11), ("next QKs -> retrieval (11->15)", 11, 15)]),
        ("slot %d retrieval warps" % _x, "sigma%d" % _x, [
            ("sigma(Q), den (30->31)", 30, 31), ("sigma done -> row sums in (31->33)", 31, 33),
            ("c scaling (33->27)", 33, 27), ("scaled -> O ready (27->24)", 27, 24), ("epilogue (24->25)", 24, 25)]),
    ]


def _decode(words):
    w = np.asarray(words, dtype=np.uint64)
    t = (w & np.uint64(0xFFFFFFFFFF)).astype(np.int64)
    code = ((w >> np.uint64(40)) & np.uint64(0xFF)).astype(np.int64)
    idx = ((w >> np.uint64(48)) & np.uint64(0xFFFF)).astype(np.int64)
    return t, code, idx


def _stats(xs):
    if not xs:
        return "-"
    a = np.asarray(xs)
    return "%6.0f [%6.0f, %6.0f] n=%d  mean %6.0f  total %9.0f" % (
        np.median(a), np.percentile(a, 10), np.percentile(a, 90), len(a), a.mean(), a.sum())


def _intervals(t, code, a, b, same_index=False, idx=None):
    """Durations from each event `a` to the next event `b` on one channel."""
    out = []
    pend = None
    for k in range(len(t)):
        if code[k] == a:
            pend = k
        elif code[k] == b and pend is not None:
            if not same_index or idx[pend] == idx[k]:
                out.append(int(t[k] - t[pend]))
            pend = None
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default="tile", choices=["tile", "paired", "fused64", "bwd_kv", "bwd64_pair"],
                    help="the one-tile attention kernel (path TC), the paired one (path TC_PAIRED), the "
                         "d = 64 single-pass kernel (path TC on a d = 64, N = 64 workload), the tensor-core "
                         "backward's dK/dV kernel, or the d = 64 backward's pair kernel")
    ap.add_argument("--workload", default="profile_64k_bf16", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--calls", type=int, default=3, help="untraced warm-up calls before the traced one")
    ap.add_argument("--excerpt", type=int, default=60, help="raw events to print from the middle")
    ap.add_argument("--lib", default=None, help="a tracing build to use instead of building the package's")
    ap.add_argument("--raw", default=None, help="also save the decoded events of every channel to this .npz")
    args = ap.parse_args(argv)
    lib = ctypes.CDLL(args.lib or _build.build(trace=True))
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t

    class Shape(ctypes.Structure):
        _fields_ = [("B", i64), ("H", i64), ("L", i64), ("d", i64), ("dtype", ctypes.c_int)]

    lib.infini_attn_workspace_size.argtypes = [ctypes.POINTER(Shape), i64]
    lib.infini_attn_workspace_size.restype = sz
    lib.infini_attn_forward_ws.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp, sz,
                                           ctypes.c_int, vp]
    lib.infini_attn_trace_read.argtypes = [ctypes.c_int, vp, ctypes.c_int]
    lib.infini_attn_backward_workspace_size.argtypes = [ctypes.POINTER(Shape), i64]
    lib.infini_attn_backward_workspace_size.restype = sz
    lib.infini_attn_backward_path.argtypes = [ctypes.POINTER(Shape)] + [vp] * 6 + [i64] + [vp] * 10 + [
        sz, ctypes.c_int, vp]
    if args.kernel == "fused64" and args.workload == "profile_64k_bf16":
        args.workload = "hf_repro_bf16"
    if args.kernel == "bwd_kv" and args.workload == "profile_64k_bf16":
        args.workload = "mid_8k_outlier_bf16"
    if args.kernel == "bwd64_pair" and args.workload == "profile_64k_bf16":
        args.workload = "hf_repro_bf16"
    bwd = args.kernel in ("bwd_kv", "bwd64_pair")
    w = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    q, k, v = synth.make_qkv(w, dev)
    beta = synth.make_beta(w, dev)
    per = w.L // w.calls
    q, k, v = (x[:, :, :per].contiguous() for x in (q, k, v))
    shp = Shape(w.B, w.H, per, w.d, 1 if w.dtype == "bf16" else 0)
    out = torch.empty_like(q)
    M = torch.empty((w.B, w.H, w.d, w.d), device=dev)
    z = torch.empty((w.B, w.H, w.d), device=dev)
    ws_n = lib.infini_attn_workspace_size(ctypes.byref(shp), w.N)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)

    path = 3 if args.kernel == "paired" else 2
    if bwd:
        g = torch.Generator(device="cpu").manual_seed(w.seed)
        dout = torch.randn(q.shape, generator=g).to(q.dtype).to(dev)
        f32 = dict(dtype=torch.float32, device=dev)
        grads = [torch.empty(q.shape, **f32) for _ in range(3)] + [
            torch.empty((w.H,), **f32), torch.empty((w.B, w.H, w.d, w.d), **f32), torch.empty((w.B, w.H, w.d), **f32)]
        ws_n = lib.infini_attn_backward_workspace_size(ctypes.byref(shp), w.N)
        ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)

    def call():
        if bwd:
            rc = lib.infini_attn_backward_path(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                               beta.data_ptr(), None, None, w.N, dout.data_ptr(), None, None,
                                               *[x.data_ptr() for x in grads], ws.data_ptr(), ws_n, path, None)
        else:
            rc = lib.infini_attn_forward_ws(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            beta.data_ptr(), None, None, w.N, out.data_ptr(), M.data_ptr(),
                                            z.data_ptr(), ws.data_ptr(), ws_n, path, None)
        if rc != 0:
            raise SystemExit("call failed: %d" % rc)

    for _ in range(args.calls):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.calls):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms_untraced = e0.elapsed_time(e1) / max(args.calls, 1)
    if lib.infini_attn_trace_reset() != 0:
        raise SystemExit("trace reset failed")
    call()
    torch.cuda.synchronize()
    ch = {}
    for c, name in enumerate(CHANNELS):
        buf = np.zeros(1 << 15, dtype=np.uint64)
        n = lib.infini_attn_trace_read(c, buf.ctypes.data, buf.size)
        if n < 0:
            raise SystemExit("trace read failed: %d" % n)
        ch[name] = _decode(buf[:min(n, buf.size)])
    if args.raw:
        np.savez(args.raw, **{"%s_%s" % (name, f): arr for name, v in ch.items() for f, arr in zip("tci", v)})
    spans = [int(v[0].max() - v[0].min()) for v in ch.values() if len(v[0])]
    print("workload %s (one call of %d tokens): %.4f ms per call (whole %s, CUDA events, mean of %d); "
          "CTA 0 of the %s kernel; SM clock cycles, median [p10, p90]"
          % (w.name, per, ms_untraced, "backward" if bwd else "forward", args.calls,
             {"paired": "paired attention", "fused64": "single-pass d = 64",
              "bwd_kv": "backward dK/dV", "bwd64_pair": "backward d = 64 pair"}.get(args.kernel,
                                                                                    "one-tile attention")))
    if spans:
        print("CTA 0 trace span: %d cycles (first to last event over all channels: %d)"
              % (max(spans), int(max(v[0].max() for v in ch.values() if len(v[0])) -
                                  min(v[0].min() for v in ch.values() if len(v[0])))))
    table = {"paired": PAIRED_INTERVALS, "fused64": FUSED64_INTERVALS,
             "bwd_kv": BWD_KV_INTERVALS, "bwd64_pair": BWD64_INTERVALS}.get(args.kernel, TILE_INTERVALS)
    names = {"bwd_kv": BWD_KV_NAMES, "bwd64_pair": BWD64_NAMES}.get(args.kernel, NAMES)
    for title, chan, spec in table:
        t, c, _ = ch[chan]
        print(title + ":")
        for name, a, b in spec:
            print("  %-38s %s" % (name, _stats(_intervals(t, c, a, b))))
    ev = []
    for name, (t, c, i) in ch.items():
        if bwd and name not in ("producer", "mma0", "softmax0"):
            continue  # the statistics pass's records
        ev += [(int(a), name, names.get(int(b), str(int(b))), int(d)) for a, b, d in zip(t, c, i)]
    ev.sort()
    if ev:
        mid = len(ev) // 2
        t0 = ev[mid][0]
        print("excerpt (cycles from an event in the middle of the call):")
        for e in ev[mid:mid + args.excerpt]:
            print("%8d  %-9s %-14s %d" % (e[0] - t0, e[1], e[2], e[3]))
    return 0


if __name__ == "__main__":
    sys.exit(main())
