"""Pipeline timeline of the paired tensor-core attention kernel, from the
tracing build of the library (INFINI_TRACE; include/infini_attn_trace.h).

    python -m compressive_memory_segment_b200.trace_timeline [--workload profile_64k_bf16] [--calls 3]

Builds libinfini_attn_trace.so if needed, runs the forward on the workload
(warm-up, then one traced call) and prints, for CTA 0 of the attention
launch, the median / 10th / 90th percentile of each interval of the
pipeline in SM clock cycles, and a short excerpt of the raw event stream.
Event codes, by channel:
  0 producers  1 K tile load issued, 2 V tile load issued, 3/4 Q load of slot 0/1 issued
  1/2 MMA x    10 waits for the next unit's Q tile, 11 its first two QK^Ts issued, 12 PV begins
               (waits for P), 13 PV issued, 14 next QK^T issued (after waiting for its K tile),
               15 retrieval issued
  3/4 softmax  20 waits for S, 21 S ready, 22 row max done, 26 exponentials done (P stores issued),
               23 P handed to the MMA, 28 row sums handed over (end of the slot's unit)
  5/6 retrieval warps (warp 8) of slot 0/1: 30 sigma(Q) starts, 31 sigma(Q) and den done,
               33 row sums in (c scaling starts), 27 c scaling done, 24 O ready (epilogue starts),
               25 epilogue stored
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

NAMES = {1: "K load", 2: "V load", 3: "Q0 load", 4: "Q1 load", 10: "next Q wait", 11: "next QK0,1",
         12: "PV begin", 13: "PV issued", 14: "QK issued", 15: "R issued", 20: "S wait", 21: "S ready",
         22: "max done", 23: "P done", 24: "epi O ready", 25: "epi stored", 26: "exp done", 27: "c-scaled",
         28: "l handed", 30: "sigma start", 31: "sigma done", 33: "l in"}
CHANNELS = ["producer", "mma0", "mma1", "softmax0", "softmax1", "sigma0", "sigma1"]


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
    return "%6.0f [%6.0f, %6.0f] n=%d" % (np.median(a), np.percentile(a, 10), np.percentile(a, 90), len(a))


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
    ap.add_argument("--workload", default="profile_64k_bf16", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--calls", type=int, default=3, help="untraced warm-up calls before the traced one")
    ap.add_argument("--excerpt", type=int, default=60, help="raw events to print from the middle")
    ap.add_argument("--lib", default=None, help="a tracing build to use instead of building the package's")
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

    def call():
        rc = lib.infini_attn_forward_ws(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                        beta.data_ptr(), None, None, w.N, out.data_ptr(), M.data_ptr(),
                                        z.data_ptr(), ws.data_ptr(), ws_n, 2, None)
        if rc != 0:
            raise SystemExit("forward failed: %d" % rc)

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
    print("workload %s (one call of %d tokens): %.4f ms per call (whole forward, CUDA events, mean of %d); "
          "CTA 0 of the paired attention kernel; SM clock cycles, median [p10, p90]"
          % (w.name, per, ms_untraced, args.calls))
    for x in range(2):
        t, c, i = ch["softmax%d" % x]
        print("slot %d softmax:" % x)
        print("  S wait (20->21)              ", _stats(_intervals(t, c, 20, 21)))
        print("  load + max (21->22)          ", _stats(_intervals(t, c, 21, 22)))
        print("  exponentials (22->26)        ", _stats(_intervals(t, c, 22, 26)))
        print("  P store wait (26->23)        ", _stats(_intervals(t, c, 26, 23)))
        print("  unit end -> next S ready (28->21)", _stats(_intervals(t, c, 28, 21)))
        t, c, i = ch["mma%d" % x]
        print("slot %d MMA issuer:" % x)
        print("  wait for P and V (12->13)    ", _stats(_intervals(t, c, 12, 13)))
        print("  wait for K (13->14)          ", _stats(_intervals(t, c, 13, 14)))
        print("  wait for next Q (10->11)     ", _stats(_intervals(t, c, 10, 11)))
        print("  next QKs -> retrieval (11->15)", _stats(_intervals(t, c, 11, 15)))
        t, c, i = ch["sigma%d" % x]
        print("slot %d retrieval warps:" % x)
        print("  sigma(Q), den (30->31)       ", _stats(_intervals(t, c, 30, 31)))
        print("  sigma done -> row sums in (31->33)", _stats(_intervals(t, c, 31, 33)))
        print("  c scaling (33->27)           ", _stats(_intervals(t, c, 33, 27)))
        print("  scaled -> O ready (27->24)   ", _stats(_intervals(t, c, 27, 24)))
        print("  epilogue (24->25)            ", _stats(_intervals(t, c, 24, 25)))
    ev = []
    for name, (t, c, i) in ch.items():
        ev += [(int(a), name, NAMES.get(int(b), str(int(b))), int(d)) for a, b, d in zip(t, c, i)]
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
