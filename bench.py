#!/usr/bin/env python
"""Benchmark of the Infini-attention layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole forward (state increments, cross-segment
scan, fused attention + retrieval + gate) over the workload's full sequence,
fed in the workload's number of streamed calls that carry (M, z). Inputs are
seeded synthetic tensors resident in HBM before the timed region; they are
larger than L2, so no explicit flush is needed between steps.

Prints one JSON line on rank 0. Under torchrun (N > 1) every rank runs its own
replica of the workload (independent problems: weak scaling, no collective on
the data path); the step time is the max over ranks.

--impl reference times the CPU oracle (the reference for this layer) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import faulthandler
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from compressive_memory_segment_b200 import synth  # noqa: E402

METRIC = "Infini-attn fwd tokens/s & TFLOP/s on 1 B200; % of bf16 tensor roofline"
DEFAULT_WORKLOAD = "stream_1m_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 << 20


def kernel_names(path: int, w) -> list:
    """The three launches of a forward call on this path and shape."""
    if path == 1:
        return ["simt_state_kernel", "scan_state_kernel", "simt_attn_kernel"]
    if w.d == 64:
        return ["tc_fused64_kernel"]  # state, prefix and attention in one pass (64-token segments)
    attn = "tc_attn_pair_kernel" if path == 3 else "tc_attn_kernel"
    return ["tc_state_kernel", "scan_state_kernel", attn]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def work_counts(w: synth.Workload):
    """Algorithmic FLOPs and bytes per step (whole sequence, all calls).

    Per (b, h, segment): local causal attention 2 d N (N + 1) (QK^T and PV over
    the N(N+1)/2 visible pairs), retrieval 2 N d^2, state increment 2 N d^2.
    Bytes: q, k, v, out once each, plus (M, z) in and out per call and beta."""
    BH, S, N, d = w.B * w.H, w.S, w.N, w.d
    elt = 4 if w.dtype == "f32" else 2
    f_local = 2.0 * d * N * (N + 1)
    f_ret = 2.0 * N * d * d
    f_state = 2.0 * N * d * d
    flops = BH * S * (f_local + f_ret + f_state)
    attn_flops = BH * S * (f_local + f_ret)
    state_flops = BH * S * f_state
    bytes_ = 4.0 * BH * w.L * d * elt + w.calls * (2.0 * BH * (d * d + d) * 4) + w.H * 4
    return dict(flops=flops, attn_flops=attn_flops, state_flops=state_flops, bytes=bytes_)


class ClockSampler:
    """SM clocks and throttle reasons sampled while the timed region runs.

    NVML is polled from a thread every 5 ms (plus one sample on entry and one
    on exit), so even a timed region of a few milliseconds has samples; the
    GPU is found by its PCI bus id. Without NVML, nvidia-smi is polled every
    50 ms instead. Only reads: nothing here changes a GPU setting."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None
        self.nvml = None
        self.thread = None
        self.samples = []  # (sm_mhz, max_mhz, set of reasons)

    @staticmethod
    def pci_bus_id(props) -> str:
        """NVML's "domain:bus:device.function" string for a torch device.
        torch reports the three numbers as integers; NVML must get the
        string (an integer there would be taken for an address)."""
        dom, bus, dev = props.pci_domain_id, props.pci_bus_id, props.pci_device_id
        if not all(isinstance(x, int) for x in (dom, bus, dev)):
            raise TypeError("PCI location is not numeric")
        return "%04x:%02x:%02x.0" % (dom, bus, dev)

    def _nvml_open(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            h = pynvml.nvmlDeviceGetHandleByPciBusId(self.pci_bus_id(torch.cuda.get_device_properties(self.index)))
        except Exception:
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
        bits = (pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap)
        smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        self.nvml = (pynvml, h, bits, smax)

    def _nvml_sample(self):
        pynvml, h, bits, smax = self.nvml
        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
        self.samples.append((float(sm), float(smax), {n for n, b in zip(self.NAMES, bits) if mask & b}))

    def __enter__(self):
        try:
            self._nvml_open()
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            import threading
            self.stop = threading.Event()

            def poll():
                while not self.stop.wait(0.005):
                    try:
                        self._nvml_sample()
                    except Exception:
                        return

            self._nvml_sample()
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return self
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            try:
                self._nvml_sample()
            except Exception:
                pass
            try:
                self.nvml[0].nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def _smi_rows(self):
        self.file.flush()
        with open(self.file.name) as f:
            rows = [r.strip().split(", ") for r in f if r.strip()]
        os.unlink(self.file.name)
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm, smax = float(r[1]), float(r[2])
            except ValueError:
                continue
            self.samples.append((sm, smax, {n for n, val in zip(self.NAMES, r[5:9])
                                            if val.strip().lower() == "active"}))

    def summary(self):
        source = "nvml"
        if self.nvml is None:
            source = "nvidia-smi"
            if self.proc is None or self.file is None:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
            self._smi_rows()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": source}
        sm = [x[0] for x in self.samples]
        reasons = set().union(*(x[2] for x in self.samples))
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": sorted(reasons), "samples": len(sm), "source": source}


def tensor_peak(pk, pk_src, clocks):
    """The bf16 dense peak a kernel timed in this run is held against: the
    burst figure when the SM clock held near its maximum under load (median
    within 10 % of max), the sustained (power-capped) figure otherwise."""
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if sm and smax and sm >= 0.9 * smax:
        return pk["bf16_tflops"], "burst bf16 dense (%s; SM clock median %.0f of %.0f MHz)" % (pk_src, sm, smax)
    sus = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    return sus, "sustained bf16 dense (%s; SM clock median %s of %s MHz)" % (pk_src, sm, smax)


def step_roofline(wc, pk, pk_src, ms_step):
    """The whole step against its roofline: the step's algorithmic FLOPs at the
    burst bf16 dense peak or its bytes at HBM bandwidth, whichever takes longer."""
    t_flops = wc["flops"] / (pk["bf16_tflops"] * 1e12)
    t_bytes = wc["bytes"] / (pk["hbm_gbs"] * 1e9)
    tensor = t_flops >= t_bytes
    secs = ms_step / 1000.0
    return {"bound": "tensor" if tensor else "hbm",
            "achieved": (wc["flops"] / secs / 1e12) if tensor else (wc["bytes"] / secs / 1e9),
            "peak": pk["bf16_tflops"] if tensor else pk["hbm_gbs"],
            "unit": "TFLOP/s" if tensor else "GB/s",
            "frac": max(t_flops, t_bytes) / secs,
            "peak_kind": ("burst bf16 dense (%s)" if tensor else "HBM copy (%s)") % pk_src,
            "roofline_ms": 1000.0 * max(t_flops, t_bytes)}


def kernel_traffic(path: int):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, valid only while the kernel source is unchanged: the hash covers
    the source file's device code, up to its host-side marker line (the whole
    file when it has none)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, "compressive_memory_segment_b200", "csrc", d.get("source", ""))
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        text = f.read()
    marker = d.get("source_end_marker", "").encode()
    if marker and marker in text:
        text = text[:text.index(marker)]
    sha = hashlib.sha256(text).hexdigest()[:16]
    ent = d.get("kernels", {}).get(str(path))
    if not ent or ent.get("source_sha") != sha:
        return None
    return ent.get("bytes_per_launch")


# ----------------------------------------------------------------------------- reference arm

def oracle_sample_run(w: synth.Workload, q, k, v, beta, seg_count: int, nthreads: int):
    """Time the CPU oracle on the first seg_count segments of every (b, h)."""
    import oracle
    import numpy as np
    T = seg_count * w.N
    qs, ks, vs = (t[:, :, :T].contiguous() for t in (q, k, v))
    def bits(t):
        t = t.cpu()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()
    qh, kh, vh = bits(qs), bits(ks), bits(vs)
    bh = beta.double().cpu().numpy()
    t0 = time.perf_counter()
    oracle.forward(qh, kh, vh, bh, seg_len=w.N, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return w.B * T / dt, dt, T


def reference_arm(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    q, k, v = synth.make_qkv(w, "cpu", L=min(w.L, 4 * w.N))
    beta = synth.make_beta(w, "cpu")
    nthreads = max(1, min(w.B * w.H, os.cpu_count() or 1))
    seg_count = max(1, min(w.S, 2 if w.N >= 1024 else 16))
    for _ in range(args.warmup):
        oracle_sample_run(w, q, k, v, beta, 1, nthreads)
    vals, times = [], []
    for _ in range(args.steps):
        val, dt, T = oracle_sample_run(w, q, k, v, beta, seg_count, nthreads)
        vals.append(val)
        times.append(dt)
    value = statistics.median(vals)
    sample = "all %d (b,h) pairs x first %d segment(s) (%d tokens each) of %s" % (w.B * w.H, seg_count, seg_count * w.N, w.name)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * statistics.median(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "N": w.N, "L": w.L,
                                        "calls": w.calls, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- ranks

def init_dist(backend: str, timeout_s: int = 120):
    """One process per GPU (or per CPU rank in the gloo tests), rendezvous from
    the torchrun environment. Returns the torch.distributed module, or None for
    a single process."""
    if int(os.environ.get("WORLD_SIZE", "1")) <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def max_over_ranks(x: float, dist, device) -> float:
    """The slowest rank's value: step times are reported as the max over ranks."""
    if dist is None:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, ms_step: float) -> float:
    """Whole-job throughput: every rank runs its own replica of the workload
    (weak scaling), so the job processes world * tokens_per_rank per step."""
    return world * tokens_per_rank / (ms_step / 1000.0)


# ----------------------------------------------------------------------------- backward

# fp32 FFMA peak of the CUDA cores: 148 SMs x 128 FP32 lanes x 2 FLOP x 1965 MHz
# (the B200's SM count, lanes per SM and maximum SM clock).
FP32_FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def backward_flops(w: synth.Workload) -> float:
    """Algorithmic FLOPs of the backward per step: per visible (query, key)
    pair of a segment the score recompute, dP, dV, dQ and dK (5 d-long
    multiply-adds), and per token the retrieval and state terms (sigma(Q)^T
    dnum, dsigma(q), dv and dk from the state gradient: 4 d^2 multiply-adds)."""
    BH, S, N, d = w.B * w.H, w.S, w.N, w.d
    return BH * S * (5.0 * d * N * (N + 1) + 8.0 * N * d * d)


def backward_arm(args, w):
    """One training step of the layer: forward then backward over the
    workload's sequence (one call), inputs and dout resident in HBM."""
    from compressive_memory_segment_b200 import binding as bd
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = synth.make_qkv(w, dev)
    beta = synth.make_beta(w, dev)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    dout = torch.randn(q.shape, generator=g).to(q.dtype).to(dev)
    shp = bd.shape_of(q)
    B, H, L, d = q.shape
    out = torch.empty_like(q)
    M = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
    z = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    fws = bd.workspace_for(q, w.N)
    bws = torch.empty(bd.infini_attn_backward_workspace_size(shp, w.N), dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty((B, H, L, d), **f32) for _ in range(3))
    dbeta, dM, dz = torch.empty((H,), **f32), torch.empty((B, H, d, d), **f32), torch.empty((B, H, d), **f32)
    stream = torch.cuda.current_stream(dev)

    def fwd():
        bd.check(bd.infini_attn_forward_ws(shp, q, k, v, beta, None, None, w.N, out, M, z, fws, fws.numel(),
                                           bd.INFINI_PATH_AUTO, stream))

    def bwd():
        bd.check(bd.infini_attn_backward(shp, q, k, v, beta, None, None, w.N, dout, None, None, dq, dk, dv, dbeta,
                                         dM, dz, bws, bws.numel(), stream))

    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    t_f = t_b = 0.0
    with ClockSampler(dev.index) as clk:
        for _ in range(args.steps):
            ev[0].record(stream)
            fwd()
            ev[1].record(stream)
            bwd()
            ev[2].record(stream)
            torch.cuda.synchronize(dev)
            t_f += ev[0].elapsed_time(ev[1])
            t_b += ev[1].elapsed_time(ev[2])
    st = bd.infini_attn_device_status(stream)
    if st != 0:
        raise RuntimeError(bd.infini_attn_strerror(st))
    t_f /= args.steps
    t_b /= args.steps
    ms = t_f + t_b
    bfl = backward_flops(w)
    ach = bfl / (t_b / 1000.0) / 1e12
    tc64 = w.dtype == "bf16" and d == 64 and w.N == 64 and w.S % 2 == 0
    tc_bwd = (w.dtype == "bf16" and d == 128 and w.N % 128 == 0) or tc64
    clocks = clk.summary()
    fwd_launches = bd.infini_attn_launch_count(shp, w.N, bd.INFINI_PATH_AUTO)
    if tc_bwd:
        pk, pk_src = peaks()
        peak, peak_kind = tensor_peak(pk, pk_src, clocks)
        kern = ("backward: tc_state64_kernel, scan, tc_bwd64_pair_kernel, bwd_rscan, tc_bwd64_state_kernel"
                if tc64 else "backward: statistics pass (tc_state, scan, tc_attn_kernel<true>), tc_bwd_dq_kernel, "
                "bwd_rscan, tc_bwd_kv_kernel")
        roof = {"kernel": kern, "bound": "tensor",
                "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak, "peak_kind": peak_kind,
                "flops_per_step": bfl, "flops_note": ("algorithmic: 5 d-long multiply-adds per visible (query, key) "
                                                      "pair and 4 d^2 per token; " + (
                                                          "the pair kernel's block-diagonal tiles also multiply the "
                                                          "zero blocks" if tc64 else
                                                          "the kernels recompute S three times")), "traffic": None}
        launches = fwd_launches + (5 if tc64 else 6)
    else:
        roof = {"kernel": "backward (bwd_rows + bwd_keys and the state chain)", "bound": "alu",
                "achieved": ach, "peak": FP32_FFMA_TFLOPS, "unit": "TFLOP/s", "frac": ach / FP32_FFMA_TFLOPS,
                "peak_kind": ("fp32 FFMA: 148 SMs x 128 lanes x 2 x 1965 MHz; with bf16 inputs the tile "
                              "products run on TF32 mma.sync and are counted as the same work"),
                "flops_per_step": bfl, "traffic": None}
        launches = fwd_launches + 6
    print(json.dumps({
        "metric": "Infini-attn training step (forward + backward) tokens/s", "value": B * L / (ms / 1000.0),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": B, "H": H, "d": d, "N": w.N, "L": L,
                   "step": "forward + backward of one call; gradients fp32"},
        "ms_forward": t_f, "ms_backward": t_b, "backward_path": "tc" if tc_bwd else "simt",
        "roofline": roof, "clocks": clocks, "gpu_launches": args.steps * launches,
    }), flush=True)
    return 0


# ----------------------------------------------------------------------------- decode

def decode_bytes(w: synth.Workload) -> float:
    """Algorithmic HBM bytes of one segment of decode steps (all B*H heads):
    per step q, k, v and out rows, the cache rows 0..pos-1 of K and V read and
    row pos written, M and z read; at the segment's end the fold reads K, V once
    and reads and writes M, z."""
    BH, N, d = w.B * w.H, w.N, w.d
    elt = 2 if w.dtype == "bf16" else 4
    cache_rows = N * (N - 1) / 2.0                   # sum over pos of pos
    per_head = (N * 4 * d * elt                      # q, k, v, out
                + 2 * cache_rows * d * elt           # K, V cache reads
                + N * 2 * d * elt                    # cache row writes
                + N * (d * d + d) * 4                # M, z reads
                + 2 * N * d * elt + 2 * (d * d + d) * 4)  # fold
    return BH * per_head


def decode_step_bytes(w: synth.Workload, pos: int) -> float:
    """Algorithmic HBM bytes of one decode step at position pos (all heads,
    without the fold)."""
    BH, d = w.B * w.H, w.d
    elt = 2 if w.dtype == "bf16" else 4
    return BH * (4 * d * elt + 2 * pos * d * elt + 2 * d * elt + (d * d + d) * 4)


def decode_pos_arm(args, w, pos):
    """Single decode steps at one position of a cache filled with seeded
    values (no fold unless pos == N - 1): the per-launch figure for the
    roofline and for profiling."""
    from compressive_memory_segment_b200 import binding as bd
    dev = torch.device("cuda", torch.cuda.current_device())
    B, H, N, d = w.B, w.H, w.N, w.d
    if not 0 <= pos < N:
        raise SystemExit("--decode-pos must be in [0, %d)" % N)
    q, k, v = synth.make_qkv(w, dev, L=N)
    beta = synth.make_beta(w, dev)
    kc, vc = k.clone(), v.clone()            # rows 0..pos-1 are the cached segment
    M, z = synth.make_state(w, dev)
    qt, kt, vt = (x[:, :, pos].contiguous() for x in (q, k, v))
    out = torch.empty_like(qt)
    shp = bd.make_shape(B, H, N, d, bd.INFINI_BF16 if w.dtype == "bf16" else bd.INFINI_F32)
    ws = torch.empty(bd.infini_attn_decode_workspace_size(shp), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def one():
        rc = bd.infini_attn_decode_step(shp, qt, kt, vt, beta, kc, vc, pos, M, z, out, ws, ws.numel(), stream)
        if rc != 0:
            raise RuntimeError(bd.infini_attn_strerror(rc))

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    pk, pk_src = peaks()
    gbs = decode_step_bytes(w, pos) / (ms / 1000.0) / 1e9
    print(json.dumps({"metric": "Infini-attn decode step at one cache position", "value": B / (ms / 1000.0),
                      "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
                      "config": {"workload": w.name, "pos": pos, "B": B, "H": H, "d": d, "N": N},
                      "roofline": {"kernel": "decode_step_kernel", "bound": "hbm", "achieved": gbs,
                                   "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                                   "peak_kind": "HBM copy (%s)" % pk_src,
                                   "bytes_per_launch": decode_step_bytes(w, pos)}}), flush=True)
    return 0


def decode_arm(args, w):
    """Time whole segments of decode steps (N single-token steps, the last one
    folding the segment into (M, z)), replayed as one CUDA graph so host launch
    overhead is not timed; inputs resident in HBM."""
    from compressive_memory_segment_b200 import binding as bd
    dev = torch.device("cuda", torch.cuda.current_device())
    B, H, N, d = w.B, w.H, w.N, w.d
    q, k, v = synth.make_qkv(w, dev, L=N)
    beta = synth.make_beta(w, dev)
    steps_q = [tuple(x[:, :, t].contiguous() for x in (q, k, v)) for t in range(N)]
    kc = torch.zeros((B, H, N, d), dtype=q.dtype, device=dev)
    vc = torch.zeros_like(kc)
    M = torch.zeros((B, H, d, d), dtype=torch.float32, device=dev)
    z = torch.zeros((B, H, d), dtype=torch.float32, device=dev)
    out = torch.empty((B, H, d), dtype=q.dtype, device=dev)
    shp = bd.make_shape(B, H, N, d, bd.INFINI_BF16 if w.dtype == "bf16" else bd.INFINI_F32)
    ws = torch.empty(bd.infini_attn_decode_workspace_size(shp), dtype=torch.uint8, device=dev)
    nbytes = ws.numel()

    def segment(stream):
        for t in range(N):
            rc = bd.infini_attn_decode_step(shp, *steps_q[t], beta, kc, vc, t, M, z, out, ws, nbytes, stream)
            if rc != 0:
                raise RuntimeError(bd.infini_attn_strerror(rc))

    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        for _ in range(args.warmup):
            segment(s)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
        segment(s)
    torch.cuda.synchronize(dev)
    st = bd.infini_attn_device_status(s)
    if st != 0:
        raise RuntimeError(bd.infini_attn_strerror(st))
    reps = max(1, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk, torch.cuda.stream(s):
        e0.record(s)
        for _ in range(reps):
            g.replay()  # launches on the current stream, s
        e1.record(s)
        torch.cuda.synchronize(dev)
    ms_seg = e0.elapsed_time(e1) / reps
    pk, pk_src = peaks()
    gbs = decode_bytes(w) / (ms_seg / 1000.0) / 1e9
    line = {
        "metric": "Infini-attn decode tokens/s (one segment of single-token steps incl. the fold)",
        "value": B * N / (ms_seg / 1000.0), "unit": "tokens/s", "n_gpus": 1, "steps": reps,
        "warmup": args.warmup, "ms_per_step": ms_seg, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": B, "H": H, "d": d, "N": N, "step": "one segment of %d decode steps" % N,
                   "launch": "CUDA graph of the segment's launches",
                   "l2": "no flush: the caches total %.2f GB > 126 MB L2" % (2 * kc.numel() * kc.element_size() / 1e9)},
        "us_per_token_step": 1000.0 * ms_seg / N,
        "roofline": {"kernel": "decode_step_kernel (+ fold)", "bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / pk["hbm_gbs"], "peak_kind": "HBM copy (%s)" % pk_src,
                     "traffic": None, "bytes_per_step": decode_bytes(w)},
        "clocks": clk.summary(), "gpu_launches": reps * (N + 2),
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- sequence-sharded arm

def sharded_arm(args, w, world, rank, dev, stream):
    """Each rank holds one block of consecutive segments of the workload's
    sequence; a step is the whole sequence's forward (state phase, one
    all-gather of the block totals over NCCL, exclusive sum, finish phase)."""
    import torch.distributed as dist
    from compressive_memory_segment_b200 import sharded
    q, k, v = synth.make_qkv(w, dev)
    blk = w.L // world
    sl = slice(rank * blk, (rank + 1) * blk)
    qb, kb, vb = (t[:, :, sl].contiguous() for t in (q, k, v))
    del q, k, v
    beta = synth.make_beta(w, dev)
    ph = sharded.CudaPhases(stream)
    ws = ph.workspace(qb, w.N)

    def step():
        return sharded.forward_sequence_sharded(qb, kb, vb, beta, w.N, phases=ph, workspace=ws)

    for _ in range(args.warmup):
        step()
    dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    dist.barrier()
    ms_step = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, dev)
    wc = work_counts(w)
    pk, pk_src = peaks()
    tflops = wc["flops"] / (ms_step / 1000.0) / 1e12
    line = {
        "metric": METRIC, "value": w.B * w.L / (ms_step / 1000.0), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "N": w.N, "L": w.L,
                   "parallelism": "sequence-sharded x%d (one all-gather of %d B per rank per step)"
                                  % (world, 4 * w.B * w.H * (w.d * w.d + w.d))},
        "tflops": tflops,
        "roofline": {"kernel": "whole step", "bound": "tensor", "achieved": tflops / world,
                     "peak": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]), "unit": "TFLOP/s per GPU",
                     "frac": tflops / world / pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                     "peak_kind": "sustained bf16 dense (%s)" % pk_src, "traffic": None},
        "clocks": clk.summary(), "gpu_launches": args.steps * 6,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- our arm

def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", type=int, default=0,
                    help="0 auto, 1 CUDA-core, 2 tensor-core, 3 tensor-core with the paired-query-tile attention kernel")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-pieces", type=int, default=16,
                    help="pieces (of whole segments) the end-to-end step pipelines the sequence in")
    ap.add_argument("--shard-sequence", action="store_true",
                    help="N > 1: split the workload's sequence into one block of segments per rank "
                         "(strong scaling, one all-gather of the block totals per call) instead of replicas")
    ap.add_argument("--backward", action="store_true",
                    help="time a training step, forward + backward (default workload hf_repro_bf16)")
    ap.add_argument("--decode", action="store_true",
                    help="time streaming decode steps (default workload decode_8b_bf16) instead of the forward")
    ap.add_argument("--decode-pos", type=int, default=-1,
                    help="with --decode: time single steps at this position of a pre-filled cache")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.backward:
        wname = args.workload if args.workload != DEFAULT_WORKLOAD else "hf_repro_bf16"
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        return backward_arm(args, synth.WORKLOADS[wname])
    if args.decode:
        wname = args.workload if args.workload != DEFAULT_WORKLOAD else "decode_8b_bf16"
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        if args.decode_pos >= 0:
            return decode_pos_arm(args, synth.WORKLOADS[wname], args.decode_pos)
        return decode_arm(args, synth.WORKLOADS[wname])
    w = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        return reference_arm(args, w)

    from compressive_memory_segment_b200 import binding as bd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local_rank)
    dist = init_dist("nccl")
    dev = torch.device("cuda", local_rank if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    shard = args.shard_sequence and world > 1
    if shard:
        if w.calls != 1 or w.S % world != 0:
            raise SystemExit("--shard-sequence needs a one-call workload whose %d segments divide by %d ranks"
                             % (w.S, world))
        return sharded_arm(args, w, world, rank, dev, stream)

    # Inputs, resident in HBM: the full sequence split into the workload's calls.
    q, k, v = synth.make_qkv(w, dev)
    beta = synth.make_beta(w, dev)
    per = w.L // w.calls
    chunks = [tuple(t[:, :, c * per:(c + 1) * per].contiguous() for t in (q, k, v)) for c in range(w.calls)]
    if w.calls > 1:
        del q, k, v
    B, H, d = w.B, w.H, w.d
    out = [torch.empty_like(ch[0]) for ch in chunks]
    Ms = [torch.empty((B, H, d, d), dtype=torch.float32, device=dev) for _ in range(w.calls)]
    zs = [torch.empty((B, H, d), dtype=torch.float32, device=dev) for _ in range(w.calls)]
    shp = bd.shape_of(chunks[0][0])
    path = args.path if args.path else bd.infini_attn_select_path(shp, w.N)
    nl = bd.infini_attn_launch_count(shp, w.N, path)
    assert nl > 0, bd.infini_attn_strerror(nl)
    ws_bytes = bd.infini_attn_workspace_size(shp, w.N)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def new_events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(nl + 1)]
        for e in evs:
            e.record(stream)  # creates the handle
        return evs

    def one_step(evsets=None):
        for c in range(w.calls):
            Mi = Ms[c - 1] if c > 0 else None
            zi = zs[c - 1] if c > 0 else None
            qc, kc, vc = chunks[c]
            if evsets is None:
                rc = bd.infini_attn_forward_ws(shp, qc, kc, vc, beta, Mi, zi, w.N, out[c], Ms[c], zs[c],
                                               ws, ws_bytes, path, stream)
            else:
                rc = bd.infini_attn_forward_traced(shp, qc, kc, vc, beta, Mi, zi, w.N, out[c], Ms[c], zs[c],
                                                   ws, ws_bytes, path, evsets[c], stream)
            if rc != 0:
                raise RuntimeError(bd.infini_attn_strerror(rc))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        one_step()
    barrier()
    st = bd.infini_attn_device_status(stream)
    if st != 0:
        raise RuntimeError("device status after warm-up: " + bd.infini_attn_strerror(st))

    # Timed region: K steps, events between kernel launches for per-kernel times.
    # Inputs smaller than twice the 126 MB L2 would be served from L2 on the
    # next step: then L2 is flushed (a 512 MB write) before every step and each
    # step is timed on its own, the flush outside the events.
    in_bytes = 3 * w.B * w.H * w.L * w.d * (2 if w.dtype == "bf16" else 4)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if in_bytes < 2 * L2_BYTES else None
    evsets = [[new_events() for _ in range(w.calls)] for _ in range(args.steps)]
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    with ClockSampler(dev.index) as clk:
        for i in range(args.steps):
            if flush is not None or i == 0:
                if flush is not None:
                    flush.fill_(i & 0xff)
                starts[i].record(stream)
            one_step(evsets[i])
            if flush is not None or i == args.steps - 1:
                stops[i].record(stream)
        barrier()
    if flush is not None:
        ms_total = sum(a.elapsed_time(b) for a, b in zip(starts, stops))
    else:
        ms_total = starts[0].elapsed_time(stops[-1])
    st = bd.infini_attn_device_status(stream)
    if st != 0:
        raise RuntimeError("device status after timed region: " + bd.infini_attn_strerror(st))
    ms_total = max_over_ranks(ms_total, dist, dev)
    ms_step = ms_total / args.steps

    per_kernel = [0.0] * nl
    for i in range(args.steps):
        for c in range(w.calls):
            evs = evsets[i][c]
            for j in range(nl):
                per_kernel[j] += evs[j].elapsed_time(evs[j + 1])
    launches = args.steps * w.calls
    per_kernel = [x / launches for x in per_kernel]  # ms per launch
    clocks = clk.summary()

    wc = work_counts(w)
    tokens_step = w.B * w.L
    value = job_tokens_per_s(world, tokens_step, ms_step)
    pk, pk_src = peaks()
    tflops = wc["flops"] / (ms_step / 1000.0) / 1e12
    roof_t = max(wc["flops"] / (pk["bf16_tflops"] * 1e12), wc["bytes"] / (pk["hbm_gbs"] * 1e9))
    names = kernel_names(path, w)
    # Dominant kernel: the fused attention (last launch); tensor-core bound.
    attn_ms = per_kernel[-1]
    attn_flops_launch = wc["attn_flops"] / w.calls
    attn_tflops = attn_flops_launch / (attn_ms / 1000.0) / 1e12
    peak_sus = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    peak_t, peak_kind = tensor_peak(pk, pk_src, clocks)
    if path == 2 and w.d == 64:
        # HBM-bound shape: the single-pass kernel's algorithmic bytes per launch
        # (q, k, v read and out written once; the incoming state read and the
        # final state written once per (b, h), fp32).
        elt = 2
        a_bytes = (4.0 * w.B * w.H * (w.L // w.calls) * w.d * elt
                   + 2.0 * w.B * w.H * (w.d * w.d + w.d) * 4)
        gbs = a_bytes / (attn_ms / 1000.0) / 1e9
        roofline = {
            "kernel": names[-1], "bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / pk["hbm_gbs"], "peak_kind": "HBM copy (%s)" % pk_src, "traffic": None,
            "bytes_per_launch": a_bytes, "ms_per_launch": attn_ms,
        }
    elif path in (2, 3):
        roofline = {
            "kernel": names[-1], "bound": "tensor", "achieved": attn_tflops, "peak": peak_t, "unit": "TFLOP/s",
            "frac": attn_tflops / peak_t, "peak_kind": peak_kind,
            "frac_of_burst": attn_tflops / pk["bf16_tflops"], "frac_of_sustained": attn_tflops / peak_sus,
            "traffic": kernel_traffic(path),
            "flops_per_launch": attn_flops_launch, "ms_per_launch": attn_ms,
        }
    else:  # CUDA-core kernels: fp32 FFMA, or TF32 mma.sync tiles for bf16 inputs
        pk_note = "fp32 FFMA: 148 SMs x 128 lanes x 2 x 1965 MHz"
        if w.dtype == "bf16":
            pk_note += "; the score and P V tiles run on TF32 mma.sync (counted as the same work)"
        roofline = {
            "kernel": names[-1], "bound": "alu", "achieved": attn_tflops, "peak": FP32_FFMA_TFLOPS,
            "unit": "TFLOP/s", "frac": attn_tflops / FP32_FFMA_TFLOPS,
            "peak_kind": pk_note, "traffic": None,
            "flops_per_launch": attn_flops_launch, "ms_per_launch": attn_ms,
        }

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "N": w.N, "L": w.L, "calls": w.calls,
                   "path": {1: "cuda-core", 2: "tcgen05", 3: "tcgen05 paired"}.get(path, str(path)),
                   "l2": ("no flush: q, k, v total %.2f GB > 126 MB L2" % (in_bytes / 1e9)) if flush is None
                   else ("L2 flushed (512 MB write) before every step, each step timed alone: q, k, v total "
                         "%.1f MB" % (in_bytes / 1e6)),
                   "parallelism": "replica x%d" % world},
        "tflops": tflops, "step_roofline_frac": roof_t / (ms_step / 1000.0),
        "step_roofline": step_roofline(wc, pk, pk_src, ms_step),
        "kernel_ms_per_launch": dict(zip(names, per_kernel)),
        "roofline": roofline, "clocks": clocks, "gpu_launches": nl * launches,
    }

    # End to end through the public API: every step copies the whole sequence's
    # q, k, v from pinned host memory, runs the layer and copies out, M and z
    # back. The layer streams (only (M, z) crosses a call boundary), so the
    # sequence goes through as a pipeline of pieces of whole segments, each one
    # call carrying the state of the piece before it: the copy in of piece
    # p + 1, the forward of piece p and the copy out of piece p - 1 overlap on
    # three streams. Same calls, same work as one call per workload call.
    if not args.no_e2e:
        del chunks  # the pieces below hold the inputs
        torch.cuda.empty_cache()
        sub = max(1, min(w.S // w.calls, args.e2e_pieces // w.calls or 1))
        while (w.S // w.calls) % sub:
            sub -= 1
        seg_per_piece = w.S // w.calls // sub
        n_pieces = w.calls * sub
        Lp = seg_per_piece * w.N
        full = synth.make_qkv(w, "cpu")
        hq = [tuple(t[:, :, i * Lp:(i + 1) * Lp].contiguous().pin_memory() for t in full) for i in range(n_pieces)]
        del full
        dq_ = [tuple(torch.empty_like(t, device=dev) for t in hp) for hp in hq]
        dout_ = [torch.empty_like(hp[0], device=dev) for hp in hq]
        hout = [torch.empty(hp[0].shape, dtype=hp[0].dtype, pin_memory=True) for hp in hq]
        pM = [torch.empty((B, H, d, d), dtype=torch.float32, device=dev) for _ in range(n_pieces)]
        pz = [torch.empty((B, H, d), dtype=torch.float32, device=dev) for _ in range(n_pieces)]
        hM = torch.empty((B, H, d, d), dtype=torch.float32, pin_memory=True)
        hz = torch.empty((B, H, d), dtype=torch.float32, pin_memory=True)
        pshp = bd.shape_of(dq_[0][0])
        pws_bytes = bd.infini_attn_workspace_size(pshp, w.N)
        pws = torch.empty(pws_bytes, dtype=torch.uint8, device=dev)
        h2d = sum(t.numel() * t.element_size() for hp in hq for t in hp)
        d2h = sum(o.numel() * o.element_size() for o in hout) + hM.numel() * 4 + hz.numel() * 4
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(n_pieces)]
        ev_c = [torch.cuda.Event() for _ in range(n_pieces)]
        ev_o = [torch.cuda.Event() for _ in range(n_pieces)]
        first = [True]

        def e2e_step():
            for i in range(n_pieces):
                if not first[0]:
                    s_in.wait_event(ev_c[i])          # the previous step's forward is done with piece i
                with torch.cuda.stream(s_in):
                    for dst, src in zip(dq_[i], hq[i]):
                        dst.copy_(src, non_blocking=True)
                ev_in[i].record(s_in)
            for i in range(n_pieces):
                stream.wait_event(ev_in[i])
                if not first[0]:
                    stream.wait_event(ev_o[i])        # the previous step's copy out of piece i is done
                Mi = pM[i - 1] if i > 0 else None      # the state after the piece before
                zi = pz[i - 1] if i > 0 else None
                rc = bd.infini_attn_forward_ws(pshp, *dq_[i], beta, Mi, zi, w.N, dout_[i], pM[i], pz[i], pws,
                                               pws_bytes, path, stream)
                if rc != 0:
                    raise RuntimeError(bd.infini_attn_strerror(rc))
                ev_c[i].record(stream)
            for i in range(n_pieces):
                s_out.wait_event(ev_c[i])
                with torch.cuda.stream(s_out):
                    hout[i].copy_(dout_[i], non_blocking=True)
                ev_o[i].record(s_out)
            with torch.cuda.stream(s_out):
                hM.copy_(pM[-1], non_blocking=True)
                hz.copy_(pz[-1], non_blocking=True)
            first[0] = False

        e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        e_steps = max(1, min(args.steps, 5))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_in.wait_stream(s_out)  # start after the warm-up step has drained
        for _ in range(e_steps):
            e2e_step()
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        barrier()
        t_e = max_over_ranks(e0.elapsed_time(e1) / e_steps, dist, dev)
        line["e2e"] = {"value": job_tokens_per_s(world, tokens_step, t_e), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
                       "pipeline": "%d pieces of %d segments, copy in / forward / copy out on three streams"
                                   % (n_pieces, seg_per_piece)}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        nthreads = max(1, min(w.B * w.H, os.cpu_count() or 1))
        seg_count = max(1, min(w.S, 8 if w.N >= 1024 else 16))
        qh, kh, vh = synth.make_qkv(w, "cpu", L=seg_count * w.N)
        val, dt, T = oracle_sample_run(w, qh, kh, vh, beta.cpu(), seg_count, nthreads)
        line["cpu_baseline"] = {"value": val, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                                "sample": "all %d (b,h) pairs x first %d tokens of %s, %.1f s wall" % (
                                    w.B * w.H, T, w.name, dt)}

    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
