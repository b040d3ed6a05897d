"""Seeded synthetic inputs for the Infini-attention layer forward.

This module holds the workload shapes and a counter-based random generator and
nothing of the layer's arithmetic, so the CUDA path and the CPU oracle can be
fed the very same bits.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used in counter mode -- element ``c`` of a
stream with key ``K`` is ``mix64(K + (c + 1) * GAMMA)`` -- followed by the
Box-Muller transform for normals. Every value is a pure function of (seed,
stream, index), so any slice can be regenerated on the CPU or on the GPU.
Integer arithmetic is done in int64 torch tensors (two's-complement wrap on
multiply, masked logical shifts); transcendental steps are float64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Optional

import torch

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB

# Stream ids: one independent sub-stream per tensor of a workload.
STREAM_Q, STREAM_K, STREAM_V, STREAM_BETA, STREAM_OUTLIER, STREAM_MIN, STREAM_ZIN = 1, 2, 3, 4, 5, 6, 7


def _s64(x: int) -> int:
    """Python int in [0, 2^64) -> the same bits as a signed int64."""
    x &= MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


def mix64_int(x: int) -> int:
    """SplitMix64 finaliser on Python ints (exact mod 2^64); the reference the
    tensor version is checked against."""
    z = x & MASK64
    z = ((z ^ (z >> 30)) * _C1) & MASK64
    z = ((z ^ (z >> 27)) * _C2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    return mix64_int(((seed & 0xFFFFFFFFFFFF) << 8) + stream)


def _srl(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 bits."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _s64(_C1)
    z = (z ^ _srl(z, 27)) * _s64(_C2)
    return z ^ _srl(z, 31)


def raw64(key: int, start: int, n: int, device) -> torch.Tensor:
    """Counters start..start+n-1 of the stream with the given key, as int64 bits."""
    c = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    return _mix64(c * _s64(GAMMA) + _s64(key))


def uniform53(bits: torch.Tensor) -> torch.Tensor:
    """Top 53 bits -> float64 in [0, 1)."""
    return _srl(bits, 11).to(torch.float64) * (2.0 ** -53)


def uniform(seed: int, stream: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    return uniform53(raw64(stream_key(seed, stream), start, n, device))


def normal(seed: int, stream: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    """Standard normals; element i uses counters 2i and 2i+1 (Box-Muller)."""
    key = stream_key(seed, stream)
    bits = raw64(key, 2 * start, 2 * n, device).view(n, 2)
    u1 = (_srl(bits[:, 0], 11).to(torch.float64) + 0.5) * (2.0 ** -53)  # (0, 1)
    u2 = uniform53(bits[:, 1])
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


@dataclass(frozen=True)
class Workload:
    """One workload: shapes, value recipe and seed."""
    name: str
    B: int
    H: int
    d: int
    N: int           # segment length
    S: int           # segments per (b, h) over the whole sequence
    dtype: str       # "f32" or "bf16"
    seed: int
    qkv_scale: float = 1.0          # Q, K, V ~ N(0, 1) * qkv_scale
    beta: str = "zero"              # "zero" | "normal" | "uniform:<a>"
    outlier_p: float = 0.0          # probability that a K row is scaled ...
    outlier_scale: float = 1.0      # ... by this factor
    calls: int = 1                  # the sequence is fed in this many streamed calls
    note: str = ""

    @property
    def L(self) -> int:
        return self.N * self.S

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads of the layer's specification, seeds 1001..1005.
WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload("tiny_f32", 1, 1, 64, 64, 4, "f32", 1001,
                         note="B1 H1 d64 N64 L256, N(0,1), beta=0, zero state"),
    "hf_repro_bf16": Workload("hf_repro_bf16", 8, 12, 64, 64, 16, "bf16", 1002,
                              qkv_scale=1.0 / 8.0, beta="uniform:3",
                              note="HF reproduction shape: segment 64, 16 segments"),
    "llama8b_32k_bf16": Workload("llama8b_32k_bf16", 1, 32, 128, 2048, 16, "bf16", 1003,
                                 beta="normal", calls=4,
                                 note="8B-like layer, L=32768 fed as 4 calls of 8192"),
    "mid_8k_outlier_bf16": Workload("mid_8k_outlier_bf16", 16, 16, 128, 1024, 8, "bf16", 1004,
                                    beta="uniform:4", outlier_p=0.01, outlier_scale=8.0,
                                    note="1% of K rows scaled x8"),
    "stream_1m_bf16": Workload("stream_1m_bf16", 1, 8, 128, 2048, 512, "bf16", 1005,
                               beta="normal", note="L=1,048,576 in one call"),
    # The 1M workload's first 64K tokens: the same kernels and tile shapes at
    # 1/16 of the size, small enough for a full profiler capture.
    # Streaming decode: one segment of single-token steps for 8 sequences of an
    # 8B-like layer (32 heads, d = 128, segment 2048), state carried in (M, z).
    "decode_8b_bf16": Workload("decode_8b_bf16", 8, 32, 128, 2048, 1, "bf16", 1006, beta="normal",
                               note="B8 H32 d128 N2048: 2048 decode steps incl. one fold"),
    "profile_64k_bf16": Workload("profile_64k_bf16", 1, 8, 128, 2048, 32, "bf16", 1005,
                                 beta="normal", note="1/16 of the 1M workload, for profiling"),
}


def _fill_normal(out: torch.Tensor, seed: int, stream: int, scale: float, chunk: int = 1 << 24):
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        x = normal(seed, stream, m, out.device, start=s)
        if scale != 1.0:
            x = x * scale
        flat[s:s + m] = x.to(out.dtype)


def make_beta(w: Workload, device="cpu") -> torch.Tensor:
    if w.beta == "zero":
        return torch.zeros(w.H, dtype=torch.float32, device=device)
    if w.beta == "normal":
        return normal(w.seed, STREAM_BETA, w.H, device).to(torch.float32)
    if w.beta.startswith("uniform:"):
        a = float(w.beta.split(":")[1])
        return (uniform(w.seed, STREAM_BETA, w.H, device) * (2 * a) - a).to(torch.float32)
    raise ValueError(w.beta)


def make_qkv(w: Workload, device="cpu", L: Optional[int] = None, B: Optional[int] = None,
             H: Optional[int] = None):
    """Q, K, V of shape [B, H, L, d] in the workload dtype (values are a pure
    function of the element index in the full-size tensor only when B, H and L
    are the workload's own; overriding them gives a smaller case with the same
    recipe)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    L = w.L if L is None else L
    shape = (B, H, L, w.d)
    q = torch.empty(shape, dtype=w.torch_dtype, device=device)
    k = torch.empty(shape, dtype=w.torch_dtype, device=device)
    v = torch.empty(shape, dtype=w.torch_dtype, device=device)
    _fill_normal(q, w.seed, STREAM_Q, w.qkv_scale)
    _fill_normal(v, w.seed, STREAM_V, w.qkv_scale)
    if w.outlier_p > 0.0:
        # Scale whole K rows: generate in float64, scale the chosen rows, round once.
        kk = torch.empty(shape, dtype=torch.float64, device=device)
        _fill_normal(kk, w.seed, STREAM_K, w.qkv_scale)
        rows = B * H * L
        hit = uniform(w.seed, STREAM_OUTLIER, rows, device) < w.outlier_p
        kk.view(rows, w.d)[hit] *= w.outlier_scale
        k.copy_(kk.to(w.torch_dtype))
        del kk
    else:
        _fill_normal(k, w.seed, STREAM_K, w.qkv_scale)
    return q, k, v


def make_state(w: Workload, device="cpu", scale: float = 1.0, B=None, H=None):
    """A non-zero incoming state (M_in, z_in) in fp32 for streaming tests:
    M_in ~ N(0,1)*scale, z_in = |N(0,1)|*scale + scale (positive, as a sum of
    sigma values always is)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    M = torch.empty((B, H, w.d, w.d), dtype=torch.float32, device=device)
    z = torch.empty((B, H, w.d), dtype=torch.float32, device=device)
    _fill_normal(M, w.seed, STREAM_MIN, scale)
    zz = normal(w.seed, STREAM_ZIN, B * H * w.d, device).abs() * scale + scale
    z.view(-1).copy_(zz.to(torch.float32))
    return M, z


def bf16_bits(t: torch.Tensor):
    """A bf16 tensor's bit patterns as a numpy uint16 array (for the oracle)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
