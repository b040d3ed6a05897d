"""Pins for the CPU oracle: checks against facts fixed by the mathematics or by
library routines, never against a retyped copy of the oracle's own formula.

Each pin takes the oracle's ``forward`` function as an argument so the same
checks can be run against copies of the oracle with a planted mistake (see
test_oracle_mutants.py) to show each mistake fails at least one pin.

Passages (page title and section):
  [HF] "Hugging Face Infini-Attention reproduction analysis", "Infini-Attention
       mechanism": Segmentation / Local Attention / Memory Retrieval (ELU + 1)
       / Integration (sigmoid gate on beta) / Memory Update / State Transfer.
  [KV] "KV linear-addition Infini-attention": causal dot-product attention per
       segment, scaled dot-product attention, linear long-term attention,
       streaming.
"""
import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _elu1(x):
    """sigma via the library ELU (torch), independent of the oracle's code."""
    return torch.nn.functional.elu(torch.as_tensor(x, dtype=torch.float64), alpha=1.0).numpy() + 1.0


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def pin_p1_single_segment_is_causal_sdpa(fwd):
    """L = N and beta = -inf: the layer is plain causal softmax attention with
    the 1/sqrt(d) scale [HF Local Attention; KV scaled dot-product]. Checked
    against torch's scaled_dot_product_attention in float64."""
    r = _rng(11)
    B, H, L, d = 2, 3, 24, 8
    q, k, v = (r.standard_normal((B, H, L, d)) for _ in range(3))
    beta = np.full(H, -np.inf)
    out, _, _ = fwd(q, k, v, beta, seg_len=L)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True).numpy()
    assert _rel(out, ref) < 1e-12, _rel(out, ref)


def pin_p1b_segments_are_independent_attention(fwd):
    """beta = -inf with several segments: each segment is its own causal
    attention; no key of another segment is visible [HF Segmentation]."""
    r = _rng(12)
    B, H, N, S, d = 1, 2, 8, 3, 4
    q, k, v = (r.standard_normal((B, H, N * S, d)) for _ in range(3))
    out, _, _ = fwd(q, k, v, np.full(H, -np.inf), seg_len=N)
    for s in range(S):
        sl = slice(s * N, (s + 1) * N)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[:, :, sl]), torch.from_numpy(k[:, :, sl]),
            torch.from_numpy(v[:, :, sl]), is_causal=True).numpy()
        assert _rel(out[:, :, sl], ref) < 1e-12


def _amem_bruteforce(q, k, v, N, M_in=None, z_in=None):
    """A_mem for every row without forming M: for a row in segment s,
    sum over all earlier tokens j of (sigma(q).sigma(k_j)) v_j divided by the
    sum of sigma(q).sigma(k_j), plus the incoming state's share."""
    B, H, L, d = q.shape
    sq, sk = _elu1(q), _elu1(k)
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            for t in range(L):
                start = (t // N) * N
                w = sk[b, h, :start] @ sq[b, h, t]          # [start]
                num = w @ v[b, h, :start]                   # [d]
                den = w.sum()
                if M_in is not None:
                    num = num + sq[b, h, t] @ M_in[b, h]
                    den = den + sq[b, h, t] @ z_in[b, h]
                out[b, h, t] = 0.0 if den == 0 else num / den
    return out


def pin_p2_memory_only_matches_bruteforce(fwd):
    """beta = +inf: out is the retrieval alone; it must equal the kernel-sum
    form of linear attention over every earlier segment (and the incoming
    state), computed without the d x d matrix [HF Memory Retrieval; KV linear
    attention]."""
    r = _rng(21)
    B, H, N, S, d = 2, 2, 4, 4, 6
    q, k, v = (r.standard_normal((B, H, N * S, d)) for _ in range(3))
    beta = np.full(H, np.inf)
    out, _, _ = fwd(q, k, v, beta, seg_len=N)
    ref = _amem_bruteforce(q, k, v, N)
    assert _rel(out, ref) < 1e-12, _rel(out, ref)
    # With an incoming state (streaming) the state's share is added.
    M_in = r.standard_normal((B, H, d, d))
    z_in = np.abs(r.standard_normal((B, H, d))) + 1.0
    out2, _, _ = fwd(q, k, v, beta, M_in, z_in, seg_len=N)
    ref2 = _amem_bruteforce(q, k, v, N, M_in, z_in)
    assert _rel(out2, ref2) < 1e-12, _rel(out2, ref2)


def pin_p3_final_state_is_matmul_for_any_segment_length(fwd):
    """M_out = M_in + sigma(K)^T V and z_out = z_in + sum sigma(K) over all
    tokens, whatever the segment length [HF Memory Update, State Transfer]."""
    r = _rng(31)
    B, H, L, d = 1, 2, 64, 5
    q, k, v = (r.standard_normal((B, H, L, d)) for _ in range(3))
    M_in = r.standard_normal((B, H, d, d))
    z_in = np.abs(r.standard_normal((B, H, d)))
    sk = torch.from_numpy(_elu1(k))
    M_ref = M_in + torch.matmul(sk.transpose(-1, -2), torch.from_numpy(v)).numpy()
    z_ref = z_in + sk.sum(dim=2).numpy()
    for N in (1, 16, 64, L):
        _, M, z = fwd(q, k, v, np.zeros(H), M_in, z_in, seg_len=N)
        assert _rel(M, M_ref) < 1e-12 and _rel(z, z_ref) < 1e-12, (N, _rel(M, M_ref), _rel(z, z_ref))


def pin_p4_streaming_equals_one_call(fwd):
    """Feeding the sequence as consecutive calls that carry (M, z) gives
    exactly the single call's result [HF State Transfer; KV streaming]."""
    r = _rng(41)
    B, H, N, S, d = 2, 2, 8, 8, 4
    q, k, v = (r.standard_normal((B, H, N * S, d)) for _ in range(3))
    beta = r.standard_normal(H)
    out, M, z = fwd(q, k, v, beta, seg_len=N)
    Mc = zc = None
    parts = []
    for c in range(4):
        sl = slice(c * 2 * N, (c + 1) * 2 * N)
        o, Mc, zc = fwd(q[:, :, sl], k[:, :, sl], v[:, :, sl], beta, Mc, zc, seg_len=N)
        parts.append(o)
    assert np.array_equal(np.concatenate(parts, axis=2), out)
    assert np.array_equal(Mc, M) and np.array_equal(zc, z)


def pin_p5_constant_values(fwd):
    """All value rows equal c: every softmax average and every retrieval is a
    convex combination of c, so segments s >= 1 output c; segment 0 from the
    zero state has no memory (A_mem = 0 by the zero-denominator rule) and
    outputs (1 - g) c."""
    r = _rng(51)
    B, H, N, S, d = 1, 3, 4, 3, 5
    q = r.standard_normal((B, H, N * S, d))
    k = r.standard_normal((B, H, N * S, d))
    c = r.standard_normal(d)
    v = np.broadcast_to(c, (B, H, N * S, d)).copy()
    beta = np.array([-1.5, 0.0, 2.0])
    out, _, _ = fwd(q, k, v, beta, seg_len=N)
    g = 1.0 / (1.0 + np.exp(-beta))
    for h in range(H):
        assert np.allclose(out[0, h, N:], c, rtol=0, atol=1e-13)
        assert np.allclose(out[0, h, :N], (1 - g[h]) * c, rtol=0, atol=1e-13)


def pin_p6_linear_in_values(fwd):
    """Scaling V by alpha scales out and M by alpha and leaves z unchanged."""
    r = _rng(61)
    B, H, N, S, d = 1, 2, 4, 3, 4
    q, k, v = (r.standard_normal((B, H, N * S, d)) for _ in range(3))
    beta = r.standard_normal(H)
    o1, M1, z1 = fwd(q, k, v, beta, seg_len=N)
    o2, M2, z2 = fwd(q, k, 3.0 * v, beta, seg_len=N)
    assert _rel(o2, 3.0 * o1) < 1e-13 and _rel(M2, 3.0 * M1) < 1e-13
    assert np.array_equal(z1, z2)


def pin_p7_hand_case(fwd):
    """d = 1, N = 1: the softmax over one key returns v_t; sigma(q) cancels in
    A_mem, leaving the sigma(k)-weighted mean of the earlier values. The
    fixture holds values worked out by hand."""
    with open(os.path.join(GOLDEN, "hand_d1_n1.json")) as f:
        cases = json.load(f)["cases"]
    for cs in cases:
        q = np.array(cs["q"], dtype=np.float64).reshape(1, 1, -1, 1)
        k = np.array(cs["k"], dtype=np.float64).reshape(1, 1, -1, 1)
        v = np.array(cs["v"], dtype=np.float64).reshape(1, 1, -1, 1)
        beta = np.array([float(cs["beta"])])
        out, M, z = fwd(q, k, v, beta, seg_len=1)
        assert np.allclose(out.reshape(-1), cs["out"], rtol=1e-14, atol=1e-14), (cs["name"], out.reshape(-1))
        assert np.allclose(M.reshape(-1), cs["M_out"], rtol=1e-14), cs["name"]
        assert np.allclose(z.reshape(-1), cs["z_out"], rtol=1e-14), cs["name"]


def pin_p8_earlier_segment_order_is_irrelevant(fwd):
    """Permuting tokens inside an earlier segment leaves every later
    segment's retrieval unchanged: the memory is a sum over tokens."""
    r = _rng(81)
    B, H, N, S, d = 1, 2, 6, 3, 4
    q, k, v = (r.standard_normal((B, H, N * S, d)) for _ in range(3))
    beta = np.full(H, np.inf)
    o1, M1, z1 = fwd(q, k, v, beta, seg_len=N)
    perm = np.concatenate([r.permutation(N), np.arange(N, N * S)])
    o2, M2, z2 = fwd(q[:, :, perm], k[:, :, perm], v[:, :, perm], beta, seg_len=N)
    assert _rel(o2[:, :, N:], o1[:, :, N:]) < 1e-13
    assert _rel(M2, M1) < 1e-13 and _rel(z2, z1) < 1e-13


def pin_p9_gate_blend(fwd):
    """out(beta) = sigmoid(beta) out(+inf) + (1 - sigmoid(beta)) out(-inf):
    the gate mixes the two branches and nothing else depends on beta
    [HF Integration]. Also pins the gate's orientation: large beta -> memory."""
    r = _rng(91)
    B, H, N, S, d = 1, 2, 4, 3, 4
    q, k, v = (r.standard_normal((B, H, N * S, d)) for _ in range(3))
    beta = np.array([0.7, -2.3])
    o, _, _ = fwd(q, k, v, beta, seg_len=N)
    o_mem, _, _ = fwd(q, k, v, np.full(H, np.inf), seg_len=N)
    o_dot, _, _ = fwd(q, k, v, np.full(H, -np.inf), seg_len=N)
    g = (1.0 / (1.0 + np.exp(-beta))).reshape(1, H, 1, 1)
    assert _rel(o, g * o_mem + (1 - g) * o_dot) < 1e-13
    # Orientation: beta=+inf reproduces the memory-only brute force.
    assert _rel(o_mem, _amem_bruteforce(q, k, v, N)) < 1e-12


def pin_p10_bf16_inputs_widen_exactly(fwd):
    """bf16 bit patterns are widened exactly: the result equals the run on the
    same values given as float64."""
    r = _rng(101)
    B, H, N, S, d = 1, 2, 8, 2, 8
    x = torch.from_numpy(r.standard_normal((3, B, H, N * S, d))).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    dbl = x.to(torch.float64).numpy()
    beta = r.standard_normal(H)
    o1, M1, z1 = fwd(bits[0], bits[1], bits[2], beta, seg_len=N)
    o2, M2, z2 = fwd(dbl[0], dbl[1], dbl[2], beta, seg_len=N)
    assert np.array_equal(o1, o2) and np.array_equal(M1, M2) and np.array_equal(z1, z2)


ALL_PINS = [
    pin_p1_single_segment_is_causal_sdpa,
    pin_p1b_segments_are_independent_attention,
    pin_p2_memory_only_matches_bruteforce,
    pin_p3_final_state_is_matmul_for_any_segment_length,
    pin_p4_streaming_equals_one_call,
    pin_p5_constant_values,
    pin_p6_linear_in_values,
    pin_p7_hand_case,
    pin_p8_earlier_segment_order_is_irrelevant,
    pin_p9_gate_blend,
    pin_p10_bf16_inputs_widen_exactly,
]
