"""Pins for the oracle's decode step: one new token at position pos of its
segment attends causally to the segment's cached keys 0..pos, reads the memory
of earlier segments, and after the segment's last token the segment is folded
into (M, z) [HF State Transfer; KV streaming].

Each pin takes the oracle's forward function ``fwd`` (with the decode step as
``fwd.decode``) so test_oracle_decode.py can run them against copies of the
oracle with a planted mistake.
"""
import math

import numpy as np
import torch

from tests.oracle_pins import _amem_bruteforce, _rel


def _decode_sequence(dec, q, k, v, beta, N, M0=None, z0=None):
    """Feed a [B, H, L, d] sequence token by token, keeping the current
    segment's keys and values in a cache; returns out [B, H, L, d] and the
    final state."""
    B, H, L, d = q.shape
    kc = np.zeros((B, H, N, d), q.dtype)
    vc = np.zeros((B, H, N, d), q.dtype)
    M = np.zeros((B, H, d, d)) if M0 is None else M0.copy()
    z = np.zeros((B, H, d)) if z0 is None else z0.copy()
    out = np.empty((B, H, L, d))
    for t in range(L):
        pos = t % N
        o, M, z = dec(q[:, :, t], k[:, :, t], v[:, :, t], kc, vc, pos, beta, M, z)
        out[:, :, t] = o
        kc[:, :, pos] = k[:, :, t]
        vc[:, :, pos] = v[:, :, t]
    return out, M, z


def pin_d1_decode_matches_forward(fwd):
    """Decoding a sequence token by token gives the forward's output rows and
    final state, bit for bit (same definition, same summation order)."""
    r = np.random.default_rng(71)
    B, H, N, S, d = 2, 2, 5, 3, 6
    q, k, v = (r.standard_normal((B, H, N * S, d)) for _ in range(3))
    beta = r.standard_normal(H)
    M0 = r.standard_normal((B, H, d, d))
    z0 = np.abs(r.standard_normal((B, H, d))) + 1.0
    ref_out, ref_M, ref_z = fwd(q, k, v, beta, M0, z0, seg_len=N)
    out, M, z = _decode_sequence(fwd.decode, q, k, v, beta, N, M0, z0)
    assert np.array_equal(out, ref_out), _rel(out, ref_out)
    assert np.array_equal(M, ref_M) and np.array_equal(z, ref_z)


def pin_d2_first_token_zero_state(fwd):
    """pos = 0 with the zero state: one visible key (softmax weight 1) and a
    zero retrieval denominator, so out = (1 - sigmoid(beta)) v exactly."""
    r = np.random.default_rng(72)
    B, H, N, d = 2, 3, 4, 8
    q, k, v = (r.standard_normal((B, H, d)) for _ in range(3))
    beta = r.standard_normal(H)
    cache = np.zeros((B, H, N, d))
    out, M, z = fwd.decode(q, k, v, cache, cache, 0, beta, np.zeros((B, H, d, d)), np.zeros((B, H, d)))
    g = 1.0 / (1.0 + np.exp(-beta))
    assert np.allclose(out, (1.0 - g)[None, :, None] * v, rtol=0, atol=1e-15)
    assert not M.any() and not z.any()


def pin_d3_local_part_is_causal_sdpa(fwd):
    """beta = -inf: the step at position pos equals row pos of causal softmax
    attention over the segment (torch SDPA in float64)."""
    r = np.random.default_rng(73)
    B, H, N, d = 1, 2, 7, 8
    q, k, v = (r.standard_normal((B, H, N, d)) for _ in range(3))
    beta = np.full(H, -np.inf)
    out, _, _ = _decode_sequence(fwd.decode, q, k, v, beta, N)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True).numpy()
    assert _rel(out, ref) < 1e-12


def pin_d4_memory_part_is_bruteforce(fwd):
    """beta = +inf: the step's output is the memory-only sum over all tokens of
    earlier segments, computed without forming M."""
    r = np.random.default_rng(74)
    B, H, N, S, d = 1, 2, 4, 3, 5
    q, k, v = (r.standard_normal((B, H, N * S, d)) for _ in range(3))
    beta = np.full(H, np.inf)
    out, _, _ = _decode_sequence(fwd.decode, q, k, v, beta, N)
    ref = _amem_bruteforce(q, k, v, N)
    assert _rel(out[:, :, N:], ref[:, :, N:]) < 1e-12
    assert np.all(out[:, :, :N] == 0.0)  # no memory yet: A_mem = 0 and g = 1


ALL_DECODE_PINS = [pin_d1_decode_matches_forward, pin_d2_first_token_zero_state,
                   pin_d3_local_part_is_causal_sdpa, pin_d4_memory_part_is_bruteforce]
