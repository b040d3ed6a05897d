"""Pins for the oracle's backward: the gradients it returns against central
finite differences of the oracle's forward (itself pinned in oracle_pins.py).
A scalar loss L = sum(W_o * out) + sum(W_M * M_out) + sum(W_z * z_out) with
random weights makes every input's gradient observable; the backward gets
dout = W_o, dM_out = W_M, dz_out = W_z.

Each pin takes the oracle's forward function ``fwd`` (its backward as
``fwd.backward``) so test_oracle_backward.py can run them against copies of
the oracle with a planted mistake."""
import numpy as np


def _loss(fwd, q, k, v, beta, M_in, z_in, N, W):
    out, M, z = fwd(q, k, v, beta, M_in, z_in, seg_len=N)
    return float(np.sum(W[0] * out) + np.sum(W[1] * M) + np.sum(W[2] * z))


def _fd_check(fwd, seed, with_state, beta_scale=1.0, h=1e-6):
    r = np.random.default_rng(seed)
    B, H, N, S, d = 1, 2, 4, 3, 3
    L = N * S
    q, k, v = (r.standard_normal((B, H, L, d)) for _ in range(3))
    beta = r.standard_normal(H) * beta_scale
    M_in = r.standard_normal((B, H, d, d)) if with_state else None
    z_in = (np.abs(r.standard_normal((B, H, d))) + 0.5) if with_state else None
    W = (r.standard_normal((B, H, L, d)), r.standard_normal((B, H, d, d)), r.standard_normal((B, H, d)))
    dq, dk, dv, dbeta, dM_in, dz_in = fwd.backward(q, k, v, beta, W[0], M_in, z_in, W[1], W[2], seg_len=N)
    args = dict(q=q, k=k, v=v, beta=beta, M_in=M_in, z_in=z_in)
    grads = dict(q=dq, k=dk, v=dv, beta=dbeta, M_in=dM_in, z_in=dz_in)
    worst = 0.0
    for name, x in args.items():
        if x is None:
            continue
        g = grads[name]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            orig = x[idx]
            x[idx] = orig + h
            lp = _loss(fwd, args["q"], args["k"], args["v"], args["beta"], args["M_in"], args["z_in"], N, W)
            x[idx] = orig - h
            lm = _loss(fwd, args["q"], args["k"], args["v"], args["beta"], args["M_in"], args["z_in"], N, W)
            x[idx] = orig
            num[idx] = (lp - lm) / (2 * h)
        scale = max(np.max(np.abs(num)), 1e-3)
        worst = max(worst, float(np.max(np.abs(num - g)) / scale))
        assert np.max(np.abs(num - g)) <= 1e-6 * scale, (name, float(np.max(np.abs(num - g))), scale)
    return worst


def pin_b1_gradients_match_finite_differences(fwd):
    """All gradients (q, k, v, beta, M_in, z_in) with an incoming state and a
    gradient on the output state, three segments."""
    _fd_check(fwd, 81, with_state=True)


def pin_b2_zero_state_first_segment(fwd):
    """The zero state: segment 0 has a zero retrieval denominator, so its
    memory part is identically 0 and passes no gradient; later segments do."""
    _fd_check(fwd, 82, with_state=False)


def pin_b3_saturated_gate(fwd):
    """Large |beta|: the gate's derivative g (1 - g) is tiny, the split of the
    gradient between the two branches must follow g."""
    _fd_check(fwd, 83, with_state=True, beta_scale=6.0)


ALL_BACKWARD_PINS = [pin_b1_gradients_match_finite_differences, pin_b2_zero_state_first_segment,
                     pin_b3_saturated_gate]
