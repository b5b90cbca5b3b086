"""Pins for the front-end oracle (oracle/frontend.py), no GPU needed: closed forms of
softplus and SiLU, convolutions with one-hot filters (identity, pure delays), the bias,
the conv-state hand-off between pieces of a sequence, and a brute-force loop on a tiny
input.  The definitions are those of "Engineering Hybrid State-Space Models", section 3
(width-4 conv + SiLU; Delta = Softplus(Linear(x) + bias); convState [dConv - 1, dModel])."""
import math

import numpy as np

import oracle


def test_softplus_closed_forms():
    assert oracle.softplus(0.0) == math.log(2.0)
    assert abs(oracle.softplus(1.0) - math.log(1.0 + math.e)) < 1e-15
    assert oracle.softplus(800.0) == 800.0                       # no overflow; log(1 + e^z) -> z
    assert abs(oracle.softplus(-40.0) - math.exp(-40.0)) < 1e-30  # -> e^z for very negative z
    z = np.linspace(-5, 5, 11)
    assert np.allclose(oracle.softplus(z) - oracle.softplus(-z), z)  # softplus(z) - softplus(-z) = z


def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    v = np.linspace(-6, 6, 13)
    assert np.allclose(oracle.silu(v) - oracle.silu(-v), v)  # silu(v) - silu(-v) = v


def test_conv_with_one_hot_filters_is_identity_and_delay():
    rng = np.random.default_rng(1)
    u = rng.standard_normal((2, 9, 5))
    ident = np.zeros((5, 4)); ident[:, 3] = 1.0
    out, st = oracle.causal_conv(u, ident)
    assert np.array_equal(out, u)
    assert np.array_equal(st, u[:, -3:])
    for lag in (1, 2, 3):
        w = np.zeros((5, 4)); w[:, 3 - lag] = 1.0
        out, _ = oracle.causal_conv(u, w)
        assert np.array_equal(out[:, lag:], u[:, :-lag])
        assert np.array_equal(out[:, :lag], np.zeros_like(out[:, :lag]))  # zero history


def test_conv_bias_and_history():
    rng = np.random.default_rng(2)
    u = rng.standard_normal((1, 4, 3))
    hist = rng.standard_normal((1, 3, 3))
    w = np.zeros((3, 4)); w[:, 0] = 1.0   # out[t] = u[t - 3]: the history for t < 3
    bias = np.array([0.5, -1.0, 2.0])
    out, st = oracle.causal_conv(u, w, bias, hist)
    assert np.array_equal(out[:, :3], hist + bias)
    assert np.array_equal(out[:, 3], u[:, 0] + bias)
    assert np.array_equal(st, u[:, 1:])


def test_conv_state_hand_off_between_pieces():
    """Processing a sequence in two pieces, the second from the first's conv state,
    equals one pass (also when a piece is shorter than the filter)."""
    rng = np.random.default_rng(3)
    u = rng.standard_normal((2, 20, 6))
    w = rng.standard_normal((6, 4))
    bias = rng.standard_normal(6)
    full, st_full = oracle.causal_conv(u, w, bias)
    for cut in (1, 2, 3, 7, 19):
        a, st = oracle.causal_conv(u[:, :cut], w, bias)
        bb, st2 = oracle.causal_conv(u[:, cut:], w, bias, st)
        assert np.allclose(np.concatenate([a, bb], axis=1), full, rtol=0, atol=1e-14)
        assert np.array_equal(st2, st_full)


def test_frontend_against_a_brute_force_loop():
    rng = np.random.default_rng(4)
    b, L, H, P, G, N = 2, 5, 2, 3, 1, 4
    Cch = H * P + 2 * G * N
    xbc = rng.standard_normal((b, L, Cch))
    w = rng.standard_normal((Cch, 4))
    bias = rng.standard_normal(Cch)
    dt_raw = rng.standard_normal((b, L, H))
    dt_bias = rng.standard_normal(H)
    hist = rng.standard_normal((b, 3, Cch))
    x, B, C, dt, st = oracle.frontend(xbc, w, bias, dt_raw, dt_bias, H, P, G, N, state=hist)
    for bi in range(b):
        for t in range(L):
            for c in range(Cch):
                acc = bias[c]
                for k in range(4):
                    tt = t - 3 + k
                    acc += w[c, k] * (xbc[bi, tt, c] if tt >= 0 else hist[bi, 3 + tt, c])
                act = acc / (1.0 + math.exp(-acc))
                if c < H * P:
                    got = x[bi, t, c // P, c % P]
                elif c < H * P + G * N:
                    got = B[bi, t, (c - H * P) // N, (c - H * P) % N]
                else:
                    got = C[bi, t, (c - H * P - G * N) // N, (c - H * P - G * N) % N]
                assert abs(got - act) < 1e-12
            for h in range(H):
                assert abs(dt[bi, t, h] - math.log1p(math.exp(dt_raw[bi, t, h] + dt_bias[h]))) < 1e-12
    assert np.array_equal(st, xbc[:, -3:])
