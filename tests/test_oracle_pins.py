"""Pins for the fp64 CPU oracle (no GPU needed).

The oracle's sequential recurrence is what the CUDA path is checked against, so it is
itself checked here against things other than itself:
  * values worked out by hand (tests/golden/hand_worked_ssd.json),
  * a closed form (geometric decay with constant dt and one-hot B/C),
  * the special cases of the selection mechanism ("Mamba and Selective State Space
    Models", section 4: dt -> 0 keeps the state, a large step flushes it),
  * trivial cases (B = 0, C = 0, a single token), linearity in x, head permutation,
  * the semiseparable and chunked forms ("Engineering Hybrid State-Space Models",
    section 2: the two are algebraically the same layer) and chunk-size invariance,
  * the prefill/decode split: a prefix followed by single-token steps equals the full
    prefill ("Compiler-First State Space Duality ...", abstract: the O(1) cache).
Finally every independent pin is run against recurrences with one planted mistake each
(tests/oracle_mutants.c); each mistake must make at least one pin fail.
"""
import ctypes
import json
import math
import os
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "hand_worked_ssd.json")


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    scale = max(np.abs(b).max(), 1e-300)
    return np.abs(a - b).max() / scale


def _rand_problem(rng, b=2, L=37, H=4, P=3, N=5, G=2, dt_range=(0.01, 0.5)):
    x = rng.standard_normal((b, L, H, P))
    dt = rng.uniform(*dt_range, (b, L, H))
    A = -rng.uniform(0.5, 3.0, H)
    B = rng.standard_normal((b, L, G, N))
    C = rng.standard_normal((b, L, G, N))
    D = rng.standard_normal(H)
    return x, dt, A, B, C, D


def _parse_A(v):
    if isinstance(v, str):
        assert v.startswith("-ln")
        return -math.log(float(v[3:]))
    return float(v)


# ------------------------------------------------------------------ pin functions
# Each takes `rec(x, dt, A, B, C, D, state=None) -> (y, final_state)` and raises
# AssertionError if the recurrence it is given is wrong.

def pin_golden(rec):
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        A = np.array([_parse_A(v) for v in case["A"]])
        args = [np.array(case[k], dtype=np.float64) for k in ("x", "dt")]
        y, st = rec(args[0], args[1], A, np.array(case["B"], float), np.array(case["C"], float),
                    np.array(case["D"], float))
        assert np.allclose(y, np.array(case["y"]), rtol=0, atol=1e-12), case["name"]
        assert np.allclose(st, np.array(case["final_state"]), rtol=0, atol=1e-12), case["name"]


def pin_closed_form(rec):
    """Constant dt and A, x = 1, group 0 has B = e_i, group 1 has B = e_k, C = e_j for
    all groups: with a = exp(dt A), the state is the geometric sum
    h_t[p][i] = dt (1 - a^(t+1)) / (1 - a) and y_t = [i == j] h_t + D."""
    b, L, H, P, N, G = 1, 50, 4, 2, 3, 2
    dtv, Av = 0.07, -1.3
    i0, i1, j = 1, 2, 1
    x = np.ones((b, L, H, P))
    dt = np.full((b, L, H), dtv)
    A = np.full(H, Av)
    B = np.zeros((b, L, G, N))
    B[:, :, 0, i0] = 1.0
    B[:, :, 1, i1] = 1.0
    C = np.zeros((b, L, G, N))
    C[:, :, :, j] = 1.0
    D = np.array([0.5, -0.25, 2.0, 1.0])
    y, st = rec(x, dt, A, B, C, D)
    a = math.exp(dtv * Av)
    t = np.arange(L)
    geo = dtv * (1.0 - a ** (t + 1)) / (1.0 - a)
    for h in range(H):
        g = h // (H // G)
        i = i0 if g == 0 else i1
        for p in range(P):
            expect = (geo if i == j else 0.0) + D[h]
            assert np.allclose(y[0, :, h, p], expect, rtol=0, atol=1e-12), (h, p)
            hrow = np.zeros(N)
            hrow[i] = geo[-1]
            assert np.allclose(st[0, h, p], hrow, rtol=0, atol=1e-12), (h, p)


def pin_dt_to_zero(rec):
    """dt -> 0: exp(dt A) -> 1 and dt B -> 0, so the state is kept and y = C h0 + D x."""
    rng = np.random.default_rng(1)
    x, _, A, B, C, D = _rand_problem(rng, b=1, L=9, H=2, P=3, N=4, G=1)
    dt = np.full((1, 9, 2), 1e-13)
    h0 = rng.standard_normal((1, 2, 3, 4))
    y, st = rec(x, dt, A, B, C, D, state=h0)
    assert _rel(st, h0) < 1e-10
    expect = np.einsum("btn,bhpn->bthp", C[:, :, 0], h0) + D[None, None, :, None] * x
    assert np.allclose(y, expect, rtol=0, atol=1e-10 * np.abs(expect).max())


def pin_large_step_flushes(rec):
    """dt |A| large: exp(dt A) ~ 0, so h_t = dt x_t B_t^T (the past is forgotten) and
    y_t = dt (C_t . B_t) x_t + D x_t."""
    rng = np.random.default_rng(2)
    x, _, _, B, C, D = _rand_problem(rng, b=1, L=6, H=3, P=2, N=4, G=1)
    dt = np.full((1, 6, 3), 5.0)
    A = np.full(3, -20.0)  # exp(-100) ~ 4e-44
    h0 = rng.standard_normal((1, 3, 2, 4)) * 100
    y, st = rec(x, dt, A, B, C, D, state=h0)
    cb = np.einsum("btn,btn->bt", C[:, :, 0], B[:, :, 0])
    expect = 5.0 * cb[:, :, None, None] * x + D[None, None, :, None] * x
    assert np.allclose(y, expect, rtol=1e-12, atol=1e-12)
    expect_st = 5.0 * np.einsum("bhp,bn->bhpn", x[:, -1], B[:, -1, 0])
    assert np.allclose(st, expect_st, rtol=1e-12, atol=1e-12)


def pin_zero_B_or_C(rec):
    rng = np.random.default_rng(3)
    x, dt, A, B, C, D = _rand_problem(rng, b=2, L=11, H=4, P=3, N=5, G=2)
    y, st = rec(x, dt, A, np.zeros_like(B), C, D)
    assert np.allclose(y, D[None, None, :, None] * x, rtol=0, atol=1e-14)
    assert np.abs(st).max() == 0.0
    h0 = rng.standard_normal((2, 4, 3, 5))
    y, st = rec(x, dt, A, B, np.zeros_like(C), D, state=h0)
    assert np.allclose(y, D[None, None, :, None] * x, rtol=0, atol=1e-14)


def pin_single_token(rec):
    """L = 1: h = exp(dt A) h0 + dt x B^T and y = C . h + D x, written out per element."""
    rng = np.random.default_rng(4)
    x, dt, A, B, C, D = _rand_problem(rng, b=2, L=1, H=4, P=3, N=5, G=2)
    h0 = rng.standard_normal((2, 4, 3, 5))
    y, st = rec(x, dt, A, B, C, D, state=h0)
    for bi in range(2):
        for h in range(4):
            g = h // 2
            a = math.exp(dt[bi, 0, h] * A[h])
            for p in range(3):
                hrow = [a * h0[bi, h, p, n] + dt[bi, 0, h] * x[bi, 0, h, p] * B[bi, 0, g, n]
                        for n in range(5)]
                assert np.allclose(st[bi, h, p], hrow, rtol=1e-13, atol=1e-13)
                yv = sum(C[bi, 0, g, n] * hrow[n] for n in range(5)) + D[h] * x[bi, 0, h, p]
                assert abs(y[bi, 0, h, p] - yv) < 1e-12


def pin_linear_in_x(rec):
    rng = np.random.default_rng(5)
    x1, dt, A, B, C, D = _rand_problem(rng)
    x2 = rng.standard_normal(x1.shape)
    y1, s1 = rec(x1, dt, A, B, C, D)
    y2, s2 = rec(x2, dt, A, B, C, D)
    y3, s3 = rec(2.0 * x1 - 3.0 * x2, dt, A, B, C, D)
    assert _rel(y3, 2.0 * y1 - 3.0 * y2) < 1e-12
    assert _rel(s3, 2.0 * s1 - 3.0 * s2) < 1e-12


def pin_head_permutation(rec):
    """With one group, heads are independent: permuting heads (x, dt, A, D together)
    permutes the outputs and states the same way."""
    rng = np.random.default_rng(6)
    x, dt, A, B, C, D = _rand_problem(rng, b=1, L=13, H=5, P=2, N=3, G=1)
    perm = np.array([3, 0, 4, 1, 2])
    y, st = rec(x, dt, A, B, C, D)
    yp, stp = rec(x[:, :, perm], dt[:, :, perm], A[perm], B, C, D[perm])
    assert _rel(yp, y[:, :, perm]) < 1e-14
    assert _rel(stp, st[:, perm]) < 1e-14


INDEPENDENT_PINS = [pin_golden, pin_closed_form, pin_dt_to_zero, pin_large_step_flushes,
                    pin_zero_B_or_C, pin_single_token, pin_linear_in_x, pin_head_permutation]


def _forms():
    return {
        "recurrence": lambda *a, state=None: oracle.recurrence(*a, state=state),
        "quadratic": lambda *a, state=None: oracle.quadratic(*a, state=state),
        "chunked_q3": lambda *a, state=None: oracle.chunked(*a, 3, state=state),
        "chunked_q16": lambda *a, state=None: oracle.chunked(*a, 16, state=state),
    }


@pytest.mark.parametrize("form", list(_forms()))
@pytest.mark.parametrize("pin", INDEPENDENT_PINS, ids=lambda f: f.__name__)
def test_pin(form, pin):
    pin(_forms()[form])


# ------------------------------------------------------------------ duality / invariants

@pytest.mark.parametrize("chunk", [1, 2, 5, 8, 16, 37, 64])
def test_three_forms_agree(chunk):
    rng = np.random.default_rng(10 + chunk)
    args = _rand_problem(rng)
    h0 = rng.standard_normal((2, 4, 3, 5))
    yr, sr = oracle.recurrence(*args, state=h0)
    yq, sq = oracle.quadratic(*args, state=h0)
    yc, sc = oracle.chunked(*args, chunk, state=h0)
    assert _rel(yq, yr) < 1e-12 and _rel(sq, sr) < 1e-12
    assert _rel(yc, yr) < 1e-12 and _rel(sc, sr) < 1e-12


def test_chunk_invariance_long():
    """Chunk sizes 16..256 (and a non-divisor) give the same layer on a 300-token input."""
    rng = np.random.default_rng(20)
    args = _rand_problem(rng, b=1, L=300, H=2, P=4, N=6, G=1, dt_range=(1e-3, 0.1))
    ref_y, ref_s = oracle.chunked(*args, 256)
    for q in (16, 32, 64, 128, 100):
        y, s = oracle.chunked(*args, q)
        assert _rel(y, ref_y) < 1e-12 and _rel(s, ref_s) < 1e-12, q


@pytest.mark.parametrize("k", [1, 16, 64, 65])
def test_prefill_then_decode_split(k):
    """prefill(L) == prefill(L - k) followed by k single-token steps (chunk 64)."""
    rng = np.random.default_rng(30 + k)
    L = 200
    x, dt, A, B, C, D = _rand_problem(rng, b=2, L=L, H=3, P=4, N=5, G=1, dt_range=(1e-3, 0.1))
    y_full, s_full = oracle.quadratic(x, dt, A, B, C, D)
    m = L - k
    y_pre, s = oracle.chunked(x[:, :m], dt[:, :m], A, B[:, :m], C[:, :m], D, 64)
    ys = [y_pre]
    for t in range(m, L):
        yt, s = oracle.recurrence(x[:, t:t + 1], dt[:, t:t + 1], A, B[:, t:t + 1],
                                  C[:, t:t + 1], D, state=s)
        ys.append(yt)
    assert _rel(np.concatenate(ys, axis=1), y_full) < 1e-12
    assert _rel(s, s_full) < 1e-12


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(40)
    args = _rand_problem(rng, b=3, L=40, H=6, P=3, N=4, G=3)
    y1, s1 = oracle.recurrence(*args, nthreads=1)
    y8, s8 = oracle.recurrence(*args, nthreads=8)
    assert np.array_equal(y1, y8) and np.array_equal(s1, s8)


def test_empty_sequence_keeps_state():
    rng = np.random.default_rng(41)
    x, dt, A, B, C, D = _rand_problem(rng, b=2, L=0, H=2, P=2, N=3, G=1)
    h0 = rng.standard_normal((2, 2, 2, 3))
    for f in (lambda: oracle.recurrence(x, dt, A, B, C, D, state=h0),
              lambda: oracle.quadratic(x, dt, A, B, C, D, state=h0),
              lambda: oracle.chunked(x, dt, A, B, C, D, 8, state=h0)):
        y, s = f()
        assert y.shape == (2, 0, 2, 2) and np.array_equal(s, h0)


def test_rejects_bad_groups():
    rng = np.random.default_rng(42)
    args = _rand_problem(rng, H=3, G=2)
    with pytest.raises(ValueError):
        oracle.recurrence(*args)


# ------------------------------------------------------------------ planted mistakes

@pytest.fixture(scope="module")
def mutant_lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("mutants") / "libmutants.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", out,
                    os.path.join(HERE, "oracle_mutants.c"), "-lm"], check=True)
    lib = ctypes.CDLL(out)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.ssd_mutant_recurrence.argtypes = [ctypes.c_int] + [ctypes.c_int64] * 6 + [dp] * 8
    lib.ssd_mutant_recurrence.restype = ctypes.c_int
    return lib


def _mutant_rec(lib, which):
    def rec(x, dt, A, B, C, D, state=None):
        f = lambda a: np.ascontiguousarray(np.asarray(a, np.float64))
        x, dt, A, B, C, D = map(f, (x, dt, A, B, C, D))
        b, L, H, P = x.shape
        G, N = B.shape[2], B.shape[3]
        st = np.zeros((b, H, P, N)) if state is None else f(state).copy()
        y = np.zeros((b, L, H, P))
        p = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
        lib.ssd_mutant_recurrence(which, b, L, H, P, N, G, p(x), p(dt), p(A), p(B), p(C),
                                  p(D), p(st), p(y))
        return y, st
    return rec


def test_mutant_zero_is_the_correct_recurrence(mutant_lib):
    """which = 0 plants nothing: every pin passes (checks the harness itself)."""
    rec = _mutant_rec(mutant_lib, 0)
    for pin in INDEPENDENT_PINS:
        pin(rec)


@pytest.mark.parametrize("which", range(1, 9))
def test_every_planted_mistake_is_caught(mutant_lib, which):
    rec = _mutant_rec(mutant_lib, which)
    failed = []
    for pin in INDEPENDENT_PINS:
        try:
            pin(rec)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"planted mistake {which} passed every pin"
