"""GPU parity of the fused front end (ssd_frontend) against the fp64 front-end oracle on
the same seeded inputs: conv + SiLU outputs within 2^-8 relative (bf16 outputs: one
rounding) or 1e-5 (fp32), plus 1e-5 RMS absolute; dt the same way; the conv state
exactly (it holds inputs).  Also: a sequence processed in pieces with the conv state updated in place, and
token-by-token decode (seqlen 1) against one pass."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_10_b200 import ssd as mod
    return mod


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).bfloat16()


def _make(b, L, H, P, G, N, dtype, seed):
    rng = np.random.default_rng(seed)
    CH = H * P + 2 * G * N
    xbc = rng.standard_normal((b, L, CH)).astype(np.float32)
    w = (rng.standard_normal((CH, 4)) * 0.5).astype(np.float32)
    bias = (rng.standard_normal(CH) * 0.1).astype(np.float32)
    dt_raw = rng.standard_normal((b, L, H)).astype(np.float32)
    dt_bias = rng.uniform(-4, 0, H).astype(np.float32)
    if dtype == "bf16":  # the oracle sees exactly what the GPU gets
        xbc = _bf16(xbc).float().numpy()
    return xbc, w, bias, dt_raw, dt_bias


def _dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return t.bfloat16() if dtype == "bf16" else t


def _close(got, ref, rel):
    """|got - ref| <= rel |ref| + 1e-5 RMS(ref): the output's own rounding (bf16: 2^-9) plus
    fp32 arithmetic, whose error near a cancelling width-4 sum is absolute, not relative."""
    got = got.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(got).all()
    bound = rel * np.abs(ref) + 1e-5 * np.sqrt(np.mean(ref * ref))
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} elements off, worst |d| {np.abs(got - ref)[bad].max():.3e}"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [
    dict(b=2, L=300, H=4, P=64, G=1, N=128),
    dict(b=1, L=37, H=4, P=16, G=2, N=32),
    dict(b=3, L=2, H=2, P=8, G=1, N=16),      # shorter than the filter
    dict(b=4, L=16390, H=2, P=32, G=1, N=16),  # long enough for the streaming kernel (ragged last range)
    dict(b=2, L=300, H=2, P=6, G=1, N=16),     # x width a multiple of 4 channels but not of 8
    dict(b=1, L=37, H=3, P=5, G=1, N=16),      # odd x width: one channel a thread
])
def test_frontend_matches_oracle(ssd, dtype, shape):
    s = shape
    xbc, w, bias, dt_raw, dt_bias = _make(s["b"], s["L"], s["H"], s["P"], s["G"], s["N"], dtype, 11)
    hist = np.random.default_rng(5).standard_normal((s["b"], 3, xbc.shape[2])).astype(np.float32)
    if dtype == "bf16":
        hist = _bf16(hist).float().numpy()
    st = torch.from_numpy(hist).cuda()
    x, B, C, dt = ssd.frontend(_dev(xbc, dtype), torch.from_numpy(w).cuda(), torch.from_numpy(dt_raw).cuda(),
                               torch.from_numpy(dt_bias).cuda(), s["H"], s["P"], s["G"], s["N"],
                               conv_b=torch.from_numpy(bias).cuda(), conv_state_in=st, conv_state_out=st)
    torch.cuda.synchronize()
    xr, Br, Cr, dtr, str_ = oracle.frontend(xbc, w, bias, dt_raw, dt_bias, s["H"], s["P"], s["G"], s["N"],
                                            state=hist)
    rel = 2.0 ** -8 if dtype == "bf16" else 1e-5
    _close(x, xr, rel)
    _close(B, Br, rel)
    _close(C, Cr, rel)
    _close(dt, dtr, 1e-5)
    assert np.array_equal(st.cpu().numpy().astype(np.float64), str_)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_frontend_in_pieces_and_token_by_token(ssd, dtype):
    """A 40-token sequence: one pass, the same in pieces of 17, 2 and 21 tokens with the conv
    state carried in place, and as 40 single-token calls (decode) -- all equal."""
    H, P, G, N = 2, 16, 1, 32
    xbc, w, bias, dt_raw, dt_bias = _make(2, 40, H, P, G, N, dtype, 21)
    args = lambda lo, hi: (_dev(xbc[:, lo:hi], dtype), torch.from_numpy(w).cuda(),
                           torch.from_numpy(np.ascontiguousarray(dt_raw[:, lo:hi])).cuda(),
                           torch.from_numpy(dt_bias).cuda(), H, P, G, N)
    bias_t = torch.from_numpy(bias).cuda()
    x1, _, C1, dt1 = ssd.frontend(*args(0, 40), conv_b=bias_t)
    st = torch.zeros(2, 3, xbc.shape[2], device="cuda")
    xs, cs = [], []
    for lo, hi in ((0, 17), (17, 19), (19, 40)):
        x, _, C, _ = ssd.frontend(*args(lo, hi), conv_b=bias_t, conv_state_in=st, conv_state_out=st)
        xs.append(x); cs.append(C)
    st2 = torch.zeros_like(st)
    xt = []
    for t in range(40):
        x, _, _, _ = ssd.frontend(*args(t, t + 1), conv_b=bias_t, conv_state_in=st2, conv_state_out=st2)
        xt.append(x)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(xs, 1), x1) and torch.equal(torch.cat(cs, 1), C1)
    assert torch.equal(torch.cat(xt, 1), x1)
    assert torch.equal(st, st2)
