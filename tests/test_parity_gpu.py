"""GPU parity: libssd (through its C ABI) against the fp64 CPU oracle on the same seeded
inputs.  Tolerances: max|y - y_ref| <= 1e-4 RMS(y_ref) for fp32 inputs, <= 2e-2 RMS for
bf16 inputs (fp32 accumulation, fp32 state); the final state within the same bounds."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_10_b200 import inputs
from helpers import TOL, assert_close, decode_args, rel_err, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_10_b200 import ssd as mod
    return mod


def run_prefill(ssd, si, chunk):
    t = to_device(si)
    y, fs = ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=chunk)
    torch.cuda.synchronize()
    return y.cpu().numpy(), fs.cpu().numpy()


def check_prefill(ssd, si, chunk, what):
    y, fs = run_prefill(ssd, si, chunk)
    y_ref, fs_ref = oracle.recurrence(si.x, si.dt, si.A, si.B, si.C, si.D)
    tol = TOL[si.dtype]
    ey = assert_close(y, y_ref, tol, f"{what} y")
    es = assert_close(fs, fs_ref, tol, f"{what} final state")
    return ey, es


# ----------------------------------------------------------------- small cases

def test_tiny_fp32_prefill_then_decode(ssd):
    """fp32 workload: prefill of 256 tokens, then 16 decode steps of the following tokens;
    checked against one oracle recurrence over all 272 tokens."""
    w = inputs.BY_NAME["tiny_fp32"]
    full = inputs.workload_sequence(w, seqlen=w.seqlen + w.decode_steps)
    pre = full.token_slice(0, w.seqlen)
    y, fs = run_prefill(ssd, pre, w.chunk)
    state = torch.from_numpy(fs).cuda()
    ys = [y]
    for k in range(w.decode_steps):
        tok = to_device(full.token_slice(w.seqlen + k, w.seqlen + k + 1))
        yk = ssd.decode_step(state, **decode_args(tok))
        ys.append(yk.cpu().numpy()[:, None])
    y_all = np.concatenate(ys, axis=1)
    y_ref, fs_ref = oracle.recurrence(full.x, full.dt, full.A, full.B, full.C, full.D)
    assert_close(y_all, y_ref, 1e-4, "y over 272 tokens")
    assert_close(state.cpu().numpy(), fs_ref, 1e-4, "state after 272 tokens")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [
    dict(b=2, L=600, H=4, P=64, N=128, G=1, Q=256),   # several chunks, ragged tail
    dict(b=1, L=300, H=4, P=64, N=128, G=2, Q=128),   # two groups
    dict(b=1, L=257, H=3, P=32, N=64, G=1, Q=64),
    dict(b=2, L=100, H=2, P=100, N=32, G=1, Q=32),    # P not a multiple of 64
    dict(b=1, L=70, H=2, P=8, N=256, G=1, Q=16),
    dict(b=1, L=50, H=1, P=1, N=16, G=1, Q=8),
    dict(b=1, L=130, H=2, P=256, N=128, G=1, Q=64),
])
def test_prefill_shapes(ssd, dtype, shape):
    s = shape
    si = inputs.sequence(s["b"], s["L"], s["H"], s["P"], s["N"], s["G"], dtype, seed=123)
    check_prefill(ssd, si, s["Q"], f"{dtype} {s}")


@pytest.mark.parametrize("shape", [
    dict(b=2, L=128 * 100 + 5, H=4, G=2, Q=128),   # 404 work items of one head pair, ragged last chunk
    dict(b=1, L=256 * 30 + 200, H=26, G=1, Q=256),  # 279 items of 3 heads (the last block 2), ragged last chunk
])
def test_prefill_more_work_items_than_sms(ssd, shape):
    """Tensor-core prefills whose chunk-state launch has more work items than the GPU has
    SMs (the persistent grid, each CTA taking several items in turn), checked in full
    against the oracle."""
    s = shape
    si = inputs.sequence(s["b"], s["L"], s["H"], 64, 128, s["G"], "bf16", seed=321)
    check_prefill(ssd, si, s["Q"], f"bf16 {s}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("chunk", [1, 2, 16, 32, 64, 128, 256])
def test_chunk_sizes(ssd, dtype, chunk):
    si = inputs.sequence(1, 333, 2, 64, 128, 1, dtype, seed=7)
    check_prefill(ssd, si, chunk, f"{dtype} chunk {chunk}")


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 255, 256, 257])
def test_lengths_around_chunk(ssd, L):
    si = inputs.sequence(2, L, 4, 64, 128, 1, "bf16", seed=L)
    check_prefill(ssd, si, 64 if L < 200 else 256, f"L={L}")


def test_empty_sequence_gives_zero_state(ssd):
    x = torch.empty((2, 0, 4, 64), dtype=torch.bfloat16, device="cuda")
    dt = torch.empty((2, 0, 4), device="cuda")
    B = torch.empty((2, 0, 1, 128), dtype=torch.bfloat16, device="cuda")
    A = -torch.ones(4, device="cuda")
    D = torch.ones(4, device="cuda")
    fs = torch.full((2, 4, 64, 128), 7.0, device="cuda")
    y, fs = ssd.prefill(x, dt, A, B, B, D, chunk=256, final_state=fs)
    torch.cuda.synchronize()
    assert y.shape == (2, 0, 4, 64)
    assert torch.count_nonzero(fs).item() == 0


def test_empty_batch(ssd):
    x = torch.empty((0, 10, 4, 64), dtype=torch.bfloat16, device="cuda")
    B = torch.empty((0, 10, 1, 128), dtype=torch.bfloat16, device="cuda")
    y, fs = ssd.prefill(x, torch.empty((0, 10, 4), device="cuda"), -torch.ones(4, device="cuda"), B, B,
                        torch.ones(4, device="cuda"), chunk=64)
    assert y.shape == (0, 10, 4, 64) and fs.shape == (0, 4, 64, 128)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_from_random_state(ssd, dtype):
    w = replace(inputs.BY_NAME["mamba2_2.7b_decode_b256"], batch=3, nheads=8, ngroups=2, dtype=dtype)
    state0 = inputs.decode_initial_state(w)
    state = torch.from_numpy(state0).cuda()
    st_ref = state0.astype(np.float64)
    for step in range(5):
        tok = inputs.decode_token(w, step)
        y = ssd.decode_step(state, **decode_args(to_device(tok)))
        y_ref, st_ref = oracle.recurrence(tok.x, tok.dt, tok.A, tok.B, tok.C, tok.D, state=st_ref)
        assert_close(y.cpu().numpy(), y_ref[:, 0], TOL[dtype], f"decode step {step} y")
    assert_close(state.cpu().numpy(), st_ref, TOL[dtype], "decode state")


@pytest.mark.parametrize("N", [16, 32, 64, 256])
def test_decode_dstates(ssd, N):
    w = replace(inputs.BY_NAME["mamba2_2.7b_decode_b256"], batch=2, nheads=4, headdim=48, dstate=N)
    state0 = inputs.decode_initial_state(w)
    state = torch.from_numpy(state0).cuda()
    tok = inputs.decode_token(w, 0)
    y = ssd.decode_step(state, **decode_args(to_device(tok)))
    y_ref, st_ref = oracle.recurrence(tok.x, tok.dt, tok.A, tok.B, tok.C, tok.D, state=state0)
    assert_close(y.cpu().numpy(), y_ref[:, 0], 2e-2, f"N={N} y")
    assert_close(state.cpu().numpy(), st_ref, 2e-2, f"N={N} state")


def test_prefill_is_deterministic(ssd):
    si = inputs.sequence(1, 700, 8, 64, 128, 1, "bf16", seed=3)
    t = to_device(si)
    y1, f1 = ssd.prefill(**t, chunk=256)
    y2, f2 = ssd.prefill(**t, chunk=256)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(f1, f2)


def test_binding_and_abi_errors(ssd):
    si = inputs.sequence(1, 64, 2, 64, 128, 1, "bf16", seed=1)
    t = to_device(si)
    with pytest.raises(ValueError):
        ssd.prefill(t["x"].float(), t["dt"], t["A"], t["B"], t["C"], t["D"])   # mixed dtypes
    with pytest.raises(ValueError):
        ssd.prefill(t["x"], t["dt"].double(), t["A"], t["B"], t["C"], t["D"])
    # x at a 4-byte offset: the C ABI rejects it (SSD_ERR_INVALID_ARG), nothing launched
    buf = torch.empty(t["x"].numel() + 2, dtype=torch.bfloat16, device="cuda")
    xm = buf[2:].view(t["x"].shape)
    xm.copy_(t["x"])
    with pytest.raises(ssd.SSDError) as e:
        ssd.prefill(xm, t["dt"], t["A"], t["B"], t["C"], t["D"])
    assert e.value.status == ssd.ERR_INVALID_ARG
    need = ssd.prefill_workspace_size(ssd.dims_of_prefill(t["x"], t["B"]), ssd.BF16, 64)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ssd.SSDError) as e:
        ssd.prefill(**t, chunk=64, workspace=small)
    assert e.value.status == ssd.ERR_WORKSPACE


# ----------------------------------------------------------------- full workloads

@pytest.mark.parametrize("name", ["mamba2_130m_prefill", "mamba2_2.7b_prefill"])
def test_full_prefill_workloads(ssd, name):
    w = inputs.BY_NAME[name]
    si = inputs.workload_sequence(w)
    ey, es = check_prefill(ssd, si, w.chunk, name)
    print(f"{name}: y err {ey:.2e}, state err {es:.2e} (RMS-relative max)")


def test_long_context_prefill_then_decode(ssd):
    """b=4, L=16384 prefill, then 256 decode steps from its final state, against (i) one
    GPU prefill of all 16640 tokens (every head) and (ii) the oracle over all 16640
    tokens, every (batch row, head) pair: y of every token and the final state."""
    w = inputs.BY_NAME["mamba2_130m_long_b4"]
    full = inputs.workload_sequence(w, seqlen=w.seqlen + w.decode_steps)
    pre = full.token_slice(0, w.seqlen)
    t_pre = to_device(pre)
    y_pre, state = ssd.prefill(**t_pre, chunk=w.chunk)
    del t_pre
    t_full = to_device(full)
    ys = []
    for k in range(w.decode_steps):
        tok = {kk: (v[:, w.seqlen + k:w.seqlen + k + 1] if v.dim() > 1 else v) for kk, v in t_full.items()}
        ys.append(ssd.decode_step(state, **decode_args(tok))[:, None])
    y_split = torch.cat([y_pre] + ys, dim=1)
    y_one, fs_one = ssd.prefill(**t_full, chunk=w.chunk)
    torch.cuda.synchronize()
    y_split, y_one = y_split.cpu().numpy(), y_one.cpu().numpy()
    assert_close(y_split, y_one, 2e-2, "split vs one prefill y")
    assert_close(state.cpu().numpy(), fs_one.cpu().numpy(), 2e-2, "split vs one prefill state")
    y_ref, fs_ref = oracle.recurrence(full.x, full.dt, full.A, full.B, full.C, full.D)
    st = state.cpu().numpy()
    assert_close(y_split, y_ref, 2e-2, "oracle y, all 96 (batch row, head) pairs")
    assert_close(st, fs_ref, 2e-2, "oracle final state, all 96 pairs")
    for bi in range(w.batch):  # and each pair on its own scale, so that no small head hides
        for h in range(w.nheads):
            assert_close(y_split[bi, :, h], y_ref[bi, :, h], 2e-2, f"oracle y (b={bi}, h={h})")
            assert_close(st[bi, h], fs_ref[bi, h], 2e-2, f"oracle state (b={bi}, h={h})")


def test_batched_decode_workload(ssd):
    """batch 256 x 80 heads, 1024 decode steps from a seeded N(0, 0.1^2) state.  Every one
    of the 20480 heads is checked against the oracle (y and the whole state) after step 0
    and after step 15, the oracle stepping all heads; then y at steps 31, 63, ..., 1023
    and the final state on a sample of (batch row, head) pairs, the oracle continuing
    only those."""
    w = inputs.BY_NAME["mamba2_2.7b_decode_b256"]
    state0 = inputs.decode_initial_state(w)
    state = torch.from_numpy(state0).cuda()
    rng = np.random.default_rng(1)
    pairs = [(0, 0), (255, 79)] + [tuple(v) for v in rng.integers((0, 0), (256, 80), (10, 2))]
    full_steps = 16
    st_all = state0.astype(np.float64)
    checks = set(range(16)) | {31, 63, 127, 255, 511, 1023}
    worst = 0.0
    st_ref = {}
    for step in range(w.decode_steps):
        tok = inputs.decode_token(w, step)
        y = ssd.decode_step(state, **decode_args(to_device(tok)))
        if step < full_steps:  # the oracle steps every head
            y_ref, st_all = oracle.recurrence(tok.x, tok.dt, tok.A, tok.B, tok.C, tok.D, state=st_all)
            if step in (0, full_steps - 1):
                worst = max(worst, assert_close(y.cpu().numpy(), y_ref[:, 0], 2e-2, f"step {step}: y, all heads"))
                assert_close(state.cpu().numpy(), st_all, 2e-2, f"step {step}: state, all heads")
            if step == full_steps - 1:
                st_ref = {p: st_all[p[0]:p[0] + 1, p[1]:p[1] + 1].copy() for p in pairs}
                del st_all
            continue
        for (bi, h) in pairs:
            hs = tok.head_slice(bi, h)
            y_ref, st_ref[(bi, h)] = oracle.recurrence(hs.x, hs.dt, hs.A, hs.B, hs.C, hs.D,
                                                       state=st_ref[(bi, h)], nthreads=1)
            if step in checks:
                got = y[bi, h].cpu().numpy()
                worst = max(worst, assert_close(got, y_ref[0, 0, 0], 2e-2, f"step {step} (b={bi}, h={h})"))
    st = state.cpu().numpy()
    for (bi, h) in pairs:
        assert_close(st[bi, h], st_ref[(bi, h)][0, 0], 2e-2, f"final state (b={bi}, h={h})")
    print(f"batched decode: worst y err {worst:.2e}")


# ----------------------------------------------------------------- initial state, chunk states

def _random_state(si, seed):
    b, _, H, P = si.x.shape
    N = si.B.shape[3]
    return np.random.default_rng(seed).standard_normal((b, H, P, N)) * 0.1


@pytest.mark.parametrize("dtype,shape", [
    ("bf16", dict(b=2, L=600, H=4, P=64, N=128, G=1, Q=256)),   # tensor-core path
    ("f32", dict(b=1, L=200, H=3, P=32, N=64, G=1, Q=64)),      # CUDA-core path
])
def test_prefill_host_equals_the_device_call(ssd, dtype, shape):
    """ssd_prefill_host (host arrays in and out, the copies enqueued by the library) gives
    exactly the results of ssd_prefill on device copies, from page-locked and from
    pageable host memory."""
    s = shape
    si = inputs.sequence(s["b"], s["L"], s["H"], s["P"], s["N"], s["G"], dtype, seed=404)
    t = to_device(si)
    y, fs = ssd.prefill(**t, chunk=s["Q"])
    torch.cuda.synchronize()
    for pinned in (True, False):
        host = {k: (v.cpu().pin_memory() if pinned else v.cpu()) for k, v in t.items()}
        yh, fsh = ssd.prefill_host(**host, chunk=s["Q"])
        torch.cuda.synchronize()
        assert torch.equal(yh, y.cpu()) and torch.equal(fsh, fs.cpu())


def test_prefill_host_on_two_streams_matches_each_device_call(ssd):
    """Independent sequences alternating between two streams, each stream with its own
    device buffer, so that one call's copies back overlap the next call's copies in and
    kernels: every sequence's host y and final state equal its own device call bit for bit."""
    Q = 256
    seqs = [to_device(inputs.sequence(1, 700, 4, 64, 128, 1, "bf16", seed=500 + i)) for i in range(4)]
    refs = []
    for t in seqs:
        y, fs = ssd.prefill(**t, chunk=Q)
        refs.append((y.cpu(), fs.cpu()))
    dims = ssd.dims_of_prefill(seqs[0]["x"], seqs[0]["B"])
    lanes = [torch.cuda.Stream() for _ in range(2)]
    bufs = [torch.empty(ssd.prefill_host_buffer_size(dims, ssd.BF16, Q), dtype=torch.uint8, device="cuda")
            for _ in lanes]
    hosts = [{k: v.cpu().pin_memory() for k, v in t.items()} for t in seqs]
    torch.cuda.synchronize()
    outs = [ssd.prefill_host(**h, chunk=Q, device_buffer=bufs[i % 2], stream=lanes[i % 2])
            for i, h in enumerate(hosts)]
    torch.cuda.synchronize()
    for (yh, fsh), (y, fs) in zip(outs, refs):
        assert torch.equal(yh, y) and torch.equal(fsh, fs)


def test_decode_with_copies_on_side_streams_matches_in_order_steps(ssd):
    """Decode steps in order on the compute stream while each step's inputs go up on one
    copy stream and its y comes back on another (device inputs and y double-buffered, their
    reuse ordered by events): every y and the final state equal those of the same steps run
    plainly on one stream, bit for bit."""
    b, H, P, N, G, steps = 8, 6, 64, 128, 1, 12
    g = torch.Generator().manual_seed(91)
    hx = torch.randn((steps, b, H, P), generator=g).bfloat16().pin_memory()
    hdt = (torch.rand((steps, b, H), generator=g) * 0.1 + 1e-3).pin_memory()
    hB = (torch.randn((steps, b, G, N), generator=g) / N ** 0.5).bfloat16().pin_memory()
    hC = (torch.randn((steps, b, G, N), generator=g) / N ** 0.5).bfloat16().pin_memory()
    A = (-torch.exp(torch.rand((H,), generator=g) * np.log(16.0))).cuda()
    D = torch.randn((H,), generator=g).cuda()
    state0 = (torch.randn((b, H, P, N), generator=g) * 0.1).cuda()

    state = state0.clone()
    ref = []
    for k in range(steps):
        ref.append(ssd.decode_step(state, hx[k].cuda(), hdt[k].cuda(), A, hB[k].cuda(), hC[k].cuda(), D).cpu())
    ref_state = state.cpu()

    state = state0.clone()
    main = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    dx = [torch.empty((b, H, P), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    ddt = [torch.empty((b, H), device="cuda") for _ in range(2)]
    dB = [torch.empty((b, G, N), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    dC = [torch.empty((b, G, N), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    dy = [torch.empty((b, H, P), device="cuda") for _ in range(2)]
    y_h = torch.empty((steps, b, H, P), pin_memory=True)
    ev_in, ev_done, ev_out = ([torch.cuda.Event() for _ in range(steps)] for _ in range(3))
    torch.cuda.synchronize()
    for k in range(steps):
        j = k % 2
        with torch.cuda.stream(up):
            if k >= 2:
                up.wait_event(ev_done[k - 2])
            dx[j].copy_(hx[k], non_blocking=True)
            ddt[j].copy_(hdt[k], non_blocking=True)
            dB[j].copy_(hB[k], non_blocking=True)
            dC[j].copy_(hC[k], non_blocking=True)
            ev_in[k].record(up)
        main.wait_event(ev_in[k])
        if k >= 2:
            main.wait_event(ev_out[k - 2])
        ssd.decode_step(state, dx[j], ddt[j], A, dB[j], dC[j], D, y=dy[j], stream=main)
        ev_done[k].record(main)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[k])
            y_h[k].copy_(dy[j], non_blocking=True)
            ev_out[k].record(down)
    torch.cuda.synchronize()
    for k in range(steps):
        assert torch.equal(y_h[k], ref[k]), f"step {k}"
    assert torch.equal(state.cpu(), ref_state)


@pytest.mark.parametrize("L", [500, 400])
def test_wide_decay_ranges_take_every_factorisation(ssd, L):
    """The tensor-core chunk scan factorises a tile's decays three ways: one reference token
    when the tile's decay spans less than 2^100, two (one per 64-row half) when it spans
    more but each half less, and the decay folded into W per element otherwise.  Heads
    built to land in each (log2 ranges per 128 tokens of about 50; 150 and 190 with even
    halves; 260; and 138 packed into one half, either half) against the recurrence; with
    L = 500 the last tile is ragged past its split point, with L = 400 before it."""
    H = 6
    si = inputs.sequence(1, L, H, 64, 128, 1, "bf16", seed=77)
    log2e = 1.0 / np.log(2.0)
    dt = np.full((1, L, H), 0.1, dtype=np.float32)
    tok = np.arange(L) % 128
    dt[0, :, 4] = np.where(tok < 64, 0.15, 0.01)
    dt[0, :, 5] = np.where(tok < 64, 0.01, 0.15)
    A = -np.array([50.0, 150.0, 190.0, 260.0, 0.0, 0.0]) / (128 * 0.1 * log2e)
    A[4] = A[5] = -10.0
    si = replace(si, dt=dt, A=A.astype(np.float32))
    check_prefill(ssd, si, 256, f"wide decay ranges, L={L}")


@pytest.mark.parametrize("dtype,shape", [
    ("bf16", dict(b=2, L=600, H=4, P=64, N=128, G=1, Q=256)),   # tensor-core path, ragged tail
    ("bf16", dict(b=1, L=300, H=4, P=64, N=128, G=2, Q=128)),   # tensor-core path, two groups
    ("f32", dict(b=2, L=200, H=3, P=32, N=64, G=1, Q=64)),      # CUDA-core path
    ("bf16", dict(b=1, L=100, H=2, P=16, N=32, G=1, Q=32)),     # CUDA-core path, bf16 inputs
])
def test_prefill_from_initial_state(ssd, dtype, shape):
    """Prefill from a non-zero state equals the recurrence started from that state; the
    state after every chunk equals the recurrence's state at that chunk's last token."""
    s = shape
    si = inputs.sequence(s["b"], s["L"], s["H"], s["P"], s["N"], s["G"], dtype, seed=321)
    h0 = _random_state(si, 5)
    t = to_device(si)
    init = torch.from_numpy(h0.astype(np.float32)).cuda()
    y, fs, cs = ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=s["Q"], initial_state=init,
                            chunk_states=True)
    torch.cuda.synchronize()
    y_ref, fs_ref = oracle.recurrence(si.x, si.dt, si.A, si.B, si.C, si.D, state=h0)
    tol = TOL[dtype]
    assert_close(y.cpu().numpy(), y_ref, tol, "y from an initial state")
    assert_close(fs.cpu().numpy(), fs_ref, tol, "final state from an initial state")
    cs = cs.cpu().numpy()
    nc = -(-s["L"] // s["Q"])
    assert cs.shape == (s["b"], nc, s["H"], s["P"], s["N"])
    for c in range(nc):
        end = min((c + 1) * s["Q"], s["L"])
        pre = si.token_slice(0, end)
        _, st_ref = oracle.recurrence(pre.x, pre.dt, pre.A, pre.B, pre.C, pre.D, state=h0)
        assert_close(cs[:, c], st_ref, tol, f"state after chunk {c}")
    assert np.array_equal(cs[:, -1], fs.cpu().numpy())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_prefill_in_pieces_equals_one_prefill(ssd, dtype):
    """Chunked continuation: prefill of 300 tokens, then of the next 220 from its final
    state (updated in place), matches the recurrence over all 520 tokens."""
    P, N, Q = (64, 128, 256) if dtype == "bf16" else (16, 32, 64)
    full = inputs.sequence(2, 520, 4, P, N, 1, dtype, seed=77)
    a, b = full.token_slice(0, 300), full.token_slice(300, 520)
    ta, tb = to_device(a), to_device(b)
    ya, state = ssd.prefill(ta["x"], ta["dt"], ta["A"], ta["B"], ta["C"], ta["D"], chunk=Q)
    yb, state2 = ssd.prefill(tb["x"], tb["dt"], tb["A"], tb["B"], tb["C"], tb["D"], chunk=Q, initial_state=state,
                             final_state=state)
    torch.cuda.synchronize()
    assert state2.data_ptr() == state.data_ptr()
    y_ref, fs_ref = oracle.recurrence(full.x, full.dt, full.A, full.B, full.C, full.D)
    tol = TOL[dtype]
    assert_close(np.concatenate([ya.cpu().numpy(), yb.cpu().numpy()], axis=1), y_ref, tol, "y over both pieces")
    assert_close(state.cpu().numpy(), fs_ref, tol, "state after both pieces")


def test_prefill_ex_without_tokens_copies_the_state(ssd):
    si = inputs.sequence(1, 0, 2, 64, 128, 1, "bf16", seed=3)
    t = to_device(si)
    h0 = torch.randn(1, 2, 64, 128, device="cuda")
    y, fs, cs = ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=256, initial_state=h0,
                            chunk_states=True)
    torch.cuda.synchronize()
    assert cs.shape[1] == 0
    assert torch.equal(fs, h0)


# ----------------------------------------------------------------- windowed decode

@pytest.mark.parametrize("dtype,shape,W", [
    ("bf16", dict(b=3, H=4, P=64, N=128, G=1), 16),
    ("bf16", dict(b=2, H=4, P=64, N=128, G=2), 5),
    ("f32", dict(b=2, H=3, P=32, N=64, G=1), 16),
    ("f32", dict(b=1, H=2, P=100, N=16, G=1), 7),
    ("bf16", dict(b=1, H=2, P=256, N=256, G=1), 1),
])
def test_windowed_decode_matches_the_recurrence(ssd, dtype, shape, W):
    """ReplaySSM-style decode after a prefill: per token y from the committed state and the
    buffered window, the state written only at flushes (every W tokens, and a partial
    window at the end), against the fp64 recurrence over all tokens."""
    s = shape
    L0, K = 200, 2 * W + 3
    full = inputs.sequence(s["b"], L0 + K, s["H"], s["P"], s["N"], s["G"], dtype, seed=99)
    pre = full.token_slice(0, L0)
    t = to_device(pre)
    _, state = ssd.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk=64)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    bufs = ssd.window_buffers(state, W, dtype=tdt, ngroups=s["G"])
    ys, pos = [], 0
    for k in range(K):
        tok = decode_args(to_device(full.token_slice(L0 + k, L0 + k + 1)))
        ys.append(ssd.decode_window_step(state, bufs, pos, **tok).cpu().numpy())
        pos += 1
        if pos == W:
            ssd.decode_window_flush(state, bufs, pos, tok["A"])
            pos = 0
    ssd.decode_window_flush(state, bufs, pos, tok["A"])
    torch.cuda.synchronize()
    y_ref, st_ref = oracle.recurrence(full.x, full.dt, full.A, full.B, full.C, full.D)
    y_w = np.stack(ys, axis=1)
    tol = TOL[dtype]
    for k in range(K):  # per-step bound, as for the decode workloads
        assert_close(y_w[:, k], y_ref[:, L0 + k], tol, f"windowed y at step {k}")
    assert_close(state.cpu().numpy(), st_ref, tol, "state after the windows")


# ----------------------------------------------------------------- failure detection

def test_bounded_device_wait_expires_and_the_context_stays_usable(ssd):
    """A wait that nothing satisfies gives up after its limit and reports SSD_ERR_TIMEOUT
    through the workspace's error word (no trap, no hang); the same wait satisfied reports
    OK; a prefill on the same context afterwards still matches the oracle."""
    import time
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    assert ssd.wait_selftest(ws, limit_ns=2_000_000, expire=True) == ssd.ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert ssd.wait_selftest(ws, limit_ns=2_000_000, expire=False) == ssd.OK
    si = inputs.sequence(1, 300, 2, 64, 128, 1, "bf16", seed=8)
    check_prefill(ssd, si, 256, "prefill after an expired wait")
