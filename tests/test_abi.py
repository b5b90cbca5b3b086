"""The C-ABI library loads and exports what include/ssd.h declares; host-side validation
rejects bad arguments before anything is enqueued.  No GPU needed: every call here fails
validation (or only queries sizes), so no kernel is ever launched, and the pointers are
never dereferenced."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def ssd():
    from selective_state_space_10_b200 import build
    build.build()
    from selective_state_space_10_b200 import ssd as mod
    return mod


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    from selective_state_space_10_b200 import build  # noqa: F401
    declared = _declared_functions()
    assert declared, "no functions found in include/ssd.h"
    src = open(os.path.join(ROOT, "selective_state_space_10_b200", "ssd.py")).read()
    m = re.search(r"EXPORTS = \((.*?)\)", src, re.S)
    listed = sorted(re.findall(r'"(ssd_[a-z0-9_]+)"', m.group(1)))
    assert listed == declared


def test_library_exports_every_declared_symbol(ssd):
    lib = ctypes.CDLL(ssd.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), f"libssd.so does not export {name}"


def test_library_exports_nothing_else(ssd):
    out = os.popen(f"nm -D --defined-only {ssd.LIB_PATH}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {s for s in exported if s.startswith("ssd_")}
    assert ours == set(_declared_functions())


def test_status_strings_and_version(ssd):
    for s in range(6):
        assert ssd.status_string(s).startswith("SSD_")
    assert ssd.status_string(99) == "unknown ssd_status"
    assert ssd.version() >= 100


def _dims(ssd, b=1, L=512, H=8, P=64, N=128, G=1):
    return ssd._dims(b, L, H, P, N, G)


def test_workspace_size_and_launches(ssd):
    d = _dims(ssd)
    ws = ssd.prefill_workspace_size(d, ssd.BF16, 256)
    # cumulative decays + one P x N fp32 state per (chunk, head), 256-byte aligned regions
    nc = 2
    expect = -(-(1 * 8 * nc * 256 * 4) // 256) * 256 + 1 * nc * 8 * 64 * 128 * 4
    assert ws >= expect
    assert ssd.prefill_kernel_launches(d, ssd.BF16, 256) >= 1
    assert ssd.prefill_workspace_size(d, ssd.BF16, 48) == 0          # not a power of two
    assert ssd.prefill_workspace_size(d, ssd.BF16, 512) == 0         # > 256
    assert ssd.prefill_kernel_launches(d, ssd.BF16, 48) == -1
    assert ssd.prefill_workspace_size(_dims(ssd, L=0), ssd.BF16, 64) == 0
    assert ssd.prefill_workspace_size(_dims(ssd, b=0), ssd.BF16, 64) == 0


FAKE = 1 << 20  # an aligned, never-dereferenced address: validation must fail first


def _prefill(ssd, dims, dtype=1, ptrs=None, chunk=256, ws=FAKE, ws_bytes=1 << 40):
    p = dict(x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, D=FAKE, y=FAKE, fs=FAKE)
    p.update(ptrs or {})
    v = lambda k: ctypes.c_void_p(p[k]) if p[k] is not None else None
    return ssd.lib.ssd_prefill(ctypes.byref(dims) if dims is not None else None, dtype, v("x"), v("dt"),
                               v("A"), v("B"), v("C"), v("D"), chunk, v("y"), v("fs"),
                               ctypes.c_void_p(ws) if ws else None, ws_bytes, None)


@pytest.mark.parametrize("case", [
    dict(dims=None),
    dict(dtype=7),
    dict(chunk=0), dict(chunk=48), dict(chunk=512), dict(chunk=-4),
    dict(dims_kw=dict(H=6, G=4)),
    dict(dims_kw=dict(P=0)), dict(dims_kw=dict(P=257)),
    dict(dims_kw=dict(N=0)),
    dict(dims_kw=dict(b=-1)), dict(dims_kw=dict(L=-5)), dict(dims_kw=dict(H=0)), dict(dims_kw=dict(G=0)),
    dict(ptrs=dict(x=None)), dict(ptrs=dict(dt=None)), dict(ptrs=dict(B=None)), dict(ptrs=dict(C=None)),
    dict(ptrs=dict(y=None)), dict(ptrs=dict(fs=None)), dict(ptrs=dict(A=None)), dict(ptrs=dict(D=None)),
    dict(ptrs=dict(x=FAKE + 8)), dict(ptrs=dict(B=FAKE + 4)), dict(ptrs=dict(y=FAKE + 2)),
    dict(ptrs=dict(fs=FAKE + 8)), dict(ptrs=dict(dt=FAKE + 2)),
])
def test_prefill_rejects_invalid(ssd, case):
    dims = None if ("dims" in case and case["dims"] is None) else _dims(ssd, **case.get("dims_kw", {}))
    st = _prefill(ssd, dims, dtype=case.get("dtype", 1), ptrs=case.get("ptrs"), chunk=case.get("chunk", 256))
    assert st == ssd.ERR_INVALID_ARG, ssd.status_string(st)


def test_prefill_unsupported_dstate(ssd):
    assert _prefill(ssd, _dims(ssd, N=48)) == ssd.ERR_UNSUPPORTED
    assert _prefill(ssd, _dims(ssd, N=512)) == ssd.ERR_UNSUPPORTED


def test_prefill_workspace_checks(ssd):
    d = _dims(ssd)
    need = ssd.prefill_workspace_size(d, 1, 256)
    assert _prefill(ssd, d, ws=0) == ssd.ERR_WORKSPACE
    assert _prefill(ssd, d, ws_bytes=need - 1) == ssd.ERR_WORKSPACE
    assert _prefill(ssd, d, ws=FAKE + 8, ws_bytes=need) == ssd.ERR_WORKSPACE


def _decode(ssd, dims, dtype=1, ptrs=None):
    p = dict(state=FAKE, x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, D=FAKE, y=FAKE)
    p.update(ptrs or {})
    v = lambda k: ctypes.c_void_p(p[k]) if p[k] is not None else None
    return ssd.lib.ssd_decode_step(ctypes.byref(dims) if dims is not None else None, dtype, v("state"), v("x"),
                                   v("dt"), v("A"), v("B"), v("C"), v("D"), v("y"), None)


@pytest.mark.parametrize("case", [
    dict(dims=None), dict(dtype=3), dict(dims_kw=dict(H=5, G=2)), dict(dims_kw=dict(P=300)),
    dict(ptrs=dict(state=None)), dict(ptrs=dict(state=FAKE + 4)), dict(ptrs=dict(x=None)),
    dict(ptrs=dict(y=FAKE + 8)), dict(ptrs=dict(B=FAKE + 2)), dict(ptrs=dict(dt=None)),
])
def test_decode_rejects_invalid(ssd, case):
    dims = None if ("dims" in case and case["dims"] is None) else _dims(ssd, **case.get("dims_kw", {}))
    assert _decode(ssd, dims, dtype=case.get("dtype", 1), ptrs=case.get("ptrs")) == ssd.ERR_INVALID_ARG


def test_decode_unsupported_dstate(ssd):
    assert _decode(ssd, _dims(ssd, N=100)) == ssd.ERR_UNSUPPORTED


def test_empty_batch_is_a_no_op(ssd):
    """batch = 0: nothing to compute, NULL pointers allowed, nothing enqueued."""
    d = _dims(ssd, b=0)
    null = {k: None for k in ("x", "dt", "A", "B", "C", "D", "y", "fs")}
    assert _prefill(ssd, d, ptrs=null, ws=0, ws_bytes=0) == ssd.OK
    nd = {k: None for k in ("state", "x", "dt", "A", "B", "C", "D", "y")}
    assert _decode(ssd, d, ptrs=nd) == ssd.OK


def test_noalloc_validation_without_a_gpu(ssd):
    """ssd_prefill_noalloc rejects invalid and oversized problems before any CUDA call."""
    f = ssd.lib.ssd_prefill_noalloc
    v = ctypes.c_void_p(FAKE)
    assert ssd.prefill_noalloc_max_workspace() == 32 << 20
    assert f(None, 1, v, v, v, v, v, v, 256, v, v, None) == ssd.ERR_INVALID_ARG
    big = _dims(ssd, b=1, L=4096, H=80)
    assert ssd.prefill_workspace_size(big, 1, 256) > ssd.prefill_noalloc_max_workspace()
    assert f(ctypes.byref(big), 1, v, v, v, v, v, v, 256, v, v, None) == ssd.ERR_WORKSPACE
    assert f(ctypes.byref(_dims(ssd)), 1, v, v, v, v, v, v, 48, v, v, None) == ssd.ERR_INVALID_ARG


def _prefill_ex(ssd, dims, init=None, cs=None, ptrs=None, chunk=256):
    p = dict(x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, D=FAKE, y=FAKE, fs=FAKE)
    p.update(ptrs or {})
    v = lambda a: ctypes.c_void_p(a) if a is not None else None
    return ssd.lib.ssd_prefill_ex(ctypes.byref(dims), 1, v(p["x"]), v(p["dt"]), v(p["A"]), v(p["B"]), v(p["C"]),
                                  v(p["D"]), chunk, v(init), v(p["y"]), v(p["fs"]), v(cs), ctypes.c_void_p(FAKE),
                                  1 << 40, None)


@pytest.mark.parametrize("case", [
    dict(init=FAKE + 4), dict(init=FAKE + 8), dict(cs=FAKE + 4), dict(cs=FAKE + 12),
    dict(ptrs=dict(x=None)), dict(ptrs=dict(fs=FAKE + 8)), dict(chunk=48),
])
def test_prefill_ex_rejects_invalid(ssd, case):
    """ssd_prefill_ex validates as ssd_prefill does, plus the optional arrays' alignment."""
    st = _prefill_ex(ssd, _dims(ssd), init=case.get("init"), cs=case.get("cs"), ptrs=case.get("ptrs"),
                     chunk=case.get("chunk", 256))
    assert st == ssd.ERR_INVALID_ARG, ssd.status_string(st)


def test_prefill_ex_empty_batch_is_a_no_op(ssd):
    null = {k: None for k in ("x", "dt", "A", "B", "C", "D", "y", "fs")}
    d = _dims(ssd, b=0)
    assert ssd.lib.ssd_prefill_ex(ctypes.byref(d), 1, None, None, None, None, None, None, 256, None, None, None,
                                  None, None, 0, None) == ssd.OK


def test_window_decode_rejects_invalid(ssd):
    """Window, position and count ranges and buffer alignment are checked on the host."""
    d = _dims(ssd, L=1)
    v = ctypes.c_void_p(FAKE)
    step = lambda W, pos, wx=FAKE: ssd.lib.ssd_decode_window_step(ctypes.byref(d), 1, W, pos, v, ctypes.c_void_p(wx),
                                                                 v, v, v, v, v, v, v, v, v, None)
    flush = lambda W, cnt: ssd.lib.ssd_decode_window_flush(ctypes.byref(d), 1, W, cnt, v, v, v, v, v, None)
    for W, pos in ((0, 0), (17, 0), (16, 16), (4, -1)):
        assert step(W, pos) == ssd.ERR_INVALID_ARG
    assert step(16, 3, FAKE + 8) == ssd.ERR_INVALID_ARG
    for W, cnt in ((0, 0), (17, 1), (8, 9), (8, -1)):
        assert flush(W, cnt) == ssd.ERR_INVALID_ARG


def test_frontend_rejects_invalid(ssd):
    """ssd_frontend validates its arrays (alignment, NULL) and grid limits on the host."""
    v = lambda a: ctypes.c_void_p(a) if a is not None else None
    def call(d, **over):
        p = dict(xbc=FAKE, w=FAKE, b=None, si=None, so=None, dtr=FAKE, dtb=FAKE, x=FAKE, B=FAKE, C=FAKE, dt=FAKE)
        p.update(over)
        return ssd.lib.ssd_frontend(ctypes.byref(d), 1, v(p["xbc"]), v(p["w"]), v(p["b"]), v(p["si"]), v(p["so"]),
                                    v(p["dtr"]), v(p["dtb"]), v(p["x"]), v(p["B"]), v(p["C"]), v(p["dt"]), None)
    d = _dims(ssd)
    for over in (dict(xbc=None), dict(w=FAKE + 4), dict(x=FAKE + 8), dict(dt=FAKE + 2), dict(si=FAKE + 2),
                 dict(so=FAKE + 1), dict(dtb=None), dict(xbc=FAKE + 1)):
        assert call(d, **over) == ssd.ERR_INVALID_ARG, over
    assert call(_dims(ssd, b=70000)) == ssd.ERR_INVALID_ARG
    assert call(_dims(ssd, b=0), xbc=None, w=None, dtr=None, dtb=None, x=None, B=None, C=None, dt=None) == ssd.OK


def test_wait_selftest_validation_without_a_gpu(ssd):
    f = ssd.lib.ssd_wait_selftest
    assert f(None, 256, 1000000, 1, None) == ssd.ERR_INVALID_ARG
    assert f(ctypes.c_void_p(FAKE + 4), 256, 1000000, 1, None) == ssd.ERR_INVALID_ARG
    assert f(ctypes.c_void_p(FAKE), 2, 1000000, 1, None) == ssd.ERR_INVALID_ARG
    assert f(ctypes.c_void_p(FAKE), 256, 0, 1, None) == ssd.ERR_INVALID_ARG
    assert f(ctypes.c_void_p(FAKE), 256, 10 ** 9, 1, None) == ssd.ERR_INVALID_ARG


def test_prefill_host_validation_without_a_gpu(ssd):
    """ssd_prefill_host checks its arguments and the device buffer before any copy; host
    arrays need no alignment, the device buffer 16 bytes."""
    f = ssd.lib.ssd_prefill_host
    d = _dims(ssd)
    h = ctypes.c_void_p(FAKE + 2)
    dev = ctypes.c_void_p(FAKE)
    need = ssd.prefill_host_buffer_size(d, 1, 256)
    assert need > ssd.prefill_workspace_size(d, 1, 256)
    call = lambda dims, x=h, chunk=256, buf=dev, nbytes=need: f(dims, 1, x, h, h, h, h, h, chunk, h, h, buf, nbytes,
                                                                 None)
    assert call(None) == ssd.ERR_INVALID_ARG
    assert call(ctypes.byref(d), chunk=48) == ssd.ERR_INVALID_ARG
    assert call(ctypes.byref(d), x=None) == ssd.ERR_INVALID_ARG
    assert call(ctypes.byref(_dims(ssd, N=48))) == ssd.ERR_UNSUPPORTED
    assert call(ctypes.byref(d), buf=None) == ssd.ERR_WORKSPACE
    assert call(ctypes.byref(d), nbytes=need - 1) == ssd.ERR_WORKSPACE
    assert call(ctypes.byref(d), buf=ctypes.c_void_p(FAKE + 8)) == ssd.ERR_WORKSPACE
    e = _dims(ssd, b=0)
    assert f(ctypes.byref(e), 1, None, None, None, None, None, None, 256, None, None, None, 0, None) == ssd.OK
