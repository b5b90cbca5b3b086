"""Python binding of libssd (include/ssd.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module checks tensor
devices, dtypes and shapes, allocates outputs with torch when the caller passes none,
and forwards raw device pointers and the current CUDA stream through ctypes.  Importing
it loads libssd.so and raises if the library has not been built: there is no fallback.
"""
import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(6)
F32, BF16 = 0, 1
_DTYPES = {torch.float32: F32, torch.bfloat16: BF16}


class SSDError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64)]


# Every symbol include/ssd.h declares.
EXPORTS = ("ssd_status_string", "ssd_version", "ssd_prefill_workspace_size",
           "ssd_prefill_kernel_launches", "ssd_prefill", "ssd_prefill_ex", "ssd_prefill_timed",
           "ssd_prefill_kernel_name", "ssd_prefill_device_status", "ssd_prefill_noalloc",
           "ssd_prefill_noalloc_max_workspace", "ssd_prefill_noalloc_device_status", "ssd_decode_step",
           "ssd_frontend", "ssd_decode_window_step", "ssd_decode_window_flush", "ssd_wait_selftest",
           "ssd_prefill_host_buffer_size", "ssd_prefill_host")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libssd.so is not built ({LIB_PATH}); run "
                          "`python -m selective_state_space_10_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, fp, i64, ci, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    dp = ctypes.POINTER(Dims)
    lib.ssd_status_string.argtypes = [ci]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_version.argtypes = []
    lib.ssd_version.restype = ci
    lib.ssd_prefill_workspace_size.argtypes = [dp, ci, ci]
    lib.ssd_prefill_workspace_size.restype = sz
    lib.ssd_prefill_kernel_launches.argtypes = [dp, ci, ci]
    lib.ssd_prefill_kernel_launches.restype = ci
    lib.ssd_prefill.argtypes = [dp, ci, vp, fp, fp, vp, vp, fp, ci, fp, fp, vp, sz, vp]
    lib.ssd_prefill.restype = ci
    lib.ssd_prefill_ex.argtypes = [dp, ci, vp, fp, fp, vp, vp, fp, ci, fp, fp, fp, fp, vp, sz, vp]
    lib.ssd_prefill_ex.restype = ci
    lib.ssd_prefill_timed.argtypes = [dp, ci, vp, fp, fp, vp, vp, fp, ci, fp, fp, vp, sz, vp,
                                      ctypes.POINTER(ctypes.c_void_p), ci]
    lib.ssd_prefill_timed.restype = ci
    lib.ssd_prefill_kernel_name.argtypes = [dp, ci, ci, ci]
    lib.ssd_prefill_kernel_name.restype = ctypes.c_char_p
    lib.ssd_prefill_device_status.argtypes = [vp, sz, vp]
    lib.ssd_prefill_device_status.restype = ci
    lib.ssd_prefill_noalloc.argtypes = [dp, ci, vp, fp, fp, vp, vp, fp, ci, fp, fp, vp]
    lib.ssd_prefill_noalloc.restype = ci
    lib.ssd_prefill_noalloc_max_workspace.argtypes = []
    lib.ssd_prefill_noalloc_max_workspace.restype = sz
    lib.ssd_prefill_noalloc_device_status.argtypes = [vp]
    lib.ssd_prefill_noalloc_device_status.restype = ci
    lib.ssd_prefill_host_buffer_size.argtypes = [dp, ci, ci]
    lib.ssd_prefill_host_buffer_size.restype = sz
    lib.ssd_prefill_host.argtypes = [dp, ci, vp, fp, fp, vp, vp, fp, ci, fp, fp, vp, sz, vp]
    lib.ssd_prefill_host.restype = ci
    lib.ssd_decode_step.argtypes = [dp, ci, fp, vp, fp, fp, vp, vp, fp, fp, vp]
    lib.ssd_decode_step.restype = ci
    lib.ssd_wait_selftest.argtypes = [vp, sz, ctypes.c_uint64, ci, vp]
    lib.ssd_wait_selftest.restype = ci
    lib.ssd_frontend.argtypes = [dp, ci, vp, fp, fp, fp, fp, fp, fp, vp, vp, vp, fp, vp]
    lib.ssd_frontend.restype = ci
    lib.ssd_decode_window_step.argtypes = [dp, ci, ci, ci, fp, vp, fp, vp, vp, fp, fp, vp, vp, fp, fp, vp]
    lib.ssd_decode_window_step.restype = ci
    lib.ssd_decode_window_flush.argtypes = [dp, ci, ci, ci, fp, vp, fp, vp, fp, vp]
    lib.ssd_decode_window_flush.restype = ci
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.ssd_status_string(int(status)).decode()


def version() -> int:
    return lib.ssd_version()


def _dims(batch, seqlen, nheads, headdim, dstate, ngroups) -> Dims:
    return Dims(int(batch), int(seqlen), int(nheads), int(headdim), int(dstate), int(ngroups))


def dims_of_prefill(x: torch.Tensor, B: torch.Tensor) -> Dims:
    b, L, H, P = x.shape
    return _dims(b, L, H, P, B.shape[3], B.shape[2])


def prefill_workspace_size(dims: Dims, dtype: int, chunk: int) -> int:
    return lib.ssd_prefill_workspace_size(ctypes.byref(dims), int(dtype), int(chunk))


def prefill_kernel_launches(dims: Dims, dtype: int, chunk: int) -> int:
    return lib.ssd_prefill_kernel_launches(ctypes.byref(dims), int(dtype), int(chunk))


def prefill_kernel_names(dims: Dims, dtype: int, chunk: int):
    n = prefill_kernel_launches(dims, dtype, chunk)
    return [lib.ssd_prefill_kernel_name(ctypes.byref(dims), int(dtype), int(chunk), i).decode()
            for i in range(max(n, 0))]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(t: torch.Tensor, name: str, shape, dtype, device):
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def prefill(x, dt, A, B, C, D, chunk: int = 256, y=None, final_state=None, workspace=None,
            stream=None, events=None, initial_state=None, chunk_states=None):
    """Chunked prefill.  Returns (y fp32 [b,L,H,P], final_state fp32 [b,H,P,N]).
    x, B, C are fp32 or bf16 (the same dtype); dt, A, D are fp32.

    `initial_state` (fp32 [b,H,P,N], optional): the state before the first token (zero if
    None); it may be `final_state` itself.  `chunk_states`: None, True (allocate), or an
    fp32 tensor [b, ceil(L/chunk), H, P, N] that receives the state after every chunk;
    when given, the return value is (y, final_state, chunk_states).  Either one routes the
    call through ssd_prefill_ex.

    `events`: optional list of torch.cuda.Event(enable_timing=True), at least
    prefill_kernel_launches() + 1 of them, already recorded once (so their handles
    exist); the call then goes through ssd_prefill_timed, which records events[i] before
    kernel i and events[-1] after the last kernel (not with initial_state/chunk_states)."""
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [b,L,H,P] and B, C [b,L,G,N]")
    if x.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {x.dtype}")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("libssd runs on CUDA tensors only")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _check(x, "x", (b, L, H, P), x.dtype, dev)
    _check(dt, "dt", (b, L, H), torch.float32, dev)
    _check(A, "A", (H,), torch.float32, dev)
    _check(B, "B", (b, L, G, N), x.dtype, dev)
    _check(C, "C", (b, L, G, N), x.dtype, dev)
    _check(D, "D", (H,), torch.float32, dev)
    if y is None:
        y = torch.empty((b, L, H, P), dtype=torch.float32, device=dev)
    if final_state is None:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    _check(y, "y", (b, L, H, P), torch.float32, dev)
    _check(final_state, "final_state", (b, H, P, N), torch.float32, dev)
    if initial_state is not None:
        _check(initial_state, "initial_state", (b, H, P, N), torch.float32, dev)
    want_cs = chunk_states is not None and chunk_states is not False
    if chunk_states is True:
        chunk_states = torch.empty((b, -(-L // int(chunk)) if chunk > 0 else 0, H, P, N), dtype=torch.float32,
                                   device=dev)
    if want_cs:
        _check(chunk_states, "chunk_states", (b, -(-L // int(chunk)) if chunk > 0 else 0, H, P, N),
               torch.float32, dev)
    extended = initial_state is not None or want_cs
    if extended and events is not None:
        raise ValueError("events cannot be combined with initial_state or chunk_states")
    dims = dims_of_prefill(x, B)
    dtype = _DTYPES[x.dtype]
    need = prefill_workspace_size(dims, dtype, chunk)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if extended:
        st = lib.ssd_prefill_ex(ctypes.byref(dims), dtype, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                int(chunk), _ptr(initial_state), _ptr(y), _ptr(final_state),
                                _ptr(chunk_states if want_cs else None), _ptr(workspace), ws_bytes, _stream(stream))
        if st != OK:
            raise SSDError(st, "ssd_prefill_ex")
        return (y, final_state, chunk_states) if want_cs else (y, final_state)
    args = (ctypes.byref(dims), dtype, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
            int(chunk), _ptr(y), _ptr(final_state), _ptr(workspace), ws_bytes, _stream(stream))
    if events is None:
        st = lib.ssd_prefill(*args)
    else:
        handles = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
        st = lib.ssd_prefill_timed(*args, handles, len(events))
    if st != OK:
        raise SSDError(st, "ssd_prefill")
    return y, final_state


def prefill_host_buffer_size(dims: Dims, dtype: int, chunk: int) -> int:
    return int(lib.ssd_prefill_host_buffer_size(ctypes.byref(dims), int(dtype), int(chunk)))


def prefill_host(x, dt, A, B, C, D, chunk: int = 256, y=None, final_state=None, device_buffer=None,
                 stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """ssd_prefill_host: the prefill end to end from host tensors (page-locked for
    asynchronous copies).  The library copies the inputs to `device_buffer` (a CUDA uint8
    tensor of at least prefill_host_buffer_size() bytes; allocated if None), runs the
    prefill, and copies y and final_state into host tensors, all on `stream`.  Returns the
    host (y, final_state); read them after synchronising the stream."""
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [b,L,H,P] and B, C [b,L,G,N]")
    if x.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {x.dtype}")
    host = torch.device("cpu")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    for t, name, shape, dtype in ((x, "x", (b, L, H, P), x.dtype), (dt, "dt", (b, L, H), torch.float32),
                                  (A, "A", (H,), torch.float32), (B, "B", (b, L, G, N), x.dtype),
                                  (C, "C", (b, L, G, N), x.dtype), (D, "D", (H,), torch.float32)):
        _check(t, name, shape, dtype, host)
    pin = x.is_pinned()
    if y is None:
        y = torch.empty((b, L, H, P), dtype=torch.float32, pin_memory=pin)
    if final_state is None:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, pin_memory=pin)
    _check(y, "y", (b, L, H, P), torch.float32, host)
    _check(final_state, "final_state", (b, H, P, N), torch.float32, host)
    dims = dims_of_prefill(x, B)
    dtype = _DTYPES[x.dtype]
    need = prefill_host_buffer_size(dims, dtype, chunk)
    if device_buffer is None:
        device_buffer = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    if device_buffer.device.type != "cuda":
        raise ValueError("device_buffer must be a CUDA tensor")
    st = lib.ssd_prefill_host(ctypes.byref(dims), dtype, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                              int(chunk), _ptr(y), _ptr(final_state), _ptr(device_buffer),
                              device_buffer.numel() * device_buffer.element_size(), _stream(stream))
    if st != OK:
        raise SSDError(st, "ssd_prefill_host")
    return y, final_state


def prefill_noalloc(x, dt, A, B, C, D, chunk: int = 256, y=None, final_state=None,
                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """ssd_prefill_noalloc: the same prefill, with no workspace argument.  For callers
    that cannot allocate device memory, the library takes its scratch from a fixed array
    of prefill_noalloc_max_workspace() bytes; calls that overlap on the GPU race on it.
    (Outputs are still allocated here when not given; pass y and final_state to avoid
    that.)"""
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    for name, t, shape, dtype in (("dt", dt, (b, L, H), torch.float32), ("A", A, (H,), torch.float32),
                                  ("B", B, (b, L, G, N), x.dtype), ("C", C, (b, L, G, N), x.dtype),
                                  ("D", D, (H,), torch.float32)):
        _check(t, name, shape, dtype, dev)
    if x.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {x.dtype}")
    if y is None:
        y = torch.empty((b, L, H, P), dtype=torch.float32, device=dev)
    if final_state is None:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    _check(y, "y", (b, L, H, P), torch.float32, dev)
    _check(final_state, "final_state", (b, H, P, N), torch.float32, dev)
    st = lib.ssd_prefill_noalloc(ctypes.byref(dims_of_prefill(x, B)), _DTYPES[x.dtype], _ptr(x), _ptr(dt),
                                 _ptr(A), _ptr(B), _ptr(C), _ptr(D), int(chunk), _ptr(y), _ptr(final_state),
                                 _stream(stream))
    if st != OK:
        raise SSDError(st, "ssd_prefill_noalloc")
    return y, final_state


def prefill_noalloc_max_workspace() -> int:
    return lib.ssd_prefill_noalloc_max_workspace()


def prefill_noalloc_device_status(stream=None) -> int:
    """ssd_prefill_noalloc_device_status: waits for the stream and returns OK or
    ERR_TIMEOUT from the error word of the library's scratch array."""
    return lib.ssd_prefill_noalloc_device_status(_stream(stream))


def prefill_device_status(workspace, stream=None) -> int:
    """Blocks until `stream` is idle, then returns the status word the prefill kernels
    left in `workspace` (OK, or ERR_TIMEOUT if a bounded device-side wait expired)."""
    return lib.ssd_prefill_device_status(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream(stream))


def decode_step(state, x, dt, A, B, C, D, y=None, stream=None) -> torch.Tensor:
    """One cached decode step: updates `state` [b,H,P,N] fp32 in place, returns y fp32
    [b,H,P].  x [b,H,P] and B, C [b,G,N] are fp32 or bf16; dt [b,H], A, D [H] fp32."""
    if x.dim() != 3 or B.dim() != 3 or state.dim() != 4:
        raise ValueError("state must be [b,H,P,N], x [b,H,P], B and C [b,G,N]")
    if x.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {x.dtype}")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("libssd runs on CUDA tensors only")
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    _check(state, "state", (b, H, P, N), torch.float32, dev)
    _check(dt, "dt", (b, H), torch.float32, dev)
    _check(A, "A", (H,), torch.float32, dev)
    _check(B, "B", (b, G, N), x.dtype, dev)
    _check(C, "C", (b, G, N), x.dtype, dev)
    _check(D, "D", (H,), torch.float32, dev)
    if y is None:
        y = torch.empty((b, H, P), dtype=torch.float32, device=dev)
    _check(y, "y", (b, H, P), torch.float32, dev)
    dims = _dims(b, 1, H, P, N, G)
    st = lib.ssd_decode_step(ctypes.byref(dims), _DTYPES[x.dtype], _ptr(state), _ptr(x), _ptr(dt),
                             _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y), _stream(stream))
    if st != OK:
        raise SSDError(st, "ssd_decode_step")
    return y


def window_buffers(state: torch.Tensor, window: int, dtype=torch.bfloat16, ngroups: int = 1):
    """Device buffers for the windowed decode of a state [b,H,P,N]: (win_x [b,W,H,P],
    win_dt [b,W,H] fp32, win_B [b,W,G,N]), in the call's input dtype."""
    b, H, P, N = state.shape
    dev = state.device
    return (torch.empty((b, window, H, P), dtype=dtype, device=dev),
            torch.empty((b, window, H), dtype=torch.float32, device=dev),
            torch.empty((b, window, ngroups, N), dtype=dtype, device=dev))


def decode_window_step(state, buffers, pos: int, x, dt, A, B, C, D, y=None, stream=None) -> torch.Tensor:
    """ssd_decode_window_step: this token's y from the committed `state` (not modified) and
    the `pos` tokens buffered since the last flush; stores the token in slot `pos`."""
    win_x, win_dt, win_B = buffers
    b, H, P, N = state.shape
    G = B.shape[1]
    dev = state.device
    if x.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {x.dtype}")
    W = win_x.shape[1]
    _check(state, "state", (b, H, P, N), torch.float32, dev)
    _check(win_x, "win_x", (b, W, H, P), x.dtype, dev)
    _check(win_dt, "win_dt", (b, W, H), torch.float32, dev)
    _check(win_B, "win_B", (b, W, G, N), x.dtype, dev)
    for name, t, shape, dtype in (("x", x, (b, H, P), x.dtype), ("dt", dt, (b, H), torch.float32),
                                  ("A", A, (H,), torch.float32), ("B", B, (b, G, N), x.dtype),
                                  ("C", C, (b, G, N), x.dtype), ("D", D, (H,), torch.float32)):
        _check(t, name, shape, dtype, dev)
    if y is None:
        y = torch.empty((b, H, P), dtype=torch.float32, device=dev)
    _check(y, "y", (b, H, P), torch.float32, dev)
    st = lib.ssd_decode_window_step(ctypes.byref(_dims(b, 1, H, P, N, G)), _DTYPES[x.dtype], W, int(pos),
                                    _ptr(state), _ptr(win_x), _ptr(win_dt), _ptr(win_B), _ptr(x), _ptr(dt),
                                    _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y), _stream(stream))
    if st != OK:
        raise SSDError(st, "ssd_decode_window_step")
    return y


def decode_window_flush(state, buffers, count: int, A, stream=None) -> torch.Tensor:
    """ssd_decode_window_flush: folds the first `count` buffered tokens into `state`."""
    win_x, win_dt, win_B = buffers
    b, H, P, N = state.shape
    W, G = win_x.shape[1], win_B.shape[2]
    if win_x.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {win_x.dtype}")
    st = lib.ssd_decode_window_flush(ctypes.byref(_dims(b, 1, H, P, N, G)), _DTYPES[win_x.dtype], W, int(count),
                                     _ptr(state), _ptr(win_x), _ptr(win_dt), _ptr(win_B), _ptr(A),
                                     _stream(stream))
    if st != OK:
        raise SSDError(st, "ssd_decode_window_flush")
    return state


def frontend(xbc, conv_w, dt_raw, dt_bias, nheads: int, headdim: int, ngroups: int, dstate: int, conv_b=None,
             conv_state_in=None, conv_state_out=None, x=None, B=None, C=None, dt=None, stream=None):
    """ssd_frontend: conv (width 4, causal, depthwise) + SiLU over xbc [b, L, H*P + 2*G*N],
    split into x [b,L,H,P], B and C [b,L,G,N] (xbc's dtype), and dt = softplus(dt_raw +
    dt_bias) [b,L,H] fp32.  conv_state_in / conv_state_out: fp32 [b, 3, channels] or None;
    they may be the same tensor.  Returns (x, B, C, dt)."""
    b, L, CH = xbc.shape
    H, P, G, N = int(nheads), int(headdim), int(ngroups), int(dstate)
    if CH != H * P + 2 * G * N:
        raise ValueError(f"xbc has {CH} channels, expected {H * P + 2 * G * N}")
    if xbc.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {xbc.dtype}")
    dev = xbc.device
    _check(xbc, "xbc", (b, L, CH), xbc.dtype, dev)
    _check(conv_w, "conv_w", (CH, 4), torch.float32, dev)
    _check(dt_raw, "dt_raw", (b, L, H), torch.float32, dev)
    _check(dt_bias, "dt_bias", (H,), torch.float32, dev)
    if conv_b is not None:
        _check(conv_b, "conv_b", (CH,), torch.float32, dev)
    for name, t in (("conv_state_in", conv_state_in), ("conv_state_out", conv_state_out)):
        if t is not None:
            _check(t, name, (b, 3, CH), torch.float32, dev)
    x = torch.empty((b, L, H, P), dtype=xbc.dtype, device=dev) if x is None else x
    B = torch.empty((b, L, G, N), dtype=xbc.dtype, device=dev) if B is None else B
    C = torch.empty((b, L, G, N), dtype=xbc.dtype, device=dev) if C is None else C
    dt = torch.empty((b, L, H), dtype=torch.float32, device=dev) if dt is None else dt
    st = lib.ssd_frontend(ctypes.byref(_dims(b, L, H, P, N, G)), _DTYPES[xbc.dtype], _ptr(xbc), _ptr(conv_w),
                          _ptr(conv_b), _ptr(conv_state_in), _ptr(conv_state_out), _ptr(dt_raw), _ptr(dt_bias),
                          _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _stream(stream))
    if st != OK:
        raise SSDError(st, "ssd_frontend")
    return x, B, C, dt


def wait_selftest(workspace, limit_ns: int = 1_000_000, expire: bool = True, stream=None) -> int:
    """ssd_wait_selftest, then ssd_prefill_device_status: ERR_TIMEOUT when the bounded
    device wait ran out (expire=True), OK when it completed."""
    nbytes = workspace.numel() * workspace.element_size()
    st = lib.ssd_wait_selftest(_ptr(workspace), nbytes, int(limit_ns), 1 if expire else 0, _stream(stream))
    if st != OK:
        raise SSDError(st, "ssd_wait_selftest")
    return prefill_device_status(workspace, stream)
