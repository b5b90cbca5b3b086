"""Shared helpers of the GPU parity tests: upload seeded inputs, call libssd through its
binding, compare against the oracle with the stated tolerances."""
import numpy as np
import torch

# Max |y - y_ref| <= TOL * RMS(y_ref); the same relative bound applies to the final state.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def to_device(si, device="cuda"):
    """SeqInputs -> dict of device tensors with the dtypes libssd takes."""
    def inp(name):
        if si.dtype == "bf16":
            bits = si.bits[name]
            return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(getattr(si, name))).to(device)
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    return dict(x=inp("x"), dt=f(si.dt), A=f(si.A), B=inp("B"), C=inp("C"), D=f(si.D))


def decode_args(t):
    """Prefill-shaped token tensors (seqlen 1) -> decode-shaped ones."""
    return dict(x=t["x"][:, 0].contiguous(), dt=t["dt"][:, 0].contiguous(), A=t["A"],
                B=t["B"][:, 0].contiguous(), C=t["C"][:, 0].contiguous(), D=t["D"])


def rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.abs(got - ref).max() / max(rms, 1e-300))


def assert_close(got, ref, tol, what=""):
    e = rel_err(got, ref)
    assert np.isfinite(np.asarray(got)).all(), f"{what}: non-finite values"
    assert e <= tol, f"{what}: max|d| / RMS = {e:.3e} > {tol:.1e}"
    return e
