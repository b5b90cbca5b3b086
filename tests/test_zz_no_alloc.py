"""ssd_prefill_noalloc, the prefill for callers that cannot allocate device memory.

Plugins inside a host process whose device allocator belongs to the host framework, and
serving loops that forbid allocation once running, cannot hand libssd a workspace; this
entry point takes its scratch from a fixed array inside the library instead.  Its
results must match ssd_prefill's on the same inputs, call after call (the array keeps
the previous call's contents, which must not leak into the next result).

Collected last on purpose (file name), so that a run stopping at the first failure has
run every other test first; it passes alone in a fresh process and after the others.
"""
import numpy as np
import pytest
import torch

from selective_state_space_10_b200 import inputs
from helpers import TOL, assert_close, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_10_b200 import ssd as mod
    return mod


CASES = [  # (batch, seqlen, heads, headdim, dstate, groups, dtype, chunk)
    (1, 1024, 8, 64, 128, 1, "bf16", 256),   # tensor-core path
    (2, 700, 4, 64, 128, 2, "bf16", 128),    # tensor-core path, ragged tail, two groups
    (1, 300, 4, 16, 16, 1, "f32", 64),       # CUDA-core fp32 path
]


def test_noalloc_matches_prefill_on_consecutive_calls(ssd):
    for i, (b, L, H, P, N, G, dtype, Q) in enumerate(CASES + CASES[:1]):
        si = inputs.sequence(b, L, H, P, N, G, dtype, seed=900 + i)
        t = to_device(si)
        need = ssd.prefill_workspace_size(ssd.dims_of_prefill(t["x"], t["B"]),
                                          ssd.BF16 if dtype == "bf16" else ssd.F32, Q)
        assert 0 < need <= ssd.prefill_noalloc_max_workspace()
        y_ref, fs_ref = ssd.prefill(**t, chunk=Q)
        y, fs = ssd.prefill_noalloc(**t, chunk=Q)
        torch.cuda.synchronize()
        y_ref, fs_ref, y, fs = (a.cpu().numpy() for a in (y_ref, fs_ref, y, fs))
        assert_close(y, y_ref, TOL[dtype], f"call {i}: y")
        assert_close(fs, fs_ref, TOL[dtype], f"call {i}: final state")
        assert np.array_equal(y, y_ref) and np.array_equal(fs, fs_ref), "same kernels: results should be identical"
        # the caller holds no workspace: the scratch array's own error word reports the waits
        assert ssd.prefill_noalloc_device_status() == ssd.OK


def test_noalloc_rejects_problems_larger_than_its_scratch(ssd):
    w = inputs.BY_NAME["mamba2_2.7b_prefill"]
    x = torch.empty((1, w.seqlen, w.nheads, w.headdim), dtype=torch.bfloat16, device="cuda")
    dt = torch.empty((1, w.seqlen, w.nheads), device="cuda")
    Bm = torch.empty((1, w.seqlen, 1, w.dstate), dtype=torch.bfloat16, device="cuda")
    hv = torch.zeros(w.nheads, device="cuda")
    with pytest.raises(ssd.SSDError) as e:
        ssd.prefill_noalloc(x, dt, hv, Bm, Bm, hv, chunk=w.chunk)
    assert e.value.status == ssd.ERR_WORKSPACE
