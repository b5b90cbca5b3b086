"""Seeded synthetic inputs for the SSD layer, shared by the tests, the smoke check and the
benchmark.  This module holds no arithmetic of the layer itself: it only draws numbers,
rounds them to the storage dtype the GPU receives, and names the workload shapes.

Value recipe (the same for every workload):
    x      ~ N(0, 1)
    dt     = clamp(softplus(0.5 z + dt_bias_h), 1e-3, 0.1),  z ~ N(0, 1),
             dt_bias_h = inverse-softplus(dt0_h),  dt0_h = exp(U(log 1e-3, log 0.1))
    A_h    = -exp(U(log 1, log 16))
    B, C   ~ N(0, 1) / sqrt(N)
    D_h    ~ N(0, 1)
    decode initial state (batched decode workload) ~ N(0, 0.1^2)
Values are drawn in float32; for bf16 workloads x, B and C are then rounded to bf16
(round-to-nearest-even) and the rounded values are what both the GPU and the oracle see.

Every array has its own random stream keyed by (seed, array id), and per-token arrays are
drawn token-major, so the first L tokens of an (L + k)-token sequence are exactly the
L-token sequence: a prefill of L tokens followed by k decode steps sees the same tokens as
a prefill of L + k tokens.
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

SEED_BASE = 20260000


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str            # "f32" or "bf16": dtype of x, B, C
    decode_steps: int = 0
    decode_only: bool = False
    index: int = 0

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index


# The five workloads: a tiny fp32 layer, the 130M- and 2.7B-shaped prefills, the batched
# 2.7B-shaped decode and the long-context 130M-shaped prefill + decode.
WORKLOADS = [
    Workload("tiny_fp32", 1, 256, 4, 16, 16, 1, 64, "f32", decode_steps=16, index=0),
    Workload("mamba2_130m_prefill", 1, 4096, 24, 64, 128, 1, 256, "bf16", index=1),
    Workload("mamba2_2.7b_prefill", 1, 4096, 80, 64, 128, 1, 256, "bf16", index=2),
    Workload("mamba2_2.7b_decode_b256", 256, 0, 80, 64, 128, 1, 256, "bf16",
             decode_steps=1024, decode_only=True, index=3),
    Workload("mamba2_130m_long_b4", 4, 16384, 24, 64, 128, 1, 256, "bf16",
             decode_steps=256, index=4),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def round_to_bf16(a: np.ndarray):
    """Round float32 -> bf16 (nearest-even).  Returns (bits uint16, values float32)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    bits = rounded.astype(np.uint16)
    vals = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return bits, vals


@dataclass
class SeqInputs:
    """One batch of token sequences.  float32 arrays hold the exact values the GPU sees."""
    x: np.ndarray       # [b, L, H, P]
    dt: np.ndarray      # [b, L, H]
    A: np.ndarray       # [H]
    B: np.ndarray       # [b, L, G, N]
    C: np.ndarray       # [b, L, G, N]
    D: np.ndarray       # [H]
    dtype: str
    bits: dict = field(default_factory=dict)   # bf16 storage (uint16) of x, B, C

    def token_slice(self, t0: int, t1: int) -> "SeqInputs":
        sl = slice(t0, t1)
        bits = {k: np.ascontiguousarray(v[:, sl]) for k, v in self.bits.items()}
        return SeqInputs(np.ascontiguousarray(self.x[:, sl]), np.ascontiguousarray(self.dt[:, sl]),
                         self.A, np.ascontiguousarray(self.B[:, sl]),
                         np.ascontiguousarray(self.C[:, sl]), self.D, self.dtype, bits)

    def head_slice(self, bi, h) -> "SeqInputs":
        """Inputs of a single (batch row, head) pair, as a b=1, H=1, G=1 problem."""
        H = self.x.shape[2]
        G = self.B.shape[2]
        g = h // (H // G)
        return SeqInputs(self.x[bi:bi + 1, :, h:h + 1], self.dt[bi:bi + 1, :, h:h + 1],
                         self.A[h:h + 1], self.B[bi:bi + 1, :, g:g + 1],
                         self.C[bi:bi + 1, :, g:g + 1], self.D[h:h + 1], self.dtype)


def _rng(*key):
    return np.random.default_rng(list(key))


def head_params(nheads: int, seed: int):
    """Per-head A_h, D_h and dt bias."""
    r = _rng(seed, 0)
    A = -np.exp(r.uniform(np.log(1.0), np.log(16.0), nheads)).astype(np.float32)
    D = r.standard_normal(nheads).astype(np.float32)
    dt0 = np.exp(r.uniform(np.log(1e-3), np.log(1e-1), nheads))
    dt_bias = dt0 + np.log(-np.expm1(-dt0))  # inverse softplus of dt0
    return A, D, dt_bias


def _dt_from(z: np.ndarray, dt_bias: np.ndarray) -> np.ndarray:
    v = 0.5 * z.astype(np.float64) + dt_bias
    sp = np.where(v > 20.0, v, np.log1p(np.exp(np.minimum(v, 20.0))))
    return np.clip(sp, 1e-3, 0.1).astype(np.float32)


def _maybe_bf16(a: np.ndarray, dtype: str, name: str, bits: dict) -> np.ndarray:
    if dtype == "bf16":
        b, v = round_to_bf16(a)
        bits[name] = b
        return v
    return np.ascontiguousarray(a, dtype=np.float32)


def sequence(batch, seqlen, nheads, headdim, dstate, ngroups, dtype, seed) -> SeqInputs:
    """Prefill inputs; token-major streams make prefixes of longer sequences identical."""
    A, D, dt_bias = head_params(nheads, seed)
    L, b, H, P, N, G = seqlen, batch, nheads, headdim, dstate, ngroups
    x = _rng(seed, 1).standard_normal((L, b, H, P), dtype=np.float32).transpose(1, 0, 2, 3)
    z = _rng(seed, 2).standard_normal((L, b, H), dtype=np.float32).transpose(1, 0, 2)
    Bm = _rng(seed, 3).standard_normal((L, b, G, N), dtype=np.float32).transpose(1, 0, 2, 3)
    Cm = _rng(seed, 4).standard_normal((L, b, G, N), dtype=np.float32).transpose(1, 0, 2, 3)
    scale = np.float32(1.0 / np.sqrt(N))
    bits = {}
    x = _maybe_bf16(x, dtype, "x", bits)
    Bm = _maybe_bf16(Bm * scale, dtype, "B", bits)
    Cm = _maybe_bf16(Cm * scale, dtype, "C", bits)
    dt = np.ascontiguousarray(_dt_from(z, dt_bias[None, None, :]))
    return SeqInputs(x, dt, A, Bm, Cm, D, dtype, bits)


def workload_sequence(w: Workload, seqlen: Optional[int] = None, batch: Optional[int] = None,
                      seed: Optional[int] = None) -> SeqInputs:
    return sequence(batch or w.batch, w.seqlen if seqlen is None else seqlen, w.nheads,
                    w.headdim, w.dstate, w.ngroups, w.dtype, w.seed if seed is None else seed)


def decode_initial_state(w: Workload, seed: Optional[int] = None) -> np.ndarray:
    seed = w.seed if seed is None else seed
    shape = (w.batch, w.nheads, w.headdim, w.dstate)
    return (_rng(seed, 6).standard_normal(shape, dtype=np.float32) * np.float32(0.1))


def decode_token(w: Workload, step: int, seed: Optional[int] = None) -> SeqInputs:
    """Fresh inputs of one decode step (seqlen axis of length 1)."""
    seed = w.seed if seed is None else seed
    A, D, dt_bias = head_params(w.nheads, seed)
    r = _rng(seed, 5, step)
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    x = r.standard_normal((b, 1, H, P), dtype=np.float32)
    z = r.standard_normal((b, 1, H), dtype=np.float32)
    Bm = r.standard_normal((b, 1, G, N), dtype=np.float32) * np.float32(1.0 / np.sqrt(N))
    Cm = r.standard_normal((b, 1, G, N), dtype=np.float32) * np.float32(1.0 / np.sqrt(N))
    bits = {}
    x = _maybe_bf16(x, w.dtype, "x", bits)
    Bm = _maybe_bf16(Bm, w.dtype, "B", bits)
    Cm = _maybe_bf16(Cm, w.dtype, "C", bits)
    dt = _dt_from(z, dt_bias[None, None, :])
    return SeqInputs(x, dt, A, Bm, Cm, D, w.dtype, bits)
