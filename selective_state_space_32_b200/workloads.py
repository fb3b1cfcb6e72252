"""Workload table and seeded synthetic inputs for the selective-scan forward.

This module only draws inputs.  It holds none of the scan's arithmetic, so the
CUDA path and the fp64 oracle can both be fed from it without sharing any of
the method: it produces u, delta, A, B, C (and h0) as plain arrays, in the
shapes of "Mamba & Mamba-2 Architecture", section 1 (u, delta: [B, L, D];
B, C: [B, L, N]; A: [D, N]) and "tm_ssm_selective", section "The mechanism:
parameters as functions of the input".

Distributions (the same for every workload unless noted):
  * dt[d]  log-uniform in [1e-3, 1e-1] per channel,
  * z ~ N(0, 1), delta = softplus(0.5 z + softplus^-1(dt[d])): the softplus
    parametrisation of the step and the [0.001, 0.1] initial range described
    in "tm_ssm_selective", sections "The mechanism ..." and "Reading delta as
    a memory horizon",
  * u, B, C ~ N(0, 1),
  * A = -exp(A_log) with A_log[d, n] = log(n + 1) (S4D-real), so A[d, n] = -(n + 1),
  * h0 ~ N(0, 0.1^2) where a workload has a nonzero initial state,
  * the long-sequence workload marks round(0.32 L) time positions per batch row
    as reset tokens (delta + 3) and scales delta by 0.01 elsewhere,
  * fused workloads (the kernel applies delta <- softplus(delta + bias) and
    y <- y * silu(z) itself) store the raw delta 0.5 z and the per-channel
    bias softplus^-1(dt[d]) (fp32), so the effective delta has the same
    distribution as above; their gate z ~ N(0, 1) is drawn after everything
    else.

Draw order from numpy PCG64(seed): dt, reset mask, z, u, B, C, h0, all fp64 in
C order.  Values are then rounded to fp32 (numpy, round-to-nearest-even) and,
for bf16 workloads, from fp32 to bf16 (round-to-nearest-even on the bit
pattern); A and h0 stay fp32.  bf16 arrays are returned as uint16 bit patterns.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

SEED_BASE = 20261202


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    D: int
    N: int
    dtype: str            # "f32" or "bf16": dtype of u, delta, B, C and y
    h0_std: float         # 0.0: no initial state (h0 = 0)
    zoh: bool             # exact zero-order-hold input term instead of Euler
    reset_frac: float     # fraction of time positions that are reset tokens (0: none)
    index: int            # seed offset
    fused: bool = False   # raw delta + bias + gate z (the kernel's fused prologue / epilogue)

    @property
    def elements(self) -> int:
        """Scanned elements B*L*D (the throughput unit)."""
        return self.B * self.L * self.D

    @property
    def updates(self) -> int:
        """State updates B*L*D*N."""
        return self.B * self.L * self.D * self.N

    @property
    def itemsize(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def algorithmic_bytes(self) -> int:
        """Bytes that must cross HBM once: u, delta, y ([B,L,D]), B, C ([B,L,N]),
        A ([D,N] fp32), h_final and, when given, h0 ([B,D,N] fp32)."""
        s = self.itemsize
        return (3 * s * self.B * self.L * self.D + 2 * s * self.B * self.L * self.N
                + 4 * self.D * self.N + 4 * self.B * self.D * self.N * (1 + (self.h0_std > 0))
                + (s * self.B * self.L * self.D + 4 * self.D if self.fused else 0))

    def shape_dict(self) -> dict:
        return {"B": self.B, "L": self.L, "D": self.D, "N": self.N, "dtype": self.dtype,
                "h0": self.h0_std > 0, "zoh": self.zoh, "fused": self.fused}


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 256, 64, 16, "f32", 0.0, False, 0.0, 0),
    "mamba130m_f32": Workload("mamba130m_f32", 8, 2048, 1536, 16, "f32", 0.0, False, 0.0, 1),
    "mamba1p4b_bf16": Workload("mamba1p4b_bf16", 2, 8192, 4096, 16, "bf16", 0.1, False, 0.0, 2),
    "longseq_bf16": Workload("longseq_bf16", 1, 131072, 2048, 16, "bf16", 0.1, False, 0.32, 3),
    "zoh_n64_bf16": Workload("zoh_n64_bf16", 16, 1024, 5120, 64, "bf16", 0.0, True, 0.0, 4),
    # one decode step (a single token per sequence, state carried in and out) for a
    # batch of 256 sequences of a layer with D = 2048, N = 16
    "decode_b256_f32": Workload("decode_b256_f32", 256, 1, 2048, 16, "f32", 0.1, False, 0.0, 5),
    # the bench shape with the Mamba block's softplus(delta + bias) and silu(z) gate fused
    "mamba130m_fused_f32": Workload("mamba130m_fused_f32", 8, 2048, 1536, 16, "f32", 0.0, False, 0.0, 6,
                                    fused=True),
    "mamba1p4b_fused_bf16": Workload("mamba1p4b_fused_bf16", 2, 8192, 4096, 16, "bf16", 0.1, False, 0.0, 7,
                                     fused=True),
}
ORDER = ["tiny_f32", "mamba130m_f32", "mamba1p4b_bf16", "longseq_bf16", "zoh_n64_bf16"]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def as_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    """The fp32 values an array of the given storage dtype holds (exact)."""
    return bf16_bits_to_f32(x) if dtype == "bf16" else np.asarray(x, dtype=np.float32)


def _store(v64: np.ndarray, dtype: str) -> np.ndarray:
    v32 = v64.astype(np.float32)
    return f32_to_bf16_bits(v32) if dtype == "bf16" else v32


def _softplus(v):
    return np.logaddexp(0.0, v)


def _inv_softplus(y):
    return y + np.log(-np.expm1(-y))


def generate(B: int, L: int, D: int, N: int, dtype: str = "f32", h0_std: float = 0.0,
             reset_frac: float = 0.0, seed: int = SEED_BASE, A_jitter: float = 0.0,
             block: int = 1 << 22, fused: bool = False) -> dict:
    """Seeded inputs of the given shape (see the module docstring for the recipe).

    A_jitter > 0 adds N(0, A_jitter^2) to A_log (drawn last), so tests can use
    a non-integer A.  Large arrays are drawn in blocks of ``block`` values; the
    stream is the same as a single draw.
    Returns a dict with u, delta ([B,L,D]), A ([D,N] fp32), B, C ([B,L,N]),
    h0 ([B,D,N] fp32 or None) and dtype; with ``fused`` also delta_bias ([D]
    fp32) and z ([B,L,D]), and delta is the raw (pre-softplus) value.
    """
    assert dtype in ("f32", "bf16")
    assert not (fused and reset_frac > 0)
    rng = np.random.Generator(np.random.PCG64(seed))
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), size=D))
    reset = None
    if reset_frac > 0:
        k = int(round(reset_frac * L))
        reset = np.zeros((B, L), dtype=bool)
        for b in range(B):
            reset[b, rng.permutation(L)[:k]] = True
    bias = _inv_softplus(dt)
    bias32 = bias.astype(np.float32)

    total = B * L * D
    sdt = np.uint16 if dtype == "bf16" else np.float32
    delta = np.empty(total, dtype=sdt)
    for s in range(0, total, block):
        e = min(total, s + block)
        z = rng.standard_normal(e - s)
        idx = np.arange(s, e)
        d = idx % D
        v = 0.5 * z if fused else _softplus(0.5 * z + bias[d])
        if reset is not None:
            bt = idx // D
            r = reset.reshape(-1)[bt]
            v = np.where(r, v + 3.0, v * 0.01)
        delta[s:e] = _store(v, dtype)
    u = np.empty(total, dtype=sdt)
    for s in range(0, total, block):
        e = min(total, s + block)
        u[s:e] = _store(rng.standard_normal(e - s), dtype)
    Bm = _store(rng.standard_normal(B * L * N), dtype).reshape(B, L, N)
    Cm = _store(rng.standard_normal(B * L * N), dtype).reshape(B, L, N)
    h0 = None
    if h0_std > 0:
        h0 = (h0_std * rng.standard_normal(B * D * N)).astype(np.float32).reshape(B, D, N)
    A_log = np.log(np.arange(1, N + 1, dtype=np.float64))[None, :].repeat(D, axis=0)
    if A_jitter > 0:
        A_log = A_log + A_jitter * rng.standard_normal((D, N))
    A = (-np.exp(A_log)).astype(np.float32)
    out = {"u": u.reshape(B, L, D), "delta": delta.reshape(B, L, D), "A": A,
           "B": Bm, "C": Cm, "h0": h0, "dtype": dtype, "delta_bias": None, "z": None}
    if fused:
        out["delta_bias"] = bias32
        zg = np.empty(B * L * D, dtype=sdt)
        for s in range(0, B * L * D, block):
            e = min(B * L * D, s + block)
            zg[s:e] = _store(rng.standard_normal(e - s), dtype)
        out["z"] = zg.reshape(B, L, D)
    return out


def make_inputs(w: Workload) -> dict:
    """Inputs of a named workload, seeded with SEED_BASE + its index."""
    return generate(w.B, w.L, w.D, w.N, w.dtype, w.h0_std, w.reset_frac, SEED_BASE + w.index,
                    fused=w.fused)


# --------------------------------------------------------------------------
# Mamba-2 SSD form ("Mamba & Mamba-2 Architecture", section 3): one scalar
# transition per head, B and C shared by the heads.

@dataclasses.dataclass(frozen=True)
class SsdWorkload:
    name: str
    B: int
    L: int
    H: int
    P: int
    N: int
    h0_std: float
    index: int

    @property
    def elements(self) -> int:
        """Scanned elements B*L*H*P (the heads' channels, as B*L*D for the selective scan)."""
        return self.B * self.L * self.H * self.P

    def algorithmic_bytes(self) -> int:
        """x and y (bf16), delta (fp32, [B,L,H]), B and C (bf16), A, h_final and h0 (fp32)."""
        return (2 * 2 * self.B * self.L * self.H * self.P + 4 * self.B * self.L * self.H
                + 2 * 2 * self.B * self.L * self.N + 4 * self.H
                + 4 * self.B * self.H * self.N * self.P * (1 + (self.h0_std > 0)))

    def flops(self) -> int:
        """Useful multiply-adds x 2 of the block algorithm with 128-token blocks: per block
        and head, C B^T (Q*Q*N; counted once per batch row and block, shared by the heads),
        the causal half of (S o L) X (Q*(Q+1)/2*P), C h_in and B^T (w X) (Q*N*P each)."""
        q = 128
        nblk = -(-self.L // q)
        per_bh = nblk * (q * (q + 1) // 2 * self.P + 2 * q * self.N * self.P)
        return 2 * (self.B * self.H * per_bh + self.B * nblk * q * q * self.N)


SSD_WORKLOADS = {
    # parity-sized: two full blocks and a ragged one, a nonzero initial state
    "ssd_small": SsdWorkload("ssd_small", 2, 300, 4, 64, 128, 0.1, 20),
    # a Mamba-2 1.3B-like layer (d_model 2048, expand 2 -> 4096 channels = 64 heads of 64,
    # state 128, one group), 8 sequences of 2048 tokens
    "ssd_mamba2_1p3b": SsdWorkload("ssd_mamba2_1p3b", 8, 2048, 64, 64, 128, 0.0, 21),
}


def generate_ssd(B: int, L: int, H: int, P: int, N: int, h0_std: float = 0.0, seed: int = SEED_BASE,
                 reset_frac: float = 0.0, A_zero: bool = False) -> dict:
    """Seeded inputs of the SSD form.

    Draw order from PCG64(seed), fp64: dt[h] log-uniform in [1e-3, 1e-1] per head;
    A_log[h] = log(U[1, 16]) (A = -exp(A_log) in [-16, -1], the Mamba-2 range);
    the reset mask (reset_frac > 0: round(reset_frac * L) positions per batch row get
    delta + 3, the others delta * 0.01, as for the long-sequence selective scan);
    z ~ N(0, 1) [B, L, H] -> delta = softplus(0.5 z + softplus^-1(dt[h])) kept in fp32;
    x ~ N(0, 1) [B, L, H, P]; B, C ~ N(0, 1) [B, L, N]; h0 ~ N(0, h0_std^2)
    [B, H, N, P] fp32 when h0_std > 0.  x, B, C are rounded to bf16 (uint16 bit
    patterns).  A_zero sets A = 0 (every decay 1: causal linear attention)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), size=H))
    A_log = np.log(rng.uniform(1.0, 16.0, size=H))
    reset = None
    if reset_frac > 0:
        k = int(round(reset_frac * L))
        reset = np.zeros((B, L), dtype=bool)
        for b in range(B):
            reset[b, rng.permutation(L)[:k]] = True
    z = rng.standard_normal((B, L, H))
    delta = _softplus(0.5 * z + _inv_softplus(dt)[None, None, :])
    if reset is not None:
        delta = np.where(reset[:, :, None], delta + 3.0, delta * 0.01)
    x = _store(rng.standard_normal(B * L * H * P), "bf16").reshape(B, L, H, P)
    Bm = _store(rng.standard_normal(B * L * N), "bf16").reshape(B, L, N)
    Cm = _store(rng.standard_normal(B * L * N), "bf16").reshape(B, L, N)
    h0 = None
    if h0_std > 0:
        h0 = (h0_std * rng.standard_normal(B * H * N * P)).astype(np.float32).reshape(B, H, N, P)
    A = np.zeros(H, np.float32) if A_zero else (-np.exp(A_log)).astype(np.float32)
    return {"x": x, "delta": delta.astype(np.float32), "A": A, "B": Bm, "C": Cm, "h0": h0}


def make_ssd_inputs(w: SsdWorkload) -> dict:
    return generate_ssd(w.B, w.L, w.H, w.P, w.N, w.h0_std, SEED_BASE + w.index)
