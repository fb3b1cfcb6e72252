"""fp64 CPU oracle for the selective-scan forward -- Python side.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
and the benchmark's CPU-baseline / reference legs may import this module.  It
shares nothing with the CUDA path: it compiles and loads its own C library
(``sscan_oracle.c``) with gcc and never touches the product package.

The C code computes the plain definition (one sequential loop over tokens per
(batch, channel) row, in double precision):

    Abar = exp(delta * A)                                   per token, per state
    Euler  bu = delta * B * u      |  ZOH  bu = (exp(delta*A) - 1) / A * B * u
    h      = Abar * h + bu                                  h before token 0 = h0 or 0
    y      = sum_n C[n] * h[n]                              state after the update
    h_final = h after the last token

and, optionally, the fused prologue delta <- softplus(delta + delta_bias[d]) and
epilogue y <- y * silu(z) ("tm_ssm_selective", section "The mechanism:
parameters as functions of the input"; "Selective State-Space Models (Mamba)
and Hardware-Aware Scans", section 4), following "tm_ssm_selective" (Transformer Math), section "Discretization becomes
a per-token operation", and the selective_scan reference loop of "12. Selective
State Space".  The header comment of ``sscan_oracle.c`` lists the readings taken
where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sscan_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libsscan_oracle.so")

_lock = threading.Lock()
_lib = None


def compile_source(src: str, out: str) -> str:
    """gcc the oracle's C source into a shared library (no fast-math, no FMA contraction)."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-pthread", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle's own library if missing or older than its source."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        compile_source(_SRC, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str):
    """ctypes handle of a build of the oracle's C source at ``path``."""
    return _bind(path)


def _bind(path):
    lib = ctypes.CDLL(path)
    i64, dp, ip = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.sscan_oracle_forward.argtypes = [i64, i64, i64, i64, dp, dp, dp, dp, dp, dp,
                                         ip, dp, dp, ip]
    lib.sscan_oracle_forward.restype = ip
    lib.sscan_oracle_rows.argtypes = [i64, i64, i64, i64, dp, dp, dp, dp, dp, dp, dp,
                                      ip, dp, dp, ip]
    lib.sscan_oracle_rows.restype = ip
    lib.sscan_oracle_forward_ex.argtypes = [i64, i64, i64, i64, dp, dp, dp, dp, dp, dp,
                                            ip, dp, ip, dp, dp, dp, ip]
    lib.sscan_oracle_forward_ex.restype = ip
    lib.sscan_oracle_rows_ex.argtypes = [i64, i64, i64, i64, dp, dp, dp, dp, dp, dp, dp,
                                         ip, dp, ip, dp, dp, dp, ip]
    lib.sscan_oracle_rows_ex.restype = ip
    lib.sscan_oracle_backward.argtypes = [i64, i64, i64, i64] + [dp] * 6 + [ip] + [dp] * 8 + [ip]
    lib.sscan_oracle_backward.restype = ip
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def host_threads() -> int:
    """Threads the oracle uses by default: every core this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _f64(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data


def forward(u, delta, A, B, C, h0=None, zoh=False, nthreads=None, lib=None,
            delta_bias=None, softplus=False, z=None):
    """Selective-scan forward in fp64 over full tensors.

    u, delta: [Bt, L, D]; A: [D, N]; B, C: [Bt, L, N]; h0: [Bt, D, N] or None.
    delta_bias: [D] or None; softplus: apply softplus to delta (+ bias);
    z: [Bt, L, D] gate or None (y is multiplied by silu(z)).
    Inputs are widened to fp64 exactly (fp32 and bf16 values are exact in fp64).
    Returns (y [Bt, L, D], h_final [Bt, D, N]) as float64 arrays.
    ``lib`` selects another build of the same C source (default: the oracle's own).
    """
    u, delta, A, B, C, h0, delta_bias, z = map(_f64, (u, delta, A, B, C, h0, delta_bias, z))
    Bt, L, D = u.shape
    N = A.shape[1]
    assert delta.shape == (Bt, L, D) and A.shape == (D, N)
    assert B.shape == (Bt, L, N) and C.shape == (Bt, L, N)
    assert h0 is None or h0.shape == (Bt, D, N)
    assert delta_bias is None or delta_bias.shape == (D,)
    assert z is None or z.shape == (Bt, L, D)
    y = np.empty((Bt, L, D), dtype=np.float64)
    hf = np.empty((Bt, D, N), dtype=np.float64)
    rc = (lib or _load()).sscan_oracle_forward_ex(
        Bt, L, D, N, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0), int(bool(zoh)),
        _ptr(delta_bias), int(bool(softplus)), _ptr(z), _ptr(y), _ptr(hf),
        int(nthreads or host_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return y, hf


def forward_rows(rows, u, delta, A, B, C, h0=None, zoh=False, nthreads=None, lib=None,
                 delta_bias=None, softplus=False, z=None):
    """The recurrence on selected (b, d) rows only (rows are independent, so exact).

    rows: sequence of (b, d) pairs.  u, delta: [Bt, L, D] arrays of any float
    dtype (only the selected channels are gathered and widened); A: [D, N];
    B, C: [Bt, L, N]; h0: [Bt, D, N] or None; delta_bias [D], softplus and the
    gate z [Bt, L, D] as in ``forward``.
    Returns (y_rows [R, L], h_final_rows [R, N]) as float64.
    """
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
    R = rows.shape[0]
    Bt, L, D = u.shape
    N = A.shape[1]
    rb = np.ascontiguousarray(rows[:, 0])
    rd = rows[:, 1]
    u_r = np.ascontiguousarray(np.asarray(u)[rb, :, rd].astype(np.float64))
    d_r = np.ascontiguousarray(np.asarray(delta)[rb, :, rd].astype(np.float64))
    A_r = np.ascontiguousarray(np.asarray(A, dtype=np.float64)[rd])
    h0_r = None if h0 is None else np.ascontiguousarray(np.asarray(h0, dtype=np.float64)[rb, rd])
    bias_r = None if delta_bias is None else np.ascontiguousarray(
        np.asarray(delta_bias, dtype=np.float64)[rd])
    z_r = None if z is None else np.ascontiguousarray(np.asarray(z)[rb, :, rd].astype(np.float64))
    B64, C64 = _f64(B), _f64(C)
    y = np.empty((R, L), dtype=np.float64)
    hf = np.empty((R, N), dtype=np.float64)
    rc = (lib or _load()).sscan_oracle_rows_ex(
        R, L, N, Bt, _ptr(rb), _ptr(u_r), _ptr(d_r), _ptr(A_r), _ptr(B64), _ptr(C64), _ptr(h0_r),
        int(bool(zoh)), _ptr(bias_r), int(bool(softplus)), _ptr(z_r), _ptr(y), _ptr(hf),
        int(nthreads or host_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return y, hf


def backward(u, delta, A, B, C, h0=None, zoh=False, dy=None, dh_final=None, nthreads=None, lib=None):
    """Gradients of the plain forward in fp64: given dy [Bt, L, D] (and optionally
    dh_final [Bt, D, N]) returns a dict with du, ddelta ([Bt, L, D]), dA ([D, N]),
    dB, dC ([Bt, L, N]) and dh0 ([Bt, D, N]).  See ``sscan_oracle.c`` ("backward")."""
    u, delta, A, B, C, h0, dy, dh_final = map(_f64, (u, delta, A, B, C, h0, dy, dh_final))
    Bt, L, D = u.shape
    N = A.shape[1]
    assert dy is not None and dy.shape == (Bt, L, D)
    out = {"du": np.empty((Bt, L, D)), "ddelta": np.empty((Bt, L, D)), "dA": np.empty((D, N)),
           "dB": np.empty((Bt, L, N)), "dC": np.empty((Bt, L, N)), "dh0": np.empty((Bt, D, N))}
    rc = (lib or _load()).sscan_oracle_backward(
        Bt, L, D, N, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0), int(bool(zoh)),
        _ptr(dy), _ptr(dh_final), _ptr(out["du"]), _ptr(out["ddelta"]), _ptr(out["dA"]), _ptr(out["dB"]),
        _ptr(out["dC"]), _ptr(out["dh0"]), int(nthreads or host_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle backward failed with code {rc}")
    return out


def backward_fused(u, delta_raw, A, B, C, h0=None, zoh=False, dy=None, dh_final=None,
                   delta_bias=None, softplus=True, z=None, nthreads=None):
    """Gradients of the fused forward (delta' = softplus(delta_raw + bias), y = scan * silu(z))
    in fp64, by the chain rule around the plain backward:

        scan output ys = y / silu(z);   dys = dy * silu(z);   dz = dy * ys * silu'(z),
        silu'(z) = sigmoid(z) (1 + z (1 - sigmoid(z)));
        d delta_raw = d delta' * sigmoid(delta_raw + bias)   (softplus' = sigmoid; 1 without softplus),
        d bias[d] = sum over b and t of d delta_raw.

    Returns the plain backward's dict (ddelta replaced by the gradient w.r.t. delta_raw)
    plus ddelta_bias ([D]) and dz ([Bt, L, D]) when those inputs are given."""
    u, delta_raw, A, B, C, h0, dy, dh_final, delta_bias, z = map(
        _f64, (u, delta_raw, A, B, C, h0, dy, dh_final, delta_bias, z))
    s = delta_raw if delta_bias is None else delta_raw + delta_bias[None, None, :]
    dprime = (np.maximum(s, 0.0) + np.log1p(np.exp(-np.abs(s)))) if softplus else s
    dys = dy
    out_extra = {}
    if z is not None:
        sig = 1.0 / (1.0 + np.exp(-z))
        ys, _ = forward(u, dprime, A, B, C, h0, zoh, nthreads=nthreads)
        dys = dy * z * sig
        out_extra["dz"] = dy * ys * sig * (1.0 + z * (1.0 - sig))
    g = backward(u, dprime, A, B, C, h0, zoh, dys, dh_final, nthreads=nthreads)
    if softplus:
        g["ddelta"] = g["ddelta"] / (1.0 + np.exp(-s))
    if delta_bias is not None:
        out_extra["ddelta_bias"] = g["ddelta"].sum(axis=(0, 1))
    g.update(out_extra)
    return g
