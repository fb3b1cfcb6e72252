"""Parity of the CUDA backward pass with the fp64 oracle's backward (B200).

The oracle's backward, plain and fused, is pinned by finite differences of the
forward oracle (tests/test_oracle_backward.py).  Cases cover N = 16, 32 and 64,
Euler and ZOH (with some A = 0, the limit branch), fp32 and bf16 I/O, ragged
channel counts (D not a multiple of a block's channels) and ragged sequences
(L not a multiple of the 8-token recompute chunk), with and without h0 and
dh_final, and the fused layer (softplus(delta + bias) and the silu(z) gate:
gradients of the raw delta, the bias and z).  Tolerances are those of the
forward: fp32 relative L2 <= 1e-5 and |err| <= 1e-4 (1 + |ref|) elementwise on
every gradient; bf16 inputs relative L2 <= 5e-3.  dA, dB, dC and the bias
gradient are fp32 sums over many terms accumulated with atomics, well inside
those bounds.

One allowance, from the arithmetic: the per-token gradients du, ddelta and dz
are products of the reverse-scan state g, which is multiplied by one Abar per
token over the whole horizon, and every Abar comes from the MUFU 2^x with a
relative error up to 2^-22.  Over L tokens that error compounds: a fp32 model
of the backward with exact exponentials stays at 4.5e-5 (scaled elementwise)
on the 512-token case below, and with exponentials perturbed by 2^-22 reaches
2.7e-4.  Their elementwise bound is therefore 1e-4 (1 + |ref|) max(1, L/256):
the forward's bound up to a 256-token horizon, growing with the horizon beyond.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import oracle as O
from selective_state_space_32_b200 import sscan as S
from selective_state_space_32_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_32_b200 import build
    build.build()
    S.lib()


def _rel(got, ref):
    got = np.asarray(got, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))


TOKENWISE = ("du", "ddelta", "dz")


def _check(got, ref, keys, dt, L=1):
    for k in keys:
        gv = got[k].float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(gv)), k
        r = _rel(gv, ref[k])
        if dt == "f32":
            assert r <= 1e-5, f"{k}: rel L2 {r:.3e} > 1e-5"
            m = float((np.abs(gv - ref[k]) / (1.0 + np.abs(ref[k]))).max()) if gv.size else 0.0
            bound = 1e-4 * (max(1.0, L / 256) if k in TOKENWISE else 1.0)
            assert m <= bound, f"{k}: max |err|/(1+|ref|) {m:.3e} > {bound:.1e}"
        else:
            assert r <= 5e-3, f"{k}: rel L2 {r:.3e} > 5e-3"


def _dy(shape, dt, seed):
    rng = np.random.default_rng(seed)
    dy32 = rng.standard_normal(shape).astype(np.float32)
    return dy32 if dt == "f32" else W.f32_to_bf16_bits(dy32)


CASES = [
    # (B, L, D, N, dtype, h0, dhf, zoh, zero_a)
    (2, 37, 70, 16, "f32", True, True, False, False),     # ragged D and L
    (2, 64, 128, 16, "f32", False, False, False, False),
    (3, 45, 200, 16, "f32", True, True, True, True),       # ZOH with A = 0 entries
    (2, 512, 256, 16, "f32", True, True, False, False),    # longer sequence
    (2, 100, 96, 16, "bf16", True, True, False, False),
    (1, 80, 64, 16, "bf16", True, False, True, False),
    (1, 1, 32, 16, "f32", True, True, False, False),       # a single token
    (2, 75, 44, 32, "f32", True, True, True, False),       # N = 32, ZOH
    (2, 130, 36, 32, "bf16", True, True, False, False),
    (2, 50, 21, 64, "f32", True, True, True, True),        # N = 64, ZOH with A = 0, ragged D
    (1, 200, 40, 64, "bf16", False, True, True, False),
    (2, 77, 45, 16, "bf16", True, True, False, False),     # odd D with bf16: rows not 4-byte aligned, unstaged
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}{'_zoh' if c[7] else ''}"
                                              f"{'_a0' if c[8] else ''}{'_h0' if c[5] else ''}{'_dhf' if c[6] else ''}"
                                              for c in CASES])
def test_backward_matches_oracle(case):
    Bt, L, D, N, dt, with_h0, with_dhf, zoh, zero_a = case
    g = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, seed=8000 + L + D + N, A_jitter=0.3)
    if zero_a:
        g["A"][::7, 3] = 0.0
    dy = _dy((Bt, L, D), dt, L + D)
    dhf = np.random.default_rng(N).standard_normal((Bt, D, N)).astype(np.float32) if with_dhf else None
    d = P.to_device(g)
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    dy_d = P.to_device({**g, "u": dy})["u"]
    dhf_d = None if dhf is None else torch.from_numpy(dhf).cuda()
    plan = S.Plan(Bt, L, D, N, tdt, zoh)
    got = plan.backward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"], dy_d, dhf_d)
    torch.cuda.synchronize()
    v = P.host_values(g)
    ref = O.backward(v["u"], v["delta"], v["A"], v["B"], v["C"], v["h0"], zoh, W.as_f32(dy, dt), dhf)
    _check(got, ref, ("du", "ddelta", "dA", "dB", "dC", "dh0"), dt, L)
    plan.close()


FUSED = [
    # (B, L, D, N, dtype, zoh, softplus, bias, gate)
    (2, 70, 64, 16, "f32", False, True, True, True),
    (2, 45, 40, 32, "f32", True, True, True, True),
    (1, 66, 24, 64, "f32", False, True, False, True),
    (2, 90, 96, 16, "bf16", False, True, True, True),
    (2, 40, 48, 16, "f32", False, False, True, False),      # bias only, no softplus, no gate
    (1, 33, 16, 16, "f32", False, True, True, False),       # softplus + bias, no gate
    (2, 50, 33, 16, "bf16", False, True, True, True),       # odd D with bf16 (unstaged)
]


@pytest.mark.parametrize("case", FUSED, ids=[f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}{'_zoh' if c[5] else ''}"
                                              f"{'_sp' if c[6] else ''}{'_bias' if c[7] else ''}{'_gate' if c[8] else ''}"
                                              for c in FUSED])
def test_fused_backward_matches_oracle(case):
    Bt, L, D, N, dt, zoh, sp, with_bias, with_gate = case
    g = W.generate(Bt, L, D, N, dt, 0.1, seed=8500 + L + D + N, A_jitter=0.3, fused=True)
    if not sp:
        # without softplus the step is raw + bias itself: keep it positive (a negative step
        # makes Abar > 1 and the state grow without bound)
        raw = np.abs(W.as_f32(g["delta"], dt)) * np.float32(0.05)
        g["delta"] = raw if dt == "f32" else W.f32_to_bf16_bits(raw)
        g["delta_bias"] = np.abs(g["delta_bias"]) * np.float32(0.01)
    if not with_bias:
        g["delta_bias"] = None
    if not with_gate:
        g["z"] = None
    dy = _dy((Bt, L, D), dt, 3 * L + D)
    dhf = np.random.default_rng(D).standard_normal((Bt, D, N)).astype(np.float32)
    d = P.to_device(g)
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    dy_d = P.to_device({**g, "u": dy})["u"]
    plan = S.Plan(Bt, L, D, N, tdt, zoh, delta_softplus=sp)
    got = plan.backward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"], dy_d, torch.from_numpy(dhf).cuda(),
                        delta_bias=d["delta_bias"], z=d["z"])
    torch.cuda.synchronize()
    v = P.host_values(g)
    ref = O.backward_fused(v["u"], v["delta"], v["A"], v["B"], v["C"], v["h0"], zoh, W.as_f32(dy, dt), dhf,
                           delta_bias=v["delta_bias"], softplus=sp, z=v["z"])
    keys = ["du", "ddelta", "dA", "dB", "dC", "dh0"] + (["ddelta_bias"] if with_bias else []) + \
        (["dz"] if with_gate else [])
    _check(got, ref, keys, dt, L)
    plan.close()


def test_backward_forward_consistency():
    # the backward's recomputed states agree with the forward: with dy = 0 and
    # dh_final = e_k, dh0 is the k-th row of d h_final / d h0 = prod Abar (diagonal)
    Bt, L, D, N = 1, 50, 32, 16
    g = W.generate(Bt, L, D, N, "f32", 0.1, seed=8100, A_jitter=0.2)
    d = P.to_device(g)
    plan = S.Plan(Bt, L, D, N, torch.float32, False)
    dhf = torch.ones((Bt, D, N), device="cuda")
    got = plan.backward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"], torch.zeros_like(d["u"]), dhf)
    torch.cuda.synchronize()
    v = P.host_values(g)
    prod = np.exp(np.einsum("bld,dn->bdn", v["delta"].astype(np.float64), v["A"].astype(np.float64)))
    assert _rel(got["dh0"].cpu().numpy(), prod) <= 1e-5
    assert float(got["dC"].abs().max()) == 0.0  # dC_t = sum_d dy_t h_t = 0
    plan.close()


def test_backward_argument_errors():
    """Every call below fails a check before any launch; the buffers are real and large
    enough for the stated shape, so a check that wrongly passed could not make a kernel
    touch memory it does not own."""
    Bt, L, D, N = 1, 16, 32, 16
    lib = S.lib()
    buf = [torch.zeros(Bt * L * D * N + 64, device="cuda") for _ in range(16)]
    p = [ctypes.c_void_p(t.data_ptr()) for t in buf]
    # u, delta, A, B, C, h0, dy, dh_final, du, ddelta, dA, dB, dC, dh0, workspace
    ok_args = p[:15]
    assert lib.sscan_backward(Bt, L, D, 24, S.F32, 0, *ok_args, None) == S.ERR_UNSUPPORTED   # N = 24
    assert lib.sscan_backward(Bt, L, D, N, S.F32, 1 << 5, *ok_args, None) == S.ERR_INVALID   # bad flag
    q = ctypes.c_void_p(buf[0].data_ptr() + 4)
    assert lib.sscan_backward(Bt, L, D, N, S.F32, 0, q, *ok_args[1:], None) == S.ERR_ALIGN
    bad = list(ok_args)
    bad[8] = p[0]                                                                        # du over u
    assert lib.sscan_backward(Bt, L, D, N, S.F32, 0, *bad, None) == S.ERR_INVALID
    # gated: a bias without its gradient output, a gate without dz
    g = p[:6] + [p[15], None] + p[6:14] + [None, None, p[14], None]
    assert lib.sscan_backward_gated(Bt, L, D, N, S.F32, 0, *g) == S.ERR_INVALID
    g = p[:6] + [None, p[15]] + p[6:14] + [None, None, p[14], None]
    assert lib.sscan_backward_gated(Bt, L, D, N, S.F32, 0, *g) == S.ERR_INVALID
