"""Parity of the CUDA backward pass with the fp64 oracle's backward (B200).

The oracle's backward is pinned by finite differences of the forward oracle
(tests/test_oracle_backward.py).  Cases cover Euler and ZOH (with some A = 0,
the limit branch), fp32 and bf16 I/O, a ragged channel count (D not a multiple
of the 128-channel block) and ragged sequence (L not a multiple of the 8-token
recompute chunk), with and without h0 and dh_final.  dA, dB, dC are fp32 sums
over many terms accumulated with atomics; the tolerances are those of the
forward (fp32: relative L2 1e-5; bf16 inputs: 5e-3).
"""
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


CASES = [
    # (B, L, D, N, dtype, h0, dhf, zoh, zero_a)
    (2, 37, 70, 16, "f32", True, True, False, False),     # ragged D and L
    (2, 64, 128, 16, "f32", False, False, False, False),
    (3, 45, 200, 16, "f32", True, True, True, True),       # ZOH with A = 0 entries
    (2, 512, 256, 16, "f32", True, True, False, False),    # longer sequence
    (2, 100, 96, 16, "bf16", True, True, False, False),
    (1, 80, 64, 16, "bf16", True, False, True, False),
    (1, 1, 32, 16, "f32", True, True, False, False),       # a single token
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}L{c[1]}D{c[2]}{c[4]}{'_zoh' if c[7] else ''}"
                                              f"{'_a0' if c[8] else ''}{'_h0' if c[5] else ''}{'_dhf' if c[6] else ''}"
                                              for c in CASES])
def test_backward_matches_oracle(case):
    Bt, L, D, N, dt, with_h0, with_dhf, zoh, zero_a = case
    g = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, seed=8000 + L + D, A_jitter=0.3)
    if zero_a:
        g["A"][::7, 3] = 0.0
    rng = np.random.default_rng(L + D)
    dy32 = rng.standard_normal((Bt, L, D)).astype(np.float32)
    dy = dy32 if dt == "f32" else W.f32_to_bf16_bits(dy32)
    dhf = rng.standard_normal((Bt, D, N)).astype(np.float32) if with_dhf else None
    d = P.to_device(g)
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    dy_d = P.to_device({**g, "u": dy})["u"]
    dhf_d = None if dhf is None else torch.from_numpy(dhf).cuda()
    plan = S.Plan(Bt, L, D, N, tdt, zoh)
    got = plan.backward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"], dy_d, dhf_d)
    torch.cuda.synchronize()
    v = P.host_values(g)
    ref = O.backward(v["u"], v["delta"], v["A"], v["B"], v["C"], v["h0"], zoh, W.as_f32(dy, dt), dhf)
    tol = 1e-5 if dt == "f32" else 5e-3
    for k in ("du", "ddelta", "dA", "dB", "dC", "dh0"):
        r = _rel(got[k].float().cpu().numpy(), ref[k])
        assert np.all(np.isfinite(got[k].float().cpu().numpy())), k
        assert r <= tol, f"{k}: rel L2 {r:.3e} > {tol}"
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
    import ctypes
    Bt, L, D = 1, 16, 32
    z = torch.zeros(16, device="cuda")
    p = ctypes.c_void_p(z.data_ptr())
    # N = 32 and the fused softplus flag are not supported by the backward
    assert S.lib().sscan_backward(Bt, L, D, 32, S.F32, 0, *([p] * 15), None) == S.ERR_UNSUPPORTED
    assert S.lib().sscan_backward(Bt, L, D, 16, S.F32, S.DELTA_SOFTPLUS, *([p] * 15), None) == S.ERR_UNSUPPORTED
    # a bad flag bit and a misaligned pointer
    assert S.lib().sscan_backward(Bt, L, D, 16, S.F32, 1 << 5, *([p] * 15), None) == S.ERR_INVALID
    q = ctypes.c_void_p(z.data_ptr() + 4)
    assert S.lib().sscan_backward(Bt, L, D, 16, S.F32, 0, q, *([p] * 14), None) == S.ERR_ALIGN
