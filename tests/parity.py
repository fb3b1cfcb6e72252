"""Shared helpers for the GPU parity tests: move generated inputs to the device,
run the CUDA path through the C ABI, and compare with the fp64 oracle.

Tolerances (fixed by the workload specification):
  * fp32 I/O: relative L2 error <= 1e-5 and |err| <= 1e-4 * (1 + |ref|) elementwise,
  * bf16 I/O: relative L2 error <= 5e-3 (inputs rounded to bf16 first and fed
    identically to both sides; the GPU keeps the state in fp32 and rounds y to bf16).
The same bounds apply to y and to the final state.
"""
import numpy as np
import torch

from oracle import oracle as O
from selective_state_space_32_b200 import sscan as S
from selective_state_space_32_b200 import workloads as W

TOL_F32_REL_L2 = 1e-5
TOL_F32_ABS = 1e-4
TOL_BF16_REL_L2 = 5e-3


def to_device(g, device="cuda"):
    """Generated arrays -> CUDA tensors in the storage dtype (bf16 bit patterns -> bfloat16)."""
    def t(x, dtype):
        if x is None:
            return None
        if dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)
    dt = g["dtype"]
    return {"u": t(g["u"], dt), "delta": t(g["delta"], dt), "A": t(g["A"], "f32"),
            "B": t(g["B"], dt), "C": t(g["C"], dt), "h0": t(g["h0"], "f32"),
            "delta_bias": t(g.get("delta_bias"), "f32"), "z": t(g.get("z"), dt)}


def host_values(g):
    """The exact fp32 values of every generated input (bf16 widened)."""
    dt = g["dtype"]
    z = g.get("z")
    return {"u": W.as_f32(g["u"], dt), "delta": W.as_f32(g["delta"], dt), "A": g["A"],
            "B": W.as_f32(g["B"], dt), "C": W.as_f32(g["C"], dt), "h0": g["h0"],
            "delta_bias": g.get("delta_bias"), "z": None if z is None else W.as_f32(z, dt)}


def run_gpu(g, zoh=False, device="cuda", softplus=False):
    d = to_device(g, device)
    y, hf = S.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"], zoh=zoh,
                      delta_bias=d["delta_bias"], delta_softplus=softplus, z=d["z"])
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), hf.cpu().numpy()


def run_oracle(g, zoh=False, softplus=False):
    v = host_values(g)
    return O.forward(v["u"], v["delta"], v["A"], v["B"], v["C"], v["h0"], zoh,
                     delta_bias=v["delta_bias"], softplus=softplus, z=v["z"])


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    return float(num / den) if den > 0 else float(num)


def check(got, ref, dtype, what=""):
    """Assert the tolerance for this I/O dtype; returns (rel_l2, max_scaled_err)."""
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    r = rel_l2(got, ref)
    scaled = np.abs(np.asarray(got, np.float64) - ref) / (1.0 + np.abs(ref))
    m = float(scaled.max()) if scaled.size else 0.0
    if dtype == "f32":
        assert r <= TOL_F32_REL_L2, f"{what}: rel L2 {r:.3e} > {TOL_F32_REL_L2}"
        assert m <= TOL_F32_ABS, f"{what}: max |err|/(1+|ref|) {m:.3e} > {TOL_F32_ABS}"
    else:
        assert r <= TOL_BF16_REL_L2, f"{what}: rel L2 {r:.3e} > {TOL_BF16_REL_L2}"
    return r, m
