"""The allocation-free entry point, sscan_forward_noalloc, against the plan-based one.

It exists for callers that cannot allocate device memory (a host whose device
memory is owned by its own pool, or a call site that cannot afford an
allocation): they pass inputs and outputs only, and the library's scratch comes
from a fixed array compiled into it.  Each case calls the new entry point twice
in a row through the C ABI and compares both results with sscan_forward's (same
tolerance as the parity tests); shapes whose workspace exceeds the fixed array
must be rejected before any launch.

This file is named so that pytest collects it last; it also passes on its own in
a fresh process (the first call performs the per-device set-up).
"""
import ctypes

import numpy as np
import pytest
import torch

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


def _noalloc(shape, dt, zoh, d, y, hf):
    Bt, L, D, N = shape
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return S.lib().sscan_forward_noalloc(
        Bt, L, D, N, S.F32 if dt == "f32" else S.BF16, S.ZOH if zoh else 0,
        p(d["u"]), p(d["delta"]), p(d["A"]), p(d["B"]), p(d["C"]), p(d["h0"]), p(y), p(hf),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


CASES = [
    # (B, L, D, N, dtype, h0, zoh, reset_frac, tune): the tune string picks the schedule
    (4, 512, 2048, 16, "f32", True, False, 0.0, None),           # chained, cuts between warps
    (1, 4096, 64, 16, "bf16", True, False, 0.32, "split=1,sms=8"),  # split mode with fix-up
    (2, 300, 96, 64, "bf16", False, True, 0.0, None),            # ZOH, N = 64
    (1, 100, 70, 16, "f32", True, False, 0.0, None),             # generic kernel (D*4 % 16 != 0)
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}_{c[8] or 'default'}"
                                            for c in CASES])
def test_noalloc_matches_plan_entry_twice(case, monkeypatch):
    Bt, L, D, N, dt, with_h0, zoh, rf, tune = case
    if tune:
        monkeypatch.setenv("SSCAN_TUNE", tune)
    g = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, rf, seed=4000 + L + D, A_jitter=0.2)
    d = P.to_device(g)
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    plan = S.Plan(Bt, L, D, N, tdt, zoh)
    y_ref, hf_ref = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    torch.cuda.synchronize()
    ref_y = y_ref.float().cpu().numpy().astype(np.float64)
    ref_h = hf_ref.cpu().numpy().astype(np.float64)
    outs = []
    for _ in range(2):
        y = torch.full((Bt, L, D), float("nan"), dtype=tdt, device="cuda")
        hf = torch.full((Bt, D, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc((Bt, L, D, N), dt, zoh, d, y, hf) == S.OK
        torch.cuda.synchronize()
        yn, hn = y.float().cpu().numpy(), hf.cpu().numpy()
        P.check(yn, ref_y, dt, "y vs sscan_forward")
        P.check(hn, ref_h, dt, "h_final vs sscan_forward")
        outs.append((yn, hn))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    plan.close()


def test_noalloc_rejects_workspace_beyond_the_fixed_array():
    # 4096 batch rows x 2048 channels (N = 64): the chained schedule needs a carry
    # slot per chain, far beyond the 32 MiB array -> rejected before any launch.
    Bt, L, D, N = 4096, 64, 2048, 64
    rc = S.lib().sscan_forward_noalloc(Bt, L, D, N, S.BF16, 0, *([ctypes.c_void_p(256)] * 5), None,
                                       ctypes.c_void_p(256), None, None)
    assert rc == S.ERR_WORKSPACE, S.status_string(rc)
