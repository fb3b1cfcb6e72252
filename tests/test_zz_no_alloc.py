"""The allocation-free entry point, sscan_forward_noalloc, against the plan-based one
and against the fp64 oracle.

It exists for callers that cannot allocate device memory (a host whose device
memory is owned by its own pool, or a call site that cannot afford an
allocation): they pass inputs and outputs only, and the library's scratch comes
from a fixed array compiled into it.  Each case calls the new entry point twice
in a row through the C ABI and compares both results with sscan_forward's (same
tolerance as the parity tests) and the first with the oracle; calls of
different shapes in a row share the array and must not disturb each other; a
wait that gives up inside it is reported by sscan_noalloc_status; shapes whose
workspace exceeds the fixed array are rejected before any launch.

Every test clears SSCAN_TUNE unless it sets it, so the schedule (and with it
the workspace a shape needs) is the library's default one.  No test passes a
pointer that is not a real device buffer of the stated size.

This file is named so that pytest collects it last; it also passes on its own in
a fresh process (the first call performs the per-device set-up).
"""
import ctypes
import time

import numpy as np
import pytest
import torch

from selective_state_space_32_b200 import sscan as S
from selective_state_space_32_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20          # the library's fixed array
WORKSPACE_ROOM = SCRATCH_BYTES - 256  # status word and alignment before the workspace


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_32_b200 import build
    build.build()
    S.lib()


@pytest.fixture(autouse=True)
def _default_schedule(monkeypatch):
    monkeypatch.delenv("SSCAN_TUNE", raising=False)


def _noalloc(shape, dt, zoh, d, y, hf):
    Bt, L, D, N = shape
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return S.lib().sscan_forward_noalloc(
        Bt, L, D, N, S.F32 if dt == "f32" else S.BF16, S.ZOH if zoh else 0,
        p(d["u"]), p(d["delta"]), p(d["A"]), p(d["B"]), p(d["C"]), p(d["h0"]), p(y), p(hf),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _status():
    return S.lib().sscan_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _outputs(shape, dt):
    Bt, L, D, N = shape
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    return (torch.full((Bt, L, D), float("nan"), dtype=tdt, device="cuda"),
            torch.full((Bt, D, N), float("nan"), dtype=torch.float32, device="cuda"))


CASES = [
    # (B, L, D, N, dtype, h0, zoh, reset_frac, tune): the tune string picks the schedule
    (4, 512, 2048, 16, "f32", True, False, 0.0, None),           # chained, cuts between warps
    (1, 4096, 64, 16, "bf16", True, False, 0.32, "split=1,sms=8"),  # split mode with fix-up
    (2, 300, 96, 64, "bf16", False, True, 0.0, None),            # ZOH, N = 64
    (4, 64, 2048, 64, "bf16", True, True, 0.0, None),            # block-tiled kernel (N = 64)
    (1, 100, 70, 16, "f32", True, False, 0.0, None),             # generic kernel (D*4 % 16 != 0)
]


def _case_inputs(case):
    Bt, L, D, N, dt, with_h0, zoh, rf, _ = case
    return W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, rf, seed=4000 + L + D, A_jitter=0.2)


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}_{c[8] or 'default'}"
                                            for c in CASES])
def test_noalloc_matches_plan_entry_and_oracle_twice(case, monkeypatch):
    Bt, L, D, N, dt, with_h0, zoh, rf, tune = case
    if tune:
        monkeypatch.setenv("SSCAN_TUNE", tune)
    g = _case_inputs(case)
    d = P.to_device(g)
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    plan = S.Plan(Bt, L, D, N, tdt, zoh)
    y_ref, hf_ref = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    torch.cuda.synchronize()
    ref_y = y_ref.float().cpu().numpy().astype(np.float64)
    ref_h = hf_ref.cpu().numpy().astype(np.float64)
    yo, ho = P.run_oracle(g, zoh)
    outs = []
    for i in range(2):
        y, hf = _outputs((Bt, L, D, N), dt)
        assert _noalloc((Bt, L, D, N), dt, zoh, d, y, hf) == S.OK
        assert _status() == S.OK
        yn, hn = y.float().cpu().numpy(), hf.cpu().numpy()
        P.check(yn, ref_y, dt, "y vs sscan_forward")
        P.check(hn, ref_h, dt, "h_final vs sscan_forward")
        if i == 0:
            P.check(yn, yo, dt, "y vs oracle")
            P.check(hn, ho, dt, "h_final vs oracle")
        outs.append((yn, hn))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    plan.close()


def test_noalloc_shapes_in_a_row_share_the_array_cleanly():
    """Shape A (chained, its carry flags at one offset), then B (another layout of the
    array), then A again: stale flags of one call must not satisfy the next call's waits."""
    a = (4, 512, 2048, 16, "f32", True, False, 0.0, None)
    b = (2, 300, 96, 64, "bf16", False, True, 0.0, None)
    runs = {}
    for case in (a, b, a):
        Bt, L, D, N, dt, _, zoh, _, _ = case
        g = _case_inputs(case)
        d = P.to_device(g)
        y, hf = _outputs((Bt, L, D, N), dt)
        assert _noalloc((Bt, L, D, N), dt, zoh, d, y, hf) == S.OK
        assert _status() == S.OK
        yo, ho = P.run_oracle(g, zoh)
        P.check(y.float().cpu().numpy(), yo, dt, f"y of {case[:5]} vs oracle")
        P.check(hf.cpu().numpy(), ho, dt, f"h_final of {case[:5]} vs oracle")
        runs.setdefault(case, []).append(y.float().cpu().numpy())
    assert np.array_equal(runs[a][0], runs[a][1])


def test_noalloc_reports_a_wait_that_gave_up(monkeypatch):
    """Failure detection through the allocation-free path: the warps that run a chain's
    head do not publish its state, the tail warps' bounded wait gives up (about a
    second) and sscan_noalloc_status reports it; the next call is clean."""
    g = W.generate(2, 300, 128, 16, "f32", 0.1, seed=77)
    d = P.to_device(g)
    shape = (2, 300, 128, 16)
    monkeypatch.setenv("SSCAN_TUNE", "cfg=3,sms=3,nopublish=1")
    plan = S.Plan(*shape, torch.float32)  # the same schedule choice, to check it cuts chains
    assert "kernel=chained" in plan.describe() and "split=0" in plan.describe()
    plan.close()
    y, hf = _outputs(shape, "f32")
    t0 = time.time()
    assert _noalloc(shape, "f32", False, d, y, hf) == S.OK
    assert _status() == S.ERR_TIMEOUT
    assert time.time() - t0 < 60
    monkeypatch.setenv("SSCAN_TUNE", "cfg=3,sms=3")
    y, hf = _outputs(shape, "f32")
    assert _noalloc(shape, "f32", False, d, y, hf) == S.OK
    assert _status() == S.OK
    yo, ho = P.run_oracle(g)
    P.check(y.cpu().numpy(), yo, "f32", "y after a failed call")
    P.check(hf.cpu().numpy(), ho, "f32", "h_final after a failed call")


def test_noalloc_rejects_workspace_beyond_the_fixed_array():
    """64 batch rows x 2048 channels (N = 64, bf16): the default block-tiled schedule
    keeps a carry slot per warp of every 48-channel block-chain, over 32 MiB in all, so
    the call is rejected before any launch.  The buffers are real device buffers of the
    stated shape, so even a failed check could not make a kernel touch memory it does
    not own."""
    Bt, L, D, N = 64, 64, 2048, 64
    plan = S.Plan(Bt, L, D, N, torch.bfloat16)
    assert "kernel=tiled" in plan.describe(), plan.describe()
    assert plan.workspace_bytes > WORKSPACE_ROOM, plan.workspace_bytes
    plan.close()
    g = W.generate(Bt, L, D, N, "bf16", seed=99)
    d = P.to_device(g)
    y, hf = _outputs((Bt, L, D, N), "bf16")
    rc = _noalloc((Bt, L, D, N), "bf16", False, d, y, hf)
    assert rc == S.ERR_WORKSPACE, S.status_string(rc)
    torch.cuda.synchronize()
    assert torch.isnan(y.float()).all()  # nothing was launched
