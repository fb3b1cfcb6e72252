"""Parity of the fused prologue / epilogue against the fp64 oracle (B200).

The kernels take delta as the raw projection and apply delta <- softplus(delta
+ delta_bias[d]) themselves ("tm_ssm_selective", section "The mechanism:
parameters as functions of the input"), and gate the output y <- y * silu(z)
("Selective State-Space Models (Mamba) and Hardware-Aware Scans", section 4).
Every schedule is covered: the chained kernel on forced shapes (chains cut
between warps, ragged last chain, bf16, ZOH, N = 32 and 64), the block-tiled
kernel (block-chains cut between blocks), the split mode,
the generic kernel, decode steps, the default schedule, and sampled rows of the
full fused workloads.  Tolerances are those of the unfused parity tests.
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


def _tdt(dt):
    return torch.float32 if dt == "f32" else torch.bfloat16


def _drop(g, bias, gate):
    g = dict(g)
    if not bias:
        g["delta_bias"] = None
    if not gate:
        g["z"] = None
    return g


def _run_plan(plan, g):
    d = P.to_device(g)
    y, hf = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"],
                         delta_bias=d["delta_bias"], z=d["z"])
    assert plan.status() == S.OK
    return y, hf, d


CHAINED = [
    # (B, L, D, N, dtype, h0, zoh, cfg, blocks, softplus, bias, gate)
    (2, 300, 128, 16, "f32", True, False, 3, 3, True, True, True),     # chains cut between warps
    (2, 300, 136, 16, "f32", True, False, 3, 2, True, True, True),     # D % 16 != 0
    (2, 300, 200, 16, "bf16", True, False, 0, 1, True, True, True),    # bf16, 8 warps/block, ragged
    (2, 300, 136, 16, "f32", True, False, 2, 2, True, True, True),     # 4 states per lane
    (2, 200, 68, 32, "f32", True, True, 5, 2, True, True, True),       # ZOH, N = 32, ragged
    (2, 100, 72, 64, "bf16", True, True, 6, 1, True, True, True),      # ZOH, N = 64
    (2, 300, 128, 16, "f32", True, False, 3, 3, True, False, False),   # softplus only
    (2, 300, 128, 16, "f32", True, False, 3, 3, False, False, True),   # gate only
    (2, 300, 128, 16, "f32", True, False, 3, 3, False, True, False),   # bias only, no softplus
    (3, 64, 128, 16, "bf16", False, False, 3, 2, True, True, True),    # L of two stages
]


@pytest.mark.parametrize("case", CHAINED, ids=[f"cfg{c[7]}_B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}_blk{c[8]}"
                                                f"{'_zoh' if c[6] else ''}_sp{int(c[9])}b{int(c[10])}g{int(c[11])}"
                                                for c in CHAINED])
def test_fused_chained_forced(case, monkeypatch):
    Bt, L, D, N, dt, with_h0, zoh, cfg, blocks, sp, bias, gate = case
    g = _drop(W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, seed=5000 + L + D, A_jitter=0.3,
                         fused=True), bias, gate)
    if not sp:  # without softplus the raw delta must itself be a valid (positive) step
        g["delta"] = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, seed=5000 + L + D,
                                A_jitter=0.3)["delta"]
        if bias:
            g["delta_bias"] = np.linspace(0.0, 0.05, D).astype(np.float32)
    monkeypatch.setenv("SSCAN_TUNE", f"cfg={cfg},sms={blocks}")
    plan = S.Plan(Bt, L, D, N, _tdt(dt), zoh, delta_softplus=sp)
    assert "kernel=chained" in plan.describe(), plan.describe()
    y, hf, d = _run_plan(plan, g)
    yr, hr = P.run_oracle(g, zoh, softplus=sp)
    P.check(y.float().cpu().numpy(), yr, dt, "y")
    P.check(hf.cpu().numpy(), hr, dt, "h_final")
    # the same plan without the fused arguments runs the unfused kernel again
    if not sp:
        y0, hf0 = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
        yr0, hr0 = P.run_oracle(_drop(g, False, False), zoh)
        P.check(y0.float().cpu().numpy(), yr0, dt, "y unfused")
        P.check(hf0.cpu().numpy(), hr0, dt, "h_final unfused")
    plan.close()


TILED = [
    # (B, L, D, N, dtype, h0, zoh, tcfg, blocks, softplus, bias, gate): the block-tiled kernel
    (2, 300, 200, 64, "bf16", True, True, 0, 3, True, True, True),     # block-chains cut, D % 48 != 0
    (2, 200, 192, 64, "f32", True, False, 1, 2, True, True, True),     # 16 warps, Euler
    (2, 200, 200, 32, "f32", True, True, 2, 2, True, False, True),     # N = 32, no bias
    (2, 300, 96, 64, "bf16", True, True, 0, 3, False, True, False),    # bias only, no softplus
]


@pytest.mark.parametrize("case", TILED, ids=[f"tcfg{c[7]}_B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}_blk{c[8]}"
                                            f"{'_zoh' if c[6] else ''}_sp{int(c[9])}b{int(c[10])}g{int(c[11])}"
                                            for c in TILED])
def test_fused_tiled_forced(case, monkeypatch):
    Bt, L, D, N, dt, with_h0, zoh, tcfg, blocks, sp, bias, gate = case
    g = _drop(W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, seed=5500 + L + D, A_jitter=0.3,
                         fused=True), bias, gate)
    if not sp:  # without softplus the raw delta must itself be a valid (positive) step
        g["delta"] = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, seed=5500 + L + D,
                                A_jitter=0.3)["delta"]
        if bias:
            g["delta_bias"] = np.linspace(0.0, 0.05, D).astype(np.float32)
    monkeypatch.setenv("SSCAN_TUNE", f"tiled={tcfg},sms={blocks}")
    plan = S.Plan(Bt, L, D, N, _tdt(dt), zoh, delta_softplus=sp)
    assert "kernel=tiled" in plan.describe(), plan.describe()
    y, hf, d = _run_plan(plan, g)
    yr, hr = P.run_oracle(g, zoh, softplus=sp)
    P.check(y.float().cpu().numpy(), yr, dt, "y")
    P.check(hf.cpu().numpy(), hr, dt, "h_final")
    if not sp:  # the same plan without the fused arguments
        y0, hf0 = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
        yr0, hr0 = P.run_oracle(_drop(g, False, False), zoh)
        P.check(y0.float().cpu().numpy(), yr0, dt, "y unfused")
        P.check(hf0.cpu().numpy(), hr0, dt, "h_final unfused")
    plan.close()


SPLIT = [
    # (B, L, D, N, dtype, zoh, blocks): split mode forced; the fix-up applies the same
    # delta transform and gates its correction
    (1, 4096, 64, 16, "bf16", False, 8),
    (1, 4096, 64, 16, "f32", False, 8),
    (2, 3000, 64, 16, "f32", True, -8),
    (1, 3000, 68, 16, "f32", False, 8),
    (2, 700, 72, 64, "bf16", True, 4),
]


@pytest.mark.parametrize("case", SPLIT, ids=[f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}_blk{c[6]}"
                                              f"{'_zoh' if c[5] else ''}" for c in SPLIT])
def test_fused_split_forced(case, monkeypatch):
    Bt, L, D, N, dt, zoh, blocks = case
    g = W.generate(Bt, L, D, N, dt, 0.1, 0.0, seed=6000 + L + D, A_jitter=0.2, fused=True)
    monkeypatch.setenv("SSCAN_TUNE", f"split=1,sms={abs(blocks)}" + (",cfg=2" if blocks < 0 else ""))
    plan = S.Plan(Bt, L, D, N, _tdt(dt), zoh, delta_softplus=True)
    desc = plan.describe()
    assert "kernel=chained" in desc and "split=1" in desc, desc
    y, hf, _ = _run_plan(plan, g)
    yr, hr = P.run_oracle(g, zoh, softplus=True)
    P.check(y.float().cpu().numpy(), yr, dt, "y")
    P.check(hf.cpu().numpy(), hr, dt, "h_final")
    plan.close()


GENERIC = [
    # (B, L, D, N, dtype, zoh, kernel): shapes the chained kernel does not take
    (2, 100, 70, 16, "f32", False, "generic"),    # D * 4 % 16 != 0
    (2, 80, 44, 32, "bf16", True, "generic"),     # ZOH, N = 32, D * 2 % 16 != 0
    (1, 70, 22, 64, "f32", True, "generic"),      # N = 64, D * 4 % 16 != 0
    (3, 37, 96, 16, "bf16", False, "step"),       # L < 64
    (2, 50, 44, 32, "bf16", True, "step"),        # ZOH, N = 32, ragged D
    (1, 45, 20, 64, "f32", True, "step"),         # N = 64
]


@pytest.mark.parametrize("case", GENERIC, ids=[f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}{'_zoh' if c[5] else ''}_{c[6]}"
                                                for c in GENERIC])
def test_fused_generic_and_step(case):
    Bt, L, D, N, dt, zoh, kernel = case
    g = W.generate(Bt, L, D, N, dt, 0.1, seed=7000 + L + D, A_jitter=0.3, fused=True)
    plan = S.Plan(Bt, L, D, N, _tdt(dt), zoh, delta_softplus=True)
    assert f"kernel={kernel}" in plan.describe(), plan.describe()
    y, hf, _ = _run_plan(plan, g)
    yr, hr = P.run_oracle(g, zoh, softplus=True)
    P.check(y.float().cpu().numpy(), yr, dt, "y")
    P.check(hf.cpu().numpy(), hr, dt, "h_final")
    plan.close()


def test_fused_decode_steps_match_full_forward():
    # one token per call, state carried in place (h_final aliases h0), gate and softplus fused
    Bt, L, D, N = 4, 12, 64, 16
    g = W.generate(Bt, L, D, N, "f32", 0.1, seed=7100, A_jitter=0.2, fused=True)
    d = P.to_device(g)
    yr, hr = P.run_oracle(g, False, softplus=True)
    state = d["h0"].clone()
    plan = S.Plan(Bt, 1, D, N, torch.float32, False, delta_softplus=True)
    ys = []
    for t in range(L):
        sl = lambda x: x[:, t:t + 1].contiguous()
        y, _ = plan.forward(sl(d["u"]), sl(d["delta"]), d["A"], sl(d["B"]), sl(d["C"]), state,
                            h_final=state, delta_bias=d["delta_bias"], z=sl(d["z"]))
        ys.append(y)
    assert plan.status() == S.OK
    P.check(torch.cat(ys, dim=1).cpu().numpy(), yr, "f32", "y (decode steps)")
    P.check(state.cpu().numpy(), hr, "f32", "state after the last step")
    plan.close()


def test_fused_default_schedule_medium():
    Bt, L, D, N = 4, 512, 2048, 16
    g = W.generate(Bt, L, D, N, "bf16", 0.1, seed=7200, A_jitter=0.2, fused=True)
    y, hf = P.run_gpu(g, False, softplus=True)
    rows = [(0, 0), (1, 777), (3, 2047), (2, 1024), (0, 1535)]
    v = P.host_values(g)
    yr, hr = O.forward_rows(rows, v["u"], v["delta"], v["A"], v["B"], v["C"], v["h0"], False,
                            delta_bias=v["delta_bias"], softplus=True, z=v["z"])
    for i, (b, dd) in enumerate(rows):
        P.check(y[b, :, dd], yr[i], "bf16", f"y row {(b, dd)}")
        P.check(hf[b, dd], hr[i], "bf16", f"h_final row {(b, dd)}")


@pytest.mark.parametrize("name", ["mamba130m_fused_f32", "mamba1p4b_fused_bf16"])
def test_fused_full_workload_sampled_rows(name):
    w = W.WORKLOADS[name]
    g = W.make_inputs(w)
    y, hf = P.run_gpu(g, w.zoh, softplus=True)
    rng = np.random.default_rng(11)
    rows = [(int(rng.integers(w.B)), int(rng.integers(w.D))) for _ in range(6)] + [(0, 0), (w.B - 1, w.D - 1)]
    v = P.host_values(g)
    yr, hr = O.forward_rows(rows, v["u"], v["delta"], v["A"], v["B"], v["C"], v["h0"], w.zoh,
                            delta_bias=v["delta_bias"], softplus=True, z=v["z"])
    for i, (b, dd) in enumerate(rows):
        P.check(y[b, :, dd], yr[i], w.dtype, f"{name} y row {(b, dd)}")
        P.check(hf[b, dd], hr[i], w.dtype, f"{name} h_final row {(b, dd)}")


def test_fused_noalloc_softplus_flag():
    # the allocation-free entry accepts SSCAN_DELTA_SOFTPLUS (no bias or gate arguments there)
    Bt, L, D, N = 2, 300, 256, 16
    g = _drop(W.generate(Bt, L, D, N, "f32", 0.1, seed=7300, A_jitter=0.2, fused=True), False, False)
    d = P.to_device(g)
    y = torch.empty((Bt, L, D), dtype=torch.float32, device="cuda")
    hf = torch.empty((Bt, D, N), dtype=torch.float32, device="cuda")
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = S.lib().sscan_forward_noalloc(Bt, L, D, N, S.F32, S.DELTA_SOFTPLUS, p(d["u"]), p(d["delta"]),
                                       p(d["A"]), p(d["B"]), p(d["C"]), p(d["h0"]), p(y), p(hf),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == S.OK, S.status_string(rc)
    torch.cuda.synchronize()
    yr, hr = P.run_oracle(g, False, softplus=True)
    P.check(y.cpu().numpy(), yr, "f32", "y")
    P.check(hf.cpu().numpy(), hr, "f32", "h_final")


def test_fused_argument_errors():
    Bt, L, D, N = 1, 64, 64, 16
    g = W.generate(Bt, L, D, N, "f32", 0.0, seed=7400, fused=True)
    d = P.to_device(g)
    plan = S.Plan(Bt, L, D, N, torch.float32, False, delta_softplus=True)
    y = torch.empty((Bt, L, D), dtype=torch.float32, device="cuda")
    args = [plan._h] + [ctypes.c_void_p(d[k].data_ptr()) for k in ("u", "delta", "A", "B", "C")] + [None]
    ws = plan.new_workspace()
    wsp = None if ws is None else ctypes.c_void_p(ws.data_ptr())
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # y overlapping the gate input is rejected
    rc = S.lib().sscan_forward_gated(*args, ctypes.c_void_p(d["delta_bias"].data_ptr()),
                                     ctypes.c_void_p(d["z"].data_ptr()), ctypes.c_void_p(d["z"].data_ptr()),
                                     None, wsp, st)
    assert rc == S.ERR_INVALID
    # a misaligned bias pointer is rejected
    rc = S.lib().sscan_forward_gated(*args, ctypes.c_void_p(d["delta_bias"].data_ptr() + 4), None,
                                     ctypes.c_void_p(y.data_ptr()), None, wsp, st)
    assert rc == S.ERR_ALIGN
    # an unknown flag bit is rejected at plan creation
    h = ctypes.c_void_p()
    assert S.lib().sscan_plan_create(ctypes.byref(h), Bt, L, D, N, S.F32, 1 << 5) == S.ERR_INVALID
    plan.close()
