"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases compare every element and span several blocks plus ragged tails;
the full-size workloads run the exact launch the benchmark times and compare a
seeded sample of (b, d) rows, each recomputed by the oracle row by row (rows
are independent, so a sampled row is an exact reference).
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


SMALL = [
    # (B, L, D, N, dtype, h0, zoh, A_jitter)
    (1, 256, 64, 16, "f32", False, False, 0.0),     # the tiny workload's shape
    (2, 257, 130, 16, "f32", True, False, 0.3),     # ragged L and D, 3 blocks
    (3, 1, 7, 16, "f32", True, True, 0.3),          # one token, D below a warp
    (1, 255, 65, 32, "f32", True, False, 0.3),
    (2, 129, 33, 64, "f32", True, True, 0.3),
    (2, 300, 96, 16, "bf16", True, False, 0.0),
    (1, 200, 40, 64, "bf16", False, True, 0.0),
    (2, 64, 200, 32, "bf16", True, True, 0.5),
    (1, 1000, 64, 16, "f32", True, True, 0.0),      # long-ish horizon, exact ZOH in fp32
    # short sequences (the step kernel): ragged channel counts, every N, both I/O types
    (5, 33, 50, 32, "bf16", True, True, 0.3),
    (7, 1, 300, 64, "f32", True, False, 0.3),
    (3, 63, 129, 16, "bf16", False, False, 0.0),
    (130, 1, 77, 16, "f32", True, True, 0.3),       # many rows, several blocks, ragged last block
]


@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}"
                                              f"{'_h0' if c[5] else ''}{'_zoh' if c[6] else ''}"
                                              for c in SMALL])
def test_small_cases_elementwise(case):
    Bt, L, D, N, dt, with_h0, zoh, jit = case
    g = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, 0.0, seed=1000 + L + D + N,
                   A_jitter=jit)
    y, hf = P.run_gpu(g, zoh)
    yr, hr = P.run_oracle(g, zoh)
    P.check(y, yr, dt, "y")
    P.check(hf, hr, dt, "h_final")


CHAINED = [
    # (B, L, D, N, dtype, h0, zoh, cfg, blocks, poly): the chained kernel forced onto a
    # small grid so that chains are cut between warps (head published, tail resumed).
    # cfg indexes the library's shape table (see csrc/sscan.cu).
    (2, 300, 128, 16, "f32", True, False, 3, 3, 1),     # 8 states/lane, FMA-pipe exp on
    (2, 300, 128, 16, "f32", True, False, 3, 3, 0),
    (2, 300, 136, 16, "f32", True, False, 2, 2, 0),     # 4 states/lane
    (2, 300, 136, 16, "f32", True, False, 3, 2, 0),     # D % 16 != 0: last chain's upper lanes idle
    (2, 300, 200, 16, "bf16", True, False, 0, 1, 0),    # the same with bf16 I/O, 8 warps/block
    (2, 200, 68, 32, "f32", True, True, 5, 2, 0),       # ZOH, N = 32, D % 8 != 0
    (1, 517, 64, 16, "bf16", True, False, 4, 1, 1),
    (2, 200, 64, 32, "f32", True, True, 5, 2, 0),
    (2, 100, 72, 64, "bf16", True, True, 6, 1, 0),
    (3, 64, 128, 16, "f32", False, False, 3, 2, 1),     # L of two stages
    (2, 300, 128, 16, "f32", True, False, 3, 20, 1),    # segment < L: chains cut many times
    (2, 300, 256, 16, "bf16", True, False, 0, 1, 0),    # 8 states/lane, 8 warps/block
    (2, 300, 128, 16, "bf16", True, False, 1, 1, 0),    # 4 states/lane, 12 warps/block
]


@pytest.mark.parametrize("case", CHAINED, ids=[f"cfg{c[7]}_B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}_blk{c[8]}"
                                                f"{'_zoh' if c[6] else ''}_poly{c[9]}" for c in CHAINED])
def test_chained_kernel_forced(case, monkeypatch):
    Bt, L, D, N, dt, with_h0, zoh, cfg, blocks, poly = case
    g = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, seed=2000 + L + D, A_jitter=0.3)
    monkeypatch.setenv("SSCAN_TUNE", f"cfg={cfg},sms={blocks},poly={poly}")
    plan = S.Plan(Bt, L, D, N, torch.float32 if dt == "f32" else torch.bfloat16, zoh)
    assert "kernel=chained" in plan.describe(), plan.describe()
    d = P.to_device(g)
    y, hf = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.OK
    yr, hr = P.run_oracle(g, zoh)
    P.check(y.float().cpu().numpy(), yr, dt, "y")
    P.check(hf.cpu().numpy(), hr, dt, "h_final")
    # a second call through the same plan and workspace (new launch epoch) is identical
    y2, hf2 = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.OK
    assert torch.equal(y, y2) and torch.equal(hf, hf2)
    plan.close()


TILED = [
    # (B, L, D, N, dtype, h0, zoh, tcfg, blocks): the block-tiled kernel forced onto a small
    # grid, so that block-chains are cut between blocks (every warp's state handed over).
    # tcfg indexes the library's tiled shape table (see csrc/sscan.cu).
    (2, 300, 200, 64, "bf16", True, True, 0, 3),    # 48 channels per block, D % 48 != 0
    (2, 300, 192, 64, "f32", True, False, 0, 2),    # Euler, fp32 I/O
    (1, 517, 96, 64, "bf16", False, False, 0, 1),   # one block, ragged last stage
    (2, 300, 200, 64, "bf16", True, True, 1, 3),    # 64 channels per block (16 warps)
    (2, 200, 200, 64, "f32", True, True, 1, 2),     # fp32 ZOH (the phi polynomial)
    (2, 200, 200, 32, "f32", True, True, 2, 2),     # N = 32, 96 channels per block
    (2, 300, 136, 32, "bf16", True, False, 2, 3),
    (2, 300, 96, 64, "bf16", True, True, 0, 10),    # segment < L: block-chains cut many times
    (3, 64, 48, 64, "bf16", False, True, 0, 2),     # L of four stages, one block-chain per row
]


@pytest.mark.parametrize("case", TILED, ids=[f"tcfg{c[7]}_B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}_blk{c[8]}"
                                            f"{'_zoh' if c[6] else ''}" for c in TILED])
def test_tiled_kernel_forced(case, monkeypatch):
    Bt, L, D, N, dt, with_h0, zoh, tcfg, blocks = case
    g = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, seed=2500 + L + D, A_jitter=0.3)
    monkeypatch.setenv("SSCAN_TUNE", f"tiled={tcfg},sms={blocks}")
    plan = S.Plan(Bt, L, D, N, torch.float32 if dt == "f32" else torch.bfloat16, zoh)
    assert "kernel=tiled" in plan.describe(), plan.describe()
    d = P.to_device(g)
    y, hf = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.OK
    yr, hr = P.run_oracle(g, zoh)
    P.check(y.float().cpu().numpy(), yr, dt, "y")
    P.check(hf.cpu().numpy(), hr, dt, "h_final")
    # a second call through the same plan and workspace (new launch epoch) is identical
    y2, hf2 = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.OK
    assert torch.equal(y, y2) and torch.equal(hf, hf2)
    plan.close()


@pytest.mark.parametrize("a_case", ["zero", "positive"])
def test_tiled_zoh_bf16_sign_of_A(a_case, monkeypatch):
    """The tiled kernel's bf16 ZOH coefficient: warps whose every A is <= 0 take the
    select-free form min(Abar/A - (1 + 2^-21)/A, delta), which must give delta where A = 0
    (the first form is NaN there); a warp with a positive A takes the select."""
    Bt, L, D, N = 2, 300, 96, 64
    g = W.generate(Bt, L, D, N, "bf16", 0.1, seed=2600, A_jitter=0.3)
    A = g["A"].copy()
    if a_case == "zero":
        A[:, 0] = 0.0          # every channel's first state, in every warp
        A[7, 5:9] = 0.0
    else:
        A[5, 3] = 0.05         # one growing state in the first warp of a block-chain
    g["A"] = A
    monkeypatch.setenv("SSCAN_TUNE", "tiled=0,sms=3")
    plan = S.Plan(Bt, L, D, N, torch.bfloat16, True)
    assert "kernel=tiled" in plan.describe(), plan.describe()
    d = P.to_device(g)
    y, hf = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.OK
    yr, hr = P.run_oracle(g, True)
    P.check(y.float().cpu().numpy(), yr, "bf16", "y")
    P.check(hf.cpu().numpy(), hr, "bf16", "h_final")
    plan.close()


def test_tiled_lost_carry_times_out_and_is_reported(monkeypatch):
    """The tiled kernel's failure detection: block-chain heads skip publishing their
    warps' states, the tails' bounded waits give up, the status word reports it, and the
    next call through a fresh plan is correct."""
    import time
    g = W.generate(2, 300, 96, 64, "bf16", 0.1, seed=78)
    d = P.to_device(g)
    monkeypatch.setenv("SSCAN_TUNE", "tiled=0,sms=3,nopublish=1")
    plan = S.Plan(2, 300, 96, 64, torch.bfloat16, True)
    assert "kernel=tiled" in plan.describe()
    t0 = time.time()
    plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.ERR_TIMEOUT
    assert time.time() - t0 < 60
    plan.close()
    monkeypatch.setenv("SSCAN_TUNE", "tiled=0,sms=3")
    plan = S.Plan(2, 300, 96, 64, torch.bfloat16, True)
    y, hf = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.OK
    yr, hr = P.run_oracle(g, True)
    P.check(y.float().cpu().numpy(), yr, "bf16", "y after a failed call")
    plan.close()


SPLIT = [
    # (B, L, D, N, dtype, h0, zoh, reset_frac, blocks, negate): split mode forced on a small
    # grid: pieces scanned from zero, exact carry-in by look-back, bounded fix-up of y
    (1, 4096, 64, 16, "bf16", True, False, 0.32, 8, False),   # resets: short fix-up windows
    (1, 4096, 64, 16, "bf16", True, False, 0.32, -8, False),  # same, 4 states per lane (cfg 2)
    (2, 3000, 64, 16, "bf16", True, True, 0.0, -8, False),    # 4 states per lane, ZOH, long windows
    (1, 4096, 64, 16, "f32", True, False, 0.32, 8, False),
    (2, 3000, 64, 16, "f32", True, False, 0.0, 8, False),     # slow decay: long windows
    (1, 2050, 128, 16, "f32", True, True, 0.0, 6, False),     # exact ZOH, ragged pieces
    (1, 1500, 64, 16, "f32", True, False, 0.32, 4, True),     # some delta < 0: no early exit
    (2, 700, 72, 64, "bf16", True, True, 0.32, 4, False),     # N = 64 (32 warps > 18 chains)
    (1, 3000, 68, 16, "f32", True, False, 0.32, 8, False),    # D % 8 != 0: idle upper lanes
]


@pytest.mark.parametrize("case", SPLIT, ids=[f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}_r{c[7]}_blk{c[8]}"
                                              f"{'_zoh' if c[6] else ''}{'_neg' if c[9] else ''}"
                                              for c in SPLIT])
def test_split_mode_forced(case, monkeypatch):
    Bt, L, D, N, dt, with_h0, zoh, rf, blocks, negate = case
    g = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, rf, seed=3000 + L + D,
                   A_jitter=0.2)
    if negate:  # a few negative steps (outside the softplus range) disable the early exit
        v = W.as_f32(g["delta"], dt).copy()
        v[:, 100:103, :] *= -0.5
        g["delta"] = v if dt == "f32" else W.f32_to_bf16_bits(v)
    # negative blocks: force the 4-states-per-lane shape (cfg 2) on |blocks| blocks
    monkeypatch.setenv("SSCAN_TUNE", f"split=1,sms={abs(blocks)}" + (",cfg=2" if blocks < 0 else ""))
    plan = S.Plan(Bt, L, D, N, torch.float32 if dt == "f32" else torch.bfloat16, zoh)
    desc = plan.describe()
    assert "kernel=chained" in desc and "split=1" in desc, desc
    d = P.to_device(g)
    y, hf = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.OK
    yr, hr = P.run_oracle(g, zoh)
    P.check(y.float().cpu().numpy(), yr, dt, "y")
    P.check(hf.cpu().numpy(), hr, dt, "h_final")
    plan.close()


def test_lost_carry_times_out_and_is_reported(monkeypatch):
    """Failure detection without a GPU fault: the warps that run a chain's head are told
    not to publish its state, so the warps running the tails wait on a flag nothing sets.
    Their bounded wait gives up (about a second), the kernel finishes, and the plan's
    status word reports SSCAN_ERR_TIMEOUT; the next call starts clean."""
    import time
    g = W.generate(2, 300, 128, 16, "f32", 0.1, seed=77)
    d = P.to_device(g)
    monkeypatch.setenv("SSCAN_TUNE", "cfg=3,sms=3,nopublish=1")
    plan = S.Plan(2, 300, 128, 16, torch.float32)
    assert "kernel=chained" in plan.describe() and "split=0" in plan.describe()
    t0 = time.time()
    plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.ERR_TIMEOUT
    assert time.time() - t0 < 60
    plan.close()
    monkeypatch.setenv("SSCAN_TUNE", "cfg=3,sms=3")
    plan = S.Plan(2, 300, 128, 16, torch.float32)
    y, hf = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    assert plan.status() == S.OK
    yr, hr = P.run_oracle(g)
    P.check(y.cpu().numpy(), yr, "f32", "y after a failed call")
    plan.close()


def test_default_schedules():
    """The full-size N = 16 workloads get the chained kernel (the 2048-channel long sequence
    split), the N = 64 bf16 one the block-tiled kernel."""
    for name, want in [("mamba130m_f32", "kernel=chained"), ("mamba1p4b_bf16", "kernel=chained"),
                       ("zoh_n64_bf16", "kernel=tiled"), ("longseq_bf16", "kernel=chained")]:
        w = W.WORKLOADS[name]
        plan = S.Plan(w.B, w.L, w.D, w.N, torch.float32 if w.dtype == "f32" else torch.bfloat16,
                      w.zoh)
        split = "split=1" if name == "longseq_bf16" else "split=0"
        assert want in plan.describe() and split in plan.describe(), (name, plan.describe())
        plan.close()


def test_tiny_workload_full():
    w = W.WORKLOADS["tiny_f32"]
    g = W.make_inputs(w)
    y, hf = P.run_gpu(g, w.zoh)
    yr, hr = P.run_oracle(g, w.zoh)
    P.check(y, yr, "f32", "y")
    P.check(hf, hr, "f32", "h_final")


def test_empty_sequence_keeps_h0():
    g = W.generate(2, 0, 70, 16, "f32", 0.1, seed=5)
    y, hf = P.run_gpu(g)
    assert y.shape == (2, 0, 70)
    assert np.array_equal(hf, g["h0"])


def test_split_call_resume_matches_one_call():
    g = W.generate(2, 700, 96, 16, "f32", 0.1, seed=6, A_jitter=0.2)
    d = P.to_device(g)
    y, hf = S.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"])
    c = 333
    y1, h1 = S.forward(d["u"][:, :c].contiguous(), d["delta"][:, :c].contiguous(), d["A"],
                       d["B"][:, :c].contiguous(), d["C"][:, :c].contiguous(), d["h0"])
    y2, h2 = S.forward(d["u"][:, c:].contiguous(), d["delta"][:, c:].contiguous(), d["A"],
                       d["B"][:, c:].contiguous(), d["C"][:, c:].contiguous(), h1)
    torch.cuda.synchronize()
    yr, hr = P.run_oracle(g)
    P.check(torch.cat([y1, y2], 1).cpu().numpy(), yr, "f32", "y split")
    P.check(h2.cpu().numpy(), hr, "f32", "h_final split")
    # the schedule does not depend on where the sequence was cut
    assert torch.allclose(torch.cat([y1, y2], 1), y, rtol=1e-5, atol=1e-6)


HOST = [
    # (B, L, D, N, dtype, h0, zoh, fused): sscan_forward_host, pieces of ceil(L/8) rounded up to 64
    # tokens, or two pieces of batch rows (ceil(B/2) rows, the last one fewer) when L < 512 and B >= 2
    (6, 300, 256, 16, "bf16", True, False, False),   # 5 pieces of 64 + a last piece of 44
    (3, 1000, 96, 32, "f32", True, True, False),     # 8 pieces of 128, the last one 104
    (2, 2048, 64, 16, "f32", False, False, True),    # 8 equal pieces; softplus(delta + bias), silu(z) gate
    (4, 700, 40, 64, "bf16", True, True, True),
    (5, 1, 300, 16, "f32", True, False, False),      # one token: pieces of 3 and 2 batch rows
    (2, 50, 33, 16, "f32", False, True, False),      # short: two pieces of one row
    (11, 100, 64, 16, "bf16", True, True, True),     # short: pieces of 6 and 5 rows; fused
    (256, 1, 2048, 16, "f32", True, False, False),   # the decode step's shape: two pieces of 128 rows
    (4, 512, 2048, 64, "bf16", True, True, False),   # 8 pieces of 64 tokens, each on the block-tiled kernel
]


@pytest.mark.parametrize("case", HOST, ids=[f"B{c[0]}L{c[1]}D{c[2]}N{c[3]}{c[4]}{'_h0' if c[5] else ''}"
                                             f"{'_zoh' if c[6] else ''}{'_fused' if c[7] else ''}" for c in HOST])
def test_forward_host_matches_oracle(case):
    """The host-buffer entry point (pinned host inputs and outputs, pieces along L with
    the state carried on the device) against the oracle, every element."""
    Bt, L, D, N, dt, with_h0, zoh, fused = case
    g = W.generate(Bt, L, D, N, dt, 0.1 if with_h0 else 0.0, seed=9000 + L + D + N, A_jitter=0.3,
                   fused=fused)
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in P.to_device(g).items()}
    y_h, hf_h = S.forward_host(host["u"], host["delta"], host["A"], host["B"], host["C"], host["h0"],
                               zoh=zoh, delta_bias=host["delta_bias"], delta_softplus=fused, z=host["z"])
    assert not y_h.is_cuda and y_h.dtype == host["u"].dtype
    yr, hr = P.run_oracle(g, zoh, softplus=fused)
    P.check(y_h.float().numpy(), yr, dt, "y host")
    P.check(hf_h.numpy(), hr, dt, "h_final host")
    plan = S.get_plan(Bt, L, D, N, host["u"].dtype, zoh, fused)
    assert plan.status() == S.OK


def test_forward_host_empty_and_no_final():
    """L = 0 returns h0 (or zeros) as h_final; h_final may be skipped; the same plan
    runs again with other buffers and gives the same result."""
    Bt, D, N = 3, 48, 16
    h0 = torch.randn(Bt, D, N).pin_memory()
    plan = S.Plan(Bt, 0, D, N, torch.float32)
    A = -torch.rand(D, N).pin_memory()
    e = torch.empty(Bt, 0, D).pin_memory()
    en = torch.empty(Bt, 0, N).pin_memory()
    hf = torch.full((Bt, D, N), 7.0).pin_memory()
    plan.forward_host(e, e, A, en, en, h0, e, hf)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(hf, h0)
    plan.forward_host(e, e, A, en, en, None, e, hf)
    torch.cuda.current_stream().synchronize()
    assert float(hf.abs().max()) == 0.0
    plan.close()
    g = W.generate(2, 333, 64, 16, "f32", 0.1, seed=21)
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in P.to_device(g).items()}
    plan = S.Plan(2, 333, 64, 16, torch.float32)
    y1 = torch.empty(2, 333, 64).pin_memory()
    y2 = torch.empty(2, 333, 64).pin_memory()
    plan.forward_host(host["u"], host["delta"], host["A"], host["B"], host["C"], host["h0"], y1, None)
    plan.forward_host(host["u"], host["delta"], host["A"], host["B"], host["C"], host["h0"], y2, None)
    torch.cuda.current_stream().synchronize()
    yr, _ = P.run_oracle(g)
    P.check(y1.numpy(), yr, "f32", "y host, no h_final")
    assert torch.equal(y1, y2)
    plan.close()


def test_forward_host_argument_errors():
    """Checks made before anything is queued: every buffer is real and of the stated size."""
    Bt, L, D, N = 2, 100, 32, 16
    lib = S.lib()
    plan = S.Plan(Bt, L, D, N, torch.float32)
    n = int(lib.sscan_host_workspace_bytes(plan._h))
    assert n > 0
    ws = torch.empty(n + 512, dtype=torch.uint8, device="cuda")
    bld = [torch.zeros(Bt, L, D).pin_memory() for _ in range(3)]
    bln = [torch.zeros(Bt, L, N).pin_memory() for _ in range(2)]
    A = torch.zeros(D, N).pin_memory()
    hf = torch.zeros(Bt, D, N).pin_memory()
    S_ = torch.cuda.current_stream().cuda_stream
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    args = lambda u, y, w: [plan._h, p(u), p(bld[1]), p(A), p(bln[0]), p(bln[1]), None, None, None, p(y), p(hf),
                            w, ctypes.c_void_p(S_)]
    assert lib.sscan_forward_host(*args(bld[0], bld[0], p(ws))) == S.ERR_INVALID        # y over u
    assert lib.sscan_forward_host(*args(bld[0], bld[2], None)) == S.ERR_WORKSPACE         # no workspace
    mis = ctypes.c_void_p(ws.data_ptr() + 16)
    assert lib.sscan_forward_host(*args(bld[0], bld[2], mis)) == S.ERR_WORKSPACE          # not 256-aligned
    a = args(bld[0], bld[2], p(ws))
    a[3] = None
    assert lib.sscan_forward_host(*a) == S.ERR_INVALID                                     # no A
    plan.close()


@pytest.mark.parametrize("dt,zoh", [("f32", False), ("bf16", True)])
def test_decode_steps_match_one_forward(dt, zoh):
    """Single-token decode: the state is carried in place (h_final aliases h0), one
    token per call; the tokens' outputs and the final state equal one forward pass."""
    Bt, L, D, N = 4, 12, 256, 16
    g = W.generate(Bt, L, D, N, dt, 0.1, seed=11, A_jitter=0.2)
    d = P.to_device(g)
    y_full, h_full = S.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], d["h0"], zoh=zoh)
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    plan = S.get_plan(Bt, 1, D, N, tdt, zoh)
    assert "kernel=decode" in plan.describe()
    state = d["h0"].clone()
    ys = []
    for t in range(L):
        yt, _ = plan.forward(d["u"][:, t:t + 1].contiguous(), d["delta"][:, t:t + 1].contiguous(),
                             d["A"], d["B"][:, t:t + 1].contiguous(), d["C"][:, t:t + 1].contiguous(),
                             h0=state, h_final=state)
        ys.append(yt)
    torch.cuda.synchronize()
    yr, hr = P.run_oracle(g, zoh)
    P.check(torch.cat(ys, 1).float().cpu().numpy(), yr, dt, "decoded y")
    P.check(state.cpu().numpy(), hr, dt, "decoded state")
    assert torch.allclose(torch.cat(ys, 1).float(), y_full.float(), rtol=2e-2 if dt == "bf16" else 1e-5,
                          atol=1e-2 if dt == "bf16" else 1e-5)


DECODE = [
    # (B, D, N, dtype, zoh, fused, in_place): one token with a state (the decode kernel when D % 8 == 0)
    (4, 256, 16, "f32", False, False, True),
    (3, 200, 16, "bf16", True, False, False),     # ragged last tile (128 + 72 channels)
    (600, 1024, 16, "f32", False, False, True),   # 4800 tiles: every block's stage ring wraps
    (5, 136, 32, "f32", True, False, True),       # N = 32: 64-channel tiles, ragged
    (7, 72, 64, "bf16", False, True, True),       # N = 64: 32-channel tiles; softplus(delta + bias), gate
    (9, 520, 16, "f32", True, True, False),
    (2, 100, 16, "f32", False, False, True),      # D % 8 != 0: the step kernel
]


@pytest.mark.parametrize("case", DECODE, ids=[f"B{c[0]}D{c[1]}N{c[2]}{c[3]}{'_zoh' if c[4] else ''}"
                                               f"{'_fused' if c[5] else ''}{'_inplace' if c[6] else ''}"
                                               for c in DECODE])
def test_decode_kernel_matches_oracle(case):
    Bt, D, N, dt, zoh, fused, in_place = case
    g = W.generate(Bt, 1, D, N, dt, 0.5, seed=9500 + Bt + D + N, A_jitter=0.3, fused=fused)
    d = P.to_device(g)
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    plan = S.Plan(Bt, 1, D, N, tdt, zoh, delta_softplus=fused)
    assert ("kernel=decode" if D % 8 == 0 else "kernel=step") in plan.describe()
    h = d["h0"].clone()
    hf = h if in_place else torch.empty_like(h)
    y, _ = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], h0=h, h_final=hf,
                        delta_bias=d["delta_bias"], z=d["z"])
    torch.cuda.synchronize()
    assert plan.status() == S.OK
    yr, hr = P.run_oracle(g, zoh, softplus=fused)
    P.check(y.float().cpu().numpy(), yr, dt, "y")
    P.check(hf.cpu().numpy(), hr, dt, "h_final")
    if not in_place:
        assert torch.equal(h, d["h0"])  # the input state is not written
    plan.close()


def test_h_final_may_alias_h0():
    g = W.generate(1, 100, 64, 16, "f32", 0.1, seed=7)
    d = P.to_device(g)
    plan = S.get_plan(1, 100, 64, 16, torch.float32)
    h = d["h0"].clone()
    y, hf = plan.forward(d["u"], d["delta"], d["A"], d["B"], d["C"], h0=h, h_final=h)
    torch.cuda.synchronize()
    yr, hr = P.run_oracle(g)
    P.check(y.cpu().numpy(), yr, "f32", "y")
    P.check(h.cpu().numpy(), hr, "f32", "h_final in place")


def test_argument_errors_are_reported_before_launch():
    g = W.generate(1, 32, 64, 16, "f32", 0.0, seed=8)
    d = P.to_device(g)
    plan = S.get_plan(1, 32, 64, 16, torch.float32)
    lib = S.lib()
    import ctypes
    p = lambda t, off=0: ctypes.c_void_p(t.data_ptr() + off)
    y = torch.empty(1, 32, 64, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # misaligned u
    assert lib.sscan_forward(plan._h, p(d["u"], 4), p(d["delta"]), p(d["A"]), p(d["B"]),
                             p(d["C"]), None, p(y), None, None, s) == S.ERR_ALIGN
    # y overlapping an input
    assert lib.sscan_forward(plan._h, p(d["u"]), p(d["delta"]), p(d["A"]), p(d["B"]),
                             p(d["C"]), None, p(d["u"]), None, None, s) == S.ERR_INVALID
    # missing B
    assert lib.sscan_forward(plan._h, p(d["u"]), p(d["delta"]), p(d["A"]), None,
                             p(d["C"]), None, p(y), None, None, s) == S.ERR_INVALID
    assert plan.status() == S.OK


# ------------------------------------------------------------- full sizes --

def _sample_rows(w, k, seed):
    rng = np.random.default_rng(seed)
    rows = {(0, 0), (w.B - 1, w.D - 1), (0, w.D - 1), (w.B - 1, 0)}
    while len(rows) < k:
        rows.add((int(rng.integers(w.B)), int(rng.integers(w.D))))
    return sorted(rows)


@pytest.mark.parametrize("name,k", [("mamba130m_f32", 256), ("mamba1p4b_bf16", 128),
                                    ("longseq_bf16", 48), ("zoh_n64_bf16", 192),
                                    ("decode_b256_f32", 2048)])
def test_full_workload_sampled_rows(name, k):
    w = W.WORKLOADS[name]
    g = W.make_inputs(w)
    y, hf = P.run_gpu(g, w.zoh)
    rows = _sample_rows(w, k, w.index)
    v = P.host_values(g)
    yr, hr = O.forward_rows(rows, v["u"], v["delta"], v["A"], v["B"], v["C"], v["h0"], w.zoh)
    rb = np.array([r[0] for r in rows])
    rd = np.array([r[1] for r in rows])
    P.check(y[rb, :, rd], yr, w.dtype, f"{name} y rows")
    P.check(hf[rb, rd], hr, w.dtype, f"{name} h_final rows")
    # whole-output properties that hold at any size
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(hf))
