"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Every pin takes the forward function under test (the oracle's own build, or a
deliberately broken copy in ``test_oracle_mutants``) so that the same checks
both pin the oracle and prove that they would catch a plausible mistake.

Pins (each cites the passage it rests on):
  * printed values: the numpy listing and the worked example of
    "Mamba & Mamba-2 Architecture" (sections "Code", "Worked Example"), and the
    memory-horizon table of "tm_ssm_selective" ("Reading delta as a memory horizon"),
  * brute force: the unrolled sum / semiseparable matrix
    y_t = sum_{j<=t} C_t (prod_{k=j+1..t} Abar_k) Bbar_j u_j  (+ the h0 term)
    ("tm_ssm_selective", "The convolution dies"; "Selective State-Space Models
    (Mamba) and Hardware-Aware Scans", Exercises, item 3),
  * LTI closed form: constant delta, B, C reduce the scan to a convolution with
    kernel K_k = C Abar^k Bbar ("Selective State-Space Models ...", section 1;
    "tm_ssm_selective", "What time-invariance forbids"),
  * GRU identity for the exact ZOH term ("tm_ssm_selective", "Delta is a gate, exactly"),
  * delta -> 0 keeps the state and ignores the input; a large delta resets it
    ("Mamba & Mamba-2 Architecture", section 1; "tm_ssm_selective", horizon table),
  * ZOH fixed point h = -B u / A (derived from the ZOH formula),
  * Abar in (0, 1) bounds the state by |h0| + sum |Bbar u|,
  * split-call resume: scan(L1) then scan(L2, h0 = h_final) equals scan(L1 + L2)
    ("tm_ssm_selective", "What it costs at inference ...": carry the block's state forward).
"""
import math
import os

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_kv(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            out[k] = [float(x) for x in v]
    return out


def _one_channel(x, delta, a, b, c, h0=None, zoh=False, fwd=O.forward):
    """Run a single (batch 1, channel 1) sequence with per-token b, c (N = len(a))."""
    x = np.asarray(x, dtype=np.float64)
    L = x.shape[0]
    a = np.atleast_1d(np.asarray(a, dtype=np.float64))
    N = a.shape[0]
    b = np.broadcast_to(np.asarray(b, dtype=np.float64), (L, N))
    c = np.broadcast_to(np.asarray(c, dtype=np.float64), (L, N))
    hh = None if h0 is None else np.asarray(h0, dtype=np.float64).reshape(1, 1, N)
    y, hf = fwd(x.reshape(1, L, 1), np.asarray(delta, dtype=np.float64).reshape(1, L, 1),
                a.reshape(1, N), b.reshape(1, L, N), c.reshape(1, L, N), hh, zoh)
    return y.reshape(L), hf.reshape(N)


def _rand_problem(rng, Bt, L, D, N, with_h0=True, dmax=1.5):
    u = rng.standard_normal((Bt, L, D))
    delta = rng.uniform(0.01, dmax, (Bt, L, D))
    A = -np.exp(rng.uniform(-1.0, 1.5, (D, N)))
    B = rng.standard_normal((Bt, L, N))
    C = rng.standard_normal((Bt, L, N))
    h0 = rng.standard_normal((Bt, D, N)) if with_h0 else None
    return u, delta, A, B, C, h0


def _brute_force(u, delta, A, B, C, h0, zoh):
    """Unrolled sum: materialise, per (b, d), the L x L lower-triangular matrix
    M[t, j] = sum_n C[t,n] * prod_{k=j+1..t} exp(delta_k A_n) * Bbar_j[n], plus the
    h0 term sum_n C[t,n] prod_{k<=t} exp(delta_k A_n) h0[n].  Products are taken
    explicitly, token by token (no recurrence is run)."""
    Bt, L, D = u.shape
    N = A.shape[1]
    y = np.zeros((Bt, L, D))
    hf = np.zeros((Bt, D, N))
    for b in range(Bt):
        for d in range(D):
            dl = delta[b, :, d]
            abar = np.exp(dl[:, None] * A[d][None, :])               # [L, N]
            if zoh:
                bbar = (np.exp(dl[:, None] * A[d][None, :]) - 1.0) / A[d][None, :] * B[b]
            else:
                bbar = dl[:, None] * B[b]                             # [L, N]
            M = np.zeros((L, L))
            for t in range(L):
                for j in range(t + 1):
                    prod = np.prod(abar[j + 1:t + 1], axis=0)          # empty -> ones
                    M[t, j] = np.sum(C[b, t] * prod * bbar[j])
            y[b, :, d] = M @ u[b, :, d]
            if h0 is not None:
                for t in range(L):
                    y[b, t, d] += np.sum(C[b, t] * np.prod(abar[:t + 1], axis=0) * h0[b, d])
            # final state: the same unrolled sum with the readout C removed
            hT = np.zeros(N) if h0 is None else np.prod(abar, axis=0) * h0[b, d]
            for j in range(L):
                hT = hT + np.prod(abar[j + 1:], axis=0) * bbar[j] * u[b, j, d]
            hf[b, d] = hT
    return y, hf


# ---------------------------------------------------------------- pins --------

def pin_p2_listing(fwd):
    g = _read_kv("p2_numpy_listing.txt")
    y, _ = _one_channel(g["x"], g["delta"], g["a"], g["b"], g["c"], fwd=fwd)
    k = int(g["pinned_count"][0])
    tol = 0.5 * 10 ** (-int(g["printed_decimals"][0])) + 1e-12
    for t in range(k):
        assert abs(y[t] - g["printed_y"][t]) <= tol, (t, y[t])
    # third token by hand: h1 = 1.5*5, h2 = e^-0.001 h1 + 0.001*100, h3 = e^-1 h2 + 1*1
    h1 = 1.5 * 5.0
    h2 = math.exp(-0.001) * h1 + 0.001 * 100.0
    h3 = math.exp(-1.0) * h2 + 1.0 * 1.0
    assert abs(y[2] - h3) <= 1e-13 * abs(h3)


def pin_p2_worked_example(fwd):
    g = _read_kv("p2_worked_example.txt")
    tol = 0.5 * 10 ** (-int(g["printed_decimals"][0])) + 1e-12
    x = g["x"]
    # contribution of the distractor alone: run with x_1 = 0
    y, _ = _one_channel([0.0, x[1]], g["delta"], g["a"], g["b"], g["c"], fwd=fwd)
    assert abs(y[1] - g["printed_x2_contribution"][0]) <= tol
    # memory of h_1 retained through the distractor step: run with x_2 = 0
    y, _ = _one_channel([x[0], 0.0], g["delta"], g["a"], g["b"], g["c"], fwd=fwd)
    assert abs(y[0] - 20.0) <= 1e-12               # h_1 = delta_1 * x_1
    assert abs(y[1] - g["printed_h1_retained"][0]) <= tol
    # both together: linear superposition
    y, _ = _one_channel(x, g["delta"], g["a"], g["b"], g["c"], fwd=fwd)
    assert abs(y[1] - (math.exp(-0.01) * 20.0 + 0.01 * 20.0)) <= 1e-12


def pin_p5_horizon_table(fwd):
    rows = []
    with open(os.path.join(GOLDEN, "p5_horizon_table.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([float(v) for v in line.split()])
    for dl, printed, dec, pct in rows:
        # one step from h0 = 1 with no input (B = 0), A = -1, readout C = 1
        y, hf = _one_channel([0.0], [dl], [-1.0], [0.0], [1.0], h0=[1.0], fwd=fwd)
        assert abs(y[0] - printed) <= 0.5 * 10 ** (-int(dec)) + 1e-12, (dl, y[0])
        assert abs(100.0 * hf[0] - pct) <= 0.5 * (1 if pct >= 1 else 0.1) + 1e-9
    for zoh in (False, True):
        y, _ = _one_channel([0.0], [5.0], [-1.0], [0.0], [1.0], h0=[1.0], zoh=zoh, fwd=fwd)
        assert abs(y[0] - math.exp(-5.0)) <= 1e-15


def pin_brute_force(fwd):
    rng = np.random.default_rng(11)
    for zoh in (False, True):
        for with_h0 in (False, True):
            u, delta, A, B, C, h0 = _rand_problem(rng, 2, 9, 3, 4, with_h0)
            y, hf = fwd(u, delta, A, B, C, h0, zoh)
            yb, hb = _brute_force(u, delta, A, B, C, h0, zoh)
            scale = 1.0 + np.abs(yb).max()
            assert np.abs(y - yb).max() <= 1e-12 * scale, (zoh, with_h0)
            assert np.abs(hf - hb).max() <= 1e-12 * (1.0 + np.abs(hb).max())


def pin_lti_convolution(fwd):
    rng = np.random.default_rng(12)
    L, N = 40, 5
    for zoh in (False, True):
        a = -np.exp(rng.uniform(-2.0, 1.0, N))
        dl = 0.3
        Bc = rng.standard_normal(N)
        Cc = rng.standard_normal(N)
        h0 = rng.standard_normal(N)
        u = rng.standard_normal(L)
        abar = np.exp(dl * a)
        bbar = (abar - 1.0) / a * Bc if zoh else dl * Bc
        K = np.array([np.sum(Cc * abar ** k * bbar) for k in range(L)])
        y_conv = np.convolve(u, K)[:L]
        y_conv = y_conv + np.array([np.sum(Cc * abar ** (t + 1) * h0) for t in range(L)])
        y, _ = _one_channel(u, np.full(L, dl), a, Bc, Cc, h0=h0, zoh=zoh, fwd=fwd)
        assert np.abs(y - y_conv).max() <= 1e-12 * (1 + np.abs(y_conv).max()), zoh


def pin_gru_identity(fwd):
    rng = np.random.default_rng(13)
    L = 30
    s = rng.normal(0.0, 2.0, L)
    u = rng.standard_normal(L)
    delta = np.log1p(np.exp(s))                     # softplus(s)
    g = 1.0 / (1.0 + np.exp(-s))                    # sigmoid(s)
    h = 0.7
    want = []
    for t in range(L):
        h = (1.0 - g[t]) * h + g[t] * u[t]
        want.append(h)
    y, hf = _one_channel(u, delta, [-1.0], [1.0], [1.0], h0=[0.7], zoh=True, fwd=fwd)
    assert np.abs(y - np.array(want)).max() <= 1e-13
    assert abs(hf[0] - want[-1]) <= 1e-13


def pin_delta_zero(fwd):
    rng = np.random.default_rng(14)
    for zoh in (False, True):
        u, delta, A, B, C, h0 = _rand_problem(rng, 2, 17, 3, 6)
        delta[:] = 0.0
        y, hf = fwd(u, delta, A, B, C, h0, zoh)
        assert np.array_equal(hf, h0)
        assert np.abs(y - np.einsum("btn,bdn->btd", C, h0)).max() <= 1e-13


def pin_reset(fwd):
    rng = np.random.default_rng(15)
    u, delta, A, B, C, h0 = _rand_problem(rng, 1, 12, 2, 4)
    delta[:, 6, :] = 60.0        # exp(60 A) < 1e-26 for A <= -1: the past is flushed
    A = np.minimum(A, -1.0)
    y, _ = fwd(u, delta, A, B, C, h0, False)
    want = np.einsum("tn,tn->t", C[0, 6:7], B[0, 6:7])[0] * 60.0 * u[0, 6]
    assert np.allclose(y[0, 6], want, rtol=1e-12, atol=0)
    y, _ = fwd(u, delta, A, B, C, h0, True)
    want = np.array([np.sum(C[0, 6] * (np.exp(60.0 * A[d]) - 1) / A[d] * B[0, 6]) * u[0, 6, d]
                     for d in range(2)])
    assert np.allclose(y[0, 6], want, rtol=1e-12, atol=0)


def pin_zoh_fixed_point(fwd):
    rng = np.random.default_rng(16)
    L, N = 25, 6
    a = -np.exp(rng.uniform(-1.0, 1.0, N))
    Bc = rng.standard_normal(N)
    Cc = rng.standard_normal(N)
    uc = 0.8
    h0 = -Bc * uc / a
    delta = rng.uniform(0.0, 3.0, L)
    y, hf = _one_channel(np.full(L, uc), delta, a, Bc, Cc, h0=h0, zoh=True, fwd=fwd)
    assert np.abs(hf - h0).max() <= 1e-12 * (1 + np.abs(h0).max())
    assert np.abs(y - np.sum(Cc * h0)).max() <= 1e-12 * (1 + abs(np.sum(Cc * h0)))


def pin_state_bound(fwd):
    rng = np.random.default_rng(17)
    L, N = 20, 4
    a = -np.exp(rng.uniform(-1.0, 1.0, N))
    delta = rng.uniform(0.0, 1.0, L)
    u = rng.standard_normal(L)
    Bm = rng.standard_normal((L, N))
    h0 = rng.standard_normal(N)
    bound = np.abs(h0).copy()
    for t in range(L):
        bound = bound + np.abs(delta[t] * Bm[t] * u[t])
        _, hf = _one_channel(u[:t + 1], delta[:t + 1], a, Bm[:t + 1], np.ones((t + 1, N)),
                             h0=h0, fwd=fwd)
        assert np.all(np.abs(hf) <= bound + 1e-12)


def pin_split_resume(fwd):
    rng = np.random.default_rng(18)
    for zoh in (False, True):
        u, delta, A, B, C, h0 = _rand_problem(rng, 2, 33, 3, 4)
        y, hf = fwd(u, delta, A, B, C, h0, zoh)
        y1, h1 = fwd(u[:, :13], delta[:, :13], A, B[:, :13], C[:, :13], h0, zoh)
        y2, h2 = fwd(u[:, 13:], delta[:, 13:], A, B[:, 13:], C[:, 13:], h1, zoh)
        assert np.array_equal(np.concatenate([y1, y2], axis=1), y)
        assert np.array_equal(h2, hf)


# ---- fused prologue (delta <- softplus(delta + bias)) and epilogue (y * silu(z)) ----

def _expit(x):
    from scipy.special import expit  # library logistic function
    return expit(x)


def pin_fused_softplus_gru(fwd):
    # "tm_ssm_selective", "Delta is a gate, exactly": N = 1, A = -1, B = 1 and
    # Delta = softplus(s) make the ZOH step the GRU update with g = sigmoid(s).
    # Here s reaches the scan as a raw delta s - b plus the channel bias b.
    rng = np.random.default_rng(31)
    L, bias = 40, 0.75
    s = rng.normal(0.0, 2.5, L)
    u = rng.standard_normal(L)
    g = _expit(s)
    h, want = -0.4, []
    for t in range(L):
        h = (1.0 - g[t]) * h + g[t] * u[t]
        want.append(h)
    ones = np.ones((1, L, 1))
    y, hf = fwd(u.reshape(1, L, 1), (s - bias).reshape(1, L, 1), np.array([[-1.0]]), ones, ones,
                np.array([[[-0.4]]]), True, delta_bias=np.array([bias]), softplus=True)
    assert np.abs(y[0, :, 0] - np.array(want)).max() <= 1e-13
    assert abs(hf[0, 0, 0] - want[-1]) <= 1e-13


def pin_fused_softplus_at_zero(fwd):
    # softplus(0) = log 2: with A = -1 the retention is exactly 1/2 and the Euler
    # input weight log 2.
    u = np.array([0.3, -1.2, 2.0])
    h, want = 0.8, []
    for t in range(3):
        h = 0.5 * h + math.log(2.0) * u[t]
        want.append(h)
    ones = np.ones((1, 3, 1))
    y, _ = fwd(u.reshape(1, 3, 1), np.zeros((1, 3, 1)), np.array([[-1.0]]), ones, ones,
               np.array([[[0.8]]]), False, softplus=True)
    assert np.abs(y[0, :, 0] - np.array(want)).max() <= 1e-15


def pin_fused_softplus_limits(fwd):
    # softplus(s) -> s for large s (gap e^-40 ~ 4e-18) and -> 0 for very negative s
    # (the "Delta -> 0 keeps the state" gate of "tm_ssm_selective").
    rng = np.random.default_rng(32)
    u, delta, A, B, C, h0 = _rand_problem(rng, 2, 9, 3, 4)
    big = np.full_like(delta, 40.0)
    y1, h1 = fwd(u, big, A, B, C, h0, False, softplus=True)
    y2, h2 = fwd(u, big, A, B, C, h0, False)
    assert np.abs(y1 - y2).max() <= 1e-12 * (1 + np.abs(y2).max())
    y3, h3 = fwd(u, np.full_like(delta, -60.0), A, B, C, h0, False, softplus=True)
    assert np.abs(h3 - h0).max() <= 1e-20 * (1 + np.abs(h0).max()) + 1e-24
    assert np.abs(y3 - np.einsum("btn,bdn->btd", C, h0)).max() <= 1e-15


def pin_fused_bias_per_channel(fwd):
    # the bias is one value per channel d, added to delta before softplus
    rng = np.random.default_rng(33)
    u, delta, A, B, C, h0 = _rand_problem(rng, 3, 11, 4, 5)
    bias = rng.normal(0.0, 1.0, 4)
    for sp, zoh in ((False, False), (True, False), (True, True)):
        y1, h1 = fwd(u, delta, A, B, C, h0, zoh, delta_bias=bias, softplus=sp)
        d2 = delta + bias[None, None, :]
        if sp:
            d2 = np.maximum(d2, 0.0) + np.log1p(np.exp(-np.abs(d2)))
        y2, h2 = fwd(u, d2, A, B, C, h0, zoh)
        assert np.abs(y1 - y2).max() <= 1e-13 * (1 + np.abs(y2).max())
        assert np.abs(h1 - h2).max() <= 1e-13 * (1 + np.abs(h2).max())


def pin_fused_gate(fwd):
    # "Selective State-Space Models (Mamba) and Hardware-Aware Scans", section 4:
    # the second branch gates the SSM output; y * silu(z), silu(z) = z * sigmoid(z).
    rng = np.random.default_rng(34)
    u, delta, A, B, C, h0 = _rand_problem(rng, 2, 13, 3, 4)
    z = rng.normal(0.0, 2.0, u.shape)
    for zoh in (False, True):
        y0, h0f = fwd(u, delta, A, B, C, h0, zoh)
        yg, hgf = fwd(u, delta, A, B, C, h0, zoh, z=z)
        assert np.abs(yg - y0 * z * _expit(z)).max() <= 1e-14 * (1 + np.abs(y0).max())
        assert np.array_equal(hgf, h0f)            # the gate acts on y only
        yz, _ = fwd(u, delta, A, B, C, h0, zoh, z=np.zeros_like(z))
        assert np.array_equal(yz, np.zeros_like(yz))


PINS = [pin_p2_listing, pin_p2_worked_example, pin_p5_horizon_table, pin_brute_force,
        pin_lti_convolution, pin_gru_identity, pin_delta_zero, pin_reset,
        pin_zoh_fixed_point, pin_state_bound, pin_split_resume,
        pin_fused_softplus_gru, pin_fused_softplus_at_zero, pin_fused_softplus_limits,
        pin_fused_bias_per_channel, pin_fused_gate]


def oracle_fwd(u, delta, A, B, C, h0, zoh, lib=None, **kw):
    return O.forward(u, delta, A, B, C, h0, zoh, lib=lib, **kw)


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle_fwd)


def test_thread_count_invariance():
    rng = np.random.default_rng(19)
    u, delta, A, B, C, h0 = _rand_problem(rng, 3, 50, 7, 8)
    y1, h1 = O.forward(u, delta, A, B, C, h0, False, nthreads=1)
    for nt in (2, 5, 64):
        y2, h2 = O.forward(u, delta, A, B, C, h0, False, nthreads=nt)
        assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


def test_rows_match_full():
    rng = np.random.default_rng(20)
    u, delta, A, B, C, h0 = _rand_problem(rng, 3, 21, 5, 4)
    for zoh in (False, True):
        y, hf = O.forward(u, delta, A, B, C, h0, zoh)
        rows = [(0, 0), (2, 4), (1, 2), (2, 0), (0, 4)]
        yr, hr = O.forward_rows(rows, u, delta, A, B, C, h0, zoh)
        for i, (b, d) in enumerate(rows):
            assert np.array_equal(yr[i], y[b, :, d])
            assert np.array_equal(hr[i], hf[b, d])


def test_empty_and_degenerate_shapes():
    rng = np.random.default_rng(21)
    u, delta, A, B, C, h0 = _rand_problem(rng, 2, 0, 3, 4)
    y, hf = O.forward(u, delta, A, B, C, h0, False)
    assert y.shape == (2, 0, 3) and np.array_equal(hf, h0)     # L = 0 keeps h0
    u, delta, A, B, C, h0 = _rand_problem(rng, 2, 5, 3, 1)     # N = 1
    y, hf = O.forward(u, delta, A, B, C, h0, False)
    yb, hb = _brute_force(u, delta, A, B, C, h0, False)
    assert np.abs(y - yb).max() <= 1e-12 * (1 + np.abs(yb).max())
