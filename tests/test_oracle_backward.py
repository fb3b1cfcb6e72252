"""Pins of the fp64 oracle's backward pass (CPU only).

The backward is pinned to something other than itself: central finite
differences of the forward oracle (an independent, already pinned routine) for
every input, Euler and ZOH, with and without an initial state and a final-state
gradient, including the A = 0 limit of ZOH; a closed form for delta = 0; and
invariance under the thread count.  Planted mistakes in a copy of the backward
source must each be caught.
"""
import os

import numpy as np
import pytest

from oracle import oracle as O

SRC = os.path.join(os.path.dirname(O.__file__), "sscan_oracle.c")


def _problem(rng, Bt=2, L=6, D=3, N=4, zero_a=False):
    u = rng.standard_normal((Bt, L, D))
    delta = rng.uniform(0.05, 0.8, (Bt, L, D))
    A = -np.exp(rng.uniform(-1.0, 1.0, (D, N)))
    if zero_a:
        A[0, 1] = 0.0
        A[2, 3] = 0.0
    B = rng.standard_normal((Bt, L, N))
    C = rng.standard_normal((Bt, L, N))
    h0 = rng.standard_normal((Bt, D, N)) * 0.5
    dy = rng.standard_normal((Bt, L, D))
    dhf = rng.standard_normal((Bt, D, N))
    return u, delta, A, B, C, h0, dy, dhf


def _loss(args, zoh, dy, dhf, fwd):
    y, hf = fwd(*args, zoh)
    return float(np.sum(y * dy) + (0.0 if dhf is None else np.sum(hf * dhf)))


def _fd_check(zoh, zero_a, with_dhf, fwd, bwd, seed):
    rng = np.random.default_rng(seed)
    u, delta, A, B, C, h0, dy, dhf = _problem(rng, zero_a=zero_a)
    dhf = dhf if with_dhf else None
    g = bwd(u, delta, A, B, C, h0, zoh, dy, dhf)
    args = [u, delta, A, B, C, h0]
    names = ["du", "ddelta", "dA", "dB", "dC", "dh0"]
    eps = 1e-6
    for i, name in enumerate(names):
        x = args[i]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            ap = list(args); ap[i] = xp
            am = list(args); am[i] = xm
            num[idx] = (_loss(ap, zoh, dy, dhf, fwd) - _loss(am, zoh, dy, dhf, fwd)) / (2 * eps)
        err = np.abs(g[name] - num).max()
        assert err <= 1e-6 * (1 + np.abs(num).max()), (name, zoh, zero_a, err)


def _fwd(u, delta, A, B, C, h0, zoh):
    return O.forward(u, delta, A, B, C, h0, zoh)


def _bwd(u, delta, A, B, C, h0, zoh, dy, dhf):
    return O.backward(u, delta, A, B, C, h0, zoh, dy, dhf)


@pytest.mark.parametrize("zoh,zero_a,with_dhf", [(False, False, True), (True, False, True),
                                                 (True, True, False), (False, False, False)])
def test_backward_matches_finite_differences(zoh, zero_a, with_dhf):
    _fd_check(zoh, zero_a, with_dhf, _fwd, _bwd, seed=41 + 2 * zoh + zero_a)


def test_backward_delta_zero_closed_form():
    # delta = 0: Abar = 1 and no input, so h_t = h0, y_t = C_t . h0; then
    # du = 0, dA = 0, dB = 0 (Euler), dC_t = sum_d dy_t h0, dh0 = sum_t C_t dy_t + dh_final
    rng = np.random.default_rng(47)
    u, delta, A, B, C, h0, dy, dhf = _problem(rng)
    delta[:] = 0.0
    g = O.backward(u, delta, A, B, C, h0, False, dy, dhf)
    assert np.array_equal(g["du"], np.zeros_like(u))
    assert np.array_equal(g["dA"], np.zeros_like(A))
    assert np.array_equal(g["dB"], np.zeros_like(B))
    assert np.allclose(g["dC"], np.einsum("btd,bdn->btn", dy, h0), rtol=1e-13, atol=1e-13)
    assert np.allclose(g["dh0"], np.einsum("btn,btd->bdn", C, dy) + dhf, rtol=1e-13, atol=1e-13)


def test_backward_thread_count_invariance():
    rng = np.random.default_rng(48)
    u, delta, A, B, C, h0, dy, dhf = _problem(rng, Bt=5, L=20, D=4, N=6)
    g1 = O.backward(u, delta, A, B, C, h0, True, dy, dhf, nthreads=1)
    g3 = O.backward(u, delta, A, B, C, h0, True, dy, dhf, nthreads=3)
    for k in g1:
        assert np.array_equal(g1[k], g3[k]), k


BWD_MUTANTS = {
    "carry_without_abar": ("g[n] *= abar;                                       /* now a_t g_t: carried to t-1 */",
                           "/* dropped */"),
    "readout_grad_uses_prev_state": ("j->dC[(b * L + t) * N + n] += dyt * ht;",
                                     "j->dC[(b * L + t) * N + n] += dyt * hprev;"),
    "ddelta_drops_decay_term": ("ddl += g[n] * (hprev * an * abar + x * dbeta_ddl);",
                                "ddl += g[n] * (x * dbeta_ddl);"),
    "zoh_dbeta_ddelta_euler": ("beta = em1 / an * Bn; dbeta_ddl = abar * Bn;",
                               "beta = em1 / an * Bn; dbeta_ddl = Bn;"),
    "zoh_dA_sign": ("dbeta_dA = Bn * (delta * abar * an - em1) / (an * an);",
                    "dbeta_dA = Bn * (em1 - delta * abar * an) / (an * an);"),
    "zoh_a0_limit": ("dbeta_dA = 0.5 * delta * delta * Bn;", "dbeta_dA = 0.0;"),
    "dB_drops_u": ("j->dB[(b * L + t) * N + n] += g[n] * x * dbeta_dB;",
                   "j->dB[(b * L + t) * N + n] += g[n] * dbeta_dB;"),
    "dh0_uncarried": ("j->dh0[(b * D + d) * N + n] = g[n];               /* a_0 g_0 */",
                      "j->dh0[(b * D + d) * N + n] = g[n] / exp(dl[0] * a_row[n]);"),
    "dhfinal_ignored": ("g[n] = j->dhf ? j->dhf[(b * D + d) * N + n] : 0.0;", "g[n] = 0.0;"),
}


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_mutant_is_caught(name, tmp_path):
    with open(SRC) as f:
        source = f.read()
    old, new = BWD_MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not unique"
    src = tmp_path / f"{name}.c"
    src.write_text(source.replace(old, new))
    lib = O.load_library(O.compile_source(str(src), str(tmp_path / f"lib{name}.so")))

    def bwd(u, delta, A, B, C, h0, zoh, dy, dhf):
        return O.backward(u, delta, A, B, C, h0, zoh, dy, dhf, lib=lib)

    caught = False
    for zoh, zero_a, with_dhf in [(False, False, True), (True, True, True)]:
        try:
            _fd_check(zoh, zero_a, with_dhf, _fwd, bwd, seed=60)
        except AssertionError:
            caught = True
    assert caught, f"no pin catches backward mutant {name}"


def test_fused_backward_matches_finite_differences():
    # delta' = softplus(delta_raw + bias), y = scan(delta') * silu(z): every gradient,
    # including the raw step, the bias and the gate, against central differences of
    # the (pinned) fused forward oracle
    rng = np.random.default_rng(49)
    u, delta, A, B, C, h0, dy, dhf = _problem(rng)
    raw = rng.normal(-1.0, 1.0, delta.shape)
    bias = rng.normal(0.0, 0.5, delta.shape[2])
    z = rng.normal(0.0, 1.5, u.shape)
    for zoh in (False, True):
        g = O.backward_fused(u, raw, A, B, C, h0, zoh, dy, dhf, delta_bias=bias, softplus=True, z=z)

        def loss(uu=u, rr=raw, AA=A, BB=B, CC=C, hh=h0, bb=bias, zz=z):
            y, hf = O.forward(uu, rr, AA, BB, CC, hh, zoh, delta_bias=bb, softplus=True, z=zz)
            return float(np.sum(y * dy) + np.sum(hf * dhf))

        eps = 1e-6
        for name, key, x in (("du", "uu", u), ("ddelta", "rr", raw), ("dA", "AA", A), ("dB", "BB", B),
                             ("dC", "CC", C), ("dh0", "hh", h0), ("ddelta_bias", "bb", bias), ("dz", "zz", z)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp = x.copy(); xp[idx] += eps
                xm = x.copy(); xm[idx] -= eps
                num[idx] = (loss(**{key: xp}) - loss(**{key: xm})) / (2 * eps)
            err = np.abs(g[name] - num).max()
            assert err <= 1e-6 * (1 + np.abs(num).max()), (name, zoh, err)
