"""Pins of the fp64 SSD oracle (Mamba-2 form), CPU only.

* it equals the already pinned recurrent oracle run with A broadcast over the
  states (scalar transition per head) and one channel per (head, p);
* with A = 0 every decay is 1 and it reduces to causal linear attention with
  Q = C, K = Bbar, V = X ("Mamba & Mamba-2 Architecture", section 3), written
  here as a double loop;
* every block of the matrix strictly below the diagonal has rank <= N (the
  1-semiseparable structure the same section names), while the full lower
  triangle has full rank.
"""
import numpy as np

from oracle import oracle as O
from oracle import ssd_oracle as S


def _problem(rng, Bt=2, L=12, H=3, P=4, N=5):
    x = rng.standard_normal((Bt, L, H, P))
    delta = rng.uniform(0.05, 0.9, (Bt, L, H))
    A = -np.exp(rng.uniform(-1.0, 1.0, H))
    B = rng.standard_normal((Bt, L, N))
    C = rng.standard_normal((Bt, L, N))
    h0 = rng.standard_normal((Bt, H, N, P)) * 0.5
    return x, delta, A, B, C, h0


def pin_recurrent(S):
    rng = np.random.default_rng(71)
    x, delta, A, B, C, h0 = _problem(rng)
    Bt, L, H, P = x.shape
    N = B.shape[2]
    y, hf = S.ssd_forward(x, delta, A, B, C, h0)
    # channel d = h * P + p: input x[..., h, p], step delta[..., h], A[d, n] = A[h] for every n
    u = x.reshape(Bt, L, H * P)
    dl = np.repeat(delta, P, axis=2)
    Afull = np.repeat(A, P)[:, None].repeat(N, axis=1)
    h0full = h0.transpose(0, 1, 3, 2).reshape(Bt, H * P, N)
    yr, hr = O.forward(u, dl, Afull, B, C, h0full, False)
    assert np.abs(y.reshape(Bt, L, H * P) - yr).max() <= 1e-12 * (1 + np.abs(yr).max())
    assert np.abs(hf.transpose(0, 1, 3, 2).reshape(Bt, H * P, N) - hr).max() <= 1e-12 * (1 + np.abs(hr).max())


def pin_linear_attention(S):
    rng = np.random.default_rng(72)
    x, delta, A, B, C, _ = _problem(rng, Bt=1, L=9, H=2)
    A[:] = 0.0
    y, _ = S.ssd_forward(x, delta, A, B, C)
    want = np.zeros_like(y)
    for h in range(x.shape[2]):
        for t in range(x.shape[1]):
            for s in range(t + 1):  # causal: keys up to the query's position
                want[0, t, h] += (C[0, t] @ B[0, s]) * delta[0, s, h] * x[0, s, h]
    assert np.abs(y - want).max() <= 1e-12 * (1 + np.abs(want).max())


def pin_semiseparable(S):
    rng = np.random.default_rng(73)
    L, N = 16, 3
    delta = rng.uniform(0.05, 0.9, L)
    B = rng.standard_normal((L, N))
    C = rng.standard_normal((L, N))
    W = S.ssd_matrix(delta, -0.7, B, C)
    assert np.array_equal(np.triu(W, 1), np.zeros_like(W))  # causal
    for j in range(1, L):
        sub = W[j:, :j]  # rows after the cut, columns before it
        assert np.linalg.matrix_rank(sub, tol=1e-10) <= N
    assert np.linalg.matrix_rank(W, tol=1e-10) == L  # nonzero diagonal: full rank overall


PINS = [pin_recurrent, pin_linear_attention, pin_semiseparable]


def test_ssd_oracle_pins():
    for pin in PINS:
        pin(S)


MUTANTS = {
    "mask_transposed": ("            M[t, s] = p\n", "            M[s, t] = p\n"),
    "decay_includes_own_step": ("            M[t, s] = p\n            p *= a[s]\n",
                                "            p *= a[s]\n            M[t, s] = p\n"),
    "no_delta_on_input": ("    return M * G * delta_bh[None, :]", "    return M * G"),
    "keys_and_queries_swapped": ("np.asarray(C_b, np.float64) @ np.asarray(B_b, np.float64).T",
                                 "np.asarray(B_b, np.float64) @ np.asarray(C_b, np.float64).T"),
    "h0_not_decayed": ("                head = np.cumprod(a)  # prod_{k=0..t} a_k",
                       "                head = np.ones_like(a)"),
    "final_state_off_by_one": ("            for s in range(L - 2, -1, -1):\n                tail[s] = tail[s + 1] * a[s + 1]",
                               "            for s in range(L - 2, -1, -1):\n                tail[s] = tail[s + 1] * a[s]"),
}


def test_ssd_mutants_are_caught():
    import os
    import types
    src_path = os.path.join(os.path.dirname(S.__file__), "ssd_oracle.py")
    with open(src_path) as f:
        source = f.read()
    for name, (old, new) in MUTANTS.items():
        assert source.count(old) == 1, f"mutation site for {name} not unique"
        mod = types.ModuleType(f"ssd_mutant_{name}")
        exec(compile(source.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
        caught = []
        for pin in PINS:
            try:
                pin(mod)
            except AssertionError:
                caught.append(pin.__name__)
        assert caught, f"no SSD pin catches mutant {name}"


def test_chunked_ssd_equals_the_quadratic_form():
    # block sizes that divide L, do not divide it, and exceed it
    rng = np.random.default_rng(74)
    x, delta, A, B, C, h0 = _problem(rng, Bt=2, L=37, H=2, P=3, N=4)
    y, hf = S.ssd_forward(x, delta, A, B, C, h0)
    for block in (1, 8, 16, 64):
        yc, hc = S.ssd_forward_chunked(x, delta, A, B, C, h0, block=block)
        assert np.abs(yc - y).max() <= 1e-12 * (1 + np.abs(y).max()), block
        assert np.abs(hc - hf).max() <= 1e-12 * (1 + np.abs(hf).max()), block
