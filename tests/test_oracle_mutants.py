"""The pins must catch plausible mistakes in the oracle.

Each mutant is a copy of the oracle's C source with one planted mistake (a
dropped term, a wrong sign, a swapped operand, a wrong index, the readout taken
before the update, ...).  Every mutant is compiled with gcc into a temporary
directory and must fail at least one pin of ``test_oracle_pins``.  Nothing here
touches the GPU; the oracle's own source file is never modified.
"""
import os

import pytest

from oracle import oracle as O
from tests import test_oracle_pins as P

SRC = os.path.join(os.path.dirname(P.O.__file__), "sscan_oracle.c")

MUTANTS = {
    "abar_sign": ("const double abar = exp(delta * a[n]);",
                  "const double abar = exp(-delta * a[n]);"),
    "abar_drop_delta": ("const double abar = exp(delta * a[n]);",
                        "const double abar = exp(a[n]);"),
    "drop_input": ("h[n] = abar * h[n] + bbar * x;", "h[n] = abar * h[n] + bbar;"),
    "euler_drop_delta": ("bbar = delta * Bt[n];\n", "bbar = Bt[n];\n"),
    "zoh_times_a": ("expm1(delta * a[n]) / a[n]", "expm1(delta * a[n]) * a[n]"),
    "zoh_as_euler": ("if (zoh)\n", "if (0)\n"),
    "readout_uses_B": ("acc += Ct[n] * h[n];", "acc += Bt[n] * h[n];"),
    "readout_before_update": (
        "            h[n] = abar * h[n] + bbar * x;\n            acc += Ct[n] * h[n];",
        "            acc += Ct[n] * h[n];\n            h[n] = abar * h[n] + bbar * x;"),
    "ignore_h0": ("h[n] = h0 ? h0[n] : 0.0;", "h[n] = 0.0;"),
    "A_row_index": ("j->A + d * N,", "j->A + d,"),
    "B_batch_index": ("j->A + d * N,\n                 j->Bm + b * L * N,",
                      "j->A + d * N,\n                 j->Bm,"),
    "u_stride": ("j->u + b * L * D + d, D,", "j->u + b * L * D + d, 1,"),
    "B_time_index": ("const double *Bt = Bm + t * N;", "const double *Bt = Bm + (t > 0 ? t - 1 : 0) * N;"),
    "hfinal_stale": ("hfin[n] = h[n];", "hfin[n] = h0 ? h0[n] : 0.0;"),
    # fused prologue / epilogue
    "softplus_as_exp": ("return (s > 0.0 ? s : 0.0) + log1p(exp(-fabs(s)));", "return exp(s);"),
    "softplus_sign": ("log1p(exp(-fabs(s)))", "log1p(exp(fabs(s)))"),
    "bias_dropped": ("double delta = dl[t * sd] + bias;", "double delta = dl[t * sd];"),
    "bias_after_softplus": ("double delta = dl[t * sd] + bias;\n        if (sp)\n            delta = softplus(delta);",
                            "double delta = dl[t * sd];\n        if (sp)\n            delta = softplus(delta);\n"
                            "        delta += bias;"),
    "bias_batch_index": ("j->bias ? j->bias[d] : 0.0", "j->bias ? j->bias[b] : 0.0"),
    "gate_sigmoid_only": ("return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    "gate_additive": ("acc * silu(z[t * sz])", "acc + silu(z[t * sz])"),
    "gate_stride": ("j->z ? j->z + b * L * D + d : NULL, D,", "j->z ? j->z + b * L * D + d : NULL, 1,"),
}


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not unique"
    mutated = source.replace(old, new)
    src = tmp_path / f"{name}.c"
    src.write_text(mutated)
    lib = O.load_library(O.compile_source(str(src), str(tmp_path / f"lib{name}.so")))

    def fwd(u, delta, A, B, C, h0, zoh, **kw):
        return O.forward(u, delta, A, B, C, h0, zoh, lib=lib, **kw)

    caught = []
    for pin in P.PINS:
        try:
            pin(fwd)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
