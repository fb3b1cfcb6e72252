"""The C-ABI library builds, loads and exports every entry point include/sscan.h declares.

These run without a GPU: no compute call is made.  Argument checks that the ABI
promises to perform before touching the device are exercised here too.
"""
import ctypes
import os
import re

import pytest

from selective_state_space_32_b200 import build as B
from selective_state_space_32_b200 import sscan as S

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "sscan.h")


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"SSCAN_API\s+[\w\s\*]+?\b(sscan_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    B.build()
    return S.lib()


def test_header_declares_the_binding_symbols():
    assert sorted(declared_symbols()) == sorted(S.SYMBOLS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.sscan_version() >= 100
    for code in range(7):
        assert S.status_string(code)
    assert S.status_string(S.ERR_ALIGN) == "pointer not 16-byte aligned"


@pytest.mark.parametrize("args,want", [
    ((0, 16, 64, 16, S.F32, 0), S.ERR_INVALID),        # B = 0
    ((1, -1, 64, 16, S.F32, 0), S.ERR_INVALID),        # L < 0
    ((1, 16, 0, 16, S.F32, 0), S.ERR_INVALID),         # D = 0
    ((1, 16, 64, 16, 7, 0), S.ERR_INVALID),            # unknown dtype
    ((1, 16, 64, 16, S.F32, 1 << 5), S.ERR_INVALID),   # unknown flag
    ((1, 16, 64, 24, S.F32, 0), S.ERR_UNSUPPORTED),    # N not in {16, 32, 64}
    ((1, 16, 64, 128, S.BF16, 1), S.ERR_UNSUPPORTED),
])
def test_plan_create_rejects_bad_sizes_without_a_device(lib, args, want):
    h = ctypes.c_void_p(123)
    assert lib.sscan_plan_create(ctypes.byref(h), *args) == want
    assert not h.value


def test_null_plan_is_rejected(lib):
    assert lib.sscan_forward(None, *([None] * 10)) == S.ERR_INVALID
    assert lib.sscan_get_status(None, None) == S.ERR_INVALID
    lib.sscan_plan_destroy(None)


def declared_param_counts():
    """{function: number of parameters} from the header's SSCAN_API declarations."""
    with open(HEADER) as f:
        text = f.read()
    out = {}
    for m in re.finditer(r"SSCAN_API\s+[\w\s\*]+?\b(sscan_\w+)\s*\(([^)]*)\)", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_argument_counts_match_the_header(lib):
    counts = declared_param_counts()
    assert set(counts) == set(S.SYMBOLS)
    for name, n in counts.items():
        assert len(getattr(lib, name).argtypes) == n, (name, n, len(getattr(lib, name).argtypes))


def test_gated_and_backward_reject_bad_arguments_without_a_device(lib):
    # every case below fails an argument check before any CUDA call; none may reach a
    # launch, so none uses a supported shape with all its pointers present and aligned
    assert lib.sscan_forward_gated(None, *([None] * 12)) == S.ERR_INVALID
    p = ctypes.c_void_p(256)  # never dereferenced: every case fails its checks first
    args16 = [p] * 15 + [None]
    assert lib.sscan_backward(1, 16, 32, 24, S.F32, 0, *args16) == S.ERR_UNSUPPORTED      # N = 24
    assert lib.sscan_backward(1, 16, 32, 128, S.F32, 0, *args16) == S.ERR_UNSUPPORTED     # N = 128
    assert lib.sscan_backward(0, 16, 32, 16, S.F32, 0, *args16) == S.ERR_INVALID          # B = 0
    assert lib.sscan_backward(1, 16, 32, 16, 7, 0, *args16) == S.ERR_INVALID              # dtype
    assert lib.sscan_backward(1, 16, 32, 16, S.F32, 1 << 5, *args16) == S.ERR_INVALID     # flag
    assert lib.sscan_backward(1, 16, 32, 16, S.F32, 0, *([p] * 6), None, *([p] * 8), None) == S.ERR_INVALID  # no dy
    assert lib.sscan_backward(1, 16, 32, 16, S.F32, 0, ctypes.c_void_p(260), *([p] * 14), None) == S.ERR_ALIGN
    # the gated backward: a gate without its gradient output, a bias without its gradient
    a = [p] * 6  # u, delta, A, B, C, h0
    assert lib.sscan_backward_gated(1, 16, 32, 16, S.F32, 0, *a, None, p, p, None, p, p, p, p, p, p, None, None,
                                    p, None) == S.ERR_INVALID
    assert lib.sscan_backward_gated(1, 16, 32, 16, S.F32, 0, *a, p, None, p, None, p, p, p, p, p, p, None, None,
                                    p, None) == S.ERR_INVALID


def test_backward_workspace_bytes(lib):
    # state checkpoints: B x channels padded to a block (4 warps x 32/(N/4) channels) x
    # ceil(L/8) chunks x N states x 4 bytes; then the per-block dB / dC partial sums:
    # (padded channels / block channels) planes x B x L x 2 N x 4 bytes; each rounded up
    # to 256 bytes
    up = lambda v: (v + 255) // 256 * 256

    def want(B, L, D, N):
        cpb = 4 * (32 // (N // 4))
        dpad = -(-D // cpb) * cpb
        return up(B * dpad * -(-L // 8) * N * 4) + up((dpad // cpb) * B * L * 2 * N * 4)
    assert lib.sscan_backward_workspace_bytes(8, 2048, 1536, 16) == 8 * 1536 * 256 * 16 * 4 + 48 * 8 * 2048 * 32 * 4
    assert lib.sscan_backward_workspace_bytes(2, 37, 70, 16) == 2 * 96 * 5 * 16 * 4 + 3 * 2 * 37 * 32 * 4
    for shape in ((2, 37, 70, 32), (2, 37, 70, 64), (3, 1, 5, 16), (1, 1000, 4096, 64)):
        assert lib.sscan_backward_workspace_bytes(*shape) == want(*shape)
    assert lib.sscan_backward_workspace_bytes(2, 37, 70, 24) == 0
    assert lib.sscan_backward_workspace_bytes(2, 0, 70, 16) == 0


def test_ssd_rejects_bad_shapes_without_a_device(lib):
    # size checks come before any CUDA call (no pointer is touched)
    assert lib.sscan_ssd_forward(1, 64, 2, 32, 128, *([None] * 10)) == S.ERR_UNSUPPORTED   # P = 32
    assert lib.sscan_ssd_forward(1, 64, 2, 64, 16, *([None] * 10)) == S.ERR_UNSUPPORTED    # N = 16
    assert lib.sscan_ssd_forward(0, 64, 2, 64, 128, *([None] * 10)) == S.ERR_INVALID       # B = 0
    assert lib.sscan_ssd_forward(1, -1, 2, 64, 128, *([None] * 10)) == S.ERR_INVALID       # L < 0
    assert lib.sscan_ssd_forward(1, 64, 2, 64, 128, *([None] * 10)) == S.ERR_INVALID       # no A
