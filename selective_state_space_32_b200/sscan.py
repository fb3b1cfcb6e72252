"""Thin ctypes binding of the C ABI in ``include/sscan.h`` (libsscan.so).

Argument marshalling only: every step of the selective-scan forward runs in the
CUDA library.  PyTorch supplies device memory and the current stream.  There is
no fallback: if the library is missing or the call fails, this module raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsscan.so")

F32, BF16 = 0, 1
ZOH = 1
DELTA_SOFTPLUS = 2
OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_ALIGN, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(7)

SYMBOLS = ("sscan_plan_create", "sscan_plan_destroy", "sscan_workspace_bytes", "sscan_forward",
           "sscan_get_status", "sscan_status_string", "sscan_plan_describe", "sscan_version",
           "sscan_forward_noalloc", "sscan_noalloc_status", "sscan_forward_gated", "sscan_backward",
           "sscan_backward_workspace_bytes", "sscan_ssd_forward", "sscan_backward_gated",
           "sscan_host_workspace_bytes", "sscan_forward_host")


class SscanError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} (code {code})")
        self.code = code


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Open libsscan.so (built in-tree by ``python -m selective_state_space_32_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                                   "`python -m selective_state_space_32_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i64, ip, u32, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                    ctypes.c_uint32, ctypes.c_size_t)
            L.sscan_plan_create.argtypes = [ctypes.POINTER(vp), i64, i64, i64, i64, ip, u32]
            L.sscan_plan_create.restype = ip
            L.sscan_plan_destroy.argtypes = [vp]
            L.sscan_plan_destroy.restype = None
            L.sscan_workspace_bytes.argtypes = [vp]
            L.sscan_workspace_bytes.restype = sz
            L.sscan_forward.argtypes = [vp] * 11
            L.sscan_forward.restype = ip
            L.sscan_get_status.argtypes = [vp, vp]
            L.sscan_get_status.restype = ip
            L.sscan_status_string.argtypes = [ip]
            L.sscan_status_string.restype = ctypes.c_char_p
            L.sscan_plan_describe.argtypes = [vp, ctypes.c_char_p, sz]
            L.sscan_plan_describe.restype = ip
            L.sscan_version.argtypes = []
            L.sscan_version.restype = ip
            L.sscan_forward_noalloc.argtypes = [i64, i64, i64, i64, ip, u32] + [vp] * 9
            L.sscan_forward_noalloc.restype = ip
            L.sscan_noalloc_status.argtypes = [vp]
            L.sscan_noalloc_status.restype = ip
            L.sscan_forward_gated.argtypes = [vp] * 13
            L.sscan_forward_gated.restype = ip
            L.sscan_backward.argtypes = [i64, i64, i64, i64, ip, u32] + [vp] * 16
            L.sscan_backward.restype = ip
            L.sscan_backward_workspace_bytes.argtypes = [i64, i64, i64, i64]
            L.sscan_backward_workspace_bytes.restype = sz
            L.sscan_ssd_forward.argtypes = [i64, i64, i64, i64, i64] + [vp] * 10
            L.sscan_ssd_forward.restype = ip
            L.sscan_backward_gated.argtypes = [i64, i64, i64, i64, ip, u32] + [vp] * 20
            L.sscan_backward_gated.restype = ip
            L.sscan_host_workspace_bytes.argtypes = [vp]
            L.sscan_host_workspace_bytes.restype = sz
            L.sscan_forward_host.argtypes = [vp] * 13
            L.sscan_forward_host.restype = ip
            _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().sscan_status_string(int(code)).decode()


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return F32
    if dt == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {dt} (float32 or bfloat16)")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class Plan:
    """A sscan_plan for one (B, L, D, N, dtype, zoh, delta_softplus) shape on the current device."""

    def __init__(self, B: int, L: int, D: int, N: int, dtype: torch.dtype = torch.float32,
                 zoh: bool = False, delta_softplus: bool = False):
        self.shape = (int(B), int(L), int(D), int(N))
        self.dtype = dtype
        self.zoh = bool(zoh)
        self.delta_softplus = bool(delta_softplus)
        h = ctypes.c_void_p()
        rc = lib().sscan_plan_create(ctypes.byref(h), *self.shape, _dtype_code(dtype),
                                     (ZOH if zoh else 0) | (DELTA_SOFTPLUS if delta_softplus else 0))
        if rc != OK:
            raise SscanError(rc, "sscan_plan_create")
        self._h = h
        self.workspace_bytes = int(lib().sscan_workspace_bytes(h))

    def close(self):
        if getattr(self, "_h", None):
            lib().sscan_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def describe(self) -> str:
        buf = ctypes.create_string_buffer(512)
        lib().sscan_plan_describe(self._h, buf, 512)
        return buf.value.decode()

    def new_workspace(self, device=None) -> Optional[torch.Tensor]:
        if self.workspace_bytes == 0:
            return None
        return torch.empty(self.workspace_bytes, dtype=torch.uint8, device=device or "cuda")

    def forward(self, u, delta, A, B, C, h0=None, y=None, h_final=None, workspace=None,
                want_final: bool = True, stream=None, delta_bias=None,
                z=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
        """Enqueue the forward on ``stream`` (default: torch's current stream).

        delta_bias ([D] float32) and z ([B, L, D], plan dtype) select the fused
        prologue / epilogue (``sscan_forward_gated``)."""
        Bt, L, D, N = self.shape
        if y is None:
            y = torch.empty((Bt, L, D), dtype=self.dtype, device=u.device)
        if h_final is None and want_final:
            h_final = torch.empty((Bt, D, N), dtype=torch.float32, device=u.device)
        for name, t, shape, dt in (("u", u, (Bt, L, D), self.dtype),
                                   ("delta", delta, (Bt, L, D), self.dtype),
                                   ("A", A, (D, N), torch.float32),
                                   ("B", B, (Bt, L, N), self.dtype),
                                   ("C", C, (Bt, L, N), self.dtype),
                                   ("h0", h0, (Bt, D, N), torch.float32),
                                   ("y", y, (Bt, L, D), self.dtype),
                                   ("h_final", h_final, (Bt, D, N), torch.float32),
                                   ("delta_bias", delta_bias, (D,), torch.float32),
                                   ("z", z, (Bt, L, D), self.dtype)):
            if t is None:
                continue
            if tuple(t.shape) != shape or t.dtype != dt or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name}: want contiguous CUDA {dt} {shape}, got "
                                 f"{t.dtype} {tuple(t.shape)} on {t.device}")
        if workspace is None and self.workspace_bytes:
            workspace = self.new_workspace(u.device)
        if stream is None:
            stream = torch.cuda.current_stream(u.device)
        if delta_bias is None and z is None:
            rc = lib().sscan_forward(self._h, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                     _ptr(h0), _ptr(y), _ptr(h_final), _ptr(workspace),
                                     ctypes.c_void_p(stream.cuda_stream))
            what = "sscan_forward"
        else:
            rc = lib().sscan_forward_gated(self._h, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                           _ptr(h0), _ptr(delta_bias), _ptr(z), _ptr(y), _ptr(h_final),
                                           _ptr(workspace), ctypes.c_void_p(stream.cuda_stream))
            what = "sscan_forward_gated"
        if rc != OK:
            raise SscanError(rc, what)
        return y, h_final

    def host_workspace_bytes(self) -> int:
        n = int(lib().sscan_host_workspace_bytes(self._h))
        if n == 0:
            raise SscanError(ERR_INVALID, "sscan_host_workspace_bytes")
        return n

    def forward_host(self, u, delta, A, B, C, h0, y, h_final, delta_bias=None, z=None, stream=None,
                     workspace=None):
        """Enqueue ``sscan_forward_host`` on ``stream``: every tensor a contiguous CPU
        tensor (pinned for overlapped copies), the device workspace allocated here
        unless given.  Returns without waiting; synchronise ``stream`` before
        reading y and h_final."""
        Bt, L, D, N = self.shape
        for name, t, shape, dt in (("u", u, (Bt, L, D), self.dtype),
                                   ("delta", delta, (Bt, L, D), self.dtype),
                                   ("A", A, (D, N), torch.float32),
                                   ("B", B, (Bt, L, N), self.dtype),
                                   ("C", C, (Bt, L, N), self.dtype),
                                   ("h0", h0, (Bt, D, N), torch.float32),
                                   ("y", y, (Bt, L, D), self.dtype),
                                   ("h_final", h_final, (Bt, D, N), torch.float32),
                                   ("delta_bias", delta_bias, (D,), torch.float32),
                                   ("z", z, (Bt, L, D), self.dtype)):
            if t is None:
                continue
            if tuple(t.shape) != shape or t.dtype != dt or t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name}: want contiguous host {dt} {shape}, got "
                                 f"{t.dtype} {tuple(t.shape)} on {t.device}")
        if stream is None:
            stream = torch.cuda.current_stream()
        if workspace is None:
            workspace = torch.empty(self.host_workspace_bytes(), dtype=torch.uint8, device=stream.device)
        rc = lib().sscan_forward_host(self._h, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0),
                                      _ptr(delta_bias), _ptr(z), _ptr(y), _ptr(h_final), _ptr(workspace),
                                      ctypes.c_void_p(stream.cuda_stream))
        if rc != OK:
            raise SscanError(rc, "sscan_forward_host")
        workspace.record_stream(stream)
        return y, h_final

    def backward(self, u, delta, A, B, C, h0, dy, dh_final=None, want_dh0: bool = True, stream=None,
                 delta_bias=None, z=None) -> dict:
        """Gradients of this plan's forward: returns a dict with du, ddelta (plan dtype), dA,
        dB, dC and dh0 (fp32) given dy (and optionally dh_final); with delta_bias and z
        (the fused layer, ``sscan_backward_gated``) also ddelta_bias (fp32) and dz."""
        Bt, L, D, N = self.shape
        dev = u.device
        out = {"du": torch.empty((Bt, L, D), dtype=self.dtype, device=dev),
               "ddelta": torch.empty((Bt, L, D), dtype=self.dtype, device=dev),
               "dA": torch.empty((D, N), dtype=torch.float32, device=dev),
               "dB": torch.empty((Bt, L, N), dtype=torch.float32, device=dev),
               "dC": torch.empty((Bt, L, N), dtype=torch.float32, device=dev),
               "dh0": torch.empty((Bt, D, N), dtype=torch.float32, device=dev) if want_dh0 else None,
               "ddelta_bias": torch.empty((D,), dtype=torch.float32, device=dev) if delta_bias is not None else None,
               "dz": torch.empty((Bt, L, D), dtype=self.dtype, device=dev) if z is not None else None}
        wsb = int(lib().sscan_backward_workspace_bytes(Bt, L, D, N))
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev) if wsb else None
        if stream is None:
            stream = torch.cuda.current_stream(dev)
        flags = (ZOH if self.zoh else 0) | (DELTA_SOFTPLUS if self.delta_softplus else 0)
        rc = lib().sscan_backward_gated(Bt, L, D, N, _dtype_code(self.dtype), flags,
                                        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0),
                                        _ptr(delta_bias), _ptr(z), _ptr(dy), _ptr(dh_final), _ptr(out["du"]),
                                        _ptr(out["ddelta"]), _ptr(out["dA"]), _ptr(out["dB"]), _ptr(out["dC"]),
                                        _ptr(out["dh0"]), _ptr(out["ddelta_bias"]), _ptr(out["dz"]), _ptr(ws),
                                        ctypes.c_void_p(stream.cuda_stream))
        if rc != OK:
            raise SscanError(rc, "sscan_backward_gated")
        return out

    def status(self, stream=None) -> int:
        """Synchronise ``stream`` and read (and clear) the plan's device status word."""
        if stream is None:
            stream = torch.cuda.current_stream()
        return int(lib().sscan_get_status(self._h, ctypes.c_void_p(stream.cuda_stream)))


_plans: dict = {}


def get_plan(B, L, D, N, dtype=torch.float32, zoh=False, delta_softplus=False) -> Plan:
    key = (int(B), int(L), int(D), int(N), dtype, bool(zoh), bool(delta_softplus),
           torch.cuda.current_device())
    p = _plans.get(key)
    if p is None:
        p = _plans[key] = Plan(B, L, D, N, dtype, zoh, delta_softplus)
    return p


def forward(u, delta, A, B, C, h0=None, zoh: bool = False, want_final: bool = True,
            delta_bias=None, delta_softplus: bool = False, z=None):
    """Selective-scan forward on CUDA tensors: returns (y [B,L,D], h_final [B,D,N] or None).

    u, delta: [B, L, D] float32 or bfloat16; A: [D, N] float32; B, C: [B, L, N]
    (dtype of u); h0: [B, D, N] float32 or None.  Fused prologue / epilogue:
    delta_bias [D] float32 and delta_softplus (delta <- softplus(delta + bias)),
    z [B, L, D] (dtype of u; y <- y * silu(z)).
    """
    Bt, L, D = u.shape
    N = A.shape[1]
    return get_plan(Bt, L, D, N, u.dtype, zoh, delta_softplus).forward(
        u, delta, A, B, C, h0, want_final=want_final, delta_bias=delta_bias, z=z)


def forward_host(u, delta, A, B, C, h0=None, zoh: bool = False, device="cuda", out=None,
                 delta_bias=None, delta_softplus: bool = False, z=None, stream=None):
    """Forward on host (CPU) tensors through ``sscan_forward_host``: the library
    copies the inputs to the device piece by piece, scans, and copies y and
    h_final back, the copies of neighbouring pieces overlapping the scan.
    Page-locked (pinned) host tensors let the copies run asynchronously;
    ``out`` = (y_host, h_final_host) reuses output buffers; delta_bias,
    delta_softplus and z select the fused prologue / epilogue.  Waits for the
    stream before returning.  Returns (y_host, h_final_host)."""
    dev = torch.device(device)
    Bt, L, D = u.shape
    N = A.shape[1]
    plan = get_plan(Bt, L, D, N, u.dtype, zoh, delta_softplus)
    if out is None:
        pin = u.is_pinned()
        out = (torch.empty((Bt, L, D), dtype=u.dtype, pin_memory=pin),
               torch.empty((Bt, D, N), dtype=torch.float32, pin_memory=pin))
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    plan.forward_host(u, delta, A, B, C, h0, out[0], out[1], delta_bias=delta_bias, z=z, stream=stream)
    stream.synchronize()
    return out


def ssd_forward(x, delta, A, B, C, h0=None, y=None, h_final=None, want_final: bool = True,
                status=None, stream=None):
    """Mamba-2 SSD forward (``sscan_ssd_forward``) on CUDA tensors.

    x: [B, L, H, P] bfloat16; delta: [B, L, H] float32; A: [H] float32; B, C:
    [B, L, N] bfloat16; h0: [B, H, N, P] float32 or None; status: a CUDA int32
    tensor of one element the kernel ORs error bits into, or None.
    Returns (y [B, L, H, P] bfloat16, h_final [B, H, N, P] float32 or None)."""
    Bt, L, H, P = x.shape
    N = B.shape[-1]
    dev = x.device
    if y is None:
        y = torch.empty((Bt, L, H, P), dtype=torch.bfloat16, device=dev)
    if h_final is None and want_final:
        h_final = torch.empty((Bt, H, N, P), dtype=torch.float32, device=dev)
    for name, t, shape, dt in (("x", x, (Bt, L, H, P), torch.bfloat16), ("delta", delta, (Bt, L, H), torch.float32),
                               ("A", A, (H,), torch.float32), ("B", B, (Bt, L, N), torch.bfloat16),
                               ("C", C, (Bt, L, N), torch.bfloat16), ("h0", h0, (Bt, H, N, P), torch.float32),
                               ("y", y, (Bt, L, H, P), torch.bfloat16),
                               ("h_final", h_final, (Bt, H, N, P), torch.float32),
                               ("status", status, (1,), torch.int32)):
        if t is None:
            continue
        if tuple(t.shape) != shape or t.dtype != dt or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name}: want contiguous CUDA {dt} {shape}, got {t.dtype} {tuple(t.shape)} on {t.device}")
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    rc = lib().sscan_ssd_forward(Bt, L, H, P, N, _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(h0),
                                 _ptr(y), _ptr(h_final), _ptr(status), ctypes.c_void_p(stream.cuda_stream))
    if rc != OK:
        raise SscanError(rc, "sscan_ssd_forward")
    return y, h_final
