"""ctypes binding of libqlora.so (C ABI in include/qlora.h).

Argument marshalling only: torch tensors are checked for dtype, device,
shape and contiguity, and their raw device pointers are handed to the
library together with the current CUDA stream. Every step of the QLoRA path
runs in the library's CUDA kernels; there is no CPU fallback, and loading
fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqlora.so")

BLOCK = 64
DQ_BLOCK = 256

_lib = None
_lock = threading.Lock()

_STATUS = {0: "QLORA_OK", 1: "QLORA_ERR_NULL", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGN",
           4: "QLORA_ERR_RANGE", 5: "QLORA_ERR_CUDA", 6: "QLORA_ERR_UNSUPPORTED",
           7: "QLORA_ERR_WORKSPACE", 8: "QLORA_ERR_TABLE"}

# every symbol include/qlora.h declares
EXPORTS = ("qlora_status_string", "qlora_abi_version", "qlora_nf4_levels", "qlora_dq_levels",
           "qlora_int4_levels", "qlora_fp4_levels", "qlora_dq_signed_levels", "qlora_dq_dynamic_levels",
           "qlora_workspace_bytes", "qlora_quantize_nf4", "qlora_double_quant", "qlora_dequant",
           "qlora_linear_fwd", "qlora_linear_bwd", "qlora_device_error", "qlora_set_trace_events",
           "qlora_launch_count", "qlora_linear_fwd_noalloc", "qlora_selftest_bounded_wait",
           "qlora_dequant_dt", "qlora_linear_fwd_dt", "qlora_linear_bwd_dt",
           "qlora_paged_adamw_create", "qlora_paged_adamw_destroy", "qlora_paged_adamw_init",
           "qlora_paged_adamw_step", "qlora_paged_adamw_set_reserve", "qlora_paged_adamw_placement",
           "qlora_paged_adamw_location", "qlora_paged_adamw_state_bytes", "qlora_paged_adamw_state",
           "qlora_block_workspace_bytes", "qlora_block_fwd", "qlora_block_bwd", "qlora_quantize_dq",
           "qlora_debug_fail_allocs")

BLOCK_STREAMS = 2


class LinearDesc(ctypes.Structure):
    """qlora_linear_desc: one linear of a decoder block (device pointers)."""
    _fields_ = [("packed", ctypes.c_void_p), ("q", ctypes.c_void_p), ("scale2", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("X", ctypes.c_void_p), ("A", ctypes.c_void_p),
                ("B", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("XA", ctypes.c_void_p), ("dY", ctypes.c_void_p),
                ("dX", ctypes.c_void_p), ("dA", ctypes.c_void_p), ("dB", ctypes.c_void_p)]

# qlora_dtype of the 16-bit tensors of a call
_DTYPE = {torch.bfloat16: 0, torch.float16: 1}

NOALLOC_SCRATCH_BYTES = 8 << 20


class QLoRAError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call} failed: {_STATUS.get(status, status)}")


def load(path: str | None = None):
    """Load libqlora.so (raises OSError if it is missing: no fallback)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise OSError(f"libqlora.so not found at {p}; build it with "
                          "`python -m bit_quantized_lora_blockwise_b200.build`")
        lib = ctypes.CDLL(p)
        P, I64, I32, F32, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                                ctypes.c_size_t)
        lib.qlora_status_string.argtypes = [I32]
        lib.qlora_status_string.restype = ctypes.c_char_p
        lib.qlora_abi_version.restype = I32
        for fn in ("qlora_nf4_levels", "qlora_dq_levels", "qlora_int4_levels", "qlora_fp4_levels",
                   "qlora_dq_signed_levels", "qlora_dq_dynamic_levels"):
            getattr(lib, fn).argtypes = [P]
            getattr(lib, fn).restype = None
        lib.qlora_workspace_bytes.argtypes = [I64, I64, I64, I32]
        lib.qlora_workspace_bytes.restype = SZ
        lib.qlora_quantize_nf4.argtypes = [P, I64, I64, P, P, P, P]
        lib.qlora_double_quant.argtypes = [P, I64, P, P, P, P]
        lib.qlora_quantize_dq.argtypes = [P, I64, I64, P, P, P, P, P, P, P]
        lib.qlora_quantize_dq.restype = I32
        lib.qlora_dequant.argtypes = [P, P, P, I64, I64, P, P, P, P]
        lib.qlora_linear_fwd.argtypes = [P, P, P, P, P, I64, I64, I64, P, P, P, I32, F32, P, P, P, SZ, P]
        lib.qlora_linear_fwd_noalloc.argtypes = [P, P, P, P, P, I64, I64, I64, P, P, P, I32, F32, P, P, P]
        lib.qlora_linear_fwd_noalloc.restype = I32
        lib.qlora_linear_bwd.argtypes = [P, P, P, P, P, I64, I64, I64, P, P, P, P, P, I32, F32, P, P, P,
                                         P, SZ, P]
        lib.qlora_dequant_dt.argtypes = [P, P, P, I64, I64, P, P, I32, P, P]
        lib.qlora_linear_fwd_dt.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P, I32, F32, P, P, P, SZ,
                                            P]
        lib.qlora_linear_bwd_dt.argtypes = [P, P, P, P, P, I32, I64, I64, I64, P, P, P, P, P, I32, F32, P, P,
                                            P, P, SZ, P]
        for fn in ("qlora_dequant_dt", "qlora_linear_fwd_dt", "qlora_linear_bwd_dt"):
            getattr(lib, fn).restype = I32
        PP = ctypes.POINTER(ctypes.c_void_p)
        lib.qlora_paged_adamw_create.argtypes = [I32, ctypes.POINTER(I64), ctypes.POINTER(P)]
        lib.qlora_paged_adamw_create.restype = I32
        lib.qlora_paged_adamw_destroy.argtypes = [P]
        lib.qlora_paged_adamw_destroy.restype = None
        lib.qlora_paged_adamw_init.argtypes = [P, PP, I32, P]
        lib.qlora_paged_adamw_init.restype = I32
        lib.qlora_paged_adamw_step.argtypes = [P, PP, PP, I32, I64, F32, F32, F32, F32, F32, P]
        lib.qlora_paged_adamw_step.restype = I32
        lib.qlora_paged_adamw_set_reserve.argtypes = [P, SZ]
        lib.qlora_paged_adamw_set_reserve.restype = I32
        lib.qlora_paged_adamw_placement.argtypes = [SZ, SZ, SZ, I32]
        lib.qlora_paged_adamw_placement.restype = I32
        lib.qlora_paged_adamw_location.argtypes = [P]
        lib.qlora_paged_adamw_location.restype = I32
        lib.qlora_paged_adamw_state_bytes.argtypes = [P]
        lib.qlora_paged_adamw_state_bytes.restype = SZ
        lib.qlora_paged_adamw_state.argtypes = [P, PP, PP, PP]
        lib.qlora_paged_adamw_state.restype = I32
        DP = ctypes.POINTER(LinearDesc)
        lib.qlora_block_workspace_bytes.argtypes = [I32, DP, I64, I32]
        lib.qlora_block_workspace_bytes.restype = SZ
        for fn in ("qlora_block_fwd", "qlora_block_bwd"):
            getattr(lib, fn).argtypes = [I32, DP, P, P, I32, I64, I32, F32, I32, P, SZ, P]
            getattr(lib, fn).restype = I32
        lib.qlora_device_error.argtypes = [I32]
        lib.qlora_device_error.restype = ctypes.c_uint32
        lib.qlora_set_trace_events.argtypes = [P, P]
        lib.qlora_set_trace_events.restype = None
        lib.qlora_launch_count.restype = ctypes.c_uint64
        lib.qlora_selftest_bounded_wait.argtypes = [P]
        lib.qlora_selftest_bounded_wait.restype = I32
        lib.qlora_debug_fail_allocs.argtypes = [I32, I32]
        lib.qlora_debug_fail_allocs.restype = I32
        for fn in ("qlora_quantize_nf4", "qlora_double_quant", "qlora_dequant", "qlora_linear_fwd",
                   "qlora_linear_bwd"):
            getattr(lib, fn).restype = I32
        _lib = lib
        return lib


def _check(status: int, call: str):
    if status != 0:
        raise QLoRAError(status, call)


def _ptr(t) -> ctypes.c_void_p | None:
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _req(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


class _HostTables:
    """Host float arrays for the code tables, kept alive across calls."""

    def __init__(self, nf4=None, t8=None):
        lib = load()
        if nf4 is None:
            self.nf4 = (ctypes.c_float * 16)()
            lib.qlora_nf4_levels(self.nf4)
        else:
            self.nf4 = (ctypes.c_float * 16)(*np.asarray(nf4, np.float32).tolist())
        if t8 is None:
            self.t8 = (ctypes.c_float * 256)()
            lib.qlora_dq_levels(self.t8)
        else:
            self.t8 = (ctypes.c_float * 256)(*np.asarray(t8, np.float32).tolist())


_default_tables = None


def _tables(nf4, t8) -> _HostTables:
    global _default_tables
    if nf4 is None and t8 is None:
        if _default_tables is None:
            _default_tables = _HostTables()
        return _default_tables
    return _HostTables(nf4, t8)


def nf4_levels() -> np.ndarray:
    """The library's default 16 NF4 levels (host computation)."""
    out = (ctypes.c_float * 16)()
    load().qlora_nf4_levels(out)
    return np.frombuffer(out, dtype=np.float32).copy()


def dq_levels() -> np.ndarray:
    out = (ctypes.c_float * 256)()
    load().qlora_dq_levels(out)
    return np.frombuffer(out, dtype=np.float32).copy()


def _table(fn: str, n: int) -> np.ndarray:
    out = (ctypes.c_float * n)()
    getattr(load(), fn)(out)
    return np.frombuffer(out, dtype=np.float32).copy()


def int4_levels() -> np.ndarray:
    """16 levels i / 7, i = -8..7 (absmax 4-bit integers), for the nf4= argument."""
    return _table("qlora_int4_levels", 16)


def fp4_levels() -> np.ndarray:
    """The E2M1 values / 6 plus an unused top level, for the nf4= argument."""
    return _table("qlora_fp4_levels", 16)


def dq_signed_levels() -> np.ndarray:
    """Signed linear 8-bit map (2k - 255) / 255, for the t8= argument."""
    return _table("qlora_dq_signed_levels", 256)


def dq_dynamic_levels() -> np.ndarray:
    """Dynamic-exponent 8-bit map over [0, 1], for the t8= argument."""
    return _table("qlora_dq_dynamic_levels", 256)


def abi_version() -> int:
    return int(load().qlora_abi_version())


def workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return int(load().qlora_workspace_bytes(M, N, K, r))


def device_error(clear: bool = False) -> int:
    return int(load().qlora_device_error(1 if clear else 0))


def selftest_bounded_wait():
    """Launch the library's failure-path self-test on the current stream: a
    kernel whose one wait never completes gives up after the bounded-wait
    limit and sets bit 0 of the device error word (read it with
    device_error)."""
    _check(load().qlora_selftest_bounded_wait(_stream()), "qlora_selftest_bounded_wait")


def debug_fail_allocs(n: int, skip: int = 0) -> int:
    """Host-side allocation fault injection: after `skip` more of the
    library's resource allocations succeed (managed optimizer state, the
    block executor's streams and events), the next `n` fail as if the driver
    were out of memory. n = 0 cancels. Returns the failures still pending
    before the call."""
    return int(load().qlora_debug_fail_allocs(int(skip), int(n)))


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(load().qlora_launch_count())


def set_trace_events(start=None, stop=None):
    """Record torch.cuda.Event `start`/`stop` around the fused GEMM kernel of
    the following linear_fwd / linear_bwd calls (None, None to stop)."""
    if start is None or stop is None:
        load().qlora_set_trace_events(None, None)
    else:
        load().qlora_set_trace_events(ctypes.c_void_p(start.cuda_event), ctypes.c_void_p(stop.cuda_event))


def quantize_nf4(W: torch.Tensor, nf4=None, packed=None, absmax=None):
    """W bf16 [N, K] -> (packed uint8 [N*K/2], absmax fp32 [N*K/64])."""
    N, K = W.shape
    _req(W, "W", torch.bfloat16)
    if packed is None:
        packed = torch.empty(N * K // 2, dtype=torch.uint8, device=W.device)
    if absmax is None:
        absmax = torch.empty(N * K // BLOCK, dtype=torch.float32, device=W.device)
    _req(packed, "packed", torch.uint8, (N * K // 2,))
    _req(absmax, "absmax", torch.float32, (N * K // BLOCK,))
    tb = _tables(nf4, None)
    _check(load().qlora_quantize_nf4(_ptr(W), N, K, tb.nf4, _ptr(packed), _ptr(absmax), _stream()),
           "qlora_quantize_nf4")
    return packed, absmax


def quantize_dq(W: torch.Tensor, nf4=None, t8=None, packed=None, q=None, scale2=None, absmax=None):
    """W bf16 [N, K] -> (packed uint8 [N*K/2], q uint8 [nb], scale2 fp32
    [ceil(nb/256)]) in one pass (qlora_quantize_dq); the fp32 block
    constants are written to `absmax` only when it is given."""
    N, K = W.shape
    _req(W, "W", torch.bfloat16)
    nb = N * K // BLOCK
    ng = (nb + DQ_BLOCK - 1) // DQ_BLOCK
    if packed is None:
        packed = torch.empty(N * K // 2, dtype=torch.uint8, device=W.device)
    if q is None:
        q = torch.empty(nb, dtype=torch.uint8, device=W.device)
    if scale2 is None:
        scale2 = torch.empty(ng, dtype=torch.float32, device=W.device)
    _req(packed, "packed", torch.uint8, (N * K // 2,))
    _req(q, "q", torch.uint8, (nb,))
    _req(scale2, "scale2", torch.float32, (ng,))
    if absmax is not None:
        _req(absmax, "absmax", torch.float32, (nb,))
    tb = _tables(nf4, t8)
    _check(load().qlora_quantize_dq(_ptr(W), N, K, tb.nf4, tb.t8, _ptr(packed), _ptr(q), _ptr(scale2), _ptr(absmax),
                                    _stream()), "qlora_quantize_dq")
    return packed, q, scale2


def double_quant(absmax: torch.Tensor, t8=None, q=None, scale2=None):
    """absmax fp32 [nb] -> (q uint8 [nb], scale2 fp32 [ceil(nb/256)])."""
    _req(absmax, "absmax", torch.float32)
    nb = absmax.numel()
    ng = (nb + DQ_BLOCK - 1) // DQ_BLOCK
    if q is None:
        q = torch.empty(nb, dtype=torch.uint8, device=absmax.device)
    if scale2 is None:
        scale2 = torch.empty(ng, dtype=torch.float32, device=absmax.device)
    _req(q, "q", torch.uint8, (nb,))
    _req(scale2, "scale2", torch.float32, (ng,))
    tb = _tables(None, t8)
    _check(load().qlora_double_quant(_ptr(absmax), nb, tb.t8, _ptr(q), _ptr(scale2), _stream()),
           "qlora_double_quant")
    return q, scale2


def _dtype_of(t, name):
    if t.dtype not in _DTYPE:
        raise TypeError(f"{name} must be torch.bfloat16 or torch.float16, got {t.dtype}")
    return t.dtype


def dequant(packed, q, scale2, N: int, K: int, nf4=None, t8=None, out=None,
            dtype=torch.bfloat16) -> torch.Tensor:
    """-> W' [N, K] in `dtype` (bf16, or fp16 through qlora_dequant_dt)."""
    _req(packed, "packed", torch.uint8, (N * K // 2,))
    _req(q, "q", torch.uint8, (N * K // BLOCK,))
    _req(scale2, "scale2", torch.float32)
    if dtype not in _DTYPE:
        raise TypeError(f"dtype must be torch.bfloat16 or torch.float16, got {dtype}")
    if out is None:
        out = torch.empty((N, K), dtype=dtype, device=packed.device)
    _req(out, "out", dtype, (N, K))
    tb = _tables(nf4, t8)
    if dtype == torch.bfloat16:
        _check(load().qlora_dequant(_ptr(packed), _ptr(q), _ptr(scale2), N, K, tb.nf4, tb.t8, _ptr(out),
                                    _stream()), "qlora_dequant")
    else:
        _check(load().qlora_dequant_dt(_ptr(packed), _ptr(q), _ptr(scale2), N, K, tb.nf4, tb.t8,
                                       _DTYPE[dtype], _ptr(out), _stream()), "qlora_dequant_dt")
    return out


def _workspace(workspace, M, N, K, r, device):
    need = workspace_bytes(M, N, K, r)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    _req(workspace, "workspace", torch.uint8)
    return workspace


def linear_fwd(packed, q, scale2, X, A, B, alpha: float, N: int, K: int, nf4=None, t8=None,
               Y=None, XA_out=None, workspace=None):
    """Y = X W'^T + (alpha/r) (X A) B  -> Y [M, N] (and XA_out if given).

    The 16-bit tensors are all bf16 or all fp16 (X's dtype decides; fp16
    goes through qlora_linear_fwd_dt)."""
    M = X.shape[0]
    r = A.shape[1]
    dt = _dtype_of(X, "X")
    _req(X, "X", dt, (M, K))
    _req(A, "A", dt, (K, r))
    _req(B, "B", dt, (r, N))
    if Y is None:
        Y = torch.empty((M, N), dtype=dt, device=X.device)
    _req(Y, "Y", dt, (M, N))
    if XA_out is not None:
        _req(XA_out, "XA_out", dt, (M, r))
    workspace = _workspace(workspace, M, N, K, r, X.device)
    tb = _tables(nf4, t8)
    if dt == torch.bfloat16:
        _check(load().qlora_linear_fwd(_ptr(packed), _ptr(q), _ptr(scale2), tb.nf4, tb.t8, M, N, K, _ptr(X),
                                       _ptr(A), _ptr(B), r, float(alpha), _ptr(Y), _ptr(XA_out),
                                       _ptr(workspace), workspace.numel(), _stream()), "qlora_linear_fwd")
    else:
        _check(load().qlora_linear_fwd_dt(_ptr(packed), _ptr(q), _ptr(scale2), tb.nf4, tb.t8, _DTYPE[dt], M, N,
                                          K, _ptr(X), _ptr(A), _ptr(B), r, float(alpha), _ptr(Y),
                                          _ptr(XA_out), _ptr(workspace), workspace.numel(), _stream()),
               "qlora_linear_fwd_dt")
    return Y


def linear_fwd_noalloc(packed, q, scale2, X, A, B, alpha: float, N: int, K: int, nf4=None, t8=None,
                       Y=None, XA_out=None):
    """linear_fwd for callers that cannot allocate device memory: no workspace
    argument; the library's fixed device scratch (NOALLOC_SCRATCH_BYTES) is
    used instead. Y must be preallocated by such a caller (pass Y=...)."""
    M = X.shape[0]
    r = A.shape[1]
    _req(X, "X", torch.bfloat16, (M, K))
    _req(A, "A", torch.bfloat16, (K, r))
    _req(B, "B", torch.bfloat16, (r, N))
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _req(Y, "Y", torch.bfloat16, (M, N))
    if XA_out is not None:
        _req(XA_out, "XA_out", torch.bfloat16, (M, r))
    tb = _tables(nf4, t8)
    _check(load().qlora_linear_fwd_noalloc(_ptr(packed), _ptr(q), _ptr(scale2), tb.nf4, tb.t8, M, N, K,
                                           _ptr(X), _ptr(A), _ptr(B), r, float(alpha), _ptr(Y),
                                           _ptr(XA_out), _stream()), "qlora_linear_fwd_noalloc")
    return Y


def linear_bwd(packed, q, scale2, X, dY, A, B, alpha: float, N: int, K: int, XA=None, nf4=None, t8=None,
               dX=None, dA=None, dB=None, workspace=None):
    """-> (dX [M, K], dA [K, r], dB [r, N]); no dW (W is frozen). The 16-bit
    tensors are all bf16 or all fp16 (X's dtype decides)."""
    M = X.shape[0]
    r = A.shape[1]
    dt = _dtype_of(X, "X")
    _req(X, "X", dt, (M, K))
    _req(dY, "dY", dt, (M, N))
    _req(A, "A", dt, (K, r))
    _req(B, "B", dt, (r, N))
    if XA is not None:
        _req(XA, "XA", dt, (M, r))
    dev = X.device
    dX = torch.empty((M, K), dtype=dt, device=dev) if dX is None else dX
    dA = torch.empty((K, r), dtype=dt, device=dev) if dA is None else dA
    dB = torch.empty((r, N), dtype=dt, device=dev) if dB is None else dB
    _req(dX, "dX", dt, (M, K))
    _req(dA, "dA", dt, (K, r))
    _req(dB, "dB", dt, (r, N))
    workspace = _workspace(workspace, M, N, K, r, dev)
    tb = _tables(nf4, t8)
    if dt == torch.bfloat16:
        _check(load().qlora_linear_bwd(_ptr(packed), _ptr(q), _ptr(scale2), tb.nf4, tb.t8, M, N, K, _ptr(X),
                                       _ptr(dY), _ptr(A), _ptr(B), _ptr(XA), r, float(alpha), _ptr(dX),
                                       _ptr(dA), _ptr(dB), _ptr(workspace), workspace.numel(), _stream()),
               "qlora_linear_bwd")
    else:
        _check(load().qlora_linear_bwd_dt(_ptr(packed), _ptr(q), _ptr(scale2), tb.nf4, tb.t8, _DTYPE[dt], M, N,
                                          K, _ptr(X), _ptr(dY), _ptr(A), _ptr(B), _ptr(XA), r, float(alpha),
                                          _ptr(dX), _ptr(dA), _ptr(dB), _ptr(workspace), workspace.numel(),
                                          _stream()), "qlora_linear_bwd_dt")
    return dX, dA, dB


def paged_adamw_placement(free_bytes: int, state_bytes: int, reserve_bytes: int, current: int) -> int:
    """The library's placement policy: 1 (state on the host) or 0 (device)."""
    return int(load().qlora_paged_adamw_placement(free_bytes, state_bytes, reserve_bytes, current))


class PagedAdamW:
    """AdamW over 16-bit adapter tensors with its fp32 state (master copy and
    moments) in unified memory that the library pages between device and
    host by free device memory (qlora_paged_adamw_*)."""

    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0):
        self.params = list(params)
        if not self.params:
            raise ValueError("no parameters")
        self.dtype = _dtype_of(self.params[0], "params[0]")
        for i, p in enumerate(self.params):
            _req(p, f"params[{i}]", self.dtype)
        self.lr, self.betas, self.eps, self.weight_decay = lr, betas, eps, weight_decay
        self.t = 0
        lib = load()
        counts = (ctypes.c_int64 * len(self.params))(*[p.numel() for p in self.params])
        h = ctypes.c_void_p()
        _check(lib.qlora_paged_adamw_create(len(self.params), counts, ctypes.byref(h)), "qlora_paged_adamw_create")
        self._h = h
        self._pp = (ctypes.c_void_p * len(self.params))(*[p.data_ptr() for p in self.params])
        _check(lib.qlora_paged_adamw_init(self._h, self._pp, _DTYPE[self.dtype], _stream()), "qlora_paged_adamw_init")

    def step(self, grads):
        grads = list(grads)
        if len(grads) != len(self.params):
            raise ValueError("one gradient per parameter")
        for i, (g, p) in enumerate(zip(grads, self.params)):
            _req(g, f"grads[{i}]", self.dtype, tuple(p.shape))
        gp = (ctypes.c_void_p * len(grads))(*[g.data_ptr() for g in grads])
        self.t += 1
        _check(load().qlora_paged_adamw_step(self._h, self._pp, gp, _DTYPE[self.dtype], self.t, float(self.lr),
                                             float(self.betas[0]), float(self.betas[1]), float(self.eps),
                                             float(self.weight_decay), _stream()), "qlora_paged_adamw_step")

    def set_reserve(self, reserve_bytes: int):
        _check(load().qlora_paged_adamw_set_reserve(self._h, int(reserve_bytes)), "qlora_paged_adamw_set_reserve")

    @property
    def location(self) -> str:
        return "host" if load().qlora_paged_adamw_location(self._h) == 1 else "device"

    @property
    def state_bytes(self) -> int:
        return int(load().qlora_paged_adamw_state_bytes(self._h))

    def state(self):
        """Host copies (numpy float32) of the master copy and the moments,
        concatenated over the tensors in order; synchronizes the device."""
        torch.cuda.synchronize()
        pm, pm1, pv = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        _check(load().qlora_paged_adamw_state(self._h, ctypes.byref(pm), ctypes.byref(pm1), ctypes.byref(pv)),
               "qlora_paged_adamw_state")
        n = sum(p.numel() for p in self.params)
        out = []
        for ptr in (pm, pm1, pv):
            a = np.empty(n, np.float32)
            ctypes.memmove(a.ctypes.data, ptr.value, n * 4)
            out.append(a)
        return tuple(out)

    def close(self):
        if getattr(self, "_h", None):
            load().qlora_paged_adamw_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


_DESC_TENSORS = ("X", "A", "B", "Y", "XA", "dY", "dX", "dA", "dB")


def _descs(linears, M: int, r: int, need):
    """ctypes array of qlora_linear_desc from dicts of tensors; `need` names
    the tensors the pass reads or writes (checked for type and shape)."""
    arr = (LinearDesc * len(linears))()
    dt = None
    for i, L in enumerate(linears):
        N, K = int(L["N"]), int(L["K"])
        shapes = {"X": (M, K), "A": (K, r), "B": (r, N), "Y": (M, N), "XA": (M, r), "dY": (M, N), "dX": (M, K),
                  "dA": (K, r), "dB": (r, N)}
        d = arr[i]
        d.packed, d.q, d.scale2 = (L[k].data_ptr() for k in ("packed", "q", "scale2"))
        d.N, d.K = N, K
        for k in _DESC_TENSORS:
            t = L.get(k)
            if k in need:
                if t is None:
                    raise ValueError(f"linear {i}: {k} is required")
                dt = dt or _dtype_of(t, k)
                _req(t, f"linear {i} {k}", dt, shapes[k])
            setattr(d, k, None if t is None else t.data_ptr())
    return arr, dt


def block_workspace_bytes(linears, M: int, r: int) -> int:
    arr, _ = _descs(linears, M, r, ())
    return int(load().qlora_block_workspace_bytes(len(linears), arr, M, r))


def _block(fn, linears, M, r, alpha, save_xa, workspace, nf4, t8, need):
    arr, dt = _descs(linears, M, r, need)
    need_ws = int(load().qlora_block_workspace_bytes(len(linears), arr, M, r))
    if workspace is None:
        workspace = torch.empty(max(need_ws, 256), dtype=torch.uint8, device=linears[0]["X"].device)
    _req(workspace, "workspace", torch.uint8)
    tb = _tables(nf4, t8)
    _check(getattr(load(), fn)(len(linears), arr, tb.nf4, tb.t8, _DTYPE[dt], M, r, float(alpha), 1 if save_xa else 0,
                               _ptr(workspace), workspace.numel(), _stream()), fn)
    return workspace


def block_fwd(linears, M: int, r: int, alpha: float, save_xa: bool = True, workspace=None, nf4=None, t8=None):
    """Forward of every linear of a decoder block in one call (qlora_block_fwd):
    each dict holds packed, q, scale2, N, K, X, A, B, Y and, with save_xa, XA."""
    need = ("X", "A", "B", "Y") + (("XA",) if save_xa else ())
    return _block("qlora_block_fwd", linears, M, r, alpha, save_xa, workspace, nf4, t8, need)


def block_bwd(linears, M: int, r: int, alpha: float, save_xa: bool = True, workspace=None, nf4=None, t8=None):
    """Backward of every linear of a decoder block in one call (qlora_block_bwd):
    each dict also holds dY, dX, dA, dB (and XA when the forward saved it)."""
    need = ("X", "A", "B", "dY", "dX", "dA", "dB") + (("XA",) if save_xa else ())
    return _block("qlora_block_bwd", linears, M, r, alpha, save_xa, workspace, nf4, t8, need)
