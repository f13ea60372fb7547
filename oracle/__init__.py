"""Plain, slow CPU oracle for the QLoRA frozen-base linear layer.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s cpu_baseline / reference leg may import this package. It
shares no code with the CUDA library in ``bit_quantized_lora_blockwise_b200``
and imports nothing from it.

Two halves:

* the codec (NF4 table, blockwise absmax, nearest-level encode, double
  quantization, dequantization) in plain C (``qlora_oracle.c``), built with
  gcc at IEEE binary32 semantics and called through ctypes;
* the linear layer forward/backward in numpy float64 (``linear.py``).

Pinned by ``tests/test_oracle_*.py`` against what the pages fix (see the
header of each test file). The exact NF4 level values are not printed on the
pages, so agreement of the table with any external NF4 table is parity
unpinned; its construction (normal quantiles, equal mass per side, [-1, 1],
exact zero) is pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .linear import (linear_fwd, linear_bwd, linear_fwd_rows, linear_bwd_rows,
                     bf16_bits_to_f64)

__all__ = [
    "BLOCK", "DQ_BLOCK", "nf4_levels", "dq_levels", "nearest_level",
    "absmax", "encode_nf4", "quantize_nf4", "double_quant", "dequant", "dequant_f16", "f32_to_f16",
    "dq_constants", "bf16_to_f32", "f32_to_bf16", "linear_fwd", "linear_bwd",
    "linear_fwd_rows", "linear_bwd_rows", "bf16_bits_to_f64", "build",
]

BLOCK = 64
DQ_BLOCK = 256

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qlora_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_liboracle.so")
_CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fexcess-precision=standard",
           "-mfpmath=sse", "-shared", "-fPIC", "-std=c11"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (in-tree ``oracle/_liboracle.so``)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.oracle_nf4_levels.argtypes = [P]
            lib.oracle_dq_levels.argtypes = [P]
            lib.oracle_nearest_level.argtypes = [ctypes.c_float, P, ctypes.c_int]
            lib.oracle_nearest_level.restype = ctypes.c_int
            lib.oracle_absmax.argtypes = [P, I64, P]
            lib.oracle_encode_nf4.argtypes = [P, I64, P, P, P]
            lib.oracle_double_quant.argtypes = [P, I64, P, P, P]
            lib.oracle_dequant.argtypes = [P, P, P, I64, P, P, P]
            lib.oracle_dq_constants.argtypes = [P, P, I64, P, P]
            lib.oracle_bf16_to_f32.argtypes = [P, I64, P]
            lib.oracle_f32_to_bf16.argtypes = [P, I64, P]
            lib.oracle_dequant_f16.argtypes = [P, P, P, I64, P, P, P]
            lib.oracle_f32_to_f16.argtypes = [P, I64, P]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 arrays are passed as their uint16 bit patterns")
    return a


def nf4_levels() -> np.ndarray:
    """The 16 ascending NF4 levels (fp32); construction in qlora_oracle.c."""
    out = np.zeros(16, np.float32)
    _load().oracle_nf4_levels(_ptr(out))
    return out


def dq_levels() -> np.ndarray:
    """The 256 ascending 8-bit constant levels T8[k] = k/255 (fp32)."""
    out = np.zeros(256, np.float32)
    _load().oracle_dq_levels(_ptr(out))
    return out


def nearest_level(x: float, levels: np.ndarray) -> int:
    lv = np.ascontiguousarray(levels, np.float32)
    return int(_load().oracle_nearest_level(ctypes.c_float(x), _ptr(lv), len(lv)))


def absmax(w_bits: np.ndarray) -> np.ndarray:
    """Blockwise absmax (one fp32 per 64 consecutive row-major elements)."""
    w = _u16(w_bits).reshape(-1)
    if w.size % BLOCK:
        raise ValueError("element count must be a multiple of 64")
    out = np.zeros(w.size // BLOCK, np.float32)
    _load().oracle_absmax(_ptr(w), w.size, _ptr(out))
    return out


def encode_nf4(w_bits: np.ndarray, amax: np.ndarray, levels: np.ndarray) -> np.ndarray:
    w = _u16(w_bits).reshape(-1)
    amax = np.ascontiguousarray(amax, np.float32)
    lv = np.ascontiguousarray(levels, np.float32)
    out = np.zeros(w.size // 2, np.uint8)
    _load().oracle_encode_nf4(_ptr(w), w.size, _ptr(amax), _ptr(lv), _ptr(out))
    return out


def quantize_nf4(w_bits: np.ndarray, levels: np.ndarray | None = None):
    """Returns (packed uint8 [N*K/2], absmax fp32 [N*K/64])."""
    lv = nf4_levels() if levels is None else levels
    amax = absmax(w_bits)
    return encode_nf4(w_bits, amax, lv), amax


def double_quant(amax: np.ndarray, t8: np.ndarray | None = None):
    """Returns (q uint8 [nb], scale2 fp32 [ceil(nb/256)])."""
    amax = np.ascontiguousarray(amax, np.float32).reshape(-1)
    t8 = dq_levels() if t8 is None else np.ascontiguousarray(t8, np.float32)
    nb = amax.size
    q = np.zeros(nb, np.uint8)
    s2 = np.zeros((nb + DQ_BLOCK - 1) // DQ_BLOCK, np.float32)
    _load().oracle_double_quant(_ptr(amax), nb, _ptr(t8), _ptr(q), _ptr(s2))
    return q, s2


def dequant(packed: np.ndarray, q: np.ndarray, scale2: np.ndarray, n_elems: int,
            levels: np.ndarray | None = None, t8: np.ndarray | None = None) -> np.ndarray:
    """bf16 bit patterns of the dequantized weight (flat, n_elems)."""
    lv = nf4_levels() if levels is None else np.ascontiguousarray(levels, np.float32)
    t8 = dq_levels() if t8 is None else np.ascontiguousarray(t8, np.float32)
    packed = np.ascontiguousarray(packed, np.uint8).reshape(-1)
    q = np.ascontiguousarray(q, np.uint8).reshape(-1)
    scale2 = np.ascontiguousarray(scale2, np.float32).reshape(-1)
    out = np.zeros(n_elems, np.uint16)
    _load().oracle_dequant(_ptr(packed), _ptr(q), _ptr(scale2), n_elems, _ptr(lv),
                           _ptr(t8), _ptr(out))
    return out


def dequant_f16(packed: np.ndarray, q: np.ndarray, scale2: np.ndarray, n_elems: int,
                levels: np.ndarray | None = None, t8: np.ndarray | None = None) -> np.ndarray:
    """fp16 bit patterns of the dequantized weight (flat, n_elems)."""
    lv = nf4_levels() if levels is None else np.ascontiguousarray(levels, np.float32)
    t8 = dq_levels() if t8 is None else np.ascontiguousarray(t8, np.float32)
    packed = np.ascontiguousarray(packed, np.uint8).reshape(-1)
    q = np.ascontiguousarray(q, np.uint8).reshape(-1)
    scale2 = np.ascontiguousarray(scale2, np.float32).reshape(-1)
    out = np.zeros(n_elems, np.uint16)
    _load().oracle_dequant_f16(_ptr(packed), _ptr(q), _ptr(scale2), n_elems, _ptr(lv),
                               _ptr(t8), _ptr(out))
    return out


def f32_to_f16(x: np.ndarray) -> np.ndarray:
    """fp16 bit patterns of x (round to nearest even)."""
    x = np.ascontiguousarray(x, np.float32)
    out = np.zeros(x.shape, np.uint16)
    _load().oracle_f32_to_f16(_ptr(x), x.size, _ptr(out))
    return out


def dq_constants(q: np.ndarray, scale2: np.ndarray, t8: np.ndarray | None = None) -> np.ndarray:
    t8 = dq_levels() if t8 is None else np.ascontiguousarray(t8, np.float32)
    q = np.ascontiguousarray(q, np.uint8).reshape(-1)
    scale2 = np.ascontiguousarray(scale2, np.float32).reshape(-1)
    out = np.zeros(q.size, np.float32)
    _load().oracle_dq_constants(_ptr(q), _ptr(scale2), q.size, _ptr(t8), _ptr(out))
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    b = _u16(bits)
    out = np.zeros(b.shape, np.float32)
    _load().oracle_bf16_to_f32(_ptr(b), b.size, _ptr(out))
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    out = np.zeros(x.shape, np.uint16)
    _load().oracle_f32_to_bf16(_ptr(x), x.size, _ptr(out))
    return out
