"""CPU-only checks of the C ABI: the library loads, exports every symbol that
include/qlora.h declares, and its host-side argument checks return the
documented status codes before anything touches a GPU (no compute calls).
"""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]*?\b(qlora_\w+)\s*\(", text)))


def test_header_declares_the_five_calls():
    syms = declared_symbols()
    for name in ("qlora_quantize_nf4", "qlora_double_quant", "qlora_dequant", "qlora_linear_fwd",
                 "qlora_linear_bwd"):
        assert name in syms
    assert set(syms) == set(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.qlora_abi_version() == 2


def test_library_has_sm100a_code():
    # the fatbin section must hold sm_100a code; nvcc records the arch in the ELF notes
    data = open(LIB, "rb").read()
    assert b"sm_100a" in data


def test_status_strings(lib):
    for code, name in binding._STATUS.items():
        assert lib.qlora_status_string(code).decode() == name


def test_host_tables_match_oracle(lib):
    import oracle
    from oracle import codebooks as cb
    assert np.array_equal(binding.nf4_levels(), oracle.nf4_levels())
    assert np.array_equal(binding.dq_levels(), oracle.dq_levels())
    # the alternative tables, bit for bit (the +0 of FP4 included)
    for got, want in ((binding.int4_levels(), cb.int4_levels()), (binding.fp4_levels(), cb.fp4_levels()),
                      (binding.dq_signed_levels(), cb.dq_signed_levels()),
                      (binding.dq_dynamic_levels(), cb.dq_dynamic_levels())):
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_argument_checks_before_any_launch(lib):
    tb = binding._tables(None, None)
    s = ctypes.c_void_p(0)
    # NULL pointers
    assert lib.qlora_quantize_nf4(None, 64, 64, tb.nf4, _fake(), _fake(), s) == 1
    assert lib.qlora_double_quant(_fake(), 10, tb.t8, None, _fake(), s) == 1
    # shapes: K % 64, K < 64, N < 1
    assert lib.qlora_quantize_nf4(_fake(), 64, 96, tb.nf4, _fake(), _fake(), s) == 2
    assert lib.qlora_quantize_nf4(_fake(), 0, 64, tb.nf4, _fake(), _fake(), s) == 2
    assert lib.qlora_double_quant(_fake(), 0, tb.t8, _fake(), _fake(), s) == 2
    # alignment
    assert lib.qlora_quantize_nf4(_fake(0x10008), 64, 64, tb.nf4, _fake(), _fake(), s) == 3
    # tables: not ascending / no exact zero
    bad = (ctypes.c_float * 16)(*np.linspace(-1, 1, 16).astype(np.float32))  # no exact 0
    assert lib.qlora_quantize_nf4(_fake(), 64, 64, bad, _fake(), _fake(), s) == 8
    desc = (ctypes.c_float * 256)(*np.linspace(1, 0, 256).astype(np.float32))
    assert lib.qlora_double_quant(_fake(), 10, desc, _fake(), _fake(), s) == 8
    # linear: r range, r % 8, N % 64, alpha finite
    args = dict(M=16, N=128, K=128, r=8, alpha=16.0)

    def fwd(**kw):
        a = {**args, **kw}
        return lib.qlora_linear_fwd(_fake(), _fake(), _fake(), tb.nf4, tb.t8, a["M"], a["N"], a["K"],
                                    _fake(), _fake(), _fake(), a["r"], a["alpha"], _fake(), None,
                                    _fake(), 1 << 30, s)
    assert fwd(r=0) == 4 and fwd(r=300) == 4 and fwd(r=12) == 4
    assert fwd(N=96) == 2 and fwd(K=32) == 2 and fwd(M=0) == 2
    assert fwd(alpha=float("inf")) == 4
    assert lib.qlora_workspace_bytes(16, 96, 128, 8) == 0
    assert lib.qlora_workspace_bytes(16, 128, 128, 8) > 0
    # a NaN level is refused like a descending table
    nan8 = np.arange(256, dtype=np.float32) / 255
    nan8[17] = np.nan
    assert lib.qlora_double_quant(_fake(), 10, (ctypes.c_float * 256)(*nan8), _fake(), _fake(), s) == 8
    # dequant: NULL output, K % 64, misaligned output
    assert lib.qlora_dequant(_fake(), _fake(), _fake(), 64, 64, tb.nf4, tb.t8, None, s) == 1
    assert lib.qlora_dequant(_fake(), _fake(), _fake(), 64, 96, tb.nf4, tb.t8, _fake(), s) == 2
    assert lib.qlora_dequant(_fake(), _fake(), _fake(), 64, 64, tb.nf4, tb.t8, _fake(0x10004), s) == 3

    def bwd(**kw):
        a = {**args, **kw}
        return lib.qlora_linear_bwd(_fake(), _fake(), _fake(), tb.nf4, tb.t8, a["M"], a["N"], a["K"],
                                    _fake(), _fake(), _fake(), _fake(), None, a["r"], a["alpha"],
                                    _fake(), _fake(), _fake(), _fake(), 1 << 30, s)
    assert bwd(r=0) == 4 and bwd(r=257) == 4 and bwd(N=100) == 2 and bwd(alpha=float("nan")) == 4


def test_dtype_argument_is_checked_first(lib):
    """A compute type other than bf16 (0) and fp16 (1) is refused before any
    other check or launch."""
    tb = binding._tables(None, None)
    s = ctypes.c_void_p(0)
    for bad in (2, -1, 7):
        assert lib.qlora_dequant_dt(_fake(), _fake(), _fake(), 64, 64, tb.nf4, tb.t8, bad, _fake(), s) == 4
        assert lib.qlora_linear_fwd_dt(_fake(), _fake(), _fake(), tb.nf4, tb.t8, bad, 16, 128, 128, _fake(),
                                       _fake(), _fake(), 8, 16.0, _fake(), None, _fake(), 1 << 30, s) == 4
        assert lib.qlora_linear_bwd_dt(_fake(), _fake(), _fake(), tb.nf4, tb.t8, bad, 16, 128, 128, _fake(),
                                       _fake(), _fake(), _fake(), None, 8, 16.0, _fake(), _fake(), _fake(),
                                       _fake(), 1 << 30, s) == 4
    # with a valid type the ordinary checks follow (r out of range)
    assert lib.qlora_linear_fwd_dt(_fake(), _fake(), _fake(), tb.nf4, tb.t8, 1, 16, 128, 128, _fake(), _fake(),
                                   _fake(), 0, 16.0, _fake(), None, _fake(), 1 << 30, s) == 4
    assert lib.qlora_dequant_dt(None, _fake(), _fake(), 64, 64, tb.nf4, tb.t8, 1, _fake(), s) == 1


def test_quantize_dq_argument_checks(lib):
    """The one-pass quantize checks its arguments like the two calls it
    replaces, before any launch."""
    tb = binding._tables(None, None)
    s = ctypes.c_void_p(0)
    f = lib.qlora_quantize_dq
    assert f(None, 64, 64, tb.nf4, tb.t8, _fake(), _fake(), _fake(), None, s) == 1
    assert f(_fake(), 64, 64, tb.nf4, tb.t8, _fake(), None, _fake(), None, s) == 1
    assert f(_fake(), 64, 96, tb.nf4, tb.t8, _fake(), _fake(), _fake(), None, s) == 2
    assert f(_fake(), 0, 64, tb.nf4, tb.t8, _fake(), _fake(), _fake(), None, s) == 2
    assert f(_fake(0x10008), 64, 64, tb.nf4, tb.t8, _fake(), _fake(), _fake(), None, s) == 3
    assert f(_fake(), 64, 64, tb.nf4, tb.t8, _fake(), _fake(), _fake(), _fake(0x10004), s) == 3
    bad = (ctypes.c_float * 16)(*np.linspace(-1, 1, 16).astype(np.float32))  # no exact 0
    assert f(_fake(), 64, 64, bad, tb.t8, _fake(), _fake(), _fake(), None, s) == 8


def test_block_and_optimizer_argument_checks(lib):
    """Block executor and paged optimizer: null, shape and range checks that
    need no device."""
    tb = binding._tables(None, None)
    s = ctypes.c_void_p(0)
    assert lib.qlora_block_fwd(0, None, tb.nf4, tb.t8, 0, 16, 8, 16.0, 1, _fake(), 1 << 20, s) == 2
    assert lib.qlora_block_bwd(1, None, tb.nf4, tb.t8, 0, 16, 8, 16.0, 1, _fake(), 1 << 20, s) == 1
    assert lib.qlora_block_fwd(1, None, tb.nf4, tb.t8, 5, 16, 8, 16.0, 1, _fake(), 1 << 20, s) == 4
    assert lib.qlora_block_workspace_bytes(0, None, 16, 8) == 0
    counts = (ctypes.c_int64 * 2)(10, 0)
    h = ctypes.c_void_p()
    assert lib.qlora_paged_adamw_create(2, counts, ctypes.byref(h)) == 2
    assert lib.qlora_paged_adamw_create(0, counts, ctypes.byref(h)) == 2
    assert lib.qlora_paged_adamw_create(1, None, ctypes.byref(h)) == 1
    assert lib.qlora_paged_adamw_location(None) == -1
    assert lib.qlora_paged_adamw_state_bytes(None) == 0
    lib.qlora_paged_adamw_destroy(None)  # a no-op


def test_alloc_fault_injection_counter(lib):
    """The injector's pending count: set, read back by the next call, and
    cancelled by n <= 0 (no allocation is made on a CPU-only host)."""
    assert binding.debug_fail_allocs(0) == 0
    assert binding.debug_fail_allocs(3, skip=2) == 0
    assert binding.debug_fail_allocs(-1) == 3
    assert binding.debug_fail_allocs(1) == 0
    assert binding.debug_fail_allocs(0) == 1
    assert binding.debug_fail_allocs(0) == 0
