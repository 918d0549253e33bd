"""The C-ABI library loads and exports every entry point include/gptq.h
declares; host-side argument checks (no GPU needed, no kernel launched)."""
import ctypes
import os
import re

import pytest

from post_weight_quantization_25_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptq.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_[a-z0-9_]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from post_weight_quantization_25_b200 import build
        build.build()
    return _lib.load()


def test_header_declares_the_expected_entry_points():
    assert _declared() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.gptq_status_string(0) == b"ok"
    assert lib.gptq_status_string(5) == b"device wait timed out"
    assert lib.gptq_status_string(99) == b"unknown status"


def test_workspace_sizes(lib):
    out = ctypes.c_size_t(0)
    cfg = _lib.GptqConfig(4, 128, 0.01, 128, 1, 0)
    # bf16: the turnstile counters of the ordered split-K reduction only
    assert lib.gptq_workspace_size(_lib.GPTQ_OP_HESSIAN, 0, 256, 2048, _lib.GPTQ_BF16, None,
                                   ctypes.byref(out)) == 0
    assert 0 < out.value <= 4096
    flags = out.value
    assert lib.gptq_workspace_size(_lib.GPTQ_OP_HESSIAN, 0, 256, 2048, _lib.GPTQ_F32, None,
                                   ctypes.byref(out)) == 0
    assert out.value >= flags + 2 * 256 * 2048 * 2
    assert lib.gptq_workspace_size(_lib.GPTQ_OP_DEQUANT_MATVEC, 8, 4096, 0, 0, None,
                                   ctypes.byref(out)) == 0
    assert out.value >= 8 * 4096 * 2
    assert lib.gptq_workspace_size(_lib.GPTQ_OP_DEQUANT_MATVEC, -1, 4096, 0, 0, None,
                                   ctypes.byref(out)) == 1
    assert lib.gptq_workspace_size(_lib.GPTQ_OP_CHOLESKY, 0, 4096, 0, 0, None,
                                   ctypes.byref(out)) == 0
    assert out.value >= 4096 * 4096 * 4
    assert lib.gptq_workspace_size(_lib.GPTQ_OP_QUANTIZE, 4096, 4096, 0, 0, ctypes.byref(cfg),
                                   ctypes.byref(out)) == 0
    assert out.value >= 4096 * 4096 * 5
    # the symmetric ruler is accepted; sym must be 0 or 1
    sym = _lib.GptqConfig(4, 128, 0.01, 128, 1, 1)
    assert lib.gptq_workspace_size(2, 16, 16, 0, 0, ctypes.byref(sym), ctypes.byref(out)) == 0
    bad = _lib.GptqConfig(4, 128, 0.01, 128, 1, 2)
    assert lib.gptq_workspace_size(2, 16, 16, 0, 0, ctypes.byref(bad), ctypes.byref(out)) == 1
    # a block other than 128 is not implemented
    bad = _lib.GptqConfig(4, 128, 0.01, 64, 1, 0)
    assert lib.gptq_workspace_size(2, 16, 16, 0, 0, ctypes.byref(bad), ctypes.byref(out)) == 2
    bad = _lib.GptqConfig(4, 48, 0.01, 128, 1, 0)
    assert lib.gptq_workspace_size(2, 16, 16, 0, 0, ctypes.byref(bad), ctypes.byref(out)) == 2
    bad = _lib.GptqConfig(1, 128, 0.01, 128, 1, 0)
    assert lib.gptq_workspace_size(2, 16, 16, 0, 0, ctypes.byref(bad), ctypes.byref(out)) == 1
    assert lib.gptq_workspace_size(7, 16, 16, 0, 0, None, ctypes.byref(out)) == 1
    assert lib.gptq_workspace_size(0, 16, 0, 16, 0, None, ctypes.byref(out)) == 1


def test_argument_checks_reject_before_any_launch(lib):
    # null H / X, bad sizes, token-major layout: rejected on the host
    assert lib.gptq_hessian_accumulate(None, None, 0, 16, 16, 16, 0, 2.0, None, 0, None,
                                       None) == 1
    assert lib.gptq_hessian_accumulate(ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 16, 16, 8,
                                       0, 2.0, None, 0, None, None) == 1      # ldx < ntok
    assert lib.gptq_hessian_accumulate(ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 16, 16, 16,
                                       1, 2.0, None, 0, None, None) == 2      # token-major
    assert lib.gptq_hessian_accumulate(ctypes.c_void_p(256), ctypes.c_void_p(256), 1, 16, 16, 16,
                                       0, 2.0, None, 0, None, None) == 3      # fp32 needs ws
    assert lib.gptq_hessian_accumulate(ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 16, 16, 16,
                                       0, 2.0, None, 0, None, None) == 3      # bf16 too
    assert lib.gptq_hessian_accumulate(ctypes.c_void_p(256), ctypes.c_void_p(258), 0, 16, 16, 16,
                                       0, 2.0, ctypes.c_void_p(512), 4096, None,
                                       None) == 1                             # misaligned X
    assert lib.gptq_hessian_accumulate(ctypes.c_void_p(256), ctypes.c_void_p(256), 0, 16, 16, 16,
                                       0, 2.0, ctypes.c_void_p(520), 4096, None,
                                       None) == 1                             # misaligned ws
    assert lib.gptq_cholesky_inverse(None, 16, 0.01, 0, None, None, None, None, None, 0,
                                     None, None) == 1
    assert lib.gptq_cholesky_inverse(ctypes.c_void_p(256), 16, 0.01, 1, ctypes.c_void_p(256),
                                     None, ctypes.c_void_p(256), ctypes.c_void_p(256), None, 0,
                                     None, None) == 1                         # act-order, no perm
    assert lib.gptq_cholesky_inverse(ctypes.c_void_p(256), 16, 0.01, 0, ctypes.c_void_p(256),
                                     None, ctypes.c_void_p(256), ctypes.c_void_p(256), None, 0,
                                     None, None) == 3                         # no workspace
    cfg = _lib.GptqConfig(4, 128, 0.01, 128, 0, 0)
    assert lib.gptq_quantize_layer(None, 0, 0, 16, None, None, None, ctypes.byref(cfg), None,
                                   None, None, None, None, None, None, 0, None, None,
                                   None) == 0                                 # empty
    assert lib.gptq_quantize_layer(None, 0, 4, 16, None, None, None, ctypes.byref(cfg), None,
                                   None, None, None, None, None, None, 0, None, None,
                                   None) == 1
    # the wait gate: a limit out of range is rejected; clearing always works
    assert lib.gptq_set_wait_gate(ctypes.c_void_p(256), 0) == 1
    assert lib.gptq_set_wait_gate(ctypes.c_void_p(256), 2_000_000_000) == 1
    assert lib.gptq_set_wait_gate(None, 0) == 0
    assert lib.gptq_pack_int4(None, 4, 12, None, None) == 1                   # n % 8
    assert lib.gptq_pack_int3(None, 4, 40, None, None) == 1                   # n % 32
    assert lib.gptq_pack_int4(None, 0, 16, None, None) == 0                   # empty
    assert lib.gptq_dequant(None, 5, 4, 16, None, None, -1, 1, None, None, 0, None) == 2


def test_hadamard_argument_checks(lib):
    """Rejected before any device work: block not a power of two in
    [32, 1024], n not a multiple of the block, strides shorter than a row,
    in place with a different type; zero rows is a no-op."""
    p = ctypes.c_void_p(0x1000)
    UNSUP, INVAL = 2, 1
    assert lib.gptq_hadamard_rows(p, 0, 4, 1024, 1024, p, 48, p, 0, 1024, None) == UNSUP
    assert lib.gptq_hadamard_rows(p, 0, 4, 1024, 1024, p, 2048, p, 0, 1024, None) == UNSUP
    assert lib.gptq_hadamard_rows(p, 0, 4, 1024, 1024, p, 16, p, 0, 1024, None) == UNSUP
    assert lib.gptq_hadamard_rows(p, 0, 4, 1000, 1000, p, 32, p, 0, 1000, None) == INVAL
    assert lib.gptq_hadamard_rows(p, 0, 4, 1024, 512, p, 1024, p, 0, 1024, None) == INVAL
    assert lib.gptq_hadamard_cols(p, 0, 1024, 16, 8, p, 1024, p, 0, 16, None) == INVAL
    assert lib.gptq_hadamard_cols(p, 0, 1024, 16, 16, p, 1024, p, 1, 16, None) == INVAL
    assert lib.gptq_hadamard_rows(p, 2, 4, 1024, 1024, p, 1024, p, 0, 1024, None) == INVAL
    assert lib.gptq_hadamard_rows(p, 0, 0, 1024, 1024, p, 1024, p, 0, 1024, None) == 0
    assert lib.gptq_hadamard_cols(p, 0, 1024, 0, 0, p, 1024, p, 0, 0, None) == 0


def test_consumer_calls_with_nothing_to_do_or_bad_arguments(lib):
    """Zero rows or zero vectors are no-ops (no pointer is touched); bad
    widths, odd n, perm with g_idx and bad dtypes are rejected before any
    launch."""
    p = ctypes.c_void_p(0x1000)
    # gptq_dequant_matvec(packed, bits, rows, n, scales, zeros, gsize, ngroups,
    #                     g_idx, perm, x, xt, batch, y, ws, ws_bytes, stream)
    assert lib.gptq_dequant_matvec(None, 4, 0, 64, None, None, 32, 2, None, None, None, 0, 1,
                                   None, None, 0, None) == 0
    assert lib.gptq_dequant_matvec(None, 4, 8, 64, None, None, 32, 2, None, None, None, 0, 0,
                                   None, None, 0, None) == 0
    assert lib.gptq_dequant_matvec(p, 5, 8, 64, p, p, 32, 2, None, None, p, 0, 1, p, p, 256,
                                   None) == 2
    assert lib.gptq_dequant_matvec(p, 4, 8, 60, p, p, 32, 2, None, None, p, 0, 1, p, p, 256,
                                   None) == 1
    assert lib.gptq_dequant_matvec(p, 3, 8, 48, p, p, 16, 3, None, None, p, 0, 1, p, p, 256,
                                   None) == 1
    assert lib.gptq_dequant_matvec(p, 4, 8, 64, p, p, 32, 2, p, p, p, 0, 1, p, p, 256,
                                   None) == 1
    assert lib.gptq_dequant_matvec(p, 4, 8, 64, p, p, 32, 2, None, None, p, 7, 1, p, p, 256,
                                   None) == 1
    assert lib.gptq_dequant_matvec(p, 4, 8, 64, p, p, 32, 1, None, None, p, 0, 1, p, p, 256,
                                   None) == 1
    # a workspace too small for the x staging, or none
    assert lib.gptq_dequant_matvec(p, 4, 8, 64, p, p, 32, 2, None, None, p, 0, 4, p, p, 256,
                                   None) == 3
    assert lib.gptq_dequant_matvec(p, 4, 8, 64, p, p, 32, 2, None, None, p, 0, 1, p, None, 0,
                                   None) == 3
    # gptq_gather_columns_u8(src, rows, n, perm, dst, stream)
    assert lib.gptq_gather_columns_u8(None, 0, 64, None, None, None) == 0
    assert lib.gptq_gather_columns_u8(p, 4, 64, p, p, None) == 1  # src == dst
    assert lib.gptq_gather_columns_u8(p, 4, 0, p, ctypes.c_void_p(0x2000), None) == 1


@pytest.fixture(scope="module")
def debug_lib():
    if not os.path.exists(_lib.DEBUG_LIB_PATH):
        from post_weight_quantization_25_b200 import build
        build.build(debug=True)
    return _lib.load(_lib.DEBUG_LIB_PATH)


def test_debug_library_exports_every_declared_symbol(debug_lib):
    for name in _declared():
        assert hasattr(debug_lib, name), name


def test_device_checks_only_in_the_debug_build(lib, debug_lib):
    flags = ctypes.c_uint32(7)
    # release: no checks compiled in (nothing touches the device)
    assert lib.gptq_device_checks(ctypes.byref(flags)) == _lib.GPTQ_ERR_UNSUPPORTED
    assert flags.value == 7
    # debug: argument check before any device call
    assert debug_lib.gptq_device_checks(None) == _lib.GPTQ_ERR_INVALID_ARG
