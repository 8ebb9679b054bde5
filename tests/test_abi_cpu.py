"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects malformed arguments on the host before touching
CUDA (every status below is returned without a device)."""

import ctypes
import os
import re

import pytest

import dequant_gemv_q4_b200 as dq
from dequant_gemv_q4_b200 import build as dqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dqgemv.h")

DQ_OK, DQ_ERR_NULL, DQ_ERR_SHAPE, DQ_ERR_ALIGN, DQ_ERR_WORKSPACE, DQ_ERR_LAYOUT, DQ_ERR_CUDA, DQ_ERR_ARG = range(8)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(dq.LIB_PATH):
        dqbuild.build()
    return dq.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[a-z_ ]*?\b(?:dq_status|size_t|int|const char \*)\s*\*?\s*([a-z_0-9]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_expected_entry_points():
    names = _declared_functions()
    assert set(names) == set(dq.EXPORTED), names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_library_is_built_for_sm_100a_only():
    # the build flags name one target; nothing here may be compiled for another GPU
    assert dqbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert "-ftz=false" in dqbuild.FLAGS


def test_status_strings(lib):
    for code in range(8):
        assert dq.status_string(code).startswith("DQ_")
    assert "unknown" in dq.status_string(99)


P = ctypes.c_void_p
A16 = P(1 << 20)          # a 16-byte aligned dummy address (never dereferenced)
A8 = P((1 << 20) + 8)     # 8-byte aligned, not 16


@pytest.mark.parametrize("args,want", [
    ((None, 0, A16, A16, 16, 256, 1, None, None, 0, None), DQ_ERR_NULL),
    ((A16, 0, None, A16, 16, 256, 1, None, None, 0, None), DQ_ERR_NULL),
    ((A16, 0, A16, None, 16, 256, 1, None, None, 0, None), DQ_ERR_NULL),
    ((A16, 2, A16, A16, 16, 256, 1, None, None, 0, None), DQ_ERR_LAYOUT),
    ((A16, 0, A16, A16, 0, 256, 1, None, None, 0, None), DQ_ERR_SHAPE),
    ((A16, 0, A16, A16, 16, 255, 1, None, None, 0, None), DQ_ERR_SHAPE),
    ((A16, 0, A16, A16, 16, 0, 1, None, None, 0, None), DQ_ERR_SHAPE),
    ((A16, 0, A16, A16, 16, 256, 0, None, None, 0, None), DQ_ERR_SHAPE),
    ((A16, 0, A16, A16, 16, 256, 9, None, None, 0, None), DQ_ERR_SHAPE),
    ((A16, 0, A16, A16, 16, 2 * 1048576, 1, None, None, 0, None), DQ_ERR_SHAPE),
    ((A16, 0, A16, A16, 16, 256, 2, A16, None, 0, None), DQ_ERR_ARG),
    ((A8, 0, A16, A16, 16, 256, 1, None, None, 0, None), DQ_ERR_ALIGN),
    ((A16, 0, A8, A16, 16, 256, 1, None, None, 0, None), DQ_ERR_ALIGN),
    ((A16, 0, A16, P((1 << 20) + 2), 16, 256, 1, None, None, 0, None), DQ_ERR_ALIGN),
])
def test_q4k_gemv_rejects_on_host(lib, args, want):
    assert lib.q4k_gemv(*args) == want


def test_other_entry_points_reject_on_host(lib):
    assert lib.q4k_swiglu_gemv(A16, None, 0, A16, A16, 16, 256, 1, None, 0, None) == DQ_ERR_NULL
    assert lib.q4k_swiglu_gemv(A16, A16, 0, A16, A16, 16, 100, 1, None, 0, None) == DQ_ERR_SHAPE
    assert lib.q8_0_gemv(None, A16, A16, 16, 64, 1, None, 0, None) == DQ_ERR_NULL
    assert lib.q8_0_gemv(A16, A16, A16, 16, 48, 1, None, 0, None) == DQ_ERR_SHAPE
    assert lib.q8_0_gemv(A16, A16, A16, 16, 64, 9, None, 0, None) == DQ_ERR_SHAPE
    assert lib.q8_0_gemv(A8, A16, A16, 16, 64, 1, None, 0, None) == DQ_ERR_ALIGN
    assert lib.q4k_repack_soa(A16, None, 4, 256, None) == DQ_ERR_NULL
    assert lib.q4k_repack_soa(A16, A16, 4, 256, None) == DQ_ERR_ARG          # overlapping
    assert lib.q4k_repack_soa(A16, A8, 4, 256, None) == DQ_ERR_ALIGN
    assert lib.q4k_repack_soa(A16, P(1 << 30), 4, 300, None) == DQ_ERR_SHAPE
    assert lib.q4k_dequant(A16, 5, A16, 4, 256, None) == DQ_ERR_LAYOUT
    assert lib.q4k_dequant(A16, 0, A16, -1, 256, None) == DQ_ERR_SHAPE
    assert lib.q8_0_dequant(None, A16, 4, 32, None) == DQ_ERR_NULL
    assert lib.q8_0_dequant(A16, A16, 4, 33, None) == DQ_ERR_SHAPE
    assert lib.dq_device_error(None, 0, None) == DQ_ERR_NULL


def test_workspace_query_rejects_bad_arguments(lib):
    bad = ctypes.c_size_t(-1).value
    assert lib.dq_workspace_bytes(7, 16, 256, 1, 0) == bad
    assert lib.dq_workspace_bytes(1, 16, 250, 1, 0) == bad
    assert lib.dq_workspace_bytes(1, 16, 256, 2, 1) == bad     # argmax needs B == 1
    assert lib.dq_workspace_bytes(2, 16, 256, 1, 1) == bad     # no argmax for SwiGLU
    assert lib.dq_workspace_bytes(0, 16, 64, 1, 0) == 0        # Q8_0 needs no scratch


def test_binding_raises_loudly_without_the_library(tmp_path):
    # The binding has no CPU path: a missing library is an error, not a fallback.
    missing = str(tmp_path / "libdqgemv.so")
    saved = dq._lib
    try:
        dq._lib = None
        with pytest.raises(RuntimeError, match="no CPU fallback"):
            dq.load_library(missing)
    finally:
        dq._lib = saved


def test_split_qg_rejects_on_host(lib):
    f = lib.q4k_gemv_split_qg
    A16b = P((1 << 20) + (1 << 16))
    # null outputs, a head that does not divide N, an unaligned G, overlapping Q and G
    assert f(A16, 0, A16, None, A16b, 512, 256, 1, 64, None, 0, None) == DQ_ERR_NULL
    assert f(A16, 0, A16, A16, A16b, 512, 256, 1, 96, None, 0, None) == DQ_ERR_SHAPE
    assert f(A16, 0, A16, A16, A16b, 512, 256, 1, 0, None, 0, None) == DQ_ERR_SHAPE
    assert f(A16, 0, A16, A16, P((1 << 20) + (1 << 16) + 2), 512, 256, 1, 64, None, 0, None) == DQ_ERR_ALIGN
    assert f(A16, 0, A16, A16, P((1 << 20) + 512), 512, 256, 1, 64, None, 0, None) == DQ_ERR_ARG
    # and the shared Q4_K checks still apply (K not a multiple of 256)
    assert f(A16, 0, A16, A16, A16b, 512, 100, 1, 64, None, 0, None) == DQ_ERR_SHAPE


def test_group_rejects_on_host(lib):
    f = lib.q4k_gemv_group
    W = (P * 2)(A16, A16)
    Y = (P * 2)(A16, A16)
    N = (ctypes.c_int64 * 2)(64, 32)
    assert f(0, W, N, Y, 0, A16, 256, None, 0, None) == DQ_ERR_ARG
    assert f(5, W, N, Y, 0, A16, 256, None, 0, None) == DQ_ERR_ARG
    assert f(2, None, N, Y, 0, A16, 256, None, 0, None) == DQ_ERR_NULL
    assert f(2, (P * 2)(A16, None), N, Y, 0, A16, 256, None, 0, None) == DQ_ERR_NULL
    assert f(2, W, (ctypes.c_int64 * 2)(64, 0), Y, 0, A16, 256, None, 0, None) == DQ_ERR_SHAPE
    assert f(2, (P * 2)(A16, A8), N, Y, 0, A16, 256, None, 0, None) == DQ_ERR_ALIGN
    assert f(2, W, N, (P * 2)(A16, P((1 << 20) + 2)), 0, A16, 256, None, 0, None) == DQ_ERR_ALIGN
    assert f(2, W, N, Y, 0, A16, 100, None, 0, None) == DQ_ERR_SHAPE
    assert f(2, W, N, Y, 7, A16, 256, None, 0, None) == DQ_ERR_LAYOUT


def test_prefill_rejects_on_host(lib):
    f = lib.q4k_prefill_gemm
    f.argtypes = [P, ctypes.c_int, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_size_t, P]
    assert f(None, 0, A16, A16, 128, 256, 16, None, 0, None) == DQ_ERR_NULL
    assert f(A16, 0, None, A16, 128, 256, 16, None, 0, None) == DQ_ERR_NULL
    assert f(A16, 2, A16, A16, 128, 256, 16, None, 0, None) == DQ_ERR_LAYOUT
    assert f(A16, 0, A16, A16, 128, 100, 16, None, 0, None) == DQ_ERR_SHAPE    # K not a multiple of 256
    assert f(A16, 0, A16, A16, 0, 256, 16, None, 0, None) == DQ_ERR_SHAPE      # N < 1
    assert f(A16, 0, A16, A16, 128, 256, 0, None, 0, None) == DQ_ERR_SHAPE     # M < 1
    assert f(A16, 0, A16, A16, 128, 256, 65537, None, 0, None) == DQ_ERR_SHAPE
    assert f(A16, 0, A16, P((1 << 20) + 4), 128, 256, 16, None, 0, None) == DQ_ERR_ALIGN   # y needs 16 B
    assert f(A16, 0, A8, A16, 128, 256, 16, None, 0, None) == DQ_ERR_ALIGN
    bad = ctypes.c_size_t(-1).value
    assert lib.dq_workspace_bytes(3, 128, 250, 16, 0) == bad
    assert lib.dq_workspace_bytes(3, 128, 256, 16, 1) == bad                    # no argmax


def test_residual_gemv_rejects_on_host(lib):
    f = lib.q4k_gemv_residual
    f.argtypes = [P, ctypes.c_int, P, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, P, P, ctypes.c_size_t, P]
    assert f(A16, 0, A16, None, A16, 64, 256, 1, None, None, 0, None) == DQ_ERR_NULL
    assert f(A16, 0, A16, P((1 << 20) + 2), A16, 64, 256, 1, None, None, 0, None) == DQ_ERR_ALIGN
    # the GEMV's own checks still apply
    assert f(A16, 0, A16, A16, A16, 64, 100, 1, None, None, 0, None) == DQ_ERR_SHAPE
    assert f(A16, 0, A16, A16, A16, 64, 256, 9, None, None, 0, None) == DQ_ERR_SHAPE


def test_ffn_block_rejects_on_host(lib):
    f = lib.q4k_ffn_block
    f.argtypes = [P, P, P, ctypes.c_int, P, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, P,
                  ctypes.c_size_t, P]
    assert f(A16, None, A16, 0, A16, None, A16, 256, 512, 1, A16, 1 << 20, None) == DQ_ERR_NULL
    assert f(A16, A16, A16, 3, A16, None, A16, 256, 512, 1, A16, 1 << 20, None) == DQ_ERR_LAYOUT
    assert f(A16, A16, A16, 0, A16, None, A16, 256, 500, 1, A16, 1 << 20, None) == DQ_ERR_SHAPE
    assert f(A16, A16, A16, 0, A16, None, A16, 256, 512, 9, A16, 1 << 20, None) == DQ_ERR_SHAPE
    assert f(A16, A16, A8, 0, A16, None, A16, 256, 512, 1, A16, 1 << 20, None) == DQ_ERR_ALIGN
    assert f(A16, A16, A16, 0, A16, P((1 << 20) + 2), A16, 256, 512, 1, A16, 1 << 20, None) == DQ_ERR_ALIGN
    bad = ctypes.c_size_t(-1).value
    assert lib.dq_workspace_bytes(4, 256, 512, 1, 1) == bad        # no argmax


def test_lost_copy_test_entry_rejects_on_host(lib):
    # wait limits outside 1 us .. 2 s are refused before anything else is looked at
    assert lib.dq_test_lost_copy(None, None, None, 64, 1024, 10, None, 0, None) == 7
    assert lib.dq_test_lost_copy(None, None, None, 64, 1024, 3_000_000_000, None, 0, None) == 7
    # then the q4k_gemv checks: null pointers
    assert lib.dq_test_lost_copy(None, None, None, 64, 1024, 1_000_000, None, 0, None) == 1
