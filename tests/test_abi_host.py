"""Host-side checks of the C ABI: the library loads, exports every symbol
include/bitlinear.h declares, and rejects bad arguments before launching
anything.  No call here reaches the GPU: every case fails a host check that
runs before the first CUDA call (fake device addresses are never touched)."""
import ctypes as C
import os
import re

import pytest

import oracle
import ternary_weight_linear_absmean_b200 as bl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")

A = 0x10000          # fake, 16-byte aligned device address (never dereferenced)
MIS = 0x10004        # fake, misaligned


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bitlinear_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from ternary_weight_linear_absmean_b200 import _build
    _build.build()
    return bl.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(bl.SIGNATURES)


def test_size_functions_match_layout_spec(L):
    for N, K in [(1, 1), (8, 64), (9, 70), (6912, 2560), (640, 2560), (28672, 8192)]:
        assert L.bitlinear_padded_k(K) == (K + 63) // 64 * 64
        assert L.bitlinear_packed_bytes(N, K) == oracle.packed_bytes(N, K)
        assert L.bitlinear_pack_workspace_bytes(N, K) >= 24
    assert L.bitlinear_packed_bytes(0, 5) == 0 and L.bitlinear_packed_bytes(5, -1) == 0


def test_status_strings(L):
    for s in range(11):
        assert bl.status_string(s).startswith("BL_")
    assert "unknown" in bl.status_string(99)


def test_pack_rejects_bad_arguments(L):
    f = L.bitlinear_pack_weights
    ws = L.bitlinear_pack_workspace_bytes(64, 64)
    assert f(None, 64, 64, 1e-5, A, A, A, A, ws, None) == bl.BL_ERR_NULL
    assert f(A, 0, 64, 1e-5, A, A, A, A, ws, None) == bl.BL_ERR_SHAPE
    assert f(A, 64, -3, 1e-5, A, A, A, A, ws, None) == bl.BL_ERR_SHAPE
    assert f(MIS, 64, 64, 1e-5, A, A, A, A, ws, None) == bl.BL_ERR_ALIGN
    assert f(A, 64, 64, -1.0, A, A, A, A, ws, None) == bl.BL_ERR_ARG
    assert f(A, 64, 64, float("nan"), A, A, A, A, ws, None) == bl.BL_ERR_ARG
    assert f(A, 64, 64, 1e-5, A, A, A, A, ws - 1, None) == bl.BL_ERR_WORKSPACE


def test_quant_rejects_bad_arguments(L):
    f = L.bitlinear_quant_act
    assert f(A, bl.BL_BF16, 4, 64, None, A, None) == bl.BL_ERR_NULL
    assert f(A, 7, 4, 64, A, A, None) == bl.BL_ERR_DTYPE
    assert f(A, bl.BL_F32, 0, 64, A, A, None) == bl.BL_ERR_SHAPE
    assert f(A, bl.BL_F32, 4, 17_000_000, A, A, None) == bl.BL_ERR_OVERFLOW
    assert f(A, bl.BL_F32, 4, 64, MIS, A, None) == bl.BL_ERR_ALIGN


def test_forward_rejects_bad_arguments(L):
    f = L.bitlinear_forward
    assert f(A, A, A, None, 1, 8, 64, A, bl.BL_F32, None, None) == bl.BL_ERR_NULL
    assert f(A, A, A, A, 1, 8, 64, A, 3, None, None) == bl.BL_ERR_DTYPE
    assert f(A, A, A, A, 1, 0, 64, A, bl.BL_F32, None, None) == bl.BL_ERR_SHAPE
    assert f(A, A, A, A, 1, 8, 16_909_321, A, bl.BL_F32, None, None) == bl.BL_ERR_OVERFLOW
    assert f(A, A, A, A, 1, 8, 64, MIS, bl.BL_F32, None, None) == bl.BL_ERR_ALIGN
    assert f(A, A, A, A, 1, 8, 64, A, bl.BL_F32, MIS, None) == bl.BL_ERR_ALIGN
    # 127 * K < 2^31 is the exact limit
    assert (2 ** 31) // 127 == 16_909_320


def test_forward_x_supported_query(L):
    # host-side query of the fused forms' limits: M' * Kp <= 160 KiB (every
    # decode kernel) or M' * Kp' <= 184 KiB with Kp' = Kp rounded up to a
    # multiple of 4096 / M' (tensor-core kernel)
    f = L.bitlinear_forward_x_supported
    assert f(1, 2560) == 1
    assert f(16, 10240) == 1                  # 160 KiB exactly
    assert f(16, 11008) == 1                  # 172 KiB: tensor-core kernel only
    assert f(16, 11776) == 1                  # 184 KiB exactly
    assert f(16, 11777) == 0
    assert f(9, 11776) == 1 and f(9, 12032) == 0   # M' = 16
    assert f(8, 23552) == 1 and f(8, 23553) == 0   # Kp' multiple of 512
    assert f(1, 188416) == 1 and f(1, 188417) == 0
    assert f(17, 64) == 0 and f(0, 64) == 0 and f(1, 0) == 0


def test_forward_x_rejects_bad_arguments(L):
    f = L.bitlinear_forward_x
    assert f(A, bl.BL_BF16, A, A, 17, 8, 64, A, bl.BL_F32, None) == bl.BL_ERR_SHAPE   # M > 16
    # activations beyond every decode kernel's shared memory (16 x 12032 B;
    # 16 x 11008 B still fits the tensor-core kernel)
    assert f(A, bl.BL_BF16, A, A, 16, 8, 12032, A, bl.BL_F32, None) == bl.BL_ERR_SHAPE
    assert f(A, bl.BL_BF16, A, A, 8, 8, 24000, A, bl.BL_F32, None) == bl.BL_ERR_SHAPE
    assert f(A, 5, A, A, 1, 8, 64, A, bl.BL_F32, None) == bl.BL_ERR_DTYPE
    assert f(MIS, bl.BL_BF16, A, A, 1, 8, 64, A, bl.BL_F32, None) == bl.BL_ERR_ALIGN
    g = L.bitlinear_forward_x_grouped
    arr = (C.c_void_p * 2)(A, A)
    i64 = (C.c_int64 * 2)(8, 64)
    assert g(0, arr, bl.BL_BF16, arr, arr, 1, i64, i64, arr, bl.BL_F32, None) == bl.BL_ERR_ARG
    assert g(17, arr, bl.BL_BF16, arr, arr, 1, i64, i64, arr, bl.BL_F32, None) == bl.BL_ERR_ARG
    bad = (C.c_void_p * 2)(A, None)
    assert g(2, bad, bl.BL_BF16, arr, arr, 1, i64, i64, arr, bl.BL_F32, None) == bl.BL_ERR_NULL


def test_decode_kernel_setting_is_host_only(L):
    # process-wide choice; no CUDA call behind it
    assert L.bitlinear_get_decode_kernel() == bl.BL_DECODE_AUTO
    for k in (bl.BL_DECODE_TENSOR, bl.BL_DECODE_DP4A, bl.BL_DECODE_TILE, bl.BL_DECODE_LUT, bl.BL_DECODE_AUTO):
        assert L.bitlinear_set_decode_kernel(k) == bl.BL_OK
        assert L.bitlinear_get_decode_kernel() == k
    assert L.bitlinear_set_decode_kernel(7) == bl.BL_ERR_ARG
    assert L.bitlinear_get_decode_kernel() == bl.BL_DECODE_AUTO


def test_rmsnorm_entries_reject_bad_arguments(L):
    f = L.bitlinear_rmsnorm_quant_act
    assert f(A, bl.BL_BF16, None, 1e-6, 4, 64, A, A, None) == bl.BL_ERR_NULL
    assert f(A, 9, A, 1e-6, 4, 64, A, A, None) == bl.BL_ERR_DTYPE
    assert f(A, bl.BL_BF16, A, 1e-6, 0, 64, A, A, None) == bl.BL_ERR_SHAPE
    assert f(A, bl.BL_BF16, MIS, 1e-6, 4, 64, A, A, None) == bl.BL_ERR_ALIGN
    assert f(A, bl.BL_BF16, A, -1.0, 4, 64, A, A, None) == bl.BL_ERR_ARG
    assert f(A, bl.BL_BF16, A, float("inf"), 4, 64, A, A, None) == bl.BL_ERR_ARG
    g = L.bitlinear_forward_x_rmsnorm_grouped
    arr = (C.c_void_p * 2)(A, A)
    i64 = (C.c_int64 * 2)(8, 64)
    assert g(0, arr, bl.BL_BF16, arr, 1e-6, arr, arr, 1, i64, i64, arr, bl.BL_F32, None) == bl.BL_ERR_ARG
    assert g(2, arr, bl.BL_BF16, None, 1e-6, arr, arr, 1, i64, i64, arr, bl.BL_F32, None) == bl.BL_ERR_NULL
    assert g(2, arr, bl.BL_BF16, arr, float("nan"), arr, arr, 1, i64, i64, arr, bl.BL_F32, None) == bl.BL_ERR_ARG
    assert g(2, arr, bl.BL_BF16, arr, 1e-6, arr, arr, 17, i64, i64, arr, bl.BL_F32, None) == bl.BL_ERR_SHAPE
    bad = (C.c_void_p * 2)(A, MIS)
    assert g(2, arr, bl.BL_BF16, bad, 1e-6, arr, arr, 1, i64, i64, arr, bl.BL_F32, None) == bl.BL_ERR_ALIGN


def test_decode_workspace_bytes(L):
    # per problem M * Kp bytes of codes and M fp32 scales, each rounded up
    # to 256 bytes
    f = L.bitlinear_decode_workspace_bytes
    K2 = (C.c_int64 * 2)(64, 100)
    assert f(2, 3, K2) == (256 + 256) + (512 + 256)
    K1 = (C.c_int64 * 1)(11008)
    assert f(1, 16, K1) == 16 * 11008 + 256
    assert f(0, 3, K2) == 0 and f(17, 3, K2) == 0 and f(2, 0, K2) == 0 and f(2, 17, K2) == 0
    assert f(2, 3, None) == 0
    assert f(1, 1, (C.c_int64 * 1)(0)) == 0
    assert f(1, 1, (C.c_int64 * 1)(16_909_321)) == 0


def test_workspace_forms_reject_bad_workspaces(L):
    # checked before any device work
    g = L.bitlinear_forward_x_grouped_ws
    arr = (C.c_void_p * 2)(A, A)
    i64 = (C.c_int64 * 2)(8, 64)
    need = L.bitlinear_decode_workspace_bytes(2, 4, i64)
    assert need > 0
    assert g(2, arr, bl.BL_BF16, arr, arr, 4, i64, i64, arr, bl.BL_F32, None, need, None) == bl.BL_ERR_NULL
    assert g(2, arr, bl.BL_BF16, arr, arr, 4, i64, i64, arr, bl.BL_F32, MIS, need, None) == bl.BL_ERR_ALIGN
    assert g(2, arr, bl.BL_BF16, arr, arr, 4, i64, i64, arr, bl.BL_F32, A, need - 1, None) == bl.BL_ERR_WORKSPACE
    assert g(2, arr, bl.BL_BF16, arr, arr, 17, i64, i64, arr, bl.BL_F32, A, need, None) == bl.BL_ERR_SHAPE
    h = L.bitlinear_forward_x_rmsnorm_grouped_ws
    assert h(2, arr, bl.BL_BF16, None, 1e-6, arr, arr, 4, i64, i64, arr, bl.BL_F32, A, need, None) == bl.BL_ERR_NULL
    assert h(2, arr, bl.BL_BF16, arr, -1.0, arr, arr, 4, i64, i64, arr, bl.BL_F32, A, need, None) == bl.BL_ERR_ARG
    assert h(2, arr, bl.BL_BF16, arr, 1e-6, arr, arr, 4, i64, i64, arr, bl.BL_F32, A, need - 1,
             None) == bl.BL_ERR_WORKSPACE
