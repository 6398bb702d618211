"""Host-side checks of the C ABI that need no GPU: the library loads, it
exports every entry point the public header declares, and argument errors
come back as status codes before anything is enqueued."""

import ctypes as C
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    import dequantize_absmax_reduce_b200 as m
    return m._bq


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "bq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for must in ("bq_quantize_per_tensor", "bq_quantize_per_channel", "bq_quantize_per_token",
                 "bq_quantize_per_group", "bq_dequantize_per_group", "bq_fake_quantize",
                 "bq_quantize_per_group_backward", "bq_fake_quantize_backward",
                 "bq_dequantize_per_token_backward", "bq_nvfp4_quantize", "bq_nvfp4_dequantize",
                 "bq_mxfp8_quantize", "bq_fp8_block_quantize", "bq_packed_transpose",
                 "bq_packed_transpose_concat", "bq_nvfp4_concat_rows", "bq_nvfp4_predequant_to_fp8"):
        assert must in names


def test_library_exports_every_declared_symbol(B):
    lib = C.CDLL(B.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_misc_host_functions(B):
    assert B.bq_default_q_range(torch.int8) == (-128, 127)
    assert B.bq_default_q_range(torch.uint8) == (0, 255)
    assert B.bq_default_q_range("s4") == (-8, 7) and B.bq_default_q_range("u4") == (0, 15)
    assert [B.bq_granularity_name(g) for g in ("tensor", "channel", "group")] == ["tensor", "channel", "group"]
    assert B.lib.bq_granularity_name(7) is None
    assert B.bq_packed_transpose_stride(4097, 16) == 4112
    assert B.bq_packed_transpose_stride(4096, 16) == 4096
    assert B.bq_packed_transpose_stride(5, 1) == 5
    assert B.bq_packed_transpose_stride(-1, 16) == -1 and B.bq_packed_transpose_stride(5, 0) == -1
    assert B.bq_status_string(0) == "ok"


def test_group_count_matches_reading(B):
    d = B.make_desc((4, 6, 10), torch.float32)
    assert B.bq_group_count(d, "tensor") == (1, 240)
    assert B.bq_group_count(d, "channel", 0) == (4, 60)
    assert B.bq_group_count(d, "channel", 2) == (240, 1)
    assert B.bq_group_count(d, "group", 1, 3) == (8, 30)
    assert B.bq_group_count(d, "group", 2, 5) == (48, 5)
    # column groups: one per (outer, block, inner index), gs elements each
    assert B.bq_group_count(d, "column_group", 1, 3) == (4 * 2 * 10, 3)
    assert B.bq_group_count(d, "column_group", 0, 2) == (2 * 60, 2)
    assert B.bq_group_count(d, "column_group", 2, 5) == B.bq_group_count(d, "group", 2, 5)
    assert B.bq_granularity_name("column_group") == "column_group"
    with pytest.raises(B.BqError):
        B.bq_group_count(d, "column_group", 1, 4)
    with pytest.raises(B.BqError):
        B.bq_group_count(d, "group", 1, 4)          # 4 does not divide 6
    with pytest.raises(B.BqError):
        B.bq_group_count(d, "channel", 3)


def test_workspace_size(B):
    d = B.make_desc((8192, 4096), torch.bfloat16)
    assert B.bq_quantize_workspace_size(d, "channel", 0) == 0          # one pass per row
    assert B.bq_quantize_workspace_size(d, "tensor") == 16             # two passes
    assert B.bq_quantize_workspace_size(d, "group", 1, 128, "static") == 0
    assert B.bq_quantize_workspace_size(d, "group", 1, 128, "from_range") == 16 * 8192 * 32
    d64 = B.make_desc((8, 64), torch.float64)
    assert B.bq_quantize_workspace_size(d64, "channel", 0) == 16 * 8
    drh = B.make_desc((8, 64), torch.float32, rnd="rhaz")
    assert B.bq_quantize_workspace_size(drh, "channel", 0) == 16 * 8
    for mode in ("dynamic", "static"):                          # one pass, no records
        assert B.bq_quantize_workspace_size(d, "column_group", 0, 128, mode) == 0
    assert B.bq_quantize_workspace_size(d, "column_group", 0, 128, "from_range") == 16 * 64 * 4096


def _status(fn):
    try:
        fn()
    except Exception as e:  # BqError
        return getattr(e, "status", None)
    return 0


def test_argument_errors_return_status_without_launching(B):
    P = 0x10000  # never dereferenced: every call below fails validation first
    d = B.make_desc((4, 64), torch.float32)
    st = lambda: B.lib.bq_quantize_per_token(None, C.byref(d), P, P, P, 0, None, 0, None)
    assert st() == B.BQ_ERR_INVALID_ARG                              # null x
    du = B.make_desc((4, 64), torch.float32, torch.uint8, symmetric=True)
    assert B.lib.bq_quantize_per_token(P, C.byref(du), P, P, P, 0, None, 0, None) == B.BQ_ERR_UNSUPPORTED
    dq = B.make_desc((4, 64), torch.float32, qmin=5, qmax=5)
    assert B.lib.bq_quantize_per_token(P, C.byref(dq), P, P, P, 0, None, 0, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_quantize_per_group(P, C.byref(d), 1, 48, P, P, P, 0, None, 0, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_quantize_per_channel(P, C.byref(d), 2, P, P, P, 0, None, 0, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_quantize_per_token(P + 1, C.byref(d), P, P, P, 0, None, 0, None) == B.BQ_ERR_MISALIGNED
    assert B.lib.bq_quantize_per_token(P, C.byref(d), P, P, P, 9, None, 0, None) == B.BQ_ERR_INVALID_ARG
    # FROM_RANGE without a large enough range buffer
    assert B.lib.bq_quantize_per_token(P, C.byref(d), P, P, P, 2, P, 16, None) == B.BQ_ERR_INVALID_ARG
    # asymmetric static scale without a zero-point
    da = B.make_desc((4, 64), torch.float32, torch.uint8, symmetric=False)
    assert B.lib.bq_quantize_per_token(P, C.byref(da), P, P, None, 1, None, 0, None) == B.BQ_ERR_INVALID_ARG
    # dtype errors
    dbad = B.make_desc((4, 64), B.BQ_E4M3)
    assert B.lib.bq_quantize_per_token(P, C.byref(dbad), P, P, P, 0, None, 0, None) == B.BQ_ERR_UNSUPPORTED
    assert B.lib.bq_dequantize_per_token(P, P, None, C.byref(d), P, B.BQ_S8, None) == B.BQ_ERR_UNSUPPORTED
    # backward of an asymmetric code without a zero-point
    assert B.lib.bq_quantize_per_token_backward(P, P, P, None, C.byref(da), P, None) == B.BQ_ERR_INVALID_ARG
    # microscaled formats
    assert B.lib.bq_nvfp4_quantize(P, B.BQ_BF16, 4, 24, P, P, P, 0, P, 16, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_nvfp4_quantize(P, B.BQ_BF16, 4, 32, P, P, P, 0, None, 0, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_nvfp4_quantize(P, B.BQ_F64, 4, 32, P, P, P, 1, None, 0, None) == B.BQ_ERR_UNSUPPORTED
    assert B.lib.bq_mxfp8_quantize(P, B.BQ_BF16, 4, 48, P, P, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_fp8_block_quantize(P, B.BQ_BF16, 4, 256, 64, 128, P, P, None) == B.BQ_ERR_UNSUPPORTED
    assert B.lib.bq_fp8_block_quantize(P, B.BQ_BF16, -1, 256, 1, 128, P, P, None) == B.BQ_ERR_INVALID_ARG
    st64 = B._I64()
    assert B.lib.bq_packed_transpose(P, P, 4, 31, 16, 16, P, P, C.byref(st64), None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_packed_transpose(P, P, 4, 32, 5, 16, P, P, C.byref(st64), None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_packed_transpose(P, None, 4, 32, 16, 16, P, P, C.byref(st64), None) == B.BQ_ERR_INVALID_ARG
    # column groups: no range records, group_size must divide the axis
    dc = B.make_desc((64, 48), torch.float32)
    # FROM_RANGE without a large enough record buffer
    assert B.lib.bq_quantize_per_column_group(P, C.byref(dc), 0, 16, P, P, P, 2, P, 16, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_quantize_per_column_group(P, C.byref(dc), 0, 48, P, P, P, 0, None, 0, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_quantize_per_column_group(P, C.byref(dc), 2, 1, P, P, P, 0, None, 0, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_quantize_per_column_group(P + 2, C.byref(dc), 0, 16, P, P, P, 0, None, 0, None) == B.BQ_ERR_MISALIGNED
    assert B.lib.bq_group_range(P + 2, C.byref(dc), B.BQ_GRAN_COLUMN_GROUP, 0, 16, P, None) == B.BQ_ERR_MISALIGNED
    assert B.lib.bq_dequantize_per_column_group(P, P, None, C.byref(dc), 0, 48, P, B.BQ_F32, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_quantize_per_column_group_backward(P, P, P, None, C.byref(da), 0, 3, P, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_dequantize_per_column_group_backward(P, P, C.byref(dc), 0, 5, P, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_quantize_dynamic_noalloc(P, C.byref(dc), 9, 0, 16, P, P, P, None) == B.BQ_ERR_INVALID_ARG
    # s4 / u4: packed codes need whole vectors and aligned tensors
    d4 = B.make_desc((4, 7), torch.float32, "s4")
    assert B.lib.bq_quantize_per_token(P, C.byref(d4), P, P, P, 0, None, 0, None) == B.BQ_ERR_UNSUPPORTED
    d4 = B.make_desc((4, 12), torch.bfloat16, "s4")                 # 12 % 8: not whole bf16 vectors
    assert B.lib.bq_quantize_per_token(P, C.byref(d4), P, P, P, 0, None, 0, None) == B.BQ_ERR_UNSUPPORTED
    d4 = B.make_desc((4, 16), torch.bfloat16, "u4", symmetric=True)
    assert B.lib.bq_quantize_per_token(P, C.byref(d4), P, P, P, 0, None, 0, None) == B.BQ_ERR_UNSUPPORTED
    d4 = B.make_desc((4, 16), torch.bfloat16, "s4")
    assert B.lib.bq_quantize_per_token(P, C.byref(d4), P + 8, P, P, 0, None, 0, None) == B.BQ_ERR_MISALIGNED
    assert B.lib.bq_dequantize_per_token(P + 4, P, None, C.byref(d4), P, B.BQ_BF16, None) == B.BQ_ERR_MISALIGNED
    # descriptor errors
    d9 = B.make_desc((4, 64), torch.float32)
    d9.ndim = 9
    assert B.lib.bq_quantize_per_token(P, C.byref(d9), P, P, P, 0, None, 0, None) == B.BQ_ERR_INVALID_ARG
    dneg = B.make_desc((4, 64), torch.float32)
    dneg.shape[0] = -4
    assert B.lib.bq_quantize_per_token(P, C.byref(dneg), P, P, P, 0, None, 0, None) == B.BQ_ERR_INVALID_ARG


def test_wait_diagnostic_refuses_out_of_range_tries(B):
    # Checked before any launch, so it runs without a device.
    assert B.lib.bq_diag_wait_timeout(0, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_diag_wait_timeout((1 << 20) + 1, None) == B.BQ_ERR_INVALID_ARG


def test_empty_calls_succeed_without_a_device(B):
    # Nothing to enqueue: an empty tensor returns OK before any CUDA call.
    d = B.make_desc((0, 64), torch.float32)
    assert B.lib.bq_quantize_per_token(None, C.byref(d), None, None, None, 0, None, 0, None) == B.BQ_OK
    assert B.lib.bq_dequantize_per_token(None, None, None, C.byref(d), None, B.BQ_F32, None) == B.BQ_OK
    assert B.lib.bq_mxfp8_quantize(None, B.BQ_BF16, 0, 64, None, None, None) == B.BQ_OK
    assert B.lib.bq_quantize_per_column_group(None, C.byref(d), 0, 1, None, None, None, 0, None, 0, None) == B.BQ_OK
    assert B.lib.bq_dequantize_per_column_group(None, None, None, C.byref(d), 1, 4, None, B.BQ_F32, None) == B.BQ_OK


def test_weight_prep_argument_errors(B):
    P = C.c_void_p(16)
    NP = (C.c_int64 * 1)(4)
    WP = (C.c_void_p * 1)(16)
    st = C.c_int64()
    # no parts, odd k, scales without sc_t
    assert B.lib.bq_packed_transpose_concat(0, WP, None, NP, 32, 16, 1, P, None, C.byref(st), None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_packed_transpose_concat(1, WP, None, NP, 31, 16, 1, P, None, C.byref(st), None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_packed_transpose_concat(1, WP, WP, NP, 32, 16, 1, P, None, C.byref(st), None) == B.BQ_ERR_INVALID_ARG
    # different per-tensor scales (bit patterns), k not a multiple of 16
    s2o = C.c_float()
    assert B.lib.bq_nvfp4_concat_rows(P, P, 1.0, 2, P, P, 1.0000001, 2, 32, P, P, C.byref(s2o), None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_nvfp4_concat_rows(P, P, 0.0, 2, P, P, -0.0, 2, 32, P, P, C.byref(s2o), None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_nvfp4_concat_rows(P, P, 1.0, 2, P, P, 1.0, 2, 24, P, P, C.byref(s2o), None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_nvfp4_predequant_to_fp8(P, P, P, 4, 24, P, None) == B.BQ_ERR_INVALID_ARG
    assert B.lib.bq_nvfp4_predequant_to_fp8(None, P, P, 4, 32, P, None) == B.BQ_ERR_INVALID_ARG
    # zero-sized calls succeed without touching the device
    assert B.lib.bq_nvfp4_concat_rows(None, None, 1.0, 0, None, None, 1.0, 0, 32, None, None, C.byref(s2o), None) == B.BQ_OK
    assert s2o.value == 1.0


def test_gemm_and_diagnostic_argument_errors(B):
    # Every call below fails validation (or is empty) before any CUDA call.
    P = 0x10000
    L = B.lib
    # fused-prologue GEMM: dtypes, k, sizes, operand outputs, alignment
    assert L.bq_fp8_block_gemm(P, B.BQ_F32, 4, 128, P, P, 16, P, B.BQ_F32, None, None, None) == B.BQ_ERR_UNSUPPORTED
    assert L.bq_fp8_block_gemm(P, B.BQ_BF16, 4, 128, P, P, 16, P, B.BQ_F16, None, None, None) == B.BQ_ERR_UNSUPPORTED
    assert L.bq_fp8_block_gemm(P, B.BQ_BF16, 4, 100, P, P, 16, P, B.BQ_F32, None, None, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_fp8_block_gemm(P, B.BQ_BF16, -1, 128, P, P, 16, P, B.BQ_F32, None, None, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_fp8_block_gemm(P, B.BQ_BF16, 4, 128, P, P, 16, P, B.BQ_F32, P, None, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_fp8_block_gemm(P + 2, B.BQ_BF16, 4, 128, P, P, 16, P, B.BQ_F32, None, None, None) == B.BQ_ERR_MISALIGNED
    assert L.bq_fp8_block_gemm(None, B.BQ_BF16, 0, 128, None, None, 16, None, B.BQ_F32, None, None, None) == B.BQ_OK
    # the same product on quantized activations
    assert L.bq_fp8_block_gemm_quantized(P, P, 4, 128, P, P, 16, P, B.BQ_F16, None) == B.BQ_ERR_UNSUPPORTED
    assert L.bq_fp8_block_gemm_quantized(P, P, 4, 100, P, P, 16, P, B.BQ_F32, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_fp8_block_gemm_quantized(P, None, 4, 128, P, P, 16, P, B.BQ_F32, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_fp8_block_gemm_quantized(P + 8, P, 4, 128, P, P, 16, P, B.BQ_F32, None) == B.BQ_ERR_MISALIGNED
    assert L.bq_fp8_block_gemm_quantized(None, None, 4, 128, None, None, 0, None, B.BQ_F32, None) == B.BQ_OK
    # the encoder and divider diagnostics
    assert L.bq_diag_encode_f32(P, 8, B.BQ_S8, P, None) == B.BQ_ERR_UNSUPPORTED
    assert L.bq_diag_encode_f32(P, 7, B.BQ_E2M1X2, P, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_diag_encode_f32(P + 4, 8, B.BQ_E4M3, P, None) == B.BQ_ERR_MISALIGNED
    assert L.bq_diag_divide_f32(P, 8, 0.0, 1, P, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_diag_divide_f32(P, 8, 2.0 ** 65, 0, P, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_diag_divide_f32(P, 7, 3.0, 1, P, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_diag_divide_f32(P, 8, 3.0, 2, P, None) == B.BQ_ERR_INVALID_ARG
    assert L.bq_diag_divide_f32(P + 4, 8, 3.0, 1, P, None) == B.BQ_ERR_MISALIGNED
    assert L.bq_diag_divide_f32(None, 0, 3.0, 1, None, None) == B.BQ_OK
