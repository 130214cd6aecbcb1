"""Host-side checks of the C ABI library (no GPU needed, no kernel launched)."""
import ctypes
import re

import pytest
import torch

import attention_dit_attn_b200 as dit


@pytest.fixture(scope="module")
def L():
    dit.ensure_built()
    return dit.lib()


def test_library_exports_every_header_function(L):
    names = dit.header_functions()
    assert set(names) == {"dit_attn_fwd", "dit_attn_status_string", "dit_attn_check_device_error",
                          "dit_attn_set_wait_limit_ns", "dit_attn_selftest_wait_timeout",
                          "dit_attn_launches_per_call", "dit_attn_lse_merge", "dit_attn_residual_diff",
                          "dit_attn_residual_diff_workspace_bytes", "dit_attn_residual_diff_noalloc",
                          "dit_attn_mxfp4_quantize", "dit_attn_block_transpose", "dit_attn_absmax_rows",
                          "dit_attn_quantize_e4m3_rows", "dit_attn_fwd_ulysses",
                          "dit_attn_ulysses_check_device_error", "dit_attn_gemm_fp8",
                          "dit_attn_gemm_check_device_error", "dit_attn_mxfp4_tiled_scale_bytes",
                          "dit_attn_mxfp4_tile_scales", "dit_attn_gemm_mxfp4"}
    for n in names:
        assert hasattr(L, n), n


def test_header_status_codes_match_binding():
    text = open(dit.HEADER).read()
    codes = dict((name, int(val)) for name, val in re.findall(r"(DIT_ATTN_(?:OK|ERR_\w+))\s*=\s*(\d+)", text))
    assert {v: k for k, v in codes.items()} == dit.STATUS


def test_status_strings(L):
    for code in dit.STATUS:
        s = dit.dit_attn_status_string(code)
        assert s and s != "unknown status"
    assert dit.dit_attn_status_string(99) == "unknown status"


@pytest.mark.parametrize("args,want", [
    ((0, 16, 16, 16, None, 1, 1, 8, 64, 0.1, 0), 1),             # q NULL
    ((16, 16, 16, 0, None, 1, 1, 8, 64, 0.1, 0), 1),             # o NULL
    ((16, 16, 16, 16, None, 1, 1, 8, 64, 0.1, 5), 3),            # bad dtype
    ((16, 16, 16, 16, None, 1, 1, 8, 64, 0.1, 1), 1),            # fp8 without scales
    ((16, 16, 16, 16, None, 1, 1, 8, 64, 0.1, 0, 16), 3),        # bf16 with a scale
    ((16, 16, 16, 16, None, 0, 1, 8, 64, 0.1, 0), 2),            # B = 0
    ((16, 16, 16, 16, None, 1, 1, 0, 64, 0.1, 0), 2),            # L = 0
    ((16, 16, 16, 16, None, 1, 1, 8, 80, 0.1, 0), 2),            # D = 80
    ((16, 16, 16, 16, None, 1 << 20, 1 << 11, 1 << 10, 128, 0.1, 0), 2),  # > 2^40 elements
    ((24, 16, 16, 16, None, 1, 1, 8, 64, 0.1, 0), 4),            # q misaligned
    ((16, 16, 16, 16, 18, 1, 1, 8, 64, 0.1, 0), 4),              # lse misaligned
    ((16, 16, 16, 16, None, 1, 1, 8, 64, float("nan"), 0), 8),   # scale NaN
    ((16, 16, 16, 16, None, 1, 1, 8, 64, -0.5, 0), 8),           # scale < 0
])
def test_argument_validation_before_any_cuda_call(L, args, want):
    assert dit.dit_attn_fwd_ptr(*args) == want


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful without a GPU")
def test_wellformed_call_without_gpu_reports_arch(L):
    assert dit.dit_attn_fwd_ptr(16, 16, 16, 16, None, 1, 1, 8, 64, 0.1, 0) == 5
    assert L.dit_attn_selftest_wait_timeout(1000, None) == 5


def test_launch_accounting(L):
    assert dit.dit_attn_launches_per_call(2, 24, 16896, 128, 0) == 1


def test_python_binding_rejects_cpu_tensors():
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        dit.dit_attn_fwd(x, x, x)


@pytest.mark.parametrize("o_parts,lse_parts,o,rows,D,want", [
    ([0], [16], 16, 4, 128, 1),                 # a part's o NULL
    ([16], [0], 16, 4, 128, 1),                 # a part's lse NULL
    ([16], [16], 0, 4, 128, 1),                 # output NULL
    ([], [], 16, 4, 128, 2),                    # no parts
    ([16] * 9, [16] * 9, 16, 4, 128, 2),        # more than DIT_ATTN_MERGE_MAX_PARTS
    ([16], [16], 16, 4, 96, 2),                 # D not 64 / 128
    ([16], [16], 16, -1, 128, 2),               # negative rows
    ([16], [16], 16, 1 << 34, 128, 2),          # rows * D >= 2^40
    ([24], [16], 16, 4, 128, 4),                # part o not 16-byte aligned
    ([16], [18], 16, 4, 128, 4),                # part lse not 4-byte aligned
    ([16], [16], 8, 4, 128, 4),                 # output not 16-byte aligned
])
def test_lse_merge_argument_validation(L, o_parts, lse_parts, o, rows, D, want):
    assert dit.dit_attn_lse_merge_ptr(o_parts, lse_parts, o, None, rows, D) == want


def test_lse_merge_wellformed_call_without_gpu_reports_arch(L):
    assert dit.dit_attn_lse_merge_ptr([16, 32], [16, 32], 16, 64, 10, 64) == 5


def test_lse_merge_zero_rows_is_a_no_op_even_with_null_buffers(L):
    assert dit.dit_attn_lse_merge_ptr([0, 0], [0, 0], 0, None, 0, 128) == 0


def test_residual_diff_workspace_size(L):
    assert dit.dit_attn_residual_diff_workspace_bytes(0) == 0
    assert dit.dit_attn_residual_diff_workspace_bytes(1) == 16 + 16
    big = dit.dit_attn_residual_diff_workspace_bytes(1 << 34)
    assert big == 16 + 16 * 1184


@pytest.mark.parametrize("args,want", [
    ((0, 16, 64, 0.12, 16, 64, 16, 16), 1),              # cur NULL
    ((16, 16, 64, 0.12, 0, 64, 16, 16), 1),              # workspace NULL
    ((16, 16, 64, 0.12, 16, 64, None, None), 1),         # no output at all
    ((16, 16, 0, 0.12, 16, 64, 16, 16), 2),              # n < 1
    ((16, 16, 64, 0.12, 16, 8, 16, 16), 2),              # workspace too small
    ((24, 16, 64, 0.12, 16, 64, 16, 16), 4),             # cur not 16-byte aligned
    ((16, 16, 64, 0.12, 16, 64, 18, 16), 4),             # diff_out not 4-byte aligned
    ((16, 16, 64, float("nan"), 16, 64, 16, 16), 8),     # NaN threshold
    ((16, 16, 64, 0.12, 16, 64, 16, 16), 5),             # well-formed: no GPU here
])
def test_residual_diff_argument_validation(L, args, want):
    assert dit.dit_attn_residual_diff_ptr(*args) == want


def test_residual_diff_noalloc_rejects_sizes_before_any_cuda_call(L):
    L.dit_attn_residual_diff_noalloc.restype = ctypes.c_int
    L.dit_attn_residual_diff_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong,
                                                 ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert L.dit_attn_residual_diff_noalloc(16, 16, 0, ctypes.c_float(0.12), 16, 16, None) == 2
    assert L.dit_attn_residual_diff_noalloc(16, 16, 1 << 40, ctypes.c_float(0.12), 16, 16, None) == 2
    # well-formed: reaches the device query, which fails here without a GPU
    assert L.dit_attn_residual_diff_noalloc(16, 16, 64, ctypes.c_float(0.12), 16, 16, None) == 5


@pytest.mark.parametrize("args,want", [
    ((16, 16, 16, 4, 48), 2),            # K not a multiple of 32
    ((16, 16, 16, 4, 0), 2),             # K = 0
    ((16, 16, 16, -1, 64), 2),           # negative rows
    ((0, 0, 0, 0, 64), 0),               # zero rows: no-op, pointers unused
    ((0, 16, 16, 4, 64), 1),             # x NULL
    ((24, 16, 16, 4, 64), 4),            # x not 16-byte aligned
    ((16, 16, 16, 4, 64), 5),            # well-formed: no GPU here
])
def test_mxfp4_quantize_argument_validation(L, args, want):
    assert dit.dit_attn_mxfp4_quantize_ptr(*args) == want


def test_ulysses_ops_argument_validation(L):
    vp = ctypes.c_void_p
    L.dit_attn_block_transpose.restype = ctypes.c_int
    L.dit_attn_block_transpose.argtypes = [vp, vp, ctypes.c_longlong, ctypes.c_longlong, ctypes.c_longlong, vp]
    L.dit_attn_absmax_rows.restype = ctypes.c_int
    L.dit_attn_absmax_rows.argtypes = [vp, vp, ctypes.c_longlong, ctypes.c_longlong, vp]
    L.dit_attn_quantize_e4m3_rows.restype = ctypes.c_int
    L.dit_attn_quantize_e4m3_rows.argtypes = [vp, vp, vp, vp, ctypes.c_longlong, ctypes.c_longlong, vp]
    assert L.dit_attn_block_transpose(16, 32, 2, 3, 6, None) == 2          # block bytes not a multiple of 4
    assert L.dit_attn_block_transpose(None, None, 0, 3, 16, None) == 0      # empty: no-op
    assert L.dit_attn_block_transpose(None, 32, 2, 3, 16, None) == 1
    assert L.dit_attn_block_transpose(18, 32, 2, 3, 16, None) == 4          # in not 4-byte aligned
    assert L.dit_attn_block_transpose(16, 32, 2, 3, 16, None) == 5          # well-formed: no GPU here
    assert L.dit_attn_absmax_rows(16, 16, 4, 12, None) == 2                 # row_len not a multiple of 8
    assert L.dit_attn_absmax_rows(16, 16, 4, 64, None) == 5
    assert L.dit_attn_quantize_e4m3_rows(16, 16, 16, None, 4, 24, None) == 2   # row_len not a multiple of 16
    assert L.dit_attn_quantize_e4m3_rows(16, 16, None, None, 4, 64, None) == 1
    assert L.dit_attn_quantize_e4m3_rows(16, 16, 16, None, 4, 64, None) == 5


def test_fused_ulysses_argument_validation(L):
    call = dit.dit_attn_fwd_ulysses_ptr
    two = [16, 16]
    assert call([16], [16], [16], [16], None, 0, 1, 1, 64, 64, 0.1, 0) == 5       # well-formed: no GPU here
    assert call(two, two, two, two, None, 0, 1, 3, 64, 64, 0.1, 0) == 2          # H % n_ranks
    assert call(two, two, two, two, None, 0, 1, 4, 100, 64, 0.1, 0) == 2         # Ls % 64
    assert call(two, two, two, two, None, 2, 1, 4, 64, 64, 0.1, 0) == 2          # rank out of range
    assert call([16] * 9, [16] * 9, [16] * 9, [16] * 9, None, 0, 1, 9, 64, 64, 0.1, 0) == 2   # > 8 ranks
    assert call(two, two, two, [16, 0], None, 0, 1, 4, 64, 64, 0.1, 0) == 1      # a NULL shard
    assert call(two, two, two, two, [16, 0], 0, 1, 4, 64, 64, 0.1, 0) == 1       # LSE for some shards only
    assert call(two, two, [16, 24], two, None, 0, 1, 4, 64, 64, 0.1, 0) == 4     # misaligned shard
    assert call(two, two, two, two, None, 0, 1, 4, 64, 96, 0.1, 0) == 2          # head dim
    assert call(two, two, two, two, None, 0, 1, 4, 64, 64, 0.1, 1) == 1          # FP8 without scales
    assert call(two, two, two, two, None, 0, 1, 4, 64, 64, -1.0, 0) == 8         # negative scale


def test_python_bindings_refuse_host_buffers_before_any_call():
    """Every caller-provided buffer must be a CUDA tensor: a host pointer reaching a kernel
    would fault.  (On this host nothing is a CUDA tensor, so each check fires on the first
    host tensor it meets.)"""
    import attention_dit_attn_b200 as d
    x = torch.zeros(64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        d.dit_attn_block_transpose(x, 2, 2)
    with pytest.raises(ValueError):
        d.dit_attn_absmax_rows(x, 4)
    with pytest.raises(ValueError):
        d.dit_attn_quantize_e4m3_rows(x, torch.ones(4))
    with pytest.raises(ValueError):
        d.dit_attn_residual_diff(x, x)
    with pytest.raises(ValueError):
        d.dit_attn_mxfp4_quantize(x.reshape(2, 32))
    shard = torch.zeros((1, 2, 64, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        d.dit_attn_fwd_ulysses([shard], [shard], [shard], [shard.clone()], rank=0)


def test_require_names_the_buffer_and_its_expected_form():
    import attention_dit_attn_b200 as d
    with pytest.raises(ValueError, match="diff must be a contiguous CUDA tensor of dtype torch.float32 with 1 elements"):
        d._require(torch.zeros(1), "diff", (torch.float32,), 1)


@pytest.mark.parametrize("args,want", [
    ((0, 0, 0, 0, 64, 64, 1.0, 1.0), 0),          # M = 0: no-op, pointers unused
    ((16, 16, 16, 4, 64, 24, 1.0, 1.0), 2),       # K not a multiple of 16
    ((16, 16, 16, 4, 60, 64, 1.0, 1.0), 2),       # N not a multiple of 8
    ((16, 0, 16, 4, 64, 64, 1.0, 1.0), 1),        # w NULL
    ((16, 24, 16, 4, 64, 64, 1.0, 1.0), 4),       # w not 16-byte aligned
    ((16, 16, 16, 4, 64, 64, float("nan"), 1.0), 8),   # non-finite scale
    ((16, 16, 16, 4, 64, 64, 1.0, 1.0), 5),       # well-formed: no GPU here
])
def test_gemm_fp8_argument_validation(L, args, want):
    assert dit.dit_attn_gemm_fp8_ptr(*args) == want


def test_gemm_binding_refuses_host_buffers():
    import attention_dit_attn_b200 as d
    a = torch.zeros((4, 64), dtype=torch.uint8)
    with pytest.raises(ValueError):
        d.dit_attn_gemm_fp8(a, a.clone(), 1.0, 1.0)


def test_mxfp4_tiled_scale_bytes(L):
    import attention_dit_attn_b200 as d
    assert d.dit_attn_mxfp4_tiled_scale_bytes(1, 32) == 1 * 2 * 512
    assert d.dit_attn_mxfp4_tiled_scale_bytes(128, 256) == 1 * 2 * 512
    assert d.dit_attn_mxfp4_tiled_scale_bytes(129, 288) == 2 * 4 * 512
    assert d.dit_attn_mxfp4_tiled_scale_bytes(33792, 3072) == 264 * 24 * 512
    assert d.dit_attn_mxfp4_tiled_scale_bytes(0, 64) == 0
    assert d.dit_attn_mxfp4_tiled_scale_bytes(4, 48) == 0


def test_gemm_mxfp4_argument_validation(L):
    call = dit.dit_attn_gemm_mxfp4_ptr
    assert call(0, 0, 0, 0, 0, 0, 64, 64) == 0                 # M = 0: no-op
    assert call(16, 16, 16, 16, 16, 4, 64, 48) == 2            # K not a multiple of 32
    assert call(16, 16, 16, 16, 16, 4, 60, 64) == 2            # N not a multiple of 8
    assert call(16, 0, 16, 16, 16, 4, 64, 64) == 1             # a_scales NULL
    assert call(16, 24, 16, 16, 16, 4, 64, 64) == 4            # a_scales not 16-byte aligned
    assert call(16, 16, 16, 16, 16, 4, 64, 64) == 5            # well-formed: no GPU here
    L.dit_attn_mxfp4_tile_scales.restype = ctypes.c_int
    L.dit_attn_mxfp4_tile_scales.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int,
                                             ctypes.c_void_p]
    assert L.dit_attn_mxfp4_tile_scales(16, 16, 4, 48, None) == 2
    assert L.dit_attn_mxfp4_tile_scales(None, None, 0, 64, None) == 0
    assert L.dit_attn_mxfp4_tile_scales(16, 24, 4, 64, None) == 4
    assert L.dit_attn_mxfp4_tile_scales(16, 16, 4, 64, None) == 5
