"""B200-native DiT joint attention: Python binding of the C ABI in include/dit_attn.h.

The binding only marshals arguments (tensor checks, device pointers, the
current CUDA stream) into ``libdit_attn.so``; every step of the attention
runs in that library's sm_100a kernel.  There is no CPU or PyTorch fallback:
if the library is missing or cannot run, calls raise.

    import attention_dit_attn_b200 as dit
    o, lse = dit.dit_attn_fwd(q, k, v)                    # bf16 [B,H,L,D] on cuda
    o, lse = dit.dit_attn_fwd(q8, k8, v8, q_scale=qs, k_scale=ks, v_scale=vs)  # e4m3
    o, lse = dit.dit_attn_lse_merge([(o0, lse0), (o1, lse1)])   # combine key chunks
    diff, reuse = dit.dit_attn_residual_diff(r_now, r_prev, 0.12)  # step-cache decision
"""
from __future__ import annotations

import ctypes
import math
import os
import re

from . import _build

__all__ = [
    "DIT_ATTN_BF16", "DIT_ATTN_FP8_E4M3", "DitAttnError", "dit_attn_fwd", "dit_attn_fwd_ptr",
    "dit_attn_status_string", "dit_attn_check_device_error", "dit_attn_set_wait_limit_ns",
    "dit_attn_selftest_wait_timeout", "dit_attn_launches_per_call", "dit_attn_lse_merge",
    "dit_attn_lse_merge_ptr", "DIT_ATTN_MERGE_MAX_PARTS", "dit_attn_residual_diff",
    "dit_attn_residual_diff_ptr", "dit_attn_residual_diff_workspace_bytes", "dit_attn_residual_diff_noalloc",
    "dit_attn_mxfp4_quantize", "dit_attn_mxfp4_quantize_ptr", "dit_attn_block_transpose",
    "dit_attn_absmax_rows", "dit_attn_quantize_e4m3_rows", "dit_attn_fwd_ulysses", "dit_attn_fwd_ulysses_ptr",
    "dit_attn_ulysses_check_device_error", "dit_attn_gemm_fp8", "dit_attn_gemm_fp8_ptr",
    "dit_attn_gemm_check_device_error", "dit_attn_mxfp4_tiled_scale_bytes", "dit_attn_mxfp4_tile_scales",
    "dit_attn_gemm_mxfp4", "dit_attn_gemm_mxfp4_ptr",
    "ensure_built", "lib",
    "header_functions", "STATUS",
]

DIT_ATTN_BF16 = 0
DIT_ATTN_FP8_E4M3 = 1
DIT_ATTN_MERGE_MAX_PARTS = 8

STATUS = {
    0: "DIT_ATTN_OK", 1: "DIT_ATTN_ERR_NULL", 2: "DIT_ATTN_ERR_SHAPE", 3: "DIT_ATTN_ERR_DTYPE",
    4: "DIT_ATTN_ERR_ALIGN", 5: "DIT_ATTN_ERR_ARCH", 6: "DIT_ATTN_ERR_LAUNCH",
    7: "DIT_ATTN_ERR_TIMEOUT", 8: "DIT_ATTN_ERR_VALUE", 9: "DIT_ATTN_ERR_DEVICE",
}

HEADER = os.path.join(_build.INCLUDE, "dit_attn.h")

_lib = None


class DitAttnError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}{STATUS.get(status, status)}: {dit_attn_status_string(status)}")


def ensure_built() -> str:
    """Build libdit_attn.so in-tree if it is missing or older than its sources."""
    return _build.build()


def lib() -> ctypes.CDLL:
    """Load the C-ABI library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_build.LIB):
            raise RuntimeError(f"{_build.LIB} is missing: run attention_dit_attn_b200.ensure_built()")
        L = ctypes.CDLL(_build.LIB)
        vp, i32, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64
        L.dit_attn_fwd.restype = i32
        L.dit_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float, i32,
                                   vp, vp, vp, vp]
        L.dit_attn_status_string.restype = ctypes.c_char_p
        L.dit_attn_status_string.argtypes = [i32]
        L.dit_attn_check_device_error.restype = i32
        L.dit_attn_check_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.dit_attn_set_wait_limit_ns.restype = None
        L.dit_attn_set_wait_limit_ns.argtypes = [u64]
        L.dit_attn_selftest_wait_timeout.restype = i32
        L.dit_attn_selftest_wait_timeout.argtypes = [u64, vp]
        L.dit_attn_launches_per_call.restype = i32
        L.dit_attn_launches_per_call.argtypes = [i32, i32, i32, i32, i32]
        L.dit_attn_residual_diff_workspace_bytes.restype = ctypes.c_size_t
        L.dit_attn_residual_diff_workspace_bytes.argtypes = [ctypes.c_longlong]
        L.dit_attn_residual_diff.restype = i32
        L.dit_attn_residual_diff.argtypes = [vp, vp, ctypes.c_longlong, ctypes.c_float, vp, ctypes.c_size_t,
                                             vp, vp, vp]
        L.dit_attn_residual_diff_noalloc.restype = i32
        L.dit_attn_residual_diff_noalloc.argtypes = [vp, vp, ctypes.c_longlong, ctypes.c_float, vp, vp, vp]
        L.dit_attn_mxfp4_quantize.restype = i32
        L.dit_attn_mxfp4_quantize.argtypes = [vp, vp, vp, ctypes.c_longlong, i32, vp]
        L.dit_attn_block_transpose.restype = i32
        L.dit_attn_block_transpose.argtypes = [vp, vp, ctypes.c_longlong, ctypes.c_longlong, ctypes.c_longlong, vp]
        L.dit_attn_absmax_rows.restype = i32
        L.dit_attn_absmax_rows.argtypes = [vp, vp, ctypes.c_longlong, ctypes.c_longlong, vp]
        L.dit_attn_quantize_e4m3_rows.restype = i32
        L.dit_attn_quantize_e4m3_rows.argtypes = [vp, vp, vp, vp, ctypes.c_longlong, ctypes.c_longlong, vp]
        L.dit_attn_lse_merge.restype = i32
        L.dit_attn_lse_merge.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), i32, vp, vp,
                                         ctypes.c_longlong, i32, vp]
        L.dit_attn_fwd_ulysses.restype = i32
        L.dit_attn_fwd_ulysses.argtypes = [ctypes.POINTER(vp)] * 5 + [i32] * 6 + [ctypes.c_float, i32, vp, vp, vp,
                                                                                vp]
        L.dit_attn_ulysses_check_device_error.restype = i32
        L.dit_attn_ulysses_check_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.dit_attn_gemm_fp8.restype = i32
        L.dit_attn_gemm_fp8.argtypes = [vp, vp, vp, ctypes.c_longlong, i32, i32, ctypes.c_float, ctypes.c_float, vp]
        L.dit_attn_mxfp4_tiled_scale_bytes.restype = ctypes.c_longlong
        L.dit_attn_mxfp4_tiled_scale_bytes.argtypes = [ctypes.c_longlong, i32]
        L.dit_attn_mxfp4_tile_scales.restype = i32
        L.dit_attn_mxfp4_tile_scales.argtypes = [vp, vp, ctypes.c_longlong, i32, vp]
        L.dit_attn_gemm_mxfp4.restype = i32
        L.dit_attn_gemm_mxfp4.argtypes = [vp, vp, vp, vp, vp, ctypes.c_longlong, i32, i32, vp]
        L.dit_attn_gemm_check_device_error.restype = i32
        L.dit_attn_gemm_check_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/dit_attn.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?(?:\w+\s+)*\w+\s*\**\s*(dit_attn_\w+)\s*\(", text, flags=re.M)


def dit_attn_status_string(status: int) -> str:
    return lib().dit_attn_status_string(int(status)).decode()


def _stream_handle(stream, device=None) -> int:
    import torch
    if stream is None:
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        if raw is not None:
            # The raw handle of torch's current stream, without building a Stream object.
            index = device.index if device is not None and device.index is not None else torch.cuda.current_device()
            return int(raw(index))
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


class _Nothing:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


_NOTHING = _Nothing()


def _on_device(dev):
    """Context that makes ``dev`` current: a no-op when it already is (the common
    case, and a few microseconds less per call)."""
    import torch
    if dev.index is None or dev.index == torch.cuda.current_device():
        return _NOTHING
    return torch.cuda.device(dev)


def _one_device(*tensors):
    """The one CUDA device all given tensors (None entries skipped) live on.  Every
    call runs with that device current and on its stream: the library launches on
    the current device, and a kernel given another GPU's memory would read it
    across the link or fault."""
    import torch
    devs = {t.device for t in tensors if isinstance(t, torch.Tensor)}
    if len(devs) != 1 or next(iter(devs)).type != "cuda":
        raise ValueError("all tensors of one call must be on the same CUDA device, got "
                         + ", ".join(sorted(str(d) for d in devs)))
    return next(iter(devs))


def dit_attn_fwd_ptr(q: int, k: int, v: int, o: int, lse: int | None, B: int, H: int, L: int,
                     D: int, scale: float, dtype: int, q_scale: int | None = None,
                     k_scale: int | None = None, v_scale: int | None = None,
                     stream: int = 0) -> int:
    """Raw C-ABI call with integer device pointers; returns the status code."""
    return lib().dit_attn_fwd(q, k, v, o, lse, B, H, L, D, ctypes.c_float(scale), dtype,
                              q_scale, k_scale, v_scale, stream)


def dit_attn_fwd(q, k, v, o=None, lse=None, *, scale: float | None = None, q_scale=None,
                 k_scale=None, v_scale=None, want_lse: bool = True, stream=None):
    """Attention forward on torch CUDA tensors [B, H, L, D] (bf16, or float8_e4m3fn with
    [B, H] fp32 dequant scales).  Allocates o (bf16) and lse (fp32 [B, H, L]) when not
    given.  Asynchronous on ``stream`` (default: torch's current stream).
    Returns (o, lse); lse is None when want_lse is False and none was given."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [B, H, L, D] tensor")
    if q.shape != k.shape or q.shape != v.shape or not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share shape and dtype")
    B, H, L, D = q.shape
    if q.dtype == torch.bfloat16:
        dtype = DIT_ATTN_BF16
        scales = (None, None, None)
        if q_scale is not None or k_scale is not None or v_scale is not None:
            raise ValueError("scales are only for float8_e4m3fn inputs")
    elif q.dtype == torch.float8_e4m3fn:
        dtype = DIT_ATTN_FP8_E4M3
        scales = []
        for name, s in (("q_scale", q_scale), ("k_scale", k_scale), ("v_scale", v_scale)):
            if s is None or not s.is_cuda or s.dtype != torch.float32 or s.numel() != B * H \
                    or not s.is_contiguous():
                raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor with B*H elements")
            scales.append(s.data_ptr())
    else:
        raise TypeError(f"unsupported dtype {q.dtype}")
    if o is None:
        o = torch.empty((B, H, L, D), dtype=torch.bfloat16, device=q.device)
    elif o.shape != q.shape or o.dtype != torch.bfloat16 or not o.is_contiguous() or not o.is_cuda:
        raise ValueError("o must be a contiguous bf16 CUDA tensor shaped like q")
    if lse is None and want_lse:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    elif lse is not None and (lse.numel() != B * H * L or lse.dtype != torch.float32
                              or not lse.is_contiguous() or not lse.is_cuda):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor with B*H*L elements")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dev = _one_device(q, k, v, o, lse, q_scale, k_scale, v_scale)
    with _on_device(dev):
        rc = dit_attn_fwd_ptr(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              None if lse is None else lse.data_ptr(), B, H, L, D, float(scale), dtype,
                              *scales, stream=_stream_handle(stream, dev))
    if rc != 0:
        raise DitAttnError(rc, "dit_attn_fwd: ")
    return o, lse


def dit_attn_check_device_error(stream=None) -> tuple[int, int]:
    """Synchronise, read and clear the device error word: (status, raw word)."""
    word = ctypes.c_uint32(0)
    rc = lib().dit_attn_check_device_error(_stream_handle(stream), ctypes.byref(word))
    return rc, word.value


def dit_attn_set_wait_limit_ns(ns: int) -> None:
    lib().dit_attn_set_wait_limit_ns(int(ns))


def dit_attn_selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    return lib().dit_attn_selftest_wait_timeout(int(limit_ns), _stream_handle(stream))


def dit_attn_launches_per_call(B: int, H: int, L: int, D: int, dtype: int) -> int:
    return lib().dit_attn_launches_per_call(B, H, L, D, dtype)


def dit_attn_lse_merge_ptr(o_parts: list[int], lse_parts: list[int], o: int, lse: int | None,
                           rows: int, D: int, stream: int = 0) -> int:
    """Raw C-ABI call with integer device pointers; returns the status code."""
    n = len(o_parts)
    if n != len(lse_parts):
        raise ValueError("one lse pointer per partial output")
    op = (ctypes.c_void_p * max(n, 1))(*o_parts)
    lp = (ctypes.c_void_p * max(n, 1))(*lse_parts)
    return lib().dit_attn_lse_merge(op, lp, n, o, lse, rows, D, stream)


def dit_attn_lse_merge(parts, o=None, lse=None, *, want_lse: bool = True, stream=None):
    """Merge partial attention results over disjoint key chunks.

    parts: sequence of (o_c, lse_c) pairs as returned by dit_attn_fwd for the same
    query rows: o_c bf16 [..., D] and lse_c fp32 [...] on CUDA, all of one shape.
    Allocates o and lse when not given (either may be parts[0]'s own tensors, for
    an in-place merge).  Asynchronous on ``stream``.  Returns (o, lse)."""
    import torch
    if not 1 <= len(parts) <= DIT_ATTN_MERGE_MAX_PARTS:
        raise ValueError(f"between 1 and {DIT_ATTN_MERGE_MAX_PARTS} parts")
    o0, l0 = parts[0]
    shape, D = tuple(o0.shape), o0.shape[-1]
    rows = o0.numel() // D
    for oc, lc in parts:
        if not (isinstance(oc, torch.Tensor) and oc.is_cuda and oc.dtype == torch.bfloat16
                and oc.is_contiguous() and tuple(oc.shape) == shape):
            raise ValueError("every partial o must be a contiguous bf16 CUDA tensor of one shape")
        if not (isinstance(lc, torch.Tensor) and lc.is_cuda and lc.dtype == torch.float32
                and lc.is_contiguous() and lc.numel() == rows):
            raise ValueError("every partial lse must be a contiguous fp32 CUDA tensor with one value per row")
    if o is None:
        o = torch.empty(shape, dtype=torch.bfloat16, device=o0.device)
    elif tuple(o.shape) != shape or o.dtype != torch.bfloat16 or not o.is_contiguous() or not o.is_cuda:
        raise ValueError("o must be a contiguous bf16 CUDA tensor shaped like the parts")
    if lse is None and want_lse:
        lse = torch.empty(tuple(l0.shape), dtype=torch.float32, device=o0.device)
    elif lse is not None and (lse.numel() != rows or lse.dtype != torch.float32
                              or not lse.is_contiguous() or not lse.is_cuda):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor with one value per row")
    dev = _one_device(o, lse, *[t for part in parts for t in part])
    with _on_device(dev):
        rc = dit_attn_lse_merge_ptr([oc.data_ptr() for oc, _ in parts], [lc.data_ptr() for _, lc in parts],
                                    o.data_ptr(), None if lse is None else lse.data_ptr(), rows, D,
                                    _stream_handle(stream, dev))
    if rc != 0:
        raise DitAttnError(rc, "dit_attn_lse_merge: ")
    return o, lse


def dit_attn_residual_diff_workspace_bytes(n: int) -> int:
    return int(lib().dit_attn_residual_diff_workspace_bytes(int(n)))


def dit_attn_residual_diff_ptr(cur: int, prev: int, n: int, threshold: float, workspace: int,
                               workspace_bytes: int, diff_out: int | None, reuse_out: int | None,
                               stream: int = 0) -> int:
    """Raw C-ABI call with integer device pointers; returns the status code."""
    return lib().dit_attn_residual_diff(cur, prev, n, ctypes.c_float(threshold), workspace, workspace_bytes,
                                        diff_out, reuse_out, stream)


def dit_attn_residual_diff(cur, prev, threshold: float = 0.12, *, workspace=None, diff=None, reuse=None,
                           stream=None):
    """Step-cache decision on two bf16 CUDA tensors of equal size (the first blocks'
    residual now and at the previous step): relative L1 change and reuse flag, as
    one-element fp32 / int32 CUDA tensors (not synchronised).  ``workspace`` (a zeroed
    uint8 CUDA tensor of dit_attn_residual_diff_workspace_bytes(n) bytes) may be kept
    and passed again; it is allocated zeroed when not given."""
    import torch
    for name, t in (("cur", cur), ("prev", prev)):
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if cur.numel() != prev.numel():
        raise ValueError("cur and prev must have the same number of elements")
    n = cur.numel()
    need = dit_attn_residual_diff_workspace_bytes(n)
    if workspace is None:
        workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=cur.device)
    elif not (workspace.is_cuda and workspace.dtype == torch.uint8 and workspace.is_contiguous()
              and workspace.numel() >= need):
        raise ValueError(f"workspace must be a contiguous uint8 CUDA tensor of at least {need} bytes")
    if diff is None:
        diff = torch.empty(1, dtype=torch.float32, device=cur.device)
    if reuse is None:
        reuse = torch.empty(1, dtype=torch.int32, device=cur.device)
    _require(diff, "diff", (torch.float32,), 1)
    _require(reuse, "reuse", (torch.int32,), 1)
    dev = _one_device(cur, prev, workspace, diff, reuse)
    with _on_device(dev):
        rc = dit_attn_residual_diff_ptr(cur.data_ptr(), prev.data_ptr(), n, float(threshold),
                                        workspace.data_ptr(), workspace.numel(), diff.data_ptr(), reuse.data_ptr(),
                                        _stream_handle(stream, dev))
    if rc != 0:
        raise DitAttnError(rc, "dit_attn_residual_diff: ")
    return diff, reuse


def dit_attn_residual_diff_noalloc(cur, prev, threshold: float = 0.12, *, diff=None, reuse=None, stream=None):
    """dit_attn_residual_diff without a workspace: the library's fixed device scratch is
    used (calls on one device must be ordered).  Returns one-element fp32 / int32 CUDA
    tensors (allocated here when not given; the C call itself allocates nothing)."""
    import torch
    for name, t in (("cur", cur), ("prev", prev)):
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if cur.numel() != prev.numel():
        raise ValueError("cur and prev must have the same number of elements")
    if diff is None:
        diff = torch.empty(1, dtype=torch.float32, device=cur.device)
    if reuse is None:
        reuse = torch.empty(1, dtype=torch.int32, device=cur.device)
    _require(diff, "diff", (torch.float32,), 1)
    _require(reuse, "reuse", (torch.int32,), 1)
    dev = _one_device(cur, prev, diff, reuse)
    with _on_device(dev):
        rc = lib().dit_attn_residual_diff_noalloc(cur.data_ptr(), prev.data_ptr(), cur.numel(),
                                                  ctypes.c_float(threshold), diff.data_ptr(), reuse.data_ptr(),
                                                  _stream_handle(stream, dev))
    if rc != 0:
        raise DitAttnError(rc, "dit_attn_residual_diff_noalloc: ")
    return diff, reuse


def dit_attn_mxfp4_quantize_ptr(x: int, q: int, scales: int, rows: int, K: int, stream: int = 0) -> int:
    """Raw C-ABI call with integer device pointers; returns the status code."""
    return lib().dit_attn_mxfp4_quantize(x, q, scales, rows, K, stream)


def dit_attn_mxfp4_quantize(x, q=None, scales=None, *, stream=None):
    """MXFP4 (1x32 blocks) quantisation of a bf16 CUDA tensor [..., K] (K % 32 == 0).
    Returns (q uint8 [..., K/2] packed E2M1 codes, scales uint8 [..., K/32] E8M0)."""
    import torch
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()):
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    K = x.shape[-1]
    rows = x.numel() // K if K else 0
    lead = tuple(x.shape[:-1])
    if q is None:
        q = torch.empty(lead + (K // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(lead + (K // 32,), dtype=torch.uint8, device=x.device)
    for name, t, cols in (("q", q, K // 2), ("scales", scales, K // 32)):
        if not (t.is_cuda and t.dtype == torch.uint8 and t.is_contiguous() and t.numel() == rows * cols):
            raise ValueError(f"{name} must be a contiguous uint8 CUDA tensor with {rows * cols} elements")
    dev = _one_device(x, q, scales)
    with _on_device(dev):
        rc = dit_attn_mxfp4_quantize_ptr(x.data_ptr(), q.data_ptr(), scales.data_ptr(), rows, K,
                                         _stream_handle(stream, dev))
    if rc != 0:
        raise DitAttnError(rc, "dit_attn_mxfp4_quantize: ")
    return q, scales


def _check(rc: int, what: str):
    if rc != 0:
        raise DitAttnError(rc, what + ": ")


def _require(t, name: str, dtypes=None, numel: int | None = None, nbytes: int | None = None):
    """A caller-provided tensor must be a contiguous CUDA tensor (a host pointer reaching
    a kernel would fault), of one of `dtypes`, with `numel` elements or `nbytes` bytes."""
    import torch
    ok = isinstance(t, torch.Tensor) and t.is_cuda and t.is_contiguous()
    ok = ok and (dtypes is None or t.dtype in dtypes)
    ok = ok and (numel is None or t.numel() == numel)
    ok = ok and (nbytes is None or t.numel() * t.element_size() == nbytes)
    if not ok:
        want = "" if dtypes is None else " of dtype " + "/".join(str(d) for d in dtypes)
        size = "" if numel is None else f" with {numel} elements"
        size += "" if nbytes is None else f" of {nbytes} bytes"
        raise ValueError(f"{name} must be a contiguous CUDA tensor{want}{size}")


def dit_attn_block_transpose(x, R: int, C: int, out=None, *, stream=None):
    """out[c][r] = x[r][c] over an R x C grid of equal contiguous blocks of a CUDA tensor
    (its bytes split into R*C blocks).  Returns a tensor of x's dtype and numel."""
    import torch
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.is_contiguous()):
        raise ValueError("x must be a contiguous CUDA tensor")
    nbytes = x.numel() * x.element_size()
    if R * C == 0 or nbytes % (R * C):
        raise ValueError("x's bytes must split into R*C equal blocks")
    if out is None:
        out = torch.empty_like(x)
    _require(out, "out", nbytes=nbytes)
    dev = _one_device(x, out)
    with _on_device(dev):
        _check(lib().dit_attn_block_transpose(x.data_ptr(), out.data_ptr(), R, C, nbytes // (R * C),
                                              _stream_handle(stream, dev)), "dit_attn_block_transpose")
    return out


def dit_attn_absmax_rows(x, rows: int, out=None, *, stream=None):
    """max |x| of each of `rows` equal rows of a bf16 CUDA tensor -> fp32 [rows]."""
    import torch
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()):
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    if rows < 0 or (rows == 0 and x.numel()) or (rows > 0 and x.numel() % rows):
        raise ValueError("x must split into `rows` equal rows")
    if out is None:
        out = torch.empty(rows, dtype=torch.float32, device=x.device)
    _require(out, "out", (torch.float32,), rows)
    dev = _one_device(x, out)
    with _on_device(dev):
        _check(lib().dit_attn_absmax_rows(x.data_ptr(), out.data_ptr(), rows, x.numel() // max(rows, 1),
                                          _stream_handle(stream, dev)), "dit_attn_absmax_rows")
    return out


def dit_attn_quantize_e4m3_rows(x, amax, q=None, scale=None, *, stream=None):
    """e4m3(x / (amax / 448)) per row (rows = amax.numel()); returns (q float8_e4m3fn like x,
    fp32 dequantisation scales [rows])."""
    import torch
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous()):
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    _require(amax, "amax", (torch.float32,))
    rows = amax.numel()
    if (rows == 0 and x.numel()) or (rows > 0 and x.numel() % rows):
        raise ValueError("x must split into amax.numel() equal rows")
    if q is None:
        q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    if scale is None:
        scale = torch.empty(rows, dtype=torch.float32, device=x.device)
    _require(q, "q", (torch.float8_e4m3fn, torch.uint8), x.numel())
    _require(scale, "scale", (torch.float32,), rows)
    dev = _one_device(x, amax, q, scale)
    with _on_device(dev):
        _check(lib().dit_attn_quantize_e4m3_rows(x.data_ptr(), amax.data_ptr(), q.data_ptr(), scale.data_ptr(),
                                                 rows, x.numel() // max(rows, 1), _stream_handle(stream, dev)),
               "dit_attn_quantize_e4m3_rows")
    return q, scale


def dit_attn_fwd_ulysses_ptr(q: list[int], k: list[int], v: list[int], o: list[int], lse: list[int] | None,
                             rank: int, B: int, H: int, Ls: int, D: int, scale: float, dtype: int,
                             q_scale: int | None = None, k_scale: int | None = None, v_scale: int | None = None,
                             stream: int = 0) -> int:
    """Raw C-ABI call: per-shard integer device pointers (lists of n_ranks); returns the status."""
    n = len(q)
    arr = lambda xs: (ctypes.c_void_p * max(n, 1))(*[ctypes.c_void_p(x) for x in xs])
    return lib().dit_attn_fwd_ulysses(arr(q), arr(k), arr(v), arr(o), None if lse is None else arr(lse), n, rank,
                                      B, H, Ls, D, ctypes.c_float(scale), dtype, q_scale, k_scale, v_scale, stream)


def dit_attn_fwd_ulysses(q_shards, k_shards, v_shards, o_shards, lse_shards=None, *, rank: int,
                         scale: float | None = None, q_scale=None, k_scale=None, v_scale=None, stream=None):
    """Ulysses attention with the exchanges fused into the kernel.  Shard c of each
    list is a contiguous CUDA tensor [B, H, Ls, D] holding tokens c*Ls .. c*Ls + Ls of
    all heads (q/k/v bf16, or float8_e4m3fn with [B, H] fp32 scales of all heads; o bf16;
    lse fp32 [B, H, Ls] or None).  Computes attention over all n*Ls tokens for head group
    `rank` (H/n heads) and writes those heads' rows of every o/lse shard.  The tensors may
    live on other GPUs if their memory is mapped into this context."""
    import torch
    n = len(q_shards)
    if not (len(k_shards) == len(v_shards) == len(o_shards) == n) or (lse_shards is not None and len(lse_shards) != n):
        raise ValueError("one shard of each tensor per rank")
    B, H, Ls, D = q_shards[0].shape
    for t in (*q_shards, *k_shards, *v_shards):
        _require(t, "every q/k/v shard", (q_shards[0].dtype,))
        if t.shape != (B, H, Ls, D):
            raise ValueError("q/k/v shards must all be [B, H, Ls, D]")
    for t in o_shards:
        _require(t, "every o shard", (torch.bfloat16,), B * H * Ls * D)
    if lse_shards is not None:
        for t in lse_shards:
            _require(t, "every lse shard", (torch.float32,), B * H * Ls)
    if q_shards[0].dtype == torch.bfloat16:
        dtype, scales = DIT_ATTN_BF16, (None, None, None)
    elif q_shards[0].dtype == torch.float8_e4m3fn:
        dtype = DIT_ATTN_FP8_E4M3
        scales = []
        for name, s in (("q_scale", q_scale), ("k_scale", k_scale), ("v_scale", v_scale)):
            if s is None or not s.is_cuda or s.dtype != torch.float32 or s.numel() != B * H or not s.is_contiguous():
                raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor with B*H elements")
            scales.append(s.data_ptr())
    else:
        raise TypeError(f"unsupported dtype {q_shards[0].dtype}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if not 0 <= rank < n:
        raise ValueError(f"rank {rank} outside 0..{n - 1}")
    # Peers' shards may live on other GPUs (mapped into this context); the call
    # runs on the device of this rank's own shards, where the scales live too.
    own = [q_shards[rank], k_shards[rank], v_shards[rank], o_shards[rank]]
    dev = _one_device(*own, None if lse_shards is None else lse_shards[rank], q_scale, k_scale, v_scale)
    ptrs = lambda ts: [t.data_ptr() for t in ts]
    with _on_device(dev):
        rc = dit_attn_fwd_ulysses_ptr(ptrs(q_shards), ptrs(k_shards), ptrs(v_shards), ptrs(o_shards),
                                      None if lse_shards is None else ptrs(lse_shards), rank, B, H, Ls, D,
                                      float(scale), dtype, *scales, stream=_stream_handle(stream, dev))
    _check(rc, "dit_attn_fwd_ulysses")


def dit_attn_ulysses_check_device_error(stream=None) -> tuple[int, int]:
    """The fused Ulysses kernel's device error word: synchronise, read, clear: (status, raw word)."""
    word = ctypes.c_uint32(0)
    rc = lib().dit_attn_ulysses_check_device_error(_stream_handle(stream), ctypes.byref(word))
    return rc, word.value


def dit_attn_gemm_fp8_ptr(a: int, w: int, y: int, M: int, N: int, K: int, a_scale: float, w_scale: float,
                          stream: int = 0) -> int:
    """Raw C-ABI call with integer device pointers; returns the status code."""
    return lib().dit_attn_gemm_fp8(a, w, y, M, N, K, ctypes.c_float(a_scale), ctypes.c_float(w_scale), stream)


def dit_attn_gemm_fp8(a, w, a_scale: float, w_scale: float, y=None, *, stream=None):
    """FP8 linear layer y = a_scale * w_scale * (a @ w^T): a [..., K] and w [N, K] float8_e4m3fn
    (or uint8 codes) CUDA tensors, y bf16 [..., N] (allocated when not given).
    Asynchronous on ``stream``."""
    import torch
    for name, t in (("a", a), ("w", w)):
        _require(t, name, (torch.float8_e4m3fn, torch.uint8))
    if w.dim() != 2 or a.shape[-1] != w.shape[1]:
        raise ValueError("w must be [N, K] with K = a.shape[-1]")
    N, K = w.shape
    M = a.numel() // K if K else 0
    if y is None:
        y = torch.empty(tuple(a.shape[:-1]) + (N,), dtype=torch.bfloat16, device=a.device)
    _require(y, "y", (torch.bfloat16,), M * N)
    dev = _one_device(a, w, y)
    with _on_device(dev):
        _check(dit_attn_gemm_fp8_ptr(a.data_ptr(), w.data_ptr(), y.data_ptr(), M, N, K, float(a_scale),
                                     float(w_scale), _stream_handle(stream, dev)), "dit_attn_gemm_fp8")
    return y


def dit_attn_gemm_check_device_error(stream=None) -> tuple[int, int]:
    """The GEMM kernels' device error word: synchronise, read, clear: (status, raw word)."""
    word = ctypes.c_uint32(0)
    rc = lib().dit_attn_gemm_check_device_error(_stream_handle(stream), ctypes.byref(word))
    return rc, word.value


def dit_attn_mxfp4_tiled_scale_bytes(rows: int, K: int) -> int:
    return int(lib().dit_attn_mxfp4_tiled_scale_bytes(int(rows), int(K)))


def dit_attn_mxfp4_tile_scales(scales, K: int, tiled=None, *, stream=None):
    """Plain [rows, K/32] E8M0 scales (uint8 CUDA tensor, as dit_attn_mxfp4_quantize writes
    them) -> the tiled layout dit_attn_gemm_mxfp4 reads (uint8, allocated when not given)."""
    import torch
    _require(scales, "scales", (torch.uint8,))
    if K % 32 or K < 32 or scales.numel() % (K // 32):
        raise ValueError("scales must hold K/32 bytes per row, K a multiple of 32")
    rows = scales.numel() // (K // 32)
    nbytes = dit_attn_mxfp4_tiled_scale_bytes(rows, K)
    if tiled is None:
        tiled = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=scales.device)
    _require(tiled, "tiled", (torch.uint8,))
    if tiled.numel() < nbytes:
        raise ValueError(f"tiled must hold {nbytes} bytes")
    dev = _one_device(scales, tiled)
    with _on_device(dev):
        _check(lib().dit_attn_mxfp4_tile_scales(scales.data_ptr(), tiled.data_ptr(), rows, K,
                                                _stream_handle(stream, dev)), "dit_attn_mxfp4_tile_scales")
    return tiled


def dit_attn_gemm_mxfp4_ptr(a: int, a_scales: int, w: int, w_scales: int, y: int, M: int, N: int, K: int,
                            stream: int = 0) -> int:
    """Raw C-ABI call with integer device pointers; returns the status code."""
    return lib().dit_attn_gemm_mxfp4(a, a_scales, w, w_scales, y, M, N, K, stream)


def dit_attn_gemm_mxfp4(a, a_scales_tiled, w, w_scales_tiled, y=None, *, stream=None):
    """MXFP4 linear layer y = A W^T: a [..., K/2] and w [N, K/2] packed E2M1 codes (uint8 CUDA
    tensors), their scales in the tiled layout (dit_attn_mxfp4_tile_scales); y bf16 [..., N]
    (allocated when not given).  Asynchronous on ``stream``."""
    import torch
    for name, t in (("a", a), ("w", w), ("a_scales_tiled", a_scales_tiled), ("w_scales_tiled", w_scales_tiled)):
        _require(t, name, (torch.uint8,))
    if w.dim() != 2 or a.shape[-1] != w.shape[1]:
        raise ValueError("w must be [N, K/2] with K/2 = a.shape[-1]")
    N, K = w.shape[0], 2 * w.shape[1]
    M = a.numel() // (K // 2) if K else 0
    for name, t, rows in (("a_scales_tiled", a_scales_tiled, M), ("w_scales_tiled", w_scales_tiled, N)):
        if t.numel() < dit_attn_mxfp4_tiled_scale_bytes(rows, K):
            raise ValueError(f"{name} must hold dit_attn_mxfp4_tiled_scale_bytes({rows}, {K}) bytes")
    if y is None:
        y = torch.empty(tuple(a.shape[:-1]) + (N,), dtype=torch.bfloat16, device=a.device)
    _require(y, "y", (torch.bfloat16,), M * N)
    dev = _one_device(a, w, a_scales_tiled, w_scales_tiled, y)
    with _on_device(dev):
        _check(dit_attn_gemm_mxfp4_ptr(a.data_ptr(), a_scales_tiled.data_ptr(), w.data_ptr(),
                                       w_scales_tiled.data_ptr(), y.data_ptr(), M, N, K,
                                       _stream_handle(stream, dev)), "dit_attn_gemm_mxfp4")
    return y
