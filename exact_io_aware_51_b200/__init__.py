"""Exact IO-aware attention for B200 (sm_100a): Python binding of ``libfa.so``.

This module only marshals arguments: it checks tensor shapes, dtypes and
devices, allocates outputs with PyTorch (PyTorch is used for device memory and
streams only), and calls the C ABI declared in ``include/fa.h`` through
ctypes.  Every step of the computation runs in the library's CUDA kernels;
there is no CPU fallback.  If the library is missing, every call raises.

    o, lse = fwd(q, k, v, causal=False)          # q, k, v: [B, N, H, d] cuda
    dq, dk, dv = bwd(q, k, v, o, do, lse, causal=False)
"""

from __future__ import annotations

import ctypes
import os
import math
import pathlib

import torch

__all__ = [
    "FAError", "FA_BF16", "FA_FP32", "lib", "lib_path", "fwd", "fwd_fp8", "bwd", "bwd_workspace_size",
    "merge_partial", "accumulate", "cast_bf16", "decode_paged", "decode_workspace_size",
    "last_device_status", "set_wait_limit_ms", "debug_inject", "debug_umma", "debug_umma_f8", "debug_umma_2cta",
    "debug_mma_rate",
    "status_string",
    "set_kernel_events",
    "attention", "EXPORTED",
]

FA_BF16 = 0
FA_FP32 = 1
_PKG = pathlib.Path(__file__).resolve().parent
_LIB = None

# Every symbol include/fa.h declares.
EXPORTED = ("fa_fwd", "fa_bwd_workspace_size", "fa_bwd", "fa_status_string", "fa_last_cuda_error",
            "fa_last_device_status", "fa_set_wait_limit_ms",
            "fa_version", "fa_set_kernel_events", "fa_bwd_static_scratch", "fa_fwd_gqa", "fa_bwd_gqa",
            "fa_fwd_window", "fa_bwd_window", "fa_fwd_fp8",
            "fa_fwd_blocksparse", "fa_bwd_blocksparse", "fa_merge_partial", "fa_accumulate_bf16",
            "fa_cast_bf16", "fa_bwd_workspace_size_gqa", "fa_decode_paged", "fa_decode_workspace_size",
            "fa_fwd_fp8_blocksparse")
# Test-only symbols (csrc/fa_testing.h): the first in libfa.so, the others in the
# separate test library libfa_probe.so.
TESTING_EXPORTED = {"libfa.so": ("fa_debug_inject",),
                    "libfa_probe.so": ("fa_debug_umma", "fa_debug_umma_f8", "fa_debug_umma_2cta",
                                       "fa_debug_mma_rate")}
_PROBE = None


class FAError(RuntimeError):
    """A non-zero status from the C library (``status`` holds the code)."""

    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        msg = status_string(status) if _LIB is not None else f"status {status}"
        if self.status == -6 and _LIB is not None:
            msg += f" (cudaError {_LIB.fa_last_cuda_error()})"
        super().__init__(f"{what}: {msg}" if what else msg)


def lib_path() -> pathlib.Path:
    """The library the binding loads: ``libfa.so``, or the checking build
    ``libfa_debug.so`` (device-side bounds checks, see ``fa_last_device_status``)
    when the environment variable ``FA_LIBRARY`` names it."""
    name = os.environ.get("FA_LIBRARY", "libfa.so")
    if name not in ("libfa.so", "libfa_debug.so"):
        raise FAError(-1, f"FA_LIBRARY={name!r}: expected libfa.so or libfa_debug.so")
    return _PKG / name


def lib() -> ctypes.CDLL:
    """Load ``libfa.so`` (built by ``python -m exact_io_aware_51_b200.build``)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = lib_path()
    if not path.exists():
        raise FAError(-6, f"{path} is missing; build it with `python -m exact_io_aware_51_b200.build`")
    L = ctypes.CDLL(str(path))
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
    L.fa_fwd.restype = i
    L.fa_bwd_workspace_size.argtypes = [i, i, i, i, i]
    L.fa_bwd_workspace_size.restype = sz
    L.fa_bwd_workspace_size_gqa.argtypes = [i, i, i, i, i, i]
    L.fa_bwd_workspace_size_gqa.restype = sz
    L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp, sz, vp]
    L.fa_bwd.restype = i
    L.fa_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    L.fa_fwd_gqa.restype = i
    L.fa_bwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, sz, vp]
    L.fa_bwd_gqa.restype = i
    L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, f, f, i, i, vp]
    L.fa_fwd_fp8.restype = i
    L.fa_fwd_fp8_blocksparse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, f, f, i, i, vp, i, vp]
    L.fa_fwd_fp8_blocksparse.restype = i
    L.fa_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, i, i, vp]
    L.fa_fwd_blocksparse.restype = i
    L.fa_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, i, i, vp, sz, vp]
    L.fa_bwd_blocksparse.restype = i
    L.fa_merge_partial.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    L.fa_merge_partial.restype = i
    L.fa_accumulate_bf16.argtypes = [vp, vp, ctypes.c_longlong, i, vp]
    L.fa_accumulate_bf16.restype = i
    L.fa_cast_bf16.argtypes = [vp, vp, ctypes.c_longlong, vp]
    L.fa_cast_bf16.restype = i
    L.fa_fwd_window.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp]
    L.fa_fwd_window.restype = i
    L.fa_bwd_window.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp, sz, vp]
    L.fa_bwd_window.restype = i
    L.fa_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp, sz, vp]
    L.fa_decode_paged.restype = i
    L.fa_decode_workspace_size.argtypes = [i, i, i, i, i, i]
    L.fa_decode_workspace_size.restype = sz
    L.fa_status_string.argtypes = [i]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_last_cuda_error.argtypes = []
    L.fa_last_cuda_error.restype = i
    L.fa_last_device_status.argtypes = [vp, ctypes.POINTER(i)]
    L.fa_last_device_status.restype = i
    L.fa_set_wait_limit_ms.argtypes = [i]
    L.fa_set_wait_limit_ms.restype = None
    L.fa_debug_inject.argtypes = [i]
    L.fa_debug_inject.restype = None
    L.fa_bwd_static_scratch.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
    L.fa_bwd_static_scratch.restype = i
    L.fa_set_kernel_events.argtypes = [vp, vp]
    L.fa_set_kernel_events.restype = None
    L.fa_version.argtypes = []
    L.fa_version.restype = i
    _LIB = L
    return L


def probe_lib() -> ctypes.CDLL:
    """Load the test library ``libfa_probe.so`` (single MMA tile probes, test-only)."""
    global _PROBE
    if _PROBE is not None:
        return _PROBE
    path = _PKG / "libfa_probe.so"
    if not path.exists():
        raise FAError(-6, f"{path} is missing; build it with `python -m exact_io_aware_51_b200.build`")
    P = ctypes.CDLL(str(path))
    vp, i = ctypes.c_void_p, ctypes.c_int
    P.fa_debug_umma.argtypes = [vp, vp, vp, i, i, i, i, i, vp]
    P.fa_debug_umma.restype = i
    P.fa_debug_umma_f8.argtypes = [vp, vp, vp, i, i, i, vp]
    P.fa_debug_umma_f8.restype = i
    P.fa_debug_umma_2cta.argtypes = [vp, vp, vp, i, i, i, i, vp, vp]
    P.fa_debug_umma_2cta.restype = i
    P.fa_debug_mma_rate.argtypes = [i, i, i, i, i, vp, vp, vp, vp, vp]
    P.fa_debug_mma_rate.restype = i
    _PROBE = P
    return P


def status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float32:
        return FA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _stream_handle(stream, device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _check_inputs(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *qlike: torch.Tensor) -> int:
    """Validate [B, N, H, d] q (and o, do) against [B, N, Hkv, d] k, v; returns Hkv."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("expected [B, N, H, d] tensors")
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    grouped = (Hkv == 0 and H == 0) or (Hkv >= 1 and H % Hkv == 0)  # no heads at all is an empty problem
    if k.shape != (B, N, Hkv, d) or not grouped:
        raise ValueError("k, v must be [B, N, Hkv, d] with Hkv dividing the query heads H")
    for t in (q, k, v, *qlike):
        want = k.shape if t is k or t is v else q.shape
        if t.shape != want or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, o, do must share one shape; k, v another; all one dtype and device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, N, heads, d]")
    if not q.is_cuda:
        raise ValueError("tensors must live on a CUDA device (there is no CPU path)")
    return Hkv


def _scale(scale, d):
    return float(1.0 / math.sqrt(d)) if scale is None else float(scale)


def _window_bounds(causal, window):
    """(left, right) bounds for fa_*_window: None -> -1 (open); causal closes the right side at 0."""
    left, right = window
    for x in (left, right):
        if x is not None and (int(x) != x or x < 0):
            raise ValueError("window bounds must be None or integers >= 0")
    if causal:
        right = 0 if right is None else min(int(right), 0)
    return (-1 if left is None else int(left)), (-1 if right is None else int(right))


def _mask_args(block_mask, q):
    """(pointer, mask_heads) for a uint8 cuda block mask [nb, nb] or [H, nb, nb]."""
    B, N, H, d = q.shape
    nb = (N + 127) // 128
    if block_mask.dtype not in (torch.uint8, torch.bool) or not block_mask.is_contiguous():
        raise ValueError("block_mask must be a contiguous uint8 (or bool) tensor")
    if block_mask.device != q.device:
        raise ValueError("block_mask must live on the device of q")
    if block_mask.shape == (nb, nb):
        return block_mask.data_ptr(), 1
    if block_mask.shape == (H, nb, nb):
        return block_mask.data_ptr(), H
    raise ValueError(f"block_mask must be [{nb}, {nb}] or [{H}, {nb}, {nb}] (128 x 128 blocks)")


def fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None, stream=None,
        window=None, block_mask=None):
    """Forward pass: returns (o [B, N, H, d], lse [B, H, N] fp32).

    k and v may have fewer heads than q (grouped-query attention, fa_fwd_gqa).
    ``window`` = (left, right) restricts query i to keys i - left .. i + right
    (None on a side: open), fa_fwd_window.  ``block_mask`` (uint8 [nb, nb] or
    [H, nb, nb] over 128 x 128 blocks) selects the blocks each query block sees,
    fa_fwd_blocksparse.
    """
    Hkv = _check_inputs(q, k, v)
    B, N, H, d = q.shape
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    tail = (_scale(scale, d), int(bool(causal)), _dtype_code(q), _stream_handle(stream, q.device))
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr())
    if block_mask is not None:
        wl, wr = _window_bounds(causal, (None, None) if window is None else window)
        mp, mh = _mask_args(block_mask, q)
        rc, name = lib().fa_fwd_blocksparse(*ptrs, B, H, Hkv, N, d, tail[0], wl, wr, mp, mh, *tail[2:]), \
            "fa_fwd_blocksparse"
    elif window is not None:
        wl, wr = _window_bounds(causal, window)
        rc, name = lib().fa_fwd_window(*ptrs, B, H, Hkv, N, d, tail[0], wl, wr, *tail[2:]), "fa_fwd_window"
    elif Hkv == H:
        rc, name = lib().fa_fwd(*ptrs, B, H, N, d, *tail), "fa_fwd"
    else:
        rc, name = lib().fa_fwd_gqa(*ptrs, B, H, Hkv, N, d, *tail), "fa_fwd_gqa"
    if rc != 0:
        raise FAError(rc, name)
    return o, l


def fwd_fp8(q, k, v, scale_q: float, scale_k: float, scale_v: float, causal: bool = False,
            scale: float | None = None, window=None, out=None, lse=None, stream=None, block_mask=None):
    """Forward with 8-bit inputs: q [B, N, H, 128], k, v [B, N, Hkv, 128] as torch.float8_e4m3fn
    (or their uint8 codes), each dequantised by its scale; returns (o bf16, lse fp32).
    ``block_mask`` as in ``fwd`` (fa_fwd_fp8_blocksparse)."""
    for t in (q, k, v):
        if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
            raise TypeError("fwd_fp8 takes torch.float8_e4m3fn (or uint8 e4m3 codes)")
    Hkv = _check_inputs(q, k, v)
    B, N, H, d = q.shape
    o = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=q.device) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    wl, wr = _window_bounds(causal, (None, None) if window is None else window)
    mp, mh = _mask_args(block_mask, q) if block_mask is not None else (None, 0)
    rc = lib().fa_fwd_fp8_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(), B, H,
                                      Hkv, N, d, _scale(scale, d), float(scale_q), float(scale_k), float(scale_v),
                                      wl, wr, mp, mh, _stream_handle(stream, q.device))
    if rc != 0:
        raise FAError(rc, "fa_fwd_fp8_blocksparse")
    return o, l


def decode_workspace_size(B: int, H: int, Hkv: int, d: int, page_size: int, max_pages: int) -> int:
    """Workspace bytes with which ``decode_paged`` splits long sequences as it would unconstrained."""
    return int(lib().fa_decode_workspace_size(B, H, Hkv, d, page_size, max_pages))


def decode_paged(q, k_cache, v_cache, block_table, seqlens, scale: float | None = None, out=None, lse=None,
                 workspace=None, stream=None):
    """One decode step over a paged KV cache (fa_decode_paged): returns (o [B, H, d] bf16, lse [B, H] fp32).

    q: [B, H, d] bf16; k_cache, v_cache: [num_pages, page_size, Hkv, d] bf16;
    block_table: [B, max_pages] int32; seqlens: [B] int32; all on one CUDA
    device.  ``workspace`` (uint8 cuda tensor) defaults to a fresh buffer of
    ``decode_workspace_size`` bytes; pass one to avoid the allocation.
    """
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("expected q [B, H, d] and k_cache, v_cache [num_pages, page_size, Hkv, d]")
    B, H, d = q.shape
    num_pages, page_size, Hkv, dk = k_cache.shape
    if v_cache.shape != k_cache.shape or dk != d:
        raise ValueError("k_cache and v_cache must be [num_pages, page_size, Hkv, d] with q's d")
    if block_table.dim() != 2 or block_table.shape[0] != B or seqlens.shape != (B,):
        raise ValueError("block_table must be [B, max_pages] and seqlens [B]")
    for t in (q, k_cache, v_cache):
        if t.dtype != torch.bfloat16:
            raise TypeError("decode_paged takes bfloat16 q, k_cache, v_cache")
    for t in (block_table, seqlens):
        if t.dtype != torch.int32:
            raise TypeError("block_table and seqlens must be int32")
    for t in (q, k_cache, v_cache, block_table, seqlens):
        if not t.is_contiguous():
            raise ValueError("decode_paged tensors must be contiguous")
        if t.device != q.device:
            raise ValueError("decode_paged tensors must share one device")
    if not q.is_cuda:
        raise ValueError("tensors must live on a CUDA device (there is no CPU path)")
    max_pages = block_table.shape[1]
    o = torch.empty((B, H, d), dtype=torch.bfloat16, device=q.device) if out is None else out
    l = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    if workspace is None:
        n = decode_workspace_size(B, H, Hkv, d, page_size, max(max_pages, 1))
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    rc = lib().fa_decode_paged(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(),
                               seqlens.data_ptr(), o.data_ptr(), l.data_ptr(), B, H, Hkv, d, page_size, num_pages,
                               max_pages, _scale(scale, d), workspace.data_ptr(), workspace.numel(),
                               _stream_handle(stream, q.device))
    if rc != 0:
        raise FAError(rc, "fa_decode_paged")
    return o, l


def merge_partial(o_acc, lse_acc, o_part, lse_part, init: bool = False, o_out=None, stream=None):
    """Fold one key chunk's partial result (o_part bf16, lse_part) into (o_acc fp32, lse_acc), in place."""
    B, N, H, d = o_part.shape
    for t, dt in ((o_acc, torch.float32), (lse_acc, torch.float32), (o_part, torch.bfloat16), (lse_part, torch.float32)):
        if t.dtype != dt or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("merge_partial: contiguous cuda tensors (o_acc fp32, o_part bf16, LSEs fp32)")
    if o_acc.shape != o_part.shape or lse_acc.shape != (B, H, N) or lse_part.shape != (B, H, N):
        raise ValueError("merge_partial: shape mismatch")
    rc = lib().fa_merge_partial(o_acc.data_ptr(), lse_acc.data_ptr(), o_part.data_ptr(), lse_part.data_ptr(),
                                None if o_out is None else o_out.data_ptr(), B, H, N, d, int(bool(init)),
                                _stream_handle(stream, o_acc.device))
    if rc != 0:
        raise FAError(rc, "fa_merge_partial")


def accumulate(acc, part, init: bool = False, stream=None):
    """acc (fp32) += part (bf16), or acc = part with init; same shapes, contiguous cuda tensors."""
    if acc.dtype != torch.float32 or part.dtype != torch.bfloat16 or acc.shape != part.shape:
        raise ValueError("accumulate: fp32 accumulator and bf16 part of one shape")
    if not (acc.is_cuda and part.is_cuda and acc.is_contiguous() and part.is_contiguous()):
        raise ValueError("accumulate: contiguous cuda tensors")
    rc = lib().fa_accumulate_bf16(acc.data_ptr(), part.data_ptr(), acc.numel(), int(bool(init)),
                                  _stream_handle(stream, acc.device))
    if rc != 0:
        raise FAError(rc, "fa_accumulate_bf16")


def cast_bf16(x, out=None, stream=None):
    """bf16 copy of a contiguous fp32 cuda tensor (round to nearest even)."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("cast_bf16: contiguous fp32 cuda tensor")
    out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device) if out is None else out
    rc = lib().fa_cast_bf16(out.data_ptr(), x.data_ptr(), x.numel(), _stream_handle(stream, x.device))
    if rc != 0:
        raise FAError(rc, "fa_cast_bf16")
    return out


def bwd_workspace_size(B: int, H: int, N: int, d: int, dtype: int = FA_BF16, kv_heads: int | None = None) -> int:
    """Backward workspace bytes (with the split accumulators small problems use)."""
    if kv_heads is None:
        return int(lib().fa_bwd_workspace_size(B, H, N, d, dtype))
    return int(lib().fa_bwd_workspace_size_gqa(B, H, kv_heads, N, d, dtype))


def bwd(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None, workspace=None,
        dq=None, dk=None, dv=None, stream=None, window=None, block_mask=None):
    """Backward pass by recomputation: returns (dq, dk, dv), shaped like (q, k, v).

    With fewer K/V heads than query heads (fa_bwd_gqa), dk and dv are summed
    over each K/V head's query-head group.  ``window`` as in ``fwd`` (the same
    one the forward used), fa_bwd_window.
    """
    Hkv = _check_inputs(q, k, v, o, do)
    B, N, H, d = q.shape
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, N] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_workspace_size(B, H, N, d, _dtype_code(q), kv_heads=Hkv)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr())
    tail = (_scale(scale, d), int(bool(causal)), _dtype_code(q), workspace.data_ptr(), workspace.numel(),
            _stream_handle(stream, q.device))
    if block_mask is not None:
        wl, wr = _window_bounds(causal, (None, None) if window is None else window)
        mp, mh = _mask_args(block_mask, q)
        rc, name = lib().fa_bwd_blocksparse(*ptrs, B, H, Hkv, N, d, tail[0], wl, wr, mp, mh, *tail[2:]), \
            "fa_bwd_blocksparse"
    elif window is not None:
        wl, wr = _window_bounds(causal, window)
        rc, name = lib().fa_bwd_window(*ptrs, B, H, Hkv, N, d, tail[0], wl, wr, *tail[2:]), "fa_bwd_window"
    elif Hkv == H:
        rc, name = lib().fa_bwd(*ptrs, B, H, N, d, *tail), "fa_bwd"
    else:
        rc, name = lib().fa_bwd_gqa(*ptrs, B, H, Hkv, N, d, *tail), "fa_bwd_gqa"
    if rc != 0:
        raise FAError(rc, name)
    return dq, dk, dv


def last_device_status(stream=None, device=None):
    """Synchronise and read/clear the device status word: (status, raw word)."""
    detail = ctypes.c_int(0)
    dev = device if device is not None else torch.cuda.current_device()
    rc = lib().fa_last_device_status(_stream_handle(stream, dev), ctypes.byref(detail))
    return rc, detail.value


def set_wait_limit_ms(ms: int):
    lib().fa_set_wait_limit_ms(int(ms))


def debug_inject(mode: int):
    lib().fa_debug_inject(int(mode))


def set_kernel_events(start=None, stop=None):
    """Record torch.cuda.Event pairs around the next calls' tensor-core kernel (None, None: off)."""
    lib().fa_set_kernel_events(start.cuda_event if start is not None else None,
                               stop.cuda_event if stop is not None else None)


def debug_umma(a: torch.Tensor, b: torch.Tensor, a_mn_major: int, b_mn_major: int, a_tmem: int = 0,
               stream=None) -> torch.Tensor:
    """One tcgen05 MMA tile D = A B^T (test-only): a [128, K], b [N, K] bf16 cuda."""
    n, kdim = b.shape
    dmat = torch.empty((128, n), dtype=torch.float32, device=a.device)
    rc = probe_lib().fa_debug_umma(a.data_ptr(), b.data_ptr(), dmat.data_ptr(), n, kdim, int(a_mn_major),
                             int(b_mn_major), int(a_tmem), _stream_handle(stream, a.device))
    if rc != 0:
        raise FAError(rc, "fa_debug_umma")
    return dmat


def debug_umma_f8(a: torch.Tensor, b: torch.Tensor, b_mn_major: int, a_tmem: int = 0, stream=None) -> torch.Tensor:
    """One 8-bit tcgen05 MMA tile D = A B^T (test-only): a [128, 128], b [N, 128] e4m3 (uint8 bytes) cuda."""
    n = b.shape[0]
    dmat = torch.empty((128, n), dtype=torch.float32, device=a.device)
    rc = probe_lib().fa_debug_umma_f8(a.data_ptr(), b.data_ptr(), dmat.data_ptr(), n, int(b_mn_major), int(a_tmem),
                                _stream_handle(stream, a.device))
    if rc != 0:
        raise FAError(rc, "fa_debug_umma_f8")
    return dmat


def debug_umma_2cta(a: torch.Tensor, b: torch.Tensor, b_mn_major: int, a_tmem: int = 0, stream=None) -> torch.Tensor:
    """One M = 256 tcgen05 tile over a two-CTA cluster, D = A B^T (test-only): a [256, K], b [128, K] bf16 cuda.
    Raises if the MMAs did not complete."""
    n, kdim = b.shape
    dmat = torch.empty((256, n), dtype=torch.float32, device=a.device)
    status = torch.zeros(1, dtype=torch.int32, device=a.device)
    rc = probe_lib().fa_debug_umma_2cta(a.data_ptr(), b.data_ptr(), dmat.data_ptr(), n, kdim, int(b_mn_major),
                                        int(a_tmem), status.data_ptr(), _stream_handle(stream, a.device))
    if rc != 0:
        raise FAError(rc, "fa_debug_umma_2cta")
    if int(status.item()) != 0:
        raise FAError(-7, "fa_debug_umma_2cta: the MMAs did not complete")
    return dmat


MMA_RATE_KINDS = ("none", "tcgen05.ld", "tcgen05.st", "st.shared", "ld.shared", "bulk copy smem->global",
                  "bulk reduce-add smem->global", "red.global.add.v4", "ld.global (L1)", "quad transpose + red.v4",
                  "FFMA-bound warp on every SMSP", "FFMA-bound warp on the issuer's SMSP only",
                  "FFMA-bound warps on the other SMSPs only", "FFMA-bound warp on every SMSP, two issuers",
                  "FFMA-bound warp on the issuer's SMSP, converged-warp issue")


def debug_mma_rate(mode: int, n: int, kind: int = 0, grid: int | None = None, reps: int = 1500, device=None) -> dict:
    """Tensor-pipe rate probe (test-only): one CTA (mode 2: a CTA pair) per SM issues reps x 8 back-to-back
    128 x n x 16 bf16 MMAs (mode 0: both operands in shared memory, 1: A in TMEM, 2: M = 256 over a CTA pair)
    while four warps generate traffic of one kind (MMA_RATE_KINDS).  Returns the median SM clocks per MMA
    instruction, per 128 x 128 x 16 of work on one SM, and the traffic warps' bytes per clock."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if grid is None:
        grid = torch.cuda.get_device_properties(dev).multi_processor_count
        grid -= grid % 2
    cyc = torch.zeros(grid, dtype=torch.int64, device=dev)
    ops = torch.zeros(grid, dtype=torch.int64, device=dev)
    scratch = torch.zeros(grid * 4 * 16384, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = probe_lib().fa_debug_mma_rate(int(mode), int(n), int(kind), int(grid), int(reps), cyc.data_ptr(),
                                       ops.data_ptr(), scratch.data_ptr(), status.data_ptr(), _stream_handle(None, dev))
    if rc != 0:
        raise FAError(rc, "fa_debug_mma_rate")
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise FAError(-7, "fa_debug_mma_rate: the MMAs did not complete")
    c = float(cyc.median().item())
    o = float(ops.median().item())
    per = c / (reps * 8)
    m = 256 if mode == 2 else 128
    ctas = 2 if mode == 2 else 1
    return {"mode": mode, "n": n, "kind": MMA_RATE_KINDS[kind], "grid": grid, "clk_per_mma": per,
            "clk_per_128x128x16": per * (128 * 128) / (m // ctas * n),
            "traffic_bytes_per_clk": o * (16384.0 if kind == 9 else 4096.0) / c if 0 < kind < 10 else 0.0}


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, window, block_mask):
        o, lse = fwd(q, k, v, causal=causal, scale=scale, window=window, block_mask=block_mask)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale, ctx.window, ctx.block_mask = causal, scale, window, block_mask
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = bwd(q, k, v, o, do.contiguous(), lse, causal=ctx.causal, scale=ctx.scale, window=ctx.window,
                         block_mask=ctx.block_mask)
        return dq, dk, dv, None, None, None, None


def attention(q, k, v, causal: bool = False, scale: float | None = None, window=None, block_mask=None):
    """Differentiable attention: q [B, N, H, d], k and v [B, N, Hkv, d] (Hkv divides H);
    optional sliding ``window`` = (left, right) and 128 x 128 ``block_mask``."""
    return _Attention.apply(q, k, v, causal, scale, window, block_mask)
