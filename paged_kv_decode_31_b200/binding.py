"""ctypes binding of libpagedkv.so (C ABI in include/pagedkv.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  torch provides device memory and the current
stream.  If the library is not built, every call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedkv.so")
_lib = None

# Mirrors of the constants in include/pagedkv.h
SPLIT_TOKENS = 4096
TILE_TOKENS = 128
DEVERR_BAD_BLOCK = 1
DEVERR_TABLE_WIDTH = 2
DEVERR_TIMEOUT = 4
DEVERR_QUERY_LEN = 8
DEVERR_SEQ_LEN = 16

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_ATTN_ARGS = [_P, _P, _P, _P, _P, _P, _I64, _P, _I64, _I, _P, _I,
              _I, _I, _I, _I, _I, _I, ctypes.c_float, _I,
              _P, _P, _P, _P, ctypes.c_size_t, _P, _P]


class PagedKVError(RuntimeError):
    """A C-ABI call returned an error status."""


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with `python -m paged_kv_decode_31_b200.build` "
                "(there is no CPU fallback)")
        L = ctypes.CDLL(_LIB_PATH)
        L.pkv_kv_append.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _I64, _I, _P,
                                    _I, _I, _I, _I, _I, _P, _P]
        L.pkv_kv_append.restype = _I
        L.pkv_paged_decode_attn.argtypes = _ATTN_ARGS
        L.pkv_paged_decode_attn.restype = _I
        L.pkv_paged_prefill_attn.argtypes = _ATTN_ARGS
        L.pkv_paged_prefill_attn.restype = _I
        L.pkv_workspace_size.argtypes = [_I, _I, _I, _I, _I]
        L.pkv_workspace_size.restype = ctypes.c_size_t
        L.pkv_strerror.argtypes = [_I]
        L.pkv_strerror.restype = ctypes.c_char_p
        L.pkv_split_tokens.argtypes = []
        L.pkv_split_tokens.restype = _I
        L.pkv_paged_varlen_attn.argtypes = [_P, _P, _P, _I, _I, _P, _P, _P, _P, _I64, _P, _I64,
                                            _I, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I,
                                            _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]
        L.pkv_paged_varlen_attn.restype = _I
        L.pkv_varlen_workspace_size.argtypes = [_I, _I, _I, _I]
        L.pkv_varlen_workspace_size.restype = ctypes.c_size_t
        L.pkv_kv_append_varlen.argtypes = [_P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _I64, _P,
                                           _I64, _I, _P, _I, _I, _I, _I, _P, _P]
        L.pkv_kv_append_varlen.restype = _I
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().pkv_strerror(int(code)).decode()


def _check(name: str, rc: int) -> None:
    if rc != 0:
        raise PagedKVError(f"{name}: {strerror(rc)} (status {rc})")


def _st3(t: torch.Tensor) -> ctypes.Array:
    return (ctypes.c_int64 * 3)(int(t.stride(0)), int(t.stride(1)), int(t.stride(2)))


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _need_cuda_bf16(name: str, t: torch.Tensor) -> None:
    if not t.is_cuda or t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be a bf16 CUDA tensor (got {t.dtype} on {t.device})")
    if t.dim() != 4 or t.stride(-1) != 1:
        raise ValueError(f"{name} must be 4-D with a unit stride on the last axis")


def _need_cuda_i32(name: str, t: torch.Tensor) -> None:
    if not t.is_cuda or t.dtype != torch.int32:
        raise TypeError(f"{name} must be an int32 CUDA tensor")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


# The library sees pointers, strides and the sizes passed beside them, nothing
# else: a tensor smaller than those sizes say would be read or written out of
# bounds on the device.  These checks tie every tensor to the sizes passed.

def _need_err(err: Optional[torch.Tensor]) -> None:
    if err is not None and (not err.is_cuda or err.dtype != torch.int32 or err.numel() < 1):
        raise TypeError("err must be an int32 CUDA tensor with at least one element")


def _need_cache_and_table(B: int, Hkv: Optional[int], D: int, k_cache: torch.Tensor,
                          v_cache: torch.Tensor, block_table: torch.Tensor,
                          seqlens: torch.Tensor) -> None:
    """k_cache and v_cache of one shape [num_blocks, block_size, Hkv, D]; a
    2-D block table of at least B rows with a unit column stride; at least B
    contiguous sequence lengths."""
    if tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError(f"k_cache {tuple(k_cache.shape)} and v_cache {tuple(v_cache.shape)} "
                         "must have the same shape")
    if int(k_cache.shape[3]) != D or (Hkv is not None and int(k_cache.shape[2]) != Hkv):
        raise ValueError(f"the caches {tuple(k_cache.shape)} disagree with Hkv {Hkv}, D {D}")
    if block_table.dim() != 2 or block_table.shape[0] < B:
        raise ValueError(f"block_table must be 2-D with at least batch = {B} rows")
    if block_table.stride(1) != 1:
        raise ValueError("block_table must have a unit column stride")
    if seqlens.dim() != 1 or seqlens.shape[0] < B or not seqlens.is_contiguous():
        raise ValueError(f"seqlens must be a contiguous 1-D tensor of at least batch = {B} "
                         "entries")


def _need_one_device(*tensors: Optional[torch.Tensor]) -> None:
    dev = tensors[0].device
    for t in tensors:
        if t is not None and t.device != dev:
            raise ValueError(f"every tensor must be on {dev} (found one on {t.device})")


def _need_rows(name: str, t: torch.Tensor, shape: tuple) -> None:
    """A bf16 tensor of exactly `shape` with a unit last stride."""
    if t.dtype != torch.bfloat16 or tuple(t.shape) != tuple(shape) or t.stride(-1) != 1:
        raise ValueError(f"{name} must be bf16 {list(shape)} with a unit last stride "
                         f"(got {t.dtype} {list(t.shape)})")


def _need_lse(name: str, t: torch.Tensor, shape: tuple) -> None:
    if t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous fp32 {list(shape)} tensor")


def workspace_size(batch: int, seqlen_q: int, Hq: int, D: int, max_seqlen_k: int) -> int:
    return int(lib().pkv_workspace_size(batch, seqlen_q, Hq, D, max_seqlen_k))


def kv_append(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
              v_cache: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor, *,
              err: Optional[torch.Tensor] = None, stream=None) -> None:
    """Write k_new/v_new [B, n, Hkv, D] into the caches at positions
    seqlens[b] + t (bits unchanged).  seqlens is not advanced."""
    for name, t in (("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need_cuda_bf16(name, t)
    _need_cuda_i32("block_table", block_table)
    _need_cuda_i32("seqlens", seqlens)
    _need_err(err)
    B, n, Hkv, D = k_new.shape
    if tuple(v_new.shape) != tuple(k_new.shape):
        raise ValueError("k_new and v_new must have the same shape")
    _need_cache_and_table(B, Hkv, D, k_cache, v_cache, block_table, seqlens)
    _need_one_device(k_new, v_new, k_cache, v_cache, block_table, seqlens, err)
    rc = lib().pkv_kv_append(
        k_new.data_ptr(), _st3(k_new), v_new.data_ptr(), _st3(v_new),
        k_cache.data_ptr(), _st3(k_cache), v_cache.data_ptr(), _st3(v_cache),
        int(k_cache.shape[0]), block_table.data_ptr(), int(block_table.stride(0)),
        int(block_table.shape[1]), seqlens.data_ptr(), B, n, Hkv, D, int(k_cache.shape[1]),
        _ptr(err), _stream_handle(stream))
    _check("pkv_kv_append", rc)


def _attn(fn_name: str, q, k_cache, v_cache, block_table, seqlens, max_seqlen_k, scale,
          causal, out, lse, workspace, err, stream,
          extra=()) -> Tuple[torch.Tensor, torch.Tensor]:
    _need_cuda_bf16("q", q)
    _need_cuda_bf16("k_cache", k_cache)
    _need_cuda_bf16("v_cache", v_cache)
    _need_cuda_i32("block_table", block_table)
    _need_cuda_i32("seqlens", seqlens)
    _need_err(err)
    B, sq, Hq, D = q.shape
    num_blocks, bs, Hkv, _ = k_cache.shape
    _need_cache_and_table(B, None, D, k_cache, v_cache, block_table, seqlens)
    if max_seqlen_k is None:
        max_seqlen_k = int(seqlens.max().item()) if seqlens.numel() else 0
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(B, sq, Hq, D, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(B, Hq, sq, dtype=torch.float32, device=q.device)
    _need_lse("lse", lse, (B, Hq, sq))
    _need_rows("out", out, (B, sq, Hq, D))
    need = workspace_size(B, sq, Hq, D, max_seqlen_k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _need_one_device(q, k_cache, v_cache, block_table, seqlens, out, lse, workspace, err)
    rc = getattr(lib(), fn_name)(
        q.data_ptr(), _st3(q), k_cache.data_ptr(), _st3(k_cache), v_cache.data_ptr(),
        _st3(v_cache), num_blocks, block_table.data_ptr(), int(block_table.stride(0)),
        int(block_table.shape[1]), seqlens.data_ptr(), int(max_seqlen_k), B, sq, Hq, Hkv, D, bs,
        float(scale), int(bool(causal)), out.data_ptr(), _st3(out), lse.data_ptr(),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), _ptr(err),
        _stream_handle(stream), *extra)
    _check(fn_name, rc)
    return out, lse


def paged_decode_attn(q, k_cache, v_cache, block_table, seqlens, *, max_seqlen_k=None,
                      scale=None, causal=False, out=None, lse=None, workspace=None, err=None,
                      stream=None):
    """Attention of q [B, sq, Hq, D] against the paged cache; returns
    (out [B, sq, Hq, D] bf16, lse [B, Hq, sq] fp32).  See include/pagedkv.h."""
    return _attn("pkv_paged_decode_attn", q, k_cache, v_cache, block_table, seqlens,
                 max_seqlen_k, scale, causal, out, lse, workspace, err, stream)


def debug_paged_decode_attn(q, k_cache, v_cache, block_table, seqlens, *, wait_limit_ns,
                            max_seqlen_k=None, scale=None, causal=False, out=None, lse=None,
                            workspace=None, err=None, stream=None):
    """paged_decode_attn with every internal pipeline wait limited to
    wait_limit_ns (at most the library's 2 s): the failure path under test.
    A wait that runs out makes the call give up: it returns, PKV_DEVERR_TIMEOUT
    is set in err and out / lse hold no result."""
    fn = lib().pkv_debug_paged_decode_attn
    if not fn.argtypes:
        fn.argtypes = _ATTN_ARGS + [ctypes.c_uint64]
        fn.restype = _I
    return _attn("pkv_debug_paged_decode_attn", q, k_cache, v_cache, block_table, seqlens,
                 max_seqlen_k, scale, causal, out, lse, workspace, err, stream,
                 extra=(int(wait_limit_ns),))


def debug_final_out(A, L, out=None, stream=None):
    """The library's final division of a folded row, A / L elementwise (0
    where L <= 0), on the device: float32 CUDA tensors of one shape."""
    L_ = lib()
    fn = L_.pkv_debug_final_out
    if not fn.argtypes:
        fn.argtypes = [_P, _P, _P, _I64, _P]
        fn.restype = _I
    for name, t in (("A", A), ("L", L)):
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.float32
                and t.is_contiguous()):
            raise TypeError(f"{name} must be a contiguous float32 CUDA tensor")
    if A.shape != L.shape:
        raise ValueError(f"A {tuple(A.shape)} and L {tuple(L.shape)} must have one shape")
    if out is None:
        out = torch.empty_like(A)
    _check("pkv_debug_final_out",
           fn(A.data_ptr(), L.data_ptr(), out.data_ptr(), A.numel(), _stream_handle(stream)))
    return out


def paged_decode_attn_append(q, k_new, v_new, k_cache, v_cache, block_table, seqlens, *,
                             max_seqlen_k=None, scale=None, causal=False, out=None, lse=None,
                             workspace=None, err=None, stream=None):
    """kv_append fused into decode: writes k_new/v_new [B, n_new, Hkv, D] at
    positions seqlens[b] - n_new + t (seqlens already count them), then attends.
    Bitwise equal to kv_append(seqlens - n_new) followed by paged_decode_attn."""
    _need_cuda_bf16("k_new", k_new)
    _need_cuda_bf16("v_new", v_new)
    L = lib()
    fn = L.pkv_paged_decode_attn_append
    if not fn.argtypes:
        fn.argtypes = [_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _I64, _P, _I64, _I, _P, _I,
                       _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P, _P, _P, _P,
                       ctypes.c_size_t, _P, _P]
        fn.restype = _I
    _need_cuda_bf16("q", q)
    _need_cuda_bf16("k_cache", k_cache)
    _need_cuda_bf16("v_cache", v_cache)
    _need_cuda_i32("block_table", block_table)
    _need_cuda_i32("seqlens", seqlens)
    _need_err(err)
    B, sq, Hq, D = q.shape
    num_blocks, bs, Hkv, _ = k_cache.shape
    _need_cache_and_table(B, None, D, k_cache, v_cache, block_table, seqlens)
    if tuple(v_new.shape) != tuple(k_new.shape) or int(k_new.shape[0]) != B or \
            tuple(k_new.shape[2:]) != (Hkv, D):
        raise ValueError(f"k_new and v_new must both be [{B}, n_new, {Hkv}, {D}]")
    if max_seqlen_k is None:
        max_seqlen_k = int(seqlens.max().item()) if seqlens.numel() else 0
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(B, sq, Hq, D, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(B, Hq, sq, dtype=torch.float32, device=q.device)
    _need_lse("lse", lse, (B, Hq, sq))
    _need_rows("out", out, (B, sq, Hq, D))
    if workspace is None:
        workspace = torch.empty(workspace_size(B, sq, Hq, D, max_seqlen_k), dtype=torch.uint8,
                                device=q.device)
    _need_one_device(q, k_new, v_new, k_cache, v_cache, block_table, seqlens, out, lse,
                     workspace, err)
    rc = fn(q.data_ptr(), _st3(q), k_new.data_ptr(), _st3(k_new), v_new.data_ptr(), _st3(v_new),
            int(k_new.shape[1]), k_cache.data_ptr(), _st3(k_cache), v_cache.data_ptr(),
            _st3(v_cache), num_blocks, block_table.data_ptr(), int(block_table.stride(0)),
            int(block_table.shape[1]), seqlens.data_ptr(), int(max_seqlen_k), B, sq, Hq, Hkv, D, bs,
            float(scale), int(bool(causal)), out.data_ptr(), _st3(out), lse.data_ptr(),
            workspace.data_ptr(), workspace.numel() * workspace.element_size(), _ptr(err),
            _stream_handle(stream))
    _check("pkv_paged_decode_attn_append", rc)
    return out, lse


def paged_prefill_attn(q, k_cache, v_cache, block_table, seqlens, *, max_seqlen_k=None,
                       scale=None, causal=True, out=None, lse=None, workspace=None, err=None,
                       stream=None):
    """Causal or chunked prefill over the paged cache; same contract as decode."""
    return _attn("pkv_paged_prefill_attn", q, k_cache, v_cache, block_table, seqlens,
                 max_seqlen_k, scale, causal, out, lse, workspace, err, stream)


def _st2(t: torch.Tensor) -> ctypes.Array:
    return (ctypes.c_int64 * 2)(int(t.stride(0)), int(t.stride(1)))


def _need_packed_bf16(name: str, t: torch.Tensor) -> None:
    if not t.is_cuda or t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be a bf16 CUDA tensor (got {t.dtype} on {t.device})")
    if t.dim() != 3 or t.stride(-1) != 1:
        raise ValueError(f"{name} must be 3-D [tokens, heads, D] with a unit last stride")


def varlen_workspace_size(total_q: int, Hq: int, D: int, max_seqlen_k: int) -> int:
    return int(lib().pkv_varlen_workspace_size(total_q, Hq, D, max_seqlen_k))


def paged_varlen_attn(q, k_cache, v_cache, block_table, seqlens, cu_seqlens_q, max_seqlen_q, *,
                      max_seqlen_k=None, scale=None, causal=True, out=None, lse=None,
                      final=False, final_out=None, final_lse=None, workspace=None, err=None,
                      stream=None):
    """Packed multi-request attention: request b's queries are rows
    cu_seqlens_q[b] .. cu_seqlens_q[b+1] - 1 of q [total_q, Hq, D] (the last
    n_b positions of its context).  Returns (out [total_q, Hq, D], lse
    [Hq, total_q]); with final=True also (final_out [B, Hq, D], final_lse
    [B, Hq]), each request's last query row.  See include/pagedkv.h."""
    _need_packed_bf16("q", q)
    _need_cuda_bf16("k_cache", k_cache)
    _need_cuda_bf16("v_cache", v_cache)
    _need_cuda_i32("block_table", block_table)
    _need_cuda_i32("seqlens", seqlens)
    _need_cuda_i32("cu_seqlens_q", cu_seqlens_q)
    _need_err(err)
    total_q, Hq, D = q.shape
    B = int(seqlens.shape[0])
    if tuple(cu_seqlens_q.shape) != (B + 1,) or not cu_seqlens_q.is_contiguous():
        raise ValueError("cu_seqlens_q must be a contiguous tensor of batch + 1 entries")
    num_blocks, bs, Hkv, _ = k_cache.shape
    _need_cache_and_table(B, None, D, k_cache, v_cache, block_table, seqlens)
    if max_seqlen_k is None:
        max_seqlen_k = int(seqlens.max().item()) if seqlens.numel() else 0
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(total_q, Hq, D, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(Hq, total_q, dtype=torch.float32, device=q.device)
    _need_packed_bf16("out", out)
    if tuple(out.shape) != (total_q, Hq, D):
        raise ValueError("out must be [total_q, Hq, D]")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (Hq, total_q):
        raise ValueError("lse must be a contiguous fp32 [Hq, total_q] tensor")
    if final and final_out is None:
        final_out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=q.device)
    if final and final_lse is None:
        final_lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    if final_out is not None:
        _need_packed_bf16("final_out", final_out)
        if tuple(final_out.shape) != (B, Hq, D) or final_lse is None or \
                tuple(final_lse.shape) != (B, Hq) or not final_lse.is_contiguous() or \
                final_lse.dtype != torch.float32:
            raise ValueError("final_out must be [B, Hq, D] and final_lse a contiguous [B, Hq]")
    need = varlen_workspace_size(total_q, Hq, D, max_seqlen_k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _need_one_device(q, k_cache, v_cache, block_table, seqlens, cu_seqlens_q, out, lse,
                     final_out, final_lse, workspace, err)
    rc = lib().pkv_paged_varlen_attn(
        q.data_ptr(), _st2(q), cu_seqlens_q.data_ptr(), total_q, int(max_seqlen_q),
        k_cache.data_ptr(), _st3(k_cache), v_cache.data_ptr(), _st3(v_cache), num_blocks,
        block_table.data_ptr(), int(block_table.stride(0)), int(block_table.shape[1]),
        seqlens.data_ptr(), int(max_seqlen_k), B, Hq, Hkv, D, bs, float(scale),
        int(bool(causal)), out.data_ptr(), _st2(out), lse.data_ptr(), _ptr(final_out),
        None if final_out is None else _st2(final_out), _ptr(final_lse), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _ptr(err), _stream_handle(stream))
    _check("pkv_paged_varlen_attn", rc)
    if final_out is not None:
        return out, lse, final_out, final_lse
    return out, lse


def kv_append_varlen(k_new, v_new, k_cache, v_cache, block_table, seqlens, cu_seqlens_new, *,
                     err=None, stream=None) -> None:
    """Write packed k_new/v_new [total_new, Hkv, D] (sequence b's tokens are
    rows cu_seqlens_new[b] .. cu_seqlens_new[b+1] - 1) at positions
    seqlens[b] + t.  seqlens is not advanced."""
    _need_packed_bf16("k_new", k_new)
    _need_packed_bf16("v_new", v_new)
    _need_cuda_bf16("k_cache", k_cache)
    _need_cuda_bf16("v_cache", v_cache)
    _need_cuda_i32("block_table", block_table)
    _need_cuda_i32("seqlens", seqlens)
    _need_cuda_i32("cu_seqlens_new", cu_seqlens_new)
    _need_err(err)
    total, Hkv, D = k_new.shape
    B = int(seqlens.shape[0])
    if tuple(v_new.shape) != tuple(k_new.shape):
        raise ValueError("k_new and v_new must have the same shape")
    if tuple(cu_seqlens_new.shape) != (B + 1,) or not cu_seqlens_new.is_contiguous():
        raise ValueError("cu_seqlens_new must be a contiguous tensor of batch + 1 entries")
    _need_cache_and_table(B, Hkv, D, k_cache, v_cache, block_table, seqlens)
    _need_one_device(k_new, v_new, k_cache, v_cache, block_table, seqlens, cu_seqlens_new, err)
    rc = lib().pkv_kv_append_varlen(
        k_new.data_ptr(), _st2(k_new), v_new.data_ptr(), _st2(v_new), cu_seqlens_new.data_ptr(),
        total, k_cache.data_ptr(), _st3(k_cache), v_cache.data_ptr(), _st3(v_cache),
        int(k_cache.shape[0]), block_table.data_ptr(), int(block_table.stride(0)),
        int(block_table.shape[1]), seqlens.data_ptr(), B, Hkv, D, int(k_cache.shape[1]),
        _ptr(err), _stream_handle(stream))
    _check("pkv_kv_append_varlen", rc)


def partials_size(batch: int, seqlen_q: int, Hq: int, D: int, n_splits_local: int) -> int:
    L = lib()
    fn = L.pkv_partials_size
    if not fn.argtypes:
        fn.argtypes = [_I, _I, _I, _I, _I]
        fn.restype = ctypes.c_size_t
    return int(fn(batch, seqlen_q, Hq, D, n_splits_local))


def paged_attn_partials(q, k_cache, v_cache, block_table, seqlens, split_begin, n_splits_local,
                        *, scale=None, causal=False, partials=None, err=None, stream=None):
    """Split partials of absolute splits [split_begin, split_begin +
    n_splits_local) for every row of q [B, sq, Hq, D] (one context-parallel
    rank's share).  Returns the partial buffer (uint8, pkv_partials_size
    bytes).  seqlens are the full context lengths."""
    L = lib()
    fn = L.pkv_paged_attn_partials
    if not fn.argtypes:
        fn.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _P, _I64, _I, _P, _I, _I, _I, _I, _I, _I,
                       ctypes.c_float, _I, _I, _I, _P, ctypes.c_size_t, _P, _P]
        fn.restype = _I
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need_cuda_bf16(name, t)
    _need_cuda_i32("block_table", block_table)
    _need_cuda_i32("seqlens", seqlens)
    _need_err(err)
    B, sq, Hq, D = q.shape
    num_blocks, bs, Hkv, _ = k_cache.shape
    _need_cache_and_table(B, None, D, k_cache, v_cache, block_table, seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    need = partials_size(B, sq, Hq, D, n_splits_local)
    if partials is None:
        partials = torch.empty(need, dtype=torch.uint8, device=q.device)
    _need_one_device(q, k_cache, v_cache, block_table, seqlens, partials, err)
    rc = fn(q.data_ptr(), _st3(q), k_cache.data_ptr(), _st3(k_cache), v_cache.data_ptr(),
            _st3(v_cache), num_blocks, block_table.data_ptr(), int(block_table.stride(0)),
            int(block_table.shape[1]), seqlens.data_ptr(), B, sq, Hq, Hkv, D, bs, float(scale),
            int(bool(causal)), int(split_begin), int(n_splits_local), partials.data_ptr(),
            partials.numel() * partials.element_size(), _ptr(err), _stream_handle(stream))
    _check("pkv_paged_attn_partials", rc)
    return partials


def merge_partials(gathered, world, n_splits_local, seqlens, q_shape, *, causal=False, out=None,
                   lse=None, stream=None):
    """Merge `world` partial buffers laid side by side in `gathered` (uint8,
    world x partials_size bytes, rank r's block holding global splits
    [r n_local, (r + 1) n_local)) into (out, lse) for q_shape (B, sq, Hq, D)."""
    L = lib()
    fn = L.pkv_merge_partials
    if not fn.argtypes:
        fn.argtypes = [_P, _I, _I, ctypes.c_size_t, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]
        fn.restype = _I
    _need_cuda_i32("seqlens", seqlens)
    if not gathered.is_cuda or not gathered.is_contiguous():
        raise TypeError("gathered must be a contiguous CUDA tensor")
    B, sq, Hq, D = q_shape
    if seqlens.dim() != 1 or seqlens.shape[0] < B or not seqlens.is_contiguous():
        raise ValueError(f"seqlens must be a contiguous 1-D tensor of at least batch = {B} "
                         "entries")
    nbytes = gathered.numel() * gathered.element_size()
    if nbytes % world != 0:
        raise ValueError("gathered buffer is not world equal blocks")
    if out is None:
        out = torch.empty(B, sq, Hq, D, dtype=torch.bfloat16, device=gathered.device)
    if lse is None:
        lse = torch.empty(B, Hq, sq, dtype=torch.float32, device=gathered.device)
    _need_rows("out", out, (B, sq, Hq, D))
    _need_lse("lse", lse, (B, Hq, sq))
    _need_one_device(gathered, seqlens, out, lse)
    rc = fn(gathered.data_ptr(), int(world), int(n_splits_local), nbytes // world,
            seqlens.data_ptr(), B, sq, Hq, D, int(bool(causal)), out.data_ptr(), _st3(out),
            lse.data_ptr(), _stream_handle(stream))
    _check("pkv_merge_partials", rc)
    return out, lse


def paged_prefill_attn_bwd(q, k_cache, v_cache, block_table, seqlens, out, lse, dout, *,
                           max_seqlen_k=None, scale=None, causal=True, dq=None, dk_cache=None,
                           dv_cache=None, workspace=None, err=None, stream=None):
    """Deterministic backward of paged attention: returns (dq [B, sq, Hq, D],
    dk_cache, dv_cache) with the gradients of the cache rows laid out like
    k_cache / v_cache (new zero-filled buffers unless given)."""
    L = lib()
    fn = L.pkv_paged_prefill_attn_bwd
    if not fn.argtypes:
        fn.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _P, _I64, _I, _P, _I, _I, _I, _I, _I, _I,
                       _I, ctypes.c_float, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                       ctypes.c_size_t, _P, _P]
        fn.restype = _I
        L.pkv_bwd_workspace_size.argtypes = [_I, _I, _I]
        L.pkv_bwd_workspace_size.restype = ctypes.c_size_t
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("out", out),
                    ("dout", dout)):
        _need_cuda_bf16(name, t)
    _need_cuda_i32("block_table", block_table)
    _need_cuda_i32("seqlens", seqlens)
    _need_err(err)
    B, sq, Hq, D = q.shape
    num_blocks, bs, Hkv, _ = k_cache.shape
    _need_cache_and_table(B, None, D, k_cache, v_cache, block_table, seqlens)
    _need_rows("out", out, (B, sq, Hq, D))
    _need_rows("dout", dout, (B, sq, Hq, D))
    _need_lse("lse", lse, (B, Hq, sq))
    if max_seqlen_k is None:
        max_seqlen_k = int(seqlens.max().item()) if seqlens.numel() else 0
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if dq is None:
        dq = torch.empty_like(q, memory_format=torch.contiguous_format)
    if dk_cache is None:
        dk_cache = torch.zeros(k_cache.shape, dtype=torch.bfloat16, device=q.device)
    if dv_cache is None:
        dv_cache = torch.zeros(v_cache.shape, dtype=torch.bfloat16, device=q.device)
    for name, t in (("dq", dq), ("dk_cache", dk_cache), ("dv_cache", dv_cache)):
        _need_cuda_bf16(name, t)
    _need_rows("dq", dq, (B, sq, Hq, D))
    _need_rows("dk_cache", dk_cache, tuple(k_cache.shape))
    _need_rows("dv_cache", dv_cache, tuple(v_cache.shape))
    if workspace is None:
        workspace = torch.empty(int(L.pkv_bwd_workspace_size(B, sq, Hq)), dtype=torch.uint8,
                                device=q.device)
    _need_one_device(q, k_cache, v_cache, block_table, seqlens, out, lse, dout, dq, dk_cache,
                     dv_cache, workspace, err)
    rc = fn(q.data_ptr(), _st3(q), k_cache.data_ptr(), _st3(k_cache), v_cache.data_ptr(),
            _st3(v_cache), num_blocks, block_table.data_ptr(), int(block_table.stride(0)),
            int(block_table.shape[1]), seqlens.data_ptr(), int(max_seqlen_k), B, sq, Hq, Hkv, D,
            bs, float(scale), int(bool(causal)), out.data_ptr(), _st3(out), lse.data_ptr(),
            dout.data_ptr(), _st3(dout), dq.data_ptr(), _st3(dq), dk_cache.data_ptr(),
            _st3(dk_cache), dv_cache.data_ptr(), _st3(dv_cache), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), _ptr(err), _stream_handle(stream))
    _check("pkv_paged_prefill_attn_bwd", rc)
    return dq, dk_cache, dv_cache


# Allocation-free decode (see pkv_paged_decode_attn_static_ws in pagedkv.h).
STATIC_WORKSPACE_BYTES = 8 << 20


def paged_decode_attn_static_ws(q, k_cache, v_cache, block_table, seqlens, *, max_seqlen_k,
                                scale=None, causal=False, out, lse, err=None, stream=None):
    """Decode attention whose scratch lives in a device array the library owns,
    for callers that cannot allocate device memory when they call: the caller
    passes every input and output (out, lse, and max_seqlen_k as a host int),
    and nothing is allocated here or in the library.  Calls on one device
    share that array, so calls that overlap on the GPU race; serialise them.
    The first call on a device looks up the array's address: make it before
    any stream capture."""
    L = lib()
    fn = L.pkv_paged_decode_attn_static_ws
    if not fn.argtypes:
        fn.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _P, _I64, _I, _P, _I,
                       _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P, _P, _P, _P, _P]
        fn.restype = _I
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("out", out)):
        _need_cuda_bf16(name, t)
    _need_cuda_i32("block_table", block_table)
    _need_cuda_i32("seqlens", seqlens)
    _need_err(err)
    B, sq, Hq, D = q.shape
    num_blocks, bs, Hkv, _ = k_cache.shape
    _need_cache_and_table(B, None, D, k_cache, v_cache, block_table, seqlens)
    _need_lse("lse", lse, (B, Hq, sq))
    _need_rows("out", out, (B, sq, Hq, D))
    _need_one_device(q, k_cache, v_cache, block_table, seqlens, out, lse, err)
    need = workspace_size(B, sq, Hq, D, max_seqlen_k)
    if need > STATIC_WORKSPACE_BYTES:
        raise PagedKVError(f"this problem needs {need} bytes of scratch; the library's static "
                           f"workspace holds {STATIC_WORKSPACE_BYTES} (use paged_decode_attn)")
    rc = fn(q.data_ptr(), _st3(q), k_cache.data_ptr(), _st3(k_cache), v_cache.data_ptr(),
            _st3(v_cache), num_blocks, block_table.data_ptr(), int(block_table.stride(0)),
            int(block_table.shape[1]), seqlens.data_ptr(), int(max_seqlen_k), B, sq, Hq, Hkv, D,
            bs, float(1.0 / math.sqrt(D) if scale is None else scale), int(bool(causal)),
            out.data_ptr(), _st3(out), lse.data_ptr(), _ptr(err), _stream_handle(stream))
    _check("pkv_paged_decode_attn_static_ws", rc)
    return out, lse
