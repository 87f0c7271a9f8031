"""Thin ctypes binding of ``libpa.so`` (C ABI in ``include/pa.h``).

Each function has the name of the C entry point it calls and only marshals
arguments: torch tensors become device pointers and sizes, the current torch
CUDA stream becomes the ``cudaStream_t``, and a non-OK status becomes
:class:`PAError`. Every step of the computation runs in the library's CUDA
kernels. The library must have been built (``python -m
pagedattention_paged_kv_02_b200.build``); loading fails loudly otherwise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE = 0, 1, 2, 3
PA_ERR_BAD_TABLE, PA_ERR_TIMEOUT, PA_ERR_CUDA = 4, 5, 6
PA_F32, PA_BF16 = 0, 1

EXPORTS = ("pa_reshape_and_cache", "pa_decode_workspace_size", "pa_decode_partition_tokens",
           "pa_decode", "pa_prefill_chunk", "pa_check_tables", "pa_device_error",
           "pa_selftest_bounded_wait", "pa_status_string", "pa_version",
           "pa_decode_static_workspace", "pa_copy_blocks", "pa_swap_blocks",
           "pa_reshape_and_cache_fp8", "pa_decode_fp8", "pa_decode_sliding_window",
           "pa_prefill_chunk_sliding_window", "pa_reshape_and_cache_int8", "pa_decode_int8",
           "pa_decode_shared_prefix", "pa_decode_shared_prefix_workspace_size")


class PAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded on first use)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m pagedattention_paged_kv_02_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, F, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float,
                            ctypes.c_size_t)
        L.pa_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P]
        L.pa_decode_workspace_size.argtypes = [I, I, I, I, I]
        L.pa_decode_workspace_size.restype = SZ
        L.pa_decode_partition_tokens.argtypes = [I, I]
        L.pa_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, P, SZ, I, P]
        L.pa_decode_static_workspace.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I,
                                                 I, P]
        L.pa_prefill_chunk.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, I, P]
        L.pa_prefill_chunk_sliding_window.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I,
                                                      I, I, F, I, I, P]
        L.pa_decode_sliding_window.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, I,
                                               P, SZ, I, P]
        L.pa_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, I, P]
        L.pa_reshape_and_cache_int8.argtypes = L.pa_reshape_and_cache_fp8.argtypes
        L.pa_decode_fp8.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, P, SZ,
                                    P]
        L.pa_decode_int8.argtypes = L.pa_decode_fp8.argtypes
        L.pa_decode_shared_prefix.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I,
                                              I, I, I, F, I, P, SZ, I, P]
        L.pa_decode_shared_prefix_workspace_size.argtypes = [I, I, I, I, I, I, I, I, I]
        L.pa_decode_shared_prefix_workspace_size.restype = SZ
        L.pa_copy_blocks.argtypes = [P, P, P, I, I, I, I, I, I, P]
        L.pa_swap_blocks.argtypes = [P, P, I, P, P, I, P, I, I, I, I, I, P]
        L.pa_check_tables.argtypes = [P, P, I, I, I, I, P, ctypes.POINTER(I), P]
        L.pa_device_error.argtypes = [ctypes.POINTER(I), I]
        L.pa_selftest_bounded_wait.argtypes = [I64, P]
        L.pa_status_string.argtypes = [I]
        L.pa_status_string.restype = ctypes.c_char_p
        for f in ("pa_reshape_and_cache", "pa_decode", "pa_decode_static_workspace",
                  "pa_prefill_chunk", "pa_check_tables", "pa_copy_blocks", "pa_swap_blocks",
                  "pa_reshape_and_cache_fp8", "pa_decode_fp8", "pa_decode_sliding_window",
                  "pa_prefill_chunk_sliding_window", "pa_reshape_and_cache_int8",
                  "pa_decode_int8", "pa_decode_shared_prefix", "pa_device_error",
                  "pa_selftest_bounded_wait", "pa_decode_partition_tokens", "pa_version"):
            getattr(L, f).restype = I
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().pa_status_string(int(status)).decode()


def _call(fn: str, *args):
    st = getattr(lib(), fn)(*args)
    if st != PA_OK:
        raise PAError(fn, st)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float32:
        return PA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensors expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensors expected")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check_int(t: torch.Tensor, dtype, name):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


# ---------------------------------------------------------------------------
def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """Scatter ``key``/``value`` [T, H_kv, D] into the caches [NB, H_kv, bs, D]
    at ``slot_mapping`` (int64 [T])."""
    _check_int(slot_mapping, torch.int64, "slot_mapping")
    NB, H_kv, bs, D = k_cache.shape
    T = slot_mapping.numel()
    if key.shape != (T, H_kv, D) or value.shape != (T, H_kv, D):
        raise ValueError("key/value must be [num_tokens, num_kv_heads, head_dim]")
    if not (key.dtype == value.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("key, value and caches must share one dtype")
    _call("pa_reshape_and_cache", _p(key), _p(value), _p(k_cache), _p(v_cache),
          _p(slot_mapping), T, H_kv, D, bs, NB, _dt(k_cache), _stream(stream))


def pa_decode_workspace_size(num_seqs: int, num_q_heads: int, head_dim: int,
                             max_context_len: int, partition_size: int = 0) -> int:
    return int(lib().pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len,
                                              partition_size))


def pa_decode_partition_tokens(max_context_len: int, partition_size: int = 0) -> int:
    return int(lib().pa_decode_partition_tokens(max_context_len, partition_size))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
              scale: float, partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
              stream=None) -> None:
    """Paged decode attention into ``out`` [B, H_q, D]. ``workspace`` is a
    device byte buffer of at least :func:`pa_decode_workspace_size` bytes
    (may be None when that size is 0)."""
    _check_int(block_tables, torch.int32, "block_tables")
    _check_int(context_lens, torch.int32, "context_lens")
    B, H_q, D = q.shape
    NB, H_kv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or out.dtype != q.dtype:
        raise ValueError("out must match q; caches must share head_dim")
    if not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("q and caches must share one dtype")
    MB = block_tables.shape[1]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _call("pa_decode", _p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables),
          _p(context_lens), B, H_q, H_kv, D, bs, NB, MB, int(max_context_len), float(scale),
          int(partition_size), _p(workspace), ws_bytes, _dt(q), _stream(stream))


def pa_decode_shared_prefix_workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                                           head_dim: int, num_groups: int, max_group_size: int,
                                           max_prefix_len: int, max_context_len: int,
                                           partition_size: int = 0) -> int:
    """Bytes of workspace ``pa_decode_shared_prefix`` needs (0: invalid arguments)."""
    return int(lib().pa_decode_shared_prefix_workspace_size(
        int(num_seqs), int(num_q_heads), int(num_kv_heads), int(head_dim), int(num_groups),
        int(max_group_size), int(max_prefix_len), int(max_context_len), int(partition_size)))


def prepare_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, context_lens,
                                 group_start, prefix_lens, max_group_size: int,
                                 max_prefix_len: int, max_context_len: int, scale: float,
                                 partition_size: int = 0,
                                 workspace: Optional[torch.Tensor] = None) -> "Prepared":
    """``pa_decode_shared_prefix``: sequences listed group by group (group g =
    ``[group_start[g], group_start[g+1])``) sharing their first
    ``prefix_lens[g]`` positions."""
    for t, n in ((block_tables, "block_tables"), (context_lens, "context_lens"),
                 (group_start, "group_start"), (prefix_lens, "prefix_lens")):
        _check_int(t, torch.int32, n)
    B, H_q, D = q.shape
    NB, H_kv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or out.dtype != q.dtype:
        raise ValueError("out must match q; caches must share head_dim")
    if not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("q and caches must share one dtype")
    G = prefix_lens.numel()
    if group_start.numel() != G + 1:
        raise ValueError("group_start must have num_groups + 1 entries")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return Prepared("pa_decode_shared_prefix",
                    (_p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables),
                     _p(context_lens), _p(group_start), _p(prefix_lens), G, int(max_group_size),
                     int(max_prefix_len), B, H_q, H_kv, D, bs, NB, block_tables.shape[1],
                     int(max_context_len), float(scale), int(partition_size), _p(workspace),
                     ws_bytes, _dt(q)))


def pa_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, context_lens, group_start,
                            prefix_lens, max_group_size: int, max_prefix_len: int,
                            max_context_len: int, scale: float, partition_size: int = 0,
                            workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Paged decode reading each group's shared prefix once for all its
    sequences; same result as :func:`pa_decode`. ``workspace``: at least
    :func:`pa_decode_shared_prefix_workspace_size` bytes."""
    prepare_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, context_lens,
                                 group_start, prefix_lens, max_group_size, max_prefix_len,
                                 max_context_len, scale, partition_size, workspace)(stream)


def pa_decode_sliding_window(out, q, k_cache, v_cache, block_tables, context_lens,
                             max_context_len: int, scale: float, sliding_window: int,
                             partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
                             stream=None) -> None:
    """pa_decode attending only the last ``sliding_window`` positions."""
    _check_int(block_tables, torch.int32, "block_tables")
    _check_int(context_lens, torch.int32, "context_lens")
    B, H_q, D = q.shape
    NB, H_kv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or out.dtype != q.dtype:
        raise ValueError("out must match q; caches must share head_dim")
    if not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("q and caches must share one dtype")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _call("pa_decode_sliding_window", _p(out), _p(q), _p(k_cache), _p(v_cache),
          _p(block_tables), _p(context_lens), B, H_q, H_kv, D, bs, NB, block_tables.shape[1],
          int(max_context_len), float(scale), int(sliding_window), int(partition_size),
          _p(workspace), ws_bytes, _dt(q), _stream(stream))


def pa_decode_static_workspace(out, q, k_cache, v_cache, block_tables, context_lens,
                               max_context_len: int, scale: float, partition_size: int = 0,
                               stream=None) -> None:
    """pa_decode using the library's built-in 16 MiB scratch array instead of
    a workspace, for callers that cannot allocate device memory where they
    call decode. Calls that overlap on the GPU share that array and race."""
    _check_int(block_tables, torch.int32, "block_tables")
    _check_int(context_lens, torch.int32, "context_lens")
    B, H_q, D = q.shape
    NB, H_kv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or out.dtype != q.dtype:
        raise ValueError("out must match q; caches must share head_dim")
    if not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("q and caches must share one dtype")
    MB = block_tables.shape[1]
    _call("pa_decode_static_workspace", _p(out), _p(q), _p(k_cache), _p(v_cache),
          _p(block_tables), _p(context_lens), B, H_q, H_kv, D, bs, NB, MB, int(max_context_len),
          float(scale), int(partition_size), _dt(q), _stream(stream))


def _prefill_args(out, q, k_cache, block_tables, context_lens, query_start_loc):
    for t, n in ((block_tables, "block_tables"), (context_lens, "context_lens"),
                 (query_start_loc, "query_start_loc")):
        _check_int(t, torch.int32, n)
    total_q, H_q, D = q.shape
    NB, H_kv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or out.dtype != q.dtype:
        raise ValueError("out must match q; caches must share head_dim")
    return query_start_loc.numel() - 1, total_q, H_q, H_kv, D, bs, NB, block_tables.shape[1]


def pa_prefill_chunk(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                     max_query_len: int, scale: float, stream=None) -> None:
    """Chunked prefill into ``out`` [total_q, H_q, D]."""
    n_chunks, total_q, H_q, H_kv, D, bs, NB, MB = _prefill_args(
        out, q, k_cache, block_tables, context_lens, query_start_loc)
    _call("pa_prefill_chunk", _p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables),
          _p(context_lens), _p(query_start_loc), n_chunks, total_q, int(max_query_len), H_q,
          H_kv, D, bs, NB, MB, float(scale), _dt(q), _stream(stream))


def pa_prefill_chunk_sliding_window(out, q, k_cache, v_cache, block_tables, context_lens,
                                    query_start_loc, max_query_len: int, scale: float,
                                    sliding_window: int, stream=None) -> None:
    """Chunked prefill where the query at position p sees positions
    p - sliding_window + 1 .. p only."""
    n_chunks, total_q, H_q, H_kv, D, bs, NB, MB = _prefill_args(
        out, q, k_cache, block_tables, context_lens, query_start_loc)
    _call("pa_prefill_chunk_sliding_window", _p(out), _p(q), _p(k_cache), _p(v_cache),
          _p(block_tables), _p(context_lens), _p(query_start_loc), n_chunks, total_q,
          int(max_query_len), H_q, H_kv, D, bs, NB, MB, float(scale), int(sliding_window),
          _dt(q), _stream(stream))


def _q8_pool(k_cache, v_cache, k_scale, v_scale, code_dtype=torch.uint8):
    if k_cache.dtype != code_dtype or v_cache.dtype != code_dtype:
        raise TypeError("FP8 caches are uint8 tensors of E4M3 codes, INT8 caches int8 tensors")
    H_kv = k_cache.shape[1]
    for t, n in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        if t.dtype != torch.float32 or t.numel() != H_kv:
            raise ValueError(f"{n} must be float32 [num_kv_heads]")


def _reshape_q8(fn, code_dtype, key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                stream):
    _check_int(slot_mapping, torch.int64, "slot_mapping")
    _q8_pool(k_cache, v_cache, k_scale, v_scale, code_dtype)
    NB, H_kv, bs, D = k_cache.shape
    T = slot_mapping.numel()
    if key.shape != (T, H_kv, D) or value.shape != (T, H_kv, D) or key.dtype != value.dtype:
        raise ValueError("key/value must be [num_tokens, num_kv_heads, head_dim], one dtype")
    _call(fn, _p(key), _p(value), _p(k_cache), _p(v_cache), _p(slot_mapping), T, H_kv, D, bs, NB,
          _p(k_scale), _p(v_scale), _dt(key), _stream(stream))


def _decode_q8(fn, code_dtype, out, q, k_cache, v_cache, k_scale, v_scale, block_tables,
               context_lens, max_context_len, scale, partition_size, workspace, stream):
    _check_int(block_tables, torch.int32, "block_tables")
    _check_int(context_lens, torch.int32, "context_lens")
    _q8_pool(k_cache, v_cache, k_scale, v_scale, code_dtype)
    B, H_q, D = q.shape
    NB, H_kv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or q.dtype != torch.bfloat16 or out.dtype != q.dtype:
        raise ValueError("q and out must be bf16 [B, H_q, head_dim]")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _call(fn, _p(out), _p(q), _p(k_cache), _p(v_cache), _p(k_scale), _p(v_scale),
          _p(block_tables), _p(context_lens), B, H_q, H_kv, D, bs, NB, block_tables.shape[1],
          int(max_context_len), float(scale), int(partition_size), _p(workspace), ws_bytes,
          _stream(stream))


def pa_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                             stream=None) -> None:
    """Quantising append into E4M3 caches (codes of x / scale[h])."""
    _reshape_q8("pa_reshape_and_cache_fp8", torch.uint8, key, value, k_cache, v_cache,
                slot_mapping, k_scale, v_scale, stream)


def pa_reshape_and_cache_int8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                              stream=None) -> None:
    """Quantising append into INT8 caches (nearest integers of x / scale[h])."""
    _reshape_q8("pa_reshape_and_cache_int8", torch.int8, key, value, k_cache, v_cache,
                slot_mapping, k_scale, v_scale, stream)


def pa_decode_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                  max_context_len: int, scale: float, partition_size: int = 0,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Paged decode over E4M3 caches; q/out bf16 [B, H_q, 128]."""
    _decode_q8("pa_decode_fp8", torch.uint8, out, q, k_cache, v_cache, k_scale, v_scale,
               block_tables, context_lens, max_context_len, scale, partition_size, workspace,
               stream)


def pa_decode_int8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                   max_context_len: int, scale: float, partition_size: int = 0,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Paged decode over INT8 caches; q/out bf16 [B, H_q, 128]."""
    _decode_q8("pa_decode_int8", torch.int8, out, q, k_cache, v_cache, k_scale, v_scale,
               block_tables, context_lens, max_context_len, scale, partition_size, workspace,
               stream)


def _addressable(t: torch.Tensor):
    """Device tensors, or pinned host tensors the GPU reaches directly."""
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError("device or pinned host tensors expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensors expected")
    return ctypes.c_void_p(t.data_ptr())


def pa_copy_blocks(k_cache, v_cache, block_mapping, stream=None) -> None:
    """Copy-on-write: block ``block_mapping[i, 1]`` := block
    ``block_mapping[i, 0]`` in the same pool (int64 [n, 2])."""
    _check_int(block_mapping, torch.int64, "block_mapping")
    NB, H_kv, bs, D = k_cache.shape
    n = block_mapping.shape[0] if block_mapping.numel() else 0
    _call("pa_copy_blocks", _p(k_cache), _p(v_cache), _addressable(block_mapping), n, H_kv, D,
          bs, NB, _dt(k_cache), _stream(stream))


def pa_swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping, stream=None) -> None:
    """Block ``block_mapping[i, 1]`` of the destination pool := block
    ``block_mapping[i, 0]`` of the source pool; either pool may be pinned
    host memory."""
    _check_int(block_mapping, torch.int64, "block_mapping")
    if src_k.shape[1:] != dst_k.shape[1:] or src_k.dtype != dst_k.dtype:
        raise ValueError("pools must share block shape and dtype")
    _, H_kv, bs, D = src_k.shape
    n = block_mapping.shape[0] if block_mapping.numel() else 0
    _call("pa_swap_blocks", _addressable(src_k), _addressable(src_v), src_k.shape[0],
          _addressable(dst_k), _addressable(dst_v), dst_k.shape[0], _addressable(block_mapping),
          n, H_kv, D, bs, _dt(src_k), _stream(stream))


def pa_check_tables(block_tables, context_lens, block_size: int, num_blocks: int,
                    scratch: Optional[torch.Tensor] = None, stream=None) -> int:
    """Synchronous device check of tables/lengths; returns the number of bad
    rows (0 when all are valid)."""
    rows, MB = block_tables.shape
    if scratch is None:
        scratch = torch.empty(1, dtype=torch.int32, device=block_tables.device)
    bad = ctypes.c_int(0)
    st = lib().pa_check_tables(_p(block_tables), _p(context_lens), rows, MB, block_size,
                               num_blocks, _p(scratch), ctypes.byref(bad), _stream(stream))
    if st not in (PA_OK, PA_ERR_BAD_TABLE):
        raise PAError("pa_check_tables", st)
    return int(bad.value)


def pa_device_error(clear: bool = False) -> int:
    """The sticky device error word (synchronous)."""
    v = ctypes.c_int(0)
    _call("pa_device_error", ctypes.byref(v), 1 if clear else 0)
    return int(v.value)


def pa_selftest_bounded_wait(timeout_ns: int, stream=None) -> None:
    _call("pa_selftest_bounded_wait", int(timeout_ns), _stream(stream))


def pa_version() -> int:
    return int(lib().pa_version())


# ---------------------------------------------------------------------------
# prepared calls: arguments marshalled once, for loops that issue the same
# call every step (the tensors' storage must stay alive and unmoved)
# ---------------------------------------------------------------------------
class Prepared:
    """One C-ABI call with its pointer and size arguments fixed. Calling it
    launches on the given (or current) stream and raises on a non-OK status."""

    def __init__(self, fn: str, args):
        self.name = fn
        self._fn = getattr(lib(), fn)
        self._args = tuple(args)

    def __call__(self, stream=None):
        st = self._fn(*self._args, _stream(stream))
        if st != PA_OK:
            raise PAError(self.name, st)


def prepare_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping) -> Prepared:
    _check_int(slot_mapping, torch.int64, "slot_mapping")
    NB, H_kv, bs, D = k_cache.shape
    T = slot_mapping.numel()
    if key.shape != (T, H_kv, D) or value.shape != (T, H_kv, D):
        raise ValueError("key/value must be [num_tokens, num_kv_heads, head_dim]")
    return Prepared("pa_reshape_and_cache", (_p(key), _p(value), _p(k_cache), _p(v_cache),
                                             _p(slot_mapping), T, H_kv, D, bs, NB,
                                             _dt(k_cache)))


def prepare_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int,
                   scale: float, partition_size: int = 0,
                   workspace: Optional[torch.Tensor] = None,
                   sliding_window: int = 0) -> Prepared:
    """``pa_decode`` (or, with ``sliding_window`` > 0, ``pa_decode_sliding_window``)."""
    _check_int(block_tables, torch.int32, "block_tables")
    _check_int(context_lens, torch.int32, "context_lens")
    B, H_q, D = q.shape
    NB, H_kv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or out.dtype != q.dtype:
        raise ValueError("out must match q; caches must share head_dim")
    if not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("q and caches must share one dtype")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    head = (_p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables), _p(context_lens), B,
            H_q, H_kv, D, bs, NB, block_tables.shape[1], int(max_context_len), float(scale))
    tail = (int(partition_size), _p(workspace), ws_bytes, _dt(q))
    if sliding_window > 0:
        return Prepared("pa_decode_sliding_window", head + (int(sliding_window),) + tail)
    return Prepared("pa_decode", head + tail)


def prepare_prefill_chunk(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                          max_query_len: int, scale: float, sliding_window: int = 0) -> Prepared:
    """``pa_prefill_chunk`` (or, with ``sliding_window`` > 0,
    ``pa_prefill_chunk_sliding_window``)."""
    for t, n in ((block_tables, "block_tables"), (context_lens, "context_lens"),
                 (query_start_loc, "query_start_loc")):
        _check_int(t, torch.int32, n)
    total_q, H_q, D = q.shape
    NB, H_kv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or out.dtype != q.dtype:
        raise ValueError("out must match q; caches must share head_dim")
    head = (_p(out), _p(q), _p(k_cache), _p(v_cache), _p(block_tables), _p(context_lens),
            _p(query_start_loc), query_start_loc.numel() - 1, total_q, int(max_query_len), H_q,
            H_kv, D, bs, NB, block_tables.shape[1], float(scale))
    if sliding_window > 0:
        return Prepared("pa_prefill_chunk_sliding_window",
                        head + (int(sliding_window), _dt(q)))
    return Prepared("pa_prefill_chunk", head + (_dt(q),))


def prepare_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale,
                                  v_scale) -> Prepared:
    """``pa_reshape_and_cache_fp8``, or ``pa_reshape_and_cache_int8`` for int8 caches."""
    _check_int(slot_mapping, torch.int64, "slot_mapping")
    int8 = k_cache.dtype == torch.int8
    _q8_pool(k_cache, v_cache, k_scale, v_scale, torch.int8 if int8 else torch.uint8)
    NB, H_kv, bs, D = k_cache.shape
    return Prepared("pa_reshape_and_cache_int8" if int8 else "pa_reshape_and_cache_fp8",
                    (_p(key), _p(value), _p(k_cache), _p(v_cache), _p(slot_mapping),
                     slot_mapping.numel(), H_kv, D, bs, NB, _p(k_scale), _p(v_scale), _dt(key)))


def prepare_decode_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                       max_context_len: int, scale: float, partition_size: int = 0,
                       workspace: Optional[torch.Tensor] = None) -> Prepared:
    """``pa_decode_fp8``, or ``pa_decode_int8`` for int8 caches."""
    int8 = k_cache.dtype == torch.int8
    _q8_pool(k_cache, v_cache, k_scale, v_scale, torch.int8 if int8 else torch.uint8)
    B, H_q, D = q.shape
    NB, H_kv, bs, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return Prepared("pa_decode_int8" if int8 else "pa_decode_fp8",
                    (_p(out), _p(q), _p(k_cache), _p(v_cache), _p(k_scale), _p(v_scale),
                     _p(block_tables), _p(context_lens), B, H_q, H_kv, D, bs, NB,
                     block_tables.shape[1], int(max_context_len), float(scale),
                     int(partition_size), _p(workspace), ws_bytes))

