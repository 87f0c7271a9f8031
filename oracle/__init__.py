"""Plain fp64 CPU oracle for the paged-KV attention path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The product path (the CUDA library and its binding) never does, and
the two share no code: this side is the C file ``pa_oracle.c`` (built with gcc
into ``liboracle.so``) plus the ctypes marshalling below, and the closed forms
the pages print.

Sources, by page title and section:

* page "字节跳动 AI Infra (2)", question "KV Cache原理与优化": the per-step
  append of K_t/V_t to the cache and Attention_t = softmax(Q_t K^T / sqrt(d)) V.
* same page, question "vLLM与PagedAttention的原理": physical block pool, per
  request block table, block pointer = base + physical_block*block_size*head_dim.
* page "LLM推理优化", section 1.2: KV cache bytes = 2 x layers x heads x
  seq_len x head_dim x dtype bytes (closed form, :func:`kv_cache_bytes`).
* page "LLM推理优化", section 3.2: blocks of 16 tokens allocated on demand
  (block counts, :func:`blocks_needed`).
* page "LLM推理优化", section 1.3: GQA / MQA head sharing.
* page "字节跳动 AI Infra (2)", table of algorithm-level optimisations,
  FlashDecoding row: split along the KV length (:func:`decode_partials`,
  :func:`lse_merge`).
* page "字节跳动 AI Infra (2)", optimisation table, KV quantisation row, and
  page "LLM推理优化", section 1.3 (quantised KV cache): FP8 E4M3 codes with a
  scale per K/V head (:func:`e4m3_encode`, :func:`reshape_and_cache_e4m3`,
  :func:`decode_e4m3`).
* page "LLM推理优化", section 2.3 (window_size) and page "vLLM框架是怎么做推理加速的",
  追问 3 (sliding window attention): :func:`decode_window`.
* page "vLLM框架是怎么做推理加速的", section 3: chunked prefill; page
  "LLM推理优化", section 2.3: causal attention (:func:`prefill`).

Every function here is pinned by ``tests/test_oracle_pins.py`` against values
the pages print, closed forms, library routines and invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OR_F32, OR_BF16 = 0, 1
_ERRORS = {1: "slot outside the pool", 2: "block id outside the pool",
           3: "bad argument", 4: "out of host memory"}


def build(force: bool = False) -> str:
    """Compile ``pa_oracle.c`` into ``liboracle.so`` with gcc (OpenMP, fp64, no
    contraction of multiply-adds so the arithmetic is the plain one)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_num_threads.restype = I
            lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, I64, I, I, I, I64, I]
            lib.oracle_decode.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, I64, D, P]
            lib.oracle_decode_partials.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, I64,
                                                   D, I, I]
            lib.oracle_lse_merge.argtypes = [P, P, P, P, I64, I, I]
            lib.oracle_lse_merge.restype = None
            lib.oracle_prefill.argtypes = [P, P, P, P, P, I, P, P, P, I, I, I, I, I, I, I64, D, P]
            lib.oracle_prefill_window.argtypes = [P, P, P, P, P, I, P, P, P, I, I, I, I, I, I,
                                                  I64, D, I, P]
            lib.oracle_copy_blocks.argtypes = [P, P, I64, P, P, I64, P, I64, I64]
            lib.oracle_decode_window.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, I64,
                                                 D, I, P]
            lib.oracle_e4m3_encode_array.argtypes = [P, P, I64]
            lib.oracle_int8_encode_array.argtypes = [P, P, I64]
            lib.oracle_int8_encode_array.restype = None
            lib.oracle_reshape_and_cache_int8.argtypes = [P, P, I, P, P, P, I64, I, I, I, I64, P,
                                                          P]
            lib.oracle_decode_int8.argtypes = [P, P, P, I, P, P, P, P, P, P, I, I, I, I, I, I,
                                               I64, D, P]
            lib.oracle_e4m3_encode_array.restype = None
            lib.oracle_e4m3_decode_array.argtypes = [P, P, I64]
            lib.oracle_e4m3_decode_array.restype = None
            lib.oracle_reshape_and_cache_e4m3.argtypes = [P, P, I, P, P, P, I64, I, I, I, I64, P,
                                                          P]
            lib.oracle_decode_e4m3.argtypes = [P, P, P, I, P, P, P, P, P, P, I, I, I, I, I, I,
                                               I64, D, P]
            for f in ("oracle_reshape_and_cache", "oracle_decode", "oracle_decode_partials",
                      "oracle_prefill", "oracle_copy_blocks", "oracle_reshape_and_cache_e4m3",
                      "oracle_decode_e4m3", "oracle_decode_window", "oracle_prefill_window",
                      "oracle_reshape_and_cache_int8", "oracle_decode_int8"):
                getattr(lib, f).restype = I
            _lib = lib
    return _lib


def num_threads() -> int:
    """Host threads the oracle's OpenMP loops use."""
    return int(_load().oracle_num_threads())


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: {_ERRORS.get(rc, rc)}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return OR_F32
    if t.dtype == torch.bfloat16:
        return OR_BF16
    raise TypeError(f"oracle takes float32 or bfloat16 storage, got {t.dtype}")


def _cpu(t: torch.Tensor, dtype=None) -> torch.Tensor:
    t = t.detach()
    if t.device.type != "cpu":
        raise ValueError("oracle inputs live on the host")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    return t.contiguous()


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


# --------------------------------------------------------------------------
# closed forms the pages print
# --------------------------------------------------------------------------
def kv_cache_bytes(num_layers: int, num_heads: int, seq_len: int, head_dim: int,
                   dtype_bytes: int) -> int:
    """Bytes of K and V cache for one sequence: 2 (K and V) x layers x heads x
    tokens x head_dim x element bytes (page "LLM推理优化", section 1.2)."""
    return 2 * num_layers * num_heads * seq_len * head_dim * dtype_bytes


def blocks_needed(num_tokens: int, block_size: int = 16) -> int:
    """Physical blocks a sequence of ``num_tokens`` occupies when blocks are
    allocated on demand: the smallest count whose capacity covers every token
    (page "LLM推理优化", section 3.2; 16-token blocks)."""
    if num_tokens <= 0:
        return 0
    return (num_tokens + block_size - 1) // block_size


# --------------------------------------------------------------------------
# the path's steps
# --------------------------------------------------------------------------
def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping) -> None:
    """Scatter new tokens' K/V rows into the pool in place (the append step in
    paged form). ``key``/``value``: [T, H_kv, D]; caches: [NB, H_kv, bs, D];
    ``slot_mapping``: int64 [T], negative entries skipped."""
    key, value = _cpu(key), _cpu(value)
    slot_mapping = _cpu(slot_mapping, torch.int64)
    for c in (k_cache, v_cache):
        if not c.is_contiguous() or c.device.type != "cpu":
            raise ValueError("caches must be contiguous host tensors (updated in place)")
    NB, H_kv, bs, D = k_cache.shape
    T = slot_mapping.numel()
    assert key.shape == (T, H_kv, D) and value.shape == (T, H_kv, D)
    assert key.dtype == value.dtype == k_cache.dtype == v_cache.dtype
    rc = _load().oracle_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(slot_mapping), T, H_kv, D, bs, NB,
                                          key.element_size())
    _check(rc, "reshape_and_cache")


def _select(sel, n):
    if sel is None:
        return None
    s = torch.as_tensor(sel).reshape(-1).to(torch.uint8).contiguous()
    assert s.numel() == n
    return s


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, select=None):
    """fp64 paged decode attention. ``q``: [B, H_q, D] in the cache's dtype.
    Returns (out [B, H_q, D] float64, lse [B, H_q] float64). With ``select``
    (bool [B, H_q]) only those pairs are computed; the rest stay 0."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    block_tables = _cpu(block_tables, torch.int32)
    context_lens = _cpu(context_lens, torch.int32)
    B, H_q, D = q.shape
    NB, H_kv, bs, D2 = k_cache.shape
    assert D == D2 and q.dtype == k_cache.dtype == v_cache.dtype
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    sel = _select(select, B * H_q)
    out = torch.zeros(B, H_q, D, dtype=torch.float64)
    lse = torch.full((B, H_q), float("-inf"), dtype=torch.float64)
    rc = _load().oracle_decode(_ptr(out), _ptr(lse), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                               _dtype_code(q), _ptr(block_tables), _ptr(context_lens), B, H_q,
                               H_kv, D, bs, MB, NB, float(scale), _ptr(sel))
    _check(rc, "decode")
    return out, lse


def decode_partials(q, k_cache, v_cache, block_tables, context_lens, scale, partition_tokens):
    """Per-partition partial results (o_s, lse_s) over KV partitions of
    ``partition_tokens`` positions. Returns ([B, H_q, S, D], [B, H_q, S])."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    block_tables = _cpu(block_tables, torch.int32)
    context_lens = _cpu(context_lens, torch.int32)
    B, H_q, D = q.shape
    NB, H_kv, bs, _ = k_cache.shape
    MB = block_tables.shape[1]
    max_ctx = int(context_lens.max()) if B else 0
    S = max(1, -(-max_ctx // partition_tokens))
    o = torch.zeros(B, H_q, S, D, dtype=torch.float64)
    lse = torch.full((B, H_q, S), float("-inf"), dtype=torch.float64)
    rc = _load().oracle_decode_partials(_ptr(o), _ptr(lse), _ptr(q), _ptr(k_cache),
                                        _ptr(v_cache), _dtype_code(q), _ptr(block_tables),
                                        _ptr(context_lens), B, H_q, H_kv, D, bs, MB, NB,
                                        float(scale), int(partition_tokens), S)
    _check(rc, "decode_partials")
    return o, lse


def lse_merge(o_parts, lse_parts):
    """Merge partials ([..., S, D], [..., S]) by log-sum-exp into ([..., D], [...])."""
    o_parts = _cpu(o_parts, torch.float64)
    lse_parts = _cpu(lse_parts, torch.float64)
    lead = o_parts.shape[:-2]
    S, D = o_parts.shape[-2:]
    R = int(np.prod(lead)) if len(lead) else 1
    out = torch.zeros(*lead, D, dtype=torch.float64)
    lse = torch.zeros(*lead, dtype=torch.float64)
    _load().oracle_lse_merge(_ptr(out), _ptr(lse), _ptr(o_parts), _ptr(lse_parts), R, S, D)
    return out, lse


def prefill(q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale,
            select=None):
    """fp64 chunked-prefill attention. ``q``: [total_q, H_q, D]; chunk c owns
    rows [qsl[c], qsl[c+1]), table row c and total context context_lens[c]
    (its own tokens included). Returns (out [total_q, H_q, D], lse [total_q, H_q])."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    block_tables = _cpu(block_tables, torch.int32)
    context_lens = _cpu(context_lens, torch.int32)
    qsl = _cpu(query_start_loc, torch.int32)
    total_q, H_q, D = q.shape
    NB, H_kv, bs, _ = k_cache.shape
    n_chunks = qsl.numel() - 1
    MB = block_tables.shape[1]
    assert int(qsl[-1]) == total_q
    sel = _select(select, total_q * H_q)
    out = torch.zeros(total_q, H_q, D, dtype=torch.float64)
    lse = torch.full((total_q, H_q), float("-inf"), dtype=torch.float64)
    rc = _load().oracle_prefill(_ptr(out), _ptr(lse), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                _dtype_code(q), _ptr(block_tables), _ptr(context_lens), _ptr(qsl),
                                n_chunks, H_q, H_kv, D, bs, MB, NB, float(scale), _ptr(sel))
    _check(rc, "prefill")
    return out, lse


def prefill_window(q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale,
                   window, select=None):
    """fp64 chunked prefill with a sliding window: query i of chunk c, at
    position pos = ctx - C + i, attends positions [max(0, pos - window + 1),
    pos] only. Shapes as ``prefill``."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    block_tables = _cpu(block_tables, torch.int32)
    context_lens = _cpu(context_lens, torch.int32)
    qsl = _cpu(query_start_loc, torch.int32)
    total_q, H_q, D = q.shape
    NB, H_kv, bs, _ = k_cache.shape
    n_chunks = qsl.numel() - 1
    MB = block_tables.shape[1]
    assert int(qsl[-1]) == total_q
    sel = _select(select, total_q * H_q)
    out = torch.zeros(total_q, H_q, D, dtype=torch.float64)
    lse = torch.full((total_q, H_q), float("-inf"), dtype=torch.float64)
    rc = _load().oracle_prefill_window(_ptr(out), _ptr(lse), _ptr(q), _ptr(k_cache),
                                       _ptr(v_cache), _dtype_code(q), _ptr(block_tables),
                                       _ptr(context_lens), _ptr(qsl), n_chunks, H_q, H_kv, D, bs,
                                       MB, NB, float(scale), int(window), _ptr(sel))
    _check(rc, "prefill_window")
    return out, lse


def copy_blocks(src_k, src_v, dst_k, dst_v, mapping) -> None:
    """Whole-block copies between pools (or within one): for each row (s, d)
    of ``mapping`` (int64 [n, 2]), block d of dst := block s of src, K and
    V. Copy-on-write and swap-out/in are both this operation."""
    mapping = _cpu(mapping, torch.int64)
    for t in (src_k, src_v, dst_k, dst_v):
        if not t.is_contiguous() or t.device.type != "cpu":
            raise ValueError("pools must be contiguous host tensors")
    assert src_k.shape[1:] == dst_k.shape[1:] and src_k.dtype == dst_k.dtype
    block_bytes = src_k[0].numel() * src_k.element_size()
    rc = _load().oracle_copy_blocks(_ptr(src_k), _ptr(src_v), src_k.shape[0], _ptr(dst_k),
                                    _ptr(dst_v), dst_k.shape[0], _ptr(mapping),
                                    mapping.shape[0] if mapping.numel() else 0, block_bytes)
    _check(rc, "copy_blocks")


# --------------------------------------------------------------------------
# FP8 (E4M3) KV cache
# --------------------------------------------------------------------------
def e4m3_encode(x) -> torch.Tensor:
    """E4M3 codes (uint8) of fp32 values: nearest value, ties to the even
    code, finite magnitudes beyond 448 saturated, NaN to 0x7F."""
    x = _cpu(torch.as_tensor(x, dtype=torch.float32))
    out = torch.empty(x.shape, dtype=torch.uint8)
    _load().oracle_e4m3_encode_array(_ptr(x), _ptr(out), x.numel())
    return out


def e4m3_decode(codes) -> torch.Tensor:
    """Values (float64) of E4M3 codes."""
    codes = _cpu(torch.as_tensor(codes, dtype=torch.uint8))
    out = torch.empty(codes.shape, dtype=torch.float64)
    _load().oracle_e4m3_decode_array(_ptr(codes), _ptr(out), codes.numel())
    return out


def reshape_and_cache_e4m3(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale) -> None:
    """The append step into uint8 E4M3 caches: code of fp32(x) / scale[h]."""
    key, value = _cpu(key), _cpu(value)
    slot_mapping = _cpu(slot_mapping, torch.int64)
    k_scale = _cpu(k_scale, torch.float32)
    v_scale = _cpu(v_scale, torch.float32)
    for c in (k_cache, v_cache):
        if not c.is_contiguous() or c.device.type != "cpu" or c.dtype != torch.uint8:
            raise ValueError("caches must be contiguous uint8 host tensors")
    NB, H_kv, bs, D = k_cache.shape
    T = slot_mapping.numel()
    rc = _load().oracle_reshape_and_cache_e4m3(_ptr(key), _ptr(value), _dtype_code(key),
                                               _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                                               T, H_kv, D, bs, NB, _ptr(k_scale), _ptr(v_scale))
    _check(rc, "reshape_and_cache_e4m3")


def decode_e4m3(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale,
                select=None):
    """fp64 paged decode over uint8 E4M3 caches with per-K/V-head scales."""
    q = _cpu(q)
    k_cache, v_cache = _cpu(k_cache, torch.uint8), _cpu(v_cache, torch.uint8)
    k_scale, v_scale = _cpu(k_scale, torch.float32), _cpu(v_scale, torch.float32)
    block_tables = _cpu(block_tables, torch.int32)
    context_lens = _cpu(context_lens, torch.int32)
    B, H_q, D = q.shape
    NB, H_kv, bs, _ = k_cache.shape
    MB = block_tables.shape[1]
    sel = _select(select, B * H_q)
    out = torch.zeros(B, H_q, D, dtype=torch.float64)
    lse = torch.full((B, H_q), float("-inf"), dtype=torch.float64)
    rc = _load().oracle_decode_e4m3(_ptr(out), _ptr(lse), _ptr(q), _dtype_code(q), _ptr(k_cache),
                                    _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
                                    _ptr(block_tables), _ptr(context_lens), B, H_q, H_kv, D, bs,
                                    MB, NB, float(scale), _ptr(sel))
    _check(rc, "decode_e4m3")
    return out, lse


def int8_encode(q) -> torch.Tensor:
    """INT8 codes (int8) of fp32 quotients x / scale: nearest integer, ties to
    even, saturated to [-127, 127], NaN to 0."""
    q = _cpu(torch.as_tensor(q, dtype=torch.float32))
    out = torch.empty(q.shape, dtype=torch.int8)
    _load().oracle_int8_encode_array(_ptr(q), _ptr(out), q.numel())
    return out


def reshape_and_cache_int8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale) -> None:
    """The append step into int8 caches: code of fp32(x) / scale[h]."""
    key, value = _cpu(key), _cpu(value)
    slot_mapping = _cpu(slot_mapping, torch.int64)
    k_scale = _cpu(k_scale, torch.float32)
    v_scale = _cpu(v_scale, torch.float32)
    for c in (k_cache, v_cache):
        if not c.is_contiguous() or c.device.type != "cpu" or c.dtype != torch.int8:
            raise ValueError("caches must be contiguous int8 host tensors")
    NB, H_kv, bs, D = k_cache.shape
    T = slot_mapping.numel()
    rc = _load().oracle_reshape_and_cache_int8(_ptr(key), _ptr(value), _dtype_code(key),
                                               _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                                               T, H_kv, D, bs, NB, _ptr(k_scale), _ptr(v_scale))
    _check(rc, "reshape_and_cache_int8")


def decode_int8(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale,
                select=None):
    """fp64 paged decode over int8 caches with per-K/V-head scales."""
    q = _cpu(q)
    k_cache, v_cache = _cpu(k_cache, torch.int8), _cpu(v_cache, torch.int8)
    k_scale, v_scale = _cpu(k_scale, torch.float32), _cpu(v_scale, torch.float32)
    block_tables = _cpu(block_tables, torch.int32)
    context_lens = _cpu(context_lens, torch.int32)
    B, H_q, D = q.shape
    NB, H_kv, bs, _ = k_cache.shape
    MB = block_tables.shape[1]
    sel = _select(select, B * H_q)
    out = torch.zeros(B, H_q, D, dtype=torch.float64)
    lse = torch.full((B, H_q), float("-inf"), dtype=torch.float64)
    rc = _load().oracle_decode_int8(_ptr(out), _ptr(lse), _ptr(q), _dtype_code(q), _ptr(k_cache),
                                    _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
                                    _ptr(block_tables), _ptr(context_lens), B, H_q, H_kv, D, bs,
                                    MB, NB, float(scale), _ptr(sel))
    _check(rc, "decode_int8")
    return out, lse


def decode_window(q, k_cache, v_cache, block_tables, context_lens, scale, window, select=None):
    """fp64 paged decode attending only the last ``window`` positions."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    block_tables = _cpu(block_tables, torch.int32)
    context_lens = _cpu(context_lens, torch.int32)
    B, H_q, D = q.shape
    NB, H_kv, bs, _ = k_cache.shape
    MB = block_tables.shape[1]
    sel = _select(select, B * H_q)
    out = torch.zeros(B, H_q, D, dtype=torch.float64)
    lse = torch.full((B, H_q), float("-inf"), dtype=torch.float64)
    rc = _load().oracle_decode_window(_ptr(out), _ptr(lse), _ptr(q), _ptr(k_cache),
                                      _ptr(v_cache), _dtype_code(q), _ptr(block_tables),
                                      _ptr(context_lens), B, H_q, H_kv, D, bs, MB, NB,
                                      float(scale), int(window), _ptr(sel))
    _check(rc, "decode_window")
    return out, lse

