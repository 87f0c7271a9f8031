"""pa_decode_static_workspace: decode for callers that cannot allocate device
memory where they call it -- a plugin that a host engine hands only its input
and output buffers, or a latency-critical caller that may not run cudaMalloc
because it can synchronise the whole device. The entry point keeps its
partial results in a fixed 16 MiB array inside the library instead of a
caller workspace.

Checked here, through the C ABI: two calls in a row (the second reuses the
array the first left behind) each agree with pa_decode on the same inputs
and with the fp64 oracle, within the tolerance of the other decode tests; a
call after set-up leaves the device's free memory unchanged; and a request
whose partials would not fit is refused before anything runs. This file is
collected last so that a run stopping at its first failure has already run
everything else."""
import ctypes

import pytest
import torch

from helpers import assert_close, oracle_after_append, oracle_decode
from pagedattention_paged_kv_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def pa():
    from pagedattention_paged_kv_02_b200 import build, pa as _pa
    build.build()
    torch.cuda.init()
    return _pa


def _static_call(pa, out, d, part):
    """The entry point called directly through ctypes."""
    B, H_q, D = d.q.shape
    NB, H_kv, bs, _ = d.k_cache.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return pa.lib().pa_decode_static_workspace(
        p(out), p(d.q), p(d.k_cache), p(d.v_cache), p(d.block_tables), p(d.context_lens), B, H_q,
        H_kv, D, bs, NB, d.block_tables.shape[1], d.max_context_len, d.scale, part,
        pa.PA_BF16 if d.q.dtype == torch.bfloat16 else pa.PA_F32,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _prepared(pa, ctxs, seed, hq, hkv):
    nb = sum(-(-c // 16) for c in ctxs) + 5
    host = W.decode_batch(ctxs, hq, hkv, 128, 16, nb, torch.bfloat16, seed=seed)
    d = host.to(DEV)
    pa.pa_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    return host, d


def test_static_workspace_matches_pa_decode_twice(pa):
    part = 256  # several partitions per sequence, so the scratch array is used
    batches = [_prepared(pa, [3000, 517, 1, 2048, 4096], 21, 32, 8),
               _prepared(pa, [700, 2900, 64, 1500], 22, 16, 16)]
    for host, d in batches:
        B, H_q, D = d.q.shape
        need = pa.pa_decode_workspace_size(B, H_q, D, d.max_context_len, part)
        assert 0 < need <= 16 << 20
        ws = torch.empty(need, dtype=torch.uint8, device=DEV)
        ref = torch.empty_like(d.q)
        pa.pa_decode(ref, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                     d.max_context_len, d.scale, part, ws)
        got = torch.full_like(d.q, float("nan"))
        assert _static_call(pa, got, d, part) == pa.PA_OK
        torch.cuda.synchronize()
        assert_close(got, ref.double().cpu(), "static workspace vs pa_decode")
        k, v = oracle_after_append(host)
        want, _ = oracle_decode(host, k, v)
        assert_close(got, want, "static workspace vs the oracle")
    assert pa.pa_device_error() == 0


def test_static_workspace_allocates_nothing(pa):
    """After the set-up call (num_seqs = 0: address lookup, module loaded) a
    decode through the entry point leaves the device's free memory as it
    was: the partials went to the built-in array, not to new memory."""
    host, d = _prepared(pa, [2500, 900, 4000], 23, 32, 8)
    empty = torch.empty(0, d.q.shape[1], d.q.shape[2], dtype=d.q.dtype, device=DEV)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = pa.lib().pa_decode_static_workspace(
        p(empty), p(empty), p(d.k_cache), p(d.v_cache), p(d.block_tables), p(d.context_lens), 0,
        d.q.shape[1], d.k_cache.shape[1], d.q.shape[2], d.k_cache.shape[2], d.k_cache.shape[0],
        d.block_tables.shape[1], d.max_context_len, d.scale, 256, pa.PA_BF16,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pa.PA_OK
    got = torch.full_like(d.q, float("nan"))
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert _static_call(pa, got, d, 256) == pa.PA_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    k, v = oracle_after_append(host)
    want, _ = oracle_decode(host, k, v)
    assert_close(got, want, "static workspace after set-up vs the oracle")


def test_static_workspace_refuses_oversized_request(pa):
    """64 sequences x 64 heads x 256 partitions of partials is far beyond
    16 MiB: refused with PA_ERR_WORKSPACE and nothing launched. The buffers
    are real and sized for the request (all sequences empty), so even a
    launch would stay in bounds."""
    B, H_q, H_kv, D, bs, NB, MB = 64, 64, 8, 128, 16, 4, 8192
    q = torch.zeros(B, H_q, D, dtype=torch.bfloat16, device=DEV)
    out = torch.ones_like(q)
    kc = torch.zeros(NB, H_kv, bs, D, dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    tables = torch.zeros(B, MB, dtype=torch.int32, device=DEV)
    lens = torch.zeros(B, dtype=torch.int32, device=DEV)
    assert pa.pa_decode_workspace_size(B, H_q, D, 131072, 512) > 16 << 20
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = pa.lib().pa_decode_static_workspace(
        p(out), p(q), p(kc), p(vc), p(tables), p(lens), B, H_q, H_kv, D, bs, NB, MB, 131072,
        0.1, 512, pa.PA_BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pa.PA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 1)
