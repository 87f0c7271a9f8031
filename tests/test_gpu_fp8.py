"""GPU parity of the FP8 (E4M3) KV cache path against the oracle: the
quantising append bit for bit (bf16 and fp32 inputs, saturation), and decode
over E4M3 pools with per-head scales on ragged small cases, every head
grouping, block size and partitioning, and the FP8 variants of the Llama-7B
and GQA decode batches at full size."""
import pytest
import torch

import oracle
from helpers import assert_close, bits
from pagedattention_paged_kv_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def pa():
    from pagedattention_paged_kv_02_b200 import build, pa as _pa
    build.build()
    torch.cuda.init()
    return _pa


@pytest.fixture(autouse=True)
def clean_error_word(pa):
    pa.pa_device_error(clear=True)
    yield
    torch.cuda.synchronize()


def oracle_after_append_fp8(b):
    k, v = b.k_cache.clone(), b.v_cache.clone()
    oracle.reshape_and_cache_e4m3(b.key, b.value, k, v, b.slot_mapping, b.k_scale, b.v_scale)
    return k, v


def gpu_step_fp8(pa, b, part=None):
    d = b.to(DEV)
    pa.pa_reshape_and_cache_fp8(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping, d.k_scale,
                                d.v_scale)
    part = b.partition_size if part is None else part
    B, H_q, D = d.q.shape
    n = pa.pa_decode_workspace_size(B, H_q, D, b.max_context_len, part)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(d.q)
    pa.pa_decode_fp8(out, d.q, d.k_cache, d.v_cache, d.k_scale, d.v_scale, d.block_tables,
                     d.context_lens, b.max_context_len, b.scale, part, ws if n else None)
    torch.cuda.synchronize()
    return d, out


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fp8_append_bit_exact(pa, dtype):
    base = W.decode_batch([5, 40, 17, 128], 4, 4, 128, 16, 32, dtype, std=3.0, seed=61)
    b = W.to_fp8(base, k_amax=2.0, v_amax=6.0)  # k values beyond 2 saturate
    d = b.to(DEV)
    pa.pa_reshape_and_cache_fp8(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping, d.k_scale,
                                d.v_scale)
    torch.cuda.synchronize()
    k, v = oracle_after_append_fp8(b)
    assert torch.equal(d.k_cache.cpu(), k) and torch.equal(d.v_cache.cpu(), v)


CASES = [
    ([1, 15, 16, 17, 100, 513, 1500], 8, 8, 16, 0),
    ([1, 15, 16, 17, 100, 513, 1500], 8, 8, 16, 64),
    ([33, 700, 1024, 2047], 32, 4, 32, 512),
    ([5, 64, 65, 999], 16, 1, 64, -1),
    ([200, 1200], 32, 1, 16, 256),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0][-1]}tok-h{c[1]}kv{c[2]}-bs{c[3]}-p{c[4]}")
def test_fp8_decode_small(pa, case):
    ctxs, Hq, Hkv, bs, part = case
    nb = sum(-(-c // bs) for c in ctxs) + 7
    b = W.to_fp8(W.decode_batch(ctxs, Hq, Hkv, 128, bs, nb, torch.bfloat16, seed=len(ctxs) + Hq))
    d, out = gpu_step_fp8(pa, b, part)
    k, v = oracle_after_append_fp8(b)
    ref, _ = oracle.decode_e4m3(b.q, k, v, b.k_scale, b.v_scale, b.block_tables, b.context_lens,
                                b.scale)
    assert_close(out, ref, f"fp8 decode {case}")
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("name", ["llama7b_decode_fp8", "gqa_decode_fp8"])
def test_fp8_workload_full(pa, name):
    b = W.WORKLOADS[name]()
    d, out = gpu_step_fp8(pa, b)
    k, v = oracle_after_append_fp8(b)
    assert torch.equal(d.k_cache.cpu(), k), "quantising append not bit-exact (K)"
    assert torch.equal(d.v_cache.cpu(), v), "quantising append not bit-exact (V)"
    ref, _ = oracle.decode_e4m3(b.q, k, v, b.k_scale, b.v_scale, b.block_tables, b.context_lens,
                                b.scale)
    assert_close(out, ref, name)
    assert pa.pa_device_error() == 0
