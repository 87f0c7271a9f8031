"""GPU parity of sliding-window decode against the oracle: windows smaller
than one chunk, across chunk and block boundaries, larger than every context,
with every partitioning; and table entries of blocks wholly before the window
set out of range (an engine may free them), which the kernels must never read."""
import pytest
import torch

import oracle
from helpers import assert_close
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


def run(pa, b, window, part, d=None):
    d = d or b.to(DEV)
    pa.pa_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    B, H_q, D = d.q.shape
    n = pa.pa_decode_workspace_size(B, H_q, D, b.max_context_len, part)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(d.q)
    pa.pa_decode_sliding_window(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                                b.max_context_len, b.scale, window, part, ws if n else None)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("window", [1, 5, 16, 17, 100, 700, 5000])
@pytest.mark.parametrize("dtype,part", [(torch.bfloat16, 0), (torch.bfloat16, 64),
                                        (torch.bfloat16, -1), (torch.float32, 128)])
def test_window_decode(pa, window, dtype, part):
    ctxs = [1, 15, 16, 17, 100, 513, 1500]
    b = W.decode_batch(ctxs, 8, 2, 128, 16, sum(-(-c // 16) for c in ctxs) + 7, dtype,
                       seed=window + part)
    out = run(pa, b, window, part)
    k, v = b.k_cache.clone(), b.v_cache.clone()
    oracle.reshape_and_cache(b.key, b.value, k, v, b.slot_mapping)
    ref, _ = oracle.decode_window(b.q, k, v, b.block_tables, b.context_lens, b.scale, window)
    assert_close(out, ref, f"window {window} part {part}")
    assert pa.pa_device_error() == 0


def test_blocks_before_the_window_are_never_read(pa):
    ctxs = [300, 1000, 77]
    window = 100
    b = W.decode_batch(ctxs, 4, 4, 128, 16, 120, torch.bfloat16, seed=81)
    d = b.to(DEV)
    for i, c in enumerate(ctxs):
        first_needed = max(0, c - window) // 16
        d.block_tables[i, :first_needed] = 1 << 20  # freed: out of the pool
    out = run(pa, b, window, 0, d=d)
    assert pa.pa_device_error() == 0
    k, v = b.k_cache.clone(), b.v_cache.clone()
    oracle.reshape_and_cache(b.key, b.value, k, v, b.slot_mapping)
    ref, _ = oracle.decode_window(b.q, k, v, b.block_tables, b.context_lens, b.scale, window)
    assert_close(out, ref, "freed prefix")
