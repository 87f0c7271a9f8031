"""GPU parity of the persistent chunked prefill when every CTA works through
several items (one CTA per SM deals out the items, so small batches give a
CTA one item each and only large ones exercise what carries across items:
the K/V rings, the S/P phases, the Q tiles loaded behind the previous item's
last S, and the epilogues between two items' key tiles).

Batches of 288 to 1152 items, against the fp64 oracle on every output: a
GQA group of three (two consecutive 128-row tiles of one head per item, the
second often short or absent), groups of four and two (the same rows of two
query heads per item), head_dim 64 and 128, causal and sliding-window,
ragged chunk lengths and cached lengths from 0 to 2000 tokens."""
import pytest
import torch

import oracle
from helpers import assert_close, oracle_after_append
from test_gpu_prefill import mixed_chunks

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


def _chunks(n, seed, cmin, cmax, lmin, lmax):
    g = torch.Generator().manual_seed(seed)
    cached = torch.randint(cmin, cmax + 1, (n,), generator=g).tolist()
    lens = torch.randint(lmin, lmax + 1, (n,), generator=g).tolist()
    return cached, lens


CASES = [
    # name, chunks, H_q, H_kv, D, bs, window (0: causal)
    ("group3-rows-d128", 24, 24, 8, 128, 16, 0),     # 24 x 2 x 24 = 1152 items
    ("group4-heads-d64-w700", 24, 16, 4, 64, 32, 700),  # 8 x 3 x 24 = 576 items
    ("group2-heads-d128-w512", 24, 8, 4, 128, 64, 512),  # 4 x 3 x 24 = 288 items
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_many_items_per_cta(pa, case):
    name, n, Hq, Hkv, D, bs, window = case
    cached, lens = _chunks(n, seed=len(name) + n, cmin=0, cmax=2000, lmin=1, lmax=384)
    lens[0], lens[1] = 384, 1  # a longest and a one-query chunk
    batch = mixed_chunks(cached, lens, Hq, Hkv, bs, seed=sum(lens), D=D)
    d = batch.to(DEV)
    pa.pa_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    out = torch.full_like(d.prefill_q, float("nan"))
    max_q = max(lens)
    if window:
        pa.pa_prefill_chunk_sliding_window(out, d.prefill_q, d.k_cache, d.v_cache,
                                           d.prefill_block_tables, d.prefill_context_lens,
                                           d.query_start_loc, max_q, batch.scale, window)
    else:
        pa.pa_prefill_chunk(out, d.prefill_q, d.k_cache, d.v_cache, d.prefill_block_tables,
                            d.prefill_context_lens, d.query_start_loc, max_q, batch.scale)
    torch.cuda.synchronize()
    k, v = oracle_after_append(batch)
    if window:
        ref, _ = oracle.prefill_window(batch.prefill_q, k, v, batch.prefill_block_tables,
                                       batch.prefill_context_lens, batch.query_start_loc,
                                       batch.scale, window)
    else:
        ref, _ = oracle.prefill(batch.prefill_q, k, v, batch.prefill_block_tables,
                                batch.prefill_context_lens, batch.query_start_loc, batch.scale)
    assert_close(out, ref, name)
    assert pa.pa_device_error() == 0
