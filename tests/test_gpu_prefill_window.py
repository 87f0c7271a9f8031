"""GPU parity of sliding-window chunked prefill against the oracle: bands of
one key, shorter than a tile, exactly a tile, across tile and block edges and
longer than every context; ragged chunks with every block size and head
grouping; table entries of blocks wholly before a chunk's first band set out
of range (an engine may free them), which the kernel must never read; and a
window covering every context giving plain prefill's bits."""
import pytest
import torch

import oracle
from helpers import assert_close, oracle_after_append
from test_gpu_prefill import CASES, mixed_chunks

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


def run(pa, batch, window, d=None):
    d = d or batch.to(DEV)
    pa.pa_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    out = torch.full_like(d.prefill_q, float("nan"))
    qsl = batch.query_start_loc
    max_q = int((qsl[1:] - qsl[:-1]).max())
    pa.pa_prefill_chunk_sliding_window(out, d.prefill_q, d.k_cache, d.v_cache,
                                       d.prefill_block_tables, d.prefill_context_lens,
                                       d.query_start_loc, max_q, batch.scale, window)
    torch.cuda.synchronize()
    return d, out


def reference(batch, window):
    k, v = oracle_after_append(batch)
    ref, _ = oracle.prefill_window(batch.prefill_q, k, v, batch.prefill_block_tables,
                                   batch.prefill_context_lens, batch.query_start_loc,
                                   batch.scale, window)
    return ref


@pytest.mark.parametrize("window", [1, 7, 128, 129, 300, 1000])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"h{c[1]}kv{c[2]}-bs{c[3]}-{max(c[0][1])}q")
def test_prefill_window(pa, case, window):
    (cached, lens), Hq, Hkv, bs = case
    batch = mixed_chunks(cached, lens, Hq, Hkv, bs, seed=sum(lens) + Hq + window)
    _, out = run(pa, batch, window)
    assert_close(out, reference(batch, window), f"prefill window {window} {case}")
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("window", [1, 100, 300])
def test_blocks_before_the_band_are_never_read(pa, window):
    cached, lens, bs = [1000, 300, 0, 700], [64, 1, 257, 300], 16
    batch = mixed_chunks(cached, lens, 8, 2, bs, seed=90 + window)
    d = batch.to(DEV)
    for c, (n_cached, C) in enumerate(zip(cached, lens)):
        first_needed = max(0, n_cached - window + 1) // bs
        d.prefill_block_tables[c, :first_needed] = 1 << 20  # freed: out of the pool
    _, out = run(pa, batch, window, d=d)
    assert pa.pa_device_error() == 0
    assert_close(out, reference(batch, window), f"freed prefix, window {window}")


@pytest.mark.parametrize("window", [1, 100, 129])
def test_prefill_window_head_dim_64(pa, window):
    (cached, lens), Hq, Hkv, bs = CASES[0]
    batch = mixed_chunks(cached, lens, Hq, Hkv, bs, seed=97 + window, D=64)
    _, out = run(pa, batch, window)
    assert_close(out, reference(batch, window), f"prefill D64 window {window}")
    assert pa.pa_device_error() == 0


def test_window_covering_everything_is_plain_prefill(pa):
    (cached, lens), Hq, Hkv, bs = CASES[1]
    batch = mixed_chunks(cached, lens, Hq, Hkv, bs, seed=95)
    d, out = run(pa, batch, 1 << 20)
    plain = torch.full_like(d.prefill_q, float("nan"))
    qsl = batch.query_start_loc
    pa.pa_prefill_chunk(plain, d.prefill_q, d.k_cache, d.v_cache, d.prefill_block_tables,
                        d.prefill_context_lens, d.query_start_loc,
                        int((qsl[1:] - qsl[:-1]).max()), batch.scale)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), plain.view(torch.int16))
