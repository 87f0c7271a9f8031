"""GPU edge cases at the limits of the arguments: the largest explicit
partition (16384 tokens) and a split at it; 64 query heads on one KV head (four
16-head tiles); an empty decode batch; prefill chunks of no queries between
real ones, a single-query chunk with nothing cached, and a chunk whose
queries end exactly on a 128-key tile; all against the oracle."""
import pytest
import torch

import oracle
from helpers import assert_close, gpu_decode, oracle_after_append, oracle_decode
from pagedattention_paged_kv_02_b200 import workloads as W
from test_gpu_prefill import mixed_chunks, oracle_prefill, run_prefill

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


def decode_step(pa, batch, part):
    dev = batch.to(DEV)
    pa.pa_reshape_and_cache(dev.key, dev.value, dev.k_cache, dev.v_cache, dev.slot_mapping)
    out = gpu_decode(pa, dev, part)
    torch.cuda.synchronize()
    return out


def test_largest_partition(pa):
    """16384-token partitions: one whole partition, and a split at it."""
    ctxs = [16384, 20000, 3]
    batch = W.decode_batch(ctxs, 8, 2, 128, 64, sum(-(-c // 64) for c in ctxs) + 3,
                           torch.bfloat16, seed=101)
    out = decode_step(pa, batch, 16384)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_decode(batch, k, v)
    assert_close(out, ref, "16384-token partitions")
    assert pa.pa_device_error() == 0


def test_sixty_four_heads_per_kv_head(pa):
    batch = W.decode_batch([700, 33], 64, 1, 128, 16, 60, torch.bfloat16, seed=102)
    out = decode_step(pa, batch, 256)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_decode(batch, k, v)
    assert_close(out, ref, "MQA with 64 query heads")
    assert pa.pa_device_error() == 0


def test_empty_decode_batch_is_a_no_op(pa):
    q = torch.empty(0, 8, 128, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16, device=DEV)
    tables = torch.zeros(0, 4, dtype=torch.int32, device=DEV)
    lens = torch.zeros(0, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    pa.pa_decode(out, q, k, k, tables, lens, 64, 0.1)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("cached,lens", [
    ([100, 0, 50, 0], [40, 0, 1, 0]),     # empty chunks between and after real ones
    ([0], [1]),                           # one query, nothing cached
    ([128, 0], [128, 256]),               # queries ending exactly on a key tile
])
def test_prefill_edge_chunks(pa, cached, lens):
    batch = mixed_chunks(cached, lens, 8, 2, 16, seed=sum(cached) + sum(lens) + 103)
    d, out = run_prefill(pa, batch)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_prefill(batch, k, v)
    if ref.numel():
        assert_close(out, ref, f"prefill edge {cached} {lens}")
    assert pa.pa_device_error() == 0


def test_prefill_chunk_longer_than_max_query_len(pa):
    """A chunk of 300 queries launched with max_query_len 200: the grid covers
    256 rows of it (200 rounded up to a multiple of the CTA's 128). Rows
    0..255 are computed as usual, rows 256..299 are left as they were (NaN
    poison) and the chunk is recorded as PA_ERR_BAD_TABLE."""
    batch = mixed_chunks([40], [300], 8, 2, 16, seed=104)
    d = batch.to(DEV)
    pa.pa_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    out = torch.full_like(d.prefill_q, float("nan"))
    pa.pa_prefill_chunk(out, d.prefill_q, d.k_cache, d.v_cache, d.prefill_block_tables,
                        d.prefill_context_lens, d.query_start_loc, 200, batch.scale)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == pa.PA_ERR_BAD_TABLE
    got = out.cpu()
    assert torch.isnan(got[256:].float()).all(), "rows past the launch were written"
    k, v = oracle_after_append(batch)
    ref, _ = oracle_prefill(batch, k, v)
    assert_close(got[:256], ref[:256], "covered rows of the over-long chunk")


def test_prefill_decreasing_query_start_loc_is_recorded(pa):
    """query_start_loc going backwards (C < 0) is a malformed chunk: skipped
    and recorded, whatever its row count; the well-formed chunk beside it is
    still computed."""
    batch = mixed_chunks([10, 20], [64, 64], 8, 2, 16, seed=105)
    d = batch.to(DEV)
    pa.pa_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    qsl = torch.tensor([0, 64, 32], dtype=torch.int32, device=DEV)  # chunk 1: C = -32
    out = torch.full_like(d.prefill_q, float("nan"))
    pa.pa_prefill_chunk(out, d.prefill_q, d.k_cache, d.v_cache, d.prefill_block_tables,
                        d.prefill_context_lens, qsl, 64, batch.scale)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == pa.PA_ERR_BAD_TABLE
    k, v = oracle_after_append(batch)
    ref, _ = oracle_prefill(batch, k, v)
    assert_close(out.cpu()[:64], ref[:64], "well-formed chunk beside a malformed one")
