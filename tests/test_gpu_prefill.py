"""GPU parity of chunked prefill (tcgen05 tensor-core kernel) against the fp64
oracle, through the C ABI: ragged chunks that start mid-tile, span several
128-key tiles, end in partial blocks and partial tiles, with every block size
and head grouping; chunk length 1 against decode; and the mixed workload
(8 x 512-token chunks after 0..4096 cached tokens plus 192 shared-prefix
decode sequences) at full size, every output of both."""
import pytest
import torch

import oracle
from helpers import assert_close, bits, gpu_decode, oracle_after_append
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


def run_prefill(pa, batch):
    d = batch.to(DEV)
    pa.pa_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    out = torch.full_like(d.prefill_q, float("nan"))
    qsl = batch.query_start_loc
    max_q = int((qsl[1:] - qsl[:-1]).max())
    pa.pa_prefill_chunk(out, d.prefill_q, d.k_cache, d.v_cache, d.prefill_block_tables,
                        d.prefill_context_lens, d.query_start_loc, max_q, batch.scale)
    torch.cuda.synchronize()
    return d, out


def oracle_prefill(batch, k, v, select=None):
    return oracle.prefill(batch.prefill_q, k, v, batch.prefill_block_tables,
                          batch.prefill_context_lens, batch.query_start_loc, batch.scale,
                          select=select)


CASES = [
    # (cached per chunk, chunk lengths), H_q, H_kv, bs
    # groups of even size put two query heads' same rows in one CTA, odd ones
    # (1, 3) two consecutive 128-row tiles of one head
    (([0, 0, 100, 37], [5, 128, 129, 300]), 8, 2, 16),
    (([1000, 300, 0], [64, 1, 257]), 4, 4, 32),
    (([250, 700], [200, 77]), 8, 1, 64),
    (([16, 127, 128], [16, 1, 129]), 32, 8, 16),
    (([0, 333], [384, 130]), 4, 2, 16),   # group 2: each head pair is a whole group
    (([40, 0], [300, 129]), 6, 2, 32),    # group 3: row pairs
]


def mixed_chunks(cached, lens, Hq, Hkv, bs, seed, D=128):
    """Chunks of differing lengths: built one length at a time, then merged."""
    nb = sum(-(-(c + n) // bs) for c, n in zip(cached, lens)) + 8
    gen = torch.Generator().manual_seed(seed)
    from pagedattention_paged_kv_02_b200.workloads import SeqSpec, build_pool, Batch, _randn
    specs = [SeqSpec(c + n, n) for c, n in zip(cached, lens)]
    k, v, tables, key, value, slots, poison = build_pool(specs, Hkv, D, bs, nb,
                                                         torch.bfloat16, 1.0, gen)
    qsl = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32)
    q = _randn(gen, (int(qsl[-1]), Hq, D), 1.0, torch.bfloat16)
    return Batch(name="chunks", k_cache=k, v_cache=v, key=key, value=value, slot_mapping=slots,
                 scale=D ** -0.5, block_size=bs, poison_block=poison, prefill_q=q,
                 prefill_block_tables=tables,
                 prefill_context_lens=torch.tensor([s.ctx for s in specs], dtype=torch.int32),
                 query_start_loc=qsl)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"h{c[1]}kv{c[2]}-bs{c[3]}-{max(c[0][1])}q")
def test_prefill_small(pa, case):
    (cached, lens), Hq, Hkv, bs = case
    batch = mixed_chunks(cached, lens, Hq, Hkv, bs, seed=sum(lens) + Hq)
    d, out = run_prefill(pa, batch)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_prefill(batch, k, v)
    assert_close(out, ref, f"prefill {case}")
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"h{c[1]}kv{c[2]}-bs{c[3]}-{max(c[0][1])}q")
def test_prefill_head_dim_64(pa, case):
    (cached, lens), Hq, Hkv, bs = case
    batch = mixed_chunks(cached, lens, Hq, Hkv, bs, seed=sum(lens) + Hq + 64, D=64)
    d, out = run_prefill(pa, batch)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_prefill(batch, k, v)
    assert_close(out, ref, f"prefill D64 {case}")
    assert pa.pa_device_error() == 0


def test_prefill_single_query_equals_decode(pa):
    """A chunk of one query is a decode step over the same context."""
    batch = mixed_chunks([500, 2000, 31], [1, 1, 1], 8, 2, 16, seed=77)
    d, out = run_prefill(pa, batch)
    dec = torch.empty_like(d.prefill_q)
    pa.pa_decode(dec, d.prefill_q, d.k_cache, d.v_cache, d.prefill_block_tables,
                 d.prefill_context_lens, int(batch.prefill_context_lens.max()), batch.scale,
                 -1)  # one partition per sequence: no workspace needed
    torch.cuda.synchronize()
    assert_close(out, dec.double().cpu(), "prefill C=1 vs decode")


def test_mixed_workload_full(pa):
    """The mixed prefill + shared-prefix decode step at full size."""
    batch = W.mixed_prefill_decode()
    d, out = run_prefill(pa, batch)
    k, v = oracle_after_append(batch)
    assert torch.equal(bits(d.k_cache.cpu()), bits(k)), "cache scatter not bit-exact"
    assert torch.equal(bits(d.v_cache.cpu()), bits(v)), "cache scatter not bit-exact"
    # prefill: every query row of every chunk, all heads
    ref, _ = oracle_prefill(batch, k, v)
    assert_close(out, ref, "mixed prefill")
    for c in range(batch.query_start_loc.numel() - 1):  # each chunk on its own too
        r0, r1 = int(batch.query_start_loc[c]), int(batch.query_start_loc[c + 1])
        assert_close(out[r0:r1], ref[r0:r1], f"mixed prefill chunk {c}")
    # decode part, every output
    dec = gpu_decode(pa, d)
    torch.cuda.synchronize()
    dref, _ = oracle.decode(batch.q, k, v, batch.block_tables, batch.context_lens, batch.scale)
    assert_close(dec, dref, "mixed decode")
    assert pa.pa_device_error() == 0
