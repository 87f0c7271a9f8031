"""GPU parity of the decode step (reshape_and_cache then pa_decode) against the
fp64 oracle, through the C ABI: small ragged cases spanning many chunks and
partitions, every head-grouping the kernels tile differently, the five
workloads at full size, and the edge cases (empty, single-token and
block-boundary contexts, padding slots, bad table entries, bounded waits)."""
import pytest
import torch

import oracle
from helpers import (assert_close, bits, gpu_decode, oracle_after_append, oracle_decode)
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


def step(pa, batch, partition_size=None):
    dev = batch.to(DEV)
    pa.pa_reshape_and_cache(dev.key, dev.value, dev.k_cache, dev.v_cache, dev.slot_mapping)
    out = gpu_decode(pa, dev, partition_size)
    torch.cuda.synchronize()
    return dev, out


CASES = [
    # ctxs, H_q, H_kv, D, bs, dtype, partition
    ([1, 15, 16, 17, 100, 513, 1500], 8, 8, 128, 16, torch.bfloat16, 0),
    ([1, 15, 16, 17, 100, 513, 1500], 8, 8, 128, 16, torch.bfloat16, 64),
    ([1, 15, 16, 17, 100, 513, 1500], 8, 8, 128, 16, torch.bfloat16, -1),
    ([33, 700, 1024, 2047], 32, 4, 128, 32, torch.bfloat16, 512),
    ([5, 64, 65, 999], 16, 1, 64, 64, torch.bfloat16, 128),
    ([200, 1200], 32, 1, 128, 16, torch.bfloat16, 256),      # 32 heads per kv head: 2 tiles
    ([300, 17], 16, 16, 64, 16, torch.bfloat16, 0),
    ([1, 15, 16, 17, 100, 513], 8, 2, 64, 16, torch.float32, 0),
    ([1, 15, 16, 17, 100, 513], 8, 2, 128, 32, torch.float32, 64),
    ([40, 900], 12, 1, 128, 64, torch.float32, 256),         # 12 heads per kv head: 2 tiles
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0][-1]}tok-h{c[1]}kv{c[2]}-d{c[3]}"
                         f"-bs{c[4]}-{str(c[5])[6:]}-p{c[6]}")
def test_decode_small(pa, case):
    ctxs, Hq, Hkv, D, bs, dt, part = case
    nb = sum(-(-c // bs) for c in ctxs) + 7
    batch = W.decode_batch(ctxs, Hq, Hkv, D, bs, nb, dt, seed=len(ctxs) * 31 + Hq)
    dev, out = step(pa, batch, part)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_decode(batch, k, v)
    assert_close(out, ref, f"decode {case}")
    assert pa.pa_device_error() == 0


def test_reshape_bit_exact_tiny(pa):
    batch = W.tiny_fp32()
    dev, _ = step(pa, batch)
    k, v = oracle_after_append(batch)
    assert torch.equal(bits(dev.k_cache.cpu()), bits(k))
    assert torch.equal(bits(dev.v_cache.cpu()), bits(v))


@pytest.mark.parametrize("name", ["tiny_fp32", "llama7b_decode", "gqa_decode",
                                  "long_context_decode"])
def test_workload_full(pa, name):
    """The decode workloads at full size, every output compared."""
    batch = W.WORKLOADS[name]()
    dev, out = step(pa, batch)
    k, v = oracle_after_append(batch)
    assert torch.equal(bits(dev.k_cache.cpu()), bits(k)), "cache scatter not bit-exact"
    ref, _ = oracle_decode(batch, k, v)
    assert_close(out, ref, name)
    assert pa.pa_device_error() == 0


def test_partition_choices_agree(pa):
    """Automatic, fixed and no split give the same answer within tolerance,
    and repeated runs are bit-identical."""
    batch = W.decode_batch([512, 1024, 1536, 1, 1500], 16, 2, 128, 16, 400, torch.bfloat16,
                           seed=9)
    dev, out0 = step(pa, batch, 0)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_decode(batch, k, v)
    for part in (16, 512, 1024, -1):
        out = gpu_decode(pa, dev, part)
        assert_close(out, ref, f"partition {part}")
    again = gpu_decode(pa, dev, 0)
    assert torch.equal(bits(out0), bits(again))


def test_empty_sequence_gives_zero(pa):
    batch = W.decode_batch([0, 37, 0], 4, 2, 128, 16, 16, torch.bfloat16, seed=4)
    dev, out = step(pa, batch)
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_decode(batch, k, v)
    assert_close(out, ref, "empty")


def test_shared_prefix_beams(pa):
    """Beams sharing prefix blocks, including a partially filled shared block
    copied on write, match the oracle."""
    batch = W.decode_batch([100, 130, 77, 95], 8, 2, 128, 16, 64, torch.bfloat16, seed=12,
                           groups=[0, 0, 1, 1], prefix=70)
    dev, out = step(pa, batch)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_decode(batch, k, v)
    assert_close(out, ref, "beams")


def test_padding_and_bad_slots(pa):
    """A negative slot is skipped; a slot past the pool is skipped and
    recorded; nothing else in the pool changes."""
    batch = W.decode_batch([20, 40], 4, 4, 64, 16, 8, torch.float32, seed=2)
    dev = batch.to(DEV)
    slots = dev.slot_mapping.clone()
    slots[0] = -1
    slots[1] = dev.k_cache.shape[0] * 16
    before = dev.k_cache.clone()
    pa.pa_reshape_and_cache(dev.key, dev.value, dev.k_cache, dev.v_cache, slots)
    torch.cuda.synchronize()
    assert torch.equal(bits(before), bits(dev.k_cache))
    assert pa.pa_device_error() == pa.PA_ERR_BAD_TABLE


def test_bad_block_id_recorded_not_read(pa):
    """A table entry outside the pool is caught by the table check, skipped by
    the kernel (never dereferenced) and recorded; other sequences are
    unaffected."""
    batch = W.decode_batch([50, 60], 4, 2, 128, 16, 16, torch.bfloat16, seed=3)
    clean, out_clean = step(pa, batch)
    dev = batch.to(DEV)
    pa.pa_reshape_and_cache(dev.key, dev.value, dev.k_cache, dev.v_cache, dev.slot_mapping)
    assert pa.pa_check_tables(dev.block_tables, dev.context_lens, 16, 16) == 0
    dev.block_tables[1, 1] = 1 << 20
    assert pa.pa_check_tables(dev.block_tables, dev.context_lens, 16, 16) == 1
    pa.pa_device_error(clear=True)
    out = gpu_decode(pa, dev)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == pa.PA_ERR_BAD_TABLE
    assert torch.equal(bits(out[0]), bits(out_clean[0]))


def test_bounded_wait_times_out_and_context_survives(pa):
    pa.pa_device_error(clear=True)
    pa.pa_selftest_bounded_wait(2_000_000)  # 2 ms on a barrier nothing completes
    torch.cuda.synchronize()
    assert pa.pa_device_error(clear=True) == pa.PA_ERR_TIMEOUT
    batch = W.tiny_fp32()
    dev, out = step(pa, batch)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_decode(batch, k, v)
    assert_close(out, ref, "after timeout")
    assert pa.pa_device_error() == 0
