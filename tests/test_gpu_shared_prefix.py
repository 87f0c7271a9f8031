"""GPU parity of the shared-prefix decode (pa_decode_shared_prefix) against
the fp64 oracle's plain decode, through the C ABI. The result must be
pa_decode's: reading a shared prefix once for all the sequences of a group
is a reformulation, not a different attention.

Cases: the mixed workload's 192 beams (24 groups of 8 sharing a 1024-token
prefix) at full size; 8 beams of a GQA model (8 query heads per KV head:
64 rows per CTA) whose prefix ends inside a block copied on write; groups of
different sizes beside sequences that share nothing, with a group larger
than one CTA's rows; head_dim 64 with 64-token blocks; partition sizes that
give many slots (the many-partition merge) or one; a member whose context
is shorter than the declared prefix; and malformed groups, which are
recorded."""
import pytest
import torch

import oracle
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


@pytest.fixture(autouse=True)
def clean_error_word(pa):
    pa.pa_device_error(clear=True)
    yield
    torch.cuda.synchronize()


def shared_decode(pa, batch, d, part=0, context_lens=None, group_start=None, prefix_lens=None):
    """pa_decode_shared_prefix on a device batch whose step was appended."""
    B, H_q, D = d.q.shape
    H_kv = d.k_cache.shape[1]
    gs = d.decode_group_start if group_start is None else group_start
    pl = d.decode_prefix_lens if prefix_lens is None else prefix_lens
    lens = d.context_lens if context_lens is None else context_lens
    n = pa.pa_decode_shared_prefix_workspace_size(B, H_q, H_kv, D, pl.numel(),
                                                  batch.max_group_size, batch.max_prefix_len,
                                                  batch.max_context_len, part)
    assert n > 0
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    out = torch.full_like(d.q, float("nan"))
    pa.pa_decode_shared_prefix(out, d.q, d.k_cache, d.v_cache, d.block_tables, lens, gs, pl,
                               batch.max_group_size, batch.max_prefix_len,
                               batch.max_context_len, batch.scale, part, ws)
    torch.cuda.synchronize()
    return out


def appended(pa, batch):
    d = batch.to(DEV)
    pa.pa_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    return d


def test_mixed_workload_beams_full(pa):
    """The mixed batch's decode part: 24 groups x 8 beams, 1024 shared tokens."""
    batch = W.mixed_prefill_decode()
    d = appended(pa, batch)
    out = shared_decode(pa, batch, d)
    k, v = oracle_after_append(batch)
    ref, _ = oracle.decode(batch.q, k, v, batch.block_tables, batch.context_lens, batch.scale)
    assert_close(out, ref, "shared-prefix decode, mixed batch")
    assert pa.pa_device_error() == 0


def _grouped(ctxs, groups, prefix, Hq, Hkv, D, bs, seed):
    nb = sum(-(-c // bs) for c in ctxs) + 8
    return W.decode_batch(ctxs, Hq, Hkv, D, bs, nb, torch.bfloat16, seed=seed, groups=groups,
                          prefix=prefix)


CASES = [
    # ctxs, groups, prefix, H_q, H_kv, D, bs, partition
    # 8 GQA beams (8 q heads per kv head: 64 rows), prefix ending mid-block
    ([1000 + t for t in (1, 17, 100, 333, 64, 500, 2, 250)], [0] * 8, 1000, 64, 8, 128, 16, 0),
    # groups of 3 and 20 (80 rows: two row tiles) between sequences sharing nothing
    ([400, 350, 301, 900, 310 + 7] + [300 + 13 * i for i in range(1, 20)] + [5, 2000],
     [0, 0, 0, -1] + [1] * 20 + [-1, -1], 300, 32, 8, 128, 32, 0),
    # head_dim 64, 64-token blocks, 8 heads per kv head
    ([130 + t for t in (1, 64, 65, 700)] + [131, 600], [0, 0, 0, 0, 1, 1], 130, 16, 2, 64, 64,
     0),
    # 64-token partitions: 16 prefix slots + 24 tail slots (the many-slot merge)
    ([1024 + t for t in (3, 100, 511, 64)], [0] * 4, 1024, 32, 8, 128, 16, 64),
    # one partition each
    ([1024 + t for t in (3, 100, 511, 64)], [0] * 4, 1024, 32, 8, 128, 16, -1),
    # MQA-like: 16 q heads on one kv head, 3 beams (48 rows)
    ([200 + t for t in (9, 40, 1)], [0] * 3, 200, 16, 1, 128, 16, 0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"n{len(c[0])}-p{c[2]}-h{c[3]}kv{c[4]}"
                         f"-d{c[5]}-bs{c[6]}-part{c[7]}")
def test_shared_prefix_cases(pa, case):
    ctxs, groups, prefix, Hq, Hkv, D, bs, part = case
    batch = _grouped(ctxs, groups, prefix, Hq, Hkv, D, bs, seed=sum(ctxs) + Hq)
    d = appended(pa, batch)
    out = shared_decode(pa, batch, d, part)
    k, v = oracle_after_append(batch)
    ref, _ = oracle_decode(batch, k, v)
    assert_close(out, ref, f"shared-prefix decode {case[2:]}")
    assert pa.pa_device_error() == 0


def test_member_shorter_than_the_prefix(pa):
    """Member 2's context is cut to 600 tokens, inside the declared 1000-token
    prefix: the group's shared part shrinks to 600 for every member (the
    others read positions 600..999 through their own tables)."""
    ctxs = [1000 + t for t in (40, 7, 300)]
    batch = _grouped(ctxs, [0, 0, 0], 1000, 32, 8, 128, 16, seed=5)
    d = appended(pa, batch)
    lens = batch.context_lens.clone()
    lens[2] = 600
    out = shared_decode(pa, batch, d, context_lens=lens.to(DEV))
    k, v = oracle_after_append(batch)
    ref, _ = oracle.decode(batch.q, k, v, batch.block_tables, lens, batch.scale)
    assert_close(out, ref, "member shorter than the prefix")
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("bad", ["decreasing", "not_covering", "too_long_prefix"])
def test_malformed_groups_are_recorded(pa, bad):
    ctxs = [500 + t for t in (1, 2, 3, 4)]
    batch = _grouped(ctxs, [0, 0, 1, 1], 400, 8, 2, 128, 16, seed=6)
    d = appended(pa, batch)
    gs = batch.decode_group_start.clone()
    pl = batch.decode_prefix_lens.clone()
    if bad == "decreasing":
        gs[1] = 3
        gs[2] = 1
    elif bad == "not_covering":
        gs[2] = 3
    else:
        pl[1] = batch.max_prefix_len + 16
    shared_decode(pa, batch, d, group_start=gs.to(DEV), prefix_lens=pl.to(DEV))
    assert pa.pa_device_error() == pa.PA_ERR_BAD_TABLE
