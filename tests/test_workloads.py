"""The seeded input generators build what the workload recipes say: shapes,
length distributions, poisoned unused slots, shared-prefix blocks, and slot
mappings that point at each sequence's appended positions."""
import math

import torch

from pagedattention_paged_kv_02_b200 import workloads as W


def _positions(batch, b, tables, lens):
    bs = batch.block_size
    return [(int(tables[b, j // bs]), j % bs) for j in range(int(lens[b]))]


def test_decode_batch_poison_and_slots():
    bt = W.decode_batch([1, 16, 17, 40], 4, 2, 8, 16, 32, torch.float32, seed=3)
    H = bt.num_kv_heads
    assert bt.q.shape == (4, 4, 8) and bt.block_tables.shape == (4, 3)
    assert bt.key.shape == (4, H, 8) and bt.slot_mapping.dtype == torch.int64
    pool_k = bt.k_cache
    for b in range(4):
        pos = _positions(bt, b, bt.block_tables, bt.context_lens)
        # cached positions are finite, the appended one is NaN until written
        for blk, off in pos[:-1]:
            assert torch.isfinite(pool_k[blk, :, off]).all()
        blk, off = pos[-1]
        assert torch.isnan(pool_k[blk, :, off]).all()
        assert int(bt.slot_mapping[b]) == blk * 16 + off
        # past ctx in the last block: NaN
        n = int(bt.context_lens[b])
        for j in range(n, -(-n // 16) * 16):
            assert torch.isnan(pool_k[int(bt.block_tables[b, j // 16]), :, j % 16]).all()
        # unused table entries point at the NaN block
        used = -(-n // 16)
        assert torch.all(bt.block_tables[b, used:] == bt.poison_block)
    assert torch.isnan(pool_k[bt.poison_block]).all()


def test_seeded_and_distinct():
    a = W.decode_batch([5, 9], 2, 2, 8, 4, 8, torch.bfloat16, seed=1)
    b = W.decode_batch([5, 9], 2, 2, 8, 4, 8, torch.bfloat16, seed=1)
    c = W.decode_batch([5, 9], 2, 2, 8, 4, 8, torch.bfloat16, seed=2)
    for k, v in a.tensors().items():
        assert torch.equal(v.view(torch.uint8) if v.is_floating_point() else v,
                           getattr(b, k).view(torch.uint8) if v.is_floating_point()
                           else getattr(b, k)), k
    assert not torch.equal(a.q, c.q)


def test_shared_prefix_blocks():
    bt = W.decode_batch([40, 50, 45], 2, 1, 8, 16, 20, torch.float32, seed=4,
                        groups=[0, 0, 0], prefix=37)
    # 37 tokens: blocks 0 and 1 shared, block 2 a private copy of the partial
    assert torch.equal(bt.block_tables[0, :2], bt.block_tables[1, :2])
    assert torch.equal(bt.block_tables[0, :2], bt.block_tables[2, :2])
    third = bt.block_tables[:, 2].tolist()
    assert len(set(third)) == 3
    k = bt.k_cache
    for b in (1, 2):
        assert torch.equal(k[third[0], :, :5], k[third[b], :, :5])
        assert not torch.equal(k[third[0], :, 5:7], k[third[b], :, 5:7])


def test_tiny_recipe():
    bt = W.tiny_fp32()
    assert bt.context_lens.tolist() == [5, 17, 33, 40]
    assert bt.k_cache.shape == (16, 4, 16, 64) and bt.dtype == torch.float32
    used = set()
    for b, n in enumerate([1, 2, 3, 3]):
        used.update(bt.block_tables[b, :n].tolist())
    assert len(used) == 9 and bt.poison_block not in used
    assert bt.scale == 1 / 8


def test_mixed_recipe_structure():
    bt = W.mixed_prefill_decode()
    assert bt.prefill_q.shape == (8 * 512, 32, 128)
    assert bt.query_start_loc.tolist() == [512 * i for i in range(9)]
    cached = [round(i * 4096 / 7) for i in range(8)]
    assert bt.prefill_context_lens.tolist() == [c + 512 for c in cached]
    assert bt.q.shape == (192, 32, 128) and bt.slot_mapping.numel() == 8 * 512 + 192
    lens = bt.context_lens
    assert int(lens.min()) >= 1024 + 64 and int(lens.max()) <= 1024 + 512
    for g in range(24):
        rows = bt.block_tables[8 * g:8 * g + 8, :64]
        assert torch.all(rows == rows[0])
    assert len(set(bt.block_tables[:8, 0].tolist())) == 1
    assert len(set(bt.block_tables[::8, 0].tolist())) == 24


def test_gqa_lengths():
    z = torch.randn(128, generator=torch.Generator().manual_seed(104729), dtype=torch.float64)
    lens = torch.exp(math.log(1024.0) + 0.75 * z).round().clamp(16, 4096)
    assert 600 < float(lens.median()) < 1700
