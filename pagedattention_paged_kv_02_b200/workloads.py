"""Seeded synthetic inputs for the paged-KV attention path.

This module only builds inputs: random tensors from a seeded generator, a
host-side block allocator that fills block tables the way a serving engine's
block manager would, and the five workload recipes. It holds no attention
arithmetic. The CUDA path's tests, the benchmark and the CPU oracle all consume
what it builds; nothing here calls either of them.

Pool contents are poisoned so that a read past a sequence's valid tokens shows
up as NaN in the result:

* the whole pool starts as NaN;
* one reserved physical block stays NaN and every unused block-table entry
  points at it (a valid id, so a stray read cannot leave the pool);
* positions a step is about to append (written by reshape_and_cache) and
  positions past ``context_len`` in a sequence's last block are NaN.

Sequences can share a prefix: full prefix blocks are the same physical ids in
several table rows, and a partially filled last prefix block is duplicated
(copied on write) into each sharer's first private block, as in the pages'
beam-search example (page "字节跳动 AI Infra (2)", question
"vLLM与PagedAttention的原理": beams share B1 and B3, B6' is a copy).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch


@dataclass
class SeqSpec:
    """One sequence in a step: ``ctx`` valid tokens after the step, of which the
    last ``new_tokens`` are appended by this step (1 for decode, C for a
    prefill chunk). ``group`` >= 0 shares a ``prefix``-token prefix with the
    other sequences of that group."""
    ctx: int
    new_tokens: int = 1
    group: int = -1
    prefix: int = 0


@dataclass
class Batch:
    """A step's inputs. Decode part: ``q`` [B, H_q, D], ``block_tables`` int32
    [B, MB], ``context_lens`` int32 [B]. Prefill part (optional):
    ``prefill_q`` [total_q, H_q, D], ``prefill_block_tables`` int32
    [n_chunks, MBp], ``prefill_context_lens`` int32 [n_chunks],
    ``query_start_loc`` int32 [n_chunks + 1]. Shared: the pool
    ``k_cache``/``v_cache`` [NB, H_kv, bs, D] and the step's new K/V rows
    ``key``/``value`` [T, H_kv, D] with their ``slot_mapping`` int64 [T]
    (prefill tokens first, then one per decode sequence)."""
    name: str
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    key: torch.Tensor
    value: torch.Tensor
    slot_mapping: torch.Tensor
    scale: float
    block_size: int
    poison_block: int
    q: Optional[torch.Tensor] = None
    block_tables: Optional[torch.Tensor] = None
    context_lens: Optional[torch.Tensor] = None
    prefill_q: Optional[torch.Tensor] = None
    prefill_block_tables: Optional[torch.Tensor] = None
    prefill_context_lens: Optional[torch.Tensor] = None
    query_start_loc: Optional[torch.Tensor] = None
    partition_size: int = 0
    k_scale: Optional[torch.Tensor] = None  # 8-bit pools: float32 [H_kv] per-head scales
    v_scale: Optional[torch.Tensor] = None
    sliding_window: int = 0  # > 0: every query sees only its last sliding_window positions
    # shared prefixes of the decode sequences, as the engine's block manager
    # knows them: group g = sequences [decode_group_start[g],
    # decode_group_start[g+1]) sharing their first decode_prefix_lens[g]
    # positions (int32; None when the batch has no groups)
    decode_group_start: Optional[torch.Tensor] = None
    decode_prefix_lens: Optional[torch.Tensor] = None
    max_group_size: int = 0
    max_prefix_len: int = 0

    @property
    def num_blocks(self) -> int:
        return self.k_cache.shape[0]

    @property
    def num_kv_heads(self) -> int:
        return self.k_cache.shape[1]

    @property
    def head_dim(self) -> int:
        return self.k_cache.shape[3]

    @property
    def num_q_heads(self) -> int:
        t = self.q if self.q is not None else self.prefill_q
        return t.shape[1]

    @property
    def dtype(self) -> torch.dtype:
        """Element type of q, out and the new K/V rows."""
        t = self.q if self.q is not None else self.prefill_q
        return t.dtype

    @property
    def fp8(self) -> bool:
        return self.k_cache.dtype == torch.uint8

    @property
    def int8(self) -> bool:
        return self.k_cache.dtype == torch.int8

    @property
    def quantized(self) -> bool:
        """The pool holds 8-bit codes (FP8 E4M3 or INT8) with per-head scales."""
        return self.fp8 or self.int8

    @property
    def num_seqs(self) -> int:
        return 0 if self.q is None else self.q.shape[0]

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    def tensors(self):
        return {k: v for k, v in self.__dict__.items() if isinstance(v, torch.Tensor)}

    def to(self, device) -> "Batch":
        """A copy with every tensor moved to ``device``."""
        kw = dict(self.__dict__)
        for k, v in kw.items():
            if isinstance(v, torch.Tensor):
                kw[k] = v.to(device)
        return Batch(**kw)


class BlockAllocator:
    """Hands out physical block ids in a seeded random order (a block-manager
    fixture: placement in the pool is arbitrary, as paging allows)."""

    def __init__(self, num_blocks: int, gen: torch.Generator):
        self.order = torch.randperm(num_blocks, generator=gen).tolist()
        self.next = 0

    def alloc(self, n: int) -> List[int]:
        if self.next + n > len(self.order):
            raise RuntimeError(f"pool of {len(self.order)} blocks exhausted")
        ids = self.order[self.next:self.next + n]
        self.next += n
        return ids


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _randn(gen, shape, std, dtype):
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * std).to(dtype)


def build_pool(specs: Sequence[SeqSpec], num_kv_heads: int, head_dim: int, block_size: int,
               num_blocks: int, dtype: torch.dtype, std: float, gen: torch.Generator,
               max_blocks_per_seq: Optional[int] = None):
    """Allocate and fill a pool for ``specs``. Returns (k_cache, v_cache,
    block_tables int32 [len(specs), MB], key, value, slot_mapping, poison_block)
    where key/value/slot_mapping list every sequence's appended tokens in spec
    order."""
    H, D, bs = num_kv_heads, head_dim, block_size
    nan = float("nan")
    k_cache = torch.full((num_blocks, H, bs, D), nan, dtype=dtype)
    v_cache = torch.full((num_blocks, H, bs, D), nan, dtype=dtype)
    alloc = BlockAllocator(num_blocks, gen)
    poison = alloc.alloc(1)[0]

    # shared prefixes: full blocks are shared ids, a partial last block is
    # drawn once per group and copied into each sharer's first private block
    groups = {}
    for s in specs:
        if s.group >= 0 and s.group not in groups:
            full = s.prefix // bs
            ids = alloc.alloc(full)
            groups[s.group] = {"ids": ids, "prefix": s.prefix, "partial": None}
    for g in sorted(groups):
        info = groups[g]
        ids = info["ids"]
        if ids:
            idx = torch.tensor(ids)
            k_cache[idx] = _randn(gen, (len(ids), H, bs, D), std, dtype)
            v_cache[idx] = _randn(gen, (len(ids), H, bs, D), std, dtype)
        rem = info["prefix"] % bs
        if rem:
            info["partial"] = (_randn(gen, (H, rem, D), std, dtype),
                               _randn(gen, (H, rem, D), std, dtype))

    rows, private_ids = [], []
    for s in specs:
        if s.ctx < s.new_tokens or s.ctx < 0:
            raise ValueError("ctx must cover the appended tokens")
        shared = groups[s.group]["ids"] if s.group >= 0 else []
        if s.group >= 0 and s.prefix > s.ctx:
            raise ValueError("prefix longer than the sequence")
        need = _ceil_div(s.ctx, bs)
        own = alloc.alloc(max(0, need - len(shared)))
        rows.append(list(shared) + own)
        private_ids.extend(own)
    MB = max_blocks_per_seq if max_blocks_per_seq is not None else max(
        [len(r) for r in rows] + [1])
    if any(len(r) > MB for r in rows):
        raise ValueError("max_blocks_per_seq too small")
    tables = torch.full((len(specs), MB), poison, dtype=torch.int32)
    for i, r in enumerate(rows):
        if r:
            tables[i, :len(r)] = torch.tensor(r, dtype=torch.int32)

    if private_ids:
        idx = torch.tensor(private_ids)
        k_cache[idx] = _randn(gen, (len(private_ids), H, bs, D), std, dtype)
        v_cache[idx] = _randn(gen, (len(private_ids), H, bs, D), std, dtype)

    keys, values, slots = [], [], []
    for i, s in enumerate(specs):
        r = rows[i]
        if s.group >= 0 and groups[s.group]["partial"] is not None:
            pk, pv = groups[s.group]["partial"]
            blk = r[s.prefix // bs]
            k_cache[blk, :, :pk.shape[1]] = pk
            v_cache[blk, :, :pv.shape[1]] = pv
        # positions appended this step and positions past ctx are NaN
        for j in range(s.ctx - s.new_tokens, _ceil_div(s.ctx, bs) * bs):
            blk, off = r[j // bs], j % bs
            k_cache[blk, :, off] = nan
            v_cache[blk, :, off] = nan
        n = s.new_tokens
        keys.append(_randn(gen, (n, H, D), std, dtype))
        values.append(_randn(gen, (n, H, D), std, dtype))
        pos = torch.arange(s.ctx - n, s.ctx)
        blk = torch.tensor(r, dtype=torch.int64)[pos // bs] if n else pos
        slots.append(blk * bs + pos % bs)
    key = torch.cat(keys) if keys else torch.empty(0, H, D, dtype=dtype)
    value = torch.cat(values) if values else torch.empty(0, H, D, dtype=dtype)
    slot_mapping = torch.cat(slots).to(torch.int64) if slots else torch.empty(0, dtype=torch.int64)
    return k_cache, v_cache, tables, key, value, slot_mapping, poison


def prefix_groups(groups: Sequence[int], prefix: int):
    """The group structure of a list of per-sequence group ids (-1: shares
    nothing): (group_start int32 [G+1], prefix_lens int32 [G], largest group,
    longest prefix). Sharing sequences must be listed group by group; each
    non-sharing sequence is a group of one with prefix 0."""
    starts, lens = [0], []
    for i, g in enumerate(groups):
        if i > 0 and g >= 0 and g == groups[i - 1]:
            continue  # same group as the previous sequence
        if g >= 0 and g in groups[:i]:
            raise ValueError("sequences of a group must be consecutive")
        if i > 0:
            starts.append(i)
        lens.append(prefix if g >= 0 else 0)
    if groups:
        starts.append(len(groups))
    else:
        starts = [0]
    sizes = [b - a for a, b in zip(starts[:-1], starts[1:])]
    return (torch.tensor(starts, dtype=torch.int32), torch.tensor(lens, dtype=torch.int32),
            max(sizes + [1]), max(lens + [0]))


def decode_batch(context_lens: Sequence[int], num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, num_blocks: int, dtype=torch.bfloat16,
                 std: float = 1.0, seed: int = 0, scale: Optional[float] = None,
                 groups: Optional[Sequence[int]] = None, prefix: int = 0,
                 max_blocks_per_seq: Optional[int] = None, partition_size: int = 0,
                 name: str = "decode") -> Batch:
    """A decode step: one query per sequence, the last token of each sequence
    appended by this step. ``groups[b]`` >= 0 makes sequences share a
    ``prefix``-token prefix."""
    gen = torch.Generator().manual_seed(seed)
    specs = [SeqSpec(int(c), 1 if c > 0 else 0,
                     -1 if groups is None else int(groups[i]), prefix)
             for i, c in enumerate(context_lens)]
    k, v, tables, key, value, slots, poison = build_pool(
        specs, num_kv_heads, head_dim, block_size, num_blocks, dtype, std, gen,
        max_blocks_per_seq)
    q = _randn(gen, (len(specs), num_q_heads, head_dim), std, dtype)
    grp = {}
    if groups is not None:
        gs, pl, mg, mp = prefix_groups([int(x) for x in groups], prefix)
        grp = dict(decode_group_start=gs, decode_prefix_lens=pl, max_group_size=mg,
                   max_prefix_len=mp)
    return Batch(name=name, k_cache=k, v_cache=v, key=key, value=value, slot_mapping=slots,
                 scale=scale if scale is not None else 1.0 / math.sqrt(head_dim),
                 block_size=block_size, poison_block=poison, q=q, block_tables=tables,
                 context_lens=torch.tensor([int(c) for c in context_lens], dtype=torch.int32),
                 partition_size=partition_size, **grp)


def mixed_batch(cached: Sequence[int], chunk: int, decode_ctx: Sequence[int],
                decode_groups: Optional[Sequence[int]], prefix: int, num_q_heads: int,
                num_kv_heads: int, head_dim: int, block_size: int, num_blocks: int,
                dtype=torch.bfloat16, std: float = 1.0, seed: int = 0,
                name: str = "mixed") -> Batch:
    """Prefill chunks (chunk c: ``chunk`` new query tokens after ``cached[c]``
    cached ones) plus decode sequences, over one pool. The step appends every
    chunk's tokens and one token per decode sequence."""
    gen = torch.Generator().manual_seed(seed)
    pre = [SeqSpec(int(c) + chunk, chunk) for c in cached]
    dec = [SeqSpec(int(c), 1, -1 if decode_groups is None else int(decode_groups[i]), prefix)
           for i, c in enumerate(decode_ctx)]
    k, v, tables, key, value, slots, poison = build_pool(
        pre + dec, num_kv_heads, head_dim, block_size, num_blocks, dtype, std, gen)
    n_pre = len(pre)
    mb_p = max(1, max(_ceil_div(s.ctx, block_size) for s in pre)) if pre else 1
    mb_d = max(1, max(_ceil_div(s.ctx, block_size) for s in dec)) if dec else 1
    pq = _randn(gen, (n_pre * chunk, num_q_heads, head_dim), std, dtype)
    dq = _randn(gen, (len(dec), num_q_heads, head_dim), std, dtype)
    grp = {}
    if decode_groups is not None:
        gs, pl, mg, mp = prefix_groups([int(x) for x in decode_groups], prefix)
        grp = dict(decode_group_start=gs, decode_prefix_lens=pl, max_group_size=mg,
                   max_prefix_len=mp)
    return Batch(name=name, k_cache=k, v_cache=v, key=key, value=value, slot_mapping=slots,
                 scale=1.0 / math.sqrt(head_dim), block_size=block_size, poison_block=poison,
                 q=dq, block_tables=tables[n_pre:, :mb_d].contiguous(),
                 context_lens=torch.tensor([s.ctx for s in dec], dtype=torch.int32),
                 prefill_q=pq, prefill_block_tables=tables[:n_pre, :mb_p].contiguous(),
                 prefill_context_lens=torch.tensor([s.ctx for s in pre], dtype=torch.int32),
                 query_start_loc=torch.arange(0, n_pre + 1, dtype=torch.int32) * chunk, **grp)


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------
def tiny_fp32(seed: int = 0) -> Batch:
    """4 sequences of 5/17/33/40 tokens, 4 q = 4 kv heads, head_dim 64,
    16-token blocks in a 16-block pool, fp32, N(0,1), scale 1/8."""
    return decode_batch([5, 17, 33, 40], 4, 4, 64, 16, 16, torch.float32, 1.0, seed,
                        scale=1.0 / 8.0, name="tiny_fp32_b4_d64")


def llama7b_decode(seed: int = 0, num_blocks: int = 16384, block_size: int = 16,
                   head_dim: int = 128) -> Batch:
    """Llama-2-7B-shaped decode: 64 sequences with lengths uniform in
    [128, 2048], 32/32 heads, head_dim 128, 16-token blocks, 16384-block pool,
    bf16, N(0,1). Other block sizes and head_dim 64 keep the lengths (and,
    for block sizes, the pool's bytes)."""
    gen = torch.Generator().manual_seed(seed + 7919)
    lens = torch.randint(128, 2049, (64,), generator=gen).tolist()
    nb, mb = num_blocks * 16 // block_size, 2048 // block_size  # same pool bytes
    return decode_batch(lens, 32, 32, head_dim, block_size, nb, torch.bfloat16, 1.0, seed,
                        max_blocks_per_seq=mb,
                        name=f"llama7b_decode_b64_h32_d{head_dim}_bs{block_size}")


def gqa_decode(seed: int = 0, num_blocks: int = 32768, block_size: int = 16,
               head_dim: int = 128) -> Batch:
    """GQA decode: 128 sequences, lengths log-normal with median 1024 and
    sigma 0.75 (natural-log scale) clipped to [16, 4096], 64 q / 8 kv heads,
    head_dim 128, 16-token blocks, 32768-block pool, bf16, N(0,1)."""
    gen = torch.Generator().manual_seed(seed + 104729)
    z = torch.randn(128, generator=gen, dtype=torch.float64)
    lens = torch.exp(math.log(1024.0) + 0.75 * z).round().clamp(16, 4096).to(torch.int64).tolist()
    nb, mb = num_blocks * 16 // block_size, 4096 // block_size  # same pool bytes
    return decode_batch(lens, 64, 8, head_dim, block_size, nb, torch.bfloat16, 1.0, seed,
                        max_blocks_per_seq=mb,
                        name=f"gqa_decode_b128_h64kv8_d{head_dim}_bs{block_size}")


def long_context_decode(seed: int = 0, num_blocks: int = 8192) -> Batch:
    """Long-context split-KV decode: 4 sequences of 32K/64K/96K/128K tokens,
    32 q / 8 kv heads, head_dim 128, 64-token blocks, 8192-block pool, bf16,
    N(0, 0.5), 512-token KV partitions."""
    return decode_batch([32768, 65536, 98304, 131072], 32, 8, 128, 64, num_blocks, torch.bfloat16,
                        0.5, seed, max_blocks_per_seq=2048, partition_size=512,
                        name="long_ctx_decode_b4_h32kv8_d128_bs64_p512")


def mixed_prefill_decode(seed: int = 0, num_blocks: int = 16384, head_dim: int = 128) -> Batch:
    """8 prefill chunks of 512 query tokens after round(i*4096/7) cached tokens
    (i = 0..7), plus 192 decode sequences in 24 groups of 8 beams sharing a
    1024-token prefix (64 shared blocks) with private tails uniform in
    [64, 512]; 32 q / 8 kv heads, head_dim 128, 16-token blocks, bf16, N(0,1)."""
    gen = torch.Generator().manual_seed(seed + 1299709)
    cached = [round(i * 4096 / 7) for i in range(8)]
    tails = torch.randint(64, 513, (192,), generator=gen).tolist()
    ctx = [1024 + t for t in tails]
    groups = [b // 8 for b in range(192)]
    return mixed_batch(cached, 512, ctx, groups, 1024, 32, 8, head_dim, 16, num_blocks,
                       torch.bfloat16, 1.0, seed,
                       name=f"mixed_prefill8x512_decode192_h32kv8_d{head_dim}_bs16")


def to_fp8(batch: Batch, k_amax: float = 4.0, v_amax: float = 4.0) -> Batch:
    """A copy of a decode batch whose pool holds FP8 E4M3 codes: each cached
    value divided by its K/V head's scale (amax / 448, one per head for K
    and one for V) and cast with torch's float8_e4m3fn conversion after
    clamping to the E4M3 range. NaN poison stays NaN (code 0x7F). q and the
    step's new K/V rows keep their type (the append quantises them)."""
    H = batch.num_kv_heads
    ks = torch.full((H,), k_amax / 448.0, dtype=torch.float32)
    vs = torch.full((H,), v_amax / 448.0, dtype=torch.float32)

    def enc(pool, sc):
        x = pool.float() / sc[None, :, None, None]
        x = torch.where(torch.isnan(x), x, x.clamp(-448.0, 448.0))
        return x.to(torch.float8_e4m3fn).view(torch.uint8)

    kw = dict(batch.__dict__)
    kw.update(k_cache=enc(batch.k_cache, ks), v_cache=enc(batch.v_cache, vs), k_scale=ks,
              v_scale=vs, name=batch.name + "_fp8")
    return Batch(**kw)


def to_int8(batch: Batch, k_amax: float = 4.0, v_amax: float = 4.0) -> Batch:
    """A copy of a decode batch whose pool holds INT8 codes: each cached value
    divided by its K/V head's scale (amax / 127) and rounded to the nearest
    integer (torch.round: ties to even), clamped to [-127, 127]. NaN poison
    becomes 0 (INT8 has no NaN). q and the step's new K/V rows keep their
    type (the append quantises them)."""
    H = batch.num_kv_heads
    ks = torch.full((H,), k_amax / 127.0, dtype=torch.float32)
    vs = torch.full((H,), v_amax / 127.0, dtype=torch.float32)

    def enc(pool, sc):
        x = pool.float() / sc[None, :, None, None]
        x = torch.nan_to_num(x, nan=0.0).round().clamp(-127.0, 127.0)
        return x.to(torch.int8)

    kw = dict(batch.__dict__)
    kw.update(k_cache=enc(batch.k_cache, ks), v_cache=enc(batch.v_cache, vs), k_scale=ks,
              v_scale=vs, name=batch.name + "_int8")
    return Batch(**kw)


def llama7b_decode_fp8(seed: int = 0, num_blocks: int = 16384, block_size: int = 16) -> Batch:
    """The Llama-2-7B-shaped decode batch with an FP8 E4M3 pool."""
    return to_fp8(llama7b_decode(seed, num_blocks, block_size))


def gqa_decode_fp8(seed: int = 0, num_blocks: int = 32768, block_size: int = 16) -> Batch:
    """The GQA decode batch with an FP8 E4M3 pool."""
    return to_fp8(gqa_decode(seed, num_blocks, block_size))


def llama7b_decode_int8(seed: int = 0, num_blocks: int = 16384, block_size: int = 16) -> Batch:
    """The Llama-2-7B-shaped decode batch with an INT8 pool."""
    return to_int8(llama7b_decode(seed, num_blocks, block_size))


def gqa_decode_int8(seed: int = 0, num_blocks: int = 32768, block_size: int = 16) -> Batch:
    """The GQA decode batch with an INT8 pool."""
    return to_int8(gqa_decode(seed, num_blocks, block_size))


WORKLOADS = {
    "tiny_fp32": tiny_fp32,
    "llama7b_decode": llama7b_decode,
    "gqa_decode": gqa_decode,
    "long_context_decode": long_context_decode,
    "mixed_prefill_decode": mixed_prefill_decode,
    "llama7b_decode_fp8": llama7b_decode_fp8,
    "gqa_decode_fp8": gqa_decode_fp8,
    "llama7b_decode_int8": llama7b_decode_int8,
    "gqa_decode_int8": gqa_decode_int8,
}
