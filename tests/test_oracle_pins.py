"""Pins for the fp64 CPU oracle, against things other than the oracle itself:
values the pages print, a library attention routine (torch's fp64
scaled_dot_product_attention on contiguous K/V), closed forms, special cases
and invariants that a dropped term, a wrong index or sign, or a transposed
operand would break.

Pages cited by title and section:
* «字节跳动 AI Infra (2)», question «vLLM与PagedAttention的原理»: block pool,
  block tables (A: 40 tokens -> [B2, B5, B7]; B: 20 tokens -> [B0, B4]),
  beams sharing B1, B3 with a copy-on-write B6'.
* same page, question «KV Cache原理与优化»: step-t formulas.
* «LLM推理优化», section 1.2 (KV size example), 1.3 (GQA/MQA), 2.3 (causal),
  3.2 (block counts).
* «字节跳动 AI Infra (2)», FlashDecoding row: split along the KV length.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

F64 = torch.float64


# ---------------------------------------------------------------------------
# helpers (test-side, independent of the oracle's C code)
# ---------------------------------------------------------------------------
def place(seqs_k, seqs_v, tables, num_blocks, bs, dtype=torch.float32, fill=float("nan")):
    """Write contiguous per-sequence K/V ([H_kv, ctx, D] each) into a fresh pool
    following the given block tables; everything else holds ``fill``."""
    H, _, D = seqs_k[0].shape
    kc = torch.full((num_blocks, H, bs, D), fill, dtype=dtype)
    vc = torch.full((num_blocks, H, bs, D), fill, dtype=dtype)
    for k, v, row in zip(seqs_k, seqs_v, tables):
        for j in range(k.shape[1]):
            kc[row[j // bs], :, j % bs] = k[:, j].to(dtype)
            vc[row[j // bs], :, j % bs] = v[:, j].to(dtype)
    return kc, vc


def pad_tables(rows, width, pad):
    t = torch.full((len(rows), width), pad, dtype=torch.int32)
    for i, r in enumerate(rows):
        t[i, :len(r)] = torch.tensor(r, dtype=torch.int32)
    return t


def sdpa(q, k, v, scale, causal=False):
    """torch's attention routine in fp64: q [H_q, Lq, D], k/v [H_kv, Lk, D]."""
    return F.scaled_dot_product_attention(q[None].to(F64), k[None].to(F64), v[None].to(F64),
                                          scale=scale, is_causal=causal,
                                          enable_gqa=q.shape[0] != k.shape[0])[0]


def random_paged(ctxs, H_q, H_kv, D, bs, seed, dtype=torch.float32, spare=3):
    """Random contiguous K/V per sequence placed in a pool at random block ids."""
    g = torch.Generator().manual_seed(seed)
    need = [-(-c // bs) for c in ctxs]
    NB = sum(need) + spare
    perm = torch.randperm(NB, generator=g).tolist()
    rows, at = [], 0
    for n in need:
        rows.append(perm[at:at + n])
        at += n
    pad = perm[-1]  # an unused id: every padded entry points at a NaN block
    ks = [torch.randn(H_kv, c, D, generator=g).to(dtype) for c in ctxs]
    vs = [torch.randn(H_kv, c, D, generator=g).to(dtype) for c in ctxs]
    q = torch.randn(len(ctxs), H_q, D, generator=g).to(dtype)
    kc, vc = place(ks, vs, rows, NB, bs, dtype)
    MB = max(need + [1])
    return q, ks, vs, kc, vc, pad_tables(rows, MB, pad), torch.tensor(ctxs, dtype=torch.int32)


# ---------------------------------------------------------------------------
# values the pages print
# ---------------------------------------------------------------------------
def test_kv_cache_size_example(golden):
    ex = golden["kv_cache_size"]
    n = oracle.kv_cache_bytes(ex["num_layers"], ex["num_heads"], ex["seq_len"], ex["head_dim"],
                              ex["dtype_bytes"])
    assert round(n / 1e9, 1) == ex["printed_gb"]
    # the reading "GB = 10^9 bytes": the same count is exactly 10 GiB
    assert n == 10 * 2 ** 30
    # linear in every factor, and K and V both counted
    assert oracle.kv_cache_bytes(1, 1, 1, 1, 1) == 2
    assert oracle.kv_cache_bytes(80, 64, 8192, 128, 2) == 2 * n


def test_block_counts_example(golden):
    ex = golden["block_counts"]
    counts = [oracle.blocks_needed(t, ex["block_size"]) for t, _ in ex["sequences"]]
    assert counts == [c for _, c in ex["sequences"]]
    assert sum(counts) == ex["printed_total"]
    assert oracle.blocks_needed(0) == 0
    assert oracle.blocks_needed(16) == 1 and oracle.blocks_needed(17) == 2


def test_block_table_example_counts(golden):
    ex = golden["block_tables"]
    for req in ex["requests"].values():
        assert oracle.blocks_needed(req["tokens"], ex["block_size"]) == len(req["table"])


def test_block_table_example_gather(golden):
    """Requests A and B of the diagram: with all keys equal the weights are
    uniform, so the output is the mean of exactly the values the table
    reaches. Each token's V carries its own position, so a wrong block or
    offset changes the mean."""
    ex = golden["block_tables"]
    bs, NB, D = ex["block_size"], ex["pool"], 4
    reqs = [ex["requests"]["A"], ex["requests"]["B"]]
    ks = [torch.zeros(1, r["tokens"], D) for r in reqs]
    vs = []
    for i, r in enumerate(reqs):
        pos = torch.arange(r["tokens"], dtype=torch.float32)
        v = torch.stack([pos, pos * pos, torch.full_like(pos, i + 1.0), pos ** 3], dim=-1)
        vs.append(v[None])
    kc, vc = place(ks, vs, [r["table"] for r in reqs], NB, bs)
    tables = pad_tables([r["table"] for r in reqs], 3, 3)  # B3 is not used by A or B
    lens = torch.tensor([r["tokens"] for r in reqs], dtype=torch.int32)
    q = torch.randn(2, 1, D)
    out, lse = oracle.decode(q, kc, vc, tables, lens, 1.0)
    for i, r in enumerate(reqs):
        n = r["tokens"]
        pos = np.arange(n, dtype=np.float64)
        expect = [pos.mean(), (pos * pos).mean(), i + 1.0, (pos ** 3).mean()]
        np.testing.assert_allclose(out[i, 0].numpy(), expect, rtol=1e-14, atol=1e-12)
        assert lse[i, 0].item() == pytest.approx(math.log(n), abs=1e-14)


def test_block_table_example_one_hot(golden):
    """The diagram's request A: a query aligned with one key under a large
    scale returns that key's value, for every position of the sequence."""
    ex = golden["block_tables"]
    bs, NB, D = ex["block_size"], ex["pool"], 8
    A = ex["requests"]["A"]
    g = torch.Generator().manual_seed(5)
    k = torch.nn.functional.normalize(torch.randn(1, A["tokens"], D, generator=g), dim=-1)
    v = torch.randn(1, A["tokens"], D, generator=g)
    kc, vc = place([k], [v], [A["table"]], NB, bs)
    tables = pad_tables([A["table"]], 3, 0)
    for j in range(A["tokens"]):
        q = k[0, j][None, None] * 1.0
        out, _ = oracle.decode(q, kc, vc, tables, torch.tensor([A["tokens"]], dtype=torch.int32),
                               1e4)
        np.testing.assert_allclose(out[0, 0].numpy(), v[0, j].double().numpy(), atol=1e-9)


def test_reshape_example_slots(golden):
    """The new (last) token of request A lands in B7 at offset 7 (slot 119) and
    of request B in B4 at offset 3 (slot 67); nothing else in the pool moves;
    a negative slot is skipped."""
    ex = golden["block_tables"]
    bs, NB, H, D = ex["block_size"], ex["pool"], 2, 4
    A, Bq = ex["requests"]["A"], ex["requests"]["B"]
    slotA = A["table"][(A["tokens"] - 1) // bs] * bs + (A["tokens"] - 1) % bs
    slotB = Bq["table"][(Bq["tokens"] - 1) // bs] * bs + (Bq["tokens"] - 1) % bs
    assert (slotA, slotB) == (119, 67)
    g = torch.Generator().manual_seed(1)
    kc = torch.randn(NB, H, bs, D, generator=g)
    vc = torch.randn(NB, H, bs, D, generator=g)
    key = torch.randn(3, H, D, generator=g)
    value = torch.randn(3, H, D, generator=g)
    slots = torch.tensor([slotA, -1, slotB], dtype=torch.int64)
    k2, v2 = kc.clone(), vc.clone()
    oracle.reshape_and_cache(key, value, k2, v2, slots)
    ek, ev = kc.clone(), vc.clone()
    ek[7, :, 7], ev[7, :, 7] = key[0], value[0]
    ek[4, :, 3], ev[4, :, 3] = key[2], value[2]
    assert torch.equal(k2, ek) and torch.equal(v2, ev)


def test_reshape_bytes_and_errors():
    """bf16 rows are copied bit for bit; a slot past the pool is an error and
    leaves the pool untouched."""
    g = torch.Generator().manual_seed(2)
    kc = torch.randn(4, 3, 16, 8, generator=g).to(torch.bfloat16)
    vc = kc.clone()
    key = torch.randn(2, 3, 8, generator=g).to(torch.bfloat16)
    oracle.reshape_and_cache(key, key, kc, vc, torch.tensor([63, 0]))
    assert torch.equal(kc[3, :, 15].view(torch.int16), key[0].view(torch.int16))
    assert torch.equal(vc[0, :, 0].view(torch.int16), key[1].view(torch.int16))
    before = kc.clone()
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(key, key, kc, vc, torch.tensor([1, 64]))
    assert torch.equal(before, kc)


# ---------------------------------------------------------------------------
# against a library routine
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("H_q,H_kv", [(4, 4), (4, 2), (8, 1)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_matches_sdpa(H_q, H_kv, dtype):
    """Paged decode at random placements equals torch's attention on the same
    K/V laid out contiguously (GQA by torch's own grouping, MQA with one kv
    head). Ragged lengths span several blocks and partial last blocks."""
    ctxs, D, bs = [1, 7, 16, 17, 40, 65], 8, 4
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, H_q, H_kv, D, bs, seed=H_q * 10 + H_kv,
                                                   dtype=dtype)
    scale = 1 / math.sqrt(D)
    out, lse = oracle.decode(q, kc, vc, tables, lens, scale)
    for b, c in enumerate(ctxs):
        ref = sdpa(q[b][:, None], ks[b], vs[b], scale)[:, 0]
        torch.testing.assert_close(out[b], ref, rtol=1e-12, atol=1e-12)
        # lse against the library's logsumexp of the scores
        kk = ks[b].to(F64).repeat_interleave(H_q // H_kv, 0)
        sc = torch.einsum("hd,hjd->hj", q[b].to(F64), kk) * scale
        torch.testing.assert_close(lse[b], torch.logsumexp(sc, -1), rtol=1e-13, atol=1e-13)


def test_decode_numpy_brute_force():
    """A dense numpy evaluation on tiny inputs (explicit exponentials, no
    max-shift) agrees with the oracle."""
    ctxs, H_q, H_kv, D, bs = [3, 9], 2, 1, 4, 4
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, H_q, H_kv, D, bs, seed=11)
    out, _ = oracle.decode(q, kc, vc, tables, lens, 0.5)
    for b in range(2):
        K, V = ks[b][0].double().numpy(), vs[b][0].double().numpy()
        for h in range(H_q):
            e = np.exp(0.5 * (K @ q[b, h].double().numpy()))
            np.testing.assert_allclose(out[b, h].numpy(), (e[:, None] * V).sum(0) / e.sum(),
                                       rtol=1e-12)


def test_gqa_head_mapping():
    """With 4 q heads over 2 kv heads, heads 2 and 3 read kv head 1: a
    constant V there gives that constant (up to the rounding of weights that
    sum to one), and heads 0 and 1 do not."""
    ctxs, D, bs = [20], 8, 16
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, 4, 2, D, bs, seed=3)
    vs[0][1] = 0.375
    kc, vc = place(ks, vs, [tables[0, :2].tolist()], kc.shape[0], bs)
    out, _ = oracle.decode(q, kc, vc, tables, lens, 0.3)
    torch.testing.assert_close(out[0, 2:], torch.full_like(out[0, 2:], 0.375), rtol=1e-15,
                               atol=0)
    assert torch.all((out[0, :2] - 0.375).abs() > 1e-3)


# ---------------------------------------------------------------------------
# special cases
# ---------------------------------------------------------------------------
def test_single_token_returns_its_value():
    q, ks, vs, kc, vc, tables, lens = random_paged([1, 1], 2, 2, 8, 16, seed=4)
    out, lse = oracle.decode(q, kc, vc, tables, lens, 0.7)
    for b in range(2):
        assert torch.equal(out[b], vs[b][:, 0].double())
        sc = 0.7 * (q[b].double() * ks[b][:, 0].double()).sum(-1)
        torch.testing.assert_close(lse[b], sc, rtol=0, atol=1e-15)


def test_equal_keys_and_zero_scale_give_mean():
    q, ks, vs, kc, vc, tables, lens = random_paged([33], 2, 2, 8, 16, seed=6)
    out0, _ = oracle.decode(q, kc, vc, tables, lens, 0.0)
    mean = vs[0].double().mean(1)
    torch.testing.assert_close(out0[0], mean, rtol=1e-13, atol=1e-14)
    ks[0][:] = ks[0][:, :1]
    kc2, vc2 = place(ks, vs, [tables[0].tolist()], kc.shape[0], 16)
    out1, lse1 = oracle.decode(q, kc2, vc2, tables, lens, 0.9)
    torch.testing.assert_close(out1[0], mean, rtol=1e-13, atol=1e-14)
    sc = 0.9 * (q[0].double() * ks[0][:, 0].double()).sum(-1)
    torch.testing.assert_close(lse1[0], sc + math.log(33), rtol=1e-13, atol=1e-13)


def test_empty_sequence():
    q, ks, vs, kc, vc, tables, lens = random_paged([5], 2, 1, 4, 4, seed=8)
    lens = torch.tensor([0], dtype=torch.int32)
    out, lse = oracle.decode(q, kc, vc, tables, lens, 1.0)
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_bad_inputs_rejected():
    q, ks, vs, kc, vc, tables, lens = random_paged([5], 2, 1, 4, 4, seed=9)
    bad = tables.clone()
    bad[0, 0] = kc.shape[0]
    with pytest.raises(ValueError):
        oracle.decode(q, kc, vc, bad, lens, 1.0)
    with pytest.raises(ValueError):
        oracle.decode(q, kc, vc, tables, torch.tensor([tables.shape[1] * 4 + 1],
                                                      dtype=torch.int32), 1.0)


# ---------------------------------------------------------------------------
# invariants of paging
# ---------------------------------------------------------------------------
def test_block_permutation_invariance():
    """Moving physical blocks (and remapping the tables) leaves the result
    bit-identical: the gather reaches the same tokens in the same order."""
    ctxs, H_q, H_kv, D, bs = [9, 30, 47], 4, 2, 16, 8
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, H_q, H_kv, D, bs, seed=12,
                                                   dtype=torch.bfloat16)
    out, lse = oracle.decode(q, kc, vc, tables, lens, 0.25)
    perm = torch.randperm(kc.shape[0], generator=torch.Generator().manual_seed(13))
    kc2 = torch.empty_like(kc)
    vc2 = torch.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc  # block i moves to perm[i]
    t2 = perm[tables.long()].to(torch.int32)
    out2, lse2 = oracle.decode(q, kc2, vc2, t2, lens, 0.25)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_shared_prefix_equals_private_copies():
    """Beams sharing prefix blocks (and a copied partial block, like B6') give
    bit-identical results to beams with private copies of everything."""
    bs, D, H = 16, 8, 2
    g = torch.Generator().manual_seed(14)
    prefix_k, prefix_v = torch.randn(H, 37, D, generator=g), torch.randn(H, 37, D, generator=g)
    tails = [11, 25]
    ks = [torch.cat([prefix_k, torch.randn(H, t, D, generator=g)], 1) for t in tails]
    vs = [torch.cat([prefix_v, torch.randn(H, t, D, generator=g)], 1) for t in tails]
    # shared: blocks 1 and 3 hold prefix positions 0..31 for both beams;
    # positions 32..36 are in each beam's own block (6 and 8), copied
    shared_rows = [[1, 3, 6, 2], [1, 3, 8, 9, 0]]
    kc, vc = place(ks, vs, shared_rows, 12, bs)
    private_rows = [[0, 2, 4, 5], [6, 7, 8, 9, 10]]
    kp, vp = place(ks, vs, private_rows, 12, bs)
    q = torch.randn(2, 4, D, generator=g)
    lens = torch.tensor([37 + t for t in tails], dtype=torch.int32)
    a = oracle.decode(q, kc, vc, pad_tables(shared_rows, 5, 11), lens, 0.3)
    b = oracle.decode(q, kp, vp, pad_tables(private_rows, 5, 11), lens, 0.3)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ---------------------------------------------------------------------------
# KV split and log-sum-exp merge
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("part", [1, 3, 16, 64, 1000])
def test_split_merge_equals_unsplit(part):
    ctxs, H_q, H_kv, D, bs = [1, 16, 50, 130], 4, 2, 8, 16
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, H_q, H_kv, D, bs, seed=15)
    out, lse = oracle.decode(q, kc, vc, tables, lens, 0.4)
    op, lp = oracle.decode_partials(q, kc, vc, tables, lens, 0.4, part)
    assert op.shape[2] == -(-max(ctxs) // part)
    mo, ml = oracle.lse_merge(op, lp)
    torch.testing.assert_close(mo, out, rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(ml, lse, rtol=1e-12, atol=1e-12)


def test_lse_merge_closed_forms():
    """Two partials: the merged lse is log(e^a + e^b) and the output the
    correspondingly weighted mean; -inf partials carry no weight."""
    o = torch.tensor([[[1.0, 2.0], [3.0, -1.0], [9.0, 9.0]]], dtype=F64)
    lse = torch.tensor([[math.log(1.0), math.log(3.0), float("-inf")]], dtype=F64)
    mo, ml = oracle.lse_merge(o, lse)
    torch.testing.assert_close(ml, torch.tensor([math.log(4.0)], dtype=F64))
    torch.testing.assert_close(mo, torch.tensor([[2.5, -0.25]], dtype=F64))
    mo, ml = oracle.lse_merge(o[:, :1], lse[:, :1])
    assert torch.equal(mo, o[:, 0]) and ml.item() == 0.0
    mo, ml = oracle.lse_merge(o[:, 2:], lse[:, 2:])
    assert torch.all(mo == 0) and torch.isneginf(ml).all()


# ---------------------------------------------------------------------------
# chunked prefill
# ---------------------------------------------------------------------------
def test_prefill_no_cache_is_causal_attention():
    """Chunks with nothing cached and identity tables equal torch's causal
    attention over each chunk."""
    Cs, H_q, H_kv, D, bs = [5, 16, 23], 4, 2, 8, 4
    g = torch.Generator().manual_seed(16)
    ks = [torch.randn(H_kv, c, D, generator=g) for c in Cs]
    vs = [torch.randn(H_kv, c, D, generator=g) for c in Cs]
    rows, at = [], 0
    for c in Cs:
        n = -(-c // bs)
        rows.append(list(range(at, at + n)))
        at += n
    kc, vc = place(ks, vs, rows, at + 1, bs)
    tables = pad_tables(rows, max(len(r) for r in rows), at)
    qsl = torch.tensor([0] + list(np.cumsum(Cs)), dtype=torch.int32)
    q = torch.randn(sum(Cs), H_q, D, generator=g)
    out, _ = oracle.prefill(q, kc, vc, tables, torch.tensor(Cs, dtype=torch.int32), qsl, 0.35)
    for c, C in enumerate(Cs):
        qc = q[qsl[c]:qsl[c + 1]].transpose(0, 1)
        ref = sdpa(qc, ks[c], vs[c], 0.35, causal=True).transpose(0, 1)
        torch.testing.assert_close(out[qsl[c]:qsl[c + 1]], ref, rtol=1e-12, atol=1e-12)


def test_prefill_query_equals_decode_at_its_position():
    """Query i of a chunk after ``cached`` tokens equals a decode over the
    first cached+i+1 tokens (chunk length 1 is exactly decode)."""
    ctxs, H_q, H_kv, D, bs = [37, 70], 4, 1, 8, 16
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, H_q, H_kv, D, bs, seed=17)
    Cs = [9, 1]
    g = torch.Generator().manual_seed(18)
    qp = torch.randn(sum(Cs), H_q, D, generator=g)
    qsl = torch.tensor([0, Cs[0], Cs[0] + Cs[1]], dtype=torch.int32)
    out, lse = oracle.prefill(qp, kc, vc, tables, lens, qsl, 0.3)
    for c, C in enumerate(Cs):
        for i in range(C):
            row = int(qsl[c]) + i
            pos = ctxs[c] - C + i
            d, dl = oracle.decode(qp[row][None], kc, vc, tables[c:c + 1],
                                  torch.tensor([pos + 1], dtype=torch.int32), 0.3)
            assert torch.equal(out[row], d[0]) and torch.equal(lse[row], dl[0])


def test_prefill_ignores_future_keys():
    """Changing keys/values at positions after a query's own leaves that
    query's output bit-identical (causality)."""
    ctxs, H_q, H_kv, D, bs = [40], 2, 1, 8, 8
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, H_q, H_kv, D, bs, seed=19)
    qp = torch.randn(12, H_q, D, generator=torch.Generator().manual_seed(20))
    qsl = torch.tensor([0, 12], dtype=torch.int32)
    out, _ = oracle.prefill(qp, kc, vc, tables, lens, qsl, 0.3)
    ks[0][:, 35:] += 3.0
    vs[0][:, 35:] -= 2.0
    kc2, vc2 = place(ks, vs, [tables[0].tolist()], kc.shape[0], bs)
    out2, _ = oracle.prefill(qp, kc2, vc2, tables, lens, qsl, 0.3)
    # query i sits at position 28 + i: rows 0..6 (positions 28..34) unchanged
    assert torch.equal(out[:7], out2[:7])
    assert not torch.equal(out[7:], out2[7:])


def test_select_computes_only_selected():
    q, ks, vs, kc, vc, tables, lens = random_paged([9, 30], 4, 2, 8, 8, seed=21)
    full, _ = oracle.decode(q, kc, vc, tables, lens, 0.5)
    sel = torch.zeros(2, 4, dtype=torch.bool)
    sel[1, 3] = sel[0, 0] = True
    part, _ = oracle.decode(q, kc, vc, tables, lens, 0.5, select=sel)
    assert torch.equal(part[sel], full[sel]) and torch.all(part[~sel] == 0)


# ---------------------------------------------------------------------------
# whole-block copies (copy-on-write, swap)
# ---------------------------------------------------------------------------
def test_cow_copy_then_diverge(golden):
    """The beam example: beams share B1, B3 and B6; before beam 2 appends,
    B6 is copied to B6'. Afterwards beam 1 and beam 2 read the same prefix
    and differ only in what each appended; the copy is bit-exact and nothing
    else in the pool moves."""
    ex = golden["block_tables"]
    bs, H, D = ex["block_size"], 2, 8
    g = torch.Generator().manual_seed(30)
    NB = 9  # B0..B7 plus B6' at id 8
    kc = torch.randn(NB, H, bs, D, generator=g)
    vc = torch.randn(NB, H, bs, D, generator=g)
    before_k, before_v = kc.clone(), vc.clone()
    oracle.copy_blocks(kc, vc, kc, vc, torch.tensor([[6, 8]]))
    assert torch.equal(kc[8], before_k[6]) and torch.equal(vc[8], before_v[6])
    assert torch.equal(kc[:8], before_k[:8]) and torch.equal(vc[:8], before_v[:8])
    # beam 2 appends at offset 5 of its copy; beam 1 at offset 5 of B6
    shared = ex["beams"]["shared"]
    b1 = shared + [6]
    b2 = shared + [8]
    key = torch.randn(2, H, D, generator=g)
    oracle.reshape_and_cache(key, key, kc, vc, torch.tensor([6 * bs + 5, 8 * bs + 5]))
    ctx = 2 * bs + 6
    q = torch.randn(2, 2, D, generator=g)
    tables = torch.tensor([b1, b2], dtype=torch.int32)
    lens = torch.tensor([ctx, ctx], dtype=torch.int32)
    out, _ = oracle.decode(q, kc, vc, tables, lens, 0.3)
    # same query against beam 1's table with beam 2's appended row gives beam 2's answer
    kc2, vc2 = kc.clone(), vc.clone()
    kc2[6, :, 5], vc2[6, :, 5] = key[1], key[1]
    out_b2_via_b1, _ = oracle.decode(q[1:], kc2, vc2, tables[:1], lens[:1], 0.3)
    assert torch.equal(out[1], out_b2_via_b1[0])
    assert not torch.equal(out[0], out[1])


def test_swap_round_trip_and_errors():
    g = torch.Generator().manual_seed(31)
    dev_k = torch.randn(6, 2, 16, 8, generator=g).to(torch.bfloat16)
    dev_v = torch.randn(6, 2, 16, 8, generator=g).to(torch.bfloat16)
    host_k = torch.zeros(4, 2, 16, 8, dtype=torch.bfloat16)
    host_v = torch.zeros_like(host_k)
    out_map = torch.tensor([[5, 0], [1, 3]])
    oracle.copy_blocks(dev_k, dev_v, host_k, host_v, out_map)
    assert torch.equal(host_k[0], dev_k[5]) and torch.equal(host_v[3], dev_v[1])
    assert torch.all(host_k[1] == 0) and torch.all(host_k[2] == 0)
    back_k, back_v = torch.zeros_like(dev_k), torch.zeros_like(dev_v)
    oracle.copy_blocks(host_k, host_v, back_k, back_v, out_map.flip(1))
    assert torch.equal(back_k[5], dev_k[5]) and torch.equal(back_v[1], dev_v[1])
    with pytest.raises(ValueError):
        oracle.copy_blocks(dev_k, dev_v, host_k, host_v, torch.tensor([[6, 0]]))
    with pytest.raises(ValueError):
        oracle.copy_blocks(dev_k, dev_v, host_k, host_v, torch.tensor([[0, 4]]))


# ---------------------------------------------------------------------------
# FP8 (E4M3) KV cache
# ---------------------------------------------------------------------------
def test_e4m3_decode_matches_library_for_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ours = oracle.e4m3_decode(codes)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64)
    nan = torch.isnan(lib)
    assert torch.equal(torch.isnan(ours), nan) and int(nan.sum()) == 2  # 0x7F, 0xFF
    assert torch.equal(ours[~nan], lib[~nan])
    assert ours.abs()[~nan].max() == 448.0


def test_e4m3_encode_matches_library_in_range():
    """Every bf16 bit pattern whose magnitude is below 448 (exhaustive)
    encodes to the same code as torch's float8_e4m3fn conversion (nearest,
    ties to even); outside that range the oracle saturates instead."""
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    x = bits.view(torch.bfloat16).to(torch.float32)
    keep = torch.isfinite(x) & (x.abs() < 448)
    x = x[keep]
    ours = oracle.e4m3_encode(x)
    lib = x.to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(ours, lib)


def test_e4m3_saturation_and_ties():
    x = torch.tensor([448.0, 460.0, 1e6, float("inf"), -1e30, float("-inf"), float("nan"),
                      1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, -0.0])
    c = oracle.e4m3_encode(x).tolist()
    assert c[:6] == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert c[6] == 0x7F
    # halfway cases go to the even code
    assert c[7:11] == [0x38, 0x3A, 0x00, 0x02]
    assert c[11] == 0x80


def test_e4m3_reshape_is_divide_then_encode():
    g = torch.Generator().manual_seed(50)
    key = (torch.randn(3, 2, 8, generator=g) * 3).to(torch.bfloat16)
    value = (torch.randn(3, 2, 8, generator=g) * 3).to(torch.bfloat16)
    ks, vs = torch.tensor([0.05, 0.3]), torch.tensor([0.02, 7.0])
    kc = torch.zeros(4, 2, 16, 8, dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    slots = torch.tensor([5, -1, 63])
    oracle.reshape_and_cache_e4m3(key, value, kc, vc, slots, ks, vs)
    for t, s in ((0, 5), (2, 63)):
        for h in range(2):
            want_k = oracle.e4m3_encode(key[t, h].float() / ks[h])
            want_v = oracle.e4m3_encode(value[t, h].float() / vs[h])
            assert torch.equal(kc[s // 16, h, s % 16], want_k)
            assert torch.equal(vc[s // 16, h, s % 16], want_v)
    untouched = torch.ones(4, 16, dtype=torch.bool)
    untouched[0, 5] = untouched[3, 15] = False
    assert torch.all(kc.permute(0, 2, 1, 3)[untouched] == 0)


def test_e4m3_decode_equals_decode_of_dequantized_cache():
    """With power-of-two scales code*scale is exact in fp32, so decode over
    the E4M3 cache equals decode over the dequantized fp32 cache bit for bit
    (and it is close to torch's attention on the same values)."""
    ctxs, H_q, H_kv, D, bs = [7, 33, 50], 8, 2, 16, 16
    g = torch.Generator().manual_seed(51)
    NB = 12
    kc = torch.randint(0, 256, (NB, H_kv, bs, D), generator=g, dtype=torch.int32).to(torch.uint8)
    vc = torch.randint(0, 256, (NB, H_kv, bs, D), generator=g, dtype=torch.int32).to(torch.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x38  # no NaN codes
    vc[(vc & 0x7F) == 0x7F] = 0x30
    ks, vs = torch.tensor([0.0625, 0.5]), torch.tensor([0.25, 2.0 ** -6])
    tables = torch.tensor([[3, 0, 0, 0], [1, 7, 2, 0], [4, 5, 6, 11]], dtype=torch.int32)
    lens = torch.tensor(ctxs, dtype=torch.int32)
    q = torch.randn(3, H_q, D, generator=g).to(torch.bfloat16)
    out, lse = oracle.decode_e4m3(q, kc, vc, ks, vs, tables, lens, 0.2)
    kd = (oracle.e4m3_decode(kc) * ks.double()[None, :, None, None]).float()
    vd = (oracle.e4m3_decode(vc) * vs.double()[None, :, None, None]).float()
    ref, ref_lse = oracle.decode(q.float(), kd, vd, tables, lens, 0.2)
    assert torch.equal(out, ref) and torch.equal(lse, ref_lse)


# ---------------------------------------------------------------------------
# INT8 KV cache
# ---------------------------------------------------------------------------
def test_int8_encode_special_values():
    """Halfway cases go to the even integer; integers stay; the range is the
    symmetric [-127, 127]; NaN encodes as 0."""
    q = torch.tensor([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -126.5, 3.0, -7.0, 0.49999997,
                      127.0, 127.49, 128.0, 1e30, float("inf"), -127.6, -1e30, float("-inf"),
                      float("nan"), -0.0])
    want = [0, 2, 2, 0, -2, -2, 126, -126, 3, -7, 0, 127, 127, 127, 127, 127, -127, -127, -127,
            0, 0]
    assert oracle.int8_encode(q).tolist() == want


def test_int8_encode_is_nearest_integer():
    """Over a dense grid of fp32 quotients every code is an integer within
    1/2 of the quotient, and the encoding never decreases."""
    q = torch.arange(-130 * 256, 130 * 256 + 1, dtype=torch.float32) / 256
    c = oracle.int8_encode(q).double()
    inside = q.abs() <= 127
    assert torch.all((c[inside] - q[inside].double()).abs() <= 0.5)
    assert torch.all(c[~inside].abs() == 127)
    assert torch.all(c[1:] >= c[:-1])


def test_int8_reshape_is_divide_then_encode():
    g = torch.Generator().manual_seed(52)
    key = (torch.randn(3, 2, 8, generator=g) * 3).to(torch.bfloat16)
    value = (torch.randn(3, 2, 8, generator=g) * 3).to(torch.bfloat16)
    ks, vs = torch.tensor([0.05, 0.3]), torch.tensor([0.01, 7.0])  # some values saturate
    kc = torch.zeros(4, 2, 16, 8, dtype=torch.int8)
    vc = torch.zeros_like(kc)
    slots = torch.tensor([5, -1, 63])
    oracle.reshape_and_cache_int8(key, value, kc, vc, slots, ks, vs)
    for t, s in ((0, 5), (2, 63)):
        for h in range(2):
            want_k = oracle.int8_encode(key[t, h].float() / ks[h])
            want_v = oracle.int8_encode(value[t, h].float() / vs[h])
            assert torch.equal(kc[s // 16, h, s % 16], want_k)
            assert torch.equal(vc[s // 16, h, s % 16], want_v)
    assert vc.abs().max() == 127  # value / 0.01 saturates
    untouched = torch.ones(4, 16, dtype=torch.bool)
    untouched[0, 5] = untouched[3, 15] = False
    assert torch.all(kc.permute(0, 2, 1, 3)[untouched] == 0)


def test_int8_decode_equals_decode_of_dequantized_cache():
    """code*scale is exact in fp32 for power-of-two scales, so decode over the
    INT8 cache equals decode over the dequantized fp32 cache bit for bit."""
    ctxs, H_q, H_kv, D, bs = [7, 33, 50], 8, 2, 16, 16
    g = torch.Generator().manual_seed(53)
    NB = 12
    kc = torch.randint(-127, 128, (NB, H_kv, bs, D), generator=g, dtype=torch.int32).to(torch.int8)
    vc = torch.randint(-127, 128, (NB, H_kv, bs, D), generator=g, dtype=torch.int32).to(torch.int8)
    ks, vs = torch.tensor([0.0625, 2.0 ** -7]), torch.tensor([0.25, 2.0 ** -6])
    tables = torch.tensor([[3, 0, 0, 0], [1, 7, 2, 0], [4, 5, 6, 11]], dtype=torch.int32)
    lens = torch.tensor(ctxs, dtype=torch.int32)
    q = torch.randn(3, H_q, D, generator=g).to(torch.bfloat16)
    out, lse = oracle.decode_int8(q, kc, vc, ks, vs, tables, lens, 0.2)
    kd = (kc.double() * ks.double()[None, :, None, None]).float()
    vd = (vc.double() * vs.double()[None, :, None, None]).float()
    ref, ref_lse = oracle.decode(q.float(), kd, vd, tables, lens, 0.2)
    assert torch.equal(out, ref) and torch.equal(lse, ref_lse)


# ---------------------------------------------------------------------------
# sliding window
# ---------------------------------------------------------------------------
def test_window_covering_everything_is_plain_decode():
    q, ks, vs, kc, vc, tables, lens = random_paged([9, 30, 47], 4, 2, 8, 8, seed=70)
    a = oracle.decode(q, kc, vc, tables, lens, 0.3)
    b = oracle.decode_window(q, kc, vc, tables, lens, 0.3, 47)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_window_of_one_is_the_last_value():
    q, ks, vs, kc, vc, tables, lens = random_paged([9, 30], 2, 2, 8, 8, seed=71)
    out, _ = oracle.decode_window(q, kc, vc, tables, lens, 0.3, 1)
    for b, c in enumerate([9, 30]):
        assert torch.equal(out[b], vs[b][:, c - 1].double())


def test_window_equals_decode_of_the_dropped_prefix():
    """A window of W over ctx tokens equals plain decode of the sequence with
    its first ctx - W tokens removed (here a whole number of blocks, so the
    shortened table is the original minus its leading entries)."""
    bs = 8
    ctxs = [48, 37]
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, 4, 1, 8, bs, seed=72)
    W = 24
    out, lse = oracle.decode_window(q, kc, vc, tables, lens, 0.4, W)
    for b, c in enumerate(ctxs):
        drop = (c - W) // bs * bs
        rest = c - drop
        t = tables[b:b + 1, drop // bs:].contiguous()
        ref, ref_lse = oracle.decode_window(q[b:b + 1], kc, vc, t,
                                            torch.tensor([rest], dtype=torch.int32), 0.4, W)
        plain, plain_lse = oracle.decode(q[b:b + 1], kc, vc, t,
                                         torch.tensor([rest], dtype=torch.int32), 0.4)
        if rest == W:
            assert torch.equal(out[b], plain[0]) and torch.equal(lse[b], plain_lse[0])
        assert torch.equal(out[b], ref[0])


def test_prefill_window_no_cache_is_banded_attention():
    """Chunks with nothing cached and identity tables equal torch's attention
    under an explicit band mask: query i sees keys j with i - W < j <= i."""
    Cs, H_q, H_kv, D, bs, W = [5, 16, 23], 4, 2, 8, 4, 6
    g = torch.Generator().manual_seed(73)
    ks = [torch.randn(H_kv, c, D, generator=g) for c in Cs]
    vs = [torch.randn(H_kv, c, D, generator=g) for c in Cs]
    rows, at = [], 0
    for c in Cs:
        n = -(-c // bs)
        rows.append(list(range(at, at + n)))
        at += n
    kc, vc = place(ks, vs, rows, at + 1, bs)
    tables = pad_tables(rows, max(len(r) for r in rows), at)
    qsl = torch.tensor([0] + list(np.cumsum(Cs)), dtype=torch.int32)
    q = torch.randn(sum(Cs), H_q, D, generator=g)
    out, _ = oracle.prefill_window(q, kc, vc, tables, torch.tensor(Cs, dtype=torch.int32), qsl,
                                   0.35, W)
    for c, C in enumerate(Cs):
        i = torch.arange(C)[:, None]
        j = torch.arange(C)[None, :]
        band = (j <= i) & (j > i - W)
        qc = q[qsl[c]:qsl[c + 1]].transpose(0, 1).to(F64)
        ref = F.scaled_dot_product_attention(qc[None], ks[c][None].to(F64), vs[c][None].to(F64),
                                             attn_mask=band, scale=0.35,
                                             enable_gqa=True)[0].transpose(0, 1)
        torch.testing.assert_close(out[qsl[c]:qsl[c + 1]], ref, rtol=1e-12, atol=1e-12)


def test_prefill_window_covering_everything_is_plain_prefill():
    ctxs, H_q, H_kv, D, bs = [37, 70], 4, 2, 8, 16
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, H_q, H_kv, D, bs, seed=74)
    qp = torch.randn(21, H_q, D, generator=torch.Generator().manual_seed(75))
    qsl = torch.tensor([0, 9, 21], dtype=torch.int32)
    a = oracle.prefill(qp, kc, vc, tables, lens, qsl, 0.3)
    b = oracle.prefill_window(qp, kc, vc, tables, lens, qsl, 0.3, 70)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_prefill_window_query_equals_windowed_decode_at_its_position():
    """Query i of a windowed chunk equals a windowed decode over the first
    pos + 1 tokens (the decode query sits at position pos)."""
    ctxs, H_q, H_kv, D, bs, W = [37, 70], 4, 1, 8, 16, 13
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, H_q, H_kv, D, bs, seed=76)
    Cs = [9, 20]
    qp = torch.randn(sum(Cs), H_q, D, generator=torch.Generator().manual_seed(77))
    qsl = torch.tensor([0, Cs[0], Cs[0] + Cs[1]], dtype=torch.int32)
    out, lse = oracle.prefill_window(qp, kc, vc, tables, lens, qsl, 0.3, W)
    for c, C in enumerate(Cs):
        for i in range(C):
            row = int(qsl[c]) + i
            pos = ctxs[c] - C + i
            d, dl = oracle.decode_window(qp[row][None], kc, vc, tables[c:c + 1],
                                         torch.tensor([pos + 1], dtype=torch.int32), 0.3, W)
            assert torch.equal(out[row], d[0]) and torch.equal(lse[row], dl[0])


def test_prefill_window_ignores_keys_outside_the_band():
    """Changing keys/values more than W - 1 positions before a query, or
    after it, leaves that query's output bit-identical; changing one inside
    its band does not."""
    ctxs, H_q, H_kv, D, bs, W = [40], 2, 1, 8, 8, 10
    q, ks, vs, kc, vc, tables, lens = random_paged(ctxs, H_q, H_kv, D, bs, seed=78)
    qp = torch.randn(12, H_q, D, generator=torch.Generator().manual_seed(79))
    qsl = torch.tensor([0, 12], dtype=torch.int32)
    out, _ = oracle.prefill_window(qp, kc, vc, tables, lens, qsl, 0.3, W)
    # query i sits at position 28 + i and sees [19 + i, 28 + i]
    ks2 = [ks[0].clone()]
    vs2 = [vs[0].clone()]
    ks2[0][:, :19] += 3.0
    vs2[0][:, :19] -= 2.0
    ks2[0][:, 39:] += 3.0
    kc2, vc2 = place(ks2, vs2, [tables[0].tolist()], kc.shape[0], bs)
    out2, _ = oracle.prefill_window(qp, kc2, vc2, tables, lens, qsl, 0.3, W)
    assert torch.equal(out[:11], out2[:11])  # rows 0..10 see [19, 38]
    assert not torch.equal(out[11], out2[11])  # row 11 sees position 39
    vs3 = [vs[0].clone()]
    vs3[0][:, 25] += 1.0  # inside the band of rows 0..6
    kc3, vc3 = place(ks, vs3, [tables[0].tolist()], kc.shape[0], bs)
    out3, _ = oracle.prefill_window(qp, kc3, vc3, tables, lens, qsl, 0.3, W)
    assert not torch.equal(out[:7], out3[:7]) and torch.equal(out[7:], out3[7:])
