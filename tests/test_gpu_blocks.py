"""GPU parity of the whole-block copies against the oracle, bit for bit:
copy-on-write inside one pool, swap out to a pinned host pool and back in,
out-of-pool ids recorded and skipped, and the beam example end to end (share,
copy the partial block, append divergent tokens, decode)."""
import pytest
import torch

import oracle
from helpers import assert_close, bits, gpu_decode
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


def pool(nb, h, bs, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(nb, h, bs, d, generator=g).to(dtype),
            torch.randn(nb, h, bs, d, generator=g).to(dtype))


@pytest.mark.parametrize("dtype,h,bs,d", [(torch.bfloat16, 8, 16, 128), (torch.float32, 4, 64, 64),
                                          (torch.bfloat16, 32, 32, 128)])
def test_copy_blocks_bit_exact(pa, dtype, h, bs, d):
    k, v = pool(200, h, bs, d, dtype, seed=h + bs)
    perm = torch.randperm(200, generator=torch.Generator().manual_seed(1))
    mapping = torch.stack([perm[:60], perm[60:120]], 1).contiguous()  # dsts disjoint from srcs
    dk, dv = k.to(DEV), v.to(DEV)
    pa.pa_copy_blocks(dk, dv, mapping.to(DEV))
    torch.cuda.synchronize()
    oracle.copy_blocks(k, v, k, v, mapping)
    assert torch.equal(bits(dk.cpu()), bits(k)) and torch.equal(bits(dv.cpu()), bits(v))
    assert pa.pa_device_error() == 0


def test_swap_out_and_in_through_pinned_host(pa):
    k, v = pool(64, 8, 16, 128, torch.bfloat16, seed=5)
    dk, dv = k.to(DEV), v.to(DEV)
    hk = torch.zeros(32, 8, 16, 128, dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    out_map = torch.tensor([[3, 0], [40, 7], [63, 31], [0, 12]], dtype=torch.int64)
    pa.pa_swap_blocks(dk, dv, hk, hv, out_map.to(DEV))
    torch.cuda.synchronize()
    ek, ev = torch.zeros_like(hk), torch.zeros_like(hv)
    oracle.copy_blocks(k, v, ek, ev, out_map)
    assert torch.equal(bits(hk), bits(ek)) and torch.equal(bits(hv), bits(ev))
    # back in, to different device blocks, with the mapping itself in pinned memory
    in_map = torch.tensor([[0, 10], [7, 11], [31, 12], [12, 13]], dtype=torch.int64).pin_memory()
    dk2, dv2 = torch.zeros_like(dk), torch.zeros_like(dv)
    pa.pa_swap_blocks(hk, hv, dk2, dv2, in_map)
    torch.cuda.synchronize()
    assert torch.equal(bits(dk2[10].cpu()), bits(k[3])) and torch.equal(bits(dv2[13].cpu()), bits(v[0]))
    assert torch.all(dk2[:10] == 0) and torch.all(dk2[14:] == 0)


def test_bad_ids_skipped_and_recorded(pa):
    k, v = pool(16, 2, 16, 64, torch.float32, seed=6)
    dk, dv = k.to(DEV), v.to(DEV)
    mapping = torch.tensor([[1, 2], [3, 16], [-1, 4]], dtype=torch.int64)
    pa.pa_copy_blocks(dk, dv, mapping.to(DEV))
    torch.cuda.synchronize()
    assert pa.pa_device_error() == pa.PA_ERR_BAD_TABLE
    ek, ev = k.clone(), v.clone()
    oracle.copy_blocks(k, v, ek, ev, mapping[:1])
    assert torch.equal(bits(dk.cpu()), bits(ek)) and torch.equal(bits(dv.cpu()), bits(ev))


def test_beam_fork_copy_on_write_then_decode(pa):
    """Two beams share a 37-token prefix (two full blocks shared, the partial
    third block shared until the fork). At the fork beam 2's partial block is
    copied on write, then each beam appends its own tokens; decode of both
    matches the oracle on the same operations."""
    bs, H, D = 16, 4, 128
    nb = 16
    g = torch.Generator().manual_seed(40)
    k = torch.full((nb, H, bs, D), float("nan"), dtype=torch.bfloat16)
    v = torch.full_like(k, float("nan"))
    shared = [3, 9, 5]  # tokens 0..36: blocks 3 and 9 full, block 5 holds 5 tokens
    for blk, n in zip(shared, [16, 16, 5]):
        k[blk, :, :n] = torch.randn(H, n, D, generator=g).to(torch.bfloat16)
        v[blk, :, :n] = torch.randn(H, n, D, generator=g).to(torch.bfloat16)
    fork = torch.tensor([[5, 11]], dtype=torch.int64)  # beam 2's copy of the partial block
    tables = torch.tensor([[3, 9, 5, 0], [3, 9, 11, 0]], dtype=torch.int32)
    # each beam appends 4 tokens at positions 37..40
    key = torch.randn(8, H, D, generator=g).to(torch.bfloat16)
    val = torch.randn(8, H, D, generator=g).to(torch.bfloat16)
    slots = torch.tensor([5 * bs + 5 + i for i in range(4)] + [11 * bs + 5 + i for i in range(4)])
    q = torch.randn(2, 8, D, generator=g).to(torch.bfloat16)
    lens = torch.tensor([41, 41], dtype=torch.int32)
    # GPU
    dk, dv = k.to(DEV), v.to(DEV)
    pa.pa_copy_blocks(dk, dv, fork.to(DEV))
    pa.pa_reshape_and_cache(key.to(DEV), val.to(DEV), dk, dv, slots.to(DEV))
    out = torch.empty(2, 8, D, dtype=torch.bfloat16, device=DEV)
    pa.pa_decode(out, q.to(DEV), dk, dv, tables.to(DEV), lens.to(DEV), 41, D ** -0.5)
    torch.cuda.synchronize()
    # oracle
    oracle.copy_blocks(k, v, k, v, fork)
    oracle.reshape_and_cache(key, val, k, v, slots)
    ref, _ = oracle.decode(q, k, v, tables, lens, D ** -0.5)
    assert_close(out, ref, "beam fork")
    assert torch.equal(bits(dk.cpu()), bits(k))
