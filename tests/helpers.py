"""Shared pieces of the GPU parity tests: run a step through the CUDA library,
run the same step through the fp64 oracle, and compare with the tolerances
the method states (fp32: max-abs 1e-5; bf16 with fp32 accumulation: max-abs
2e-2 and relative L2 3e-3; the cache scatter: bit-exact)."""
import torch

import oracle

FP32_MAX_ABS = 1e-5
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 3e-3


def bits(t: torch.Tensor) -> torch.Tensor:
    """Bit patterns, so NaN payloads compare exactly."""
    return t.contiguous().view(torch.int16 if t.element_size() == 2 else torch.int32)


def assert_close(gpu: torch.Tensor, ref64: torch.Tensor, what: str = ""):
    got = gpu.detach().cpu().double()
    ref = ref64.double()
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    err = (got - ref).abs()
    max_abs = err.max().item() if err.numel() else 0.0
    if gpu.dtype == torch.float32:
        assert max_abs <= FP32_MAX_ABS, f"{what}: max-abs {max_abs:.3e}"
    else:
        rel = ((got - ref).norm() / ref.norm().clamp_min(1e-30)).item()
        assert max_abs <= BF16_MAX_ABS, f"{what}: max-abs {max_abs:.3e}"
        assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel:.3e}"
    return max_abs


def oracle_after_append(batch):
    """Host copies of the caches with the step's tokens appended by the oracle."""
    k, v = batch.k_cache.clone(), batch.v_cache.clone()
    oracle.reshape_and_cache(batch.key, batch.value, k, v, batch.slot_mapping)
    return k, v


def oracle_decode(batch, k, v, select=None):
    return oracle.decode(batch.q, k, v, batch.block_tables, batch.context_lens, batch.scale,
                         select=select)


def gpu_decode(pa, dev, partition_size=None, out=None):
    """Run pa_decode on a device batch (caches already appended)."""
    part = dev.partition_size if partition_size is None else partition_size
    B, H_q, D = dev.q.shape
    ws_bytes = pa.pa_decode_workspace_size(B, H_q, D, dev.max_context_len, part)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev.q.device)
    if out is None:
        out = torch.empty_like(dev.q)
    pa.pa_decode(out, dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens,
                 dev.max_context_len, dev.scale, part, ws if ws_bytes else None)
    return out
