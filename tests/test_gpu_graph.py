"""The hot path captured in a CUDA graph: a decode step (scatter, split
kernel, and the log-sum-exp merge launched as a programmatic dependent) and a
prefill step, captured once through the C ABI and replayed, give the same
bits as the eager calls; replays after changing the inputs in place follow
the new inputs."""
import pytest
import torch

from helpers import bits
from pagedattention_paged_kv_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def pa():
    from pagedattention_paged_kv_02_b200 import build, pa as _pa
    build.build()
    torch.cuda.init()
    return _pa


def test_decode_step_in_a_graph(pa):
    batch = W.decode_batch([1500, 40, 700, 2047], 16, 2, 128, 16, 400, torch.bfloat16, seed=111)
    d = batch.to(DEV)
    B, H_q, D = d.q.shape
    n = pa.pa_decode_workspace_size(B, H_q, D, batch.max_context_len, 512)
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    out = torch.empty_like(d.q)
    scatter = pa.prepare_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    decode = pa.prepare_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                               batch.max_context_len, batch.scale, 512, ws)
    scatter()
    decode()
    torch.cuda.synchronize()
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            scatter(stream=s)
            decode(stream=s)
    torch.cuda.current_stream().wait_stream(s)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(bits(out), bits(eager))
    # new queries, same graph
    d.q.mul_(-1.0)
    g.replay()
    torch.cuda.synchronize()
    decode()
    torch.cuda.synchronize()
    again = out.clone()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(bits(out), bits(again)) and not torch.equal(bits(out), bits(eager))
    assert pa.pa_device_error() == 0


def test_prefill_step_in_a_graph(pa):
    batch = W.mixed_prefill_decode()
    d = batch.to(DEV)
    pa.pa_reshape_and_cache(d.key, d.value, d.k_cache, d.v_cache, d.slot_mapping)
    out = torch.empty_like(d.prefill_q)
    qsl = batch.query_start_loc
    prefill = pa.prepare_prefill_chunk(out, d.prefill_q, d.k_cache, d.v_cache,
                                       d.prefill_block_tables, d.prefill_context_lens,
                                       d.query_start_loc, int((qsl[1:] - qsl[:-1]).max()),
                                       batch.scale)
    prefill()
    torch.cuda.synchronize()
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            prefill(stream=s)
    torch.cuda.current_stream().wait_stream(s)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(bits(out), bits(eager))
    assert pa.pa_device_error() == 0
