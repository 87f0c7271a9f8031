"""Host-side arithmetic of bench.py: algorithmic bytes and FLOPs with and
without a sliding window, and the reference arm (the oracle) with a window."""
import json

import bench
from pagedattention_paged_kv_02_b200 import workloads as W


def test_window_covering_every_context_changes_nothing():
    b = W.llama7b_decode()
    full = bench.decode_bytes(b)
    b.sliding_window = 4096
    assert bench.decode_bytes(b) == full
    m = W.mixed_prefill_decode()
    f = bench.prefill_flops(m)
    m.sliding_window = 1 << 20
    assert bench.prefill_flops(m) == f


def test_window_bytes_and_flops_closed_forms():
    b = W.tiny_fp32()
    b.sliding_window = 8
    ctx = b.context_lens.tolist()  # 5, 17, 33, 40
    H_kv, D, bs, e = b.num_kv_heads, b.head_dim, b.block_size, 4
    kv = sum(2 * min(c, 8) * H_kv * D * e for c in ctx)
    blocks = sum((c - 1) // bs - max(0, c - 8) // bs + 1 for c in ctx)
    qo = 2 * b.num_seqs * b.num_q_heads * D * e
    assert bench.decode_bytes(b) == kv + qo + 4 * blocks * H_kv + 4 * b.num_seqs
    m = W.mixed_prefill_decode()
    m.sliding_window = 1  # every query sees one key
    assert bench.prefill_flops(m) == 4 * m.head_dim * m.num_q_heads * m.prefill_q.shape[0]


def test_reference_arm_with_window(capsys, monkeypatch):
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    bench.main(["--impl", "reference", "--workload", "tiny_fp32", "--window", "8",
                "--steps", "2", "--warmup", "3", "--reference-seconds", "1"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"]["sliding_window"] == 8
    assert line["value"] > 0
