"""Host-side arithmetic of bench.py: algorithmic bytes and FLOPs with and
without a sliding window, and the reference arm (the oracle) with a window."""
import json

import torch

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


def test_profiled_traffic_follows_the_source_digest_and_workload(tmp_path, monkeypatch):
    """The DRAM bytes of a committed ncu summary are reported only while the
    kernel source still hashes to the digest recorded beside them and the run
    is on the workload the summary was taken on (the same batch name: head
    dim, block size and cache type are part of it)."""
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cuh"
    src.write_text("kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.source_digest(["k.cuh"])
    (tmp_path / "profiles" / "p.md").write_text(
        f"# summary\n\n- workload: `wl_d128_bs16`\n- source-sha256: `{digest}`\n"
        "- dram-bytes-per-launch: `123456`\n")
    assert bench.profiled_traffic("p.md", ["k.cuh"], "wl_d128_bs16") == 123456.0
    assert bench.profiled_traffic("p.md", ["k.cuh"], "wl_d64_bs16") is None
    assert bench.profiled_traffic("p.md", ["k.cuh"], None) is None
    assert bench.profiled_traffic("missing.md", ["k.cuh"], "wl_d128_bs16") is None
    src.write_text("kernel v2\n")
    assert bench.profiled_traffic("p.md", ["k.cuh"], "wl_d128_bs16") is None
    # a summary without a workload field is never used
    (tmp_path / "profiles" / "q.md").write_text(
        f"- source-sha256: `{bench.source_digest(['k.cuh'])}`\n- dram-bytes-per-launch: `7`\n")
    assert bench.profiled_traffic("q.md", ["k.cuh"], "wl_d128_bs16") is None


def test_committed_profiles_carry_a_source_digest():
    """Every committed kernel summary names the workload and the digest of the
    kernel sources it was taken on and its DRAM bytes per launch; bench
    reports that traffic only while both match (a summary taken before a
    kernel change, or on another workload, yields traffic = null, never a
    stale number)."""
    import glob
    import os
    import re
    for path in glob.glob(os.path.join(bench.ROOT, "profiles", "*.md")):
        text = open(path).read()
        name = os.path.basename(path)
        assert re.search(r"source-sha256: `[0-9a-f]{16}`", text), f"{name}: no digest"
        assert re.search(r"dram-bytes-per-launch: `[0-9]+`", text), f"{name}: no DRAM bytes"
        # a batch name: the workload with its heads, head dim and block size
        assert re.search(r"workload: `\w+_d(64|128)_bs(16|32|64)\w*`", text), \
            f"{name}: no workload"


def test_unique_bytes_count_shared_prefix_blocks_once():
    """Without sharing, the distinct K/V bytes are the logical K/V bytes; the
    mixed batch's 24 beam groups share a 64-block prefix, read 8 times each."""
    b = W.llama7b_decode()
    ctx = b.context_lens.to(torch.int64)
    kv = int((2 * ctx * b.num_kv_heads * b.head_dim * b.k_cache.element_size()).sum())
    assert bench.decode_unique_bytes(b) == kv
    m = W.mixed_prefill_decode()
    per_token = 2 * m.num_kv_heads * m.head_dim * m.k_cache.element_size()
    logical = int(m.context_lens.to(torch.int64).sum()) * per_token
    shared = 24 * 7 * 1024 * per_token  # 7 of each group's 8 readers of its prefix
    assert bench.decode_unique_bytes(m) == logical - shared
