"""The C-ABI library loads on a host without a GPU, exports every entry point
include/pa.h declares, and rejects bad arguments on the host before any
launch. Nothing here touches a device: every call below fails its host-side
checks (or is pure host arithmetic) before the library would reach CUDA."""
import ctypes
import os
import re

import pytest

from pagedattention_paged_kv_02_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")

# addresses that are aligned but never dereferenced: each call using them
# must fail a host check first
FAKE = ctypes.c_void_p(0x10000)


@pytest.fixture(scope="module")
def L():
    pa_build.build()
    from pagedattention_paged_kv_02_b200 import pa
    return pa.lib()


def declared():
    text = open(HEADER).read()
    return re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = declared()
    for n in ("pa_reshape_and_cache", "pa_decode", "pa_prefill_chunk",
              "pa_decode_workspace_size", "pa_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    from pagedattention_paged_kv_02_b200 import pa
    names = declared()
    assert set(names) == set(pa.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    from pagedattention_paged_kv_02_b200 import pa
    for code in range(7):
        assert pa.status_string(code)
    assert pa.status_string(99) == "unknown status"
    assert pa.pa_version() >> 16 == 1


def test_partition_and_workspace_arithmetic(L):
    from pagedattention_paged_kv_02_b200 import pa
    # explicit 512-token partitions over 128K tokens: 256 partials per (seq, head)
    assert pa.pa_decode_partition_tokens(131072, 512) == 512
    S = 256
    o = 4 * 32 * S * 128 * 4
    l_ = 4 * 32 * S * 4
    assert pa.pa_decode_workspace_size(4, 32, 128, 131072, 512) == o + l_
    # one partition: no workspace
    assert pa.pa_decode_workspace_size(4, 32, 128, 500, 512) == 0
    assert pa.pa_decode_workspace_size(64, 32, 128, 40, 0) == 0
    # never split: one partition covering the longest context
    assert pa.pa_decode_partition_tokens(1000, -1) == 1008
    assert pa.pa_decode_partition_tokens(1 << 20, -1) == -1
    # invalid explicit sizes
    assert pa.pa_decode_partition_tokens(1000, 24) == -1
    assert pa.pa_decode_partition_tokens(1000, 32768) == -1
    # automatic: one partition for short contexts, 1024 tokens otherwise
    assert pa.pa_decode_partition_tokens(40, 0) == 48
    assert pa.pa_decode_partition_tokens(4096, 0) == 1024


def _decode(L, **kw):
    args = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, lens=FAKE, B=4, Hq=8, Hkv=2,
                D=128, bs=16, NB=64, MB=8, max_ctx=128, scale=0.1, part=0, ws=None, ws_bytes=0,
                dtype=1)
    args.update(kw)
    return L.pa_decode(args["out"], args["q"], args["k"], args["v"], args["tables"],
                       args["lens"], args["B"], args["Hq"], args["Hkv"], args["D"], args["bs"],
                       args["NB"], args["MB"], args["max_ctx"], args["scale"], args["part"],
                       args["ws"], args["ws_bytes"], args["dtype"], None)


def test_decode_host_checks(L):
    from pagedattention_paged_kv_02_b200 import pa
    assert _decode(L, D=96) == pa.PA_ERR_UNSUPPORTED
    assert _decode(L, bs=8) == pa.PA_ERR_UNSUPPORTED
    assert _decode(L, Hq=6, Hkv=4) == pa.PA_ERR_UNSUPPORTED
    assert _decode(L, dtype=7) == pa.PA_ERR_INVALID_ARG
    assert _decode(L, q=None) == pa.PA_ERR_INVALID_ARG
    assert _decode(L, out=ctypes.c_void_p(0x10008)) == pa.PA_ERR_INVALID_ARG
    assert _decode(L, B=-1) == pa.PA_ERR_INVALID_ARG
    assert _decode(L, max_ctx=8 * 16 + 1) == pa.PA_ERR_INVALID_ARG
    assert _decode(L, scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    assert _decode(L, part=24) == pa.PA_ERR_INVALID_ARG
    # 1024 tokens in 512-token partitions need a workspace
    big = dict(MB=64, max_ctx=1024, part=512)
    assert _decode(L, **big) == pa.PA_ERR_WORKSPACE
    need = pa.pa_decode_workspace_size(4, 8, 128, 1024, 512)
    assert need > 0
    assert _decode(L, ws=FAKE, ws_bytes=need - 1, **big) == pa.PA_ERR_WORKSPACE
    assert _decode(L, ws=ctypes.c_void_p(0x10010), ws_bytes=need, **big) == pa.PA_ERR_WORKSPACE
    # zero sequences: nothing to do, no device needed
    assert _decode(L, B=0) == pa.PA_OK


def test_reshape_host_checks(L):
    from pagedattention_paged_kv_02_b200 import pa
    f = L.pa_reshape_and_cache
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 96, 16, 8, 1, None) == pa.PA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 2, 128, 16, 8, 1, None) == pa.PA_ERR_INVALID_ARG
    assert f(None, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 16, 8, 1, None) == pa.PA_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(0x10004), FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 16, 8, 1,
             None) == pa.PA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 16, 8, 5, None) == pa.PA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 128, 16, 8, 1, None) == pa.PA_OK


def test_prefill_host_checks(L):
    from pagedattention_paged_kv_02_b200 import pa
    f = L.pa_prefill_chunk
    # out, q, k, v, tables, lens, qsl, chunks, tokens, max_q, Hq, Hkv, D, bs, NB, MB, scale,
    # dtype, stream
    base = [FAKE] * 7 + [2, 1024, 512, 32, 8, 128, 16, 64, 64, 0.1, 1, None]
    assert len(base) == 19
    assert f(*base[:17], 0, None) == pa.PA_ERR_UNSUPPORTED  # fp32 has no tensor-core path
    b = list(base)
    b[12] = 96  # head_dim 64 and 128 only
    assert f(*b) == pa.PA_ERR_UNSUPPORTED
    b = list(base)
    b[10], b[11] = 12, 8
    assert f(*b) == pa.PA_ERR_UNSUPPORTED
    b = list(base)
    b[8] = -1
    assert f(*b) == pa.PA_ERR_INVALID_ARG
    b = list(base)
    b[1] = None
    assert f(*b) == pa.PA_ERR_INVALID_ARG
    b = list(base)
    b[7] = 0
    assert f(*b) == pa.PA_OK
    # work items are (query head or head pair, row tile, chunk): at most 65535 row
    # tiles and 65535 chunks; any number of query heads
    b = list(base)
    b[8], b[9] = 65536 * 256, 65536 * 256
    assert f(*b) == pa.PA_ERR_UNSUPPORTED
    b = list(base)
    b[7] = 65536
    assert f(*b) == pa.PA_ERR_UNSUPPORTED


def test_prefill_window_host_checks(L):
    from pagedattention_paged_kv_02_b200 import pa
    f = L.pa_prefill_chunk_sliding_window
    # as pa_prefill_chunk with the window before dtype
    base = [FAKE] * 7 + [2, 1024, 512, 32, 8, 128, 16, 64, 64, 0.1, 256, 1, None]
    assert len(base) == 20
    for w in (0, -5):
        b = list(base)
        b[17] = w
        assert f(*b) == pa.PA_ERR_INVALID_ARG
    b = list(base)
    b[18] = 0
    assert f(*b) == pa.PA_ERR_UNSUPPORTED  # fp32 has no tensor-core path
    b = list(base)
    b[7] = 0
    assert f(*b) == pa.PA_OK


def test_service_host_checks(L):
    from pagedattention_paged_kv_02_b200 import pa
    bad = ctypes.c_int(-1)
    assert L.pa_check_tables(FAKE, FAKE, 0, 4, 16, 8, FAKE, ctypes.byref(bad), None) == pa.PA_OK
    assert bad.value == 0
    assert L.pa_check_tables(FAKE, FAKE, -1, 4, 16, 8, FAKE, None, None) == pa.PA_ERR_INVALID_ARG
    assert L.pa_selftest_bounded_wait(0, None) == pa.PA_ERR_INVALID_ARG
    assert L.pa_selftest_bounded_wait(20_000_000_000, None) == pa.PA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from pagedattention_paged_kv_02_b200 import pa
    monkeypatch.setattr(pa, "_lib", None)
    monkeypatch.setattr(pa, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        pa.lib()


def test_shared_prefix_workspace_arithmetic(L):
    """Slots: prefix partitions then tail partitions per (sequence, head)."""
    from pagedattention_paged_kv_02_b200 import pa
    f = pa.pa_decode_shared_prefix_workspace_size

    def ws(B, Hq, D, S):
        o = B * Hq * S * D * 4
        return (o + 255) // 256 * 256 + (B * Hq * S * 4 + 255) // 256 * 256

    # explicit 256-token partitions: 1024-token prefix -> 4 slots, 1536-token
    # contexts -> 6 tail slots
    assert f(192, 32, 8, 128, 24, 8, 1024, 1536, 256) == ws(192, 32, 128, 10)
    # never split: one prefix slot and one tail slot
    assert f(192, 32, 8, 128, 24, 8, 1024, 1536, -1) == ws(192, 32, 128, 2)
    # automatic: 24 groups x 8 KV heads x 1 row tile x 2 partitions of 512
    # -> 384 prefix CTAs (>= 2 per SM), tails in one partition up to 2048
    assert f(192, 32, 8, 128, 24, 8, 1024, 1536, 0) == ws(192, 32, 128, 3)
    # few groups: 256-token prefix partitions
    assert f(16, 32, 8, 128, 2, 8, 1024, 1536, 0) == ws(16, 32, 128, 5)
    # no prefix at all: tail slots only
    assert f(8, 8, 8, 64, 8, 1, 0, 100, 0) == ws(8, 8, 64, 1)
    # invalid: odd partition, heads not grouped, prefix bound above context bound
    assert f(8, 8, 8, 128, 8, 1, 64, 100, 24) == 0
    assert f(8, 6, 4, 128, 8, 1, 64, 100, 0) == 0
    assert f(8, 8, 8, 128, 8, 0, 64, 100, 0) == 0


def _shared(L, **kw):
    args = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, lens=FAKE, gs=FAKE, pl=FAKE,
                G=2, maxg=4, maxp=64, B=8, Hq=8, Hkv=2, D=128, bs=16, NB=64, MB=8, max_ctx=128,
                scale=0.1, part=0, ws=None, ws_bytes=0, dtype=1)
    args.update(kw)
    a = args
    return L.pa_decode_shared_prefix(a["out"], a["q"], a["k"], a["v"], a["tables"], a["lens"],
                                     a["gs"], a["pl"], a["G"], a["maxg"], a["maxp"], a["B"],
                                     a["Hq"], a["Hkv"], a["D"], a["bs"], a["NB"], a["MB"],
                                     a["max_ctx"], a["scale"], a["part"], a["ws"], a["ws_bytes"],
                                     a["dtype"], None)


def test_shared_prefix_host_checks(L):
    from pagedattention_paged_kv_02_b200 import pa
    assert _shared(L, dtype=0) == pa.PA_ERR_UNSUPPORTED     # fp32: not offered
    assert _shared(L, D=96) == pa.PA_ERR_UNSUPPORTED
    assert _shared(L, Hq=6, Hkv=4) == pa.PA_ERR_UNSUPPORTED
    assert _shared(L, gs=None) == pa.PA_ERR_INVALID_ARG
    assert _shared(L, pl=ctypes.c_void_p(0x10002)) == pa.PA_ERR_INVALID_ARG
    assert _shared(L, maxg=0) == pa.PA_ERR_INVALID_ARG
    assert _shared(L, maxp=129) == pa.PA_ERR_INVALID_ARG   # prefix bound above the context bound
    assert _shared(L, G=0) == pa.PA_ERR_INVALID_ARG        # sequences but no groups
    assert _shared(L, part=24) == pa.PA_ERR_INVALID_ARG
    # the workspace is always needed: both passes leave partials
    assert _shared(L) == pa.PA_ERR_WORKSPACE
    need = pa.pa_decode_shared_prefix_workspace_size(8, 8, 2, 128, 2, 4, 64, 128, 0)
    assert _shared(L, ws=FAKE, ws_bytes=need - 1) == pa.PA_ERR_WORKSPACE
    assert _shared(L, ws=ctypes.c_void_p(0x10010), ws_bytes=need) == pa.PA_ERR_WORKSPACE
    assert _shared(L, B=0, G=0) == pa.PA_OK
