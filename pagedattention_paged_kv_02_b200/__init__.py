"""PagedAttention paged-KV decode for B200 (sm_100a).

The compute lives in ``libpa.so`` (hand-written CUDA, C ABI declared in
``include/pa.h``). ``pagedattention_paged_kv_02_b200.pa`` is the thin ctypes
binding with the same entry-point names; ``pagedattention_paged_kv_02_b200.workloads``
builds seeded synthetic inputs. Import the submodule you need: the package
itself loads nothing, so the input generators work on a host without the
built library.
"""
