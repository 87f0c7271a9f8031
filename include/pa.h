/*
 * pa.h -- C ABI of libpa.so: paged-KV attention on B200 (sm_100a).
 *
 * The operations, by the page and section that define them:
 *
 *  pa_reshape_and_cache
 *      page "字节跳动 AI Infra (2)", question "KV Cache原理与优化": at step t
 *      the new token's K_t and V_t are appended to the cache
 *      (K_cache = concat(K_cache, K_t)). In paged form the append is a
 *      scatter into a slot of a physical block (same page, question
 *      "vLLM与PagedAttention的原理": a block of block_size tokens starts at
 *      physical_block * block_size * head_dim).
 *
 *  pa_decode
 *      same page, "KV Cache原理与优化": Attention_t = softmax(Q_t K^T / sqrt(d)) V
 *      for the one new query of each sequence, with K/V reached through the
 *      sequence's block table ("vLLM与PagedAttention的原理"); query heads
 *      share K/V heads in groups (page "LLM推理优化", section 1.3, GQA/MQA);
 *      long contexts are split along the KV length and the partial results
 *      merged (page "字节跳动 AI Infra (2)", algorithm-level table, row
 *      FlashDecoding), using online-softmax statistics (page "LLM推理优化",
 *      section 2.1, FlashAttention's tiling and online softmax).
 *
 *  pa_prefill_chunk
 *      page "vLLM框架是怎么做推理加速的", section 3 (Chunked Prefill): a
 *      prompt is processed in chunks (512 tokens by default) that attend
 *      over the paged cache; attention within the prompt is causal (page
 *      "LLM推理优化", section 2.3, causal=True).
 *
 * Data layout (all device memory, row-major, owned by the caller):
 *   k_cache, v_cache   [num_blocks][num_kv_heads][block_size][head_dim]
 *                      One (block, kv head) page of block_size*head_dim
 *                      elements is contiguous. With num_kv_heads == 1 this is
 *                      exactly the pages' pointer formula.
 *   block_tables       int32 [rows][max_blocks_per_seq]; entry i of row r is
 *                      the physical block holding tokens [i*bs, (i+1)*bs) of
 *                      sequence (or chunk) r. Entries past the valid tokens
 *                      are never read.
 *   context_lens       int32 [rows]; valid tokens of the row, including any
 *                      token(s) appended in this step.
 *   slot_mapping       int64 [num_tokens]; slot = physical_block*bs + offset.
 *                      Negative slots are padding and are skipped.
 *   q / out (decode)   [num_seqs][num_q_heads][head_dim]
 *   q / out (prefill)  [total_q][num_q_heads][head_dim], chunk c owning rows
 *                      [query_start_loc[c], query_start_loc[c+1]).
 *   key / value        [num_tokens][num_kv_heads][head_dim]
 *   Query head h reads K/V head h / (num_q_heads / num_kv_heads).
 *   q, out, key, value and the caches all have element type `dtype`;
 *   accumulation is fp32; bf16 outputs are rounded to nearest even.
 *
 * Conventions:
 *   - Every call is asynchronous on `stream`, never allocates device memory,
 *     and never synchronises, except where a function says otherwise.
 *   - Argument checks run on the host before any launch. A failed check
 *     returns an error code, launches nothing and writes nothing.
 *   - Supported: head_dim in {64, 128}; block_size in {16, 32, 64};
 *     num_q_heads % num_kv_heads == 0. Anything else returns
 *     PA_ERR_UNSUPPORTED. Cache, q, out, key and value pointers must be
 *     16-byte aligned, table and length pointers 4-byte aligned.
 *   - Device data the host cannot see (block ids, lengths, slots) is checked
 *     on the device: an out-of-range block id or slot is skipped, never
 *     dereferenced, and recorded in a sticky device error word that
 *     pa_device_error() reads. Device-side waits are bounded; a wait that
 *     runs out records PA_ERR_TIMEOUT there and the kernel returns.
 *   - A launch failure returns PA_ERR_CUDA (cudaGetLastError is consumed).
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1, /* null pointer, negative size, misalignment, bad dtype */
    PA_ERR_UNSUPPORTED = 2, /* shape outside the supported set */
    PA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
    PA_ERR_BAD_TABLE = 4,   /* a block id, slot or length outside its range */
    PA_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out */
    PA_ERR_CUDA = 6         /* a CUDA runtime call or launch failed */
} pa_status;

typedef enum { PA_F32 = 0, PA_BF16 = 1 } pa_dtype;

/* Scatter new tokens' K/V rows into their cache slots:
 *   for t with s = slot_mapping[t] >= 0 and every kv head h:
 *     k_cache[s / block_size][h][s % block_size][:] = key[t][h][:]
 *     v_cache[s / block_size][h][s % block_size][:] = value[t][h][:]
 * Rows are copied bit for bit. A slot >= num_blocks*block_size is skipped
 * and recorded as PA_ERR_BAD_TABLE in the device error word. Slots must be
 * distinct (two tokens writing one slot race). num_tokens == 0 is a no-op. */
PA_API pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                               const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                               cudaStream_t stream);

/* Bytes of workspace pa_decode needs for these sizes and partition_size
 * (same meaning as in pa_decode). 0 when every sequence fits one partition. */
PA_API size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                int partition_size);

/* Token count of one KV partition that pa_decode uses for these arguments
 * (resolves partition_size == 0 and < 0), or -1 for invalid arguments. */
PA_API int pa_decode_partition_tokens(int max_context_len, int partition_size);

/* Paged decode attention, one query per sequence:
 *   out[b][h] = sum_j softmax_j(scale * q[b][h] . K_j) V_j
 * over positions j < context_lens[b] of sequence b, K_j/V_j read from head
 * h / (num_q_heads/num_kv_heads) of physical block block_tables[b][j / bs]
 * at offset j % bs.
 *   max_context_len   host-side upper bound of context_lens (lengths above
 *                     it, or above max_blocks_per_seq*block_size, are clamped
 *                     and recorded as PA_ERR_BAD_TABLE).
 *   partition_size    KV tokens per split (multiple of 16, <= 16384);
 *                     0 = choose automatically; < 0 = never split. Sequences
 *                     longer than one partition are computed as partial
 *                     results merged by log-sum-exp.
 *   workspace         device scratch of >= pa_decode_workspace_size(...)
 *                     bytes (may be NULL when that is 0), 256-byte aligned;
 *                     contents on entry are ignored.
 * A sequence with context_len 0 yields out = 0. */
PA_API pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                    int partition_size, void *workspace, size_t workspace_bytes, pa_dtype dtype,
                    cudaStream_t stream);

/* Paged decode for batches whose sequences share prefix blocks, reading
 * each shared block once for all its readers: page "字节跳动 AI Infra (2)",
 * question "vLLM与PagedAttention的原理" (beams of one request share prefix
 * blocks, B1 and B3 in its example; a partially filled shared block is
 * copied on write, B6'), with the split of each sequence's attention into a
 * prefix part and a private part merged by log-sum-exp (same page,
 * algorithm-level table, FlashDecoding row). The result is pa_decode's:
 *   out[b][h] = sum_{j < context_lens[b]} softmax_j(scale * q[b][h] . K_j) V_j.
 *   group_start   int32 [num_groups + 1], device: sequences are listed group
 *                 by group; group g is [group_start[g], group_start[g+1]).
 *                 The groups partition [0, num_seqs) (group_start[0] = 0,
 *                 group_start[num_groups] = num_seqs, non-decreasing); a
 *                 sequence that shares nothing is a group of one.
 *   prefix_lens   int32 [num_groups], device: group g's sequences hold the
 *                 same K/V at positions [0, prefix_lens[g]) -- shared
 *                 physical blocks, or copies of them. Those positions are
 *                 read once per KV head through the table of the group's
 *                 first sequence, for all of its sequences. The length used
 *                 is min(prefix_lens[g], every member's context_len), and it
 *                 need not be a multiple of block_size.
 *   max_group_size, max_prefix_len   host-side bounds of the group sizes and
 *                 prefix lengths. A malformed group, a group larger than
 *                 max_group_size or a prefix longer than max_prefix_len is
 *                 recorded as PA_ERR_BAD_TABLE (the outputs of that group's
 *                 sequences are then unspecified).
 *   partition_size   KV tokens per split of both the prefix and the tails
 *                 (multiple of 16, <= 16384); 0 = automatic; < 0 = one
 *                 partition each.
 *   workspace     >= pa_decode_shared_prefix_workspace_size(...) bytes,
 *                 256-byte aligned, always needed (the two passes always
 *                 leave partials).
 * bf16 only (fp32 returns PA_ERR_UNSUPPORTED); other arguments, limits and
 * errors as for pa_decode. Three launches on `stream`: the prefix pass, the
 * private-tail pass (which may start while the prefix pass runs) and the
 * log-sum-exp merge. */
PA_API size_t pa_decode_shared_prefix_workspace_size(int num_seqs, int num_q_heads,
                                                     int num_kv_heads, int head_dim,
                                                     int num_groups, int max_group_size,
                                                     int max_prefix_len, int max_context_len,
                                                     int partition_size);
PA_API pa_status pa_decode_shared_prefix(void *out, const void *q, const void *k_cache,
                                         const void *v_cache, const int32_t *block_tables,
                                         const int32_t *context_lens, const int32_t *group_start,
                                         const int32_t *prefix_lens, int num_groups,
                                         int max_group_size, int max_prefix_len, int num_seqs,
                                         int num_q_heads, int num_kv_heads, int head_dim,
                                         int block_size, int num_blocks, int max_blocks_per_seq,
                                         int max_context_len, float scale, int partition_size,
                                         void *workspace, size_t workspace_bytes,
                                         pa_dtype dtype, cudaStream_t stream);

/* FP8 KV cache (E4M3 codes, one byte per element, one dequantisation scale
 * per K/V head for K and one for V): page "字节跳动 AI Infra (2)", optimisation
 * table, KV quantisation row, and page "LLM推理优化", section 1.3 (store K/V
 * in low precision). Element value = code * scale[kv head].
 *
 * pa_reshape_and_cache_fp8: as pa_reshape_and_cache, with k_cache/v_cache
 * uint8 [num_blocks][num_kv_heads][block_size][head_dim] and key/value of
 * `dtype` (fp32 or bf16); each element is stored as the E4M3 code nearest to
 * the IEEE fp32 quotient x / scale[h] (ties to even; magnitudes beyond 448
 * saturate to +-448). k_scale/v_scale: device float [num_kv_heads]. */
PA_API pa_status pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache,
                                          void *v_cache, const int64_t *slot_mapping,
                                          int num_tokens, int num_kv_heads, int head_dim,
                                          int block_size, int num_blocks, const float *k_scale,
                                          const float *v_scale, pa_dtype dtype,
                                          cudaStream_t stream);

/* pa_decode_fp8: as pa_decode over E4M3 caches (uint8, layout as above) with
 * per-K/V-head scales; q and out are bf16; head_dim must be 128. The same
 * workspace sizes apply (pa_decode_workspace_size). */
PA_API pa_status pa_decode_fp8(void *out, const void *q, const void *k_cache, const void *v_cache,
                               const float *k_scale, const float *v_scale,
                               const int32_t *block_tables, const int32_t *context_lens,
                               int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int num_blocks, int max_blocks_per_seq,
                               int max_context_len, float scale, int partition_size,
                               void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* INT8 KV cache (one int8 code per element, one dequantisation scale per K/V
 * head for K and one for V): page "字节跳动 AI Infra (2)", optimisation table,
 * row "KV量化(INT8)", and page "LLM推理优化", section 1.3 (INT8 K/V). Element
 * value = code * scale[kv head].
 *
 * pa_reshape_and_cache_int8: as pa_reshape_and_cache_fp8 with int8 caches;
 * each element is stored as the integer nearest to the IEEE fp32 quotient
 * x / scale[h] (ties to even), saturated to [-127, 127]; NaN stores 0. */
PA_API pa_status pa_reshape_and_cache_int8(const void *key, const void *value, void *k_cache,
                                           void *v_cache, const int64_t *slot_mapping,
                                           int num_tokens, int num_kv_heads, int head_dim,
                                           int block_size, int num_blocks, const float *k_scale,
                                           const float *v_scale, pa_dtype dtype,
                                           cudaStream_t stream);

/* pa_decode_int8: as pa_decode_fp8 over INT8 caches (int8, same layout and
 * arguments). */
PA_API pa_status pa_decode_int8(void *out, const void *q, const void *k_cache, const void *v_cache,
                                const float *k_scale, const float *v_scale,
                                const int32_t *block_tables, const int32_t *context_lens,
                                int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                int block_size, int num_blocks, int max_blocks_per_seq,
                                int max_context_len, float scale, int partition_size,
                                void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* pa_decode without a caller-provided workspace. The pages have no
 * counterpart: this exists for callers that cannot allocate device memory at
 * the call site (a plugin handed only its input and output buffers, or a
 * latency-critical caller that may not run cudaMalloc, which can synchronise
 * the device). Arguments and results are those of pa_decode minus the
 * workspace; the partial results live in a 16 MiB device array built into
 * the library, which every GPU that loads the library keeps until exit.
 *   - A request whose workspace (pa_decode_workspace_size) exceeds 16 MiB is
 *     refused with PA_ERR_WORKSPACE before anything is launched.
 *   - Set-up: the first call in a CUDA context (per device; again after
 *     cudaDeviceReset) looks up the array's device address with that device
 *     current. With lazy module loading, CUDA's default, that first call --
 *     or the first launch of any libpa kernel on the device, whichever comes
 *     first -- also loads the library's device code and so reserves the
 *     16 MiB, which allocates and can synchronise. A call with num_seqs = 0
 *     does this set-up and launches nothing: make it at start-up, before
 *     any stream capture.
 *   - All calls share the one array: two calls whose kernels overlap on the
 *     GPU (different streams, no ordering between them) race and may return
 *     wrong results. Calls ordered on one stream are safe; nothing needs to
 *     be cleared between them.
 *   - After set-up, allocates nothing (no cudaMalloc, cudaFree or allocating
 *     library call). */
PA_API pa_status pa_decode_static_workspace(void *out, const void *q, const void *k_cache,
                                            const void *v_cache, const int32_t *block_tables,
                                            const int32_t *context_lens, int num_seqs,
                                            int num_q_heads, int num_kv_heads, int head_dim,
                                            int block_size, int num_blocks,
                                            int max_blocks_per_seq, int max_context_len,
                                            float scale, int partition_size, pa_dtype dtype,
                                            cudaStream_t stream);

/* pa_decode restricted to a sliding window (page "LLM推理优化", section 2.3,
 * flash_attn_func window_size; page "vLLM框架是怎么做推理加速的", 追问 3,
 * sliding window attention): sequence b's query attends only positions
 * [max(0, context_lens[b] - sliding_window), context_lens[b]). Table entries
 * of blocks wholly before the window are never read (an engine may have
 * freed them). sliding_window must be > 0; other arguments, workspace sizes
 * and errors as for pa_decode. */
PA_API pa_status pa_decode_sliding_window(void *out, const void *q, const void *k_cache,
                                          const void *v_cache, const int32_t *block_tables,
                                          const int32_t *context_lens, int num_seqs,
                                          int num_q_heads, int num_kv_heads, int head_dim,
                                          int block_size, int num_blocks,
                                          int max_blocks_per_seq, int max_context_len,
                                          float scale, int sliding_window, int partition_size,
                                          void *workspace, size_t workspace_bytes,
                                          pa_dtype dtype, cudaStream_t stream);

/* Chunked prefill: chunk c has C_c = query_start_loc[c+1] - query_start_loc[c]
 * queries and context_lens[c] tokens in the cache (its own C_c tokens
 * included, already written by pa_reshape_and_cache). Query i of the chunk
 * sits at position p = context_lens[c] - C_c + i and attends positions 0..p:
 *   out[r][h] = sum_{j<=p} softmax_j(scale * q[r][h] . K_j) V_j,  r = qsl[c]+i.
 *   num_query_tokens  rows of q and out (query_start_loc[num_chunks]); a
 *                     chunk reaching past it, with C_c < 0 (decreasing
 *                     query_start_loc), with context_lens[c] < C_c or above
 *                     max_blocks_per_seq*block_size is skipped and recorded
 *                     as PA_ERR_BAD_TABLE.
 *   max_query_len     host-side upper bound of every C_c. The work covers
 *                     max_query_len rounded up to whole row tiles per chunk
 *                     (128 rows when num_q_heads / num_kv_heads is even, else
 *                     256); the rows of a longer chunk past that are left
 *                     unwritten and the chunk is recorded as PA_ERR_BAD_TABLE.
 * bf16 with head_dim 64 or 128 (the tcgen05 tensor-core path), at most
 * 65535 chunks and max_query_len at most 65535 * 128; anything else returns
 * PA_ERR_UNSUPPORTED. */
PA_API pa_status pa_prefill_chunk(void *out, const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *block_tables, const int32_t *context_lens,
                           const int32_t *query_start_loc, int num_chunks, int num_query_tokens,
                           int max_query_len,
                           int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, int max_blocks_per_seq, float scale, pa_dtype dtype,
                           cudaStream_t stream);

/* pa_prefill_chunk restricted to a sliding window (page "LLM推理优化",
 * section 2.3, flash_attn_func window_size; page "vLLM框架是怎么做推理加速的",
 * 追问 3, sliding window attention): query i of chunk c, at position p,
 * attends positions [max(0, p - sliding_window + 1), p] only, the band a
 * pa_decode_sliding_window query at position context_lens[b] - 1 sees.
 * Table entries of blocks wholly before the chunk's first query's band are
 * never read (an engine may have freed them). sliding_window must be > 0;
 * other arguments and errors as for pa_prefill_chunk. */
PA_API pa_status pa_prefill_chunk_sliding_window(void *out, const void *q, const void *k_cache,
                                                 const void *v_cache, const int32_t *block_tables,
                                                 const int32_t *context_lens,
                                                 const int32_t *query_start_loc, int num_chunks,
                                                 int num_query_tokens, int max_query_len,
                                                 int num_q_heads, int num_kv_heads, int head_dim,
                                                 int block_size, int num_blocks,
                                                 int max_blocks_per_seq, float scale,
                                                 int sliding_window, pa_dtype dtype,
                                                 cudaStream_t stream);

/* Copy-on-write of whole blocks inside one pool: for each pair i of
 * block_mapping (int64 [num_pairs][2], device-readable), block
 * block_mapping[i][1] := block block_mapping[i][0], every kv head, K and V,
 * bit for bit. This is how a beam gets its own copy of a shared, partially
 * filled block before writing into it (page "字节跳动 AI Infra (2)", question
 * "vLLM与PagedAttention的原理": B6' is a copy-on-write copy of B6).
 * Destinations must be distinct and must not be sources of other pairs (the
 * pairs run concurrently). An id outside [0, num_blocks) skips its pair and
 * is recorded as PA_ERR_BAD_TABLE. */
PA_API pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping,
                                int num_pairs, int num_kv_heads, int head_dim, int block_size,
                                int num_blocks, pa_dtype dtype, cudaStream_t stream);

/* Whole-block copies between two pools of the same block shape, e.g. the
 * device pool and a pinned host pool holding swapped-out requests (page
 * "字节跳动 AI Infra (2)", scheduler: KV caches are swapped to CPU memory when
 * GPU memory runs short, and back). For each pair i: block mapping[i][1] of
 * (dst_k, dst_v) := block mapping[i][0] of (src_k, src_v). Every pointer must
 * be addressable by the GPU: device memory, or pinned host memory (page-
 * locked with cudaHostAlloc / cudaHostRegister, addressed through unified
 * virtual addressing); the copy then runs over the host link inside one
 * kernel. Ids outside their pool skip the pair and are recorded as
 * PA_ERR_BAD_TABLE. */
PA_API pa_status pa_swap_blocks(const void *src_k, const void *src_v, int src_blocks,
                                void *dst_k, void *dst_v, int dst_blocks,
                                const int64_t *block_mapping, int num_pairs, int num_kv_heads,
                                int head_dim, int block_size, pa_dtype dtype,
                                cudaStream_t stream);

/* Check block tables and lengths on the device: every entry a row's valid
 * tokens reach must lie in [0, num_blocks), and 0 <= context_lens[r] <=
 * max_blocks_per_seq*block_size. d_scratch is one caller-owned device int32.
 * SYNCHRONOUS: waits for `stream`, stores the number of bad rows in
 * *bad_rows (may be NULL) and returns PA_ERR_BAD_TABLE if any. */
PA_API pa_status pa_check_tables(const int32_t *block_tables, const int32_t *context_lens, int rows,
                          int max_blocks_per_seq, int block_size, int num_blocks,
                          int32_t *d_scratch, int *bad_rows, cudaStream_t stream);

/* Read (and with clear != 0 reset) the sticky device error word of the
 * current device: PA_OK, PA_ERR_BAD_TABLE or PA_ERR_TIMEOUT, the first one
 * recorded. SYNCHRONOUS: waits for all prior work on the device. */
PA_API pa_status pa_device_error(int *status, int clear);

/* Failure-detection self test: launch one CTA that waits, with a bound of
 * timeout_ns nanoseconds, on a barrier nothing will complete. The wait runs
 * out, the kernel records PA_ERR_TIMEOUT in the device error word and
 * returns; the GPU context stays usable. Asynchronous on `stream`. */
PA_API pa_status pa_selftest_bounded_wait(long long timeout_ns, cudaStream_t stream);

/* Static description of a status code. */
PA_API const char *pa_status_string(pa_status status);

/* ABI version, (major << 16) | minor. */
PA_API int pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
