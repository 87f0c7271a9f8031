// reshape_and_cache.cuh -- the append step of decode in paged form.
//
// Page "字节跳动 AI Infra (2)", question "KV Cache原理与优化": each step appends
// the new token's K_t and V_t to the cache. With the cache paged (same page,
// question "vLLM与PagedAttention的原理") the append writes each new token's
// rows into the slot the block manager assigned it: physical block
// slot / block_size, offset slot % block_size.
//
// A thread moves one 16-byte vector of K and the matching vector of V for
// each of a few tokens: blockIdx.y walks groups of tokens, blockIdx.x /
// threadIdx.x the vectors of a token (num_kv_heads rows of head_dim*elem
// bytes), so reads of key/value are fully coalesced and each (token, kv head)
// row lands contiguously in its page.
// Row length and block size are powers of two: positions are shifts and
// masks, no integer division. Memory-bound: 2 * num_tokens * num_kv_heads *
// head_dim * elem bytes read and written.
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kScatterThreads = 128;
constexpr int kScatterTokens = 4;  // tokens a thread moves per pass

struct ReshapeArgs {
    const uint4 *key;
    const uint4 *value;
    uint4 *k_cache;
    uint4 *v_cache;
    const int64_t *slot_mapping;
    long long num_tokens;
    int vecs_per_token;  // num_kv_heads * vecs_per_row
    int row_shift;       // log2(vecs_per_row), vecs_per_row = head_dim * elem / 16
    int bs_shift;        // log2(block_size)
    int num_kv_heads;
    long long num_slots;  // num_blocks * block_size
};

// Each thread moves one 16-byte vector of K and of V for kScatterTokens
// tokens (blockIdx.y walks groups of tokens): it loads all their slots and
// rows first, so the slot lookups and the row reads are in flight together,
// then stores the rows whose slots are valid.
__global__ void __launch_bounds__(kScatterThreads)
    reshape_and_cache_kernel(const __grid_constant__ ReshapeArgs a) {
    const int r = blockIdx.x * kScatterThreads + threadIdx.x;  // vector within the token
    if (r >= a.vecs_per_token) return;
    const int h = r >> a.row_shift;
    const int c = r & ((1 << a.row_shift) - 1);
    for (long long t0 = (long long)blockIdx.y * kScatterTokens; t0 < a.num_tokens;
         t0 += (long long)gridDim.y * kScatterTokens) {
        long long slot[kScatterTokens];
        uint4 kv[kScatterTokens], vv[kScatterTokens];
#pragma unroll
        for (int u = 0; u < kScatterTokens; ++u) {
            const long long t = t0 + u;
            slot[u] = -1;
            if (t < a.num_tokens) {
                slot[u] = __ldg(a.slot_mapping + t);
                const long long i = t * a.vecs_per_token + r;
                kv[u] = __ldg(a.key + i);
                vv[u] = __ldg(a.value + i);
            }
        }
#pragma unroll
        for (int u = 0; u < kScatterTokens; ++u) {
            if (slot[u] < 0) continue;  // padding token (or past the end)
            if (slot[u] >= a.num_slots) {
                flag_error(PA_ERR_BAD_TABLE);
                continue;
            }
            const long long block = slot[u] >> a.bs_shift;
            const long long offset = slot[u] & ((1LL << a.bs_shift) - 1);
            const long long dst =
                (((block * a.num_kv_heads + h) << a.bs_shift) + offset) * (1LL << a.row_shift) + c;
            a.k_cache[dst] = kv[u];
            a.v_cache[dst] = vv[u];
        }
    }
}

}  // namespace pa
