// reshape_and_cache.cuh -- the append step of decode in paged form.
//
// Page "字节跳动 AI Infra (2)", question "KV Cache原理与优化": each step appends
// the new token's K_t and V_t to the cache. With the cache paged (same page,
// question "vLLM与PagedAttention的原理") the append writes each new token's
// rows into the slot the block manager assigned it: physical block
// slot / block_size, offset slot % block_size.
//
// One thread moves one 16-byte vector of K and the matching vector of V:
// blockIdx.y walks the tokens, blockIdx.x/threadIdx.x the vectors of a token
// (num_kv_heads rows of head_dim*elem bytes), so reads of key/value are fully
// coalesced and each (token, kv head) row lands contiguously in its page.
// Row length and block size are powers of two: positions are shifts and
// masks, no integer division. Memory-bound: 2 * num_tokens * num_kv_heads *
// head_dim * elem bytes read and written.
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kScatterThreads = 128;

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

__global__ void __launch_bounds__(kScatterThreads)
    reshape_and_cache_kernel(const __grid_constant__ ReshapeArgs a) {
    const int r = blockIdx.x * kScatterThreads + threadIdx.x;  // vector within the token
    if (r >= a.vecs_per_token) return;
    const int h = r >> a.row_shift;
    const int c = r & ((1 << a.row_shift) - 1);
    for (long long t = blockIdx.y; t < a.num_tokens; t += gridDim.y) {
        const long long slot = __ldg(a.slot_mapping + t);
        if (slot < 0) continue;  // padding token
        if (slot >= a.num_slots) {
            flag_error(PA_ERR_BAD_TABLE);
            continue;
        }
        const long long block = slot >> a.bs_shift;
        const long long offset = slot & ((1LL << a.bs_shift) - 1);
        const long long dst =
            (((block * a.num_kv_heads + h) << a.bs_shift) + offset) * (1LL << a.row_shift) + c;
        const long long i = t * a.vecs_per_token + r;
        const uint4 kv = __ldg(a.key + i);
        const uint4 vv = __ldg(a.value + i);
        a.k_cache[dst] = kv;
        a.v_cache[dst] = vv;
    }
}

}  // namespace pa
