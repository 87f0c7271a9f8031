// reshape_and_cache.cuh -- the append step of decode in paged form.
//
// Page "字节跳动 AI Infra (2)", question "KV Cache原理与优化": each step appends
// the new token's K_t and V_t to the cache. With the cache paged (same page,
// question "vLLM与PagedAttention的原理") the append writes each new token's
// rows into the slot the block manager assigned it: physical block
// slot / block_size, offset slot % block_size.
//
// One thread moves one 16-byte vector of K and the matching vector of V.
// Reads of key/value are fully coalesced; each (token, kv head) row of
// head_dim*elem bytes lands contiguously in its page. Memory-bound:
// 2 * num_tokens * num_kv_heads * head_dim * elem bytes read and written.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct ReshapeArgs {
    const uint4 *key;
    const uint4 *value;
    uint4 *k_cache;
    uint4 *v_cache;
    const int64_t *slot_mapping;
    long long total_vecs;  // num_tokens * vecs_per_token
    int vecs_per_row;      // head_dim * elem / 16
    int vecs_per_token;    // num_kv_heads * vecs_per_row
    int num_kv_heads;
    int block_size;
    long long num_slots;  // num_blocks * block_size
};

__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const __grid_constant__ ReshapeArgs a) {
    const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (i >= a.total_vecs) return;
    const long long t = i / a.vecs_per_token;
    const int r = static_cast<int>(i - t * a.vecs_per_token);
    const int h = r / a.vecs_per_row;
    const int c = r - h * a.vecs_per_row;
    const long long slot = __ldg(a.slot_mapping + t);
    if (slot < 0) return;  // padding token
    if (slot >= a.num_slots) {
        flag_error(PA_ERR_BAD_TABLE);
        return;
    }
    const long long block = slot / a.block_size;
    const long long offset = slot - block * a.block_size;
    const long long dst = ((block * a.num_kv_heads + h) * a.block_size + offset) * a.vecs_per_row + c;
    const uint4 kv = __ldg(a.key + i);
    const uint4 vv = __ldg(a.value + i);
    a.k_cache[dst] = kv;
    a.v_cache[dst] = vv;
}

}  // namespace pa
