// blocks.cuh -- whole-block copies of the paged pool.
//
// Page "字节跳动 AI Infra (2)", question "vLLM与PagedAttention的原理": beams
// share prefix blocks, and a beam about to write into a shared, partially
// filled block first gets its own copy of it (B6' is a copy-on-write copy of
// B6). The same page's scheduler moves a swapped-out request's KV cache to
// CPU memory and back. Both are copies of whole physical blocks (every K/V
// head, K and V): block d of the destination pool := block s of the source.
//
// One CTA per (source, destination) pair; its threads move the block's K and
// V bytes in 16-byte vectors, fully coalesced on both sides. Either pool may
// be pinned host memory the GPU addresses directly (a swap then streams over
// the host link without staging). Bound: the copy bandwidth of the slower
// side; algorithmic bytes 2 x 2 x pairs x block bytes (read + write, K + V).
#pragma once

#include "pa_device.cuh"

namespace pa {

struct CopyArgs {
    const uint4 *src_k;
    const uint4 *src_v;
    uint4 *dst_k;
    uint4 *dst_v;
    const int64_t *mapping;  // [num_pairs][2]: (source block, destination block)
    long long src_blocks, dst_blocks;
    int vecs_per_block;      // block bytes / 16
};

__global__ void __launch_bounds__(256) copy_blocks_kernel(const __grid_constant__ CopyArgs a) {
    const long long pair = blockIdx.x;
    const long long s = a.mapping[2 * pair], d = a.mapping[2 * pair + 1];
    if (s < 0 || s >= a.src_blocks || d < 0 || d >= a.dst_blocks) {
        if (threadIdx.x == 0) flag_error(PA_ERR_BAD_TABLE);
        return;
    }
    const size_t so = (size_t)s * a.vecs_per_block, dof = (size_t)d * a.vecs_per_block;
    for (int v = threadIdx.x; v < a.vecs_per_block; v += 256) {
        const uint4 kv = a.src_k[so + v];
        const uint4 vv = a.src_v[so + v];
        a.dst_k[dof + v] = kv;
        a.dst_v[dof + v] = vv;
    }
}

}  // namespace pa
