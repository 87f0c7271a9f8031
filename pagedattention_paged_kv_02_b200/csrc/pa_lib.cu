// pa_lib.cu -- the C ABI of libpa.so (declared in include/pa.h): host-side
// argument checks, launch configuration, TMA descriptors, and the small
// service kernels (table check, error word, bounded-wait self test).
//
// Everything is one translation unit so that every kernel records into the
// same device error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "pa.h"
#include "pa_device.cuh"
#include "reshape_and_cache.cuh"
#include "decode.cuh"
#include "decode_merge.cuh"
#include "decode_prefix.cuh"
#include "decode_fp8.cuh"
#include "prefill.cuh"
#include "blocks.cuh"

namespace {

using namespace pa;

constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s per bounded wait

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool head_dim_ok(int d) { return d == 64 || d == 128; }
bool block_size_ok(int bs) { return bs == 16 || bs == 32 || bs == 64; }

pa_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime so
// that the library does not link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// A 4-D view [num_blocks][H_kv][bs][D] of a bf16 cache with a box of
// box_rows tokens x 64 dims (128 bytes) and 128-byte swizzle.
bool encode_cache_map(CUtensorMap *m, const void *cache, int NB, int H_kv, int bs, int D,
                      int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)bs, (cuuint64_t)H_kv, (cuuint64_t)NB};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)bs * D * 2,
                             (cuuint64_t)H_kv * bs * D * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(cache), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// KV tokens per partition, or -1 if the request cannot be met.
int partition_tokens(int max_ctx, int partition_size) {
    if (max_ctx < 0) return -1;
    if (partition_size > 0) {
        if (partition_size % kChunk != 0 || partition_size > kMaxPartition) return -1;
        return partition_size;
    }
    const int whole = ((max_ctx > 0 ? max_ctx : 1) + kChunk - 1) / kChunk * kChunk;
    if (partition_size < 0) return whole <= kMaxPartition ? whole : -1;
    return max_ctx <= 1024 ? whole : 1024;  // automatic
}

size_t workspace_bytes(int B, int H_q, int D, int max_ctx, int P) {
    const long long S = (max_ctx + P - 1) / P;
    if (S <= 1) return 0;
    const size_t o = (size_t)B * H_q * S * D * sizeof(float);
    const size_t l = (size_t)B * H_q * S * sizeof(float);
    return (o + 255) / 256 * 256 + (l + 255) / 256 * 256;
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// ------------------------------------------------------------- decode
// Launch shapes (measured on B200 in sweeps of warps x stages): the bf16
// and fp32 split kernels run 4 warps with 2-deep per-warp TMA rings; the
// 8-bit kernel 4 warps x 2 stages of 32 tokens.
constexpr int kDecodeWarps = 4;
constexpr int kDecodeStages = 2;
constexpr int kQ8Tokens = 32;

template <int D, int NW, int NS>
pa_status launch_decode_bf16(const DecodeArgs &a, const CUtensorMap &mk, const CUtensorMap &mv,
                             dim3 grid, cudaStream_t st) {
    constexpr int STAGE = 2 * kChunk * D * 2;
    using L = DecodeSmem<NW, NS, STAGE, kHeadsBf16, D>;
    const size_t smem = 1024 + L::kTable + ((size_t)a.P / a.bs + 2) * 4;
    auto k = decode_split_bf16<D, NW, NS>;
    if (set_smem(k, smem) != cudaSuccess) return PA_ERR_CUDA;
    k<<<grid, NW * 32, smem, st>>>(a, mk, mv);
    return launch_status();
}

template <int D, int NW, int NS>
pa_status launch_decode_f32(const DecodeArgs &a, dim3 grid, cudaStream_t st) {
    constexpr int STAGE = 2 * kChunk * D * 4;
    using L = DecodeSmem<NW, NS, STAGE, kHeadsF32, D>;
    const size_t smem = 1024 + L::kTable + ((size_t)a.P / a.bs + 2) * 4;
    auto k = decode_split_f32<D, NW, NS>;
    if (set_smem(k, smem) != cudaSuccess) return PA_ERR_CUDA;
    k<<<grid, NW * 32, smem, st>>>(a);
    return launch_status();
}

template <int D, bool WIN>
pa_status launch_prefill_tc(const PrefillArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                            const CUtensorMap &mv, dim3 grid, cudaStream_t st) {
    const size_t smem = 1024 + pf_smem_bytes(D);
    auto k = prefill_tc_kernel<D, WIN>;
    if (set_smem(k, smem) != cudaSuccess) return PA_ERR_CUDA;
    // the kernel's register split must fit the registers it launches with,
    // or the warpgroups that grow would wait forever
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, k) != cudaSuccess) return PA_ERR_CUDA;
    if ((long long)fa.numRegs * kPfThreads < kPfRegsNeeded) return PA_ERR_UNSUPPORTED;
    k<<<grid, kPfThreads, smem, st>>>(a, mq, mk, mv);
    return launch_status();
}

// A 4-D view [num_blocks][H_kv][bs][128] of a one-byte (E4M3) cache with a
// box of 16 tokens x 128 dims (128 bytes) and 128-byte swizzle.
bool encode_cache_map_u8(CUtensorMap *m, const void *cache, int NB, int H_kv, int bs) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {128, (cuuint64_t)bs, (cuuint64_t)H_kv, (cuuint64_t)NB};
    cuuint64_t strides[3] = {128, (cuuint64_t)bs * 128, (cuuint64_t)H_kv * bs * 128};
    cuuint32_t box[4] = {128, (cuuint32_t)kChunk, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(cache), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NW, int NS, int CT, bool INT8>
pa_status launch_decode_q8(const DecodeArgs &a, const CUtensorMap &mk, const CUtensorMap &mv,
                             dim3 grid, cudaStream_t st) {
    constexpr int STAGE = 2 * CT * 128;
    using L = DecodeSmem<NW, NS, STAGE, kHeadsBf16, 128>;
    const size_t smem = 1024 + L::kTable + ((size_t)a.P / a.bs + 2) * 4;
    auto k = decode_split_q8<NW, NS, CT, INT8>;
    if (set_smem(k, smem) != cudaSuccess) return PA_ERR_CUDA;
    k<<<grid, NW * 32, smem, st>>>(a, mk, mv);
    return launch_status();
}

// The LSE merge behind a split launch, as a programmatic dependent launch
// (its CTAs may start while the split grid's last CTAs run; they wait for
// that grid's completion before reading partials).
template <int D, typename OutT, bool SHARED = false>
pa_status launch_reduce(const DecodeArgs &a, cudaStream_t st) {
    const long long heads = (long long)a.num_seqs * a.H_q;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = st;
    cfg.dynamicSmemBytes = 0;
    if (a.S_max <= kWarpMergeMax) {
        cfg.gridDim = dim3((unsigned)((heads + 7) / 8));
        cfg.blockDim = dim3(256);
        if (cudaLaunchKernelEx(&cfg, decode_reduce_warp<D, OutT, SHARED>, a) != cudaSuccess)
            return PA_ERR_CUDA;
    } else {
        cfg.gridDim = dim3((unsigned)heads);
        cfg.blockDim = dim3(512);
        if (cudaLaunchKernelEx(&cfg, decode_reduce<D, OutT, SHARED>, a) != cudaSuccess)
            return PA_ERR_CUDA;
    }
    return launch_status();
}

// ------------------------------------------------------ shared-prefix decode
// Partition sizes and slot counts of the shared-prefix decode.
struct SharedPlan {
    int Pp, Pt;  // tokens per prefix / tail partition
    int Sp, St;  // partial slots of the prefix / tail passes
    int MT, row_tiles;
};

int round16(int n) { return ((n > 0 ? n : 1) + kChunk - 1) / kChunk * kChunk; }

// false if partition_size cannot be met. Automatic: a tail in one partition
// up to 2048 tokens, else 1024-token partitions; prefix partitions of 512
// tokens, 256 when that leaves fewer than two CTAs per SM of a B200.
bool shared_plan(int max_ctx, int max_prefix, int max_group, int group, int H_kv, int num_groups,
                 int partition_size, SharedPlan &p) {
    const int rows = max_group * group;
    p.MT = rows <= 16 ? 1 : rows <= 32 ? 2 : 4;
    p.row_tiles = (rows + p.MT * 16 - 1) / (p.MT * 16);
    if (partition_size > 0) {
        if (partition_size % kChunk != 0 || partition_size > kMaxPartition) return false;
        p.Pp = p.Pt = partition_size;
    } else if (partition_size < 0) {
        p.Pt = round16(max_ctx);
        p.Pp = round16(max_prefix);
        if (p.Pt > kMaxPartition || p.Pp > kMaxPartition) return false;
    } else {
        p.Pt = max_ctx <= 2048 ? round16(max_ctx) : 1024;
        p.Pp = 512;
        const long long ctas = (long long)((max_prefix + 511) / 512) * H_kv * p.row_tiles * num_groups;
        if (ctas < 2 * 148) p.Pp = 256;
        if (max_prefix < p.Pp) p.Pp = round16(max_prefix);
    }
    p.Sp = (max_prefix + p.Pp - 1) / p.Pp;
    p.St = (max_ctx + p.Pt - 1) / p.Pt;
    if (p.St < 1) p.St = 1;
    return true;
}

size_t shared_workspace_bytes(int B, int H_q, int D, const SharedPlan &p) {
    const size_t S = (size_t)p.Sp + p.St;
    const size_t o = (size_t)B * H_q * S * D * sizeof(float);
    const size_t l = (size_t)B * H_q * S * sizeof(float);
    return (o + 255) / 256 * 256 + (l + 255) / 256 * 256;
}

template <int D, int MT>
pa_status launch_prefix(const DecodeArgs &a, const CUtensorMap &mk, const CUtensorMap &mv,
                        dim3 grid, cudaStream_t st) {
    using L = PrefixSmem<D, MT>;
    const size_t smem = 1024 + L::kTable + ((size_t)a.P_prefix / a.bs + 2) * 4;
    auto k = decode_prefix_bf16<D, MT>;
    if (set_smem(k, smem) != cudaSuccess) return PA_ERR_CUDA;
    k<<<grid, kPrefixWarps * 32, smem, st>>>(a, mk, mv);
    return launch_status();
}

// The tail pass, as a programmatic dependent of the prefix pass when there
// is one (it reads nothing the prefix pass writes; it only finishes after it).
template <int D>
pa_status launch_tail(const DecodeArgs &a, const CUtensorMap &mk, const CUtensorMap &mv, dim3 grid,
                      bool dependent, cudaStream_t st) {
    constexpr int STAGE = 2 * kChunk * D * 2;
    using L = DecodeSmem<kDecodeWarps, kDecodeStages, STAGE, kHeadsBf16, D>;
    const size_t smem = 1024 + L::kTable + ((size_t)a.P / a.bs + 2) * 4;
    auto k = decode_split_bf16<D, kDecodeWarps, kDecodeStages, true>;
    if (set_smem(k, smem) != cudaSuccess) return PA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    cfg.stream = st;
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kDecodeWarps * 32);
    cfg.dynamicSmemBytes = smem;
    if (cudaLaunchKernelEx(&cfg, k, a, mk, mv) != cudaSuccess) return PA_ERR_CUDA;
    return launch_status();
}

}  // namespace

// =================================================================== C ABI
extern "C" {

int pa_version(void) { return (1 << 16) | 0; }

const char *pa_status_string(pa_status s) {
    switch (s) {
        case PA_OK: return "ok";
        case PA_ERR_INVALID_ARG: return "invalid argument";
        case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case PA_ERR_WORKSPACE: return "workspace missing or too small";
        case PA_ERR_BAD_TABLE: return "block id, slot or length out of range";
        case PA_ERR_TIMEOUT: return "bounded device wait ran out";
        case PA_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                               const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                               cudaStream_t stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0 || head_dim <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (!head_dim_ok(head_dim) || !block_size_ok(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(slot_mapping, 8))
        return PA_ERR_INVALID_ARG;
    const int elem = dtype == PA_BF16 ? 2 : 4;
    ReshapeArgs a;
    a.key = static_cast<const uint4 *>(key);
    a.value = static_cast<const uint4 *>(value);
    a.k_cache = static_cast<uint4 *>(k_cache);
    a.v_cache = static_cast<uint4 *>(v_cache);
    a.slot_mapping = slot_mapping;
    const int vecs_per_row = head_dim * elem / 16;  // 8, 16 or 32: a power of two
    if ((long long)num_kv_heads * vecs_per_row > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
    a.num_tokens = num_tokens;
    a.vecs_per_token = num_kv_heads * vecs_per_row;
    a.row_shift = __builtin_ctz((unsigned)vecs_per_row);
    a.bs_shift = __builtin_ctz((unsigned)block_size);
    a.num_kv_heads = num_kv_heads;
    a.num_slots = (long long)num_blocks * block_size;
    const long long groups = (num_tokens + kScatterTokens - 1) / kScatterTokens;
    const dim3 grid((unsigned)((a.vecs_per_token + kScatterThreads - 1) / kScatterThreads),
                    (unsigned)(groups < 65535 ? groups : 65535));
    reshape_and_cache_kernel<<<grid, kScatterThreads, 0, stream>>>(a);
    return launch_status();
}

int pa_decode_partition_tokens(int max_context_len, int partition_size) {
    return partition_tokens(max_context_len, partition_size);
}

size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                int partition_size) {
    const int P = partition_tokens(max_context_len, partition_size);
    if (P <= 0 || num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0) return 0;
    return workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len, P);
}

}  // extern "C"

static pa_status decode_impl(void *out, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, const int32_t *context_lens,
                             int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                             int block_size, int num_blocks, int max_blocks_per_seq,
                             int max_context_len, float scale, int partition_size,
                             void *workspace, size_t workspace_bytes_given, pa_dtype dtype,
                             int window, cudaStream_t stream) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0 || !head_dim_ok(head_dim) || !block_size_ok(block_size))
        return PA_ERR_UNSUPPORTED;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size)
        return PA_ERR_INVALID_ARG;
    const int P = partition_tokens(max_context_len, partition_size);
    if (P <= 0) return partition_size > 0 ? PA_ERR_INVALID_ARG : PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4))
        return PA_ERR_INVALID_ARG;
    const size_t need = workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len, P);
    if (need > 0 && (!workspace || workspace_bytes_given < need || !aligned(workspace, 256)))
        return PA_ERR_WORKSPACE;
    const int group = num_q_heads / num_kv_heads;
    const int ht = dtype == PA_BF16 ? kHeadsBf16 : kHeadsF32;
    const int n_htiles = (group + ht - 1) / ht;
    const long long S = (max_context_len + P - 1) / P;
    const long long gy = (long long)num_kv_heads * n_htiles;
    if (gy > 65535 || num_seqs > 65535 || S > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;

    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    const long long S1 = S > 0 ? S : 1;
    a.part_o = need ? static_cast<float *>(workspace) : nullptr;
    a.part_lse = need ? reinterpret_cast<float *>(
                            static_cast<char *>(workspace) +
                            ((size_t)num_seqs * num_q_heads * S1 * head_dim * 4 + 255) / 256 * 256)
                      : nullptr;
    a.num_seqs = num_seqs;
    a.H_q = num_q_heads;
    a.H_kv = num_kv_heads;
    a.group = group;
    a.bs = block_size;
    a.bs_shift = __builtin_ctz((unsigned)block_size);
    a.NB = num_blocks;
    a.MB = max_blocks_per_seq;
    a.max_ctx = max_context_len;
    a.P = P;
    a.S_max = (int)S1;
    a.n_htiles = n_htiles;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.timeout_ns = kWaitTimeoutNs;
    a.window = window;
    a.k_scale = a.v_scale = nullptr;

    const dim3 grid((unsigned)S1, (unsigned)gy, (unsigned)num_seqs);
    pa_status st;
    if (dtype == PA_BF16) {
        CUtensorMap mk, mv;
        if (!encode_cache_map(&mk, k_cache, num_blocks, num_kv_heads, block_size, head_dim,
                              kChunk) ||
            !encode_cache_map(&mv, v_cache, num_blocks, num_kv_heads, block_size, head_dim, kChunk))
            return PA_ERR_CUDA;
        st = head_dim == 128
                 ? launch_decode_bf16<128, kDecodeWarps, kDecodeStages>(a, mk, mv, grid, stream)
                 : launch_decode_bf16<64, kDecodeWarps, kDecodeStages>(a, mk, mv, grid, stream);
        if (st != PA_OK) return st;
        if (S1 > 1) {
            st = head_dim == 128 ? launch_reduce<128, __nv_bfloat16>(a, stream)
                                 : launch_reduce<64, __nv_bfloat16>(a, stream);
        }
    } else {
        st = head_dim == 128 ? launch_decode_f32<128, kDecodeWarps, kDecodeStages>(a, grid, stream)
                             : launch_decode_f32<64, kDecodeWarps, kDecodeStages>(a, grid, stream);
        if (st != PA_OK) return st;
        if (S1 > 1) {
            st = head_dim == 128 ? launch_reduce<128, float>(a, stream)
                                 : launch_reduce<64, float>(a, stream);
        }
    }
    return st;
}

extern "C" {

pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                    int partition_size, void *workspace, size_t workspace_bytes_given,
                    pa_dtype dtype, cudaStream_t stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       max_blocks_per_seq, max_context_len, scale, partition_size, workspace,
                       workspace_bytes_given, dtype, 0, stream);
}

pa_status pa_decode_sliding_window(void *out, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *block_tables,
                                   const int32_t *context_lens, int num_seqs, int num_q_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int num_blocks, int max_blocks_per_seq, int max_context_len,
                                   float scale, int sliding_window, int partition_size,
                                   void *workspace, size_t workspace_bytes_given, pa_dtype dtype,
                                   cudaStream_t stream) {
    if (sliding_window <= 0) return PA_ERR_INVALID_ARG;
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       max_blocks_per_seq, max_context_len, scale, partition_size, workspace,
                       workspace_bytes_given, dtype, sliding_window, stream);
}

static pa_status reshape_q8_impl(const void *key, const void *value, void *k_cache,
                                 void *v_cache, const int64_t *slot_mapping, int num_tokens,
                                 int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                 const float *k_scale, const float *v_scale, pa_dtype dtype,
                                 bool int8, cudaStream_t stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0 || head_dim <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (!head_dim_ok(head_dim) || !block_size_ok(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping || !k_scale || !v_scale)
        return PA_ERR_INVALID_ARG;
    if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(slot_mapping, 8) || !aligned(k_scale, 4) ||
        !aligned(v_scale, 4))
        return PA_ERR_INVALID_ARG;
    ReshapeFp8Args a;
    a.key = key;
    a.value = value;
    a.k_cache = static_cast<uint4 *>(k_cache);
    a.v_cache = static_cast<uint4 *>(v_cache);
    a.slot_mapping = slot_mapping;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    const int vecs_per_row = head_dim / 16;  // 4 or 8: a power of two
    if ((long long)num_kv_heads * vecs_per_row > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
    a.num_tokens = num_tokens;
    a.vecs_per_token = num_kv_heads * vecs_per_row;
    a.row_shift = __builtin_ctz((unsigned)vecs_per_row);
    a.bs_shift = __builtin_ctz((unsigned)block_size);
    a.num_kv_heads = num_kv_heads;
    a.num_slots = (long long)num_blocks * block_size;
    a.bf16_in = dtype == PA_BF16;
    const dim3 grid((unsigned)((a.vecs_per_token + kScatterThreads - 1) / kScatterThreads),
                    (unsigned)(num_tokens < 65535 ? num_tokens : 65535));
    if (int8)
        reshape_and_cache_int8_kernel<<<grid, kScatterThreads, 0, stream>>>(a);
    else
        reshape_and_cache_e4m3_kernel<<<grid, kScatterThreads, 0, stream>>>(a);
    return launch_status();
}

pa_status pa_reshape_and_cache_fp8(const void *key, const void *value, void *k_cache,
                                   void *v_cache, const int64_t *slot_mapping, int num_tokens,
                                   int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                   const float *k_scale, const float *v_scale, pa_dtype dtype,
                                   cudaStream_t stream) {
    return reshape_q8_impl(key, value, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads,
                           head_dim, block_size, num_blocks, k_scale, v_scale, dtype, false,
                           stream);
}

pa_status pa_reshape_and_cache_int8(const void *key, const void *value, void *k_cache,
                                    void *v_cache, const int64_t *slot_mapping, int num_tokens,
                                    int num_kv_heads, int head_dim, int block_size,
                                    int num_blocks, const float *k_scale, const float *v_scale,
                                    pa_dtype dtype, cudaStream_t stream) {
    return reshape_q8_impl(key, value, k_cache, v_cache, slot_mapping, num_tokens, num_kv_heads,
                           head_dim, block_size, num_blocks, k_scale, v_scale, dtype, true,
                           stream);
}

static pa_status decode_q8_impl(void *out, const void *q, const void *k_cache,
                                const void *v_cache, const float *k_scale, const float *v_scale,
                                const int32_t *block_tables, const int32_t *context_lens,
                                int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                int block_size, int num_blocks, int max_blocks_per_seq,
                                int max_context_len, float scale, int partition_size,
                                void *workspace, size_t workspace_bytes_given, bool int8,
                                cudaStream_t stream) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
        return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0 || head_dim != 128 || !block_size_ok(block_size))
        return PA_ERR_UNSUPPORTED;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size)
        return PA_ERR_INVALID_ARG;
    const int P = partition_tokens(max_context_len, partition_size);
    if (P <= 0) return partition_size > 0 ? PA_ERR_INVALID_ARG : PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !k_scale ||
        !v_scale)
        return PA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(k_scale, 4) ||
        !aligned(v_scale, 4))
        return PA_ERR_INVALID_ARG;
    const size_t need = workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len, P);
    if (need > 0 && (!workspace || workspace_bytes_given < need || !aligned(workspace, 256)))
        return PA_ERR_WORKSPACE;
    const int group = num_q_heads / num_kv_heads;
    const int n_htiles = (group + kHeadsBf16 - 1) / kHeadsBf16;
    const long long S = (max_context_len + P - 1) / P;
    const long long gy = (long long)num_kv_heads * n_htiles;
    if (gy > 65535 || num_seqs > 65535 || S > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    const long long S1 = S > 0 ? S : 1;
    a.part_o = need ? static_cast<float *>(workspace) : nullptr;
    a.part_lse = need ? reinterpret_cast<float *>(
                            static_cast<char *>(workspace) +
                            ((size_t)num_seqs * num_q_heads * S1 * head_dim * 4 + 255) / 256 * 256)
                      : nullptr;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.window = 0;
    a.num_seqs = num_seqs;
    a.H_q = num_q_heads;
    a.H_kv = num_kv_heads;
    a.group = group;
    a.bs = block_size;
    a.bs_shift = __builtin_ctz((unsigned)block_size);
    a.NB = num_blocks;
    a.MB = max_blocks_per_seq;
    a.max_ctx = max_context_len;
    a.P = P;
    a.S_max = (int)S1;
    a.n_htiles = n_htiles;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.timeout_ns = kWaitTimeoutNs;
    CUtensorMap mk, mv;
    if (!encode_cache_map_u8(&mk, k_cache, num_blocks, num_kv_heads, block_size) ||
        !encode_cache_map_u8(&mv, v_cache, num_blocks, num_kv_heads, block_size))
        return PA_ERR_CUDA;
    const dim3 grid((unsigned)S1, (unsigned)gy, (unsigned)num_seqs);
    const pa_status st =
        int8 ? launch_decode_q8<kDecodeWarps, kDecodeStages, kQ8Tokens, true>(a, mk, mv, grid, stream)
             : launch_decode_q8<kDecodeWarps, kDecodeStages, kQ8Tokens, false>(a, mk, mv, grid, stream);
    if (st != PA_OK) return st;
    return S1 > 1 ? launch_reduce<128, __nv_bfloat16>(a, stream) : PA_OK;
}

pa_status pa_decode_fp8(void *out, const void *q, const void *k_cache, const void *v_cache,
                        const float *k_scale, const float *v_scale, const int32_t *block_tables,
                        const int32_t *context_lens, int num_seqs, int num_q_heads,
                        int num_kv_heads, int head_dim, int block_size, int num_blocks,
                        int max_blocks_per_seq, int max_context_len, float scale,
                        int partition_size, void *workspace, size_t workspace_bytes_given,
                        cudaStream_t stream) {
    return decode_q8_impl(out, q, k_cache, v_cache, k_scale, v_scale, block_tables,
                          context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                          block_size, num_blocks, max_blocks_per_seq, max_context_len, scale,
                          partition_size, workspace, workspace_bytes_given, false, stream);
}

pa_status pa_decode_int8(void *out, const void *q, const void *k_cache, const void *v_cache,
                         const float *k_scale, const float *v_scale, const int32_t *block_tables,
                         const int32_t *context_lens, int num_seqs, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks,
                         int max_blocks_per_seq, int max_context_len, float scale,
                         int partition_size, void *workspace, size_t workspace_bytes_given,
                         cudaStream_t stream) {
    return decode_q8_impl(out, q, k_cache, v_cache, k_scale, v_scale, block_tables,
                          context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                          block_size, num_blocks, max_blocks_per_seq, max_context_len, scale,
                          partition_size, workspace, workspace_bytes_given, true, stream);
}

static pa_status prefill_impl(void *out, const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *block_tables, const int32_t *context_lens,
                              const int32_t *query_start_loc, int num_chunks,
                              int num_query_tokens, int max_query_len, int num_q_heads,
                              int num_kv_heads, int head_dim, int block_size, int num_blocks,
                              int max_blocks_per_seq, float scale, int window, pa_dtype dtype,
                              cudaStream_t stream) {
    if (num_chunks < 0 || num_query_tokens < 0 || max_query_len < 0 || num_q_heads <= 0 ||
        num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (dtype != PA_BF16 || num_q_heads % num_kv_heads != 0 || !head_dim_ok(head_dim) ||
        !block_size_ok(block_size))
        return PA_ERR_UNSUPPORTED;
    if (num_chunks == 0 || max_query_len == 0 || num_query_tokens == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start_loc)
        return PA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(query_start_loc, 4))
        return PA_ERR_INVALID_ARG;
    // a CTA's two query tiles: the same 128 rows of two query heads of one KV
    // head when the group size is even, else 256 consecutive rows of one head
    const bool pair_heads = (num_q_heads / num_kv_heads) % 2 == 0;
    const int cta_rows = pair_heads ? kPfRows : kPfRows * kPfQTiles;
    const long long qtiles = (max_query_len + cta_rows - 1) / cta_rows;
    if (qtiles > 65535 || num_chunks > 65535) return PA_ERR_UNSUPPORTED;

    EncodeTiledFn fn = encode_fn();
    if (!fn) return PA_ERR_CUDA;
    CUtensorMap mq, mk, mv;
    {
        cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads,
                              (cuuint64_t)num_query_tokens};
        cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2,
                                 (cuuint64_t)num_q_heads * head_dim * 2};
        cuuint32_t box[3] = {64, 1, kPfRows};
        cuuint32_t estr[3] = {1, 1, 1};
        if (fn(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return PA_ERR_CUDA;
    }
    if (!encode_cache_map(&mk, k_cache, num_blocks, num_kv_heads, block_size, head_dim, 16) ||
        !encode_cache_map(&mv, v_cache, num_blocks, num_kv_heads, block_size, head_dim, 16))
        return PA_ERR_CUDA;

    PrefillArgs a;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.qsl = query_start_loc;
    a.n_chunks = num_chunks;
    a.total_q = num_query_tokens;
    a.H_q = num_q_heads;
    a.H_kv = num_kv_heads;
    a.group = num_q_heads / num_kv_heads;
    a.bs = block_size;
    a.NB = num_blocks;
    a.MB = max_blocks_per_seq;
    a.window = window;
    a.pair_heads = pair_heads ? 1 : 0;
    a.bs_shift = __builtin_ctz((unsigned)block_size);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.timeout_ns = kWaitTimeoutNs;
    // persistent: one CTA per SM (its 512 TMEM columns) deals the items out
    a.gx = pair_heads ? num_q_heads / 2 : num_q_heads;
    a.gy = (int)qtiles;
    const long long n_items = (long long)a.gx * a.gy * num_chunks;
    if (n_items > (1LL << 30)) return PA_ERR_UNSUPPORTED;
    a.n_items = (int)n_items;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return PA_ERR_CUDA;
    const dim3 grid((unsigned)std::min<long long>(n_items, sms));
    if (head_dim == 64)
        return window > 0 ? launch_prefill_tc<64, true>(a, mq, mk, mv, grid, stream)
                          : launch_prefill_tc<64, false>(a, mq, mk, mv, grid, stream);
    return window > 0 ? launch_prefill_tc<128, true>(a, mq, mk, mv, grid, stream)
                      : launch_prefill_tc<128, false>(a, mq, mk, mv, grid, stream);
}

pa_status pa_prefill_chunk(void *out, const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *block_tables, const int32_t *context_lens,
                           const int32_t *query_start_loc, int num_chunks, int num_query_tokens,
                           int max_query_len, int num_q_heads, int num_kv_heads, int head_dim,
                           int block_size, int num_blocks, int max_blocks_per_seq, float scale,
                           pa_dtype dtype, cudaStream_t stream) {
    return prefill_impl(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                        num_chunks, num_query_tokens, max_query_len, num_q_heads, num_kv_heads,
                        head_dim, block_size, num_blocks, max_blocks_per_seq, scale, 0, dtype,
                        stream);
}

pa_status pa_prefill_chunk_sliding_window(void *out, const void *q, const void *k_cache,
                                          const void *v_cache, const int32_t *block_tables,
                                          const int32_t *context_lens,
                                          const int32_t *query_start_loc, int num_chunks,
                                          int num_query_tokens, int max_query_len,
                                          int num_q_heads, int num_kv_heads, int head_dim,
                                          int block_size, int num_blocks,
                                          int max_blocks_per_seq, float scale,
                                          int sliding_window, pa_dtype dtype,
                                          cudaStream_t stream) {
    if (sliding_window <= 0) return PA_ERR_INVALID_ARG;
    return prefill_impl(out, q, k_cache, v_cache, block_tables, context_lens, query_start_loc,
                        num_chunks, num_query_tokens, max_query_len, num_q_heads, num_kv_heads,
                        head_dim, block_size, num_blocks, max_blocks_per_seq, scale,
                        sliding_window, dtype, stream);
}

}  // extern "C"

namespace {

pa_status launch_copy_blocks(const void *src_k, const void *src_v, long long src_blocks,
                             void *dst_k, void *dst_v, long long dst_blocks,
                             const int64_t *mapping, int num_pairs, int num_kv_heads, int head_dim,
                             int block_size, pa_dtype dtype, cudaStream_t stream) {
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        src_blocks <= 0 || dst_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (!head_dim_ok(head_dim) || !block_size_ok(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!src_k || !src_v || !dst_k || !dst_v || !mapping) return PA_ERR_INVALID_ARG;
    if (!aligned(src_k, 16) || !aligned(src_v, 16) || !aligned(dst_k, 16) ||
        !aligned(dst_v, 16) || !aligned(mapping, 8))
        return PA_ERR_INVALID_ARG;
    const long long bytes = (long long)num_kv_heads * block_size * head_dim *
                            (dtype == PA_BF16 ? 2 : 4);
    if (bytes / 16 > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
    CopyArgs a;
    a.src_k = static_cast<const uint4 *>(src_k);
    a.src_v = static_cast<const uint4 *>(src_v);
    a.dst_k = static_cast<uint4 *>(dst_k);
    a.dst_v = static_cast<uint4 *>(dst_v);
    a.mapping = mapping;
    a.src_blocks = src_blocks;
    a.dst_blocks = dst_blocks;
    a.vecs_per_block = (int)(bytes / 16);
    copy_blocks_kernel<<<num_pairs, 256, 0, stream>>>(a);
    return launch_status();
}

}  // namespace

extern "C" {

pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping,
                         int num_pairs, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype dtype, cudaStream_t stream) {
    return launch_copy_blocks(k_cache, v_cache, num_blocks, k_cache, v_cache, num_blocks,
                              block_mapping, num_pairs, num_kv_heads, head_dim, block_size, dtype,
                              stream);
}

pa_status pa_swap_blocks(const void *src_k, const void *src_v, int src_blocks, void *dst_k,
                         void *dst_v, int dst_blocks, const int64_t *block_mapping, int num_pairs,
                         int num_kv_heads, int head_dim, int block_size, pa_dtype dtype,
                         cudaStream_t stream) {
    return launch_copy_blocks(src_k, src_v, src_blocks, dst_k, dst_v, dst_blocks, block_mapping,
                              num_pairs, num_kv_heads, head_dim, block_size, dtype, stream);
}

}  // extern "C"

extern "C" {

size_t pa_decode_shared_prefix_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                              int head_dim, int num_groups, int max_group_size,
                                              int max_prefix_len, int max_context_len,
                                              int partition_size) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        num_q_heads % num_kv_heads != 0 || num_groups < 0 || max_group_size <= 0 ||
        max_prefix_len < 0 || max_context_len < 0)
        return 0;
    SharedPlan p;
    if (!shared_plan(max_context_len, max_prefix_len, max_group_size,
                     num_q_heads / num_kv_heads, num_kv_heads, num_groups, partition_size, p))
        return 0;
    return shared_workspace_bytes(num_seqs, num_q_heads, head_dim, p);
}

pa_status pa_decode_shared_prefix(void *out, const void *q, const void *k_cache,
                                  const void *v_cache, const int32_t *block_tables,
                                  const int32_t *context_lens, const int32_t *group_start,
                                  const int32_t *prefix_lens, int num_groups, int max_group_size,
                                  int max_prefix_len, int num_seqs, int num_q_heads,
                                  int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                  int max_blocks_per_seq, int max_context_len, float scale,
                                  int partition_size, void *workspace, size_t workspace_bytes_given,
                                  pa_dtype dtype, cudaStream_t stream) {
    if (num_seqs < 0 || num_groups < 0 || max_group_size <= 0 || max_prefix_len < 0 ||
        num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F32 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (dtype != PA_BF16 || num_q_heads % num_kv_heads != 0 || !head_dim_ok(head_dim) ||
        !block_size_ok(block_size))
        return PA_ERR_UNSUPPORTED;
    if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size ||
        max_prefix_len > max_context_len)
        return PA_ERR_INVALID_ARG;
    if ((num_seqs == 0) != (num_groups == 0)) return PA_ERR_INVALID_ARG;
    const int group = num_q_heads / num_kv_heads;
    SharedPlan plan;
    if (!shared_plan(max_context_len, max_prefix_len, max_group_size, group, num_kv_heads,
                     num_groups, partition_size, plan))
        return partition_size > 0 ? PA_ERR_INVALID_ARG : PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !group_start ||
        !prefix_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(group_start, 4) ||
        !aligned(prefix_lens, 4))
        return PA_ERR_INVALID_ARG;
    const size_t need = shared_workspace_bytes(num_seqs, num_q_heads, head_dim, plan);
    if (!workspace || workspace_bytes_given < need || !aligned(workspace, 256))
        return PA_ERR_WORKSPACE;
    const int n_htiles = (group + kHeadsBf16 - 1) / kHeadsBf16;
    const long long S = (long long)plan.Sp + plan.St;
    const long long tail_x = (long long)max_group_size * plan.St;
    if (num_groups > 65535 || (long long)num_kv_heads * plan.row_tiles > 65535 ||
        (long long)num_kv_heads * n_htiles > 65535 || tail_x > 0x7fffffffLL || S > 0x7fffffffLL)
        return PA_ERR_UNSUPPORTED;

    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.part_o = static_cast<float *>(workspace);
    a.part_lse = reinterpret_cast<float *>(
        static_cast<char *>(workspace) +
        ((size_t)num_seqs * num_q_heads * S * head_dim * 4 + 255) / 256 * 256);
    a.num_seqs = num_seqs;
    a.H_q = num_q_heads;
    a.H_kv = num_kv_heads;
    a.group = group;
    a.bs = block_size;
    a.bs_shift = __builtin_ctz((unsigned)block_size);
    a.NB = num_blocks;
    a.MB = max_blocks_per_seq;
    a.max_ctx = max_context_len;
    a.P = plan.Pt;
    a.S_max = (int)S;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.timeout_ns = kWaitTimeoutNs;
    a.window = 0;
    a.group_start = group_start;
    a.prefix_lens = prefix_lens;
    a.num_groups = num_groups;
    a.max_group = max_group_size;
    a.max_prefix = max_prefix_len;
    a.P_prefix = plan.Pp;
    a.S_prefix = plan.Sp;

    CUtensorMap mk, mv;
    if (!encode_cache_map(&mk, k_cache, num_blocks, num_kv_heads, block_size, head_dim, kChunk) ||
        !encode_cache_map(&mv, v_cache, num_blocks, num_kv_heads, block_size, head_dim, kChunk))
        return PA_ERR_CUDA;
    pa_status st = PA_OK;
    if (plan.Sp > 0) {
        DecodeArgs ap = a;
        ap.n_htiles = plan.row_tiles;  // row tiles of (member, head) rows
        const dim3 grid((unsigned)plan.Sp, (unsigned)(num_kv_heads * plan.row_tiles),
                        (unsigned)num_groups);
        if (head_dim == 128)
            st = plan.MT == 1   ? launch_prefix<128, 1>(ap, mk, mv, grid, stream)
                 : plan.MT == 2 ? launch_prefix<128, 2>(ap, mk, mv, grid, stream)
                                : launch_prefix<128, 4>(ap, mk, mv, grid, stream);
        else
            st = plan.MT == 1   ? launch_prefix<64, 1>(ap, mk, mv, grid, stream)
                 : plan.MT == 2 ? launch_prefix<64, 2>(ap, mk, mv, grid, stream)
                                : launch_prefix<64, 4>(ap, mk, mv, grid, stream);
        if (st != PA_OK) return st;
    }
    a.n_htiles = n_htiles;
    const dim3 tgrid((unsigned)tail_x, (unsigned)(num_kv_heads * n_htiles), (unsigned)num_groups);
    st = head_dim == 128 ? launch_tail<128>(a, mk, mv, tgrid, plan.Sp > 0, stream)
                         : launch_tail<64>(a, mk, mv, tgrid, plan.Sp > 0, stream);
    if (st != PA_OK) return st;
    return head_dim == 128 ? launch_reduce<128, __nv_bfloat16, true>(a, stream)
                           : launch_reduce<64, __nv_bfloat16, true>(a, stream);
}

}  // extern "C"

// ------------------------------------------------------- service kernels
namespace {

__global__ void check_tables_kernel(const int32_t *tables, const int32_t *lens, int MB, int bs,
                                    int NB, int32_t *bad) {
    __shared__ int row_bad;
    const int r = blockIdx.x;
    if (threadIdx.x == 0) row_bad = 0;
    __syncthreads();
    const int len = lens[r];
    if (len < 0 || (long long)len > (long long)MB * bs) {
        if (threadIdx.x == 0) row_bad = 1;
    } else {
        const int n = (len + bs - 1) / bs;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const int id = tables[(size_t)r * MB + i];
            if (id < 0 || id >= NB) row_bad = 1;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && row_bad) atomicAdd(bad, 1);
}

__global__ void selftest_wait_kernel(unsigned long long timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // nothing arrives on this barrier: the bounded wait must run out
    if (!mbar_wait(b, 0, timeout_ns) && threadIdx.x == 0) flag_error(PA_ERR_TIMEOUT);
}

}  // namespace

extern "C" {

pa_status pa_check_tables(const int32_t *block_tables, const int32_t *context_lens, int rows,
                          int max_blocks_per_seq, int block_size, int num_blocks,
                          int32_t *d_scratch, int *bad_rows, cudaStream_t stream) {
    if (rows < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || num_blocks <= 0)
        return PA_ERR_INVALID_ARG;
    if (bad_rows) *bad_rows = 0;
    if (rows == 0) return PA_OK;
    if (!block_tables || !context_lens || !d_scratch) return PA_ERR_INVALID_ARG;
    if (cudaMemsetAsync(d_scratch, 0, sizeof(int32_t), stream) != cudaSuccess) return PA_ERR_CUDA;
    check_tables_kernel<<<rows, 128, 0, stream>>>(block_tables, context_lens, max_blocks_per_seq,
                                                  block_size, num_blocks, d_scratch);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, d_scratch, sizeof(int32_t), cudaMemcpyDeviceToHost, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return PA_ERR_CUDA;
    if (bad_rows) *bad_rows = h;
    return h ? PA_ERR_BAD_TABLE : PA_OK;
}

pa_status pa_device_error(int *status, int clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, pa::g_pa_error, sizeof(int)) != cudaSuccess) return PA_ERR_CUDA;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(pa::g_pa_error, &zero, sizeof(int)) != cudaSuccess)
            return PA_ERR_CUDA;
    }
    if (status) *status = v;
    return PA_OK;
}

pa_status pa_selftest_bounded_wait(long long timeout_ns, cudaStream_t stream) {
    if (timeout_ns <= 0 || timeout_ns > 10000000000LL) return PA_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, stream>>>((unsigned long long)timeout_ns);
    return launch_status();
}

}  // extern "C"

// ------------------------------------------------- decode without allocation
// pa_decode_static_workspace: pa_decode for callers that cannot allocate the
// workspace themselves -- for example a plugin that is handed only its input
// and output buffers by a host engine, or a caller on a latency-critical path
// where cudaMalloc (which may synchronise the whole device) is not allowed.
// Its scratch is a file-scope device array compiled into the library, so
// every GPU that loads the library holds these 16 MiB until the process
// exits. In host code the array's name is only a host-side stand-in; the
// device address is looked up with cudaGetSymbolAddress, with the device
// current, the first time the entry point runs in a CUDA context, and cached
// under that context's unique id: after cudaDeviceReset the next call runs in
// a new context and looks the address up again.
namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(16) << 20;  // 16 MiB per device

__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mutex;
void *g_static_ws_ptr[kMaxDevices] = {};
unsigned long long g_static_ws_ctx[kMaxDevices] = {};  // context id of each cached address

// Unique id (cuCtxGetId, never reused within the process) of the calling
// thread's current context, 0 when there is none or the lookup fails. The
// driver entry points are fetched through the runtime so that the library
// does not link libcuda directly.
unsigned long long current_context_id() {
    typedef CUresult (*GetCurrentFn)(CUcontext *);
    typedef CUresult (*GetIdFn)(CUcontext, unsigned long long *);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr, *q = nullptr;
        cudaDriverEntryPointQueryResult r1, r2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r1) ==
                cudaSuccess &&
            r1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &q, cudaEnableDefault, &r2) == cudaSuccess &&
            r2 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrentFn>(p);
            get_id = reinterpret_cast<GetIdFn>(q);
        }
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_static_workspace on the current device, looked up once
// per CUDA context; nullptr if the lookup fails.
void *static_workspace_address() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_static_ws_mutex);
    const unsigned long long ctx = current_context_id();
    if (!g_static_ws_ptr[dev] || ctx == 0 || ctx != g_static_ws_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess) return nullptr;
        g_static_ws_ptr[dev] = p;
        // the lookup makes the device's primary context current if no
        // context was: key the address on the context it was found in
        g_static_ws_ctx[dev] = current_context_id();
    }
    return g_static_ws_ptr[dev];
}

}  // namespace

extern "C" pa_status pa_decode_static_workspace(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, const int32_t *context_lens, int num_seqs, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
    int max_context_len, float scale, int partition_size, pa_dtype dtype, cudaStream_t stream) {
    // refuse, before touching the device, any request whose partials would
    // not fit in the fixed array
    const int P = partition_tokens(max_context_len, partition_size);
    if (P > 0 && num_seqs >= 0 && num_q_heads > 0 && head_dim > 0 &&
        workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len, P) >
            kStaticWorkspaceBytes)
        return PA_ERR_WORKSPACE;
    void *ws = static_workspace_address();
    if (!ws) return PA_ERR_CUDA;
    // the decode kernels write every partial they later read within the same
    // call, so the array needs no clearing between calls
    return pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_q_heads,
                     num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                     max_context_len, scale, partition_size, ws, kStaticWorkspaceBytes, dtype,
                     stream);
}
