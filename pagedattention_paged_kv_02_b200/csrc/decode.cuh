// decode.cuh -- paged decode attention: the split-KV kernel (the merge of
// its partials is in decode_merge.cuh).
//
// What is computed (page "字节跳动 AI Infra (2)", question "KV Cache原理与优化"):
// for each sequence b and query head h, softmax(scale * q . K^T) V over the
// sequence's context_lens[b] cached tokens. K/V are reached through the
// block table (question "vLLM与PagedAttention的原理": logical block i of the
// sequence lives in physical block block_tables[b][i]); query heads share K/V
// heads in groups (page "LLM推理优化", section 1.3). Long contexts are split
// along the KV length into partitions whose partial results are merged by
// log-sum-exp (page "字节跳动 AI Infra (2)", FlashDecoding row), each
// partition using a running max / running sum softmax (page "LLM推理优化",
// section 2.1, online softmax).
//
// Work decomposition: one CTA per (KV partition, KV head [x query-head tile],
// sequence). Every K/V byte fetched serves all query heads of the GQA group.
// Inside the CTA each warp owns every NW-th 16-token chunk of the partition
// and runs its own NS-deep pipeline: lane 0 issues TMA copies of the chunk's
// K and V rows (contiguous inside a page) into a stage and the warp waits on
// that stage's mbarrier, so up to NW*NS chunks per CTA are in flight. The
// table slice of the partition is prefetched into shared memory first.
//
// bf16: Q K^T and P V run on warp-level tensor cores (m16n8k16, fp32
// accumulate) with the GQA group as the M dimension (padded to 16); TMA
// writes K/V tiles with 128-byte swizzle so ldmatrix reads are conflict-free.
// fp32: plain FMA (tensor cores would round fp32 inputs to tf32).
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kChunk = 16;             // tokens per staged chunk
constexpr int kMaxPartition = 16384;   // tokens per KV partition, upper bound
constexpr int kHeadsBf16 = 16;         // query heads per CTA, tensor-core path
constexpr int kHeadsF32 = 8;           // query heads per CTA, fp32 path

struct DecodeArgs {
    void *out;
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *part_o;    // [B][H_q][S_max][D] (split mode only)
    float *part_lse;  // [B][H_q][S_max], base-2 log-sum-exp of scaled scores
    const float *k_scale;  // FP8 caches: per K/V head dequantisation scales
    const float *v_scale;
    int num_seqs, H_q, H_kv, group, bs, NB, MB, max_ctx, P, S_max, n_htiles;
    int bs_shift;      // log2(bs): block sizes are powers of two
    int window;        // > 0: attend only the last `window` positions
    float scale_log2;  // scale * log2(e): scores are kept in the base-2 domain
    unsigned long long timeout_ns;
    // shared-prefix decode (decode_prefix.cuh): sequences [group_start[g],
    // group_start[g+1]) share their first prefix_lens[g] positions
    const int32_t *group_start;
    const int32_t *prefix_lens;
    int num_groups, max_group, max_prefix;
    int P_prefix;      // tokens per prefix partition
    int S_prefix;      // partial slots [0, S_prefix) hold prefix partitions,
                       // [S_prefix, S_max) the private tails' partitions
};

// First attended position of a sequence of ctx tokens (the sliding window's
// start, 0 without a window), and the 16-aligned position its partitions
// count from.
__device__ __forceinline__ int window_lo(const DecodeArgs &a, int ctx) {
    return a.window > 0 && ctx > a.window ? ctx - a.window : 0;
}
__device__ __forceinline__ int span_base(const DecodeArgs &a, int ctx) {
    return window_lo(a, ctx) & ~(kChunk - 1);
}

// Context length of sequence b as the kernels use it: clamped to what the
// host bound and the table row allow (anything outside is recorded).
__device__ __forceinline__ int clamped_ctx(const DecodeArgs &a, int b, bool report) {
    int ctx = a.context_lens[b];
    const int cap = min(a.max_ctx, a.MB * a.bs);
    if (ctx < 0 || ctx > cap) {
        if (report) flag_error(PA_ERR_BAD_TABLE);
        ctx = ctx < 0 ? 0 : cap;
    }
    return ctx;
}

// A shared-prefix group as the kernels use it: its first sequence, its
// member count (capped at the host bound max_group) and its effective shared
// length L = min(prefix_lens[g], every member's context), clamped to
// [0, max_prefix]. Every warp computes it on its own (a lane per member, then
// a warp minimum). False for a malformed group: bounds outside
// [0, num_seqs], decreasing, or not starting at 0 / ending at num_seqs for
// the first / last group (the groups must partition the batch).
struct PrefixGroup {
    int first, n, L;
};

__device__ __forceinline__ bool prefix_group(const DecodeArgs &a, int g, PrefixGroup &pg,
                                             bool report) {
    const int g0 = __ldg(a.group_start + g), g1 = __ldg(a.group_start + g + 1);
    if (g0 < 0 || g1 < g0 || g1 > a.num_seqs || (g == 0 && g0 != 0) ||
        (g == a.num_groups - 1 && g1 != a.num_seqs)) {
        if (report) flag_error(PA_ERR_BAD_TABLE);
        return false;
    }
    int L = __ldg(a.prefix_lens + g);
    if (L < 0 || L > a.max_prefix || g1 - g0 > a.max_group) {
        if (report) flag_error(PA_ERR_BAD_TABLE);
        L = L < 0 ? 0 : min(L, a.max_prefix);
    }
    const int lane = threadIdx.x & 31;
    for (int i = lane; i < g1 - g0; i += 32) L = min(L, clamped_ctx(a, g0 + i, false));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L = min(L, __shfl_xor_sync(0xffffffffu, L, o));
    pg.first = g0;
    pg.n = min(g1 - g0, a.max_group);
    pg.L = L;
    return true;
}

// lse = -inf for `nh` rows (query heads h0.. of sequence b) at partial slot
// `slot`: a partition with nothing to attend, skipped by the merge.
__device__ __forceinline__ void write_empty_slot(const DecodeArgs &a, int b, int h0, int nh,
                                                 int slot) {
    for (int r = threadIdx.x; r < nh; r += blockDim.x)
        a.part_lse[((size_t)b * a.H_q + h0 + r) * a.S_max + slot] = -INFINITY;
}

// Programmatic dependent launch: a split CTA lets the merge kernel queued
// behind it (decode_merge.cuh) be scheduled as soon as every split CTA has
// started; its CTAs then fill the SMs the split grid's tail leaves idle.
__device__ __forceinline__ void allow_dependent_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Waits for the grid this one depends on to complete, with its writes
// visible (a no-op when launched without the dependency).
__device__ __forceinline__ void wait_for_primary_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Shared-memory plan of a split CTA: the stage ring (reused after the main
// loop for the cross-warp merge, so it is sized for whichever is larger),
// then NW*NS mbarriers, then the partition's block-table slice.
template <int NW, int NS, int STAGE_BYTES, int HT, int D>
struct DecodeSmem {
    static constexpr int kRing = NW * NS * STAGE_BYTES;
    static constexpr int kMerge = NW * HT * (D + 4) * 4 + 2 * NW * HT * 4;
    static constexpr int kStages = ((kRing > kMerge ? kRing : kMerge) + 1023) / 1024 * 1024;
    static constexpr int kBars = kStages;
    static constexpr int kTable = kBars + NW * NS * 8;
};

// Cross-warp merge of per-warp online-softmax states and the final write:
// the output (one partition) or the partition's normalised partial and lse.
template <int D, int NW, int HT, typename OutT>
__device__ __forceinline__ void decode_epilogue(const DecodeArgs &a, const float *red_o,
                                                const float *red_m, const float *red_l, int b,
                                                int h0, int nh, int s, int n_splits,
                                                float oscale = 1.f) {
    constexpr int OS = D + 4;  // padded row stride of red_o
    for (int idx = threadIdx.x; idx < nh * (D / 2); idx += NW * 32) {
        const int row = idx / (D / 2);
        const int d = (idx - row * (D / 2)) * 2;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w * HT + row]);
        float L = 0.f, o0 = 0.f, o1 = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = exp2f(red_m[w * HT + row] - M);
                L += f * red_l[w * HT + row];
                o0 += f * red_o[(w * HT + row) * OS + d];
                o1 += f * red_o[(w * HT + row) * OS + d + 1];
            }
        }
        const float inv = L > 0.f ? oscale / L : 0.f;
        const size_t bh = (size_t)b * a.H_q + h0 + row;
        if (n_splits <= 1) {
            if constexpr (sizeof(OutT) == 2) {
                *reinterpret_cast<uint32_t *>(reinterpret_cast<__nv_bfloat16 *>(a.out) + bh * D +
                                              d) = pack_bf16x2(o0 * inv, o1 * inv);
            } else {
                *reinterpret_cast<float2 *>(reinterpret_cast<float *>(a.out) + bh * D + d) =
                    make_float2(o0 * inv, o1 * inv);
            }
        } else {
            *reinterpret_cast<float2 *>(a.part_o + (bh * a.S_max + s) * D + d) =
                make_float2(o0 * inv, o1 * inv);
            if (d == 0) a.part_lse[bh * a.S_max + s] = L > 0.f ? M + log2f(L) : -INFINITY;
        }
    }
}

template <int D, typename OutT>
__device__ __forceinline__ void write_zero_rows(const DecodeArgs &a, int b, int h0, int nh) {
    for (int idx = threadIdx.x; idx < nh * D; idx += blockDim.x) {
        const size_t e = ((size_t)b * a.H_q + h0) * D + idx;
        reinterpret_cast<OutT *>(a.out)[e] = OutT(0.f);
    }
}

// ------------------------------------------------------------------ bf16
// SHARED: the private-tail pass of the shared-prefix decode. The grid is
// (member x tail partition, KV head [x head tile], group); sequence b of
// group g attends positions [L, ctx_b) here (L = the group's shared length,
// decode_prefix.cuh attends [0, L)) and always leaves partials, in slots
// S_prefix + s, with lse = -inf for a partition that has nothing to attend.
template <int D, int NW, int NS, bool SHARED = false>
__global__ void __launch_bounds__(NW * 32)
    decode_split_bf16(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
    constexpr int HT = kHeadsBf16;
    constexpr int KSTEPS = D / 16;
    constexpr int DTILES = D / 8;
    constexpr int HALF = kChunk * D * 2;    // bytes of one K (or V) chunk
    constexpr int STAGE = 2 * HALF;
    constexpr int SUBTILE = kChunk * 128;   // one 64-wide swizzled sub-tile
    using L = DecodeSmem<NW, NS, STAGE, HT, D>;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    int32_t *tbl = reinterpret_cast<int32_t *>(smem + L::kTable);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvh = blockIdx.y / a.n_htiles, ht = blockIdx.y - kvh * a.n_htiles;
    const int h0 = kvh * a.group + ht * HT;
    const int nh = min(HT, a.group - ht * HT);

    allow_dependent_launch();
    int s, b, ctx, lo, base, n_splits;
    if constexpr (SHARED) {
        const int St = a.S_max - a.S_prefix;
        const int member = blockIdx.x / St;
        s = blockIdx.x - member * St;
        PrefixGroup pg;
        if (!prefix_group(a, blockIdx.z, pg, false) || member >= pg.n) {
            wait_for_primary_grid();
            return;
        }
        b = pg.first + member;
        ctx = clamped_ctx(a, b, s == 0 && blockIdx.y == 0 && threadIdx.x == 0);
        lo = pg.L;
        base = lo & ~(kChunk - 1);
        n_splits = ctx > lo ? (ctx - base + a.P - 1) / a.P : 0;
        if (s >= n_splits) {
            write_empty_slot(a, b, h0, nh, a.S_prefix + s);
            wait_for_primary_grid();
            return;
        }
    } else {
        s = blockIdx.x;
        b = blockIdx.z;
        ctx = clamped_ctx(a, b, s == 0 && blockIdx.y == 0 && threadIdx.x == 0);
        lo = window_lo(a, ctx);
        base = span_base(a, ctx);
        n_splits = (ctx - base + a.P - 1) / a.P;
        if (s >= (n_splits > 0 ? n_splits : 1)) return;
        if (ctx == 0) {
            write_zero_rows<D, __nv_bfloat16>(a, b, h0, nh);
            return;
        }
    }
    const int tok0 = base + s * a.P;
    const int tok1 = min(tok0 + a.P, ctx);
    const int n_chunks = (tok1 - tok0 + kChunk - 1) / kChunk;
    const int lb0 = tok0 >> a.bs_shift;
    const int n_tbl = ((tok1 - 1) >> a.bs_shift) - lb0 + 1;

    // table slice of this partition -> shared memory (ids checked once here)
    const int32_t *row = a.block_tables + (size_t)b * a.MB + lb0;
    for (int i = threadIdx.x; i < n_tbl; i += NW * 32) {
        int id = __ldg(row + i);
        if (id < 0 || id >= a.NB) {
            flag_error(PA_ERR_BAD_TABLE);
            id = -1;
        }
        tbl[i] = id;
    }
    const uint32_t bar0 = sbase + L::kBars + warp * NS * 8;
    if (lane == 0) {
        for (int st = 0; st < NS; ++st) mbar_init(bar0 + st * 8, 1);
        fence_mbar_init();
    }
    __syncthreads();

    const int my_n = n_chunks > warp ? (n_chunks - warp + NW - 1) / NW : 0;
    const uint32_t stage0 = sbase + warp * NS * STAGE;

    auto issue = [&](int i) {  // lane 0: chunk i of this warp -> stage i % NS
        const int st = i % NS;
        const uint32_t bar = bar0 + st * 8;
        const int t = tok0 + (warp + i * NW) * kChunk;
        const int id = tbl[(t >> a.bs_shift) - lb0];
        if (id < 0) {
            mbar_arrive(bar);  // nothing to load; the chunk is skipped
            return;
        }
        mbar_arrive_expect_tx(bar, STAGE);
        const uint32_t kdst = stage0 + st * STAGE;
        const int off = t & (a.bs - 1);
#pragma unroll
        for (int sub = 0; sub < D / 64; ++sub) {
            tma_load_4d(kdst + sub * SUBTILE, &tmk, bar, sub * 64, off, kvh, id);
            tma_load_4d(kdst + HALF + sub * SUBTILE, &tmv, bar, sub * 64, off, kvh, id);
        }
    };
    if (lane == 0) {
        for (int i = 0; i < NS && i < my_n; ++i) issue(i);
    }

    // Q fragments (rows = query heads of the tile, zero past nh)
    const int g = lane >> 2, tig = lane & 3;
    uint32_t qa[KSTEPS][4];
    {
        const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                  ((size_t)b * a.H_q + h0) * D;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int qr = g + 8 * (r & 1);
                const int col = ks * 16 + 2 * tig + 8 * (r >> 1);
                qa[ks][r] = qr < nh ? __ldg(reinterpret_cast<const uint32_t *>(qb + qr * D + col))
                                    : 0u;
            }
    }

    float o[DTILES][4];
#pragma unroll
    for (int i = 0; i < DTILES; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    int done = 0;
    bool failed = false;

    for (int i = 0; i < my_n; ++i) {
        const int st = i % NS;
        // the verdict is made warp-uniform: the tensor-core steps below need
        // every lane
        const bool ok = mbar_wait(bar0 + st * 8, (i / NS) & 1, a.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) {
            failed = true;
            break;
        }
        done = i + 1;
        const int t = tok0 + (warp + i * NW) * kChunk;
        const int id = tbl[(t >> a.bs_shift) - lb0];
        if (id >= 0) {
            const int valid = min(kChunk, tok1 - t);
            const int first = max(0, lo - t);  // rows before the window start
            const uint32_t kb = stage0 + st * STAGE;
            const uint32_t vb = kb + HALF;
            if (valid < kChunk || first > 0) {
                // rows outside [first, valid) may hold anything (NaN, Inf):
                // zero those V rows so that P = 0 cannot turn them into NaN
                const int nvec = kChunk * (D / 8);
                for (int e = lane; e < nvec; e += 32) {
                    const int r = e / (D / 8);
                    if (r >= first && r < valid) continue;
                    const int u = e % (D / 8);
                    const uint32_t addr = vb + (u / 8) * SUBTILE + r * 128 + (u % 8) * 16;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0)
                                 : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            // S = Q K^T over 16 tokens (two n-tiles of 8)
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            {
                const int mi = lane >> 3;
                const int r = (mi >> 1) * 8 + (lane & 7);
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const int col = ks * 16 + (mi & 1) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kb + (col / 64) * SUBTILE + sw128(r, (col % 64) / 8), b0, b1, b2, b3);
                    mma_bf16_16816(sc[0], qa[ks], b0, b1);
                    mma_bf16_16816(sc[1], qa[ks], b2, b3);
                }
            }
            // online softmax in base 2; rows g (c0,c1) and g+8 (c2,c3)
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tok = nt * 8 + 2 * tig + (e & 1);
                    sc[nt][e] = tok < valid && tok >= first ? sc[nt][e] * a.scale_log2 : -INFINITY;
                }
            mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
            mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float c0 = exp2f(m0 - mn0), c1 = exp2f(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            uint32_t pa[4];
            pa[0] = pack_bf16x2(exp2f(sc[0][0] - mn0), exp2f(sc[0][1] - mn0));
            pa[1] = pack_bf16x2(exp2f(sc[0][2] - mn1), exp2f(sc[0][3] - mn1));
            pa[2] = pack_bf16x2(exp2f(sc[1][0] - mn0), exp2f(sc[1][1] - mn0));
            pa[3] = pack_bf16x2(exp2f(sc[1][2] - mn1), exp2f(sc[1][3] - mn1));
            // the denominator sums the same rounded weights the numerator uses
            l0 = l0 * c0 + (bf16_lo(pa[0]) + bf16_hi(pa[0]) + bf16_lo(pa[2]) + bf16_hi(pa[2]));
            l1 = l1 * c1 + (bf16_lo(pa[1]) + bf16_hi(pa[1]) + bf16_lo(pa[3]) + bf16_hi(pa[3]));
            // the running max rarely moves once a few chunks are in: rescale
            // the accumulators only when it did for some row of this warp
            if (__any_sync(0xffffffffu, c0 != 1.f || c1 != 1.f)) {
#pragma unroll
                for (int dt = 0; dt < DTILES; ++dt) {
                    o[dt][0] *= c0;
                    o[dt][1] *= c0;
                    o[dt][2] *= c1;
                    o[dt][3] *= c1;
                }
            }
            // O += P V  (V^T fragments via transposed ldmatrix)
            {
                const int mi = lane >> 3;
                const int r = (mi & 1) * 8 + (lane & 7);
#pragma unroll
                for (int dp = 0; dp < DTILES / 2; ++dp) {
                    const int col = (dp * 2 + (mi >> 1)) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vb + (col / 64) * SUBTILE + sw128(r, (col % 64) / 8), b0, b1, b2,
                              b3);
                    mma_bf16_16816(o[2 * dp], pa, b0, b1);
                    mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
                }
            }
        }
        __syncwarp();
        if (lane == 0 && i + NS < my_n) {
            fence_proxy_async_smem();  // order this warp's reads before the refill
            issue(i + NS);
        }
    }
    if (failed) {
        flag_error(PA_ERR_TIMEOUT);
        // let copies already issued into this warp's stages land (bounded)
        const int issued = min(my_n, done + NS);
        for (int i = done; i < issued; ++i)
            if (!mbar_wait(bar0 + (i % NS) * 8, (i / NS) & 1, a.timeout_ns)) break;
    }

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    __syncthreads();  // every warp is done with its stages: reuse them
    constexpr int OS = D + 4;
    float *red_o = reinterpret_cast<float *>(smem);
    float *red_m = reinterpret_cast<float *>(smem + NW * HT * OS * 4);
    float *red_l = red_m + NW * HT;
    if (tig == 0) {
        red_m[warp * HT + g] = m0;
        red_m[warp * HT + g + 8] = m1;
        red_l[warp * HT + g] = l0;
        red_l[warp * HT + g + 8] = l1;
    }
#pragma unroll
    for (int dt = 0; dt < DTILES; ++dt) {
        const int d = dt * 8 + 2 * tig;
        *reinterpret_cast<float2 *>(red_o + (warp * HT + g) * OS + d) = make_float2(o[dt][0], o[dt][1]);
        *reinterpret_cast<float2 *>(red_o + (warp * HT + g + 8) * OS + d) =
            make_float2(o[dt][2], o[dt][3]);
    }
    __syncthreads();
    if constexpr (SHARED) {  // always a partial, after the prefix slots
        decode_epilogue<D, NW, HT, __nv_bfloat16>(a, red_o, red_m, red_l, b, h0, nh,
                                                  a.S_prefix + s, 2);
        // the tail pass may start while the prefix pass runs (programmatic
        // dependent launch); it completes only after the prefix pass has, so
        // that the merge behind it sees both passes' partials
        wait_for_primary_grid();
    } else
        decode_epilogue<D, NW, HT, __nv_bfloat16>(a, red_o, red_m, red_l, b, h0, nh, s, n_splits);
}

// ------------------------------------------------------------------ fp32
template <int D, int NW, int NS>
__global__ void __launch_bounds__(NW * 32) decode_split_f32(const __grid_constant__ DecodeArgs a) {
    constexpr int HT = kHeadsF32;
    constexpr int VEC = D / 32;          // dims per lane
    constexpr int HALF = kChunk * D * 4;
    constexpr int STAGE = 2 * HALF;
    using L = DecodeSmem<NW, NS, STAGE, HT, D>;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    int32_t *tbl = reinterpret_cast<int32_t *>(smem + L::kTable);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = blockIdx.x;
    const int kvh = blockIdx.y / a.n_htiles, ht = blockIdx.y - kvh * a.n_htiles;
    const int b = blockIdx.z;
    const int h0 = kvh * a.group + ht * HT;
    const int nh = min(HT, a.group - ht * HT);

    allow_dependent_launch();
    const int ctx = clamped_ctx(a, b, s == 0 && blockIdx.y == 0 && threadIdx.x == 0);
    const int lo = window_lo(a, ctx), base = span_base(a, ctx);
    const int n_splits = (ctx - base + a.P - 1) / a.P;
    if (s >= (n_splits > 0 ? n_splits : 1)) return;
    if (ctx == 0) {
        write_zero_rows<D, float>(a, b, h0, nh);
        return;
    }
    const int tok0 = base + s * a.P;
    const int tok1 = min(tok0 + a.P, ctx);
    const int n_chunks = (tok1 - tok0 + kChunk - 1) / kChunk;
    const int lb0 = tok0 >> a.bs_shift;
    const int n_tbl = ((tok1 - 1) >> a.bs_shift) - lb0 + 1;

    const int32_t *row = a.block_tables + (size_t)b * a.MB + lb0;
    for (int i = threadIdx.x; i < n_tbl; i += NW * 32) {
        int id = __ldg(row + i);
        if (id < 0 || id >= a.NB) {
            flag_error(PA_ERR_BAD_TABLE);
            id = -1;
        }
        tbl[i] = id;
    }
    const uint32_t bar0 = sbase + L::kBars + warp * NS * 8;
    if (lane == 0) {
        for (int st = 0; st < NS; ++st) mbar_init(bar0 + st * 8, 1);
        fence_mbar_init();
    }
    __syncthreads();

    const int my_n = n_chunks > warp ? (n_chunks - warp + NW - 1) / NW : 0;
    const uint32_t stage0 = sbase + warp * NS * STAGE;
    const float *kc = reinterpret_cast<const float *>(a.k_cache);
    const float *vc = reinterpret_cast<const float *>(a.v_cache);

    auto issue = [&](int i) {
        const int st = i % NS;
        const uint32_t bar = bar0 + st * 8;
        const int t = tok0 + (warp + i * NW) * kChunk;
        const int id = tbl[(t >> a.bs_shift) - lb0];
        if (id < 0) {
            mbar_arrive(bar);
            return;
        }
        mbar_arrive_expect_tx(bar, STAGE);
        const size_t page = (((size_t)id * a.H_kv + kvh) * a.bs + (t & (a.bs - 1))) * D;
        bulk_load(stage0 + st * STAGE, kc + page, HALF, bar);
        bulk_load(stage0 + st * STAGE + HALF, vc + page, HALF, bar);
    };
    if (lane == 0) {
        for (int i = 0; i < NS && i < my_n; ++i) issue(i);
    }

    float qv[HT][VEC], acc[HT][VEC], mrow[HT], lrow[HT];
    {
        const float *qb = reinterpret_cast<const float *>(a.q) + ((size_t)b * a.H_q + h0) * D;
#pragma unroll
        for (int g = 0; g < HT; ++g) {
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                qv[g][v] = g < nh ? __ldg(qb + g * D + lane * VEC + v) : 0.f;
                acc[g][v] = 0.f;
            }
            mrow[g] = -INFINITY;
            lrow[g] = 0.f;
        }
    }
    int done = 0;
    bool failed = false;
    for (int i = 0; i < my_n; ++i) {
        const int st = i % NS;
        // the verdict is made warp-uniform: the tensor-core steps below need
        // every lane
        const bool ok = mbar_wait(bar0 + st * 8, (i / NS) & 1, a.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) {
            failed = true;
            break;
        }
        done = i + 1;
        const int t = tok0 + (warp + i * NW) * kChunk;
        const int id = tbl[(t >> a.bs_shift) - lb0];
        if (id >= 0) {
            const int valid = min(kChunk, tok1 - t);
            const int first = max(0, lo - t);
            const float *ks = reinterpret_cast<const float *>(smem + warp * NS * STAGE + st * STAGE);
            const float *vs = ks + kChunk * D;
            for (int j = first; j < valid; ++j) {  // tokens outside the span are never touched
                float kk[VEC], vv[VEC];
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    kk[v] = ks[j * D + lane * VEC + v];
                    vv[v] = vs[j * D + lane * VEC + v];
                }
#pragma unroll
                for (int g = 0; g < HT; ++g) {
                    if (g < nh) {
                        float dot = 0.f;
#pragma unroll
                        for (int v = 0; v < VEC; ++v) dot = fmaf(qv[g][v], kk[v], dot);
                        const float sc = warp_sum(dot) * a.scale_log2;
                        const float mn = fmaxf(mrow[g], sc);
                        const float c = exp2f(mrow[g] - mn);
                        const float p = exp2f(sc - mn);
                        lrow[g] = lrow[g] * c + p;
#pragma unroll
                        for (int v = 0; v < VEC; ++v) acc[g][v] = fmaf(acc[g][v], c, p * vv[v]);
                        mrow[g] = mn;
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0 && i + NS < my_n) {
            fence_proxy_async_smem();  // order this warp's reads before the refill
            issue(i + NS);
        }
    }
    if (failed) {
        flag_error(PA_ERR_TIMEOUT);
        const int issued = min(my_n, done + NS);
        for (int i = done; i < issued; ++i)
            if (!mbar_wait(bar0 + (i % NS) * 8, (i / NS) & 1, a.timeout_ns)) break;
    }

    __syncthreads();
    constexpr int OS = D + 4;
    float *red_o = reinterpret_cast<float *>(smem);
    float *red_m = reinterpret_cast<float *>(smem + NW * HT * OS * 4);
    float *red_l = red_m + NW * HT;
#pragma unroll
    for (int g = 0; g < HT; ++g) {
        if (lane == 0) {
            red_m[warp * HT + g] = mrow[g];
            red_l[warp * HT + g] = lrow[g];
        }
#pragma unroll
        for (int v = 0; v < VEC; ++v) red_o[(warp * HT + g) * OS + lane * VEC + v] = acc[g][v];
    }
    __syncthreads();
    decode_epilogue<D, NW, HT, float>(a, red_o, red_m, red_l, b, h0, nh, s, n_splits);
}

}  // namespace pa
