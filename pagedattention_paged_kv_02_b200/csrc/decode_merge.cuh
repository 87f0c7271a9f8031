// decode_merge.cuh -- the second decode kernel: log-sum-exp merge of the
// split partials.
//
// Page "字节跳动 AI Infra (2)", algorithm-level table, FlashDecoding row: the
// KV length is split, each split produces a partial result, and the partials
// are merged. Each partition s of (sequence b, query head h) left its
// normalised output o_s and the base-2 log-sum-exp lse_s of its scaled
// scores; out = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M), M = max lse_s
// (page "LLM推理优化", section 2.1: rescaling by the running max keeps the
// exponentials in range).
//
// Launched as a programmatic dependent of the split kernel: its CTAs may be
// placed while the split grid's last CTAs run and wait (griddepcontrol.wait)
// for that grid to finish, with its writes visible, before reading partials.
#pragma once

#include "decode.cuh"

namespace pa {

// ------------------------------------------------------------- LSE merge
// out = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M), M = max_s lse_s, for
// every (sequence, query head) with more than one partition.
//
// Few partitions per head (S_max <= kWarpMergeMax): one warp per
// (sequence, head), eight per CTA, each lane owning D/32 dimensions and
// walking the partitions in order; heads with one partition cost a warp a
// length read.
//
// SHARED (the shared-prefix decode): every one of the S_max slots of every
// (sequence, head) was written -- prefix partitions, then the private tail's
// -- and a slot with lse = -inf (nothing attended) has no partial output:
// its weight is zero and its output is never read.
constexpr int kWarpMergeMax = 16;

template <int D, typename OutT, bool SHARED = false>
__global__ void __launch_bounds__(256) decode_reduce_warp(const __grid_constant__ DecodeArgs a) {
    constexpr int VEC = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x * 8 + warp;
    if (bh >= a.num_seqs * a.H_q) return;
    const int b = bh / a.H_q;
    int n = a.S_max;
    if constexpr (!SHARED) {
        const int ctx = clamped_ctx(a, b, false);
        n = (ctx - span_base(a, ctx) + a.P - 1) / a.P;
        if (n <= 1) return;
    }
    wait_for_primary_grid();
    const float *lse = a.part_lse + (size_t)bh * a.S_max;
    const float *po = a.part_o + (size_t)bh * a.S_max * D + lane * VEC;
    // lane s holds lse_s: one load for all of them, then shuffles (no second
    // round trip before the partials' loads, which are independent)
    const float my_lse = lane < n ? __ldcg(lse + lane) : -INFINITY;
    float M = my_lse;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
    float W = 0.f;
    if (M != -INFINITY) {
#pragma unroll 4
        for (int s = 0; s < n; ++s) {
            const float ls = __shfl_sync(0xffffffffu, my_lse, s);
            if (SHARED && ls == -INFINITY) continue;  // an empty slot
            const float w = exp2f(ls - M);
            W += w;
            if constexpr (VEC == 4) {
                const float4 x = __ldcg(reinterpret_cast<const float4 *>(po + (size_t)s * D));
                acc[0] = fmaf(w, x.x, acc[0]);
                acc[1] = fmaf(w, x.y, acc[1]);
                acc[2] = fmaf(w, x.z, acc[2]);
                acc[3] = fmaf(w, x.w, acc[3]);
            } else {
                const float2 x = __ldcg(reinterpret_cast<const float2 *>(po + (size_t)s * D));
                acc[0] = fmaf(w, x.x, acc[0]);
                acc[1] = fmaf(w, x.y, acc[1]);
            }
        }
    }
    OutT *dst = reinterpret_cast<OutT *>(a.out) + (size_t)bh * D + lane * VEC;
#pragma unroll
    for (int v = 0; v < VEC; ++v) dst[v] = OutT(W > 0.f ? acc[v] / W : 0.f);
}

// Many partitions per head: one CTA (16 warps) per (sequence, head), the
// warps taking every 16th partition, four partitions' loads in flight per
// warp (a long context has hundreds of partials per head and only a few
// heads, so the merge is latency-bound unless many loads are outstanding).
template <int D, typename OutT, bool SHARED = false>
__global__ void __launch_bounds__(512) decode_reduce(const __grid_constant__ DecodeArgs a) {
    constexpr int NWR = 16;
    constexpr int VEC = D / 32;
    const int bh = blockIdx.x;
    const int b = bh / a.H_q;
    int n = a.S_max;
    if constexpr (!SHARED) {
        const int ctx = clamped_ctx(a, b, false);
        n = (ctx - span_base(a, ctx) + a.P - 1) / a.P;
        if (n <= 1) return;
    }
    wait_for_primary_grid();
    const float *lse = a.part_lse + (size_t)bh * a.S_max;
    const float *po = a.part_o + (size_t)bh * a.S_max * D;
    __shared__ float red[NWR][D + 1];
    __shared__ float wsum[NWR];
    __shared__ float smax[NWR];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    float M = -INFINITY;
    for (int s = threadIdx.x; s < n; s += NWR * 32) M = fmaxf(M, __ldcg(lse + s));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) smax[warp] = M;
    __syncthreads();
    M = smax[0];
#pragma unroll
    for (int w = 1; w < NWR; ++w) M = fmaxf(M, smax[w]);

    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
    float W = 0.f;
    if (M != -INFINITY) {
#pragma unroll 4
        for (int s = warp; s < n; s += NWR) {
            const float ls = __ldcg(lse + s);
            if (SHARED && ls == -INFINITY) continue;  // an empty slot
            const float w = exp2f(ls - M);
            W += w;
            const float *src = po + (size_t)s * D + lane * VEC;
            if constexpr (VEC == 4) {
                const float4 x = __ldcg(reinterpret_cast<const float4 *>(src));
                acc[0] = fmaf(w, x.x, acc[0]);
                acc[1] = fmaf(w, x.y, acc[1]);
                acc[2] = fmaf(w, x.z, acc[2]);
                acc[3] = fmaf(w, x.w, acc[3]);
            } else {
                const float2 x = __ldcg(reinterpret_cast<const float2 *>(src));
                acc[0] = fmaf(w, x.x, acc[0]);
                acc[1] = fmaf(w, x.y, acc[1]);
            }
        }
    }
#pragma unroll
    for (int v = 0; v < VEC; ++v) red[warp][lane * VEC + v] = acc[v];
    if (lane == 0) wsum[warp] = W;
    __syncthreads();
    if (threadIdx.x < D) {
        const int d = threadIdx.x;
        float Wt = 0.f, x = 0.f;
#pragma unroll
        for (int w = 0; w < NWR; ++w) {
            Wt += wsum[w];
            x += red[w][d];
        }
        const float r = Wt > 0.f ? x / Wt : 0.f;
        reinterpret_cast<OutT *>(a.out)[(size_t)bh * D + d] = OutT(r);
    }
}

}  // namespace pa
