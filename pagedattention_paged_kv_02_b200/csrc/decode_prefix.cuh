// decode_prefix.cuh -- the shared-prefix pass of paged decode: each shared
// K/V page is fetched once for every sequence that shares it.
//
// Page "字节跳动 AI Infra (2)", question "vLLM与PagedAttention的原理": beams of
// one request share their prefix blocks (B1 and B3 in the page's example),
// so the prefix's K/V live once in the pool however many sequences read it.
// The attention of each sequence's query over its context splits at the
// prefix boundary L into two partial results (page "字节跳动 AI Infra (2)",
// algorithm-level table, FlashDecoding row: partial softmax results merged by
// log-sum-exp): positions [0, L), the same K/V for every sequence of the
// group, and positions [L, ctx_b), the sequence's own. This kernel computes
// the first part for all sequences of a group at once; the private tails go
// through decode_split_bf16<..., SHARED = true> and the merge kernel
// (decode_merge.cuh) combines the partials.
//
// Work decomposition: one CTA per (prefix partition, KV head x row tile,
// group). The rows of a CTA are (member sequence, query head of the KV
// head's group) pairs, MT m-tiles of 16 rows: every K/V chunk fetched serves
// MT*16 query rows (8 beams x 4 heads = 32 rows for the beam batch), instead
// of one sequence's group of heads. Four warps: warp w computes m-tile
// w % MT over every (4/MT)-th 16-token chunk of the partition (its token
// group); the MT warps of a token group share one TMA ring of NS stages:
// lane 0 of the group's first warp issues the chunk's K and V boxes, every
// warp of the group waits on the stage's full barrier, reads it, and
// arrives on its empty barrier (MT arrivals free the stage for the next
// copy). QK^T and PV are warp-level mma.sync m16n8k16 (bf16, fp32
// accumulate) with the 16 rows of the warp's m-tile as M; the online softmax
// keeps a running max and sum per row. At the end the token groups' states
// are merged through shared memory and each row's normalised partial and
// base-2 lse go to its sequence's partial slot s.
#pragma once

#include "decode.cuh"

namespace pa {

constexpr int kPrefixWarps = 4;

template <int D, int MT>
struct PrefixSmem {
    static constexpr int TG = kPrefixWarps / MT;  // token groups
    static constexpr int NS = 8 / TG;             // ring stages per token group
    static constexpr int STAGE = 2 * kChunk * D * 2;
    static constexpr int ROWS = MT * 16;
    static constexpr int kRing = TG * NS * STAGE;
    static constexpr int kMerge = TG * ROWS * (D + 4) * 4 + 2 * TG * ROWS * 4;
    static constexpr int kStages = ((kRing > kMerge ? kRing : kMerge) + 1023) / 1024 * 1024;
    static constexpr int kBars = kStages;                 // full[TG][NS], then empty[TG][NS]
    static constexpr int kTable = kBars + 2 * TG * NS * 8;
};

template <int D, int MT>
__global__ void __launch_bounds__(kPrefixWarps * 32)
    decode_prefix_bf16(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv) {
    using L = PrefixSmem<D, MT>;
    constexpr int TG = L::TG, NS = L::NS, ROWS = L::ROWS, STAGE = L::STAGE;
    constexpr int KSTEPS = D / 16;
    constexpr int DTILES = D / 8;
    constexpr int HALF = kChunk * D * 2;
    constexpr int SUBTILE = kChunk * 128;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    int32_t *tbl = reinterpret_cast<int32_t *>(smem + L::kTable);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = warp % MT, tg = warp / MT;
    const int s = blockIdx.x;
    const int kvh = blockIdx.y / a.n_htiles, rt = blockIdx.y - kvh * a.n_htiles;

    allow_dependent_launch();
    PrefixGroup pg;
    if (!prefix_group(a, blockIdx.z, pg, s == 0 && blockIdx.y == 0 && threadIdx.x == 0)) return;
    const int grp_rows = pg.n * a.group;  // (member, head) rows of the group
    const int r0 = rt * ROWS;             // first row of this CTA
    if (r0 >= grp_rows) return;
    const int nrows = min(ROWS, grp_rows - r0);
    const int n_splits = (pg.L + a.P_prefix - 1) / a.P_prefix;
    if (s >= n_splits) {  // nothing to attend in this slot: lse = -inf
        for (int r = threadIdx.x; r < nrows; r += blockDim.x) {
            const int rr = r0 + r, b = pg.first + rr / a.group;
            a.part_lse[((size_t)b * a.H_q + kvh * a.group + rr % a.group) * a.S_max + s] =
                -INFINITY;
        }
        return;
    }
    const int tok0 = s * a.P_prefix;
    const int tok1 = min(tok0 + a.P_prefix, pg.L);
    const int n_chunks = (tok1 - tok0 + kChunk - 1) / kChunk;
    const int lb0 = tok0 >> a.bs_shift;
    const int n_tbl = ((tok1 - 1) >> a.bs_shift) - lb0 + 1;

    // the partition's slice of the group's first sequence's table (the
    // prefix's blocks), checked once
    const int32_t *row = a.block_tables + (size_t)pg.first * a.MB + lb0;
    for (int i = threadIdx.x; i < n_tbl; i += blockDim.x) {
        int id = __ldg(row + i);
        if (id < 0 || id >= a.NB) {
            flag_error(PA_ERR_BAD_TABLE);
            id = -1;
        }
        tbl[i] = id;
    }
    // stage st of token group t: full barrier at kBars + (t*NS + st)*8 (one
    // arrival + the copy's bytes), empty barrier TG*NS*8 further (MT
    // arrivals, one per warp reading the stage)
    const uint32_t full0 = sbase + L::kBars + tg * NS * 8;
    const uint32_t empty0 = full0 + TG * NS * 8;
    const bool producer = mt == 0;  // lane 0 of the token group's first warp issues
    if (producer && lane == 0) {
        for (int st = 0; st < NS; ++st) {
            mbar_init(full0 + st * 8, 1);
            mbar_init(empty0 + st * 8, MT);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const int my_n = n_chunks > tg ? (n_chunks - tg + TG - 1) / TG : 0;
    const uint32_t stage0 = sbase + tg * NS * STAGE;

    auto issue = [&](int i) {  // chunk i of this token group -> stage i % NS
        const int st = i % NS;
        const uint32_t bar = full0 + st * 8;
        const int t = tok0 + (tg + i * TG) * kChunk;
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
    int issued = 0;
    if (producer && lane == 0) {
        for (int i = 0; i < NS && i < my_n; ++i) issue(i);
        issued = min(NS, my_n);
    }

    // Q fragments of this warp's m-tile: row q of the tile is group row
    // r0 + mt*16 + q, i.e. query head kvh*G + row % G of member row / G
    const int g = lane >> 2, tig = lane & 3;
    uint32_t qa[KSTEPS][4];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int rr = mt * 16 + g + 8 * hr;  // row within the CTA
        const bool ok = rr < nrows;
        const __nv_bfloat16 *qb = nullptr;
        if (ok) {
            const int gr = r0 + rr;
            const int b = pg.first + gr / a.group;
            qb = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                 ((size_t)b * a.H_q + kvh * a.group + gr % a.group) * D;
        }
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int col = ks * 16 + 2 * tig + 8 * c;
                qa[ks][hr + 2 * c] =
                    ok ? __ldg(reinterpret_cast<const uint32_t *>(qb + col)) : 0u;
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
        const bool ok = mbar_wait(full0 + st * 8, (i / NS) & 1, a.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) {
            failed = true;
            break;
        }
        done = i + 1;
        const int t = tok0 + (tg + i * TG) * kChunk;
        const int id = tbl[(t >> a.bs_shift) - lb0];
        if (id >= 0) {
            const int valid = min(kChunk, tok1 - t);
            const uint32_t kb = stage0 + st * STAGE;
            const uint32_t vb = kb + HALF;
            if (valid < kChunk) {
                // rows past the prefix may hold anything (NaN): zero those V
                // rows so that P = 0 cannot meet a NaN there. Every warp of
                // the token group writes the same zeros before its own reads.
                for (int e = lane; e < kChunk * (D / 8); e += 32) {
                    const int r = e / (D / 8);
                    if (r < valid) continue;
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
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tok = nt * 8 + 2 * tig + (e & 1);
                    sc[nt][e] = tok < valid ? sc[nt][e] * a.scale_log2 : -INFINITY;
                }
            float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
            float mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
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
        // this warp is done with the stage: release it (its reads ordered
        // before the next copy into it, which is an async-proxy write)
        __syncwarp();
        if (lane == 0) {
            fence_proxy_async_smem();
            mbar_arrive(empty0 + st * 8);
        }
        // the producer refills the stage once every warp of the group left it
        if (producer && lane == 0 && i + NS < my_n) {
            if (!mbar_wait(empty0 + st * 8, (i / NS) & 1, a.timeout_ns)) {
                failed = true;
            } else {
                issue(i + NS);
                issued = i + NS + 1;
            }
        }
        if (__shfl_sync(0xffffffffu, failed ? 1 : 0, 0)) {
            failed = true;
            break;
        }
    }
    if (failed) {
        flag_error(PA_ERR_TIMEOUT);
        // let copies already issued into this group's stages land (bounded)
        if (producer && lane == 0)
            for (int i = done; i < issued; ++i)
                if (!mbar_wait(full0 + (i % NS) * 8, (i / NS) & 1, a.timeout_ns)) break;
    }

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    __syncthreads();  // every warp is done with the rings: reuse them
    constexpr int OS = D + 4;
    float *red_o = reinterpret_cast<float *>(smem);  // [TG][ROWS][OS]
    float *red_m = reinterpret_cast<float *>(smem + TG * ROWS * OS * 4);
    float *red_l = red_m + TG * ROWS;
    {
        const int ra = mt * 16 + g, rb = ra + 8;  // this lane's two rows in the CTA
        if (tig == 0) {
            red_m[tg * ROWS + ra] = m0;
            red_m[tg * ROWS + rb] = m1;
            red_l[tg * ROWS + ra] = l0;
            red_l[tg * ROWS + rb] = l1;
        }
#pragma unroll
        for (int dt = 0; dt < DTILES; ++dt) {
            const int d = dt * 8 + 2 * tig;
            *reinterpret_cast<float2 *>(red_o + (tg * ROWS + ra) * OS + d) =
                make_float2(o[dt][0], o[dt][1]);
            *reinterpret_cast<float2 *>(red_o + (tg * ROWS + rb) * OS + d) =
                make_float2(o[dt][2], o[dt][3]);
        }
    }
    __syncthreads();
    // merge the token groups' states per row; each row's partial goes to its
    // own sequence's slot s
    for (int idx = threadIdx.x; idx < nrows * (D / 2); idx += blockDim.x) {
        const int r = idx / (D / 2);
        const int d = (idx - r * (D / 2)) * 2;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < TG; ++w) M = fmaxf(M, red_m[w * ROWS + r]);
        float Lsum = 0.f, x0 = 0.f, x1 = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < TG; ++w) {
                const float f = exp2f(red_m[w * ROWS + r] - M);
                Lsum += f * red_l[w * ROWS + r];
                x0 += f * red_o[(w * ROWS + r) * OS + d];
                x1 += f * red_o[(w * ROWS + r) * OS + d + 1];
            }
        }
        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
        const int gr = r0 + r;
        const size_t bh = (size_t)(pg.first + gr / a.group) * a.H_q + kvh * a.group + gr % a.group;
        *reinterpret_cast<float2 *>(a.part_o + (bh * a.S_max + s) * D + d) =
            make_float2(x0 * inv, x1 * inv);
        if (d == 0) a.part_lse[bh * a.S_max + s] = Lsum > 0.f ? M + log2f(Lsum) : -INFINITY;
    }
}

}  // namespace pa
