// decode_fp8.cuh -- paged decode over an 8-bit KV cache: FP8 (E4M3) or INT8
// codes.
//
// Page "字节跳动 AI Infra (2)", optimisation table, row "KV量化(INT8)", and
// page "LLM推理优化", section 1.3 (INT8/INT4 K/V): store K/V in low precision
// to shrink the cache; decode is bound by KV reads (page
// "vLLM框架是怎么做推理加速的", section 3), so halving the bytes per element
// halves its cost. Here each element is an E4M3 or INT8 code and value =
// code * scale[kv head]; the scales fold into the score scale (K) and into
// the output (V), so the tensor-core products run on the exact code values.
//
// Same work decomposition and pipeline as the bf16 split kernel (one CTA per
// (partition, kv head [x 16-head tile], sequence), per-warp TMA rings of
// 16-token chunks, warp-level mma.sync with the GQA group as M), with these
// differences:
//   * a chunk is 16 tokens x 128 one-byte dims: one 128-byte swizzled TMA
//     box each for K and V (2 KB each);
//   * K fragments come from ldmatrix on the byte rows directly: a lane's
//     32-bit element holds 4 consecutive dims, converted to two f16 pairs.
//     That lane layout assigns dims to fragment k-slots in a fixed
//     permutation; Q's fragment is loaded with the same permutation, and a
//     dot product does not depend on the order of its terms;
//   * V fragments come from transposed ldmatrix (2 tokens x 2 dims per
//     lane) plus one byte permute, giving two f16 token pairs for two
//     adjacent dims; the output columns come out permuted accordingly and
//     are put back in order in the merge;
//   * the tensor-core type is f16 (E4M3 -> f16 and INT8 -> f16 are exact), P
//     is rounded to f16 and the denominator sums the same rounded weights.
#pragma once

#include "decode.cuh"
#include "reshape_and_cache.cuh"

namespace pa {

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
        " {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// four E4M3 codes w = [c0 c1 c2 c3] -> f16 pairs {c0, c1} and {c2, c3},
// exact: the word's two 16-bit halves feed the conversion directly (no
// shift or zero-extension per pair; 5.6 % on the FP8 Llama-7B batch)
__device__ __forceinline__ void e4m3x4_to_f16x2_hw(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// 2^x on the special-function unit, subnormal results flushed to zero (a
// softmax weight below 2^-126 of the row's largest does not register).
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Four INT8 codes w = [c0 c1 c2 c3] (c0 the low byte) -> the f16 pairs
// {c0, c2} (even) and {c1, c3} (odd), exact, without the conversion pipe:
// flipping the sign bits makes each byte c + 128 in 0..255; a byte under the
// f16 pattern 0x64 reads 1024 + (c + 128) (the ulp at 1024 is 1), and one
// packed f16 subtraction of 1152 leaves c.
__device__ __forceinline__ void int8x4_to_f16x2(uint32_t w, uint32_t &even, uint32_t &odd) {
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t e = __byte_perm(u, 0x64646464u, 0x4240);  // [c0', 0x64, c2', 0x64]
    const uint32_t o = __byte_perm(u, 0x64646464u, 0x4341);  // [c1', 0x64, c3', 0x64]
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(even) : "r"(e), "r"(0x64806480u));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(odd) : "r"(o), "r"(0x64806480u));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float f16_lo(uint32_t v) {
    return __half2float(__ushort_as_half((unsigned short)(v & 0xffffu)));
}
__device__ __forceinline__ float f16_hi(uint32_t v) {
    return __half2float(__ushort_as_half((unsigned short)(v >> 16)));
}

// CT: tokens per pipeline stage (16 or 32). A 32-token stage is two
// 16-token page pieces (each inside one physical block, so each has its own
// table lookup); it halves the softmax and hand-off work per byte.
// INT8: the code format. E4M3 codes become f16 through the conversion
// instruction; INT8 codes on the integer and FMA pipes (int8x4_to_f16x2,
// 2.5 instructions per pair).
template <int NW, int NS, int CT, bool INT8>
__global__ void __launch_bounds__(NW * 32)
    decode_split_q8(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
    constexpr int D = 128;
    constexpr int HT = kHeadsBf16;
    constexpr int PIECES = CT / kChunk;
    constexpr int HALF = CT * D;  // bytes of one K (or V) stage
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
        write_zero_rows<D, __nv_bfloat16>(a, b, h0, nh);
        return;
    }
    const int tok0 = base + s * a.P;
    const int tok1 = min(tok0 + a.P, ctx);
    const int n_chunks = (tok1 - tok0 + CT - 1) / CT;
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

    auto issue = [&](int i) {
        const int st = i % NS;
        const uint32_t bar = bar0 + st * 8;
        const int t = tok0 + (warp + i * NW) * CT;
        int ids[PIECES];
        int n = 0;
#pragma unroll
        for (int p = 0; p < PIECES; ++p) {
            const int tp = t + p * kChunk;
            ids[p] = tp < tok1 ? tbl[(tp >> a.bs_shift) - lb0] : -1;
            n += ids[p] >= 0;
        }
        if (n == 0) {
            mbar_arrive(bar);
            return;
        }
        mbar_arrive_expect_tx(bar, n * 2 * kChunk * D);
        const uint32_t kdst = stage0 + st * STAGE;
#pragma unroll
        for (int p = 0; p < PIECES; ++p) {
            if (ids[p] < 0) continue;
            const int off = (t + p * kChunk) & (a.bs - 1);
            tma_load_4d(kdst + p * kChunk * D, &tmk, bar, 0, off, kvh, ids[p]);
            tma_load_4d(kdst + HALF + p * kChunk * D, &tmv, bar, 0, off, kvh, ids[p]);
        }
    };
    if (lane == 0) {
        for (int i = 0; i < NS && i < my_n; ++i) issue(i);
    }

    const float sl2 = a.scale_log2 * __ldg(a.k_scale + kvh);
    const float vsc = __ldg(a.v_scale + kvh);

    // Q fragments in f16, dims permuted to match the K fragments: slot
    // 2c+j (j = 0,1) of k-step ks holds dim 16ks+4c+j, slot 2c+8+j holds
    // dim 16ks+4c+2+j (c = lane % 4); with K converted on the integer pipe
    // (even and odd codes of a word) slot 2c+j holds dim 16ks+4c+2j and slot
    // 2c+8+j dim 16ks+4c+1+2j
    const int g = lane >> 2, tig = lane & 3;
    uint32_t qa[8][4];
    {
        const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                  ((size_t)b * a.H_q + h0) * D;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int qr = g + 8 * hr;
                uint2 v = make_uint2(0u, 0u);
                if (qr < nh)
                    v = __ldg(reinterpret_cast<const uint2 *>(qb + qr * D + ks * 16 + 4 * tig));
                if (INT8) {
                    qa[ks][hr] = pack_f16x2(bf16_lo(v.x), bf16_lo(v.y));      // dims +0, +2
                    qa[ks][hr + 2] = pack_f16x2(bf16_hi(v.x), bf16_hi(v.y));  // dims +1, +3
                } else {
                    qa[ks][hr] = pack_f16x2(bf16_lo(v.x), bf16_hi(v.x));      // dims +0, +1
                    qa[ks][hr + 2] = pack_f16x2(bf16_lo(v.y), bf16_hi(v.y));  // dims +2, +3
                }
            }
    }

    const bool hi_rows = nh > 8;

    // O fragments of 16 virtual n-tiles: tile 2u+p, column n <-> dim 16u+2n+p
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    int done = 0;
    bool failed = false;

    for (int i = 0; i < my_n; ++i) {
        const int st = i % NS;
        const bool ok = mbar_wait(bar0 + st * 8, (i / NS) & 1, a.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) {
            failed = true;
            break;
        }
        done = i + 1;
        const int t = tok0 + (warp + i * NW) * CT;
        // pieces that were loaded (inside the span, valid table entry)
        int pok = 0;
#pragma unroll
        for (int p = 0; p < PIECES; ++p)
            if (t + p * kChunk < tok1 && tbl[((t + p * kChunk) >> a.bs_shift) - lb0] >= 0)
                pok |= 1 << p;
        if (pok) {
            const int valid = min(CT, tok1 - t);
            const int first = max(0, lo - t);  // rows before the window start
            const uint32_t kb = stage0 + st * STAGE;
            const uint32_t vb = kb + HALF;
            const bool full = valid == CT && first == 0 && pok == (1 << PIECES) - 1;
            if (!full) {
                // rows outside [first, valid) or in an unloaded piece may hold
                // anything: zero those V rows so that P = 0 cannot meet a NaN
                for (int e = lane; e < CT * 8; e += 32) {
                    const int r = e / 8;
                    if (r >= first && r < valid && ((pok >> (r / kChunk)) & 1)) continue;
                    const uint32_t addr = vb + r * 128 + (e % 8) * 16;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0)
                                 : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            // S = Q K^T per 16-token piece: matrices (tokens 0-7 | 8-15) x
            // (16-dim units u, u+1)
            float sc[2 * PIECES][4];
#pragma unroll
            for (int nt = 0; nt < 2 * PIECES; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
            {
                const int mi = lane >> 3;
                const int r = (mi & 1) * 8 + (lane & 7);
#pragma unroll
                for (int p = 0; p < PIECES; ++p)
#pragma unroll
                    for (int kp = 0; kp < 4; ++kp) {
                        const int u = kp * 2 + (mi >> 1);
                        uint32_t r0, r1, r2, r3;
                        ldsm_x4(kb + p * kChunk * D + sw128(r, u), r0, r1, r2, r3);
                        if constexpr (INT8) {
                            uint32_t e0, o0, e1, o1, e2, o2, e3, o3;
                            int8x4_to_f16x2(r0, e0, o0);
                            int8x4_to_f16x2(r1, e1, o1);
                            int8x4_to_f16x2(r2, e2, o2);
                            int8x4_to_f16x2(r3, e3, o3);
                            mma_f16_16816(sc[2 * p], qa[2 * kp], e0, o0);
                            mma_f16_16816(sc[2 * p + 1], qa[2 * kp], e1, o1);
                            mma_f16_16816(sc[2 * p], qa[2 * kp + 1], e2, o2);
                            mma_f16_16816(sc[2 * p + 1], qa[2 * kp + 1], e3, o3);
                        } else {
                            uint32_t l0, h0, l1, h1, l2, h2, l3, h3;
                            e4m3x4_to_f16x2_hw(r0, l0, h0);
                            e4m3x4_to_f16x2_hw(r1, l1, h1);
                            e4m3x4_to_f16x2_hw(r2, l2, h2);
                            e4m3x4_to_f16x2_hw(r3, l3, h3);
                            mma_f16_16816(sc[2 * p], qa[2 * kp], l0, h0);
                            mma_f16_16816(sc[2 * p + 1], qa[2 * kp], l1, h1);
                            mma_f16_16816(sc[2 * p], qa[2 * kp + 1], l2, h2);
                            mma_f16_16816(sc[2 * p + 1], qa[2 * kp + 1], l3, h3);
                        }
                    }
            }
            float mx0 = -INFINITY, mx1 = -INFINITY;
            if (full) {
#pragma unroll
                for (int nt = 0; nt < 2 * PIECES; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        sc[nt][e] *= sl2;
                        if (e < 2)
                            mx0 = fmaxf(mx0, sc[nt][e]);
                        else
                            mx1 = fmaxf(mx1, sc[nt][e]);
                    }
            } else {
#pragma unroll
                for (int nt = 0; nt < 2 * PIECES; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int tok = nt * 8 + 2 * tig + (e & 1);
                        const bool ok =
                            tok < valid && tok >= first && ((pok >> (tok / kChunk)) & 1);
                        sc[nt][e] = ok ? sc[nt][e] * sl2 : -INFINITY;
                        if (e < 2)
                            mx0 = fmaxf(mx0, sc[nt][e]);
                        else
                            mx1 = fmaxf(mx1, sc[nt][e]);
                    }
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            // a row with nothing visible yet keeps reference -inf: use 0 then
            const float r0m = mn0 == -INFINITY ? 0.f : mn0, r1m = mn1 == -INFINITY ? 0.f : mn1;
            const float c0 = ex2_fast(m0 - r0m), c1 = ex2_fast(m1 - r1m);
            m0 = mn0;
            m1 = mn1;
            uint32_t pa[PIECES][4];
            float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
            for (int p = 0; p < PIECES; ++p) {
                pa[p][0] = pack_f16x2(ex2_fast(sc[2 * p][0] - r0m), ex2_fast(sc[2 * p][1] - r0m));
                pa[p][2] =
                    pack_f16x2(ex2_fast(sc[2 * p + 1][0] - r0m), ex2_fast(sc[2 * p + 1][1] - r0m));
                ps0 += f16_lo(pa[p][0]) + f16_hi(pa[p][0]) + f16_lo(pa[p][2]) + f16_hi(pa[p][2]);
            }
            if (hi_rows) {  // rows g+8 hold query heads only when the tile has more than 8
#pragma unroll
                for (int p = 0; p < PIECES; ++p) {
                    pa[p][1] = pack_f16x2(ex2_fast(sc[2 * p][2] - r1m), ex2_fast(sc[2 * p][3] - r1m));
                    pa[p][3] = pack_f16x2(ex2_fast(sc[2 * p + 1][2] - r1m),
                                          ex2_fast(sc[2 * p + 1][3] - r1m));
                    ps1 += f16_lo(pa[p][1]) + f16_hi(pa[p][1]) + f16_lo(pa[p][3]) + f16_hi(pa[p][3]);
                }
            } else {
#pragma unroll
                for (int p = 0; p < PIECES; ++p) pa[p][1] = pa[p][3] = 0u;
            }
            l0 = l0 * c0 + ps0;
            l1 = l1 * c1 + ps1;
            // the running max rarely moves once a few chunks are in: rescale
            // the accumulators only when it did for some row of this warp
            if (__any_sync(0xffffffffu, c0 != 1.f || c1 != 1.f)) {
#pragma unroll
                for (int dt = 0; dt < 16; ++dt) {
                    o[dt][0] *= c0;
                    o[dt][1] *= c0;
                    o[dt][2] *= c1;
                    o[dt][3] *= c1;
                }
            }
            // O += P V per piece: matrices (tokens 0-7 | 8-15) x units (u,
            // u+1), transposed; each register holds a token pair (2c, 2c+1)
            // x a dim pair (2g, 2g+1) of its unit; a byte permute regroups
            // it into (dim 2g: both tokens) and (dim 2g+1: both tokens)
            {
                const int mi = lane >> 3;
                const int r = (mi & 1) * 8 + (lane & 7);
#pragma unroll
                for (int p = 0; p < PIECES; ++p)
#pragma unroll
                    for (int up = 0; up < 4; ++up) {
                        const int u = up * 2 + (mi >> 1);
                        uint32_t r0, r1, r2, r3;
                        ldsm_x4_t(vb + p * kChunk * D + sw128(r, u), r0, r1, r2, r3);
                        const int u0 = up * 2, u1 = up * 2 + 1;
                        if constexpr (INT8) {
                            // even codes of a word: dim 2g, odd codes: dim 2g+1
                            uint32_t e0, o0, e1, o1, e2, o2, e3, o3;
                            int8x4_to_f16x2(r0, e0, o0);
                            int8x4_to_f16x2(r1, e1, o1);
                            int8x4_to_f16x2(r2, e2, o2);
                            int8x4_to_f16x2(r3, e3, o3);
                            mma_f16_16816(o[2 * u0], pa[p], e0, e1);
                            mma_f16_16816(o[2 * u0 + 1], pa[p], o0, o1);
                            mma_f16_16816(o[2 * u1], pa[p], e2, e3);
                            mma_f16_16816(o[2 * u1 + 1], pa[p], o2, o3);
                            continue;
                        }
                        const uint32_t a0 = __byte_perm(r0, 0, 0x3120);
                        const uint32_t a1 = __byte_perm(r1, 0, 0x3120);
                        const uint32_t b0 = __byte_perm(r2, 0, 0x3120);
                        const uint32_t b1 = __byte_perm(r3, 0, 0x3120);
                        uint32_t la0, ha0, la1, ha1, lb0, hb0, lb1, hb1;
                        e4m3x4_to_f16x2_hw(a0, la0, ha0);
                        e4m3x4_to_f16x2_hw(a1, la1, ha1);
                        e4m3x4_to_f16x2_hw(b0, lb0, hb0);
                        e4m3x4_to_f16x2_hw(b1, lb1, hb1);
                        mma_f16_16816(o[2 * u0], pa[p], la0, la1);
                        mma_f16_16816(o[2 * u0 + 1], pa[p], ha0, ha1);
                        mma_f16_16816(o[2 * u1], pa[p], lb0, lb1);
                        mma_f16_16816(o[2 * u1 + 1], pa[p], hb0, hb1);
                    }
            }
        }
        __syncwarp();
        if (lane == 0 && i + NS < my_n) {
            fence_proxy_async_smem();
            issue(i + NS);
        }
    }
    if (failed) {
        flag_error(PA_ERR_TIMEOUT);
        const int issued = min(my_n, done + NS);
        for (int i = done; i < issued; ++i)
            if (!mbar_wait(bar0 + (i % NS) * 8, (i / NS) & 1, a.timeout_ns)) break;
    }

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    __syncthreads();
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
    // virtual tile vt = 2u + p, column n = 2*tig + j <-> dim 16u + 2n + p
#pragma unroll
    for (int vt = 0; vt < 16; ++vt) {
        const int u = vt >> 1, p = vt & 1;
        const int d0 = 16 * u + 4 * tig + p, d1 = d0 + 2;
        red_o[(warp * HT + g) * OS + d0] = o[vt][0];
        red_o[(warp * HT + g) * OS + d1] = o[vt][1];
        red_o[(warp * HT + g + 8) * OS + d0] = o[vt][2];
        red_o[(warp * HT + g + 8) * OS + d1] = o[vt][3];
    }
    __syncthreads();
    decode_epilogue<D, NW, HT, __nv_bfloat16>(a, red_o, red_m, red_l, b, h0, nh, s, n_splits, vsc);
}

// E4M3 append: each thread turns 16 elements of a new token's K (and V) row
// into 16 codes: the fp32 quotient x / scale[h] (IEEE division) rounded to
// the nearest E4M3 value, ties to even, saturating at +-448.
struct ReshapeFp8Args {
    const void *key;
    const void *value;
    uint4 *k_cache;
    uint4 *v_cache;
    const int64_t *slot_mapping;
    const float *k_scale;
    const float *v_scale;
    long long num_tokens;
    int vecs_per_token;  // num_kv_heads * head_dim / 16 (16 elements per vector)
    int row_shift;       // log2(head_dim / 16)
    int bs_shift;        // log2(block_size)
    int num_kv_heads;
    long long num_slots;
    int bf16_in;
};

__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(r)
        : "f"(lo), "f"(hi));
    return r;
}

__global__ void __launch_bounds__(kScatterThreads)
    reshape_and_cache_e4m3_kernel(const __grid_constant__ ReshapeFp8Args a) {
    // blockIdx.y walks the tokens, blockIdx.x/threadIdx.x the 16-element
    // vectors of a token (no integer division: the sizes are powers of two)
    const int r = blockIdx.x * kScatterThreads + threadIdx.x;
    if (r >= a.vecs_per_token) return;
    const int h = r >> a.row_shift;
    const int c = r & ((1 << a.row_shift) - 1);
    for (long long t = blockIdx.y; t < a.num_tokens; t += gridDim.y) {
        const long long i = t * a.vecs_per_token + r;
        const long long slot = __ldg(a.slot_mapping + t);
        if (slot < 0) continue;
        if (slot >= a.num_slots) {
            flag_error(PA_ERR_BAD_TABLE);
            continue;
        }
        const float ks = __ldg(a.k_scale + h), vs = __ldg(a.v_scale + h);
        float xk[16], xv[16];
        if (a.bf16_in) {
            const uint4 *k4 = reinterpret_cast<const uint4 *>(a.key) + 2 * i;
            const uint4 *v4 = reinterpret_cast<const uint4 *>(a.value) + 2 * i;
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                const uint4 kk = __ldg(k4 + w), vv = __ldg(v4 + w);
                const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xk[8 * w + 2 * e] = bf16_lo(kw[e]);
                    xk[8 * w + 2 * e + 1] = bf16_hi(kw[e]);
                    xv[8 * w + 2 * e] = bf16_lo(vw[e]);
                    xv[8 * w + 2 * e + 1] = bf16_hi(vw[e]);
                }
            }
        } else {
            const float4 *k4 = reinterpret_cast<const float4 *>(a.key) + 4 * i;
            const float4 *v4 = reinterpret_cast<const float4 *>(a.value) + 4 * i;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float4 kk = __ldg(k4 + w), vv = __ldg(v4 + w);
                xk[4 * w] = kk.x; xk[4 * w + 1] = kk.y; xk[4 * w + 2] = kk.z; xk[4 * w + 3] = kk.w;
                xv[4 * w] = vv.x; xv[4 * w + 1] = vv.y; xv[4 * w + 2] = vv.z; xv[4 * w + 3] = vv.w;
            }
        }
        uint32_t kc[4], vc[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const uint32_t k01 = e4m3x2_from_f32(__fdiv_rn(xk[4 * w], ks), __fdiv_rn(xk[4 * w + 1], ks));
            const uint32_t k23 =
                e4m3x2_from_f32(__fdiv_rn(xk[4 * w + 2], ks), __fdiv_rn(xk[4 * w + 3], ks));
            const uint32_t v01 = e4m3x2_from_f32(__fdiv_rn(xv[4 * w], vs), __fdiv_rn(xv[4 * w + 1], vs));
            const uint32_t v23 =
                e4m3x2_from_f32(__fdiv_rn(xv[4 * w + 2], vs), __fdiv_rn(xv[4 * w + 3], vs));
            kc[w] = k01 | (k23 << 16);
            vc[w] = v01 | (v23 << 16);
        }
        const long long block = slot >> a.bs_shift;
        const long long offset = slot & ((1LL << a.bs_shift) - 1);
        const long long dst =
            (((block * a.num_kv_heads + h) << a.bs_shift) + offset) * (1LL << a.row_shift) + c;
        a.k_cache[dst] = make_uint4(kc[0], kc[1], kc[2], kc[3]);
        a.v_cache[dst] = make_uint4(vc[0], vc[1], vc[2], vc[3]);
    }
}

// INT8 append: as the E4M3 append, each code the nearest integer of the
// fp32 quotient x / scale[h] (IEEE division; ties to even by the
// round-to-nearest-even conversion, which also turns NaN into 0), saturated
// to [-127, 127].
__device__ __forceinline__ uint32_t int8x4_from_f32(float x0, float x1, float x2, float x3) {
    auto one = [](float x) -> uint32_t {
        const int r = min(max(__float2int_rn(x), -127), 127);
        return (uint32_t)(r & 0xff);
    };
    return one(x0) | (one(x1) << 8) | (one(x2) << 16) | (one(x3) << 24);
}

__global__ void __launch_bounds__(kScatterThreads)
    reshape_and_cache_int8_kernel(const __grid_constant__ ReshapeFp8Args a) {
    // blockIdx.y walks the tokens, blockIdx.x/threadIdx.x the 16-element
    // vectors of a token (no integer division: the sizes are powers of two)
    const int r = blockIdx.x * kScatterThreads + threadIdx.x;
    if (r >= a.vecs_per_token) return;
    const int h = r >> a.row_shift;
    const int c = r & ((1 << a.row_shift) - 1);
    for (long long t = blockIdx.y; t < a.num_tokens; t += gridDim.y) {
        const long long i = t * a.vecs_per_token + r;
        const long long slot = __ldg(a.slot_mapping + t);
        if (slot < 0) continue;
        if (slot >= a.num_slots) {
            flag_error(PA_ERR_BAD_TABLE);
            continue;
        }
        const float ks = __ldg(a.k_scale + h), vs = __ldg(a.v_scale + h);
        float xk[16], xv[16];
        if (a.bf16_in) {
            const uint4 *k4 = reinterpret_cast<const uint4 *>(a.key) + 2 * i;
            const uint4 *v4 = reinterpret_cast<const uint4 *>(a.value) + 2 * i;
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                const uint4 kk = __ldg(k4 + w), vv = __ldg(v4 + w);
                const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xk[8 * w + 2 * e] = bf16_lo(kw[e]);
                    xk[8 * w + 2 * e + 1] = bf16_hi(kw[e]);
                    xv[8 * w + 2 * e] = bf16_lo(vw[e]);
                    xv[8 * w + 2 * e + 1] = bf16_hi(vw[e]);
                }
            }
        } else {
            const float4 *k4 = reinterpret_cast<const float4 *>(a.key) + 4 * i;
            const float4 *v4 = reinterpret_cast<const float4 *>(a.value) + 4 * i;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float4 kk = __ldg(k4 + w), vv = __ldg(v4 + w);
                xk[4 * w] = kk.x; xk[4 * w + 1] = kk.y; xk[4 * w + 2] = kk.z; xk[4 * w + 3] = kk.w;
                xv[4 * w] = vv.x; xv[4 * w + 1] = vv.y; xv[4 * w + 2] = vv.z; xv[4 * w + 3] = vv.w;
            }
        }
        uint32_t kc[4], vc[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            kc[w] = int8x4_from_f32(__fdiv_rn(xk[4 * w], ks), __fdiv_rn(xk[4 * w + 1], ks),
                                    __fdiv_rn(xk[4 * w + 2], ks), __fdiv_rn(xk[4 * w + 3], ks));
            vc[w] = int8x4_from_f32(__fdiv_rn(xv[4 * w], vs), __fdiv_rn(xv[4 * w + 1], vs),
                                    __fdiv_rn(xv[4 * w + 2], vs), __fdiv_rn(xv[4 * w + 3], vs));
        }
        const long long block = slot >> a.bs_shift;
        const long long offset = slot & ((1LL << a.bs_shift) - 1);
        const long long dst =
            (((block * a.num_kv_heads + h) << a.bs_shift) + offset) * (1LL << a.row_shift) + c;
        a.k_cache[dst] = make_uint4(kc[0], kc[1], kc[2], kc[3]);
        a.v_cache[dst] = make_uint4(vc[0], vc[1], vc[2], vc[3]);
    }
}

}  // namespace pa
