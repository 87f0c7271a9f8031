// prefill.cuh -- chunked prefill over the paged cache on 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// What is computed (page "vLLM框架是怎么做推理加速的", section 3, Chunked
// Prefill): a chunk of C prompt tokens, whose K/V are already appended to the
// cache, attends over everything cached before it plus itself, causally
// (page "LLM推理优化", section 2.3, causal=True): query i of the chunk sits at
// position cached + i and sees keys 0..cached+i. K/V pages are reached through
// the chunk's block table (page "字节跳动 AI Infra (2)", question
// "vLLM与PagedAttention的原理"), and the softmax is computed tile by tile with
// a running max and sum (page "LLM推理优化", section 2.1).
//
// With a sliding window of W positions (page "LLM推理优化", section 2.3 on
// attention masks, read as a band), query i sees keys cached+i-W+1 ..
// cached+i only; key tiles wholly before a query tile's band are neither
// loaded nor multiplied.
//
// Work item = two 128-row query tiles (the tcgen05 M) of one chunk sharing
// every K/V tile: when the query heads of a KV head come in pairs, the same
// 128 rows of two query heads of that KV head (both tiles then need the same
// key tiles and stay interleaved to the end); otherwise 256 consecutive rows
// of one query head (the second tile needs one key tile more, its diagonal).
// Keys are processed in tiles of 128. The kernel is persistent: one CTA per
// SM works through its share of the items (see prefill_tc_kernel), and
// across items the K/V rings and barrier phases carry on. Twelve warps:
//   warp 8   TMA: an item's Q tiles once the previous item's last S has read
//            the Q buffers, then each key tile's K and V as 16-token page
//            pieces (128-byte swizzle) gathered through the block table, one
//            piece per lane (block ids read one key tile ahead), into
//            two-stage K and V rings with full/free barriers.
//   warp 9   MMA (one lane) and the tensor-memory allocation: S_x = Q_x K^T
//            (8 x 128x128x16, both operands K-major in shared memory) into
//            tensor-memory columns [128x, 128x+128); O_x += P_x V with P_x
//            read from tensor memory (bf16, over S_x's first 64 columns) and
//            V MN-major in shared memory, into columns [256+128x, ...).
//            After P_x.V_j it issues S_x for tile j+1 (the tensor core runs
//            one thread's operations in order), so one query tile's softmax
//            overlaps the other tile's multiplications; the next item's
//            first S follows the current item's last P.V.
//   warps 0-3 / 4-7   softmax of query tile 0 / 1: thread r owns row r
//            (tensor-memory lane r): row max, exp2, the running sum, bf16 P
//            written back over the consumed S columns; O is rescaled in
//            tensor memory only when a row's max grows by more than 2^8 (the
//            result is exact for any reference max as long as O and the sum
//            share it); the epilogue divides by the sum and writes bf16 rows.
//   warps 10-11 idle (they give their registers to the softmax warpgroups).
// All waits are bounded; a wait that runs out records PA_ERR_TIMEOUT, makes
// every role leave its loop, drains outstanding copies and tensor-core work,
// and frees the tensor memory.
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kPfRows = 128;      // query rows per Q tile (the tcgen05 M)
constexpr int kPfQTiles = 2;      // Q tiles per item, sharing every K/V tile
constexpr int kPfKeys = 128;      // keys per K/V tile
constexpr int kPfStages = 2;      // K and V ring depth
constexpr int kPfThreads = 384;   // 2 softmax warpgroups + a control warpgroup
// Register split (setmaxnreg): the control warpgroup (TMA warp, MMA warp and
// two idle warps) gives registers to the two softmax warpgroups, which hold
// a full 128-column score row per thread. The shares must sum to at most the
// launch allocation (384 threads x registers per thread); the host checks
// that against the compiled kernel before launching.
constexpr int kPfCtlRegs = 56;
constexpr int kPfSoftmaxRegs = 224;
constexpr int kPfRegsNeeded = 128 * (2 * kPfSoftmaxRegs + kPfCtlRegs);
// A Q, K or V tile: 128 rows of head_dim bf16, as head_dim/64 halves of 128 x
// 128 bytes (one 128-byte swizzle atom wide), each 16 KB.
__host__ __device__ constexpr int pf_tile_bytes(int D) { return kPfRows * D * 2; }
__host__ __device__ constexpr int pf_smem_bytes(int D) {
    return (kPfQTiles + 2 * kPfStages) * pf_tile_bytes(D) + 512;
}

struct PrefillArgs {
    __nv_bfloat16 *out;
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *qsl;
    int n_chunks, total_q, H_q, H_kv, group, bs, NB, MB;
    int window;  // > 0: query at position p sees keys p-window+1 .. p only
    int pair_heads;  // 1: the two query tiles are the same rows of query heads 2x, 2x+1
    int gx, gy;      // items per row tile (query heads or head pairs), row tiles per chunk
    int n_items;     // gx * gy * n_chunks
    int bs_shift;  // log2(bs)
    float scale_log2;
    unsigned long long timeout_ns;
};

// ------------------------------------------------------------ tcgen05 PTX
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` once every tcgen05 operation this thread issued so far has
// completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
// A group of MMAs accumulating into one tensor-memory tile, issued from one
// asm block: the operand descriptors advance in place by single adds (start
// address in 16-byte units), so the issuing thread keeps two descriptors
// live instead of one per MMA.
// S = Q K^T over head_dim: NK = head_dim / 16 k-steps, both operands K-major
// SW128; a k-step moves 32 bytes inside a 64-wide half and a half is 16 KB.
// The first k-step overwrites the accumulator.
#define PA_MMA_SS(pred) "tcgen05.mma.cta_group::1.kind::f16 [%2], %0, %1, %3, " pred ";\n\t"
#define PA_MMA_SS_STEP(delta) \
    "add.s64 %0, %0, " delta ";\n\tadd.s64 %1, %1, " delta ";\n\t" PA_MMA_SS("pt")
template <int NK>
__device__ __forceinline__ void mma_ss_group(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc) {
    static_assert(NK == 4 || NK == 8, "head_dim 64 or 128");
    if constexpr (NK == 8) {
        asm volatile("{\n\t.reg .pred pt, pf;\n\t"
                     "setp.eq.b32 pt, %3, %3;\n\tsetp.ne.b32 pf, %3, %3;\n\t" PA_MMA_SS("pf")
                         PA_MMA_SS_STEP("2") PA_MMA_SS_STEP("2") PA_MMA_SS_STEP("2")
                             PA_MMA_SS_STEP("1018") PA_MMA_SS_STEP("2") PA_MMA_SS_STEP("2")
                                 PA_MMA_SS_STEP("2") "}"
                     : "+l"(a), "+l"(b)
                     : "r"(d), "r"(idesc)
                     : "memory");
    } else {
        asm volatile("{\n\t.reg .pred pt, pf;\n\t"
                     "setp.eq.b32 pt, %3, %3;\n\tsetp.ne.b32 pf, %3, %3;\n\t" PA_MMA_SS("pf")
                         PA_MMA_SS_STEP("2") PA_MMA_SS_STEP("2") PA_MMA_SS_STEP("2") "}"
                     : "+l"(a), "+l"(b)
                     : "r"(d), "r"(idesc)
                     : "memory");
    }
}
#undef PA_MMA_SS_STEP
#undef PA_MMA_SS
// O += P V over 128 keys: 8 k-steps of 16 keys, P (A) read from tensor memory
// 8 columns (16 bf16) further per step, V (B) MN-major SW128 2 KB further per
// step. The first k-step accumulates only when acc0 is non-zero.
#define PA_MMA_TS(pred) "tcgen05.mma.cta_group::1.kind::f16 [%2], [%0], %1, %3, " pred ";\n\t"
#define PA_MMA_TS_STEP "add.u32 %0, %0, 8;\n\tadd.s64 %1, %1, 128;\n\t" PA_MMA_TS("pt")
__device__ __forceinline__ void mma_ts_group(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                             uint32_t acc0) {
    asm volatile("{\n\t.reg .pred pt, p0;\n\t"
                 "setp.eq.b32 pt, %3, %3;\n\tsetp.ne.b32 p0, %4, 0;\n\t" PA_MMA_TS("p0")
                     PA_MMA_TS_STEP PA_MMA_TS_STEP PA_MMA_TS_STEP PA_MMA_TS_STEP PA_MMA_TS_STEP
                         PA_MMA_TS_STEP PA_MMA_TS_STEP "}"
                 : "+r"(a), "+l"(b)
                 : "r"(d), "r"(idesc), "r"(acc0)
                 : "memory");
}
#undef PA_MMA_TS_STEP
#undef PA_MMA_TS

#define PA_R32(r)                                                                                 \
    "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),         \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), \
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),           \
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),           \
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// its lane's 32 columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : PA_R32(r)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm100 format: start,
// leading and stride byte offsets in 16-byte units, version 1 at bit 46,
// layout type 2 = SWIZZLE_128B at bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator (bit 4), bf16 A and B
// (bits 7, 10), B MN-major when b_mn (bit 16), N>>3 at bit 17, M>>4 at bit 24.
__host__ __device__ constexpr uint32_t f16_idesc(int M, int N, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct PfBars {
    uint64_t q_full, q_free;
    uint64_t k_full[kPfStages], k_free[kPfStages], v_full[kPfStages], v_free[kPfStages];
    uint64_t s_full[kPfQTiles], p_full[kPfQTiles], o_full[kPfQTiles];
    uint64_t fin;
    uint32_t tmem_base;
    volatile int abort;
};

// Bounded wait shared by all roles: false when the CTA is aborting or the
// bound ran out (which starts the abort). Warp-uniform when `uniform`.
__device__ __forceinline__ bool pf_wait(PfBars *bars, uint64_t *bar, uint32_t parity,
                                        unsigned long long timeout_ns, bool uniform) {
    bool ok = bars->abort == 0 && mbar_wait(smem_u32(bar), parity, timeout_ns);
    if (uniform) ok = __all_sync(0xffffffffu, ok);
    if (!ok && bars->abort == 0) {
        bars->abort = 1;
        flag_error(PA_ERR_TIMEOUT);
    }
    return ok;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One work item: the two 128-row query tiles a CTA works on at a time (see
// the file header) and the key tiles [jmin, jmax) they need. Every role
// decodes the same items in the same order.
struct PfItem {
    int c, q0, C, ctx, cached, chunk_lo;
    int row0, row1, rows0, rows1;  // first row (within the chunk) and row count per tile
    int hq0, hq1, kvh;             // query head per tile, their KV head
    int jlo0, jhi0, jlo1, jhi1, jmin, jmax;
};

// Decode work item `it` (item 0 has the most work: chunks from the last,
// within a chunk row tiles from the last, query heads or head pairs
// fastest). False when the item has no rows or its chunk is malformed
// (recorded when `report`).
template <bool WIN>
__device__ __forceinline__ bool pf_item(const PrefillArgs &a, int it, bool report, PfItem &w) {
    const int hx = it % a.gx;
    const int rest = it / a.gx;
    const int tp = a.gy - 1 - rest % a.gy;
    w.c = a.n_chunks - 1 - rest / a.gy;
    w.q0 = a.qsl[w.c];
    w.C = a.qsl[w.c + 1] - w.q0;
    w.ctx = a.context_lens[w.c];
    if (w.q0 < 0 || w.C < 0 || w.q0 + w.C > a.total_q || w.ctx < w.C ||
        (long long)w.ctx > (long long)a.MB * a.bs) {
        if (report) flag_error(PA_ERR_BAD_TABLE);
        return false;
    }
    // rows past the items' reach (a chunk longer than max_query_len rounded
    // up to the item's rows) would be left unwritten: recorded
    const int item_rows = a.pair_heads ? kPfRows : kPfRows * kPfQTiles;
    if (report && hx == 0 && tp == 0 && w.C > a.gy * item_rows) flag_error(PA_ERR_BAD_TABLE);
    w.row0 = tp * item_rows;
    if (w.row0 >= w.C) return false;
    w.row1 = a.pair_heads ? w.row0 : w.row0 + kPfRows;
    w.rows0 = min(kPfRows, w.C - w.row0);
    w.rows1 = max(0, min(kPfRows, w.C - w.row1));
    w.hq0 = a.pair_heads ? 2 * hx : hx;
    w.hq1 = a.pair_heads ? w.hq0 + 1 : w.hq0;
    w.kvh = w.hq0 / a.group;
    w.cached = w.ctx - w.C;
    // key tiles of each query tile: up to its last row's position, from its
    // first row's band start. Key positions below the chunk's smallest band
    // start (chunk_lo) are never needed: their blocks may have been freed.
    const int W = WIN ? a.window : 0;
    w.chunk_lo = W > 0 ? max(0, w.cached - W + 1) : 0;
    const int pf0 = w.cached + w.row0, pf1 = w.cached + w.row1;  // first positions
    w.jlo0 = (W > 0 ? max(0, pf0 - W + 1) : 0) / kPfKeys;
    w.jlo1 = (W > 0 ? max(0, pf1 - W + 1) : 0) / kPfKeys;
    w.jhi0 = (pf0 + w.rows0 - 1) / kPfKeys + 1;
    w.jhi1 = w.rows1 > 0 ? (pf1 + w.rows1 - 1) / kPfKeys + 1 : w.jlo1;
    w.jmin = w.jlo0;
    w.jmax = max(w.jhi0, w.jhi1);
    return true;
}

// WIN: the sliding-window build; without it the band logic folds away at
// compile time and the causal kernel keeps its tighter code.
// D: head_dim, 64 or 128 (one or two 64-wide halves per row; the S tiles
// and the P.V accumulators keep their TMEM columns, O using the first D).
//
// Persistent: one CTA per SM takes items r*G + b (G CTAs, b its index; in
// odd rounds r the order is reversed, so that the longest items spread over
// all CTAs). Across items the K/V rings, the S/P phases and the Q tiles carry
// on: the next item's Q loads once the last S of the current one has read
// Q (q_free), and its first S is issued right behind the current item's
// last P.V — so the next item's loads and first S overlap the current
// item's last key tile and epilogue. The next item's first P.V into an O
// needs no barrier of its own: it waits for that item's first P, which the
// softmax warps produce only after their epilogue has read the O out.
template <int D, bool WIN>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_tc_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    constexpr int TB = pf_tile_bytes(D);
    constexpr int HALVES = D / 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(smem);            // Q tile x at sQ + x*TB
    const uint32_t sK = sQ + kPfQTiles * TB;       // K stage st at sK + st*TB
    const uint32_t sV = sK + kPfStages * TB;       // V stage st at sV + st*TB
    PfBars *bars = reinterpret_cast<PfBars *>(smem + (kPfQTiles + 2 * kPfStages) * TB);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's r-th item (or past the last)
    auto item_of = [&](int r) {
        const int G = (int)gridDim.x, b = (int)blockIdx.x;
        return r * G + ((r & 1) ? G - 1 - b : b);
    };

    if (warp == 8 && lane == 0) {
        mbar_init(smem_u32(&bars->q_full), 1);
        mbar_init(smem_u32(&bars->q_free), 1);
        for (int st = 0; st < kPfStages; ++st) {
            mbar_init(smem_u32(&bars->k_full[st]), 1);
            mbar_init(smem_u32(&bars->k_free[st]), 1);
            mbar_init(smem_u32(&bars->v_full[st]), 1);
            mbar_init(smem_u32(&bars->v_free[st]), 1);
        }
        for (int x = 0; x < kPfQTiles; ++x) {
            mbar_init(smem_u32(&bars->s_full[x]), 1);
            mbar_init(smem_u32(&bars->p_full[x]), 4);  // one arrive per softmax warp
            mbar_init(smem_u32(&bars->o_full[x]), 1);
        }
        mbar_init(smem_u32(&bars->fin), 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(&bars->tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // tensor memory: S/P of Q tile x in columns [128x, 128x+128) (P, bf16
    // pairs, over the first 64); O of Q tile x in [256+128x, 256+128x+128)
    const uint32_t tmem = bars->tmem_base;

    if (warp >= 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfCtlRegs));
      if (warp == 8) {
        // ------------------------------------------------------------ TMA
        // One box per lane: a thread issuing tensor copies back to back is
        // slow (each issue takes a while to be accepted), so the 16 boxes
        // of a K or V tile (8 pieces of 16 tokens x 2 halves of 64 dims)
        // go out from 16 lanes at once. Each lane reads its piece's block id
        // from the chunk's table row one key tile ahead, so that the read
        // overlaps the wait for a free stage. Lane 0 arms the barrier first
        // with the exact byte count of the pieces that exist.
        const int s16 = lane / HALVES, half = lane % HALVES;
        int g = 0, k_issued = 0, v_issued = 0, qn = 0;
        bool ok = true;
        for (int r = 0; ok; ++r) {
            const int it = item_of(r);
            if (it >= a.n_items) break;
            PfItem w;
            if (!pf_item<WIN>(a, it, lane == 0, w)) continue;
            const int32_t *trow = a.block_tables + (size_t)w.c * a.MB;
            // the table entry of this lane's piece of key tile j (-1: no
            // piece); read ahead of its use and checked only there, so that
            // waiting for the read never holds up the copies before it
            auto piece_raw = [&](int j) {
                const int key = j * kPfKeys + s16 * 16;
                return lane < 8 * HALVES && key < w.ctx && (!WIN || key + 15 >= w.chunk_lo)
                           ? __ldg(trow + (key >> a.bs_shift))
                           : -1;
            };
            auto checked = [&](int raw, int j) {  // -1 for no piece or a bad id (recorded)
                const int key = j * kPfKeys + s16 * 16;
                const bool piece =
                    lane < 8 * HALVES && key < w.ctx && (!WIN || key + 15 >= w.chunk_lo);
                if (piece && (raw < 0 || raw >= a.NB)) {
                    flag_error(PA_ERR_BAD_TABLE);
                    return -1;
                }
                return piece ? raw : -1;
            };
            auto issue = [&](uint32_t dst, const CUtensorMap *map, uint64_t *bar, int j, int id) {
                const int n = __popc(__ballot_sync(0xffffffffu, id >= 0));
                if (lane == 0) mbar_arrive_expect_tx(smem_u32(bar), n * 2048);
                __syncwarp();
                if (id >= 0)
                    tma_load_4d(dst + half * 16384 + s16 * 2048, map, smem_u32(bar), half * 64,
                                (j * kPfKeys + s16 * 16) & (a.bs - 1), w.kvh, id);
            };
            int raw = piece_raw(w.jmin);
            // the Q tiles, once the previous item's last S has read them
            if (qn > 0 && !pf_wait(bars, &bars->q_free, (qn - 1) & 1, a.timeout_ns, true)) {
                ok = false;
                break;
            }
            const int nq = w.rows1 > 0 ? 2 : 1;  // Q tiles with rows
            if (lane == 0) mbar_arrive_expect_tx(smem_u32(&bars->q_full), nq * TB);
            __syncwarp();
            if (lane < HALVES * nq) {
                const int x = lane / HALVES, hf = lane % HALVES;
                tma_load_3d(sQ + x * TB + hf * 16384, &tmq, smem_u32(&bars->q_full), hf * 64,
                            x == 0 ? w.hq0 : w.hq1, w.q0 + (x == 0 ? w.row0 : w.row1));
            }
            ++qn;
            int id = checked(raw, w.jmin);
            for (int j = w.jmin; j < w.jmax; ++j, ++g) {
                const int nraw = j + 1 < w.jmax ? piece_raw(j + 1) : -1;
                const int st = g % kPfStages;
                const uint32_t use = g / kPfStages;
                if (use > 0 &&
                    !pf_wait(bars, &bars->k_free[st], (use - 1) & 1, a.timeout_ns, true)) {
                    ok = false;
                    break;
                }
                issue(sK + st * TB, &tmk, &bars->k_full[st], j, id);
                k_issued = g + 1;
                if (use > 0 &&
                    !pf_wait(bars, &bars->v_free[st], (use - 1) & 1, a.timeout_ns, true)) {
                    ok = false;
                    break;
                }
                issue(sV + st * TB, &tmv, &bars->v_full[st], j, id);
                v_issued = g + 1;
                if (j + 1 < w.jmax) id = checked(nraw, j + 1);
            }
        }
        if (bars->abort && lane == 0) {  // let copies already in flight land
            if (qn > 0) mbar_wait(smem_u32(&bars->q_full), (qn - 1) & 1, a.timeout_ns);
            for (int t = max(0, k_issued - kPfStages); t < k_issued; ++t)
                mbar_wait(smem_u32(&bars->k_full[t % kPfStages]), (t / kPfStages) & 1,
                          a.timeout_ns);
            for (int t = max(0, v_issued - kPfStages); t < v_issued; ++t)
                mbar_wait(smem_u32(&bars->v_full[t % kPfStages]), (t / kPfStages) & 1,
                          a.timeout_ns);
        }
      } else if (warp == 9) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t kIdQK = f16_idesc(128, 128, false);
            constexpr uint32_t kIdPV = f16_idesc(128, D, true);
            int g = 0, qn = 0;
            int pc[kPfQTiles] = {0, 0};  // P tiles consumed per query tile
            bool ok = true;
            for (int r = 0; ok; ++r) {
                const int it = item_of(r);
                if (it >= a.n_items) break;
                PfItem w;
                if (!pf_item<WIN>(a, it, false, w)) continue;
                auto jlo = [&](int x) { return x == 0 ? w.jlo0 : w.jlo1; };
                auto jhi = [&](int x) { return x == 0 ? w.jhi0 : w.jhi1; };
                auto active = [&](int x, int j) { return j >= jlo(x) && j < jhi(x); };
                auto wait_k = [&](int t) {  // K/V tile t (counted over items) landed
                    return pf_wait(bars, &bars->k_full[t % kPfStages], (t / kPfStages) & 1,
                                   a.timeout_ns, false);
                };
                auto wait_v = [&](int t) {
                    return pf_wait(bars, &bars->v_full[t % kPfStages], (t / kPfStages) & 1,
                                   a.timeout_ns, false);
                };
                // S_x = Q_x K^T of the K/V tile counted t; K has landed
                auto issue_s = [&](int x, int t) {
                    tc_fence_after();
                    mma_ss_group<D / 16>(tmem + x * 128, sw128_desc(sQ + x * TB, 16, 1024),
                                         sw128_desc(sK + (t % kPfStages) * TB, 16, 1024), kIdQK);
                    tc_commit(smem_u32(&bars->s_full[x]));
                };
                ok = pf_wait(bars, &bars->q_full, qn & 1, a.timeout_ns, false) && wait_k(g);
                ++qn;
                if (!ok) break;
                // S of every Q tile that starts at the first K tile, then per
                // K/V tile j: P.V of each Q tile that uses it and, behind it
                // in issue order (the tensor core runs one thread's
                // operations in order, so S may reuse the P columns), S of
                // each Q tile that uses tile j+1
#pragma unroll
                for (int x = 0; x < kPfQTiles; ++x)
                    if (active(x, w.jmin)) issue_s(x, g);
                tc_commit(smem_u32(&bars->k_free[g % kPfStages]));
                if (w.jmax - w.jmin == 1) tc_commit(smem_u32(&bars->q_free));
                for (int j = w.jmin; ok && j < w.jmax; ++j) {
                    const int t = g + (j - w.jmin);
                    // the K and V tiles land long before a softmax hands
                    // over its P: waiting for them first keeps their waits
                    // off the path from P to its multiplication
                    const bool s_next = active(0, j + 1) || active(1, j + 1);
                    ok = wait_v(t) && (!s_next || wait_k(t + 1));
#pragma unroll
                    for (int x = 0; x < kPfQTiles; ++x) {
                        if (ok && active(x, j)) {
                            ok = pf_wait(bars, &bars->p_full[x], pc[x] & 1, a.timeout_ns, false);
                            ++pc[x];
                            if (ok) {
                                tc_fence_after();
                                mma_ts_group(tmem + 256 + x * 128, tmem + x * 128,
                                             sw128_desc(sV + (t % kPfStages) * TB, 16384, 1024),
                                             kIdPV, j > jlo(x) ? 1u : 0u);
                                // the epilogue waits for the item's last P.V
                                // (a rescale of O waits for the next S,
                                // committed behind the P.V before it)
                                if (j == jhi(x) - 1) tc_commit(smem_u32(&bars->o_full[x]));
                            }
                        }
                        if (ok && active(x, j + 1)) issue_s(x, t + 1);
                    }
                    if (!ok) break;
                    // the item's last S reads Q: the next item's Q may load
                    // once it completes
                    if (j + 1 == w.jmax - 1) tc_commit(smem_u32(&bars->q_free));
                    if (j + 1 < w.jmax) tc_commit(smem_u32(&bars->k_free[(t + 1) % kPfStages]));
                    tc_commit(smem_u32(&bars->v_free[t % kPfStages]));
                }
                g += w.jmax - w.jmin;
            }
            // every tensor-core operation issued above completes before teardown
            tc_commit(smem_u32(&bars->fin));
            mbar_wait(smem_u32(&bars->fin), 0, a.timeout_ns);
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPfSoftmaxRegs));
        // -------------------------------------------------------- softmax
        const int x = warp >> 2;                      // Q tile of this warpgroup
        const int r = threadIdx.x & 127;              // row of the tile == lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + x * 128 + lane_off;
        const uint32_t tO = tmem + 256 + x * 128 + lane_off;
        const float sl2 = a.scale_log2;
        int g = 0;   // K/V tiles of the items before this one
        int sc = 0;  // S tiles of this query tile consumed
        int oc = 0;  // items whose O this query tile wrote out
        bool ok = true;
        for (int rr = 0; ok; ++rr) {
            const int it = item_of(rr);
            if (it >= a.n_items) break;
            PfItem w;
            if (!pf_item<WIN>(a, it, false, w)) continue;
            const int gbase = g;
            g += w.jmax - w.jmin;
            const int j0 = x == 0 ? w.jlo0 : w.jlo1, j1 = x == 0 ? w.jhi0 : w.jhi1;
            if (j1 <= j0) continue;  // a second tile without rows
            const int W = WIN ? a.window : 0;
            const int xrow0 = x == 0 ? w.row0 : w.row1;  // first row of the tile
            const int i = xrow0 + r;                     // query index in the chunk
            const bool row_valid = i < w.C;
            const int pos = w.cached + min(i, w.C - 1);  // keys <= pos are visible
            const int lo = W > 0 ? pos - W + 1 : 0;      // ... and keys >= lo
            const int pos_first = w.cached + xrow0;      // smallest pos of the tile
            const int lo_last = W > 0 ? pos_first + (x == 0 ? w.rows0 : w.rows1) - W : 0;
            // the warpgroup that first consumes the last K/V tile clears its
            // rows past the context; query tile 0, always the first consumer
            // of the first K/V tile, clears its rows before chunk_lo
            const bool zeroes_tail = j1 == w.jmax && (x == 0 || w.jhi0 < w.jmax);
            float m = -INFINITY, l = 0.f;
            for (int j = j0; j < j1; ++j) {
                if (!pf_wait(bars, &bars->s_full[x], sc & 1, a.timeout_ns, true)) {
                    ok = false;
                    break;
                }
                ++sc;
                tc_fence_after();
                uint32_t sv[128];
                tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
                tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
                tmem_ld_wait();
                const int key0 = j * kPfKeys;
                // some key masked for some row: past the first row's
                // position, or before the last row's band start
                const bool diag = key0 + kPfKeys - 1 > pos_first || (WIN && key0 < lo_last);
                if (diag) {
#pragma unroll
                    for (int e = 0; e < 128; ++e)
                        if (key0 + e > pos || (WIN && key0 + e < lo))
                            sv[e] = __float_as_uint(sl2 >= 0.f ? -INFINITY : INFINITY);
                }
                // the row's largest scaled score (raw max, or raw min for a
                // negative scale)
                float ext;
                {
                    // eight independent running extrema, then a tree
                    float tt[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) tt[u] = __uint_as_float(sv[u]);
                    if (sl2 >= 0.f) {
#pragma unroll
                        for (int e = 8; e < 128; ++e)
                            tt[e & 7] = fmaxf(tt[e & 7], __uint_as_float(sv[e]));
#pragma unroll
                        for (int v = 4; v > 0; v >>= 1)
#pragma unroll
                            for (int u = 0; u < v; ++u) tt[u] = fmaxf(tt[u], tt[u + v]);
                    } else {
#pragma unroll
                        for (int e = 8; e < 128; ++e)
                            tt[e & 7] = fminf(tt[e & 7], __uint_as_float(sv[e]));
#pragma unroll
                        for (int v = 4; v > 0; v >>= 1)
#pragma unroll
                            for (int u = 0; u < v; ++u) tt[u] = fminf(tt[u], tt[u + v]);
                    }
                    ext = tt[0];
                }
                const float m_tile = isinf(ext) ? -INFINITY : ext * sl2;
                const float m_new = fmaxf(m, m_tile);
                if (j == j0) {
                    m = m_new;
                } else if (__any_sync(0xffffffffu, m_new > m + 8.f)) {
                    // re-reference O and the sum to the new max
                    const float corr = ex2_approx(m - m_new);
                    l *= corr;
                    m = m_new;
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t v[32];
                        tmem_ld32(tO + cc * 32, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            v[e] = __float_as_uint(__uint_as_float(v[e]) * corr);
                        tmem_st32(tO + cc * 32, v);
                    }
                }
                const float neg_m = -m;
                uint32_t pk[64];
                float ls[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
                if (diag) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const int k0 = key0 + 2 * e;
                        const float p0 = k0 <= pos && (!WIN || k0 >= lo)
                                             ? ex2_approx(fmaf(__uint_as_float(sv[2 * e]), sl2, neg_m))
                                             : 0.f;
                        const float p1 =
                            k0 + 1 <= pos && (!WIN || k0 + 1 >= lo)
                                ? ex2_approx(fmaf(__uint_as_float(sv[2 * e + 1]), sl2, neg_m))
                                : 0.f;
                        ls[e & 3] += p0 + p1;
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                } else {
                    // scale and shift as one packed f32x2 FMA per key pair,
                    // the row sum as packed adds: fewer instructions on the
                    // path between a tile's scores and its P.V
                    const float2 sl2v = make_float2(sl2, sl2), nmv = make_float2(neg_m, neg_m);
                    float2 acc2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const float2 tv = __ffma2_rn(make_float2(__uint_as_float(sv[2 * e]),
                                                                 __uint_as_float(sv[2 * e + 1])),
                                                     sl2v, nmv);
                        const float p0 = ex2_approx(tv.x), p1 = ex2_approx(tv.y);
                        acc2[e & 1] = __fadd2_rn(acc2[e & 1], make_float2(p0, p1));
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                    ls[0] = acc2[0].x;
                    ls[1] = acc2[0].y;
                    ls[2] = acc2[1].x;
                    ls[3] = acc2[1].y;
                }
                l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
                tmem_st32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
                tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
                tmem_st_wait();
                // V rows past the context, or before chunk_lo, hold stale or
                // unloaded data: zero them so that P = 0 cannot meet a NaN
                const int z0 = WIN && x == 0 && j == w.jmin ? max(0, w.chunk_lo - key0) : 0;
                const int z1 = zeroes_tail && j == j1 - 1 ? min(kPfKeys, w.ctx - key0) : kPfKeys;
                if (z0 > 0 || z1 < kPfKeys) {
                    const int t = gbase + (j - w.jmin);
                    if (!pf_wait(bars, &bars->v_full[t % kPfStages], (t / kPfStages) & 1,
                                 a.timeout_ns, true)) {
                        ok = false;
                        break;
                    }
                    const uint32_t vb = sV + (t % kPfStages) * TB;
                    const int nz = z0 + (kPfKeys - z1);  // rows [0, z0) and [z1, 128)
                    for (int e = r; e < nz * (D / 8); e += 128) {  // 16-byte units of a row
                        const int zr = e / (D / 8), u = e % (D / 8);
                        const int row = zr < z0 ? zr : z1 + (zr - z0);
                        const uint32_t addr = vb + (u / 8) * 16384 + row * 128 + (u % 8) * 16;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0)
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                }
                // the warp's P stores (and V zeroing) are complete and
                // fenced: one arrive per warp (128 arrivals on one barrier
                // serialise)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[x]));
            }
            if (!ok || !pf_wait(bars, &bars->o_full[x], oc & 1, a.timeout_ns, true)) {
                ok = false;
                break;
            }
            ++oc;
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst =
                a.out + ((size_t)(w.q0 + i) * a.H_q + (x == 0 ? w.hq0 : w.hq1)) * D;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t v[32];
                tmem_ld32(tO + cc * 32, v);
                tmem_ld_wait();
                uint32_t o[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    o[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv,
                                       __uint_as_float(v[2 * e + 1]) * inv);
                if (row_valid) {
                    // whole 32-byte sectors: a thread's row is 8 KB away from
                    // its neighbours', so 16-byte stores would each write half
                    // a sector, twice as many store instructions
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        asm volatile(
                            "st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                                dst + cc * 32 + e * 16),
                            "r"(o[8 * e]), "r"(o[8 * e + 1]), "r"(o[8 * e + 2]), "r"(o[8 * e + 3]),
                            "r"(o[8 * e + 4]), "r"(o[8 * e + 5]), "r"(o[8 * e + 6]),
                            "r"(o[8 * e + 7])
                            : "memory");
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace pa
