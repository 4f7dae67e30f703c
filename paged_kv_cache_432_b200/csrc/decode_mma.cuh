// decode_mma.cuh -- paged decode attention, bf16, one warp per work item.
//
// Decoding reads the whole KV cache once per step and does little arithmetic
// per byte: it is bound by memory bandwidth ("vLLM PagedAttention: eine
// Revolution für den Durchsatz bei der LLM-Inferenz", de.news.hada.io, the
// list of advanced features: decoding is the bandwidth-heavy phase).  So the
// design goal is to keep enough bytes in flight from HBM, and to read every
// K/V block once per kv head however many query heads share it.
//
// Structure (persistent kernel, grid = SMs x resident CTAs):
//  * Every warp walks work items (sequence, partition, kv head) of items.cuh.
//    Each warp owns a ring of STAGES shared-memory stages.  A stage holds one
//    16-token block of one kv head: K and V, head_dim <= 128 bf16.  Lane 0 fills
//    a stage with TMA 2-D tile loads (64 x 16 boxes, 128-byte swizzle) and an
//    mbarrier with an expected byte count.  The warp keeps STAGES blocks in
//    flight and refills a stage as soon as it has consumed it, crossing item
//    boundaries without draining.
//  * The physical block id comes from the sequence's block table
//    ("Was ändert PagedAttention an der KV-Speicherzuweisung für LLMs?",
//    slavadubrov.com, introduction): the warp reads 32 consecutive table
//    entries with one coalesced load, and each lane keeps one of them in a
//    register.
//  * The g = Hq/Hkv query heads of the kv head form the M dimension of
//    mma.sync m16n8k16 (bf16 in, fp32 accumulate), padded to 16 rows:
//    S = Q K^T (tokens in N), then P V (head dims in N), in the register
//    layout where the S accumulators become the A operand of P V without a
//    trip through shared memory.  K fragments come from ldmatrix and V
//    fragments from ldmatrix.trans.  Both read the swizzled tiles without bank
//    conflicts.  The tensor cores do this to relieve the fp32 pipe, which
//    could not keep up at g = 8; the kernel stays memory-bound.
//  * Softmax is online, in fp32, in the log2 domain (scale * log2 e folded
//    into the scores); each block updates the running max m and sum l, and
//    rescales the accumulators once.  Tokens past the sequence length are
//    masked with -inf.  The V rows of a partly filled last block are zeroed in
//    shared memory before P V, so stale or NaN slot contents never reach out.
//  * At the end of an item the warp writes either the final row
//    (acc / l, rounded to bf16) when the sequence has one partition, or the
//    partition's (m, l, acc) to the workspace for the log-sum-exp reduction.
//
// Every wait on an mbarrier is bounded: on timeout the warp flags
// PA_DEVERR_TIMEOUT, waits (bounded) for its copies in flight and returns.
#pragma once

#include "items.cuh"

namespace pa {

template <int D, int STAGES, int WARPS>
struct MmaCfg {
    static constexpr int kRegions = D / 64;            // 64-element (128 B) column slabs
    static constexpr int kRegionBytes = 16 * 128;      // 16 token rows x 128 B
    static constexpr int kTileBytes = kRegions * kRegionBytes;  // K (or V) of one block, one head
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kRingBytes = WARPS * STAGES * kStageBytes;
    static constexpr int kBarBytes = WARPS * STAGES * 8;
    static constexpr int kThreads = WARPS * 32;
    static size_t smem_bytes(int seq_count) {
        return 1024 + kRingBytes + kBarBytes + 8 * static_cast<size_t>(seq_count + 1);
    }
};

// Online-softmax update of one row set: x[] are four raw scores (tokens
// tq, tq+1, 8+tq, 9+tq), already masked to -inf where invalid and scaled to
// log2 units.  Returns the rescale factor for the accumulators and packs the
// probabilities as bf16 pairs (lo: tokens tq..tq+1, hi: tokens 8+tq..9+tq).
__device__ __forceinline__ float softmax_update(float& m, float& l, const float (&x)[4],
                                                uint32_t& p_lo, uint32_t& p_hi) {
    float bm = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, 1));
    bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, 2));
    const float mn = fmaxf(m, bm);
    const float mu = mn == -INFINITY ? 0.0f : mn;  // a row with nothing valid yet
    const float alpha = exp2f(m - mu);
    const __nv_bfloat162 a = __floats2bfloat162_rn(exp2f(x[0] - mu), exp2f(x[1] - mu));
    const __nv_bfloat162 b = __floats2bfloat162_rn(exp2f(x[2] - mu), exp2f(x[3] - mu));
    // the denominator sums the same (rounded) weights the numerator uses
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    l = l * alpha + ((fa.x + fa.y) + (fb.x + fb.y));
    m = mn;
    p_lo = bf162_bits(a);
    p_hi = bf162_bits(b);
    return alpha;
}

template <int D, int ROWS, int STAGES, int WARPS, int MIN_CTAS>
__global__ void __launch_bounds__(WARPS * 32, MIN_CTAS)
decode_bf16_mma_kernel(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const DecodeParams P) {
    using Cfg = MmaCfg<D, STAGES, WARPS>;
    constexpr int KSTEPS = D / 16;  // k-steps of Q K^T
    constexpr int NTD = D / 8;      // n-tiles of P V
    constexpr bool HI = ROWS > 8;   // query rows 8..15 in use
    constexpr int AR = HI ? 4 : 2;  // registers per A fragment / per C tile that are held

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = smem + warp * STAGES * Cfg::kStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kRingBytes) + warp * STAGES;
    int32_t* prefix = reinterpret_cast<int32_t*>(smem + Cfg::kRingBytes + Cfg::kBarBytes);
    int32_t* lens = prefix + P.seq_count + 1;

    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < STAGES; ++st) mbar_init(smem_u32(&bars[st]), 1);
        fence_barrier_init();
    }
    // Launched with programmatic stream serialization: the CTAs become
    // resident while the previous kernel (typically the cache write) drains,
    // and wait here until its results are visible.  Nothing above touched
    // global memory.
    grid_dependency_wait();
    allow_dependents();  // the reduction may launch and wait for this grid
    const Schedule sched = make_schedule(P, prefix, lens, WARPS);  // ends with __syncthreads
    zero_empty_sequences<__nv_bfloat16>(P, lens);

    const int32_t my_warp = blockIdx.x * WARPS + warp;
    Cursor pc;  // producer: the piece whose next block is loaded next
    sched.start(pc, my_warp);
    if (!pc.valid) return;
    Cursor cc = pc;  // consumer: the piece being computed

    const uint64_t policy = l2_policy_evict_first();
    const uint32_t ring_u32 = smem_u32(ring);
    const uint32_t bar_u32 = smem_u32(bars);
    const int g = P.group;
    const int Hkv = P.num_kv_heads;
    const CUtensorMap* map_k = &tmap_k;  // grid-constant parameters: address taken in place
    const CUtensorMap* map_v = &tmap_v;

    // ---------------- producer state (warp-uniform except `tbl`)
    int32_t pj = pc.jbeg;
    bool prod_live = true;
    int32_t tbl = 0, tbase = 0;
    bool tbl_fresh = false;  // tbl holds entries of the producer's current piece
    uint32_t oob_mask = 0;   // stages whose block id was outside the pool
    uint32_t issued = 0, consumed = 0;

    auto produce = [&](int stage) {
        if (!tbl_fresh || pj >= tbase + 32) {
            tbase = pj;
            tbl_fresh = true;
            const int32_t jj = tbase + lane;
            tbl = jj < pc.jend
                      ? __ldg(P.block_tables + static_cast<size_t>(pc.s) * P.max_blocks_per_seq + jj)
                      : 0;
        }
        int32_t pb = __shfl_sync(kFullMask, tbl, pj - tbase);
        const bool oob = static_cast<uint32_t>(pb) >= static_cast<uint32_t>(P.num_blocks);
        if (oob) {
            pb = 0;  // load a valid block; the consumer masks all its tokens
            oob_mask |= 1u << stage;
        } else {
            oob_mask &= ~(1u << stage);
        }
        if (lane == 0) {
            if (oob) flag_error(PA_DEVERR_BLOCK_OOB);
            fence_proxy_async_smem();
            const uint32_t bar = bar_u32 + stage * 8;
            mbar_arrive_expect_tx(bar, Cfg::kStageBytes);
            const int32_t row = (pb * Hkv + pc.h) * kBlockTokens;
            const uint32_t kdst = ring_u32 + stage * Cfg::kStageBytes;
#pragma unroll
            for (int r = 0; r < Cfg::kRegions; ++r) {
                tma_load_2d(kdst + r * Cfg::kRegionBytes, map_k, r * 64, row, bar, policy);
                tma_load_2d(kdst + Cfg::kTileBytes + r * Cfg::kRegionBytes, map_v, r * 64, row,
                            bar, policy);
            }
        }
        ++issued;
        if (++pj == pc.jend) {
            sched.next(pc);
            tbl_fresh = false;
            if (pc.valid) pj = pc.jbeg;
            else prod_live = false;
        }
    };

    for (int st = 0; st < STAGES && prod_live; ++st) produce(st);

    // ---------------- consumer
    int32_t cj = cc.jbeg;
    int stage = 0;
    uint32_t phase = 0;

    const int tq = 2 * (lane & 3);  // first token (S) / first dim (O) of this lane's pair
    const int r_lo = lane >> 2;     // query row within the group
    const uint32_t sw = lane & 7;   // swizzle term: ldmatrix row index mod 8
    const float sl2 = P.scale_log2;

    uint32_t qa[KSTEPS][AR];  // Q as A fragments: {lo, [hi,] lo+8 cols, [hi+8 cols]}
    float m_lo = -INFINITY, l_lo = 0.f, m_hi = -INFINITY, l_hi = 0.f;
    // this lane's two query rows in the current piece: in use?, row of q / out,
    // last key position they may see
    bool ok_lo = false, ok_hi = false;
    size_t orow_lo = 0, orow_hi = 0;
    int32_t lim_lo = 0, lim_hi = 0;
    float acc[NTD][AR];

    while (true) {
        if (cj == cc.jbeg) {  // new piece: load its query rows as A fragments
            // Row R of the unit is (query token R / g, query head h*g + R % g);
            // token k of n new tokens sits at position len - n + k and may
            // see keys 0 .. len - n + k.  One token per sequence: R = head.
            const QRows qr = query_rows(P, cc.s, cc.len);
            if (qr.clamped && cc.p == 0 && lane == 0) flag_error(PA_DEVERR_SEQ_LEN);
            const int rows_used = g * qr.n;
            const int tok_lo = r_lo / g, tok_hi = (r_lo + 8) / g;
            ok_lo = r_lo < rows_used;
            ok_hi = HI && (r_lo + 8 < rows_used);
            orow_lo = (static_cast<size_t>(qr.base) + tok_lo) * P.num_q_heads + cc.h * g + r_lo % g;
            orow_hi = (static_cast<size_t>(qr.base) + tok_hi) * P.num_q_heads + cc.h * g + (r_lo + 8) % g;
            lim_lo = cc.len - qr.n + tok_lo;
            lim_hi = cc.len - qr.n + tok_hi;
            const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(P.q);
            const uint32_t* q_lo = reinterpret_cast<const uint32_t*>(qb + (ok_lo ? orow_lo : 0) * D + tq);
            const uint32_t* q_hi = reinterpret_cast<const uint32_t*>(qb + (ok_hi ? orow_hi : 0) * D + tq);
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                if constexpr (HI) {
                    qa[ks][0] = ok_lo ? __ldg(q_lo + ks * 8) : 0u;
                    qa[ks][2] = ok_lo ? __ldg(q_lo + ks * 8 + 4) : 0u;
                    qa[ks][1] = ok_hi ? __ldg(q_hi + ks * 8) : 0u;
                    qa[ks][3] = ok_hi ? __ldg(q_hi + ks * 8 + 4) : 0u;
                } else {
                    qa[ks][0] = ok_lo ? __ldg(q_lo + ks * 8) : 0u;
                    qa[ks][1] = ok_lo ? __ldg(q_lo + ks * 8 + 4) : 0u;
                }
            }
            m_lo = m_hi = -INFINITY;
            l_lo = l_hi = 0.f;
#pragma unroll
            for (int n = 0; n < NTD; ++n)
#pragma unroll
                for (int r = 0; r < AR; ++r) acc[n][r] = 0.f;
        }

        const uint32_t bar = bar_u32 + stage * 8;
        if (!mbar_wait_bounded(bar, phase)) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            // drain: wait (bounded) for the copies still in flight, then leave
            for (uint32_t k = 1; k < issued - consumed; ++k) {
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
                mbar_wait_bounded(bar_u32 + stage * 8, phase);
            }
            return;
        }
        ++consumed;
        const uint32_t kbase = ring_u32 + stage * Cfg::kStageBytes;
        const uint32_t vbase = kbase + Cfg::kTileBytes;
        const int valid = ((oob_mask >> stage) & 1u) ? 0 : min(kBlockTokens, cc.len - cj * kBlockTokens);
        if (valid < kBlockTokens) {
            // zero V rows [valid, 16) so that 0 * (stale or NaN) never enters P V
            uint8_t* vs = ring + stage * Cfg::kStageBytes + Cfg::kTileBytes;
            const int chunks = (kBlockTokens - valid) * Cfg::kRegions * 8;
            for (int c = lane; c < chunks; c += 32) {
                const int row = valid + c / (Cfg::kRegions * 8);
                const int rem = c % (Cfg::kRegions * 8);
                *reinterpret_cast<uint4*>(vs + (rem >> 3) * Cfg::kRegionBytes + row * 128 +
                                          (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }

        // ---- S = Q K^T : two n-tiles of 8 tokens
        float s0[AR], s1[AR];
#pragma unroll
        for (int r = 0; r < AR; ++r) s0[r] = s1[r] = 0.f;
#pragma unroll
        for (int kp = 0; kp < KSTEPS / 2; ++kp) {
            const int cg = 4 * kp + (lane >> 3);  // 8-element column chunk 0 .. D/8-1
            const uint32_t col = (cg >> 3) * Cfg::kRegionBytes + ((((uint32_t)cg & 7u) ^ sw) << 4);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kbase + col + (lane & 7) * 128, b0, b1, b2, b3);
            mma_frag(s0, qa[2 * kp], b0, b1);
            mma_frag(s0, qa[2 * kp + 1], b2, b3);
            ldsm_x4(kbase + col + (8 + (lane & 7)) * 128, b0, b1, b2, b3);
            mma_frag(s1, qa[2 * kp], b0, b1);
            mma_frag(s1, qa[2 * kp + 1], b2, b3);
        }

        // ---- online softmax (rows r_lo and r_lo + 8); key t of the block is
        // visible to a row iff t < valid and cj*16 + t <= the row's limit
        uint32_t pa0, pa1 = 0u, pa2, pa3 = 0u;
        {
            const int vis = min(valid - 1, lim_lo - cj * kBlockTokens);  // last visible key
            float x[4] = {s0[0], s0[1], s1[0], s1[1]};
            x[0] = tq <= vis ? x[0] * sl2 : -INFINITY;
            x[1] = tq + 1 <= vis ? x[1] * sl2 : -INFINITY;
            x[2] = tq + 8 <= vis ? x[2] * sl2 : -INFINITY;
            x[3] = tq + 9 <= vis ? x[3] * sl2 : -INFINITY;
            const float alpha = softmax_update(m_lo, l_lo, x, pa0, pa2);
#pragma unroll
            for (int n = 0; n < NTD; ++n) {
                acc[n][0] *= alpha;
                acc[n][1] *= alpha;
            }
        }
        if constexpr (HI) {
            const int vis = min(valid - 1, lim_hi - cj * kBlockTokens);
            float x[4] = {s0[2], s0[3], s1[2], s1[3]};
            x[0] = tq <= vis ? x[0] * sl2 : -INFINITY;
            x[1] = tq + 1 <= vis ? x[1] * sl2 : -INFINITY;
            x[2] = tq + 8 <= vis ? x[2] * sl2 : -INFINITY;
            x[3] = tq + 9 <= vis ? x[3] * sl2 : -INFINITY;
            const float alpha = softmax_update(m_hi, l_hi, x, pa1, pa3);
#pragma unroll
            for (int n = 0; n < NTD; ++n) {
                acc[n][2] *= alpha;
                acc[n][3] *= alpha;
            }
        }

        uint32_t pa[AR];  // P as an A fragment
        if constexpr (HI) {
            pa[0] = pa0; pa[1] = pa1; pa[2] = pa2; pa[3] = pa3;
        } else {
            pa[0] = pa0; pa[1] = pa2;
        }

        // ---- O += P V : n-tiles of 8 head dims, K = the 16 tokens
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
            const int cg = 2 * dp + (lane >> 4);
            const int t = 8 * ((lane >> 3) & 1) + (lane & 7);
            const uint32_t addr = vbase + (cg >> 3) * Cfg::kRegionBytes + t * 128 +
                                  ((((uint32_t)cg & 7u) ^ sw) << 4);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_trans(addr, b0, b1, b2, b3);
            mma_frag(acc[2 * dp], pa, b0, b1);
            mma_frag(acc[2 * dp + 1], pa, b2, b3);
        }
        __syncwarp();

        if (prod_live) produce(stage);
        if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
        }

        if (++cj < cc.jend) continue;

        // ---- item done: final row or partition partials
        float lt_lo = l_lo + __shfl_xor_sync(kFullMask, l_lo, 1);
        lt_lo += __shfl_xor_sync(kFullMask, lt_lo, 2);
        float lt_hi = 0.f;
        if constexpr (HI) {
            lt_hi = l_hi + __shfl_xor_sync(kFullMask, l_hi, 1);
            lt_hi += __shfl_xor_sync(kFullMask, lt_hi, 2);
        }
        if (cc.parts == 1 && P.piece_base == 0) {
            __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(P.out);
            if (ok_lo) {
                const float inv = lt_lo > 0.f ? 1.0f / lt_lo : 0.f;
                __nv_bfloat16* o = ob + orow_lo * D + tq;
#pragma unroll
                for (int n = 0; n < NTD; ++n)
                    *reinterpret_cast<__nv_bfloat162*>(o + 8 * n) =
                        __floats2bfloat162_rn(acc[n][0] * inv, acc[n][1] * inv);
            }
            if constexpr (HI) {
                if (ok_hi) {
                    const float inv = lt_hi > 0.f ? 1.0f / lt_hi : 0.f;
                    __nv_bfloat16* o = ob + orow_hi * D + tq;
#pragma unroll
                    for (int n = 0; n < NTD; ++n)
                        *reinterpret_cast<__nv_bfloat162*>(o + 8 * n) =
                            __floats2bfloat162_rn(acc[n][2] * inv, acc[n][3] * inv);
                }
            }
        } else {
            constexpr float kLn2 = 0.693147180559945309f;
            if (ok_lo) {
                const size_t idx = orow_lo * P.max_parts + P.piece_base + cc.p;
                if ((lane & 3) == 0) {
                    P.ws_m[idx] = m_lo * kLn2;
                    P.ws_l[idx] = lt_lo;
                }
                float* a = P.ws_acc + idx * D + tq;
#pragma unroll
                for (int n = 0; n < NTD; ++n)
                    *reinterpret_cast<float2*>(a + 8 * n) = make_float2(acc[n][0], acc[n][1]);
            }
            if constexpr (HI) {
                if (ok_hi) {
                    const size_t idx = orow_hi * P.max_parts + P.piece_base + cc.p;
                    if ((lane & 3) == 0) {
                        P.ws_m[idx] = m_hi * kLn2;
                        P.ws_l[idx] = lt_hi;
                    }
                    float* a = P.ws_acc + idx * D + tq;
#pragma unroll
                    for (int n = 0; n < NTD; ++n)
                        *reinterpret_cast<float2*>(a + 8 * n) = make_float2(acc[n][2], acc[n][3]);
                }
            }
        }

        record_parts(P, cc, lane);
        sched.next(cc);
        if (!cc.valid) break;
        cj = cc.jbeg;
    }
}

}  // namespace pa
