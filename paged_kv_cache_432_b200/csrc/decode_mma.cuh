// decode_mma.cuh -- paged decode attention, bf16 or E4M3 caches, one warp per work item.
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
// E4M3 (fp8) caches (FP8 = true): a stage holds the 8-bit codes of the K and
// V tile, one TMA box each (16 rows x D bytes, 128-byte swizzle).  The codes
// go from shared memory straight into MMA fragments: ldmatrix on the codes
// seen as 16-bit pairs, then cvt.f16x2.e4m3x2 (exact), and the MMAs run in
// f16.  For K, a lane receives 4 consecutive dims of one token; the k index of
// Q K^T is permuted to match (the Q fragments take the same dims), which
// changes nothing in the sum.  For V, ldmatrix.trans gives each lane two
// tokens of a dim pair; one byte permute splits that into the even and the
// odd dim's token pair, so the P V n-tiles hold the even and the odd dims of
// each 16-dim chunk.  The kv head's K scale is folded into the score scale
// and its V scale multiplies the accumulators once at the end of the piece,
// so the result is that of attention over decode(code) * scale.
//
// E4M3 with at most 8 query rows (MHA, GQA up to 8 heads per kv head) runs
// the transposed products S^T = K Q^T and O^T = V^T P^T: the block's 16
// tokens (for S^T) and 16 head dims (for O^T) fill the MMA's M dimension and
// the query rows its N = 8, so no register holds padding and each product
// takes D/16 MMAs instead of D/8.  The widened codes are the A fragments
// directly (K: token rows, V: even dims in rows 0-7, odd dims in rows 8-15);
// a row's scores sit in the 8 lanes of equal lane % 4, and four shuffles plus
// two byte permutes turn P into the B fragment of P^T.  The kernel then fits
// 128 registers, four CTAs per SM.
//
// Every wait on an mbarrier is bounded: on timeout the warp flags
// PA_DEVERR_TIMEOUT, waits (bounded) for its copies in flight and returns.
#pragma once

#include "items.cuh"

namespace pa {

template <int D, int STAGES, int WARPS, bool FP8 = false>
struct MmaCfg {
    // bf16 tiles: D/64 column slabs of 16 rows x 128 B (64 values), one TMA
    // box each.  E4M3 tiles: one box of 16 rows x D bytes.  Both with the
    // 128-byte swizzle (64-byte for E4M3 at D = 64).
    static constexpr int kRegions = FP8 ? 1 : D / 64;
    static constexpr int kRowBytes = FP8 ? D : 128;
    static constexpr int kRegionBytes = 16 * kRowBytes;
    static constexpr int kTileBytes = kRegions * kRegionBytes;  // K (or V) of one block, one head
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kRingBytes = WARPS * STAGES * kStageBytes;
    static constexpr int kBarBytes = WARPS * STAGES * 8;
    static constexpr int kThreads = WARPS * 32;
    static size_t smem_bytes(int seq_count) {  // + prefix, lengths and skips of the launch's sequences
        return 1024 + kRingBytes + kBarBytes + 12 * static_cast<size_t>(seq_count + 1);
    }
    // 16-byte chunk c of row t sits at chunk c ^ swz(t) (the TMA swizzle pattern)
    static __device__ __forceinline__ uint32_t swz(int t) {
        return (FP8 && D == 64) ? static_cast<uint32_t>((t >> 1) & 3) : static_cast<uint32_t>(t & 7);
    }
};

// Online-softmax update of one row set over NB blocks: x[4b..4b+3] are four
// raw scores of block b (tokens tq, tq+1, 8+tq, 9+tq), already masked to -inf
// where invalid and scaled to log2 units.  Returns the rescale factor for the
// accumulators and packs the probabilities as bf16 (or f16) pairs: p[b][0]
// tokens tq..tq+1, p[b][1] tokens 8+tq..9+tq of block b.
template <bool F16, int NB>
__device__ __forceinline__ float softmax_update(float& m, float& l, const float (&x)[4 * NB],
                                                uint32_t (&p)[NB][2]) {
    float bm = x[0];
#pragma unroll
    for (int i = 1; i < 4 * NB; ++i) bm = fmaxf(bm, x[i]);
    bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, 1));
    bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, 2));
    const float mn = fmaxf(m, bm);
    const float mu = mn == -INFINITY ? 0.0f : mn;  // a row with nothing valid yet
    const float alpha = fast_exp2(m - mu);
    float sum = 0.f;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        p[b][0] = pack2<F16>(fast_exp2(x[4 * b] - mu), fast_exp2(x[4 * b + 1] - mu));
        p[b][1] = pack2<F16>(fast_exp2(x[4 * b + 2] - mu), fast_exp2(x[4 * b + 3] - mu));
        // the denominator sums the same (rounded) weights the numerator uses
        const float2 fa = unpack2<F16>(p[b][0]), fb = unpack2<F16>(p[b][1]);
        sum += (fa.x + fa.y) + (fb.x + fb.y);
    }
    l = l * alpha + sum;
    m = mn;
    return alpha;
}

// The same for one row of the transposed layout, where the lane holds two of
// the row's 16 scores (x0: token lane/4, x1: token 8 + lane/4) and the 8
// lanes of equal lane % 4 hold the rest.  p gets the f16 pair (x0's, x1's
// weight); l is this lane's share of the row sum.
__device__ __forceinline__ float softmax_update_col(float& m, float& l, float x0, float x1, uint32_t& p) {
    float bm = fmaxf(x0, x1);
    bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, 4));
    bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, 8));
    bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, 16));
    const float mn = fmaxf(m, bm);
    const float mu = mn == -INFINITY ? 0.0f : mn;  // a row with nothing valid yet
    const float alpha = fast_exp2(m - mu);
    p = pack2<true>(fast_exp2(x0 - mu), fast_exp2(x1 - mu));
    const float2 f = unpack2<true>(p);  // the denominator sums the rounded weights
    l = l * alpha + (f.x + f.y);
    m = mn;
    return alpha;
}

template <int D, int ROWS, int STAGES, int WARPS, int MIN_CTAS, bool FP8 = false>
__global__ void __launch_bounds__(WARPS * 32, MIN_CTAS)
decode_bf16_mma_kernel(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const DecodeParams P) {
    using Cfg = MmaCfg<D, STAGES, WARPS, FP8>;
    constexpr int KSTEPS = D / 16;  // k-steps of Q K^T
    constexpr int NTD = D / 8;      // n-tiles of P V
    constexpr bool HI = ROWS > 8;   // query rows 8..15 in use
    constexpr int AR = HI ? 4 : 2;  // registers per A fragment / per C tile that are held
    // E4M3 with <= 8 query rows: the transposed products S^T = K Q^T and
    // O^T = V^T P^T, tokens / head dims in M and the query rows in N
    constexpr bool TR = FP8 && !HI;
    // one query row (MHA): only the even columns of S^T / O^T are real, so
    // each lane keeps one row's softmax instead of two
    constexpr bool ONE = TR && ROWS == 1;
    constexpr int ACC_N = TR ? D / 16 : NTD;  // accumulator tiles
    constexpr int ACC_R = TR ? 4 : AR;        // registers held per tile
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
    // resident while the previous kernel (typically the cache write) still
    // runs.  Until grid_dependency_wait() they read only inputs that no kernel
    // of this library writes (lengths, block tables, query rows): the
    // schedule, the first table window and, into L2, the first query rows are
    // ready when the wait ends.  The pool (which the cache write fills), the
    // output and the workspace are touched only after it.
    const Schedule sched = make_schedule(P, prefix, WARPS);  // ends with __syncthreads
    const int32_t my_warp = blockIdx.x * WARPS + warp;
    Cursor pc;  // producer: the piece whose next block is loaded next
    sched.start(pc, my_warp);
    int32_t first_tbl = 0;  // lane l: table entry jbeg + l of the first piece
    if (pc.valid) {
        const int32_t jj = pc.jbeg + lane;
        first_tbl = jj < pc.jend
                        ? __ldg(P.block_tables + static_cast<size_t>(pc.s) * P.max_blocks_per_seq + jj)
                        : 0;
        if (!P.q_start && lane < P.group * D / 64)  // its g query rows of D bf16: 128-byte lines
            prefetch_l2(static_cast<const __nv_bfloat16*>(P.q) +
                        (static_cast<size_t>(pc.s) * P.num_q_heads + pc.h * P.group) * D + 64 * lane);
    }
    grid_dependency_wait();
    // Dependents may start only now, once every CTA has passed the wait: the
    // kernels launched before this one have then completed, so a following
    // grid that does not depend on this one (the shared-prefix tiles) may
    // read what they wrote without waiting for this grid.
    allow_dependents();
    zero_empty_sequences<__nv_bfloat16>(P, lens);
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
    int32_t tbl = first_tbl, tbase = pc.jbeg;
    bool tbl_fresh = true;  // tbl holds entries of the producer's current piece
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
    // The lane's two rows of S and O: r_lo and r_lo + 8, or, transposed, the
    // C columns tq and tq + 1 (its Q row stays r_lo, the B-operand column).
    const int row_a = TR ? tq : r_lo, row_b = TR ? tq + 1 : r_lo + 8;
    const uint32_t sw = lane & 7;   // swizzle term: ldmatrix row index mod 8
    float sl2 = P.scale_log2;  // times the kv head's K scale for E4M3 caches
    float vscale = 1.f;         // the kv head's V scale for E4M3 caches

    uint32_t qa[KSTEPS][AR];  // Q as A fragments: {lo, [hi,] lo+8 cols, [hi+8 cols]}
    float m_lo = -INFINITY, l_lo = 0.f, m_hi = -INFINITY, l_hi = 0.f;
    // this lane's two query rows in the current piece: in use?, row of q / out,
    // last key position they may see
    bool ok_lo = false, ok_hi = false;
    size_t orow_lo = 0, orow_hi = 0;
    int32_t lim_lo = 0, lim_hi = 0;
    float acc[ACC_N][ACC_R];

    while (true) {
        if (cj == cc.jbeg) {  // new piece: load its query rows as A fragments
            // Row R of the unit is (query token R / g, query head h*g + R % g);
            // token k of n new tokens sits at position len - n + k and may
            // see keys 0 .. len - n + k.  One token per sequence: R = head.
            const QRows qr = query_rows(P, cc.s, cc.len);
            if (qr.clamped && cc.p == 0 && lane == 0) flag_error(PA_DEVERR_SEQ_LEN);
            const int rows_used = g * qr.n;
            const int tok_lo = row_a / g, tok_hi = row_b / g;
            ok_lo = row_a < rows_used;
            ok_hi = (HI || TR) && (row_b < rows_used);
            orow_lo = (static_cast<size_t>(qr.base) + tok_lo) * P.num_q_heads + cc.h * g + row_a % g;
            orow_hi = (static_cast<size_t>(qr.base) + tok_hi) * P.num_q_heads + cc.h * g + row_b % g;
            lim_lo = cc.len - qr.n + tok_lo;
            lim_hi = cc.len - qr.n + tok_hi;
            const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(P.q);
            if constexpr (FP8) {
                // k-step ks covers dims 16ks..16ks+15; the K fragments hold
                // dims 16ks+2tq..+3 (b0: first pair, b1: second), so the A
                // fragment takes the same dims: a0/a1 the first pair, a2/a3
                // the second.  Transposed, the same registers are the B
                // fragment of Q^T (row r_lo, the same dims).  Widened to f16
                // (exact for |q| in 2^-14..65504).
                const bool ok_q = r_lo < rows_used;
                const size_t orow_q =
                    (static_cast<size_t>(qr.base) + r_lo / g) * P.num_q_heads + cc.h * g + r_lo % g;
                const uint2* q_lo = reinterpret_cast<const uint2*>(qb + (ok_q ? orow_q : 0) * D + 2 * tq);
                const uint2* q_hi = reinterpret_cast<const uint2*>(qb + (ok_hi ? orow_hi : 0) * D + 2 * tq);
                bool q_out_of_range = false;  // a value f16 cannot hold (|q| > 65504, inf, NaN)
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const uint2 lo = ok_q ? __ldg(q_lo + 4 * ks) : make_uint2(0u, 0u);
                    if constexpr (HI) {
                        const uint2 hi = ok_hi ? __ldg(q_hi + 4 * ks) : make_uint2(0u, 0u);
                        qa[ks][0] = bf16x2_to_f16x2_checked(lo.x, q_out_of_range);
                        qa[ks][1] = bf16x2_to_f16x2_checked(hi.x, q_out_of_range);
                        qa[ks][2] = bf16x2_to_f16x2_checked(lo.y, q_out_of_range);
                        qa[ks][3] = bf16x2_to_f16x2_checked(hi.y, q_out_of_range);
                    } else {
                        qa[ks][0] = bf16x2_to_f16x2_checked(lo.x, q_out_of_range);
                        qa[ks][1] = bf16x2_to_f16x2_checked(lo.y, q_out_of_range);
                    }
                }
                if (__any_sync(kFullMask, q_out_of_range) && lane == 0) flag_error(PA_DEVERR_Q_RANGE);
                sl2 = P.scale_log2 * __ldg(P.k_scale + cc.h);
                vscale = __ldg(P.v_scale + cc.h);
            } else {
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
            }
            m_lo = m_hi = -INFINITY;
            l_lo = l_hi = 0.f;
#pragma unroll
            for (int n = 0; n < ACC_N; ++n)
#pragma unroll
                for (int r = 0; r < ACC_R; ++r) acc[n][r] = 0.f;
        }

        // ---- this step's block: wait for its stage and mask what it holds
        if (!mbar_wait_bounded(bar_u32 + stage * 8, phase)) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            // drain: wait (bounded) for the copies still in flight, then leave
            int sb = stage;
            uint32_t pb = phase;
            for (uint32_t k = 1; k < issued - consumed; ++k) {
                if (++sb == STAGES) { sb = 0; pb ^= 1u; }
                mbar_wait_bounded(bar_u32 + sb * 8, pb);
            }
            return;
        }
        ++consumed;
        const int valid = ((oob_mask >> stage) & 1u) ? 0 : min(kBlockTokens, cc.len - cj * kBlockTokens);
        const uint32_t kb = ring_u32 + stage * Cfg::kStageBytes;
        const uint32_t vb = kb + Cfg::kTileBytes;
        if (valid < kBlockTokens) {
            // zero V rows [valid, 16) so that 0 * (stale or NaN) never enters P V
            uint8_t* vs = ring + stage * Cfg::kStageBytes + Cfg::kTileBytes;
            constexpr int kRowChunks = Cfg::kRegions * Cfg::kRowBytes / 16;  // 16-byte chunks per row
            constexpr int kSlabChunks = Cfg::kRowBytes / 16;
            const int chunks = (kBlockTokens - valid) * kRowChunks;
            for (int c = lane; c < chunks; c += 32) {
                const int row = valid + c / kRowChunks;
                const int rem = c % kRowChunks;
                *reinterpret_cast<uint4*>(vs + (rem / kSlabChunks) * Cfg::kRegionBytes +
                                          row * Cfg::kRowBytes + (rem % kSlabChunks) * 16) =
                    make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }

        if constexpr (TR) {
            // ---- S^T = K Q^T: M = the block's 16 tokens, N = the query
            // rows, K = head dims.  ldmatrix on the codes seen as 16-bit
            // pairs gives each lane dims 4(lane%4)..+3 of token lane/4 (and of
            // token 8 + lane/4) per 16-dim chunk: widened, those are the A
            // fragment, and Q^T takes the same dims (qa).
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const int tok = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
                for (int j = 0; j < KSTEPS; j += 2) {
                    const uint32_t ch = static_cast<uint32_t>(j + (lane >> 4));
                    uint32_t r0, r1, r2, r3, l0, h0, l1, h1;
                    ldsm_x4(kb + tok * Cfg::kRowBytes + ((ch ^ Cfg::swz(tok)) << 4), r0, r1, r2, r3);
                    e4m3x4_to_f16x2x2(r0, l0, h0);  // tokens 0-7, chunk j
                    e4m3x4_to_f16x2x2(r1, l1, h1);  // tokens 8-15, chunk j
                    mma_f16(s0, l0, l1, h0, h1, qa[j][0], qa[j][1]);
                    e4m3x4_to_f16x2x2(r2, l0, h0);  // chunk j + 1
                    e4m3x4_to_f16x2x2(r3, l1, h1);
                    mma_f16(s1, l0, l1, h0, h1, qa[j + 1][0], qa[j + 1][1]);
                }
            }
            // ---- online softmax: this lane holds tokens r_lo and r_lo + 8
            // of rows tq (s[0], s[2]) and tq + 1 (s[1], s[3]); a row's 16
            // tokens sit in the 8 lanes of equal lane % 4
            const int vis_a = min(valid - 1, lim_lo - cj * kBlockTokens);
            const int vis_b = min(valid - 1, lim_hi - cj * kBlockTokens);
            uint32_t pk_a, pk_b;  // f16 pairs (token r_lo, token r_lo + 8) of rows tq, tq + 1
            const float alpha_lo = softmax_update_col(m_lo, l_lo, r_lo <= vis_a ? (s0[0] + s1[0]) * sl2 : -INFINITY,
                                          r_lo + 8 <= vis_a ? (s0[2] + s1[2]) * sl2 : -INFINITY, pk_a);
            float alpha_hi = 1.f;
            if constexpr (ONE) {
                pk_b = pk_a;  // the odd columns only carry padding
            } else {
                alpha_hi = softmax_update_col(m_hi, l_hi, r_lo <= vis_b ? (s0[1] + s1[1]) * sl2 : -INFINITY,
                                              r_lo + 8 <= vis_b ? (s0[3] + s1[3]) * sl2 : -INFINITY, pk_b);
            }
            if (__any_sync(kFullMask, alpha_lo != 1.f || alpha_hi != 1.f)) {
#pragma unroll
                for (int c = 0; c < ACC_N; ++c) {
                    acc[c][0] *= alpha_lo;
                    acc[c][2] *= alpha_lo;
                    if constexpr (!ONE) {
                        acc[c][1] *= alpha_hi;
                        acc[c][3] *= alpha_hi;
                    }
                }
            }
            // ---- P^T as the B fragment: lane l takes row r_lo, tokens tq,
            // tq + 1 and 8 + tq, 9 + tq; token t < 8 of row n sits in lane
            // 4t + n/2 (the low half of pk_a for even n, of pk_b for odd n),
            // token 8 + t in the high half of the same register
            uint32_t pb0, pb1;
            {
                const int src = 8 * (lane & 3) + (r_lo >> 1);  // holds token tq; src + 4 token tq + 1
                const uint32_t xa = __shfl_sync(kFullMask, pk_a, src), xb = __shfl_sync(kFullMask, pk_a, src + 4);
                uint32_t wa = xa, wb = xb;
                if constexpr (!ONE) {
                    const uint32_t ya = __shfl_sync(kFullMask, pk_b, src), yb = __shfl_sync(kFullMask, pk_b, src + 4);
                    wa = (r_lo & 1) ? ya : xa;
                    wb = (r_lo & 1) ? yb : xb;
                }
                pb0 = __byte_perm(wa, wb, 0x5410);  // tokens tq, tq + 1
                pb1 = __byte_perm(wa, wb, 0x7632);  // tokens 8 + tq, 9 + tq
            }
            // ---- O^T += V^T P^T: M = 16 head dims of a chunk (rows 0-7 the
            // even dims 16c + 2(lane/4), rows 8-15 the odd ones), K = tokens.
            // ldmatrix.trans gives each lane tokens tq, tq + 1 of the dim pair
            // 2(lane/4), +1; one byte permute splits it into the even and the
            // odd dim's token pair: exactly the A fragment.
            {
                const int tok = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
                for (int c = 0; c < D / 16; c += 2) {
                    const uint32_t ch = static_cast<uint32_t>(c + (lane >> 4));
                    uint32_t r0, r1, r2, r3, e0, o0, e1, o1;
                    ldsm_x4_trans(vb + tok * Cfg::kRowBytes + ((ch ^ Cfg::swz(tok)) << 4), r0, r1, r2, r3);
                    e4m3x4_to_f16x2x2(byte_perm(r0, 0x3120), e0, o0);  // tokens tq, tq + 1
                    e4m3x4_to_f16x2x2(byte_perm(r1, 0x3120), e1, o1);  // tokens 8 + tq, 9 + tq
                    mma_f16(acc[c], e0, o0, e1, o1, pb0, pb1);
                    e4m3x4_to_f16x2x2(byte_perm(r2, 0x3120), e0, o0);  // chunk c + 1
                    e4m3x4_to_f16x2x2(byte_perm(r3, 0x3120), e1, o1);
                    mma_f16(acc[c + 1], e0, o0, e1, o1, pb0, pb1);
                }
            }
        }
        if constexpr (!TR) {
            // ---- S = Q K^T of the block: two n-tiles of 8 tokens, each with
            // two accumulators (even / odd k-steps) so that the dependent MMA
            // chains are KSTEPS/2 long
            float sc[2][AR];
            {
                float s0[AR], s1[AR], t0[AR], t1[AR];
#pragma unroll
                for (int r = 0; r < AR; ++r) s0[r] = s1[r] = t0[r] = t1[r] = 0.f;
                if constexpr (FP8) {
                    // E4M3 K: ldmatrix on the codes seen as b16 gives each lane dims
                    // 4(lane%4)..+3 of one token per 16-dim chunk; matrices: (tokens
                    // 0-7, chunk j), (8-15, j), (0-7, j+1), (8-15, j+1)
                    const int tok = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
                    for (int j = 0; j < KSTEPS; j += 2) {
                        const uint32_t ch = static_cast<uint32_t>(j + (lane >> 4));
                        uint32_t r0, r1, r2, r3, b0, b1;
                        ldsm_x4(kb + tok * Cfg::kRowBytes + ((ch ^ Cfg::swz(tok)) << 4), r0, r1, r2, r3);
                        e4m3x4_to_f16x2x2(r0, b0, b1);
                        mma_frag_t<true>(s0, qa[j], b0, b1);
                        e4m3x4_to_f16x2x2(r1, b0, b1);
                        mma_frag_t<true>(s1, qa[j], b0, b1);
                        e4m3x4_to_f16x2x2(r2, b0, b1);
                        mma_frag_t<true>(t0, qa[j + 1], b0, b1);
                        e4m3x4_to_f16x2x2(r3, b0, b1);
                        mma_frag_t<true>(t1, qa[j + 1], b0, b1);
                    }
                } else {
#pragma unroll
                    for (int kp = 0; kp < KSTEPS / 2; ++kp) {
                        const int cg = 4 * kp + (lane >> 3);  // 8-element column chunk 0 .. D/8-1
                        const uint32_t col = (cg >> 3) * Cfg::kRegionBytes + ((((uint32_t)cg & 7u) ^ sw) << 4);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(kb + col + (lane & 7) * 128, b0, b1, b2, b3);
                        mma_frag(s0, qa[2 * kp], b0, b1);
                        mma_frag(t0, qa[2 * kp + 1], b2, b3);
                        ldsm_x4(kb + col + (8 + (lane & 7)) * 128, b0, b1, b2, b3);
                        mma_frag(s1, qa[2 * kp], b0, b1);
                        mma_frag(t1, qa[2 * kp + 1], b2, b3);
                    }
                }
#pragma unroll
                for (int r = 0; r < AR; ++r) {
                    sc[0][r] = s0[r] + t0[r];
                    sc[1][r] = s1[r] + t1[r];
                }
            }

            // ---- online softmax over the block's keys (rows r_lo and r_lo + 8);
            // key t is visible to a row iff t < valid and cj*16 + t <= the
            // row's limit
            uint32_t plo[1][2], phi[1][2];  // P as bf16 / f16 pairs: tokens tq.. / 8+tq..
            float alpha_lo, alpha_hi = 1.f;
            {
                const int vis = min(valid - 1, lim_lo - cj * kBlockTokens);  // last visible key
                const float x[4] = {tq <= vis ? sc[0][0] * sl2 : -INFINITY,
                                    tq + 1 <= vis ? sc[0][1] * sl2 : -INFINITY,
                                    tq + 8 <= vis ? sc[1][0] * sl2 : -INFINITY,
                                    tq + 9 <= vis ? sc[1][1] * sl2 : -INFINITY};
                alpha_lo = softmax_update<FP8, 1>(m_lo, l_lo, x, plo);
            }
            if constexpr (HI) {
                const int vis = min(valid - 1, lim_hi - cj * kBlockTokens);
                const float x[4] = {tq <= vis ? sc[0][2] * sl2 : -INFINITY,
                                    tq + 1 <= vis ? sc[0][3] * sl2 : -INFINITY,
                                    tq + 8 <= vis ? sc[1][2] * sl2 : -INFINITY,
                                    tq + 9 <= vis ? sc[1][3] * sl2 : -INFINITY};
                alpha_hi = softmax_update<FP8, 1>(m_hi, l_hi, x, phi);
            }
            // rescale the accumulators only when some row's max moved (alpha is
            // exactly 1 otherwise): after the first blocks of a sequence it rarely does
            if (__any_sync(kFullMask, alpha_lo != 1.f || alpha_hi != 1.f)) {
#pragma unroll
                for (int n = 0; n < NTD; ++n) {
                    acc[n][0] *= alpha_lo;
                    acc[n][1] *= alpha_lo;
                    if constexpr (HI) {
                        acc[n][2] *= alpha_hi;
                        acc[n][3] *= alpha_hi;
                    }
                }
            }

            // ---- O += P V : n-tiles of 8 head dims, K = the 16 tokens of the block
            uint32_t pa[AR];  // P as an A fragment
            if constexpr (HI) {
                pa[0] = plo[0][0]; pa[1] = phi[0][0]; pa[2] = plo[0][1]; pa[3] = phi[0][1];
            } else {
                pa[0] = plo[0][0]; pa[1] = plo[0][1];
            }
            if constexpr (FP8) {
                // E4M3 V: ldmatrix.trans on the codes seen as b16 gives each lane
                // tokens 2(lane%4), +1 of the dim pair 2(lane/4), +1 of a 16-dim
                // chunk; one byte permute splits it into the even and the odd
                // dim's token pair.  n-tile 2c of the accumulators holds the even
                // dims 16c + 2n of chunk c, n-tile 2c+1 the odd dims.
                const int tok = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
                for (int c = 0; c < D / 16; c += 2) {
                    const uint32_t ch = static_cast<uint32_t>(c + (lane >> 4));
                    uint32_t r0, r1, r2, r3;
                    ldsm_x4_trans(vb + tok * Cfg::kRowBytes + ((ch ^ Cfg::swz(tok)) << 4), r0, r1, r2, r3);
                    uint32_t e0, o0, e1, o1;
                    e4m3x4_to_f16x2x2(byte_perm(r0, 0x3120), e0, o0);  // tokens 2(lane%4), +1
                    e4m3x4_to_f16x2x2(byte_perm(r1, 0x3120), e1, o1);  // tokens 8 + 2(lane%4), +1
                    mma_frag_t<true>(acc[2 * c], pa, e0, e1);
                    mma_frag_t<true>(acc[2 * c + 1], pa, o0, o1);
                    e4m3x4_to_f16x2x2(byte_perm(r2, 0x3120), e0, o0);
                    e4m3x4_to_f16x2x2(byte_perm(r3, 0x3120), e1, o1);
                    mma_frag_t<true>(acc[2 * c + 2], pa, e0, e1);
                    mma_frag_t<true>(acc[2 * c + 3], pa, o0, o1);
                }
            } else {
#pragma unroll
                for (int dp = 0; dp < D / 16; ++dp) {
                    const int cg = 2 * dp + (lane >> 4);
                    const int t = 8 * ((lane >> 3) & 1) + (lane & 7);
                    const uint32_t addr = vb + (cg >> 3) * Cfg::kRegionBytes + t * 128 +
                                          ((((uint32_t)cg & 7u) ^ sw) << 4);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(addr, b0, b1, b2, b3);
                    mma_frag(acc[2 * dp], pa, b0, b1);
                    mma_frag(acc[2 * dp + 1], pa, b2, b3);
                }
            }
        }
        __syncwarp();

        // ---- hand the stage back to the producer
        if (prod_live) produce(stage);
        if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
        }

        if (++cj < cc.jend) continue;

        // ---- item done: final row or partition partials
        if constexpr (FP8) {  // the sums of P V used the V codes: apply the V scale once
#pragma unroll
            for (int n = 0; n < ACC_N; ++n)
#pragma unroll
                for (int r = 0; r < ACC_R; ++r) acc[n][r] *= vscale;
        }
        // row sums: over the 4 lanes of a row, or (transposed) the 8 lanes of a column
        float lt_lo = l_lo, lt_hi = l_hi;
#pragma unroll
        for (int x = TR ? 4 : 1; x < (TR ? 32 : 4); x *= 2) {
            lt_lo += __shfl_xor_sync(kFullMask, lt_lo, x);
            if constexpr (HI || (TR && !ONE)) lt_hi += __shfl_xor_sync(kFullMask, lt_hi, x);
        }
        // This lane's accumulators of a row (r = 0: row r_lo, r = 2: row
        // r_lo + 8) go to dims 8n + tq, +1 of n-tile n (bf16); for E4M3 to
        // dims 16c + 2tq .. +3 of chunk c as (even, odd, even, odd) n-tiles.
        // Transposed (r = 0: row tq, r = 1: row tq + 1): acc[c][r] and
        // acc[c][r + 2] are dims 16c + 2(lane/4), +1.
        constexpr int RB = TR ? 1 : 2;  // accumulator index of the lane's second row
        auto put_out = [&](size_t orow, int r, float inv) {
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(P.out) + orow * D;
            if constexpr (TR) {
#pragma unroll
                for (int c = 0; c < D / 16; ++c)
                    *reinterpret_cast<__nv_bfloat162*>(o + 16 * c + 2 * r_lo) =
                        __floats2bfloat162_rn(acc[c][r] * inv, acc[c][r + 2] * inv);
            } else if constexpr (FP8) {
#pragma unroll
                for (int c = 0; c < D / 16; ++c) {
                    uint2 u;
                    u.x = pack2<false>(acc[2 * c][r] * inv, acc[2 * c + 1][r] * inv);
                    u.y = pack2<false>(acc[2 * c][r + 1] * inv, acc[2 * c + 1][r + 1] * inv);
                    *reinterpret_cast<uint2*>(o + 16 * c + 2 * tq) = u;
                }
            } else {
#pragma unroll
                for (int n = 0; n < NTD; ++n)
                    *reinterpret_cast<__nv_bfloat162*>(o + 8 * n + tq) =
                        __floats2bfloat162_rn(acc[n][r] * inv, acc[n][r + 1] * inv);
            }
        };
        auto put_partial = [&](size_t idx, int r) {
            float* a = P.ws_acc + idx * D;
            if constexpr (TR) {
#pragma unroll
                for (int c = 0; c < D / 16; ++c)
                    *reinterpret_cast<float2*>(a + 16 * c + 2 * r_lo) = make_float2(acc[c][r], acc[c][r + 2]);
            } else if constexpr (FP8) {
#pragma unroll
                for (int c = 0; c < D / 16; ++c)
                    *reinterpret_cast<float4*>(a + 16 * c + 2 * tq) =
                        make_float4(acc[2 * c][r], acc[2 * c + 1][r], acc[2 * c][r + 1], acc[2 * c + 1][r + 1]);
            } else {
#pragma unroll
                for (int n = 0; n < NTD; ++n)
                    *reinterpret_cast<float2*>(a + 8 * n + tq) = make_float2(acc[n][r], acc[n][r + 1]);
            }
        };
        if (cc.parts == 1 && P.piece_base == 0) {
            if (ok_lo) put_out(orow_lo, 0, lt_lo > 0.f ? 1.0f / lt_lo : 0.f);
            if constexpr (HI || (TR && !ONE)) {
                if (ok_hi) put_out(orow_hi, RB, lt_hi > 0.f ? 1.0f / lt_hi : 0.f);
            }
        } else {
            constexpr float kLn2 = 0.693147180559945309f;
            const bool stat_lane = TR ? r_lo == 0 : (lane & 3) == 0;  // one lane per row writes m, l
            if (ok_lo) {
                const size_t idx = orow_lo * P.max_parts + P.piece_base + cc.p;
                if (stat_lane) {
                    P.ws_m[idx] = m_lo * kLn2;
                    P.ws_l[idx] = lt_lo;
                }
                put_partial(idx, 0);
            }
            if constexpr (HI || (TR && !ONE)) {
                if (ok_hi) {
                    const size_t idx = orow_hi * P.max_parts + P.piece_base + cc.p;
                    if (stat_lane) {
                        P.ws_m[idx] = m_hi * kLn2;
                        P.ws_l[idx] = lt_hi;
                    }
                    put_partial(idx, RB);
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
