// decode_prefix.cuh -- attention of all sequences' queries to a prefix they share.
//
// When every sequence of a batch starts with the same prompt, their tables
// point at the same physical blocks for it ("Was ändert PagedAttention an der
// KV-Speicherzuweisung für LLMs?", slavadubrov.com, §"Gemeinsame Nutzung
// erfordert mehr als Speicherzuweisung": several requests reference one cache
// block, prefix caching finds blocks of identical prefixes; "PagedAttention
// et vLLM", aiunderstanding.org, §"Questions fréquemment posées": identical
// prefixes refer to the same physical KV pages).  The plain decode reads those
// blocks once per sequence.  Here they are read once per CTA for many
// sequences: for kv head h, the N*g query rows of all sequences form the M
// side of a real matrix product with the prefix keys, S = Q K^T, followed by
// P V, flash-attention style (online softmax per query row).
//
// Grid: (row tiles x key splits, kv heads).  A CTA owns 64 query rows (4
// consumer warps x 16 rows, any (sequence, query head) pairs of the group) and
// one key split (a run of prefix blocks).  A producer warp streams the split's
// blocks with TMA (64 x 16 boxes, 128-byte swizzle), two blocks (32 keys) per
// stage, into a 4-stage ring shared by the 4 consumers: `full` barriers carry
// the TMA byte counts, `empty` barriers collect one arrival per consumer warp
// before a stage is refilled.  Each 32-key step costs one softmax update per
// row, and the accumulators are rescaled only when some row's running max
// moved.
// Each consumer runs mma.sync m16n8k16 (bf16, fp32 accumulate) on its 16 rows,
// the same fragment layout as the decode kernel, and writes the split's
// partial (m, l, acc) per row to the workspace at piece index = split.  The
// rest of each sequence (its private blocks) is handled by the decode kernel
// with skip_blocks set, and the log-sum-exp reduction merges both.
#pragma once

#include "decode_mma.cuh"

namespace pa {

struct PrefixParams {
    const void* q;
    const int32_t* block_tables;  // [num_seqs][max_blocks_per_seq]; row 0 names the prefix blocks
    const int32_t* seq_lens;
    float* ws_m;
    float* ws_l;
    float* ws_acc;
    int32_t num_seqs;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t group;
    int32_t max_blocks_per_seq;
    int32_t num_blocks;
    int32_t shared_blocks;  // blocks of the shared prefix
    int32_t split_blocks;   // prefix blocks per key split
    int32_t row_tiles;      // ceil(num_seqs * group / 64)
    int32_t max_parts;      // pieces per row in the workspace
    float scale_log2;
};

#ifndef PA_PREFIX_MIN_CTAS
#define PA_PREFIX_MIN_CTAS 2
#endif
constexpr int kPrefixConsumers = 4;
constexpr int kPrefixStages = 4;
constexpr int kPrefixRows = 16 * kPrefixConsumers;  // query rows per CTA

constexpr int kPrefixBlocksPerStage = 2;  // 32 keys per softmax step

template <int D>
struct PrefixCfg {
    static constexpr int kRegions = D / 64;
    static constexpr int kTileBytes = kRegions * 2048;  // K (or V) of one block, one head
    // stage: K of block 0, K of block 1, V of block 0, V of block 1
    static constexpr int kStageBytes = 2 * kPrefixBlocksPerStage * kTileBytes;
    static constexpr int kThreads = (kPrefixConsumers + 1) * 32;
    static constexpr size_t kSmem = 1024 + kPrefixStages * kStageBytes + 2 * kPrefixStages * 8 + 16 * 4;
};

// Online-softmax update of one row set over a 32-key step.  x[] are the row's
// scores (log2 units, -inf where masked) for keys tq, tq+1, 8+tq, 9+tq, then
// the same + 16.  Packs the probabilities as bf16 pairs p[0..3] (keys tq..,
// 8+tq.., 16+tq.., 24+tq..) and returns the accumulator rescale factor.
__device__ __forceinline__ float softmax_update32(float& m, float& l, const float (&x)[8],
                                                  uint32_t (&p)[4]) {
    float bm = x[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) bm = fmaxf(bm, x[k]);
    bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, 1));
    bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, 2));
    const float mn = fmaxf(m, bm);
    const float mu = mn == -INFINITY ? 0.0f : mn;
    const float alpha = exp2f(m - mu);
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(exp2f(x[2 * k] - mu), exp2f(x[2 * k + 1] - mu));
        const float2 f = __bfloat1622float2(v);
        sum += f.x + f.y;
        p[k] = bf162_bits(v);
    }
    l = l * alpha + sum;
    m = mn;
    return alpha;
}

// Single-thread bounded wait (the producer lane).
__device__ __forceinline__ bool mbar_wait_bounded_thread(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        for (int k = 0; k < 32; ++k)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <int D>
__global__ void __launch_bounds__(PrefixCfg<D>::kThreads, PA_PREFIX_MIN_CTAS)
decode_prefix_mma_kernel(const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const PrefixParams P) {
    using Cfg = PrefixCfg<D>;
    constexpr int KSTEPS = D / 16;
    constexpr int NTD = D / 8;
    constexpr int S = kPrefixStages;

    grid_dependency_wait();
    allow_dependents();

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    const uint32_t ring_u32 = smem_u32(smem);
    const uint32_t full_u32 = ring_u32 + S * Cfg::kStageBytes;
    const uint32_t empty_u32 = full_u32 + S * 8;
    int32_t* oob = reinterpret_cast<int32_t*>(smem + S * Cfg::kStageBytes + 2 * S * 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int tile = blockIdx.x % P.row_tiles;
    const int split = blockIdx.x / P.row_tiles;
    const int jbeg = split * P.split_blocks;
    const int jend = min(P.shared_blocks, jbeg + P.split_blocks);
    const int nblk = jend - jbeg;
    const int g = P.group;
    const int rows_total = P.num_seqs * g;

    // Precondition check, spread over all CTAs: every table starts with the
    // prefix blocks of table 0, and no sequence is shorter than the prefix.
    {
        const int64_t nthreads = static_cast<int64_t>(gridDim.x) * gridDim.y * blockDim.x;
        const int64_t me = (static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x;
        const int64_t entries = static_cast<int64_t>(P.num_seqs) * P.shared_blocks;
        for (int64_t e = me; e < entries; e += nthreads) {
            const int64_t s = e / P.shared_blocks, j = e - s * P.shared_blocks;
            if (P.block_tables[s * P.max_blocks_per_seq + j] != P.block_tables[j]) flag_error(PA_DEVERR_PREFIX);
        }
        for (int64_t s = me; s < P.num_seqs; s += nthreads)
            if (P.seq_lens[s] < P.shared_blocks * kBlockTokens) flag_error(PA_DEVERR_PREFIX);
    }

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(full_u32 + st * 8, 1);
            mbar_init(empty_u32 + st * 8, kPrefixConsumers);
        }
        fence_barrier_init();
    }
    __syncthreads();
    if (nblk <= 0) return;

    if (warp == kPrefixConsumers) {
        // ---------------- producer: one lane streams the split's blocks
        if (lane != 0) return;
        const uint64_t policy = l2_policy_evict_last();  // every row tile of this head reads them
        const int nst = (nblk + kPrefixBlocksPerStage - 1) / kPrefixBlocksPerStage;
        for (int n = 0; n < nst; ++n) {
            const int st = n % S;
            const uint32_t fill = n / S;
            if (fill > 0 && !mbar_wait_bounded_thread(empty_u32 + st * 8, (fill - 1) & 1u)) {
                flag_error(PA_DEVERR_TIMEOUT);
                return;
            }
            // bit b: block b of the stage is absent or outside the pool (masked)
            int32_t pbs[kPrefixBlocksPerStage];
            int32_t mask = 0, loaded = 0;
#pragma unroll
            for (int b = 0; b < kPrefixBlocksPerStage; ++b) {
                const int j = jbeg + n * kPrefixBlocksPerStage + b;
                pbs[b] = -1;
                if (j >= jend) {
                    mask |= 1 << b;
                    continue;
                }
                int32_t pb = P.block_tables[j];
                if (static_cast<uint32_t>(pb) >= static_cast<uint32_t>(P.num_blocks)) {
                    flag_error(PA_DEVERR_BLOCK_OOB);
                    mask |= 1 << b;
                    continue;
                }
                pbs[b] = pb;
                ++loaded;
            }
            oob[st] = mask;  // published by the mbarrier arrive below
            fence_proxy_async_smem();
            const uint32_t bar = full_u32 + st * 8;
            mbar_arrive_expect_tx(bar, loaded * 2 * Cfg::kTileBytes);
            const uint32_t sbase = ring_u32 + st * Cfg::kStageBytes;
#pragma unroll
            for (int b = 0; b < kPrefixBlocksPerStage; ++b) {
                if (pbs[b] < 0) continue;
                const int32_t row = (pbs[b] * P.num_kv_heads + h) * kBlockTokens;
                const uint32_t kdst = sbase + b * Cfg::kTileBytes;
                const uint32_t vdst = sbase + (kPrefixBlocksPerStage + b) * Cfg::kTileBytes;
#pragma unroll
                for (int r = 0; r < Cfg::kRegions; ++r) {
                    tma_load_2d(kdst + r * 2048, &tmap_k, r * 64, row, bar, policy);
                    tma_load_2d(vdst + r * 2048, &tmap_v, r * 64, row, bar, policy);
                }
            }
        }
        return;
    }

    // ---------------- consumers: 16 query rows each
    const int tq = 2 * (lane & 3);
    const uint32_t sw = lane & 7;
    const int r_lo = tile * kPrefixRows + warp * 16 + (lane >> 2);
    const int r_hi = r_lo + 8;
    const bool lo_ok = r_lo < rows_total, hi_ok = r_hi < rows_total;
    // query row r = (sequence r / g, query head h*g + r % g)
    const size_t qrow_lo = lo_ok ? static_cast<size_t>(r_lo / g) * P.num_q_heads + h * g + r_lo % g : 0;
    const size_t qrow_hi = hi_ok ? static_cast<size_t>(r_hi / g) * P.num_q_heads + h * g + r_hi % g : 0;
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(P.q);
    const uint32_t* q_lo = reinterpret_cast<const uint32_t*>(qb + qrow_lo * D + tq);
    const uint32_t* q_hi = reinterpret_cast<const uint32_t*>(qb + qrow_hi * D + tq);
    uint32_t qa[KSTEPS][4];
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
        qa[ks][0] = lo_ok ? __ldg(q_lo + ks * 8) : 0u;
        qa[ks][1] = hi_ok ? __ldg(q_hi + ks * 8) : 0u;
        qa[ks][2] = lo_ok ? __ldg(q_lo + ks * 8 + 4) : 0u;
        qa[ks][3] = hi_ok ? __ldg(q_hi + ks * 8 + 4) : 0u;
    }
    float m_lo = -INFINITY, l_lo = 0.f, m_hi = -INFINITY, l_hi = 0.f;
    float acc[NTD][4];
#pragma unroll
    for (int n = 0; n < NTD; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    const float sl2 = P.scale_log2;

    const int nst = (nblk + kPrefixBlocksPerStage - 1) / kPrefixBlocksPerStage;
    for (int n = 0; n < nst; ++n) {
        const int st = n % S;
        if (!mbar_wait_bounded(full_u32 + st * 8, (n / S) & 1u)) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            return;
        }
        const int32_t mask = oob[st];
        const uint32_t sbase = ring_u32 + st * Cfg::kStageBytes;
        // ---- S = Q K^T over 32 keys: n-tiles 0,1 from block 0, 2,3 from block 1
        float sc[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t) sc[t][0] = sc[t][1] = sc[t][2] = sc[t][3] = 0.f;
#pragma unroll
        for (int b = 0; b < kPrefixBlocksPerStage; ++b) {
            if (mask & (1 << b)) continue;  // warp-uniform
            const uint32_t kbase = sbase + b * Cfg::kTileBytes;
#pragma unroll
            for (int kp = 0; kp < KSTEPS / 2; ++kp) {
                const int cg = 4 * kp + (lane >> 3);
                const uint32_t col = (cg >> 3) * 2048 + ((((uint32_t)cg & 7u) ^ sw) << 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kbase + col + (lane & 7) * 128, b0, b1, b2, b3);
                mma_frag(sc[2 * b], qa[2 * kp], b0, b1);
                mma_frag(sc[2 * b], qa[2 * kp + 1], b2, b3);
                ldsm_x4(kbase + col + (8 + (lane & 7)) * 128, b0, b1, b2, b3);
                mma_frag(sc[2 * b + 1], qa[2 * kp], b0, b1);
                mma_frag(sc[2 * b + 1], qa[2 * kp + 1], b2, b3);
            }
        }
        // ---- online softmax of rows r_lo (accumulator regs 0,1) and r_hi (2,3)
        const bool m0 = (mask & 1) != 0, m1 = (mask & 2) != 0;
        float xl[8], xh[8];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const bool dead = t < 2 ? m0 : m1;
            xl[2 * t] = dead ? -INFINITY : sc[t][0] * sl2;
            xl[2 * t + 1] = dead ? -INFINITY : sc[t][1] * sl2;
            xh[2 * t] = dead ? -INFINITY : sc[t][2] * sl2;
            xh[2 * t + 1] = dead ? -INFINITY : sc[t][3] * sl2;
        }
        uint32_t pl[4], ph[4];
        const float alpha_lo = softmax_update32(m_lo, l_lo, xl, pl);
        const float alpha_hi = softmax_update32(m_hi, l_hi, xh, ph);
        if (__any_sync(kFullMask, alpha_lo != 1.f || alpha_hi != 1.f)) {  // a row max moved
#pragma unroll
            for (int k = 0; k < NTD; ++k) {
                acc[k][0] *= alpha_lo;
                acc[k][1] *= alpha_lo;
                acc[k][2] *= alpha_hi;
                acc[k][3] *= alpha_hi;
            }
        }
        // ---- O += P V, one k-step of 16 keys per present block
#pragma unroll
        for (int b = 0; b < kPrefixBlocksPerStage; ++b) {
            if (mask & (1 << b)) continue;
            const uint32_t pa[4] = {pl[2 * b], ph[2 * b], pl[2 * b + 1], ph[2 * b + 1]};
            const uint32_t vbase = sbase + (kPrefixBlocksPerStage + b) * Cfg::kTileBytes;
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                const int cg = 2 * dp + (lane >> 4);
                const int t = 8 * ((lane >> 3) & 1) + (lane & 7);
                const uint32_t addr = vbase + (cg >> 3) * 2048 + t * 128 + ((((uint32_t)cg & 7u) ^ sw) << 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_trans(addr, b0, b1, b2, b3);
                mma_frag(acc[2 * dp], pa, b0, b1);
                mma_frag(acc[2 * dp + 1], pa, b2, b3);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_u32 + st * 8);  // this warp is done with the stage
    }

    // ---------------- the split's partial of every valid row
    constexpr float kLn2 = 0.693147180559945309f;
    float lt_lo = l_lo + __shfl_xor_sync(kFullMask, l_lo, 1);
    lt_lo += __shfl_xor_sync(kFullMask, lt_lo, 2);
    float lt_hi = l_hi + __shfl_xor_sync(kFullMask, l_hi, 1);
    lt_hi += __shfl_xor_sync(kFullMask, lt_hi, 2);
    if (lo_ok) {
        const size_t idx = qrow_lo * P.max_parts + split;
        if ((lane & 3) == 0) {
            P.ws_m[idx] = m_lo * kLn2;
            P.ws_l[idx] = lt_lo;
        }
        float* a = P.ws_acc + idx * D + tq;
#pragma unroll
        for (int n = 0; n < NTD; ++n) *reinterpret_cast<float2*>(a + 8 * n) = make_float2(acc[n][0], acc[n][1]);
    }
    if (hi_ok) {
        const size_t idx = qrow_hi * P.max_parts + split;
        if ((lane & 3) == 0) {
            P.ws_m[idx] = m_hi * kLn2;
            P.ws_l[idx] = lt_hi;
        }
        float* a = P.ws_acc + idx * D + tq;
#pragma unroll
        for (int n = 0; n < NTD; ++n) *reinterpret_cast<float2*>(a + 8 * n) = make_float2(acc[n][2], acc[n][3]);
    }
}

}  // namespace pa
