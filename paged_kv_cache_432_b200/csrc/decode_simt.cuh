// decode_simt.cuh -- paged decode attention, fp32, on the CUDA cores.
//
// The fp32 path must stay within 1e-5 of an fp64 reference, so it keeps
// every product in fp32 FMA and uses the accurate expf; tensor cores (tf32)
// would not meet that.  Same work items and output/partial format as the
// bf16 kernel (items.cuh): one warp per (sequence, partition, kv head),
// lanes across head dims (2 or 4 consecutive floats each, so a token row is
// one coalesced 256/512-byte load), block ids read 32 at a time from the
// block table.  Per 16-token block: scores of the valid tokens for every
// query head of the group (warp butterfly sums, identical in all lanes), one
// online-softmax rescale per block, then P V from the V rows.  Tokens past the
// sequence length are never loaded.
#pragma once

#include "items.cuh"

namespace pa {

constexpr int kSimtWarps = 4;

template <int D, int MAXG>
__global__ void __launch_bounds__(kSimtWarps * 32)
decode_f32_simt_kernel(const DecodeParams P) {
    constexpr int DPL = D / 32;  // dims per lane
    using Vec = typename std::conditional<DPL == 4, float4, float2>::type;
    extern __shared__ int32_t smem_i[];
    __shared__ float pbuf[kSimtWarps][MAXG][kBlockTokens];
    int32_t* prefix = smem_i;
    int32_t* lens = prefix + P.seq_count + 1;
    grid_dependency_wait();  // global memory only once the previous kernel is done
    allow_dependents();
    const Schedule sched = make_schedule(P, prefix, kSimtWarps);
    zero_empty_sequences<float>(P, lens);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = P.group;
    const int Hkv = P.num_kv_heads;
    const float* kc = static_cast<const float*>(P.k_cache);
    const float* vc = static_cast<const float*>(P.v_cache);

    Cursor it;
    for (sched.start(it, blockIdx.x * kSimtWarps + warp); it.valid; sched.next(it)) {
        const float* qg = static_cast<const float*>(P.q) +
                          (static_cast<size_t>(it.s) * P.num_q_heads + it.h * g) * D + lane * DPL;
        float q[MAXG][DPL], acc[MAXG][DPL], m[MAXG], l[MAXG];
#pragma unroll
        for (int i = 0; i < MAXG; ++i) {
#pragma unroll
            for (int e = 0; e < DPL; ++e) {
                q[i][e] = i < g ? qg[i * D + e] : 0.f;
                acc[i][e] = 0.f;
            }
            m[i] = -INFINITY;
            l[i] = 0.f;
        }

        int32_t tbl = 0, tbase = it.jbeg - 32;
        for (int32_t j = it.jbeg; j < it.jend; ++j) {
            if (j >= tbase + 32) {
                tbase = j;
                const int32_t jj = tbase + lane;
                tbl = jj < it.jend
                          ? P.block_tables[static_cast<size_t>(it.s) * P.max_blocks_per_seq + jj]
                          : 0;
            }
            const int32_t pb = __shfl_sync(kFullMask, tbl, j - tbase);
            if (static_cast<uint32_t>(pb) >= static_cast<uint32_t>(P.num_blocks)) {
                if (lane == 0) flag_error(PA_DEVERR_BLOCK_OOB);
                continue;  // the whole block is masked
            }
            const int valid = min(kBlockTokens, it.len - j * kBlockTokens);
            const size_t base = (static_cast<size_t>(pb) * Hkv + it.h) * kBlockTokens * D + lane * DPL;
            float kr[kBlockTokens][DPL];
#pragma unroll
            for (int t = 0; t < kBlockTokens; ++t) {
                if (t < valid) {
                    const Vec v4 = *reinterpret_cast<const Vec*>(kc + base + t * D);
                    const float* f = reinterpret_cast<const float*>(&v4);
#pragma unroll
                    for (int e = 0; e < DPL; ++e) kr[t][e] = f[e];
                } else {
#pragma unroll
                    for (int e = 0; e < DPL; ++e) kr[t][e] = 0.f;
                }
            }
#pragma unroll
            for (int i = 0; i < MAXG; ++i) {
                if (i >= g) break;
                float sc[kBlockTokens];
                float bm = -INFINITY;
#pragma unroll
                for (int t = 0; t < kBlockTokens; ++t) {
                    float d = 0.f;
#pragma unroll
                    for (int e = 0; e < DPL; ++e) d = fmaf(q[i][e], kr[t][e], d);
                    d = warp_sum(d);
                    sc[t] = t < valid ? d * P.scale : -INFINITY;
                    bm = fmaxf(bm, sc[t]);
                }
                const float mn = fmaxf(m[i], bm);  // finite: valid >= 1
                const float alpha = expf(m[i] - mn);
                float ps = 0.f;
#pragma unroll
                for (int t = 0; t < kBlockTokens; ++t) {
                    const float p = t < valid ? expf(sc[t] - mn) : 0.f;
                    ps += p;
                    if (lane == t) pbuf[warp][i][t] = p;
                }
                l[i] = l[i] * alpha + ps;
                m[i] = mn;
#pragma unroll
                for (int e = 0; e < DPL; ++e) acc[i][e] *= alpha;
            }
            __syncwarp();
            for (int t = 0; t < valid; ++t) {
                const Vec v4 = *reinterpret_cast<const Vec*>(vc + base + t * D);
                const float* f = reinterpret_cast<const float*>(&v4);
#pragma unroll
                for (int i = 0; i < MAXG; ++i) {
                    if (i >= g) break;
                    const float p = pbuf[warp][i][t];
#pragma unroll
                    for (int e = 0; e < DPL; ++e) acc[i][e] = fmaf(p, f[e], acc[i][e]);
                }
            }
            __syncwarp();
        }

        if (it.parts == 1 && P.piece_base == 0) {
            float* o = static_cast<float*>(P.out) +
                       (static_cast<size_t>(it.s) * P.num_q_heads + it.h * g) * D + lane * DPL;
#pragma unroll
            for (int i = 0; i < MAXG; ++i) {
                if (i >= g) break;
                const float inv = l[i] > 0.f ? 1.0f / l[i] : 0.f;
#pragma unroll
                for (int e = 0; e < DPL; ++e) o[i * D + e] = acc[i][e] * inv;
            }
        } else {
#pragma unroll
            for (int i = 0; i < MAXG; ++i) {
                if (i >= g) break;
                const size_t idx =
                    (static_cast<size_t>(it.s) * P.num_q_heads + it.h * g + i) * P.max_parts + P.piece_base + it.p;
                if (lane == 0) {
                    P.ws_m[idx] = m[i];
                    P.ws_l[idx] = l[i];
                }
#pragma unroll
                for (int e = 0; e < DPL; ++e) P.ws_acc[idx * D + lane * DPL + e] = acc[i][e];
            }
        }
        record_parts(P, it, lane);
    }
}

}  // namespace pa
