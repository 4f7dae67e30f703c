// lse_reduce.cuh -- log-sum-exp merge of split-K decode partials.
//
// A sequence longer than one partition is processed as independent work items
// over consecutive block ranges; each leaves (m_p, l_p, acc_p): its maximum
// score, sum of exp(score - m_p) and the matching unnormalised sum of V rows.
// The exact softmax over the whole sequence is recovered as
//   M = max_p m_p,  out = sum_p e^(m_p - M) acc_p / sum_p e^(m_p - M) l_p,
// which is the standard identity behind splitting attention over key ranges
// (the pages do not describe the split; long sequences are where paged KV
// matters most: "PagedAttention et vLLM", aiunderstanding.org,
// §"L'avenir de PagedAttention et vLLM").
//
// A warp merges one (sequence, query head) row: lanes read the pieces' m and
// l in parallel, then accumulate the pieces' acc rows (lanes across head dims,
// 16-byte loads, eight pieces in flight).  Two kernels choose the rows: the
// row-wise one (fixed partitions, shared prefix) and the boundary-walking one
// (balanced split).
#pragma once

#include "items.cuh"

namespace pa {

constexpr int kReduceWarps = 4;

template <typename T>
__device__ __forceinline__ T from_float(float x);
template <>
__device__ __forceinline__ float from_float<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// The pieces of a row: `n1` partials at indices 0 .. n1-1 (after `base`),
// then `n2` at off2 .. off2+n2-1 (a shared prefix's key chunks, then the
// decode's pieces of the private part, which start at a fixed index).
struct RowPieces {
    int n1, off2, n2;
    __device__ __forceinline__ int count() const { return n1 + n2; }
    __device__ __forceinline__ int index(int p) const { return p < n1 ? p : off2 + (p - n1); }
};

// One warp merges one row (sequence, query head) from its pieces (partial
// indices after `base`); lanes hold D/32 consecutive head dims.  The first 32
// pieces' m and l (one per lane) and the first kPre pieces' acc slices are
// loaded together, so a row of up to kPre pieces costs one round trip to L2
// before the arithmetic; the sums run in the same order as a plain loop.
template <typename OutT, int D>
__device__ __forceinline__ void merge_row_warp(const DecodeParams& P, size_t base, RowPieces pcs,
                                               OutT* o, int lane) {
    constexpr int DPL = D / 32;
    constexpr int kPre = 8;
    using Vec = typename std::conditional<DPL == 4, float4, float2>::type;
    const float* wm = P.ws_m + base;
    const float* wl = P.ws_l + base;
    const float* wa = P.ws_acc + base * D + lane * DPL;
    const int parts = pcs.count();
    float m0 = -INFINITY, l0 = 0.f;  // piece `lane`'s max and sum
    if (lane < parts) {
        const int p = pcs.index(lane);
        m0 = wm[p];
        l0 = wl[p];
    }
    Vec pre[kPre];
#pragma unroll
    for (int q = 0; q < kPre; ++q)
        if (q < parts) pre[q] = *reinterpret_cast<const Vec*>(wa + static_cast<size_t>(pcs.index(q)) * D);
    float M = m0;
    for (int p = lane + 32; p < parts; p += 32) M = fmaxf(M, wm[pcs.index(p)]);
    M = warp_max(M);
    if (M == -INFINITY) {  // every piece fully masked, or none
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[lane * DPL + e] = from_float<OutT>(0.f);
        return;
    }
    float den = lane < parts ? expf(m0 - M) * l0 : 0.f;
    for (int p = lane + 32; p < parts; p += 32) den += expf(wm[pcs.index(p)] - M) * wl[pcs.index(p)];
    den = warp_sum(den);
    // weight of piece q (warp-uniform q): its max from lane q, or from memory past 32
    auto weight = [&](int q) {
        const float mq = q < 32 ? __shfl_sync(kFullMask, m0, q & 31) : wm[pcs.index(q)];
        return expf(mq - M);
    };
    float a[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) a[e] = 0.f;
#pragma unroll
    for (int q = 0; q < kPre; ++q) {
        if (q < parts) {
            const float w = weight(q);
            const float* f = reinterpret_cast<const float*>(&pre[q]);
#pragma unroll
            for (int e = 0; e < DPL; ++e) a[e] = fmaf(w, f[e], a[e]);
        }
    }
#pragma unroll 8
    for (int q = kPre; q < parts; ++q) {
        const float w = weight(q);
        const Vec x = *reinterpret_cast<const Vec*>(wa + static_cast<size_t>(pcs.index(q)) * D);
        const float* f = reinterpret_cast<const float*>(&x);
#pragma unroll
        for (int e = 0; e < DPL; ++e) a[e] = fmaf(w, f[e], a[e]);
    }
    const float inv = den > 0.f ? 1.0f / den : 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[lane * DPL + e] = from_float<OutT>(a[e] * inv);
}

// The (sequence, query head, query-token row) of output row `row` of a
// launch: rows are sequence-major without q_start, token-row-major with it
// (the sequence then found by binary search over q_start).  Returns false
// when the row was not computed (a token beyond the clamped count).
struct RowRef {
    int32_t s, qh;
    size_t r;     // output row (query token row * Hq + qh)
    int32_t len;  // the sequence's (clamped) length
    int32_t tok;  // query token within the sequence, of
    int32_t n;    // its query tokens
};

__device__ __forceinline__ bool locate_row(const DecodeParams& P, int64_t row, RowRef* R) {
    if (!P.q_start) {
        R->s = P.seq_begin + static_cast<int32_t>(row / P.num_q_heads);
        R->qh = static_cast<int32_t>(row % P.num_q_heads);
        R->r = static_cast<size_t>(R->s) * P.num_q_heads + R->qh;
        R->len = 0;
        R->tok = 0;
        R->n = 1;
        return true;
    }
    const int32_t t = static_cast<int32_t>(row / P.num_q_heads);
    R->qh = static_cast<int32_t>(row % P.num_q_heads);
    R->s = upper_index(P.num_seqs, t, [&](int k) { return static_cast<int64_t>(__ldg(P.q_start + k)); });
    R->r = static_cast<size_t>(row);
    R->len = seq_geometry(P, P.seq_lens[R->s], 0).len;
    const QRows qr = query_rows(P, R->s, R->len);
    R->tok = t - qr.base;
    R->n = qr.n;
    return R->tok < qr.n;
}

// Which partials row R merges; false when the row needs no merge (its one
// piece was written as the final row by the decode).
__device__ __forceinline__ bool row_pieces(const DecodeParams& P, const RowRef& R, RowPieces* pcs) {
    if (P.tile_chunk > 0) {  // a prefill row of the tile kernel: its tile's key chunks
        *pcs = RowPieces{prefill_row_pieces(R.len, R.n, R.tok, P.tile_tokens, P.tile_chunk), 0, 0};
        return true;
    }
    const int32_t skip = seq_skip(P, R.s);
    const SeqGeom geo = seq_geometry(P, P.seq_lens[R.s], skip);
    const int own = geo.work > 0 ? P.ws_parts[static_cast<size_t>(R.s) * P.num_kv_heads + R.qh / P.group] : 0;
    if (P.group_start) {  // several prompt groups: this group's prefix chunks, then the own pieces
        const int pre = (skip + P.group_chunk - 1) / P.group_chunk;
        *pcs = RowPieces{pre, P.piece_base, own};
        return true;
    }
    *pcs = RowPieces{P.piece_base + own, 0, 0};
    return !(P.piece_base == 0 && own <= 1);
}

// Row-wise merge (fixed partitions, or a shared prefix): one warp per
// (sequence, query head) row, four rows per CTA.  The pieces of a row are
// piece_base partials written by another kernel (a shared prefix's key
// splits) followed by the decode kernel's pieces of blocks [first, nb), whose
// number the decode recorded in ws_parts.  Rows with a single piece of their
// own and nothing before it were written by the decode and are skipped.
template <typename OutT, int D>
__global__ void __launch_bounds__(kReduceWarps * 32) lse_reduce_kernel(const DecodeParams P) {
    grid_dependency_wait();  // the partials of the decode launched just before
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kReduceWarps + warp;
    const int64_t rows = static_cast<int64_t>(P.q_start ? P.num_q_rows : P.seq_count) * P.num_q_heads;
    if (row >= rows) return;
    RowRef R;
    if (!locate_row(P, row, &R)) return;
    RowPieces pcs;
    if (!row_pieces(P, R, &pcs)) return;
    merge_row_warp<OutT, D>(P, R.r * P.max_parts, pcs, static_cast<OutT*>(P.out) + R.r * D, lane);
}

// Row-wise merge for rows with many pieces (long sequences in fixed
// partitions): one CTA of kWideWarps warps per row.  The pieces' weights
// e^(m_p - M) are computed once, into shared memory, while the row sum is
// taken; the warps then split the pieces and accumulate their acc rows with
// eight 16-byte loads in flight per warp, and the warps' sums are added in a
// fixed order.
constexpr int kWideWarps = 8;
constexpr int kWideWeights = 1024;  // pieces whose weight is kept in shared memory
template <typename OutT, int D>
__global__ void __launch_bounds__(kWideWarps * 32) lse_reduce_wide_kernel(const DecodeParams P) {
    constexpr int DPL = D / 32;
    using Vec = typename std::conditional<DPL == 4, float4, float2>::type;
    __shared__ float wts[kWideWeights];
    __shared__ float red[kWideWarps][D];
    __shared__ float wmax[kWideWarps], wden[kWideWarps];
    grid_dependency_wait();
    RowRef R;
    if (!locate_row(P, blockIdx.x, &R)) return;
    RowPieces pcs;
    if (!row_pieces(P, R, &pcs)) return;
    const int parts = pcs.count();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t base = R.r * P.max_parts;
    const float* wm = P.ws_m + base;
    const float* wl = P.ws_l + base;
    const float* wa = P.ws_acc + base * D;
    float M = -INFINITY;
    for (int p = tid; p < parts; p += blockDim.x) M = fmaxf(M, wm[pcs.index(p)]);
    M = warp_max(M);
    if (lane == 0) wmax[warp] = M;
    __syncthreads();
    M = wmax[0];
#pragma unroll
    for (int w = 1; w < kWideWarps; ++w) M = fmaxf(M, wmax[w]);
    OutT* o = static_cast<OutT*>(P.out) + R.r * D;
    if (M == -INFINITY) {
        for (int d = tid; d < D; d += blockDim.x) o[d] = from_float<OutT>(0.f);
        return;
    }
    float den = 0.f;
    for (int p = tid; p < parts; p += blockDim.x) {
        const float w = expf(wm[pcs.index(p)] - M);
        if (p < kWideWeights) wts[p] = w;
        den += w * wl[pcs.index(p)];
    }
    den = warp_sum(den);
    if (lane == 0) wden[warp] = den;
    __syncthreads();  // the weights and the warps' sums
    float a[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) a[e] = 0.f;
#pragma unroll 8
    for (int p = warp; p < parts; p += kWideWarps) {
        const float w = p < kWideWeights ? wts[p] : expf(wm[pcs.index(p)] - M);
        const Vec x = *reinterpret_cast<const Vec*>(wa + static_cast<size_t>(pcs.index(p)) * D + lane * DPL);
        const float* f = reinterpret_cast<const float*>(&x);
#pragma unroll
        for (int e = 0; e < DPL; ++e) a[e] = fmaf(w, f[e], a[e]);
    }
#pragma unroll
    for (int e = 0; e < DPL; ++e) red[warp][lane * DPL + e] = a[e];
    __syncthreads();
    den = 0.f;
#pragma unroll
    for (int w = 0; w < kWideWarps; ++w) den += wden[w];
    const float inv = den > 0.f ? 1.0f / den : 0.f;
    for (int d = tid; d < D; d += blockDim.x) {
        float x = 0.f;
#pragma unroll
        for (int w = 0; w < kWideWarps; ++w) x += red[w][d];
        o[d] = from_float<OutT>(x * inv);
    }
}

// Balanced split: only units that cross a boundary between two decode warps'
// ranges were cut, so the merge walks those boundaries instead of every row.
// CTA b looks at the boundary between decode warps b and b + 1 (stream
// position (b + 1) * C, with C recomputed exactly as the decode did from the
// same lengths and the decode's warp count).  If a unit crosses it and this is
// the unit's first boundary, the CTA's warps merge the unit's query rows.
template <typename OutT, int D>
__global__ void __launch_bounds__(kReduceWarps * 32)
lse_reduce_balanced_kernel(const DecodeParams P, int32_t decode_warps) {
    extern __shared__ int32_t smem_i[];
    int32_t* prefix = smem_i;
    int32_t* lens = prefix + P.seq_count + 1;
    int32_t* skips = lens + P.seq_count;
    // the lengths are input no kernel of this library writes: the prefix is
    // built while the decode launched just before still runs
    const int32_t total = build_prefix(P, prefix, lens, skips);  // blocks per sequence
    grid_dependency_wait();  // the decode's partials
    const int64_t hk = P.num_kv_heads;
    const int64_t T = static_cast<int64_t>(total) * hk;
    const int64_t even = (T + decode_warps - 1) / decode_warps;
    const int64_t C = even > P.min_chunk ? even : P.min_chunk;
    const int64_t b = (static_cast<int64_t>(blockIdx.x) + 1) * C;
    if (b >= T) return;
    const int i = upper_index(P.seq_count, b, [&](int k) { return hk * prefix[k]; });
    const SeqGeom geo = seq_geometry(P, lens[i], skips[i]);
    const int64_t off = b - hk * prefix[i];
    const int32_t h = static_cast<int32_t>(off / geo.work);
    const int64_t j = off - static_cast<int64_t>(h) * geo.work;
    if (j == 0) return;  // a unit starts exactly here: nothing crosses
    const int64_t ustart = b - j;
    if (ustart / C != blockIdx.x) return;  // merged at the unit's first boundary
    const int64_t uend = ustart + geo.work;
    const int parts = static_cast<int>((uend - 1) / C - ustart / C + 1);
    const int32_t s = P.seq_begin + i;
    const QRows qr = query_rows(P, s, geo.len);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp; r < P.group * qr.n; r += kReduceWarps) {  // (query token, head) rows
        const size_t row = (static_cast<size_t>(qr.base) + r / P.group) * P.num_q_heads +
                           h * P.group + r % P.group;
        merge_row_warp<OutT, D>(P, row * P.max_parts, RowPieces{parts, 0, 0}, static_cast<OutT*>(P.out) + row * D,
                                lane);
    }
}

}  // namespace pa
