// items.cuh -- how a decode launch cuts its sequences into work items.
//
// A work item is (sequence s, partition p, kv head h): the blocks
// [p*part_blocks, min((p+1)*part_blocks, nb_s)) of sequence s, seen through
// kv head h, for all query heads of that head's group.  Items are numbered
// sequence-major, then partition, then kv head, so consecutive warps stream
// neighbouring head slices of the same physical blocks.  Every CTA of a launch
// builds the exclusive prefix sum of items per sequence in shared memory once
// and then maps an item number to (s, p, h) by binary search.
#pragma once

#include "common.cuh"

namespace pa {

struct SeqGeom {
    int32_t len;    // tokens attended (clamped)
    int32_t nb;     // blocks: ceil(len / 16)
    int32_t parts;  // partitions: ceil(nb / part_blocks), 0 for an empty sequence
};

__device__ __forceinline__ SeqGeom seq_geometry(const DecodeParams& P, int32_t len) {
    SeqGeom g;
    if (len < 0) len = 0;
    if (len > P.len_cap) len = P.len_cap;
    g.len = len;
    g.nb = (len + kBlockTokens - 1) / kBlockTokens;
    g.parts = g.nb == 0 ? 0 : 1 + (g.nb - 1) / P.part_blocks;
    return g;
}

__device__ __forceinline__ int32_t load_len_checked(const DecodeParams& P, int32_t s, bool report) {
    int32_t len = P.seq_lens[s];
    if (report && (len < 0 || len > P.len_cap)) flag_error(PA_DEVERR_SEQ_LEN);
    return len;
}

// Builds prefix[0..n] (items before each sequence of the launch, prefix[n] =
// total) and lens[0..n) (clamped lengths) in shared memory.  All threads of
// the CTA must call it.  Returns the total number of items.
__device__ __forceinline__ int32_t build_item_prefix(const DecodeParams& P, int32_t* prefix,
                                                     int32_t* lens) {
    __shared__ int32_t warp_tot[32];
    const int n = P.seq_count;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int per = (n + nthr - 1) / nthr;
    const int beg = min(n, tid * per), end = min(n, beg + per);
    // only CTA 0 reports bad lengths, so each bad length is counted once
    const bool report = blockIdx.x == 0;
    int32_t local = 0;
    for (int i = beg; i < end; ++i) {
        SeqGeom g = seq_geometry(P, load_len_checked(P, P.seq_begin + i, report));
        lens[i] = g.len;
        local += g.parts * P.num_kv_heads;
    }
    // exclusive scan of `local` over the CTA
    const int lane = tid & 31, warp = tid >> 5, nwarps = (nthr + 31) >> 5;
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int32_t v = __shfl_up_sync(kFullMask, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t t = lane < nwarps ? warp_tot[lane] : 0;
        int32_t ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t v = __shfl_up_sync(kFullMask, ti, o);
            if (lane >= o) ti += v;
        }
        warp_tot[lane] = ti - t;  // exclusive
    }
    __syncthreads();
    int32_t run = warp_tot[warp] + incl - local;
    for (int i = beg; i < end; ++i) {
        prefix[i] = run;
        SeqGeom g = seq_geometry(P, lens[i]);
        run += g.parts * P.num_kv_heads;
    }
    if (tid == nthr - 1) prefix[n] = run;  // last thread holds the grand total
    __syncthreads();
    return prefix[n];
}

struct Item {
    int32_t s;       // sequence (global index)
    int32_t h;       // kv head
    int32_t p;       // partition
    int32_t len;     // tokens of the sequence
    int32_t parts;   // partitions of the sequence
    int32_t jbeg;    // first block of the item
    int32_t jend;    // one past its last block
};

// Item number -> (s, p, h).  Warp-uniform; reads the shared prefix.
__device__ __forceinline__ Item decode_item(const DecodeParams& P, const int32_t* prefix,
                                            const int32_t* lens, int32_t item) {
    int lo = 0, hi = P.seq_count;  // prefix[lo] <= item < prefix[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= item) lo = mid;
        else hi = mid;
    }
    Item it;
    const int32_t r = item - prefix[lo];
    it.p = r / P.num_kv_heads;
    it.h = r - it.p * P.num_kv_heads;
    it.s = P.seq_begin + lo;
    SeqGeom g = seq_geometry(P, lens[lo]);
    it.len = g.len;
    it.parts = g.parts;
    it.jbeg = it.p * P.part_blocks;
    it.jend = min(g.nb, it.jbeg + P.part_blocks);
    return it;
}

// Zero-length sequences have no items; their rows of `out` are zero.  CTA b
// clears those of the sequences s = b, b + gridDim.x, ... of the launch.
template <typename OutT>
__device__ __forceinline__ void zero_empty_sequences(const DecodeParams& P, const int32_t* lens) {
    const int row = P.num_q_heads * P.head_dim;
    for (int i = blockIdx.x; i < P.seq_count; i += gridDim.x) {
        if (lens[i] != 0) continue;
        OutT* o = static_cast<OutT*>(P.out) + static_cast<size_t>(P.seq_begin + i) * row;
        for (int e = threadIdx.x; e < row; e += blockDim.x) o[e] = OutT(0.0f);
    }
}

}  // namespace pa
