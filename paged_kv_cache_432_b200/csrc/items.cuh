// items.cuh -- how a decode launch cuts its sequences into pieces of work.
//
// A unit is (sequence s, kv head h): the ceil(len_s / 16) blocks of s seen
// through kv head h, for all query heads of that head's group.  A piece is a
// run of consecutive blocks of one unit; one warp processes it and writes
// either the final rows (the piece is the whole unit) or the piece's partial
// (m, l, acc) for the log-sum-exp reduction.  Two ways to cut:
//
//  * balanced (partition_blocks = 0): the blocks of all units form one stream,
//    units ordered sequence-major then kv head (so neighbouring warps read
//    neighbouring head slices of the same physical blocks), and warp w takes
//    stream positions [w*C, (w+1)*C) with C = max(min_chunk, ceil(total / warps)).
//    Every warp gets the same number of blocks (+-1), whatever the length mix;
//    a unit that crosses a warp boundary becomes several pieces.  Piece p of a
//    unit is the part that falls in the unit's p-th warp range.
//  * fixed (partition_blocks > 0, or "never split"): piece p of a unit is
//    blocks [p*PB, (p+1)*PB); pieces are numbered sequence-major, then piece,
//    then kv head, and handed out round-robin over the warps.
//
// Every CTA builds a prefix sum over the launch's sequences in shared memory
// once (blocks per sequence, or pieces per sequence) and then locates any
// stream position or piece number by binary search.  The prefix and the
// clamped lengths take 8 bytes of shared memory per sequence.
#pragma once

#include "common.cuh"

namespace pa {

struct SeqGeom {
    int32_t len;    // tokens attended (clamped)
    int32_t nb;     // blocks: ceil(len / 16)
    int32_t first;  // first block the pieces cover (skip_blocks, at most nb)
    int32_t work;   // blocks the pieces cover: nb - first
    int32_t parts;  // fixed mode: ceil(work / part_blocks); 0 when there is no work
};

// `skip`: the leading blocks of the sequence that other kernels cover (a
// shared prefix), from seq_skip.
__device__ __forceinline__ SeqGeom seq_geometry(const DecodeParams& P, int32_t len, int32_t skip) {
    SeqGeom g;
    if (len < 0) len = 0;
    if (len > P.len_cap) len = P.len_cap;
    g.len = len;
    g.nb = (len + kBlockTokens - 1) / kBlockTokens;
    g.first = min(skip, g.nb);
    g.work = g.nb - g.first;
    g.parts = g.work == 0 ? 0 : 1 + (g.work - 1) / P.part_blocks;
    return g;
}

// Largest s in [0, n) with key(s) <= x, where key is non-decreasing and
// key(0) <= x < key(n).
template <typename Key>
__device__ __forceinline__ int upper_index(int n, int64_t x, Key key) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (key(mid) <= x) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Prefix group of sequence s (several prompt groups: group i is sequences
// group_start[i] .. group_start[i+1]-1).
__device__ __forceinline__ int32_t seq_group(const DecodeParams& P, int32_t s) {
    return upper_index(P.num_groups, s, [&](int k) { return static_cast<int64_t>(__ldg(P.group_start + k)); });
}

// Shared blocks of a group, within [0, max_shared] (larger values are clamped;
// the tile kernel flags them).
__device__ __forceinline__ int32_t group_shared(const DecodeParams& P, int32_t grp) {
    return max(0, min(__ldg(P.group_blocks + grp), P.max_shared));
}

// Leading blocks of sequence s that a shared-prefix kernel covers.
__device__ __forceinline__ int32_t seq_skip(const DecodeParams& P, int32_t s) {
    return P.group_start ? group_shared(P, seq_group(P, s)) : P.skip_blocks;
}

// Builds prefix[0..n] (exclusive sums of the per-sequence quantity: blocks in
// balanced mode, pieces x kv heads in fixed mode; prefix[n] = total), lens[0..n)
// (clamped lengths) and skips[0..n) (leading blocks covered elsewhere) in
// shared memory.  All threads of the CTA must call it.  Returns the total.
__device__ __forceinline__ int32_t build_prefix(const DecodeParams& P, int32_t* prefix,
                                                int32_t* lens, int32_t* skips) {
    __shared__ int32_t warp_tot[32];
    const int n = P.seq_count;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int per = (n + nthr - 1) / nthr;
    const int beg = min(n, tid * per), end = min(n, beg + per);
    // only CTA 0 reports bad lengths, so each is counted once per launch
    const bool report = blockIdx.x == 0;
    int32_t local = 0;
    for (int i = beg; i < end; ++i) {
        const int32_t raw = P.seq_lens[P.seq_begin + i];
        if (report && (raw < 0 || raw > P.len_cap)) flag_error(PA_DEVERR_SEQ_LEN);
        skips[i] = seq_skip(P, P.seq_begin + i);
        const SeqGeom g = seq_geometry(P, raw, skips[i]);
        lens[i] = g.len;
        local += P.balanced ? g.work : g.parts * P.num_kv_heads;
    }
    const int lane = tid & 31, warp = tid >> 5, nwarps = (nthr + 31) >> 5;
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(kFullMask, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int32_t t = lane < nwarps ? warp_tot[lane] : 0;
        int32_t ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(kFullMask, ti, o);
            if (lane >= o) ti += v;
        }
        warp_tot[lane] = ti - t;  // exclusive
    }
    __syncthreads();
    int32_t run = warp_tot[warp] + incl - local;
    for (int i = beg; i < end; ++i) {
        prefix[i] = run;
        const SeqGeom g = seq_geometry(P, lens[i], skips[i]);
        run += P.balanced ? g.work : g.parts * P.num_kv_heads;
    }
    if (tid == nthr - 1) prefix[n] = run;  // the last thread ends on the grand total
    __syncthreads();
    return prefix[n];
}

// Iterates the pieces one warp owns.  Warp-uniform.
struct Cursor {
    // the current piece
    bool valid;
    int32_t s;      // sequence (global index)
    int32_t h;      // kv head
    int32_t p;      // piece index within its unit
    int32_t parts;  // pieces of the unit
    int32_t len;    // tokens of the sequence
    int32_t jbeg;   // first block of the piece
    int32_t jend;   // one past its last block
    // iteration state
    int32_t item;    // fixed mode: piece number
    int64_t pos;     // balanced mode: stream position of the current piece
    int64_t end;     // balanced mode: end of this warp's range
    int64_t chunk;   // balanced mode: C
};

struct Schedule {
    const DecodeParams* P;
    const int32_t* prefix;
    const int32_t* lens;
    const int32_t* skips;
    int32_t total;  // blocks (balanced) or pieces (fixed)
    int64_t chunk;  // balanced: blocks per warp range
    int32_t nw;     // warps in the grid

    __device__ __forceinline__ void locate_fixed(Cursor& c) const {
        const int n = P->seq_count;
        const int i = upper_index(n, c.item, [&](int k) { return (int64_t)prefix[k]; });
        const int32_t r = c.item - prefix[i];
        c.p = r / P->num_kv_heads;
        c.h = r - c.p * P->num_kv_heads;
        c.s = P->seq_begin + i;
        const SeqGeom g = seq_geometry(*P, lens[i], skips[i]);
        c.len = g.len;
        c.parts = g.parts;
        c.jbeg = g.first + c.p * P->part_blocks;
        c.jend = min(g.nb, c.jbeg + P->part_blocks);
    }

    __device__ __forceinline__ void locate_balanced(Cursor& c) const {
        const int n = P->seq_count;
        const int64_t hk = P->num_kv_heads;
        const int i = upper_index(n, c.pos, [&](int k) { return hk * prefix[k]; });
        const SeqGeom g = seq_geometry(*P, lens[i], skips[i]);
        const int64_t off = c.pos - hk * prefix[i];
        c.h = static_cast<int32_t>(off / g.work);
        const int64_t jrel = off - static_cast<int64_t>(c.h) * g.work;
        const int64_t ustart = c.pos - jrel;
        const int64_t uend = ustart + g.work;
        c.jbeg = g.first + static_cast<int32_t>(jrel);
        c.jend = g.first + static_cast<int32_t>(min(uend, c.end) - ustart);
        c.s = P->seq_begin + i;
        c.len = g.len;
        c.p = static_cast<int32_t>(c.pos / c.chunk - ustart / c.chunk);
        c.parts = static_cast<int32_t>((uend - 1) / c.chunk - ustart / c.chunk + 1);
    }

    __device__ __forceinline__ void start(Cursor& c, int32_t warp_global) const {
        if (P->balanced) {
            c.chunk = chunk;
            c.pos = static_cast<int64_t>(warp_global) * chunk;
            c.end = min(c.pos + chunk, static_cast<int64_t>(total) * P->num_kv_heads);
            c.valid = c.pos < c.end;
            if (c.valid) locate_balanced(c);
        } else {
            c.item = warp_global;
            c.valid = c.item < total;
            if (c.valid) locate_fixed(c);
        }
    }

    // Move to the warp's next piece.
    __device__ __forceinline__ void next(Cursor& c) const {
        if (P->balanced) {
            c.pos += c.jend - c.jbeg;  // the piece's length
            c.valid = c.pos < c.end;
            if (c.valid) locate_balanced(c);
        } else {
            c.item += nw;
            c.valid = c.item < total;
            if (c.valid) locate_fixed(c);
        }
    }
};

// Sets up the schedule of a launch (all threads of the CTA call it).
// `smem_seqs` holds 3 * seq_count + 1 ints: the prefix, the lengths, the skips.
__device__ __forceinline__ Schedule make_schedule(const DecodeParams& P, int32_t* smem_seqs,
                                                  int warps_per_cta) {
    Schedule sc;
    sc.P = &P;
    int32_t* prefix = smem_seqs;
    int32_t* lens = prefix + P.seq_count + 1;
    int32_t* skips = lens + P.seq_count;
    sc.prefix = prefix;
    sc.lens = lens;
    sc.skips = skips;
    sc.total = build_prefix(P, prefix, lens, skips);
    sc.nw = gridDim.x * warps_per_cta;
    if (P.balanced) {
        const int64_t blocks = static_cast<int64_t>(sc.total) * P.num_kv_heads;
        const int64_t even = (blocks + sc.nw - 1) / sc.nw;
        sc.chunk = even > P.min_chunk ? even : P.min_chunk;
    } else {
        sc.chunk = 0;
    }
    return sc;
}

// Zero-length sequences have no pieces; their rows of `out` are zero.  CTA b
// clears those of the sequences s = b, b + gridDim.x, ... of the launch.  (With
// piece_base > 0 the rows are written by the merge instead.)
template <typename OutT>
__device__ __forceinline__ void zero_empty_sequences(const DecodeParams& P, const int32_t* lens) {
    if (P.piece_base > 0) return;
    const int row = P.num_q_heads * P.head_dim;
    for (int i = blockIdx.x; i < P.seq_count; i += gridDim.x) {
        if (lens[i] != 0) continue;
        const int32_t s = P.seq_begin + i;
        const int32_t r0 = P.q_start ? P.q_start[s] : s;
        const int32_t r1 = P.q_start ? P.q_start[s + 1] : s + 1;
        OutT* o = static_cast<OutT*>(P.out) + static_cast<size_t>(r0) * row;
        for (int64_t e = threadIdx.x; e < static_cast<int64_t>(r1 - r0) * row; e += blockDim.x)
            o[e] = OutT(0.0f);
    }
}

// Query-token rows of sequence s: first row and count (clamped to
// max_q_len and to the sequence length).  One row per sequence without
// q_start.
struct QRows {
    int32_t base;
    int32_t n;
    bool clamped;  // the raw count exceeded max_q_len or the sequence length
};

__device__ __forceinline__ QRows query_rows(const DecodeParams& P, int32_t s, int32_t len) {
    QRows q;
    q.clamped = false;
    if (!P.q_start) {
        q.base = s;
        q.n = 1;
        return q;
    }
    q.base = __ldg(P.q_start + s);
    q.n = __ldg(P.q_start + s + 1) - q.base;
    const int32_t cap = min(P.max_q_len, len);
    if (q.n > cap || q.n < 0) {
        q.clamped = true;
        q.n = q.n < 0 ? 0 : cap;
    }
    return q;
}

// Pieces a prefill row's tile wrote (for the merge): the chunks of key blocks
// up to the tile's last visible key.  Token k of a sequence of length len with
// n new tokens.
__device__ __forceinline__ int32_t prefill_row_pieces(int32_t len, int32_t n, int32_t k, int32_t tile_tokens,
                                                      int32_t chunk_blocks) {
    const int32_t t = k / tile_tokens;
    const int32_t last = min((t + 1) * tile_tokens, n) - 1;
    const int32_t kend = (len - n + last) / kBlockTokens + 1;
    return (kend + chunk_blocks - 1) / chunk_blocks;
}

// Records how many pieces unit (s, h) has (written by the warp holding piece 0;
// read by the reduction).
__device__ __forceinline__ void record_parts(const DecodeParams& P, const Cursor& c, int lane) {
    if (P.ws_parts != nullptr && c.p == 0 && lane == 0)
        P.ws_parts[static_cast<size_t>(c.s) * P.num_kv_heads + c.h] = c.parts;
}

}  // namespace pa
