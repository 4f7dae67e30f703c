// attn_tiles_tc.cuh -- attention of query tiles of up to 256 rows to paged
// keys on the 5th-generation tensor cores (tcgen05: S = Q K^T and O += P V
// accumulate in tensor memory).
//
// Two jobs are real matrix products over paged K/V and share this kernel:
//  * prefix mode.  The sequences of a group start with the same prompt, whose
//    blocks every table of the group names ("Was ändert PagedAttention an der
//    KV-Speicherzuweisung für LLMs?", slavadubrov.com, §"Gemeinsame Nutzung
//    erfordert mehr als Speicherzuweisung": several requests reference one
//    cache block; "PagedAttention et vLLM", aiunderstanding.org, §"Questions
//    fréquemment posées": identical prefixes refer to the same physical
//    pages).  For kv head h, the g query heads of all sequences of the group
//    are the rows of S = Q K^T against the shared prefix keys, so a prefix
//    block is read once per tile of rows instead of once per sequence.  The
//    tile writes each row's partial (m, l, acc); the private suffix goes
//    through the decode kernel and the log-sum-exp merge joins both.
//  * prefill mode.  The n new query tokens of one sequence (a prefill chunk,
//    "vLLM PagedAttention: eine Revolution für den Durchsatz bei der
//    LLM-Inferenz", de.news.hada.io, list of advanced features: chunked
//    prefill; "Внутреннее устройство vLLM", artificials.ru, paragraph on
//    chunked prefill) attend causally to the sequence's own blocks: token k
//    sits at position L - n + k and sees keys 0 .. L - n + k.
//
// Work: a unit is a group (prefix) or a sequence (prefill).  Its tokens (the
// group's sequences, or the new query tokens) are cut into tiles of two
// halves of T = floor(128 / g) tokens; row r of a half is token r / g, query
// head h*g + r % g, one TMEM lane, and the two halves are two accumulator
// sets in tensor memory that share every K/V stage (so a K/V block is fetched
// once per 2T tokens: the SM's TMA engine, which bounds a one-half tile, then
// delivers half the boxes per row).  The unit's key blocks are cut into
// chunks of chunk_blocks blocks (one chunk when the device is full without a
// split).  An item is (chunk c, kv head h, tile t), numbered with t fastest,
// so that the tiles reading the same keys run side by side and share them in
// L2.  The grid is persistent, one CTA per SM: CTA b starts with item b and
// then takes the next unclaimed item from a counter in global memory (one
// atomic add per item, so the CTAs finish together whatever the length mix);
// the producer warp claims items and passes them to the other roles through a
// small queue in shared memory.  Each CTA builds the per-unit item prefix once
// in shared memory and finds any item by binary search.  An item whose chunk
// lies wholly past its tile's last visible key is empty and is skipped.
//
// Roles (320 threads): warps 0-7 softmax, one thread per query row (warp w:
// half w / 4, TMEM lanes 32 (w mod 4) .. +31), warp 8 TMA producer, warp 9
// MMA issue (one thread).  Per item, the producer loads the tile's Q rows with
// one 3-D TMA box per half and 64-column slab (tokens x heads x columns, the
// 128-byte swizzle), then 64-key steps of K and V (4 blocks) into a 4-stage
// ring: K as 64 x 16 boxes per block and slab (the K-major layout of the
// scores' B operand keeps a slab's 64 keys together), V as one 3-D box per
// block (64 columns x 16 rows x 2 slabs, 4 KB), which is exactly one k-step
// of P V's MN-major B operand.  (Measured on B200: 4 KB boxes move a 32 KB
// step 20% faster than 2 KB boxes when every SM loads.)  The MMA thread
// issues S of step j + 1 (both halves) before P V of step j (two S buffers
// per half in TMEM), so the tensor cores run while the softmax works, also
// across item boundaries.  A softmax thread reads its row of S straight from
// TMEM, takes the running max with the scale folded into one multiply-add per
// key (a step that is wholly visible needs no masking), writes P as bf16
// pairs back over the first half of the S buffer it read (P V takes its A
// operand from tensor memory, as FlashAttention-4 does: no shared-memory
// round trip for P), rescales its O row in TMEM when the max moved (only
// then does it wait for the previous P V), and at the item's end writes the
// row: a partial (m, l, acc) at piece c, or the final bf16 row when the units
// have one chunk (prefill), staged through shared memory so that every store
// writes whole 128-byte lines.
// All step counters run on across items, so every mbarrier's phase follows
// from a per-CTA global step or item count.  Every wait is bounded; a role
// that gives up flags PA_DEVERR_TIMEOUT and stops issuing, the other roles'
// waits then run out too, and TMEM is freed on every path.
#pragma once

#include "items.cuh"
#include "tcgen05.cuh"

namespace pa {

constexpr int kTileModePrefix = 0;
constexpr int kTileModePrefill = 1;
constexpr int kTileStepBlocks = 4;  // 64 keys per step
constexpr int kTileHalves = 2;      // accumulator sets of 128 rows per tile
constexpr float kLazyRescale = 8.f;  // log2 units: the reference max lags the true max by at most this

struct TileParams {
    const int32_t* block_tables;  // [num_seqs][max_blocks_per_seq]
    const int32_t* seq_lens;      // [num_seqs]
    const int32_t* q_start;       // prefill: [num_seqs + 1] query-token rows of each sequence
    const int32_t* group_start;   // prefix: [groups + 1] sequences of each group (contiguous;
                                  //   null: one group of every sequence)
    const int32_t* group_blocks;  // prefix: [groups] shared blocks of each group (null: shared_blocks)
    void* out;                    // direct: final rows, bf16 [rows][Hq][D]
    float* ws_m;                  // partials (layout of the decode workspace)
    float* ws_l;
    float* ws_acc;
    int32_t* item_counter;        // items handed out after each CTA's first (zero at launch);
                                  //   null: CTA b takes items b, b + grid, b + 2 grid, ...
    int32_t mode;            // kTileModePrefix or kTileModePrefill
    int32_t unit_begin;      // first unit of this launch
    int32_t num_units;       // units of this launch
    int32_t num_seqs;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t group;           // query heads per kv head
    int32_t half_tokens;     // tokens (prefill) or sequences (prefix) per 128-row half: floor(128 / group)
    int32_t max_blocks_per_seq;
    int32_t num_blocks;
    int32_t chunk_blocks;    // key blocks per item (a multiple of 4)
    int32_t max_parts;       // workspace pieces per row
    int32_t len_cap;         // sequences longer than this are clamped
    int32_t max_q_len;       // prefill: query tokens per sequence handled
    int32_t shared_blocks;   // prefix: blocks of every group when group_blocks is null, else
                             //   the bound on group_blocks
    int32_t direct;          // 1: one chunk per unit, rows written to out as final bf16
    // 1: the grid launched just before this one in the stream (the decode of
    // the private blocks) computes something this launch does not read, and
    // lets it start only after the kernels before it have completed.  Then
    // no role waits for it at the start; one thread waits at the very end, so
    // that this grid completes after it (the merge that follows waits for
    // this grid, and so for both).
    int32_t independent;
    float scale_log2;        // softmax scale * log2(e)
};

template <int D>
struct TileCfg {
    static constexpr int kHalfRows = 128;      // TMEM lanes: rows of one half
    static constexpr int kKeys = 64;           // keys per step
    static constexpr int kStepBlocks = kKeys / kBlockTokens;
    static_assert(kStepBlocks == kTileStepBlocks, "steps of 64 keys");
    static constexpr int kSlabs = D / 64;      // 64-column slabs (128-byte rows)
    static constexpr int kQHalfBytes = kSlabs * kHalfRows * 128;
    static constexpr int kQBytes = kTileHalves * kQHalfBytes;
    static constexpr int kKVSlab = kKeys * 128;               // one slab of K (or V) for a step
    static constexpr int kStageBytes = 2 * kSlabs * kKVSlab;  // K slabs, then V blocks
    // V of a step: block after block (one TMA box each), a block's slabs after
    // each other (16 rows of 128 bytes per slab)
    static constexpr int kVBlockBytes = kSlabs * kBlockTokens * 128;
    static constexpr int kStages = 4;
    static constexpr int kPHalfBytes = kHalfRows * 128;       // epilogue staging: 128 bytes per row
    static constexpr int kPBytes = kTileHalves * kPHalfBytes;
    static constexpr int kSoftmaxWarps = 4 * kTileHalves;
    static constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
    static constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
    static constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
    static constexpr uint32_t kHalfCols = 256;  // per half: S0 | S1 | O
    static constexpr uint32_t kTmemCols = kTileHalves * kHalfCols;
    static constexpr uint32_t kColS = 0, kColO = 2 * kKeys;
    // full, empty per stage; s_full x2, p_full, o_done, o_free, q_full, q_empty, drain;
    // item queue full / empty x kItemSlots
    static constexpr int kItemSlots = 4;
    static constexpr int kBars = 2 * kStages + 8 + 2 * kItemSlots;
    static constexpr int kMaxUnits = 256;  // units whose item prefix one CTA holds (more: several launches)
    static_assert(kMaxUnits <= 256 && kMaxUnits <= kThreads, "unit positions in a byte, one thread per unit");
    // item prefix (int32 [kMaxUnits + 1]) and the units' order (uint8 [kMaxUnits])
    static constexpr int kPrefixBytes = (4 * (kMaxUnits + 1) + kMaxUnits + 15) / 16 * 16;
    static constexpr size_t kSmem = 1024 + kQBytes + kStages * kStageBytes + kPBytes + kPrefixBytes +
                                    8 * kBars + 16 + 4 * kStages + 4 * kItemSlots;
    static_assert(kColO + D <= kHalfCols, "TMEM columns");
    static_assert(kTmemCols <= 512, "TMEM columns");
    static_assert(kSmem <= 227u * 1024u, "shared memory per CTA");
};

// What one unit holds.
struct TileUnit {
    int32_t n;        // tokens: new query tokens (prefill) or sequences (prefix)
    int32_t q_base;   // q row of token 0
    int32_t table;    // block-table row the keys are read through
    int32_t len;      // key positions 0 .. len-1 exist (prefill: the sequence length)
    int32_t kblocks;  // key blocks of the unit
    int32_t tiles;
    int32_t chunks;   // 0 when the unit has no work
    bool clamped;     // prefill: more query tokens than max_q_len or the length allow
};

__device__ __forceinline__ TileUnit tile_unit(const TileParams& P, int32_t u) {
    TileUnit U;
    U.clamped = false;
    if (P.mode == kTileModePrefix) {
        // (out-of-range group bounds are clamped here and flagged by check_group_tables)
        const int32_t s0 = P.group_start ? min(max(__ldg(P.group_start + u), 0), P.num_seqs) : 0;
        const int32_t s1 = P.group_start ? min(max(__ldg(P.group_start + u + 1), s0), P.num_seqs) : P.num_seqs;
        U.n = s1 - s0;
        U.q_base = s0;
        U.table = s0;
        const int32_t kb = P.group_blocks ? __ldg(P.group_blocks + u) : P.shared_blocks;
        U.kblocks = max(0, min(kb, min(P.shared_blocks, P.max_blocks_per_seq)));
        U.len = U.kblocks * kBlockTokens;
    } else {
        int32_t L = __ldg(P.seq_lens + u);
        L = max(0, min(L, P.len_cap));
        const int32_t q0 = __ldg(P.q_start + u);
        int32_t n = __ldg(P.q_start + u + 1) - q0;
        const int32_t cap = min(P.max_q_len, L);
        if (n > cap || n < 0) {
            U.clamped = true;
            n = n < 0 ? 0 : cap;
        }
        U.n = n;
        U.q_base = q0;
        U.table = u;
        U.len = L;
        U.kblocks = (L + kBlockTokens - 1) / kBlockTokens;
    }
    const int32_t tile_tokens = kTileHalves * P.half_tokens;
    U.tiles = (U.n + tile_tokens - 1) / tile_tokens;
    U.chunks = (U.n == 0 || U.kblocks == 0) ? 0 : (U.kblocks + P.chunk_blocks - 1) / P.chunk_blocks;
    return U;
}

struct TileItem {
    TileUnit U;
    int32_t u, t, c, h;
    int32_t tok0, ntok;  // tokens of the tile (both halves)
    int32_t kb0, kb1;    // key blocks [kb0, kb1) of the item
    int32_t nsteps;      // 0: empty item
};

// Item `it` of the launch: prefix[] holds the exclusive item sums of the
// units in the order ord[] (heaviest unit first).
__device__ __forceinline__ TileItem tile_item(const TileParams& P, const int32_t* prefix, const uint8_t* ord,
                                              int32_t it) {
    TileItem I;
    const int i = upper_index(P.num_units, it, [&](int k) { return static_cast<int64_t>(prefix[k]); });
    I.u = P.unit_begin + ord[i];
    I.U = tile_unit(P, I.u);
    const int32_t j = it - prefix[i];
    const int32_t th = I.U.tiles * P.num_kv_heads;
    I.c = j / th;
    const int32_t r = j - I.c * th;
    I.h = r / I.U.tiles;
    I.t = r - I.h * I.U.tiles;
    const int32_t tile_tokens = kTileHalves * P.half_tokens;
    I.tok0 = I.t * tile_tokens;
    I.ntok = min(tile_tokens, I.U.n - I.tok0);
    int32_t kend = I.U.kblocks;
    if (P.mode == kTileModePrefill) {  // blocks up to the tile's last visible key
        const int32_t last = I.U.len - I.U.n + I.tok0 + I.ntok - 1;
        kend = min(kend, last / kBlockTokens + 1);
    }
    I.kb0 = I.c * P.chunk_blocks;
    I.kb1 = min(I.kb0 + P.chunk_blocks, kend);
    I.nsteps = I.kb1 > I.kb0 ? (I.kb1 - I.kb0 + kTileStepBlocks - 1) / kTileStepBlocks : 0;
    return I;
}

// The launch's units in order of decreasing work (items x key blocks, ties by
// index) into ord[0..num_units), and the exclusive sums of their item counts
// in that order into prefix[0..num_units]: items of the heaviest units are
// claimed first, so the last items to be claimed are short and the CTAs finish
// together.  `scratch` holds 2 * num_units words (free during the prologue).
// All threads of the CTA call it (num_units <= kMaxUnits <= blockDim.x).
// Returns the total.  Reports clamped query counts (CTA 0 only, so each is
// counted once).
__device__ __forceinline__ int32_t build_unit_prefix(const TileParams& P, int32_t* prefix, uint8_t* ord,
                                                     uint32_t* scratch) {
    __shared__ int32_t warp_tot[32];
    const int n = P.num_units;
    const int tid = threadIdx.x, nthr = blockDim.x;
    uint32_t* cost = scratch;
    int32_t* items = reinterpret_cast<int32_t*>(scratch + n);
    uint32_t my_cost = 0;
    if (tid < n) {
        const TileUnit U = tile_unit(P, P.unit_begin + tid);
        if (U.clamped && blockIdx.x == 0) flag_error(PA_DEVERR_SEQ_LEN);
        const int32_t it = U.tiles * U.chunks * P.num_kv_heads;
        my_cost = static_cast<uint32_t>(min(static_cast<int64_t>(it) * max(U.kblocks, 1), int64_t{0xffffffff}));
        cost[tid] = my_cost;
        items[tid] = it;
    }
    __syncthreads();
    if (tid < n) {
        int rank = 0;
        for (int u = 0; u < n; ++u) {
            const uint32_t c = cost[u];
            rank += (c > my_cost) || (c == my_cost && u < tid);
        }
        ord[rank] = static_cast<uint8_t>(tid);
    }
    __syncthreads();
    const int32_t local = tid < n ? items[ord[tid]] : 0;
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
        warp_tot[lane] = ti - t;
    }
    __syncthreads();
    const int32_t excl = warp_tot[warp] + incl - local;
    if (tid < n) prefix[tid] = excl;
    if (tid == n - 1) prefix[n] = excl + local;
    if (n == 0 && tid == 0) prefix[0] = 0;
    __syncthreads();
    return prefix[n];
}

// Prefix mode precondition, checked by the producer and MMA warps of the grid
// after their main work: the groups are ordered ranges of the batch with
// shared block counts within the bound, every table of a group starts with the
// group's shared blocks (those of its first sequence), and no sequence of the
// group is shorter than them.  Violations set PA_DEVERR_PREFIX.  `me` of
// `nthreads`.
__device__ __forceinline__ void check_group_tables(const TileParams& P, int64_t me, int64_t nthreads) {
    for (int32_t g = P.unit_begin; g < P.unit_begin + P.num_units; ++g) {
        if (me == 0 && P.group_start) {  // the group list itself: ordered, inside the batch, within the bound
            const int32_t s0 = P.group_start[g], s1 = P.group_start[g + 1], kb = P.group_blocks[g];
            if (s0 < 0 || s1 < s0 || s1 > P.num_seqs || kb < 0 || kb > P.shared_blocks) flag_error(PA_DEVERR_PREFIX);
        }
        const TileUnit U = tile_unit(P, g);
        const int64_t entries = static_cast<int64_t>(U.n) * U.kblocks;
        const int32_t* lead = P.block_tables + static_cast<size_t>(U.table) * P.max_blocks_per_seq;
        for (int64_t e = me; e < entries; e += nthreads) {
            const int64_t s = U.q_base + e / U.kblocks, j = e % U.kblocks;
            if (P.block_tables[s * P.max_blocks_per_seq + j] != lead[j]) flag_error(PA_DEVERR_PREFIX);
        }
        for (int64_t s = me; s < U.n; s += nthreads)
            if (P.seq_lens[U.q_base + s] < U.len) flag_error(PA_DEVERR_PREFIX);
    }
}

template <int D>
__global__ void __launch_bounds__(TileCfg<D>::kThreads, 1)
attn_tiles_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const __grid_constant__ CUtensorMap tmap_q, const TileParams P) {
    using Cfg = TileCfg<D>;
    constexpr int S = Cfg::kStages;
    constexpr int K = Cfg::kKeys;

    // Launched with programmatic stream serialization: until
    // grid_dependency_wait() the CTA reads only the lengths, q_start, the
    // groups and block tables and q (inputs no kernel of this library
    // writes); the pool is read (producer) and out / the workspace written
    // (softmax) only after the wait.
    allow_dependents();

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    // layout: Q[half][slab] | ring[S] | staging[half] | unit prefix | barriers | TMEM slot | stage masks
    const uint32_t q_u32 = smem_u32(smem);
    const uint32_t ring_u32 = q_u32 + Cfg::kQBytes;
    const uint32_t p_u32 = ring_u32 + S * Cfg::kStageBytes;
    uint8_t* ring_smem = smem + Cfg::kQBytes;
    uint8_t* p_smem = ring_smem + S * Cfg::kStageBytes;
    int32_t* prefix = reinterpret_cast<int32_t*>(p_smem + Cfg::kPBytes);
    const uint32_t bars_u32 = p_u32 + Cfg::kPBytes + Cfg::kPrefixBytes;
    const uint32_t full_u32 = bars_u32;            // [S]
    const uint32_t empty_u32 = bars_u32 + 8 * S;   // [S]
    const uint32_t sfull_u32 = bars_u32 + 16 * S;  // [2]
    const uint32_t pfull_u32 = sfull_u32 + 16;
    const uint32_t odone_u32 = pfull_u32 + 8;
    const uint32_t ofree_u32 = odone_u32 + 8;
    const uint32_t qfull_u32 = ofree_u32 + 8;
    const uint32_t qempty_u32 = qfull_u32 + 8;
    const uint32_t drain_u32 = qempty_u32 + 8;
    const uint32_t iqfull_u32 = drain_u32 + 8;                        // [kItemSlots]
    const uint32_t iqempty_u32 = iqfull_u32 + 8 * Cfg::kItemSlots;  // [kItemSlots]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (iqempty_u32 + 8 * Cfg::kItemSlots - q_u32));
    uint32_t* stage_present = tmem_slot + 4;  // [S]: blocks of the stage that were loaded
    volatile int32_t* item_q = reinterpret_cast<volatile int32_t*>(stage_present + S);  // [kItemSlots]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = P.group;
    const int half_rows = P.half_tokens * g;  // rows a half's Q box fills
    const bool prefill = P.mode == kTileModePrefill;

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(full_u32 + 8 * st, 1);
            mbar_init(empty_u32 + 8 * st, 1);
        }
        mbar_init(sfull_u32, 1);
        mbar_init(sfull_u32 + 8, 1);
        mbar_init(pfull_u32, Cfg::kSoftmaxThreads);
        mbar_init(odone_u32, 1);
        mbar_init(ofree_u32, Cfg::kSoftmaxThreads);
        mbar_init(qfull_u32, 1);
        mbar_init(qempty_u32, 1);
        mbar_init(drain_u32, 1);
        for (int i = 0; i < Cfg::kItemSlots; ++i) {
            mbar_init(iqfull_u32 + 8 * i, 1);
            mbar_init(iqempty_u32 + 8 * i, 1 + Cfg::kSoftmaxThreads);
        }
        fence_barrier_init();
    }
    // the rows past the Q boxes (128 mod g of each half) are never loaded:
    // zero them once, so that their S and P stay finite
    for (int e = threadIdx.x; e < kTileHalves * Cfg::kSlabs * (Cfg::kHalfRows - half_rows) * 8; e += blockDim.x) {
        const int chunk = e & 7, rest = e >> 3;
        const int row = half_rows + rest % (Cfg::kHalfRows - half_rows);
        const int half_slab = rest / (Cfg::kHalfRows - half_rows);
        *reinterpret_cast<uint4*>(smem + half_slab * Cfg::kHalfRows * 128 + row * 128 + chunk * 16) =
            make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    if (warp == Cfg::kMmaWarp) tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    uint8_t* unit_ord = reinterpret_cast<uint8_t*>(prefix + Cfg::kMaxUnits + 1);
    // (the staging buffer is free until the first epilogue: scratch for the ordering)
    const int32_t total = build_unit_prefix(P, prefix, unit_ord, reinterpret_cast<uint32_t*>(p_smem));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t check_me = static_cast<int64_t>(blockIdx.x) * 64 + threadIdx.x - Cfg::kProducerWarp * 32;
    const int64_t check_n = static_cast<int64_t>(gridDim.x) * 64;

    if (warp == Cfg::kProducerWarp) {
        // ---------------- producer: Q of each item, then its steps of K and V
        const uint64_t keep = l2_policy_evict_last();  // K/V and Q are read by several tiles
        bool ok = true;
        uint32_t iq = 0, gs = 0;  // items with work, global steps
        bool waited = P.independent != 0;  // grid_dependency_wait done (or not needed)
        bool first = true;         // the CTA's first item is item blockIdx.x
        int32_t cand = blockIdx.x;
        while (ok) {
            // the next item with work; it goes into the item queue the other roles read
            // (-1: none left)
            int32_t it = -1;
            TileItem I;
            while (true) {
                if (first) {
                    first = false;
                } else if (P.item_counter) {
                    if (!waited) {
                        grid_dependency_wait();  // (the counter was set to zero before this launch)
                        waited = true;
                    }
                    cand = 0;
                    if (lane == 0) cand = static_cast<int32_t>(gridDim.x) + atomicAdd(P.item_counter, 1);
                    cand = __shfl_sync(kFullMask, cand, 0);
                } else {
                    cand += gridDim.x;
                }
                if (cand >= total) break;
                I = tile_item(P, prefix, unit_ord, cand);
                if (I.nsteps > 0) {
                    it = cand;
                    break;
                }
            }
            const uint32_t slot = iq % Cfg::kItemSlots;
            if (iq >= static_cast<uint32_t>(Cfg::kItemSlots) &&
                !mbar_wait_bounded(iqempty_u32 + 8 * slot, ((iq / Cfg::kItemSlots) - 1) & 1u)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                item_q[slot] = it;
                mbar_arrive(iqfull_u32 + 8 * slot);
            }
            __syncwarp();
            if (it < 0) break;
            // Q of both halves, once the previous item's S products are done with the buffer
            // (the first item's Q, an input no kernel of this library writes, before the
            // dependency wait)
            if (iq >= 1 && !mbar_wait_bounded(qempty_u32, (iq - 1) & 1u)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(qfull_u32, kTileHalves * Cfg::kSlabs * half_rows * 128);
#pragma unroll
                for (int hh = 0; hh < kTileHalves; ++hh)
#pragma unroll
                    for (int sl = 0; sl < Cfg::kSlabs; ++sl)
                        tma_load_3d(q_u32 + hh * Cfg::kQHalfBytes + sl * Cfg::kHalfRows * 128, &tmap_q, sl * 64,
                                    I.h * g, I.U.q_base + I.tok0 + hh * P.half_tokens, qfull_u32, keep);
            }
            ++iq;
            if (!waited) {
                grid_dependency_wait();  // the pool: a cache write launched before has finished
                waited = true;
            }
            // table entries of the item's blocks, 32 at a time: lane l holds
            // block win + l (-1 where past the item or outside the pool)
            const int32_t* trow = P.block_tables + static_cast<size_t>(I.U.table) * P.max_blocks_per_seq;
            auto table_entry = [&](int jb) -> int32_t {
                if (jb >= I.kb1) return -1;
                const int32_t pb = __ldg(trow + jb);
                if (static_cast<uint32_t>(pb) >= static_cast<uint32_t>(P.num_blocks)) {
                    flag_error(PA_DEVERR_BLOCK_OOB);
                    return -1;
                }
                return pb;
            };
            int32_t win = table_entry(I.kb0 + lane);
            for (int j = 0; j < I.nsteps; ++j, ++gs) {
                const int st = gs % S;
                if (gs >= static_cast<uint32_t>(S) && !mbar_wait_bounded(empty_u32 + 8 * st, ((gs / S) - 1) & 1u)) {
                    ok = false;
                    break;
                }
                const int first = j * Cfg::kStepBlocks;  // block of the item at this step's start
                if (first > 0 && (first & 31) == 0) win = table_entry(I.kb0 + first + lane);
                const int32_t pb = __shfl_sync(kFullMask, win, (first & 31) + (lane & (Cfg::kStepBlocks - 1)));
                const uint32_t present =
                    __ballot_sync(kFullMask, lane < Cfg::kStepBlocks && pb >= 0) & ((1u << Cfg::kStepBlocks) - 1u);
                const uint32_t sbase = ring_u32 + st * Cfg::kStageBytes;
                if (present != (1u << Cfg::kStepBlocks) - 1u) {
                    // blocks past the item or outside the pool: zero their V rows
                    // so that P = 0 times them stays 0
                    for (int c = lane; c < Cfg::kStepBlocks * Cfg::kSlabs * kBlockTokens * 8; c += 32) {
                        const int bb = c / (Cfg::kSlabs * kBlockTokens * 8);
                        if ((present >> bb) & 1u) continue;
                        const int rem = c % (Cfg::kSlabs * kBlockTokens * 8);  // the block's 16-byte chunks
                        *reinterpret_cast<uint4*>(ring_smem + st * Cfg::kStageBytes + Cfg::kSlabs * Cfg::kKVSlab +
                                                  bb * Cfg::kVBlockBytes + rem * 16) = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    stage_present[st] = present;  // read by the softmax after this barrier's phase
                    mbar_arrive_expect_tx(full_u32 + 8 * st, __popc(present) * 2 * Cfg::kSlabs * 2048);
                }
#pragma unroll
                for (int bb = 0; bb < Cfg::kStepBlocks; ++bb) {
                    const int32_t pbb = __shfl_sync(kFullMask, pb, bb);
                    if (lane == 0 && pbb >= 0) {
                        const int32_t row = (pbb * P.num_kv_heads + I.h) * kBlockTokens;
#pragma unroll
                        for (int sl = 0; sl < Cfg::kSlabs; ++sl)
                            tma_load_2d(sbase + sl * Cfg::kKVSlab + bb * kBlockTokens * 128, &tmap_k, sl * 64, row,
                                        full_u32 + 8 * st, keep);
                        // V: the block's slabs in one box (the map is 3-D: 64 columns x rows x slabs)
                        const uint32_t vdst = sbase + Cfg::kSlabs * Cfg::kKVSlab + bb * Cfg::kVBlockBytes;
                        if constexpr (Cfg::kSlabs > 1)
                            tma_load_3d(vdst, &tmap_v, 0, row, 0, full_u32 + 8 * st, keep);
                        else
                            tma_load_2d(vdst, &tmap_v, 0, row, full_u32 + 8 * st, keep);
                    }
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) flag_error(PA_DEVERR_TIMEOUT);
        // this warp's last copies into every stage and into Q have landed before leaving
        for (uint32_t k = 0; k < static_cast<uint32_t>(S) && k < gs; ++k) {
            const uint32_t last = gs - 1 - k;  // one of the last S steps
            mbar_wait_bounded(full_u32 + 8 * (last % S), (last / S) & 1u);
        }
        if (iq > 0) mbar_wait_bounded(qfull_u32, (iq - 1) & 1u);
    } else if (warp == Cfg::kMmaWarp) {
        // ---------------- MMA issue (one thread): S of step j + 1, then P V of step j
        if (lane == 0) {
            constexpr uint32_t kIdescS = umma_idesc_bf16(Cfg::kHalfRows, K, 0);
            constexpr uint32_t kIdescO = umma_idesc_bf16(Cfg::kHalfRows, D, 1);
            // the step sequence of this CTA: (item, step j within it)
            struct Cur {
                int32_t it;      // item index
                int32_t j;       // step within the item
                int32_t nsteps;  // steps of the item
                uint32_t iq;     // items with work before this one
                uint32_t gs;     // global step
            };
            bool ok = true;
            // the iq-th item of the queue (false: none left, or the wait gave up)
            auto first_step = [&](uint32_t iq, uint32_t gs, Cur& c) -> bool {
                const uint32_t slot = iq % Cfg::kItemSlots;
                if (!mbar_wait_bounded_thread(iqfull_u32 + 8 * slot, (iq / Cfg::kItemSlots) & 1u)) {
                    ok = false;
                    return false;
                }
                const int32_t it = item_q[slot];
                mbar_arrive(iqempty_u32 + 8 * slot);
                if (it < 0) return false;
                const TileItem I = tile_item(P, prefix, unit_ord, it);
                c = Cur{it, 0, I.nsteps, iq, gs};
                return true;
            };
            auto next_step = [&](const Cur& c, Cur& n) -> bool {
                if (c.j + 1 < c.nsteps) {
                    n = c;
                    ++n.j;
                    ++n.gs;
                    return true;
                }
                return first_step(c.iq + 1, c.gs + 1, n);
            };
            // S of step c waits for its Q (first step of an item) and its K
            auto wait_s = [&](const Cur& c) -> bool {
                if (c.j == 0 && !mbar_wait_bounded_thread(qfull_u32, c.iq & 1u)) return false;
                return mbar_wait_bounded_thread(full_u32 + 8 * (c.gs % S), (c.gs / S) & 1u);
            };
            // P V of step c waits for its P; the first step of an item
            // overwrites O, which the softmax must have read out for the
            // previous item
            auto wait_pv = [&](const Cur& c) -> bool {
                if (c.j == 0 && c.iq > 0 && !mbar_wait_bounded_thread(ofree_u32, (c.iq - 1) & 1u)) return false;
                return mbar_wait_bounded_thread(pfull_u32, c.gs & 1u);
            };
            auto issue_s = [&](const Cur& c) {
                const int st = c.gs % S;
                tc_fence_after();
                const uint32_t kb = ring_u32 + st * Cfg::kStageBytes;
#pragma unroll
                for (int hh = 0; hh < kTileHalves; ++hh) {
                    const uint32_t qb = q_u32 + hh * Cfg::kQHalfBytes;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = (ks % 4) * 32u;  // k-step within the 128-byte row
                        const uint64_t a = umma_desc_sw128(qb + (ks / 4) * Cfg::kHalfRows * 128 + off, 16, 1024);
                        const uint64_t bd = umma_desc_sw128(kb + (ks / 4) * Cfg::kKVSlab + off, 16, 1024);
                        umma_bf16(tmem + hh * Cfg::kHalfCols + Cfg::kColS + (c.gs & 1u) * K, a, bd, kIdescS, ks > 0);
                    }
                }
                umma_commit(sfull_u32 + 8 * (c.gs & 1u));
                if (c.j + 1 == c.nsteps) umma_commit(qempty_u32);  // the item's last read of Q
            };
            auto issue_pv = [&](const Cur& c) {
                tc_fence_after();
                const uint32_t vb = ring_u32 + (c.gs % S) * Cfg::kStageBytes + Cfg::kSlabs * Cfg::kKVSlab;
#pragma unroll
                for (int hh = 0; hh < kTileHalves; ++hh) {
#pragma unroll
                    for (int ks = 0; ks < K / 16; ++ks) {  // k-step ks: the keys of block ks
                        // P: 16 keys = 8 columns of bf16 pairs in the step's S buffer
                        const uint32_t a = tmem + hh * Cfg::kHalfCols + Cfg::kColS + (c.gs & 1u) * K + ks * 8u;
                        const uint64_t bd = umma_desc_sw128(vb + ks * Cfg::kVBlockBytes, 2048, 1024);
                        umma_bf16_tmem_a(tmem + hh * Cfg::kHalfCols + Cfg::kColO, a, bd, kIdescO, c.j > 0 || ks > 0);
                    }
                }
                umma_commit(odone_u32);
                umma_commit(empty_u32 + 8 * (c.gs % S));  // the stage may be refilled
            };
            // S(j + 1) goes before P V(j), so that the tensor cores compute the
            // next scores while the softmax works on this step.  (Measured:
            // letting P V(j) go first whenever K(j + 1) lands after P(j)
            // delays the next softmax by a P V and was 27% slower.)
            Cur cur;
            bool have = first_step(0, 0, cur);
            if (have && (ok = wait_s(cur))) issue_s(cur);
            while (have && ok) {
                Cur nxt;
                const bool more = next_step(cur, nxt);
                if (!ok) break;  // the item queue's wait gave up
                if (more) {
                    if (!(ok = wait_s(nxt))) break;
                    issue_s(nxt);
                }
                if (!(ok = wait_pv(cur))) break;
                issue_pv(cur);
                if (!more) break;
                cur = nxt;
            }
            if (!ok) flag_error(PA_DEVERR_TIMEOUT);
            // every MMA this thread issued has completed before TMEM goes away
            umma_commit(drain_u32);
            mbar_wait_bounded_thread(drain_u32, 0);
        }
        __syncwarp();
    } else {
        // ---------------- softmax: one thread per query row
        const int hh = warp >> 2;                // half of the tile
        const int row = 32 * (warp & 3) + lane;  // TMEM lane = row of the half
        const uint32_t lane_base = tmem + hh * Cfg::kHalfCols + ((static_cast<uint32_t>(warp & 3) * 32u) << 16);
        const float sl2 = P.scale_log2;
        bool ok = true;  // warp-uniform: a wait that gave up stops TMEM work and arrivals
        uint32_t gs = 0;
        bool waited = P.independent != 0;  // grid_dependency_wait done (before the first output write)
        for (uint32_t iq = 0; ok; ++iq) {
            const uint32_t slot = iq % Cfg::kItemSlots;
            ok = mbar_wait_bounded(iqfull_u32 + 8 * slot, (iq / Cfg::kItemSlots) & 1u);
            if (!ok) break;
            const int32_t it = item_q[slot];
            mbar_arrive(iqempty_u32 + 8 * slot);
            if (it < 0) break;
            const TileItem I = tile_item(P, prefix, unit_ord, it);
            const int tok = hh * P.half_tokens + row / g;  // token of the tile (a sequence in prefix mode)
            const bool row_ok = row < half_rows && tok < I.ntok;
            const int32_t ktok = I.tok0 + tok;  // token within the unit
            // last key this row sees (prefill: causal; prefix: every prefix key)
            const int32_t lim = !row_ok ? -1 : prefill ? I.U.len - I.U.n + ktok : I.U.len - 1;
            const size_t orow = row_ok ? static_cast<size_t>(I.U.q_base + ktok) * P.num_q_heads + I.h * g + row % g : 0;
            float m = -INFINITY, l = 0.f;  // reference max (log2 units) and sum of the row
            for (int j = 0; j < I.nsteps; ++j, ++gs) {
                const int st = gs % S;
                ok = ok && mbar_wait_bounded(sfull_u32 + 8 * (gs & 1u), (gs >> 1) & 1u);
                ok = ok && mbar_wait_bounded(full_u32 + 8 * st, (gs / S) & 1u);
                tc_fence_after();
                const int32_t key0 = (I.kb0 + j * Cfg::kStepBlocks) * kBlockTokens;  // first key of the step
                float x[K];
                float mu = 0.f, alpha = 1.f;
                if (ok) {
                    tmem_ld64(lane_base + Cfg::kColS + (gs & 1u) * K, x);
                    const uint32_t present = stage_present[st];
                    float mx;
                    // a wholly visible step (every block loaded, every key within
                    // the row's limit) with a positive scale takes the plain max of
                    // the raw scores; otherwise mask and scale first
                    const bool plain = present == 0xFu && key0 + K - 1 <= lim && sl2 > 0.f;
                    if (plain) {
                        float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
                        for (int i = 4; i < K; ++i) m4[i & 3] = fmaxf(m4[i & 3], x[i]);
                        mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
                    } else {
                        const int32_t vis = lim - key0;  // last visible key of the step
                        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                        for (int i = 0; i < K; ++i) {
                            x[i] = (((present >> (i / kBlockTokens)) & 1u) && i <= vis) ? x[i] * sl2 : -INFINITY;
                            m4[i & 3] = fmaxf(m4[i & 3], x[i]);
                        }
                        mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                    }
                    // the reference max m (the exponents' offset) moves only when
                    // the step's max exceeds it by more than kLazyRescale: weights
                    // up to 2^kLazyRescale are exact enough in bf16 and fp32, and
                    // O and l then need no rescale (alpha = 1)
                    const float mn = mx > m + kLazyRescale ? mx : m;
                    mu = mn == -INFINITY ? 0.0f : mn;
                    alpha = fast_exp2(m - mu);
                    m = mn;
                    // P = 2^(s - mu) as bf16, the row sum in fp32
                    uint32_t pw[K / 2];
                    float s4[4] = {0.f, 0.f, 0.f, 0.f};
                    if (plain) {
#pragma unroll
                        for (int i = 0; i < K / 2; ++i) {
                            const float p0 = fast_exp2(fmaf(x[2 * i], sl2, -mu));
                            const float p1 = fast_exp2(fmaf(x[2 * i + 1], sl2, -mu));
                            s4[i & 3] += p0 + p1;
                            pw[i] = pack2<false>(p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < K / 2; ++i) {
                            const float p0 = fast_exp2(x[2 * i] - mu);
                            const float p1 = fast_exp2(x[2 * i + 1] - mu);
                            s4[i & 3] += p0 + p1;
                            pw[i] = pack2<false>(p0, p1);
                        }
                    }
                    l = l * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
                    // P V of the previous step must be done before this step's P is
                    // announced (the phase tracking of o_done stays within one
                    // step), and before O is rescaled; the P store itself need not
                    // wait for it (P goes to the other S buffer)
                    bool prev_done = j == 0;
                    if (j > 0 && __any_sync(kFullMask, alpha != 1.f)) {
                        ok = mbar_wait_bounded(odone_u32, (gs - 1) & 1u);
                        tc_fence_after();
                        prev_done = true;
                        if (ok) {
#pragma unroll
                            for (int c = 0; c < D / 32; ++c) {
                                float v[32];
                                tmem_ld32(lane_base + Cfg::kColO + 32 * c, v);
#pragma unroll
                                for (int i = 0; i < 32; ++i) v[i] *= alpha;
                                tmem_st32(lane_base + Cfg::kColO + 32 * c, v);
                            }
                        }
                    }
                    // the row's 64 weights (bf16 pairs) over the first 32 columns of
                    // the S buffer just read: P V takes its A operand from there.  S
                    // of step j + 2 overwrites them only after P V of this step.
                    if (ok) tmem_st32(lane_base + Cfg::kColS + (gs & 1u) * K, pw);
                    if (ok && !prev_done) ok = mbar_wait_bounded(odone_u32, (gs - 1) & 1u);
                }
                if (ok) {
                    // key slots at or past the sequence's length hold stale data
                    // (weight 0, but 0 * NaN is NaN): zero their V rows in the stage
                    const int32_t zero_from = I.U.len - key0;
                    if (zero_from < K) {
                        const int zrows = K - max(0, zero_from);
                        for (int e = threadIdx.x; e < zrows * Cfg::kSlabs * 8; e += Cfg::kSoftmaxThreads) {
                            const int zr = K - zrows + e / (Cfg::kSlabs * 8);
                            const int sl = (e / 8) % Cfg::kSlabs;
                            *reinterpret_cast<uint4*>(ring_smem + st * Cfg::kStageBytes + Cfg::kSlabs * Cfg::kKVSlab +
                                                      (zr / kBlockTokens) * Cfg::kVBlockBytes + sl * kBlockTokens * 128 +
                                                      (zr % kBlockTokens) * 128 + (e % 8) * 16) = make_uint4(0, 0, 0, 0);
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(pfull_u32);
                }
            }
            // ---- the item's rows, through the staging buffer: each warp's 32
            // rows, 128 bytes of each at a time
            if (!waited) {
                grid_dependency_wait();  // before the first write of out or the workspace
                waited = true;
            }
            ok = ok && mbar_wait_bounded(odone_u32, (gs - 1) & 1u);  // the item's last P V
            tc_fence_after();
            if (ok) {
                constexpr float kLn2 = 0.693147180559945309f;
                uint8_t* stage = p_smem + warp * 32 * 128;  // this warp's 4 KB
                const bool direct = P.direct != 0;
                const float inv = direct ? (l > 0.f ? 1.0f / l : 0.f) : 1.f;
                if (!direct && row_ok) {
                    const size_t idx = orow * P.max_parts + I.c;
                    P.ws_m[idx] = m * kLn2;
                    P.ws_l[idx] = l;
                }
                // 128 bytes of a row per round: 32 fp32 (partial) or 64 bf16 (final)
                constexpr int kRounds = D / 32;
                for (int rd = 0; rd < (direct ? kRounds / 2 : kRounds); ++rd) {
                    uint32_t w[32];
                    if (direct) {
                        float v[32], u[32];
                        tmem_ld32(lane_base + Cfg::kColO + 64 * rd, v);
                        tmem_ld32(lane_base + Cfg::kColO + 64 * rd + 32, u);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            w[i] = pack2<false>(v[2 * i] * inv, v[2 * i + 1] * inv);
                            w[16 + i] = pack2<false>(u[2 * i] * inv, u[2 * i + 1] * inv);
                        }
                    } else {
                        float v[32];
                        tmem_ld32(lane_base + Cfg::kColO + 32 * rd, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
                    }
                    // lane's 128 bytes -> its staging row, 16-byte chunk c at c ^ (lane mod 8)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4*>(stage + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                    __syncwarp();
                    // 4 rows per store: lanes 8 r' .. 8 r' + 7 write row 4 k + r' (128 contiguous bytes)
                    for (int k = 0; k < 8; ++k) {
                        const int rr = 4 * k + (lane >> 3), c = lane & 7;
                        const unsigned long long dst_row =
                            __shfl_sync(kFullMask, static_cast<unsigned long long>(orow), rr);
                        const bool rok = __shfl_sync(kFullMask, row_ok ? 1 : 0, rr) != 0;
                        const uint4 val = *reinterpret_cast<const uint4*>(stage + rr * 128 + ((c ^ (rr & 7)) << 4));
                        if (rok) {
                            if (direct)
                                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.out) + dst_row * D + 64 * rd +
                                                          8 * c) = val;
                            else
                                *reinterpret_cast<uint4*>(P.ws_acc + (dst_row * P.max_parts + I.c) * D + 32 * rd +
                                                          4 * c) = val;
                        }
                    }
                    __syncwarp();
                }
                tc_fence_before();
                mbar_arrive(ofree_u32);  // O may be overwritten by the next item
            }
        }
        if (!ok && lane == 0) flag_error(PA_DEVERR_TIMEOUT);
    }

    if (P.mode == kTileModePrefix && warp >= Cfg::kProducerWarp) check_group_tables(P, check_me, check_n);
    tc_fence_before();
    __syncthreads();
    if (warp == Cfg::kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
    if (P.independent && threadIdx.x == 0) grid_dependency_wait();  // complete after the grid before
}

}  // namespace pa
