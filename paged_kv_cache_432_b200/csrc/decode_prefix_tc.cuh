// decode_prefix_tc.cuh -- the shared-prefix attention on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// Same job as decode_prefix_mma_kernel: for kv head h, the N*g query rows of
// all sequences that share a prompt prefix ("Was ändert PagedAttention an der
// KV-Speicherzuweisung für LLMs?", slavadubrov.com, §"Gemeinsame Nutzung
// erfordert mehr als Speicherzuweisung"; "PagedAttention et vLLM",
// aiunderstanding.org, §"Questions fréquemment posées") attend to the prefix
// keys, which are read once per CTA for all of its query rows.  S = Q K^T
// and O += P V are real matrix products here (M = 128 query rows, N = 64 keys
// or D dims), so they run as tcgen05.mma with the accumulators in TMEM:
//
//  * one CTA per SM: T tiles of 128 query rows (PA_PREFIX_TC_TILES, 1 by
//    default; each tile's rows are the TMEM lanes of its own columns) x one
//    key split; 8T + 2 warps.  All tiles of a CTA use every K/V stage.
//    Softmax warps 0 .. 8T-1: two threads per query row.  Warp w serves tile
//    w / 8, reaches TMEM lanes 32 (w mod 4) .. +31 (its rows) and takes half
//    (w / 4) mod 2 of each step's keys and of O's columns.  They load Q into
//    shared memory, run the online softmax of their row half straight from
//    TMEM (tcgen05.ld gives a thread its own row: the max and sum of a half
//    need no shuffles; the two halves swap their maxima through shared memory
//    once per step, one named barrier per tile), write P as bf16 into shared
//    memory, rescale their half of O in TMEM when the row max moved, and
//    finally write the split's partial (m, l, acc).
//    Warp 8T: TMA producer; 4 blocks (64 keys) of K and V per stage, a ring of
//    PA_PREFIX_TC_STAGES stages (4 by default, 128 KB).  It starts as soon as
//    the barriers exist, while the softmax warps load Q.
//    Warp 8T + 1: allocates TMEM and issues the MMAs from one thread.
//  * TMEM, per tile: S in two buffers of 64 columns (the MMA of step j+1 runs
//    while the softmax of step j reads the other), O in D columns; 256
//    columns per tile.
//  * shared memory operands all use the 128-byte swizzle (rows of 128 bytes,
//    16-byte chunk c of row r at c ^ (r mod 8), 1 KB atoms of 8 rows): Q and K
//    K-major for S, P K-major and V MN-major for O.
//  * mbarriers: full/empty per stage (TMA <-> MMA); per tile s_full per S
//    buffer (tcgen05.commit -> softmax), p_full (256 softmax arrivals -> MMA),
//    o_done (tcgen05.commit after each P V -> softmax).  Every wait is
//    bounded; on timeout the CTA flags PA_DEVERR_TIMEOUT, drains what it
//    issued and still frees its TMEM.
//  * What bounds it: with one tile, the delivery of the 2 KB TMA boxes (about
//    1.1 us per 64-key stage); with two, the softmax of 256 rows per step.
//
// The partial of each row goes to the workspace at piece index = split, as
// the mma.sync kernel writes it, and the same log-sum-exp reduction merges it
// with the private suffix.
#pragma once

#include "decode_prefix.cuh"

namespace pa {

template <int D>
struct PrefixTcCfg {
// One tile per CTA measured fastest (two tiles halve the K/V boxes per row
// but double the softmax work per SM, which is what bounds the kernel).
#ifndef PA_PREFIX_TC_TILES
#define PA_PREFIX_TC_TILES 1
#endif
#ifndef PA_PREFIX_TC_STAGES
#define PA_PREFIX_TC_STAGES 4
#endif
    static constexpr int kTiles = PA_PREFIX_TC_TILES;  // 128-row query tiles sharing each K/V stage
    static constexpr int kTileRows = 128;              // rows of a tile = TMEM lanes
    static constexpr int kRows = kTiles * kTileRows;   // query rows per CTA
    static constexpr int kKeys = 64;                   // keys per step
    static constexpr int kStepBlocks = kKeys / kBlockTokens;
    static constexpr int kSlabs = D / 64;              // 64-dim slabs (128-byte rows)
    static constexpr int kQBytes = kSlabs * kTileRows * 128;  // Q of one tile
    static constexpr int kKVSlab = kKeys * 128;        // one slab of K (or V) for a step
    static constexpr int kStageBytes = 2 * kSlabs * kKVSlab;  // K slabs, then V slabs
    static constexpr int kStages = PA_PREFIX_TC_STAGES;
    static constexpr int kPBytes = kTileRows * 128;   // P of one tile (64 keys of bf16 per row)
    static constexpr int kSoftmaxWarps = 8 * kTiles;  // two per TMEM lane quarter and tile
    static constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
    static constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
    // per tile: S0 | S1 | O; 256 columns each
    static constexpr uint32_t kTileCols = 256;
    static constexpr uint32_t kTmemCols = kTiles * kTileCols;
    static constexpr uint32_t kColS = 0, kColO = 2 * kKeys;
    // full, empty per stage; s_full x2, p_full, o_done per tile; drain, q_ready
    static constexpr int kBars = 2 * kStages + 4 * kTiles + 2;
    // exchange between the two halves of a row, per tile: [3][2 halves][128 rows]
    // (maxima of even / odd steps, then the row sums)
    static constexpr int kXBytes = 3 * 2 * kTileRows * 4;
    // at least 120 KB so that one CTA fills an SM (its TMEM request never waits)
    static constexpr size_t kSmemUsed = 1024 + kTiles * kQBytes + kStages * kStageBytes + kTiles * kPBytes +
                                        kTiles * kXBytes + 8 * kBars + 16 + 8 * kStages;
    static constexpr size_t kSmem = kSmemUsed > (120u << 10) ? kSmemUsed : (120u << 10);
    static_assert(kColO + D <= kTileCols, "TMEM columns");
    static_assert(kTmemCols == 256 || kTmemCols == 512, "TMEM allocation");
    static_assert(kKeys == 64, "one 128-byte P row per query row");
    static_assert(kSmem <= 227u * 1024u, "shared memory per CTA");
    static_assert(kTiles * kQBytes + kStages * kStageBytes >= kSoftmaxWarps * 32 * (D / 2) * 4,
                  "epilogue staging fits in Q and the ring");
};

// ------------------------------------------------------------------ tcgen05 helpers
// Shared-memory matrix descriptor: start address, leading / stride byte
// offsets (16-byte units), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;  // descriptor version
    d |= 2ull << 61;  // 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> fp32, A K-major, B
// K-major (b_mn = 0) or MN-major (b_mn = 1), M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, int b_mn) {
    return (1u << 4)                                   // D: fp32
           | (1u << 7)                                 // A: bf16
           | (1u << 10)                                // B: bf16
           | (static_cast<uint32_t>(b_mn) << 16)       // B major
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u));
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot_saddr, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_saddr), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective).
// The wait is in the same statement, so the registers are defined when it ends.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// Named barrier `id` (1.. : barrier 0 is __syncthreads) over `nthreads` softmax threads.
__device__ __forceinline__ void softmax_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ... and the store, which has read its registers when the statement ends.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
        "tcgen05.wait::st.sync.aligned;"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
          "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
          "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
          "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
          "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
          "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

// Precondition of the shared-prefix decode, checked by the producer and MMA
// warps of the grid together (after their main work): every table starts with the prefix blocks of table 0, and no
// sequence is shorter than the prefix.  Violations set PA_DEVERR_PREFIX.
// `me` of `nthreads` checking threads.
__device__ __forceinline__ void check_prefix_tables(const PrefixParams& P, int64_t me, int64_t nthreads) {
    const int64_t entries = static_cast<int64_t>(P.num_seqs) * P.shared_blocks;
    for (int64_t e = me; e < entries; e += nthreads) {
        const int64_t s = e / P.shared_blocks, j = e - s * P.shared_blocks;
        if (P.block_tables[s * P.max_blocks_per_seq + j] != P.block_tables[j]) flag_error(PA_DEVERR_PREFIX);
    }
    for (int64_t s = me; s < P.num_seqs; s += nthreads)
        if (P.seq_lens[s] < P.shared_blocks * kBlockTokens) flag_error(PA_DEVERR_PREFIX);
}

// ------------------------------------------------------------------ kernel
template <int D>
__global__ void __launch_bounds__(PrefixTcCfg<D>::kThreads, 1)
decode_prefix_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const PrefixParams P) {
    using Cfg = PrefixTcCfg<D>;
    constexpr int S = Cfg::kStages;
    constexpr int T = Cfg::kTiles;
    constexpr int kHalfKeys = Cfg::kKeys / 2;      // keys of a step per softmax thread
    constexpr int kHalfD = D / 2;                  // O columns per softmax thread
    constexpr int kTileThreads = 8 * 32;           // softmax threads of one tile
    constexpr int kSoftmaxThreads = Cfg::kSoftmaxWarps * 32;
    static_assert(T == 1 || T == 2, "one or two query tiles");

    // Launched with programmatic stream serialization: the CTA starts while
    // the previous kernel (the cache write) may still run.  Setup, Q and the
    // table windows are inputs no kernel of this library writes; the pool is
    // read (producer) and the workspace written (softmax epilogue) only after
    // grid_dependency_wait().
    allow_dependents();

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    // layout: Q[T] | ring[S] | P[T] | exchange[T] | barriers | TMEM address, stage masks
    const uint32_t q_u32 = smem_u32(smem);
    const uint32_t ring_u32 = q_u32 + T * Cfg::kQBytes;
    const uint32_t p_u32 = ring_u32 + S * Cfg::kStageBytes;
    uint8_t* ring_smem = smem + T * Cfg::kQBytes;
    uint8_t* p_smem = ring_smem + S * Cfg::kStageBytes;
    float* xchg_all = reinterpret_cast<float*>(p_smem + T * Cfg::kPBytes);
    const uint32_t bars_u32 = p_u32 + T * Cfg::kPBytes + T * Cfg::kXBytes;
    const uint32_t full_u32 = bars_u32;                // [S]
    const uint32_t empty_u32 = bars_u32 + 8 * S;       // [S]
    const uint32_t tile_bars_u32 = bars_u32 + 16 * S;  // per tile: s_full[2], p_full, o_done
    const uint32_t drain_u32 = tile_bars_u32 + 32 * T;
    const uint32_t qready_u32 = drain_u32 + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (qready_u32 + 8 - q_u32));
    uint32_t* stage_present = tmem_slot + 2;  // [S]: blocks of the stage that were loaded
    auto sfull_of = [&](int t, int b) { return tile_bars_u32 + 32 * t + 8 * b; };
    auto pfull_of = [&](int t) { return tile_bars_u32 + 32 * t + 16; };
    auto odone_of = [&](int t) { return tile_bars_u32 + 32 * t + 24; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int tile = blockIdx.x % P.row_tiles;  // a group of T tiles of 128 rows
    const int split = blockIdx.x / P.row_tiles;
    const int jbeg = split * P.split_blocks;
    const int jend = min(P.shared_blocks, jbeg + P.split_blocks);
    const int nblk = max(0, jend - jbeg);
    const int nsteps = (nblk + Cfg::kStepBlocks - 1) / Cfg::kStepBlocks;
    const int g = P.group;
    const int rows_total = P.num_seqs * g;
    const int64_t check_me = static_cast<int64_t>(blockIdx.y * gridDim.x + blockIdx.x) * 64 + threadIdx.x -
                             Cfg::kProducerWarp * 32;
    const int64_t check_n = static_cast<int64_t>(gridDim.x) * gridDim.y * 64;

    if (nsteps == 0) {  // (uniform over the CTA: nothing allocated yet)
        if (warp >= Cfg::kProducerWarp) check_prefix_tables(P, check_me, check_n);
        return;
    }

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(full_u32 + 8 * st, 1);
            mbar_init(empty_u32 + 8 * st, 1);
        }
        for (int t = 0; t < T; ++t) {
            mbar_init(sfull_of(t, 0), 1);
            mbar_init(sfull_of(t, 1), 1);
            mbar_init(pfull_of(t), kTileThreads);
            mbar_init(odone_of(t), 1);
        }
        mbar_init(drain_u32, 1);
        mbar_init(qready_u32, kSoftmaxThreads);
        fence_barrier_init();
    }
    if (warp == Cfg::kMmaWarp) tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // softmax threads: tile, row of the tile (= TMEM lane), half of the keys / of O
    const bool is_softmax = warp < Cfg::kSoftmaxWarps;
    const int tl = warp >> 3;
    const int row = 32 * (warp & 3) + lane;
    const int hf = (warp >> 2) & 1;
    const int r = (tile * T + tl) * Cfg::kTileRows + row;
    const bool row_ok = is_softmax && r < rows_total;
    const size_t qrow = row_ok ? static_cast<size_t>(r / g) * P.num_q_heads + h * g + r % g : 0;
    if (is_softmax) {
        // this thread's half of the Q row into shared memory (K-major, 128-byte
        // swizzle), while the producer already streams K and V
        uint8_t* qt = smem + tl * Cfg::kQBytes;
        const uint4* q = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(P.q) + qrow * D);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
            const int cc = hf * (D / 16) + k;  // 16-byte chunk of the row
            const int sl = cc >> 3, c = cc & 7;
            const uint4 v = row_ok ? __ldg(q + cc) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(qt + sl * Cfg::kTileRows * 128 + row * 128 + ((c ^ (row & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();  // generic writes, read by the tensor cores
        mbar_arrive(qready_u32);
    }

    if (warp == Cfg::kProducerWarp) {
        // ---------------- producer: 4 blocks of K and V per stage
        const uint64_t policy = l2_policy_evict_last();  // every tile group of this head reads them
        int issued = 0;
        // table entries of the split, 32 at a time: lane l holds block
        // win + l (-1 where absent or outside the pool); the next window is
        // loaded while this one is used
        auto table_entry = [&](int jb) -> int32_t {
            if (jb >= jend) return -1;
            const int32_t pb = __ldg(P.block_tables + jb);
            if (static_cast<uint32_t>(pb) >= static_cast<uint32_t>(P.num_blocks)) {
                flag_error(PA_DEVERR_BLOCK_OOB);
                return -1;
            }
            return pb;
        };
        int32_t win_cur = table_entry(jbeg + lane);
        int32_t win_next = table_entry(jbeg + 32 + lane);
        grid_dependency_wait();  // the pool: the cache write has finished
        for (int j = 0; j < nsteps; ++j) {
            const int st = j % S;
            const int fill = j / S;
            if (fill > 0 && !mbar_wait_bounded(empty_u32 + 8 * st, (fill - 1) & 1u)) {
                if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
                break;
            }
            const uint32_t sbase = ring_u32 + st * Cfg::kStageBytes;
            const int first = j * Cfg::kStepBlocks;  // block of the split at this step's start
            if (first > 0 && (first & 31) == 0) {    // next window
                win_cur = win_next;
                win_next = table_entry(jbeg + first + 32 + lane);
            }
            // lane b < kStepBlocks: block b of the step
            const int32_t pb = __shfl_sync(kFullMask, win_cur, (first & 31) + (lane & (Cfg::kStepBlocks - 1)));
            const uint32_t present =
                __ballot_sync(kFullMask, lane < Cfg::kStepBlocks && pb >= 0) & ((1u << Cfg::kStepBlocks) - 1u);
            if (present != (1u << Cfg::kStepBlocks) - 1u) {
                // absent blocks: zero their V rows so that P = 0 times them stays 0
                for (int c = lane; c < Cfg::kStepBlocks * Cfg::kSlabs * kBlockTokens * 8; c += 32) {
                    const int b = c / (Cfg::kSlabs * kBlockTokens * 8);
                    if ((present >> b) & 1u) continue;
                    const int rem = c % (Cfg::kSlabs * kBlockTokens * 8);
                    const int sl = rem / (kBlockTokens * 8), rr = rem % (kBlockTokens * 8);
                    const int t = b * kBlockTokens + rr / 8;
                    *reinterpret_cast<uint4*>(ring_smem + st * Cfg::kStageBytes + (Cfg::kSlabs + sl) * Cfg::kKVSlab +
                                              t * 128 + (rr % 8) * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) {
                stage_present[st] = present;  // read by the softmax after this barrier's phase
                mbar_arrive_expect_tx(full_u32 + 8 * st, __popc(present) * 2 * Cfg::kSlabs * 2048);
            }
#pragma unroll
            for (int b = 0; b < Cfg::kStepBlocks; ++b) {
                const int32_t pbb = __shfl_sync(kFullMask, pb, b);
                if (lane == 0 && pbb >= 0) {
                    const int32_t trow = (pbb * P.num_kv_heads + h) * kBlockTokens;
                    const uint32_t bar = full_u32 + 8 * st;
#pragma unroll
                    for (int sl = 0; sl < Cfg::kSlabs; ++sl) {
                        tma_load_2d(sbase + sl * Cfg::kKVSlab + b * kBlockTokens * 128, &tmap_k, sl * 64, trow, bar,
                                    policy);
                        tma_load_2d(sbase + (Cfg::kSlabs + sl) * Cfg::kKVSlab + b * kBlockTokens * 128, &tmap_v,
                                    sl * 64, trow, bar, policy);
                    }
                }
            }
            __syncwarp();
            ++issued;
        }
        // wait for this warp's last copy into every stage before leaving
        for (int st = 0; st < S && st < issued; ++st) {
            const int last_fill = (issued - 1 - st) / S;
            mbar_wait_bounded(full_u32 + 8 * st, last_fill & 1u);
        }
    } else if (warp == Cfg::kMmaWarp) {
        // ---------------- MMA issue (one thread)
        if (lane == 0) {
            constexpr uint32_t kIdescS = umma_idesc_bf16(Cfg::kTileRows, Cfg::kKeys, 0);
            constexpr uint32_t kIdescO = umma_idesc_bf16(Cfg::kTileRows, D, 1);
            auto issue_s = [&](int j) -> bool {
                const int st = j % S;
                if (!mbar_wait_bounded_thread(full_u32 + 8 * st, (j / S) & 1u)) return false;
                tc_fence_after();
                const uint32_t kb = ring_u32 + st * Cfg::kStageBytes;
#pragma unroll
                for (int t = 0; t < T; ++t) {
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = (ks % 4) * 32u;  // k-step within the 128-byte row
                        const uint64_t a = umma_desc_sw128(
                            q_u32 + t * Cfg::kQBytes + (ks / 4) * Cfg::kTileRows * 128 + off, 16, 1024);
                        const uint64_t b = umma_desc_sw128(kb + (ks / 4) * Cfg::kKVSlab + off, 16, 1024);
                        umma_bf16(tmem + t * Cfg::kTileCols + Cfg::kColS + (j & 1) * Cfg::kKeys, a, b, kIdescS,
                                  ks > 0);
                    }
                    umma_commit(sfull_of(t, j & 1));
                }
                return true;
            };
            bool ok = mbar_wait_bounded_thread(qready_u32, 0);
            if (ok) {
                tc_fence_after();
                ok = issue_s(0);
            }
            for (int j = 0; j < nsteps && ok; ++j) {
                if (j + 1 < nsteps && !(ok = issue_s(j + 1))) break;
                const uint32_t vb = ring_u32 + (j % S) * Cfg::kStageBytes + Cfg::kSlabs * Cfg::kKVSlab;
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    if (!(ok = mbar_wait_bounded_thread(pfull_of(t), j & 1u))) break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < Cfg::kKeys / 16; ++ks) {
                        const uint64_t a = umma_desc_sw128(p_u32 + t * Cfg::kPBytes + ks * 32u, 16, 1024);
                        const uint64_t b = umma_desc_sw128(vb + ks * 16 * 128, Cfg::kKVSlab, 1024);
                        umma_bf16(tmem + t * Cfg::kTileCols + Cfg::kColO, a, b, kIdescO, j > 0 || ks > 0);
                    }
                    umma_commit(odone_of(t));
                }
                if (!ok) break;
                umma_commit(empty_u32 + 8 * (j % S));
            }
            if (!ok) flag_error(PA_DEVERR_TIMEOUT);
            // every MMA this thread issued has completed before TMEM goes away
            umma_commit(drain_u32);
            mbar_wait_bounded_thread(drain_u32, 0);
        }
        __syncwarp();
    } else {
        // ---------------- softmax: two threads per query row (keys and O split in halves)
        // Every softmax thread runs all nsteps steps and takes every named
        // barrier of its tile, so that the halves of a row stay paired
        // whatever happens; a wait that gives up marks the warp dead
        // (warp-uniform), and a dead warp skips its tensor-memory work and its
        // arrivals.
        const uint32_t lane_base = tmem + tl * Cfg::kTileCols + ((static_cast<uint32_t>(warp & 3) * 32u) << 16);
        uint8_t* p_tile = p_smem + tl * Cfg::kPBytes;
        float* xchg = xchg_all + tl * (Cfg::kXBytes / 4);
        const int bar_id = 1 + tl;
        const float sl2 = P.scale_log2;
        float m = -INFINITY, l = 0.f;  // l: this half's share of the row sum
        bool ok = true;
        for (int j = 0; j < nsteps; ++j) {
            const int st = j % S;
            // S of this step is in TMEM; the stage's block mask was published
            // with the stage's load barrier (already complete)
            ok = ok && mbar_wait_bounded(sfull_of(tl, j & 1), (j >> 1) & 1u);
            ok = ok && mbar_wait_bounded(full_u32 + 8 * st, (j / S) & 1u);
            tc_fence_after();
            float x[kHalfKeys];
            float mx = -INFINITY;
            if (ok) {
                const uint32_t present = stage_present[st] >> (hf * kHalfKeys / kBlockTokens);
                tmem_ld32(lane_base + Cfg::kColS + (j & 1) * Cfg::kKeys + hf * kHalfKeys, x);
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // four independent chains
#pragma unroll
                for (int i = 0; i < kHalfKeys; ++i) {
                    x[i] = ((present >> (i / kBlockTokens)) & 1u) ? x[i] * sl2 : -INFINITY;
                    m4[i & 3] = fmaxf(m4[i & 3], x[i]);
                }
                mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            } else {
#pragma unroll
                for (int i = 0; i < kHalfKeys; ++i) x[i] = -INFINITY;
            }
            // the row max over both halves
            float* xs = xchg + (j & 1) * 2 * Cfg::kTileRows;
            xs[hf * Cfg::kTileRows + row] = mx;
            softmax_bar_sync(bar_id, kTileThreads);
            mx = fmaxf(mx, xs[(1 - hf) * Cfg::kTileRows + row]);
            const float mn = fmaxf(m, mx);
            const float mu = mn == -INFINITY ? 0.0f : mn;
            const float alpha = fast_exp2(m - mu);
            m = mn;
            // P as bf16 pairs; the denominator sums the rounded weights
            uint32_t pw[kHalfKeys / 2];
            float s4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains
#pragma unroll
            for (int i = 0; i < kHalfKeys / 2; ++i) {
                pw[i] = pack2<false>(fast_exp2(x[2 * i] - mu), fast_exp2(x[2 * i + 1] - mu));
                s4[i & 3] += __uint_as_float(pw[i] << 16) + __uint_as_float(pw[i] & 0xffff0000u);
            }
            l = l * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
            if (j > 0) {
                // P V of the previous step is done: the P buffer is free, O holds the sum up to it
                ok = ok && mbar_wait_bounded(odone_of(tl), (j - 1) & 1u);
                tc_fence_after();
                if (ok && __any_sync(kFullMask, alpha != 1.f)) {
#pragma unroll
                    for (int c = 0; c < kHalfD / 32; ++c) {
                        float v[32];
                        tmem_ld32(lane_base + Cfg::kColO + hf * kHalfD + 32 * c, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= alpha;
                        tmem_st32(lane_base + Cfg::kColO + hf * kHalfD + 32 * c, v);
                    }
                }
            }
            if (ok) {
                // keys 32 hf .. 32 hf + 31 of the row: 16-byte chunks 4 hf .. 4 hf + 3
                // of its 128-byte P row, K-major, 128-byte swizzle
#pragma unroll
                for (int c = 0; c < kHalfKeys / 8; ++c) {
                    const int cc = hf * (kHalfKeys / 8) + c;
                    *reinterpret_cast<uint4*>(p_tile + row * 128 + ((cc ^ (row & 7)) << 4)) =
                        make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(pfull_of(tl));
            }
        }
        grid_dependency_wait();  // before the workspace writes below
        // the row sum over both halves (its own buffer: the partner may still
        // read the last step's maximum)
        xchg[4 * Cfg::kTileRows + hf * Cfg::kTileRows + row] = l;
        softmax_bar_sync(bar_id, kTileThreads);
        l += xchg[4 * Cfg::kTileRows + (1 - hf) * Cfg::kTileRows + row];
        ok = ok && mbar_wait_bounded(odone_of(tl), (nsteps - 1) & 1u);
        // the last tile's last commit covers every MMA the CTA issued: after
        // it, Q and the ring are idle and serve as staging below
        ok = ok && mbar_wait_bounded(odone_of(T - 1), (nsteps - 1) & 1u);
        if (ok) {
            tc_fence_after();
            // the split's partial of this row: m, l by half 0; each half its O columns
            const size_t idx = qrow * P.max_parts + split;
            constexpr float kLn2 = 0.693147180559945309f;
            if (row_ok && hf == 0) {
                P.ws_m[idx] = m * kLn2;
                P.ws_l[idx] = l;
            }
            // the warp's 32 half-rows go through shared memory (Q and the ring
            // are idle now) so that each store instruction
            // writes one contiguous half-row; 16-byte chunk c of lane l's
            // half-row sits at c ^ (l mod 16)
            constexpr int kChunks = kHalfD / 4;  // 16-byte chunks of a half-row
            float* stage = reinterpret_cast<float*>(smem) + warp * 32 * kHalfD;
#pragma unroll
            for (int c = 0; c < kHalfD / 32; ++c) {
                float v[32];
                tmem_ld32(lane_base + Cfg::kColO + hf * kHalfD + 32 * c, v);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int ch = 8 * c + i;
                    *reinterpret_cast<float4*>(stage + lane * kHalfD + 4 * ((ch ^ lane) & (kChunks - 1))) =
                        make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
            }
            __syncwarp();
            for (int rr = 0; rr < 32; ++rr) {
                const size_t ridx = __shfl_sync(kFullMask, static_cast<unsigned long long>(idx), rr);
                const bool rok = __shfl_sync(kFullMask, row_ok ? 1 : 0, rr) != 0;
                const int e = 2 * lane;  // this lane's two floats of the half-row
                if (rok && e < kHalfD) {
                    const int ch = e / 4;
                    const float2 v = *reinterpret_cast<const float2*>(
                        stage + rr * kHalfD + 4 * ((ch ^ rr) & (kChunks - 1)) + (e & 3));
                    *reinterpret_cast<float2*>(P.ws_acc + ridx * D + hf * kHalfD + e) = v;
                }
            }
        } else if (lane == 0) {
            flag_error(PA_DEVERR_TIMEOUT);
        }
    }

    if (!is_softmax) check_prefix_tables(P, check_me, check_n);
    tc_fence_before();
    __syncthreads();
    if (warp == Cfg::kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

}  // namespace pa
