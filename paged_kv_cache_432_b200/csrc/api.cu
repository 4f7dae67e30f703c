// api.cu -- the C ABI of the paged decode library (declared in pagedattn.h).
//
// Host side only: validates arguments without touching device memory, plans
// the split of long sequences into partitions, encodes the TMA tensor maps of
// the KV pools, sizes persistent grids from the SM count and occupancy, and
// enqueues the kernels on the caller's stream.  All kernels live in this one
// translation unit, so the sticky device error word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include "pagedattn.h"

#include "cache_write.cuh"
#include "common.cuh"
#include "attn_tiles_tc.cuh"
#include "decode_mma.cuh"
#include "decode_simt.cuh"
#include "items.cuh"
#include "lse_reduce.cuh"

namespace {

using namespace pa;

constexpr int32_t kNoSplit = 1 << 24;       // partition size meaning "never split"
constexpr int32_t kMaxSeqsPerLaunch = 2048; // sequences whose item prefix one CTA holds
constexpr int kMaxDevices = 64;

// bf16 kernel configuration: warps per CTA and ring stages per warp (build-time
// overridable, for tuning sweeps).
#ifndef PA_MMA_WARPS
#define PA_MMA_WARPS 4
#endif
#ifndef PA_MMA_STAGES
#define PA_MMA_STAGES 2
#endif
#ifndef PA_MMA_MIN_CTAS
#define PA_MMA_MIN_CTAS 2
#endif
// E4M3 stages are half the bytes: twice as many keep the same bytes in flight
#ifndef PA_MMA_STAGES_FP8
#define PA_MMA_STAGES_FP8 4
#endif
#ifndef PA_MMA_MIN_CTAS_FP8
#define PA_MMA_MIN_CTAS_FP8 2
#endif
// E4M3 with <= 8 query rows runs the transposed products, which hold far
// fewer registers: four CTAs per SM, each warp with a 2-stage ring (measured
// faster than 3 or 4 stages at 3-4 CTAs)
#ifndef PA_MMA_STAGES_FP8_T
#define PA_MMA_STAGES_FP8_T 2
#endif
#ifndef PA_MMA_MIN_CTAS_FP8_T
#define PA_MMA_MIN_CTAS_FP8_T 4
#endif
constexpr int kMmaWarps = PA_MMA_WARPS;
constexpr int kMmaStages = PA_MMA_STAGES;
constexpr int kMmaMinCtas = PA_MMA_MIN_CTAS;  // CTAs per SM the register budget must allow
template <bool FP8, int ROWS>
constexpr int mma_stages() {
    return !FP8 ? kMmaStages : ROWS <= 8 ? PA_MMA_STAGES_FP8_T : PA_MMA_STAGES_FP8;
}
template <bool FP8, int ROWS>
constexpr int mma_min_ctas() {
    return !FP8 ? kMmaMinCtas : ROWS <= 8 ? PA_MMA_MIN_CTAS_FP8_T : PA_MMA_MIN_CTAS_FP8;
}

thread_local char g_last_cuda_error[256] = "no CUDA error recorded";

int cuda_fail(cudaError_t e, const char* where) {
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "CUDA error in %s: %s (%s)", where,
                  cudaGetErrorName(e), cudaGetErrorString(e));
    return PA_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct DeviceInfo {
    int sms = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

int device_info(DeviceInfo* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_dev[dev].sms == 0) {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        g_dev[dev].sms = sms;
    }
    *out = g_dev[dev];
    return PA_OK;
}

// Sets the dynamic shared-memory ceiling of `kernel` once per device.
struct AttrKey {
    const void* kernel;
    int dev;
};
AttrKey g_attr_done[256];
int g_attr_count = 0;

template <typename K>
int ensure_smem_attr(K kernel, size_t bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    const void* kp = reinterpret_cast<const void*>(kernel);
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < g_attr_count; ++i)
        if (g_attr_done[i].kernel == kp && g_attr_done[i].dev == dev) return PA_OK;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(bytes));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    if (g_attr_count < 256) g_attr_done[g_attr_count++] = AttrKey{kp, dev};
    return PA_OK;
}

template <typename K>
int persistent_grid(K kernel, int threads, size_t smem, int64_t max_useful_ctas, int* grid) {
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc != PA_OK) return rc;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (per_sm < 1) per_sm = 1;
    int64_t g = static_cast<int64_t>(di.sms) * per_sm;
    if (max_useful_ctas < g) g = max_useful_ctas;
    *grid = static_cast<int>(g < 1 ? 1 : g);
    return PA_OK;
}

// ------------------------------------------------------------ TMA tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

int get_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
    std::call_once(g_encode_once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        g_encode_err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                                        cudaEnableDefault, &q);
        if (g_encode_err == cudaSuccess && q != cudaDriverEntryPointSuccess)
            g_encode_err = cudaErrorSymbolNotFound;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    if (g_encode_err != cudaSuccess) return cuda_fail(g_encode_err, "cudaGetDriverEntryPoint");
    *fn = g_encode;
    return PA_OK;
}

// The pool seen as a 2-D tensor [num_blocks*Hkv*16 rows][head_dim].  bf16:
// loaded in 64-column x 16-row boxes with the 128-byte swizzle.  E4M3 (fp8):
// one box of 16 rows x head_dim bytes, with the 128-byte swizzle (64-byte at
// head_dim 64, where a row is 64 bytes).
int encode_pool_map(CUtensorMap* map, const void* base, int64_t rows, int head_dim,
                    bool fp8 = false) {
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    int rc = get_encoder(&enc);
    if (rc != PA_OK) return rc;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * (fp8 ? 1 : 2)};
    cuuint32_t box[2] = {fp8 ? static_cast<cuuint32_t>(head_dim) : 64u, 16};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     (fp8 && head_dim == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                      "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
        return PA_ERR_CUDA;
    }
    return PA_OK;
}

// The bf16 pool seen as a 3-D tensor [slab][rows][64 columns] (slab stride
// 128 bytes, row stride head_dim * 2), for head_dim 128: one 64 x 16 x 2 box
// lands a block-head's whole tile (4 KB) as its two 128-byte-swizzled
// column slabs one after the other.  head_dim 64 has one slab: the 2-D map.
int encode_pool_map_blocks(CUtensorMap* map, const void* base, int64_t rows, int head_dim) {
    if (head_dim != 128) return encode_pool_map(map, base, rows, head_dim);
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    int rc = get_encoder(&enc);
    if (rc != PA_OK) return rc;
    cuuint64_t dims[3] = {64u, static_cast<cuuint64_t>(rows), 2u};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2, 128u};
    cuuint32_t box[3] = {64u, 16u, 2u};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                      "cuTensorMapEncodeTiled (block tiles) failed (CUresult %d)", static_cast<int>(r));
        return PA_ERR_CUDA;
    }
    return PA_OK;
}

// ------------------------------------------------------------ planning
constexpr int32_t kMinChunk = 16;  // balanced split: fewest blocks in one warp's range

// Fixed partition size for partition_blocks > 0 or -1 (never split); 0 for the
// balanced split (partition_blocks = 0).
int32_t resolve_part_blocks(int32_t partition_blocks) {
    if (partition_blocks > 0) return partition_blocks;
    if (partition_blocks == -1) return kNoSplit;
    return 0;
}

struct Plan {
    bool balanced;
    int32_t part_blocks;  // fixed mode
    int32_t max_parts;    // pieces per unit the workspace holds
    int32_t max_len;      // effective max_seq_len (the workspace is sized for it)
    bool split;
    // shared-prefix decode only
    int32_t shared_blocks;
    int32_t prefix_splits;        // key splits of the prefix = its pieces 0 .. splits-1
    int32_t prefix_split_blocks;  // blocks per key split
    int32_t prefix_row_tiles;     // ceil(num_seqs * group / rows per prefix CTA)
};

Plan make_plan(int32_t max_seq_len, int32_t partition_blocks) {
    Plan p;
    p.max_len = max_seq_len;
    p.shared_blocks = p.prefix_splits = p.prefix_split_blocks = p.prefix_row_tiles = 0;
    const int32_t nb = (max_seq_len + kBlockTokens - 1) / kBlockTokens;
    const int32_t pb = resolve_part_blocks(partition_blocks);
    p.balanced = pb == 0;
    if (p.balanced) {
        // a unit of nb blocks meets at most ceil(nb / C) + 1 warp ranges of C >= kMinChunk
        p.part_blocks = kNoSplit;
        p.max_parts = nb == 0 ? 1 : (nb + kMinChunk - 1) / kMinChunk + 1;
    } else {
        p.part_blocks = pb;
        p.max_parts = nb == 0 ? 1 : 1 + (nb - 1) / pb;
    }
    p.split = p.max_parts > 1;
    return p;
}

// Shared-prefix decode: the tile kernel's key chunks of the prefix are pieces
// 0..splits-1 of every row; the private part of each sequence (blocks from
// shared_blocks on) is cut as pa_decode would cut a sequence of the remaining
// length, and its pieces follow.  The workspace reserves kMaxTileSplits slots;
// the launch picks the chunking that fills the device (choose_tile_split).
constexpr int32_t kMaxTileSplits = 16;
constexpr int32_t kWideReducePieces = 32;  // rows that can have more pieces merge with a CTA each

// Query tokens (or sequences) per 128-row half of a tile of the tile kernel,
// and per tile (two halves).
int32_t half_tokens(int32_t group) { return 128 / group; }
int32_t tile_tokens(int32_t group) { return kTileHalves * half_tokens(group); }

Plan make_prefix_plan(int32_t max_seq_len, int32_t partition_blocks, int32_t shared_blocks,
                      int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads) {
    const int32_t rest = max_seq_len - shared_blocks * kBlockTokens;
    Plan p = make_plan(rest > 0 ? rest : 0, partition_blocks);
    p.max_len = max_seq_len;
    const int32_t tt = tile_tokens(num_q_heads / num_kv_heads);
    p.prefix_row_tiles = (num_seqs + tt - 1) / tt;
    if (p.prefix_row_tiles < 1) p.prefix_row_tiles = 1;
    p.shared_blocks = shared_blocks;
    const int32_t slots = shared_blocks < kMaxTileSplits ? shared_blocks : kMaxTileSplits;
    p.prefix_splits = slots;  // reserved; narrowed at launch
    p.prefix_split_blocks = (shared_blocks + slots - 1) / slots;
    p.max_parts += slots;
    p.split = true;
    return p;
}

// Several prompt groups: every sequence's private part can be as long as the
// whole sequence (a group may share nothing), and up to kMaxTileSplits
// prefix chunks come first.  prefix_row_tiles bounds the tiles over all
// groups.
Plan make_group_plan(int32_t max_seq_len, int32_t partition_blocks, int32_t max_shared_blocks,
                     int32_t num_groups, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads) {
    Plan p = make_plan(max_seq_len, partition_blocks);
    const int32_t tt = tile_tokens(num_q_heads / num_kv_heads);
    p.prefix_row_tiles = (num_seqs + tt - 1) / tt + num_groups;
    p.shared_blocks = max_shared_blocks;
    const int32_t slots = max_shared_blocks < kMaxTileSplits ? max_shared_blocks : kMaxTileSplits;
    p.prefix_splits = slots;
    p.prefix_split_blocks = (max_shared_blocks + slots - 1) / slots;
    p.max_parts += slots;
    p.split = true;
    return p;
}

struct WsLayout {
    size_t off_m, off_l, off_acc, off_parts, off_ctr, bytes;
};

constexpr size_t kCounterBytes = 256;  // the tile kernel's item counter (zeroed by each call)

// q_rows: query-token rows (num_seqs with one query token per sequence).
// counter: the tile kernel runs in the call and needs its item counter (last).
WsLayout ws_layout(int64_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t max_parts,
                   int32_t head_dim, bool split, int64_t q_rows = -1, bool counter = false) {
    WsLayout w{0, 0, 0, 0, 0, 0};
    if (split) {
        const int64_t rows = (q_rows >= 0 ? q_rows : num_seqs) * num_q_heads;
        const size_t ml = align256(static_cast<size_t>(rows) * max_parts * sizeof(float));
        w.off_m = 0;
        w.off_l = ml;
        w.off_acc = 2 * ml;
        w.off_parts = w.off_acc + align256(static_cast<size_t>(rows) * max_parts * head_dim * sizeof(float));
        w.bytes = w.off_parts + align256(static_cast<size_t>(num_seqs) * num_kv_heads * sizeof(int32_t));
    }
    if (counter) {
        w.off_ctr = w.bytes;
        w.bytes += kCounterBytes;
    }
    return w;
}

struct DecodeArgs {
    const float* k_scale = nullptr;    // E4M3 caches: per-kv-head scales (null: bf16/f32 caches)
    const float* v_scale = nullptr;
    const int32_t* q_start = nullptr;  // several query tokens per sequence (null: one)
    int32_t max_q_len = 1;
    int32_t num_q_rows = -1;           // query-token rows (-1: num_seqs)
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    int32_t max_blocks_per_seq;
    const int32_t* seq_lens;
    int32_t max_seq_len;
    int32_t num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size;
    float scale;
    int32_t partition_blocks;
    void* workspace;
    size_t workspace_bytes;
    void* out;
    int32_t dtype;
    cudaStream_t stream;
};

int check_shapes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                 int32_t block_size, int32_t dtype) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (block_size != kBlockTokens) return PA_ERR_UNSUPPORTED;
    if (num_q_heads / num_kv_heads > 16) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

// Validates and fills the kernel parameter block (workspace pointers included).
// shared_blocks > 0: the shared-prefix decode (plan from make_prefix_plan).
int prepare_decode(const DecodeArgs& a, bool need_inputs, DecodeParams* P, Plan* plan,
                   int32_t shared_blocks = 0, int32_t num_groups = 0) {
    int rc = check_shapes(a.num_seqs, a.num_q_heads, a.num_kv_heads, a.head_dim, a.block_size,
                          a.dtype);
    if (rc != PA_OK) return rc;
    if (a.max_blocks_per_seq <= 0 || a.partition_blocks < -1) return PA_ERR_INVALID_ARG;
    if (!a.seq_lens || !aligned(a.seq_lens, 4) || !a.out || !aligned(a.out, 16))
        return PA_ERR_INVALID_ARG;
    if (need_inputs) {
        if (!a.q || !a.k_cache || !a.v_cache || !a.block_tables) return PA_ERR_INVALID_ARG;
        if (!aligned(a.q, 16) || !aligned(a.k_cache, 16) || !aligned(a.v_cache, 16) ||
            !aligned(a.block_tables, 4))
            return PA_ERR_INVALID_ARG;
        if (a.num_blocks <= 0) return PA_ERR_INVALID_ARG;
        // TMA row coordinates and element offsets are 32-bit
        if (static_cast<int64_t>(a.num_blocks) * a.num_kv_heads * kBlockTokens > INT32_MAX)
            return PA_ERR_UNSUPPORTED;
        if (!std::isfinite(a.scale)) return PA_ERR_INVALID_ARG;
    }
    if (a.k_scale || a.v_scale) {  // E4M3 caches: bf16 queries and output
        if (a.dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
        if (!a.k_scale || !a.v_scale || !aligned(a.k_scale, 4) || !aligned(a.v_scale, 4))
            return PA_ERR_INVALID_ARG;
    }
    const int64_t table_tokens = static_cast<int64_t>(a.max_blocks_per_seq) * kBlockTokens;
    const int32_t max_len = a.max_seq_len > 0
                                ? a.max_seq_len
                                : static_cast<int32_t>(table_tokens > INT32_MAX ? INT32_MAX : table_tokens);
    if (shared_blocks > 0) {
        if (a.dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
        if (shared_blocks > a.max_blocks_per_seq ||
            static_cast<int64_t>(shared_blocks) * kBlockTokens > max_len)
            return PA_ERR_INVALID_ARG;
        *plan = num_groups > 0 ? make_group_plan(max_len, a.partition_blocks, shared_blocks, num_groups,
                                                 a.num_seqs, a.num_q_heads, a.num_kv_heads)
                               : make_prefix_plan(max_len, a.partition_blocks, shared_blocks, a.num_seqs,
                                                  a.num_q_heads, a.num_kv_heads);
    } else {
        *plan = make_plan(max_len, a.partition_blocks);
    }
    const int64_t q_rows = a.q_start ? a.num_q_rows : a.num_seqs;
    const WsLayout ws = ws_layout(a.num_seqs, a.num_q_heads, a.num_kv_heads, plan->max_parts,
                                  a.head_dim, plan->split, q_rows, shared_blocks > 0);
    std::memset(P, 0, sizeof *P);
    if (plan->split) {
        if (!a.workspace || !aligned(a.workspace, 256)) return PA_ERR_WORKSPACE;
        if (a.workspace_bytes < ws.bytes) return PA_ERR_WORKSPACE;
        char* w = static_cast<char*>(a.workspace);
        P->ws_m = reinterpret_cast<float*>(w + ws.off_m);
        P->ws_l = reinterpret_cast<float*>(w + ws.off_l);
        P->ws_acc = reinterpret_cast<float*>(w + ws.off_acc);
        P->ws_parts = reinterpret_cast<int32_t*>(w + ws.off_parts);
        if (shared_blocks > 0) P->tile_counter = reinterpret_cast<int32_t*>(w + ws.off_ctr);
    }
    P->q = a.q;
    P->q_start = a.q_start;
    P->max_q_len = a.q_start ? a.max_q_len : 1;
    P->num_q_rows = static_cast<int32_t>(q_rows);
    P->k_cache = a.k_cache;
    P->v_cache = a.v_cache;
    P->k_scale = a.k_scale;
    P->v_scale = a.v_scale;
    P->block_tables = a.block_tables;
    P->seq_lens = a.seq_lens;
    P->out = a.out;
    P->num_seqs = a.num_seqs;
    P->num_q_heads = a.num_q_heads;
    P->num_kv_heads = a.num_kv_heads;
    P->head_dim = a.head_dim;
    P->group = a.num_q_heads / a.num_kv_heads;
    P->max_blocks_per_seq = a.max_blocks_per_seq;
    P->num_blocks = a.num_blocks;
    P->part_blocks = plan->part_blocks;
    P->balanced = plan->balanced ? 1 : 0;
    P->min_chunk = kMinChunk;
    P->max_parts = plan->max_parts;
    P->len_cap = static_cast<int32_t>(max_len < table_tokens ? max_len : table_tokens);
    P->skip_blocks = num_groups > 0 ? 0 : plan->shared_blocks;
    P->piece_base = plan->prefix_splits;
    P->max_shared = plan->shared_blocks;
    P->scale = a.scale;
    P->scale_log2 = a.scale * 1.4426950408889634f;
    return PA_OK;
}

// Sequences per launch: the per-CTA prefix holds at most kMaxSeqsPerLaunch
// entries, and its running sums (blocks x kv heads) must fit in 32 bits.
int32_t seqs_per_launch(const DecodeParams& P) {
    const int64_t nb_cap = (static_cast<int64_t>(P.len_cap) + kBlockTokens - 1) / kBlockTokens;
    const int64_t per_seq = (nb_cap > 0 ? nb_cap : 1) * P.num_kv_heads;
    const int64_t lim = static_cast<int64_t>(INT32_MAX) / per_seq;
    return static_cast<int32_t>(lim < kMaxSeqsPerLaunch ? (lim < 1 ? 1 : lim) : kMaxSeqsPerLaunch);
}

// Launches `kernel` with programmatic stream serialization, so that it may
// begin while the previous kernel in the stream finishes (the kernels call
// griddepcontrol.wait before touching anything that kernel writes).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Shape of the decode launch for one chunk of sequences (shared by the decode
// launch and by the balanced reduction, which recomputes the decode's warp
// ranges).
struct LaunchShape {
    int grid;
    int threads;
    size_t smem;
};

template <int D, int ROWS, bool FP8>
auto mma_kernel() {
    return decode_bf16_mma_kernel<D, ROWS, mma_stages<FP8, ROWS>(), kMmaWarps, mma_min_ctas<FP8, ROWS>(), FP8>;
}

template <typename K>
int shape_of(K kernel, int warps, size_t smem, const DecodeParams& P, LaunchShape* L) {
    const int64_t max_pieces = static_cast<int64_t>(P.seq_count) * P.num_kv_heads * P.max_parts;
    L->threads = warps * 32;
    L->smem = smem;
    return persistent_grid(kernel, L->threads, smem, (max_pieces + warps - 1) / warps, &L->grid);
}

template <int D, int ROWS, bool FP8>
int mma_shape(const DecodeParams& P, LaunchShape* L) {
    using Cfg = MmaCfg<D, mma_stages<FP8, ROWS>(), kMmaWarps, FP8>;
    auto kernel = mma_kernel<D, ROWS, FP8>();
    int rc = ensure_smem_attr(kernel, Cfg::smem_bytes(kMaxSeqsPerLaunch));
    if (rc != PA_OK) return rc;
    return shape_of(kernel, kMmaWarps, Cfg::smem_bytes(P.seq_count), P, L);
}

template <int D, int MAXG>
int simt_shape(const DecodeParams& P, LaunchShape* L) {
    return shape_of(decode_f32_simt_kernel<D, MAXG>, kSimtWarps, 12 * static_cast<size_t>(P.seq_count + 1),
                    P, L);
}

template <bool FP8>
int mma_shape_for(const DecodeParams& P, LaunchShape* L) {
    const int rows = P.group * P.max_q_len;
    if constexpr (FP8) {  // one query row: the E4M3 kernel's single-column form
        if (rows <= 1) return P.head_dim == 128 ? mma_shape<128, 1, FP8>(P, L) : mma_shape<64, 1, FP8>(P, L);
    }
    if (P.head_dim == 128)
        return rows <= 8 ? mma_shape<128, 8, FP8>(P, L) : mma_shape<128, 16, FP8>(P, L);
    return rows <= 8 ? mma_shape<64, 8, FP8>(P, L) : mma_shape<64, 16, FP8>(P, L);
}

// fp8: the E4M3 form of the decode kernel (caches of 8-bit codes).
int decode_shape(const DecodeParams& P, int32_t dtype, bool fp8, LaunchShape* L) {
    if (dtype == PA_DTYPE_BF16)
        return fp8 ? mma_shape_for<true>(P, L) : mma_shape_for<false>(P, L);
    if (P.head_dim == 128) return P.group <= 4 ? simt_shape<128, 4>(P, L) : simt_shape<128, 16>(P, L);
    return P.group <= 4 ? simt_shape<64, 4>(P, L) : simt_shape<64, 16>(P, L);
}

// Calls fn(chunk_params) for each launch chunk of sequences.
template <typename F>
int for_each_chunk(const DecodeParams& base, F fn) {
    const int32_t chunk = seqs_per_launch(base);
    for (int32_t b = 0; b < base.num_seqs; b += chunk) {
        DecodeParams P = base;
        P.seq_begin = b;
        P.seq_count = base.num_seqs - b < chunk ? base.num_seqs - b : chunk;
        const int rc = fn(P);
        if (rc != PA_OK) return rc;
    }
    return PA_OK;
}

template <int D, int ROWS, bool FP8>
int launch_mma(const DecodeParams& base, cudaStream_t st) {
    const int64_t rows = static_cast<int64_t>(base.num_blocks) * base.num_kv_heads * kBlockTokens;
    alignas(64) CUtensorMap mk, mv;
    int rc;
    if ((rc = encode_pool_map(&mk, base.k_cache, rows, D, FP8)) != PA_OK) return rc;
    if ((rc = encode_pool_map(&mv, base.v_cache, rows, D, FP8)) != PA_OK) return rc;
    return for_each_chunk(base, [&](const DecodeParams& P) {
        LaunchShape L;
        int r = mma_shape<D, ROWS, FP8>(P, &L);
        if (r != PA_OK) return r;
        cudaError_t e = launch_pdl(mma_kernel<D, ROWS, FP8>(), dim3(L.grid), dim3(L.threads), L.smem,
                                   st, mk, mv, P);
        return e == cudaSuccess ? PA_OK : cuda_fail(e, "decode_bf16_mma_kernel launch");
    });
}

template <int D, int MAXG>
int launch_simt(const DecodeParams& base, cudaStream_t st) {
    return for_each_chunk(base, [&](const DecodeParams& P) {
        LaunchShape L;
        int r = simt_shape<D, MAXG>(P, &L);
        if (r != PA_OK) return r;
        cudaError_t e = launch_pdl(decode_f32_simt_kernel<D, MAXG>, dim3(L.grid), dim3(L.threads),
                                   L.smem, st, P);
        return e == cudaSuccess ? PA_OK : cuda_fail(e, "decode_f32_simt_kernel launch");
    });
}

template <bool FP8>
int launch_mma_for(const DecodeParams& P, cudaStream_t st) {
    const int rows = P.group * P.max_q_len;  // query rows of one (sequence, kv head) unit
    if constexpr (FP8) {  // one query row: the E4M3 kernel's single-column form
        if (rows <= 1) return P.head_dim == 128 ? launch_mma<128, 1, FP8>(P, st) : launch_mma<64, 1, FP8>(P, st);
    }
    if (P.head_dim == 128)
        return rows <= 8 ? launch_mma<128, 8, FP8>(P, st) : launch_mma<128, 16, FP8>(P, st);
    return rows <= 8 ? launch_mma<64, 8, FP8>(P, st) : launch_mma<64, 16, FP8>(P, st);
}

int run_partitions(const DecodeParams& P, int32_t dtype, cudaStream_t st) {
    if (P.num_seqs == 0) return PA_OK;
    if (dtype == PA_DTYPE_BF16)
        return P.k_scale ? launch_mma_for<true>(P, st) : launch_mma_for<false>(P, st);
    if (P.head_dim == 128) return P.group <= 4 ? launch_simt<128, 4>(P, st) : launch_simt<128, 16>(P, st);
    return P.group <= 4 ? launch_simt<64, 4>(P, st) : launch_simt<64, 16>(P, st);
}

// ------------------------------------------------------------ tile kernel (tcgen05)
// q seen as a 3-D tensor [rows][num_q_heads][head_dim], loaded in boxes of 64
// columns x `group` heads x half_tokens rows: one box lands as a half tile's
// half_tokens * group query rows of 128 bytes (one 64-column slab), in the
// 128-byte swizzle the tensor-core descriptors expect.
int encode_q_map(CUtensorMap* map, const void* q, int64_t rows, int32_t num_q_heads, int head_dim,
                 int32_t group) {
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    int rc = get_encoder(&enc);
    if (rc != PA_OK) return rc;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                          static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                             static_cast<cuuint64_t>(num_q_heads) * head_dim * 2};
    cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(half_tokens(group))};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                      "cuTensorMapEncodeTiled (q) failed (CUresult %d)", static_cast<int>(r));
        return PA_ERR_CUDA;
    }
    return PA_OK;
}

struct TileSplit {
    int32_t splits;        // key chunks of the longest unit
    int32_t chunk_blocks;  // blocks per chunk, a multiple of the 4-block step
};

// Key chunking for `work_tiles` (tile, kv head) pairs over units of at most
// nb_max key blocks: as many chunks as fill the device's SMs (one tile-kernel
// CTA each), at most kMaxTileSplits; one chunk when the tiles alone fill it.
// Long units are cut further, up to kBalanceItemsPerSm items per SM, as long
// as every chunk keeps at least kMinBalanceChunk blocks: the heaviest-first
// claiming then evens out the CTAs' work (a few items of very different
// lengths per SM would leave the last wave half empty), while an item's start
// and epilogue (~10 us) stay small next to its steps.
constexpr int64_t kBalanceItemsPerSm = 16;
constexpr int64_t kMinBalanceChunk = 256;  // 64 steps of 64 keys
TileSplit choose_tile_split(int sms, int64_t work_tiles, int32_t nb_max) {
    if (nb_max < 1) nb_max = 1;
    int64_t want = work_tiles > 0 ? sms / work_tiles : 1;
    if (want < 1) want = 1;
    if (work_tiles > 0) {
        const int64_t bal = (kBalanceItemsPerSm * sms + work_tiles - 1) / work_tiles;
        const int64_t by_len = nb_max / kMinBalanceChunk;
        const int64_t b = bal < by_len ? bal : by_len;
        if (b > want) want = b;
    }
    if (want > kMaxTileSplits) want = kMaxTileSplits;
    int32_t ch = static_cast<int32_t>((nb_max + want - 1) / want);
    ch = (ch + kTileStepBlocks - 1) / kTileStepBlocks * kTileStepBlocks;
    return TileSplit{(nb_max + ch - 1) / ch, ch};
}

// counter_zeroed: the caller set the item counter to zero before (the
// shared-prefix tiles launched after the private-block decode: a memset
// between the two would keep the tiles from starting early).
template <int D>
int launch_tiles(const TileParams& base, const void* q, int64_t q_rows, const void* k_cache,
                 const void* v_cache, int64_t items_bound, cudaStream_t st, bool counter_zeroed = false) {
    auto kernel = attn_tiles_tc_kernel<D>;
    int rc = ensure_smem_attr(kernel, TileCfg<D>::kSmem);
    if (rc != PA_OK) return rc;
    const int64_t rows = static_cast<int64_t>(base.num_blocks) * base.num_kv_heads * kBlockTokens;
    alignas(64) CUtensorMap mk, mv, mq;
    if ((rc = encode_pool_map(&mk, k_cache, rows, D)) != PA_OK) return rc;
    if ((rc = encode_pool_map_blocks(&mv, v_cache, rows, D)) != PA_OK) return rc;
    if ((rc = encode_q_map(&mq, q, q_rows > 0 ? q_rows : 1, base.num_q_heads, D, base.group)) != PA_OK) return rc;
    DeviceInfo di;
    if ((rc = device_info(&di)) != PA_OK) return rc;
    const int32_t units = base.num_units;
    for (int32_t b = 0; b < units; b += TileCfg<D>::kMaxUnits) {
        TileParams P = base;
        P.unit_begin = base.unit_begin + b;
        P.num_units = units - b < TileCfg<D>::kMaxUnits ? units - b : TileCfg<D>::kMaxUnits;
        int64_t grid = items_bound < di.sms ? items_bound : di.sms;
        if (grid < 1) grid = 1;
        cudaError_t e;
        if (items_bound > grid) {
            // more items than CTAs: they are claimed from a counter, which starts at zero
            if (!counter_zeroed) {
                e = cudaMemsetAsync(P.item_counter, 0, sizeof(int32_t), st);
                if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (tile item counter)");
            }
        } else {
            P.item_counter = nullptr;  // at most one item per CTA: no counter
        }
        e = launch_pdl(kernel, dim3(static_cast<unsigned>(grid)), dim3(TileCfg<D>::kThreads),
                                   TileCfg<D>::kSmem, st, mk, mv, mq, P);
        if (e != cudaSuccess) return cuda_fail(e, "attn_tiles_tc_kernel launch");
    }
    return PA_OK;
}

// The shared prefixes' key chunks through the tile kernel (prefix mode: one
// group of every sequence, or P.num_groups groups from P.group_start /
// P.group_blocks): the launch's parameters and item count; sets
// plan->prefix_splits / prefix_split_blocks.
struct PrefixTiles {
    TileParams T;
    int64_t items;
    int sms;
};

int plan_prefix_tiles(const DecodeParams& P, Plan* plan, PrefixTiles* pt) {
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc != PA_OK) return rc;
    const TileSplit sp = choose_tile_split(di.sms, static_cast<int64_t>(plan->prefix_row_tiles) * P.num_kv_heads,
                                           plan->shared_blocks);
    plan->prefix_splits = sp.splits;
    plan->prefix_split_blocks = sp.chunk_blocks;
    TileParams& T = pt->T;
    std::memset(&T, 0, sizeof T);
    T.block_tables = P.block_tables;
    T.seq_lens = P.seq_lens;
    T.ws_m = P.ws_m;
    T.ws_l = P.ws_l;
    T.ws_acc = P.ws_acc;
    T.item_counter = P.tile_counter;
    T.mode = kTileModePrefix;
    T.unit_begin = 0;
    T.num_units = P.group_start ? P.num_groups : 1;
    T.group_start = P.group_start;
    T.group_blocks = P.group_blocks;
    T.num_seqs = P.num_seqs;
    T.num_q_heads = P.num_q_heads;
    T.num_kv_heads = P.num_kv_heads;
    T.group = P.group;
    T.half_tokens = half_tokens(P.group);
    T.max_blocks_per_seq = P.max_blocks_per_seq;
    T.num_blocks = P.num_blocks;
    T.chunk_blocks = sp.chunk_blocks;
    T.max_parts = P.max_parts;
    T.len_cap = P.len_cap;
    T.shared_blocks = plan->shared_blocks;
    T.scale_log2 = P.scale_log2;
    pt->items = static_cast<int64_t>(plan->prefix_row_tiles) * P.num_kv_heads * sp.splits;
    pt->sms = di.sms;
    return PA_OK;
}

int launch_prefix_tiles(const DecodeParams& P, const PrefixTiles& pt, cudaStream_t st, bool counter_zeroed) {
    return P.head_dim == 128
               ? launch_tiles<128>(pt.T, P.q, P.num_seqs, P.k_cache, P.v_cache, pt.items, st, counter_zeroed)
               : launch_tiles<64>(pt.T, P.q, P.num_seqs, P.k_cache, P.v_cache, pt.items, st, counter_zeroed);
}

template <typename OutT, int D>
int launch_reduce(const DecodeParams& base, int32_t dtype, bool fp8, cudaStream_t st) {
    if (base.q_start && !(base.balanced && base.piece_base == 0)) {
        // row-wise merge over every query-token row at once (rows locate their
        // sequence through q_start)
        DecodeParams P = base;
        P.seq_begin = 0;
        P.seq_count = base.num_seqs;
        const int64_t rows = static_cast<int64_t>(P.num_q_rows) * P.num_q_heads;
        if (rows == 0) return PA_OK;
        cudaError_t e;
        if (P.max_parts > kWideReducePieces)
            e = launch_pdl(lse_reduce_wide_kernel<OutT, D>, dim3(static_cast<unsigned>(rows)),
                           dim3(kWideWarps * 32), 0, st, P);
        else
            e = launch_pdl(lse_reduce_kernel<OutT, D>,
                           dim3(static_cast<unsigned>((rows + kReduceWarps - 1) / kReduceWarps)),
                           dim3(kReduceWarps * 32), 0, st, P);
        return e == cudaSuccess ? PA_OK : cuda_fail(e, "lse_reduce_kernel launch");
    }
    return for_each_chunk(base, [&](const DecodeParams& P) {
        cudaError_t e;
        if (P.balanced && P.piece_base == 0) {
            LaunchShape L;
            int r = decode_shape(P, dtype, fp8, &L);
            if (r != PA_OK) return r;
            const int decode_warps = L.grid * (L.threads / 32);
            if (decode_warps < 2) return PA_OK;  // one warp range: nothing was cut
            e = launch_pdl(lse_reduce_balanced_kernel<OutT, D>, dim3(decode_warps - 1),
                           dim3(kReduceWarps * 32), 12 * static_cast<size_t>(P.seq_count + 1), st, P,
                           decode_warps);
        } else {
            const int64_t rows = static_cast<int64_t>(P.seq_count) * P.num_q_heads;
            if (P.max_parts > kWideReducePieces) {  // many pieces per row: a CTA per row
                e = launch_pdl(lse_reduce_wide_kernel<OutT, D>, dim3(static_cast<unsigned>(rows)),
                               dim3(kWideWarps * 32), 0, st, P);
            } else {
                const unsigned grid = static_cast<unsigned>((rows + kReduceWarps - 1) / kReduceWarps);
                e = launch_pdl(lse_reduce_kernel<OutT, D>, dim3(grid), dim3(kReduceWarps * 32), 0, st, P);
            }
        }
        return e == cudaSuccess ? PA_OK : cuda_fail(e, "lse_reduce_kernel launch");
    });
}

// fp8: the partials came from the E4M3 decode kernel (whose launch shape the
// balanced merge recomputes); by default, when P carries the E4M3 scales.
int run_reduce(const DecodeParams& P, const Plan& plan, int32_t dtype, cudaStream_t st, int fp8 = -1) {
    if (P.num_seqs == 0 || !plan.split) return PA_OK;
    const bool f8 = fp8 < 0 ? P.k_scale != nullptr : fp8 != 0;
    if (dtype == PA_DTYPE_BF16)
        return P.head_dim == 128 ? launch_reduce<__nv_bfloat16, 128>(P, dtype, f8, st)
                                 : launch_reduce<__nv_bfloat16, 64>(P, dtype, f8, st);
    return P.head_dim == 128 ? launch_reduce<float, 128>(P, dtype, f8, st)
                             : launch_reduce<float, 64>(P, dtype, f8, st);
}

// The shared-prefix decode's three steps.  The private blocks' decode goes
// first and the prefix tiles right after it, marked independent: the tiles'
// CTAs take each SM the decode leaves (its slowest warps' tail) instead of
// waiting for the whole grid, and their start-up (cold Q and K/V loads) hides
// under it.  The merge waits for the tiles, which wait for the decode before
// they complete.  With more prompt groups than one tile launch holds, the
// tiles launch in several grids and go first, each waiting as usual.
int run_shared_prefix(DecodeParams& P, Plan& plan, int32_t dtype, cudaStream_t st) {
    PrefixTiles pt;
    int rc = plan_prefix_tiles(P, &plan, &pt);
    if (rc != PA_OK) return rc;
    // the private pieces follow the chunks actually used (the most a group has);
    // a group's own chunk count follows from its shared blocks and the chunk size
    P.piece_base = plan.prefix_splits;
    P.group_chunk = plan.prefix_split_blocks;
    const int32_t max_units = P.head_dim == 128 ? TileCfg<128>::kMaxUnits : TileCfg<64>::kMaxUnits;
    if (pt.T.num_units <= max_units) {
        if (pt.items > pt.sms) {  // the tiles claim items from the counter: zero it before the decode
            cudaError_t e = cudaMemsetAsync(pt.T.item_counter, 0, sizeof(int32_t), st);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (tile item counter)");
        }
        rc = run_partitions(P, dtype, st);
        if (rc != PA_OK) return rc;
        pt.T.independent = 1;
        rc = launch_prefix_tiles(P, pt, st, true);
    } else {
        rc = launch_prefix_tiles(P, pt, st, false);
        if (rc != PA_OK) return rc;
        rc = run_partitions(P, dtype, st);
    }
    if (rc != PA_OK) return rc;
    return run_reduce(P, plan, dtype, st);
}

// Several query tokens per sequence with group * max_q_len > 16 (prefill
// chunks): the tile kernel in prefill mode, then, when the keys were cut into
// chunks, the row-wise merge of each row's chunks.
struct PrefillPlan {
    TileSplit split;
    int64_t tiles_bound;  // tiles over all sequences, at most
    WsLayout ws;
};

PrefillPlan make_prefill_plan(int sms, int32_t num_seqs, int32_t num_q_rows, int32_t num_q_heads,
                              int32_t num_kv_heads, int32_t head_dim, int32_t max_len) {
    PrefillPlan pp;
    const int32_t tt = tile_tokens(num_q_heads / num_kv_heads);
    pp.tiles_bound = (static_cast<int64_t>(num_q_rows) + tt - 1) / tt + num_seqs;
    pp.split = choose_tile_split(sms, pp.tiles_bound * num_kv_heads, (max_len + kBlockTokens - 1) / kBlockTokens);
    pp.ws = ws_layout(num_seqs, num_q_heads, num_kv_heads, pp.split.splits, head_dim, pp.split.splits > 1,
                      num_q_rows, true);
    return pp;
}

int run_prefill_tiles(const DecodeArgs& a) {
    int rc = check_shapes(a.num_seqs, a.num_q_heads, a.num_kv_heads, a.head_dim, a.block_size, a.dtype);
    if (rc != PA_OK) return rc;
    if (a.dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
    if (a.max_blocks_per_seq <= 0 || a.partition_blocks < -1 || a.num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (!a.q || !a.k_cache || !a.v_cache || !a.block_tables || !a.seq_lens || !a.out || !a.q_start)
        return PA_ERR_INVALID_ARG;
    if (!aligned(a.q, 16) || !aligned(a.k_cache, 16) || !aligned(a.v_cache, 16) || !aligned(a.out, 16) ||
        !aligned(a.block_tables, 4) || !aligned(a.seq_lens, 4) || !aligned(a.q_start, 4))
        return PA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(a.num_blocks) * a.num_kv_heads * kBlockTokens > INT32_MAX) return PA_ERR_UNSUPPORTED;
    if (!std::isfinite(a.scale)) return PA_ERR_INVALID_ARG;
    if (a.num_seqs == 0 || a.num_q_rows == 0) return PA_OK;
    const int64_t table_tokens = static_cast<int64_t>(a.max_blocks_per_seq) * kBlockTokens;
    const int32_t max_len = a.max_seq_len > 0
                                ? a.max_seq_len
                                : static_cast<int32_t>(table_tokens > INT32_MAX ? INT32_MAX : table_tokens);
    // the workspace holds at least the item counter (checked before any CUDA call)
    if (!a.workspace || !aligned(a.workspace, 256) || a.workspace_bytes < kCounterBytes) return PA_ERR_WORKSPACE;
    DeviceInfo di;
    if ((rc = device_info(&di)) != PA_OK) return rc;
    const PrefillPlan pp = make_prefill_plan(di.sms, a.num_seqs, a.num_q_rows, a.num_q_heads, a.num_kv_heads,
                                             a.head_dim, max_len);
    const bool direct = pp.split.splits == 1;
    float* ws_m = nullptr;
    float* ws_l = nullptr;
    float* ws_acc = nullptr;
    if (!a.workspace || !aligned(a.workspace, 256) || a.workspace_bytes < pp.ws.bytes) return PA_ERR_WORKSPACE;
    char* w = static_cast<char*>(a.workspace);
    if (!direct) {
        ws_m = reinterpret_cast<float*>(w + pp.ws.off_m);
        ws_l = reinterpret_cast<float*>(w + pp.ws.off_l);
        ws_acc = reinterpret_cast<float*>(w + pp.ws.off_acc);
    }
    TileParams T;
    std::memset(&T, 0, sizeof T);
    T.block_tables = a.block_tables;
    T.seq_lens = a.seq_lens;
    T.q_start = a.q_start;
    T.out = a.out;
    T.ws_m = ws_m;
    T.ws_l = ws_l;
    T.ws_acc = ws_acc;
    T.item_counter = reinterpret_cast<int32_t*>(w + pp.ws.off_ctr);
    T.mode = kTileModePrefill;
    T.unit_begin = 0;
    T.num_units = a.num_seqs;
    T.num_seqs = a.num_seqs;
    T.num_q_heads = a.num_q_heads;
    T.num_kv_heads = a.num_kv_heads;
    T.group = a.num_q_heads / a.num_kv_heads;
    T.half_tokens = half_tokens(T.group);
    T.max_blocks_per_seq = a.max_blocks_per_seq;
    T.num_blocks = a.num_blocks;
    T.chunk_blocks = pp.split.chunk_blocks;
    T.max_parts = pp.split.splits;
    T.len_cap = static_cast<int32_t>(max_len < table_tokens ? max_len : table_tokens);
    T.max_q_len = a.max_q_len;
    T.direct = direct ? 1 : 0;
    T.scale_log2 = a.scale * 1.4426950408889634f;
    const int64_t items = pp.tiles_bound * a.num_kv_heads * pp.split.splits;
    rc = a.head_dim == 128 ? launch_tiles<128>(T, a.q, a.num_q_rows, a.k_cache, a.v_cache, items, a.stream)
                           : launch_tiles<64>(T, a.q, a.num_q_rows, a.k_cache, a.v_cache, items, a.stream);
    if (rc != PA_OK || direct) return rc;
    // the row-wise merge of each row's chunks (their number follows from the row's tile)
    DecodeParams R;
    std::memset(&R, 0, sizeof R);
    R.seq_lens = a.seq_lens;
    R.q_start = a.q_start;
    R.out = a.out;
    R.ws_m = ws_m;
    R.ws_l = ws_l;
    R.ws_acc = ws_acc;
    R.max_q_len = a.max_q_len;
    R.num_q_rows = a.num_q_rows;
    R.num_seqs = a.num_seqs;
    R.seq_count = a.num_seqs;
    R.num_q_heads = a.num_q_heads;
    R.num_kv_heads = a.num_kv_heads;
    R.head_dim = a.head_dim;
    R.group = T.group;
    R.max_parts = pp.split.splits;
    R.len_cap = T.len_cap;
    R.part_blocks = kNoSplit;
    R.tile_tokens = tile_tokens(T.group);
    R.tile_chunk = pp.split.chunk_blocks;
    const int64_t rows = static_cast<int64_t>(a.num_q_rows) * a.num_q_heads;
    const unsigned grid = static_cast<unsigned>((rows + kReduceWarps - 1) / kReduceWarps);
    cudaError_t e = a.head_dim == 128
                        ? launch_pdl(lse_reduce_kernel<__nv_bfloat16, 128>, dim3(grid), dim3(kReduceWarps * 32), 0,
                                     a.stream, R)
                        : launch_pdl(lse_reduce_kernel<__nv_bfloat16, 64>, dim3(grid), dim3(kReduceWarps * 32), 0,
                                     a.stream, R);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "lse_reduce_kernel launch");
}

DecodeArgs make_args(const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                     const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                     int32_t num_blocks, int32_t block_size, float scale,
                     int32_t partition_blocks, void* workspace, size_t workspace_bytes, void* out,
                     int32_t dtype, void* stream) {
    DecodeArgs a;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.seq_lens = seq_lens;
    a.max_seq_len = max_seq_len;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.head_dim = head_dim;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    a.scale = scale;
    a.partition_blocks = partition_blocks;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    a.out = out;
    a.dtype = dtype;
    a.stream = static_cast<cudaStream_t>(stream);
    return a;
}

}  // namespace

extern "C" {

int pa_cache_write(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                   int32_t num_kv_heads, int32_t head_dim, void* k_cache, void* v_cache,
                   int32_t num_blocks, int32_t block_size, int32_t dtype, void* stream) {
    int rc = check_shapes(0, num_kv_heads, num_kv_heads, head_dim, block_size, dtype);
    if (rc != PA_OK) return rc;
    if (num_tokens < 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(slot_mapping, 8))
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    const int32_t elem = dtype == PA_DTYPE_F32 ? 4 : 2;
    const int32_t chunks_per_row = head_dim * elem / 16;
    const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * chunks_per_row;
    const int64_t grid = (total + 255) / 256;
    if (grid > INT32_MAX) return PA_ERR_UNSUPPORTED;
    cache_write_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, total,
        num_kv_heads, chunks_per_row, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
        static_cast<int64_t>(num_blocks) * kBlockTokens);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "cache_write_kernel launch");
    return PA_OK;
}

int pa_cache_write_fp8(const void* k, const void* v, const int64_t* slot_mapping,
                       int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim, void* k_cache,
                       void* v_cache, int32_t num_blocks, int32_t block_size,
                       const float* k_inv_scale, const float* v_inv_scale, void* stream) {
    int rc = check_shapes(0, num_kv_heads, num_kv_heads, head_dim, block_size, PA_DTYPE_BF16);
    if (rc != PA_OK) return rc;
    if (num_tokens < 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache || !k_inv_scale || !v_inv_scale)
        return PA_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(slot_mapping, 8) || !aligned(k_inv_scale, 4) || !aligned(v_inv_scale, 4))
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    const int32_t chunks_per_row = head_dim / 16;  // 16 values per thread
    const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * chunks_per_row;
    const int64_t grid = (total + 255) / 256;
    if (grid > INT32_MAX) return PA_ERR_UNSUPPORTED;
    cache_write_fp8_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, total,
        num_kv_heads, chunks_per_row, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
        static_cast<int64_t>(num_blocks) * kBlockTokens, k_inv_scale, v_inv_scale);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "cache_write_fp8_kernel launch");
}

int pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* src, const int32_t* dst,
                   int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                   int32_t block_size, int32_t dtype, void* stream) {
    int rc = check_shapes(0, num_kv_heads, num_kv_heads, head_dim, block_size, dtype);
    if (rc != PA_OK) return rc;
    if (num_pairs < 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !src || !dst || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(src, 4) || !aligned(dst, 4))
        return PA_ERR_INVALID_ARG;
    const int32_t elem = dtype == PA_DTYPE_F32 ? 4 : 2;
    const int64_t chunks = static_cast<int64_t>(num_kv_heads) * kBlockTokens * head_dim * elem / 16;
    DeviceInfo di;
    if ((rc = device_info(&di)) != PA_OK) return rc;
    const int64_t want = (static_cast<int64_t>(num_pairs) * chunks + 255) / 256;
    const int64_t cap = static_cast<int64_t>(di.sms) * 8;
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    copy_blocks_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), src, dst, num_pairs, chunks,
        num_blocks);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "copy_blocks_kernel launch");
}

int32_t pa_decode_partition_blocks(int32_t num_seqs, int32_t num_kv_heads, int32_t max_seq_len,
                                   int32_t block_size, int32_t partition_blocks) {
    if (num_seqs < 0 || num_kv_heads <= 0 || max_seq_len < 0 || partition_blocks < -1)
        return PA_ERR_INVALID_ARG;
    if (block_size != kBlockTokens) return PA_ERR_UNSUPPORTED;
    return resolve_part_blocks(partition_blocks);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                int32_t head_dim, int32_t max_seq_len, int32_t block_size,
                                int32_t partition_blocks) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        max_seq_len < 0 || block_size != kBlockTokens || partition_blocks < -1)
        return 0;
    const Plan plan = make_plan(max_seq_len, partition_blocks);
    return ws_layout(num_seqs, num_q_heads, num_kv_heads, plan.max_parts, head_dim, plan.split).bytes;
}

int pa_decode_partitions(const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, int32_t max_blocks_per_seq,
                         const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                         int32_t num_blocks, int32_t block_size, float scale,
                         int32_t partition_blocks, void* workspace, size_t workspace_bytes,
                         void* out, int32_t dtype, void* stream) {
    const DecodeArgs a = make_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                                   max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim,
                                   num_blocks, block_size, scale, partition_blocks, workspace,
                                   workspace_bytes, out, dtype, stream);
    DecodeParams P;
    Plan plan;
    int rc = prepare_decode(a, true, &P, &plan);
    if (rc != PA_OK) return rc;
    return run_partitions(P, dtype, a.stream);
}

int pa_decode_reduce(const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                     int32_t max_blocks_per_seq, int32_t block_size, int32_t partition_blocks,
                     const void* workspace, size_t workspace_bytes, void* out, int32_t dtype,
                     void* stream) {
    const DecodeArgs a = make_args(nullptr, nullptr, nullptr, nullptr, max_blocks_per_seq, seq_lens,
                                   max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim, 1,
                                   block_size, 1.0f, partition_blocks,
                                   const_cast<void*>(workspace), workspace_bytes, out, dtype,
                                   stream);
    DecodeParams P;
    Plan plan;
    int rc = prepare_decode(a, false, &P, &plan);
    if (rc != PA_OK) return rc;
    return run_reduce(P, plan, dtype, a.stream, 0);
}

int pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
              int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t max_seq_len,
              int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
              int32_t num_blocks, int32_t block_size, float scale, int32_t partition_blocks,
              void* workspace, size_t workspace_bytes, void* out, int32_t dtype, void* stream) {
    const DecodeArgs a = make_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                                   max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim,
                                   num_blocks, block_size, scale, partition_blocks, workspace,
                                   workspace_bytes, out, dtype, stream);
    DecodeParams P;
    Plan plan;
    int rc = prepare_decode(a, true, &P, &plan);
    if (rc != PA_OK) return rc;
    rc = run_partitions(P, dtype, a.stream);
    if (rc != PA_OK) return rc;
    return run_reduce(P, plan, dtype, a.stream);
}

int pa_decode_fp8(const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                  const float* v_scale, const int32_t* block_tables, int32_t max_blocks_per_seq,
                  const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                  int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                  int32_t block_size, float scale, int32_t partition_blocks, void* workspace,
                  size_t workspace_bytes, void* out, void* stream) {
    if (!k_scale || !v_scale) return PA_ERR_INVALID_ARG;
    DecodeArgs a = make_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                             max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                             block_size, scale, partition_blocks, workspace, workspace_bytes, out,
                             PA_DTYPE_BF16, stream);
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    DecodeParams P;
    Plan plan;
    int rc = prepare_decode(a, true, &P, &plan);
    if (rc != PA_OK) return rc;
    rc = run_partitions(P, PA_DTYPE_BF16, a.stream);
    if (rc != PA_OK) return rc;
    return run_reduce(P, plan, PA_DTYPE_BF16, a.stream);
}

int pa_decode_fp8_partitions(const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                             const float* v_scale, const int32_t* block_tables, int32_t max_blocks_per_seq,
                             const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                             int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                             int32_t block_size, float scale, int32_t partition_blocks, void* workspace,
                             size_t workspace_bytes, void* out, void* stream) {
    if (!k_scale || !v_scale) return PA_ERR_INVALID_ARG;
    DecodeArgs a = make_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                             max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                             block_size, scale, partition_blocks, workspace, workspace_bytes, out,
                             PA_DTYPE_BF16, stream);
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    DecodeParams P;
    Plan plan;
    int rc = prepare_decode(a, true, &P, &plan);
    if (rc != PA_OK) return rc;
    return run_partitions(P, PA_DTYPE_BF16, a.stream);
}

int pa_decode_fp8_reduce(const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t head_dim, int32_t max_blocks_per_seq, int32_t block_size,
                         int32_t partition_blocks, const void* workspace, size_t workspace_bytes, void* out,
                         void* stream) {
    const DecodeArgs a = make_args(nullptr, nullptr, nullptr, nullptr, max_blocks_per_seq, seq_lens,
                                   max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim, 1,
                                   block_size, 1.0f, partition_blocks,
                                   const_cast<void*>(workspace), workspace_bytes, out, PA_DTYPE_BF16,
                                   stream);
    DecodeParams P;
    Plan plan;
    int rc = prepare_decode(a, false, &P, &plan);
    if (rc != PA_OK) return rc;
    return run_reduce(P, plan, PA_DTYPE_BF16, a.stream, 1);
}

// ------------------------------------------------------------ no-allocation decode
// The split-K scratch of pa_decode_noalloc: one file-scope device array of a
// fixed size, present on every device that loads the library.  Host code must
// not pass the name itself to a kernel (on the host it is only a stand-in);
// its device address is looked up once per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device (looked up on
// the first call per device, with that device current).
int noalloc_scratch(void** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return PA_OK;
}
}  // namespace

int pa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                      const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                      int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                      int32_t num_blocks, int32_t block_size, float scale,
                      int32_t partition_blocks, void* out, int32_t dtype, void* stream) {
    int rc = check_shapes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, dtype);
    if (rc != PA_OK) return rc;
    if (max_blocks_per_seq <= 0 || partition_blocks < -1) return PA_ERR_INVALID_ARG;
    // the same effective bound pa_decode sizes its workspace with
    const int64_t table_tokens = static_cast<int64_t>(max_blocks_per_seq) * kBlockTokens;
    const int32_t max_len = max_seq_len > 0
                                ? max_seq_len
                                : static_cast<int32_t>(table_tokens > INT32_MAX ? INT32_MAX : table_tokens);
    const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                 max_len, block_size, partition_blocks);
    if (need > PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    if (need > 0 && (rc = noalloc_scratch(&scratch)) != PA_OK) return rc;
    return pa_decode(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, max_seq_len,
                     num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, scale,
                     partition_blocks, scratch, need > 0 ? PA_NOALLOC_SCRATCH_BYTES : 0, out,
                     dtype, stream);
}

int pa_decode_shared_prefix(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* seq_lens, int32_t max_seq_len, int32_t shared_blocks,
                            int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
                            int32_t partition_blocks, void* workspace, size_t workspace_bytes,
                            void* out, int32_t dtype, void* stream) {
    if (shared_blocks < 0) return PA_ERR_INVALID_ARG;
    if (shared_blocks == 0)
        return pa_decode(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                         max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                         block_size, scale, partition_blocks, workspace, workspace_bytes, out,
                         dtype, stream);
    const DecodeArgs a = make_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                                   max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim,
                                   num_blocks, block_size, scale, partition_blocks, workspace,
                                   workspace_bytes, out, dtype, stream);
    DecodeParams P;
    Plan plan;
    int rc = prepare_decode(a, true, &P, &plan, shared_blocks);
    if (rc != PA_OK) return rc;
    if (num_seqs == 0) return PA_OK;
    return run_shared_prefix(P, plan, dtype, a.stream);
}

int pa_decode_shared_prefix_groups(const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* block_tables, int32_t max_blocks_per_seq,
                                   const int32_t* seq_lens, int32_t max_seq_len, const int32_t* group_start,
                                   const int32_t* group_shared_blocks, int32_t num_groups,
                                   int32_t max_shared_blocks, int32_t num_seqs, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks, int32_t block_size,
                                   float scale, int32_t partition_blocks, void* workspace, size_t workspace_bytes,
                                   void* out, int32_t dtype, void* stream) {
    if (!group_start || !group_shared_blocks || !aligned(group_start, 4) || !aligned(group_shared_blocks, 4) ||
        num_groups < 1 || max_shared_blocks < 0)
        return PA_ERR_INVALID_ARG;
    if (max_shared_blocks == 0)
        return pa_decode(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, max_seq_len, num_seqs,
                         num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, scale, partition_blocks,
                         workspace, workspace_bytes, out, dtype, stream);
    const DecodeArgs a = make_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                                   max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim,
                                   num_blocks, block_size, scale, partition_blocks, workspace,
                                   workspace_bytes, out, dtype, stream);
    DecodeParams P;
    Plan plan;
    int rc = prepare_decode(a, true, &P, &plan, max_shared_blocks, num_groups);
    if (rc != PA_OK) return rc;
    if (num_seqs == 0) return PA_OK;
    P.group_start = group_start;
    P.group_blocks = group_shared_blocks;
    P.num_groups = num_groups;
    return run_shared_prefix(P, plan, dtype, a.stream);
}

size_t pa_decode_shared_prefix_groups_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                                     int32_t head_dim, int32_t max_seq_len,
                                                     int32_t max_shared_blocks, int32_t num_groups,
                                                     int32_t block_size, int32_t partition_blocks) {
    if (max_shared_blocks == 0)
        return pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len,
                                        block_size, partition_blocks);
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_seq_len < 0 ||
        block_size != kBlockTokens || partition_blocks < -1 || max_shared_blocks < 0 || num_groups < 1 ||
        num_q_heads % num_kv_heads != 0 || static_cast<int64_t>(max_shared_blocks) * kBlockTokens > max_seq_len)
        return 0;
    const Plan plan = make_group_plan(max_seq_len, partition_blocks, max_shared_blocks, num_groups, num_seqs,
                                      num_q_heads, num_kv_heads);
    return ws_layout(num_seqs, num_q_heads, num_kv_heads, plan.max_parts, head_dim, plan.split, -1, true).bytes;
}

int pa_decode_multi(const void* q, const int32_t* q_start, int32_t num_q_rows, int32_t max_q_len,
                    const void* k_cache, const void* v_cache, const int32_t* block_tables,
                    int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t max_seq_len,
                    int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                    int32_t num_blocks, int32_t block_size, float scale, int32_t partition_blocks,
                    void* workspace, size_t workspace_bytes, void* out, int32_t dtype,
                    void* stream) {
    if (!q_start || !aligned(q_start, 4) || num_q_rows < 0 || max_q_len < 1) return PA_ERR_INVALID_ARG;
    if (dtype != PA_DTYPE_BF16) return PA_ERR_UNSUPPORTED;
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    DecodeArgs a = make_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                             max_seq_len, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                             block_size, scale, partition_blocks, workspace, workspace_bytes, out,
                             dtype, stream);
    a.q_start = q_start;
    a.max_q_len = max_q_len;
    a.num_q_rows = num_q_rows;
    // more rows per (sequence, kv head) than one warp-level MMA tile holds: the
    // tensor-memory tile kernel (prefill chunks)
    if (static_cast<int64_t>(num_q_heads / num_kv_heads) * max_q_len > 16) return run_prefill_tiles(a);
    DecodeParams P;
    Plan plan;
    int rc = prepare_decode(a, true, &P, &plan);
    if (rc != PA_OK) return rc;
    rc = run_partitions(P, dtype, a.stream);
    if (rc != PA_OK) return rc;
    return run_reduce(P, plan, dtype, a.stream);
}

size_t pa_decode_multi_workspace_size(int32_t num_seqs, int32_t num_q_rows, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t head_dim, int32_t max_seq_len,
                                      int32_t block_size, int32_t partition_blocks) {
    if (num_seqs < 0 || num_q_rows < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        max_seq_len < 0 || block_size != kBlockTokens || partition_blocks < -1)
        return 0;
    if (num_q_heads % num_kv_heads != 0) return 0;
    const Plan plan = make_plan(max_seq_len, partition_blocks);
    const size_t dec = ws_layout(num_seqs, num_q_heads, num_kv_heads, plan.max_parts, head_dim, plan.split,
                                 num_q_rows).bytes;
    // the tile path (group * max_q_len > 16) keeps its chunks' partials; its
    // chunking follows the device's SM count (the most chunks if unknown)
    DeviceInfo di;
    const int sms = device_info(&di) == PA_OK ? di.sms : (1 << 30);
    const size_t til = make_prefill_plan(sms, num_seqs, num_q_rows, num_q_heads, num_kv_heads, head_dim,
                                         max_seq_len).ws.bytes;
    return dec > til ? dec : til;
}

size_t pa_decode_shared_prefix_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                              int32_t num_kv_heads, int32_t head_dim,
                                              int32_t max_seq_len, int32_t shared_blocks,
                                              int32_t block_size, int32_t partition_blocks) {
    if (shared_blocks == 0)
        return pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len,
                                        block_size, partition_blocks);
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        max_seq_len < 0 || block_size != kBlockTokens || partition_blocks < -1 ||
        shared_blocks < 0 || num_q_heads % num_kv_heads != 0 ||
        static_cast<int64_t>(shared_blocks) * kBlockTokens > max_seq_len)
        return 0;
    const Plan plan = make_prefix_plan(max_seq_len, partition_blocks, shared_blocks, num_seqs,
                                       num_q_heads, num_kv_heads);
    return ws_layout(num_seqs, num_q_heads, num_kv_heads, plan.max_parts, head_dim, plan.split, -1, true).bytes;
}

int pa_get_device_error(uint32_t* bits, int32_t clear, void* stream) {
    if (!bits) return PA_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int v = 0;
    e = cudaMemcpyFromSymbol(&v, pa::g_error_bits, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol");
    if (clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(pa::g_error_bits, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol");
    }
    *bits = v;
    return PA_OK;
}

const char* pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "ok";
        case PA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad sizes)";
        case PA_ERR_UNSUPPORTED: return "unsupported dtype, head_dim, block size or group size";
        case PA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case PA_ERR_CUDA: return g_last_cuda_error;
        case PA_ERR_OUT_OF_BLOCKS: return "the block pool has too few free blocks";
        case PA_ERR_SCRATCH_LIMIT:
            return "sizes need more split-K scratch than pa_decode_noalloc's built-in 32 MiB buffer "
                   "(use larger partitions, or pa_decode with a caller-owned workspace)";
        default: return "unknown status";
    }
}

}  // extern "C"
