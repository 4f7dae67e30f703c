// cache_write.cuh -- scatter of newly computed K/V into the paged pool.
//
// Token t with slot s >= 0 lands in physical block s / 16 at offset s % 16 of
// every kv head: the inverse of the block-table lookup that maps logical
// positions to physical blocks ("Was ändert PagedAttention an der
// KV-Speicherzuweisung für LLMs?", slavadubrov.com, introduction; 16-token
// blocks: "Внутреннее устройство vLLM", artificials.ru).
//
// One thread moves one 16-byte chunk of K and the same chunk of V; a head row
// is head_dim * elem bytes (128..512 B), so a warp covers whole rows with
// fully coalesced 16-byte loads and stores.  Pure data movement: bytes are
// copied unchanged.
#pragma once

#include "common.cuh"

namespace pa {

__global__ void __launch_bounds__(256)
cache_write_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                   const int64_t* __restrict__ slot_mapping, int64_t total_chunks,
                   int32_t num_kv_heads, int32_t chunks_per_row, uint4* __restrict__ k_cache,
                   uint4* __restrict__ v_cache, int64_t num_slots) {
    allow_dependents();  // a dependent decode may become resident now
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= total_chunks) return;
    const int64_t row = i / chunks_per_row;  // (token, head)
    const int32_t c = static_cast<int32_t>(i - row * chunks_per_row);
    const int64_t t = row / num_kv_heads;
    const int32_t h = static_cast<int32_t>(row - t * num_kv_heads);
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;  // padding token
    if (slot >= num_slots) {
        if (h == 0 && c == 0) flag_error(PA_DEVERR_SLOT_OOB);
        return;
    }
    const int64_t blk = slot / kBlockTokens;
    const int64_t off = slot - blk * kBlockTokens;
    const int64_t dst = ((blk * num_kv_heads + h) * kBlockTokens + off) * chunks_per_row + c;
    const uint4 kv = __ldcs(k + i);
    const uint4 vv = __ldcs(v + i);
    k_cache[dst] = kv;
    v_cache[dst] = vv;
}

// Cache write into E4M3 caches: one thread quantises 16 consecutive elements
// of one (token, head) row: bf16 -> fp32, times the head's inverse scale (fp32
// multiply, round to nearest), then round to E4M3 (nearest even, saturating at
// 448, NaN to 0x7F); one 16-byte store per cache.
__global__ void __launch_bounds__(256)
cache_write_fp8_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                       const int64_t* __restrict__ slot_mapping, int64_t total_chunks,
                       int32_t num_kv_heads, int32_t chunks_per_row, uint4* __restrict__ k_cache,
                       uint4* __restrict__ v_cache, int64_t num_slots,
                       const float* __restrict__ k_inv_scale, const float* __restrict__ v_inv_scale) {
    allow_dependents();
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= total_chunks) return;
    const int64_t row = i / chunks_per_row;  // (token, head)
    const int32_t c = static_cast<int32_t>(i - row * chunks_per_row);
    const int64_t t = row / num_kv_heads;
    const int32_t h = static_cast<int32_t>(row - t * num_kv_heads);
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (h == 0 && c == 0) flag_error(PA_DEVERR_SLOT_OOB);
        return;
    }
    const int64_t blk = slot / kBlockTokens;
    const int64_t off = slot - blk * kBlockTokens;
    const int64_t dst = ((blk * num_kv_heads + h) * kBlockTokens + off) * chunks_per_row + c;
    const float kis = k_inv_scale[h], vis = v_inv_scale[h];
#pragma unroll
    for (int which = 0; which < 2; ++which) {
        const uint4* src = (which == 0 ? k : v) + 2 * i;  // 16 bf16 = two 16-byte loads
        const float inv = which == 0 ? kis : vis;
        const uint4 a = __ldcs(src), b = __ldcs(src + 1);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint16_t q[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
            q[j] = f32x2_to_e4m3x2(__fmul_rn(f.x, inv), __fmul_rn(f.y, inv));
        }
        uint4 o;
        o.x = e4m3x4_canonical_nan(q[0] | (static_cast<uint32_t>(q[1]) << 16));
        o.y = e4m3x4_canonical_nan(q[2] | (static_cast<uint32_t>(q[3]) << 16));
        o.z = e4m3x4_canonical_nan(q[4] | (static_cast<uint32_t>(q[5]) << 16));
        o.w = e4m3x4_canonical_nan(q[6] | (static_cast<uint32_t>(q[7]) << 16));
        (which == 0 ? k_cache : v_cache)[dst] = o;
    }
}

// Block copy for copy-on-write: grid-stride over (pair, 16-byte chunk) of a
// whole physical block (all kv heads, both pools); consecutive threads move
// consecutive chunks of one block, so both the reads and the writes are fully
// coalesced.
__global__ void __launch_bounds__(256)
copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                   const int32_t* __restrict__ src, const int32_t* __restrict__ dst,
                   int32_t num_pairs, int64_t chunks_per_block, int32_t num_blocks) {
    const int64_t total = static_cast<int64_t>(num_pairs) * chunks_per_block;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t pair = i / chunks_per_block;
        const int64_t c = i - pair * chunks_per_block;
        const int32_t s = src[pair], d = dst[pair];
        if (static_cast<uint32_t>(s) >= static_cast<uint32_t>(num_blocks) ||
            static_cast<uint32_t>(d) >= static_cast<uint32_t>(num_blocks)) {
            if (c == 0) flag_error(PA_DEVERR_BLOCK_OOB);
            continue;
        }
        const uint4 kv = k_cache[static_cast<int64_t>(s) * chunks_per_block + c];
        const uint4 vv = v_cache[static_cast<int64_t>(s) * chunks_per_block + c];
        k_cache[static_cast<int64_t>(d) * chunks_per_block + c] = kv;
        v_cache[static_cast<int64_t>(d) * chunks_per_block + c] = vv;
    }
}

}  // namespace pa
