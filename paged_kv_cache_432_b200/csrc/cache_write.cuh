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
