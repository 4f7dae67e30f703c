// common.cuh -- shared device helpers of the paged decode library (sm_100a).
//
// Inline-PTX wrappers for the async-copy machinery (mbarrier, TMA tile loads),
// the legacy warp-level tensor-core path (ldmatrix / mma.sync m16n8k16 bf16),
// bounded waits, and the parameter block every decode kernel receives.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "pagedattn.h"

namespace pa {

constexpr int kBlockTokens = 16;           // tokens per physical block
constexpr unsigned kFullMask = 0xffffffffu;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bounded waits give up after 1 s

// Sticky device error word (PA_DEVERR_* bits).  The library is one translation
// unit, so this header is compiled once and the word exists once per device.
__device__ unsigned int g_error_bits = 0u;

__device__ __forceinline__ void flag_error(unsigned bits) { atomicOr(&g_error_bits, bits); }

// Everything a decode launch needs; passed by value (kernel parameter space).
struct DecodeParams {
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    const float* k_scale;  // E4M3 caches: dequantisation scale per kv head (else null)
    const float* v_scale;
    void* out;
    float* ws_m;    // [num_seqs*num_q_heads][max_parts]        (null: no split)
    float* ws_l;    // [num_seqs*num_q_heads][max_parts]
    float* ws_acc;  // [num_seqs*num_q_heads][max_parts][head_dim]
    int32_t* ws_parts;  // [num_seqs*num_kv_heads] pieces of each unit (split only)
    int32_t* tile_counter;  // shared-prefix calls: the tile kernel's item counter (host use only)
    const int32_t* q_start;  // several query tokens per sequence: rows q_start[s] .. q_start[s+1]-1
                             // (null: one query token per sequence, row = sequence)
    int32_t max_q_len;       // bound on query tokens per sequence (1 without q_start)
    int32_t num_q_rows;      // query token rows (num_seqs without q_start)
    int32_t num_seqs;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t group;               // num_q_heads / num_kv_heads
    int32_t max_blocks_per_seq;  // table row width
    int32_t num_blocks;          // pool size in blocks
    int32_t part_blocks;         // fixed mode: blocks per partition (huge = never split)
    int32_t balanced;            // 1: balanced stream split, 0: fixed partitions
    int32_t min_chunk;           // balanced mode: fewest blocks a warp range holds
    int32_t max_parts;           // pieces per row the workspace holds
    int32_t len_cap;             // longest sequence handled; longer ones are clamped
    int32_t skip_blocks;         // pieces cover blocks [skip_blocks, nb) of each sequence
    int32_t piece_base;          // > 0: pieces are written as partials at index piece_base + p
                                 //      (the first piece_base partials come from elsewhere)
    const int32_t* group_start;  // several prompt groups: sequences of group i are
                                 //   group_start[i] .. group_start[i+1]-1 (null: one or no prefix)
    const int32_t* group_blocks; //   and group i shares its first group_blocks[i] blocks
    int32_t num_groups;
    int32_t max_shared;          //   bound on group_blocks
    int32_t group_chunk;         //   key blocks per prefix chunk of the tile kernel
    int32_t tile_tokens;         // merge of tile-kernel prefill rows: query tokens per tile
    int32_t tile_chunk;          //   and key blocks per chunk (0: not a tile-kernel merge)
    int32_t seq_begin;           // first sequence of this launch
    int32_t seq_count;           // sequences in this launch
    float scale;                 // softmax scale (natural units)
    float scale_log2;            // scale * log2(e)
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- dependent launch
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream is still
// running; grid_dependency_wait() blocks until that kernel has completed and
// its memory is visible (a no-op for a normal launch).  allow_dependents()
// lets the next kernel in the stream begin launching.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of an mbarrier with a wall-clock limit; every lane
// of the warp polls, and the result is made warp-uniform.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    bool ok = mbar_try_wait(bar, parity);
    if (!__all_sync(kFullMask, ok)) {
        const uint64_t t0 = globaltimer_ns();
        while (!ok) {
            for (int k = 0; k < 32 && !ok; ++k) ok = mbar_try_wait(bar, parity);
            if (!ok && globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
        ok = __all_sync(kFullMask, ok);
    }
    return ok;
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
// 2-D tile load global -> shared, completion counted on `bar` in bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

// 3-D tile load global -> shared (innermost coordinate first).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy)
        : "memory");
}

// Brings the 128-byte line holding p into L2 ahead of a dependent load.  p
// must lie inside an allocation the kernel may read.
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// L2 policy for data read once (the KV stream): evict first.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// L2 policy for data many CTAs read (a shared prefix): keep it.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------- tensor cores (warp level)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same with rows 8..15 of A and C known to be zero: only the two
// accumulators of rows 0..7 are kept (the other two outputs are discarded), so
// a query group of <= 8 heads holds half the accumulator registers.
__device__ __forceinline__ void mma_bf16_rows8(float (&d)[2], uint32_t a0, uint32_t a2, uint32_t b0,
                                               uint32_t b1) {
    float z2, z3;
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(z2), "=f"(z3)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d[0]), "f"(d[1]), "f"(0.f),
          "f"(0.f));
    (void)z2;
    (void)z3;
}

// Fragment-array forms: 4 registers = all 16 rows, 2 registers = rows 0..7.
__device__ __forceinline__ void mma_frag(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    mma_bf16(d, a[0], a[1], a[2], a[3], b0, b1);
}
__device__ __forceinline__ void mma_frag(float (&d)[2], const uint32_t (&a)[2], uint32_t b0,
                                         uint32_t b1) {
    mma_bf16_rows8(d, a[0], a[1], b0, b1);
}

// f16 inputs (the FP8 path widens E4M3 to f16, which is exact).
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_rows8(float (&d)[2], uint32_t a0, uint32_t a2, uint32_t b0,
                                              uint32_t b1) {
    float z2, z3;
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(z2), "=f"(z3)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d[0]), "f"(d[1]), "f"(0.f),
          "f"(0.f));
    (void)z2;
    (void)z3;
}

template <bool F16>
__device__ __forceinline__ void mma_frag_t(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                           uint32_t b1) {
    if constexpr (F16) mma_f16(d, a[0], a[1], a[2], a[3], b0, b1);
    else mma_bf16(d, a[0], a[1], a[2], a[3], b0, b1);
}
template <bool F16>
__device__ __forceinline__ void mma_frag_t(float (&d)[2], const uint32_t (&a)[2], uint32_t b0,
                                           uint32_t b1) {
    if constexpr (F16) mma_f16_rows8(d, a[0], a[1], b0, b1);
    else mma_bf16_rows8(d, a[0], a[1], b0, b1);
}

// Two fp32 values to a packed pair (lo in the low half) of bf16 or f16.
template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (F16) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    } else {
        __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&b);
    }
}
template <bool F16>
__device__ __forceinline__ float2 unpack2(uint32_t u) {
    if constexpr (F16) return __half22float2(*reinterpret_cast<__half2*>(&u));
    else return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
}

// Four E4M3 codes (bytes 0..3 of x) -> two f16 pairs: lo = (byte 0, byte 1),
// hi = (byte 2, byte 3), first value in the low half; exact.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(x));
}

// 2^x with the hardware approximation (relative error about 2^-22; -inf
// gives 0, results below 2^-126 flush to 0).  The softmax weights it feeds
// are rounded to 16-bit floats right after.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Byte i of the result is byte (sel >> 4i) & 7 of {x (bytes 0..3), x (4..7)}.
__device__ __forceinline__ uint32_t byte_perm(uint32_t x, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %1, %2;" : "=r"(r) : "r"(x), "r"(sel));
    return r;
}

// A bf16 pair -> an f16 pair (round to nearest; exact for magnitudes in
// 2^-14 .. 65504).  `bad` is set when a value lies outside the f16 range
// (magnitude above 65504, infinity or NaN).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_checked(uint32_t u, bool& bad) {
    const float2 f = unpack2<false>(u);
    bad |= !(fabsf(f.x) <= 65504.f && fabsf(f.y) <= 65504.f);
    return pack2<true>(f.x, f.y);
}

// Two fp32 values to an E4M3 pair (first value in the low byte), rounding to
// nearest even and saturating at +-448.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float first, float second) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(second), "f"(first));
    return r;
}

// Four packed E4M3 codes with every NaN (S.1111.111) made the one NaN code
// 0x7F, whatever its sign.
__device__ __forceinline__ uint32_t e4m3x4_canonical_nan(uint32_t w) {
    const uint32_t nan = __vcmpeq4(w & 0x7f7f7f7fu, 0x7f7f7f7fu);  // 0xff in each NaN byte
    return (w & ~nan) | (0x7f7f7f7fu & nan);
}

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) {
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFullMask, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFullMask, v, o));
    return v;
}

}  // namespace pa
