/*
 * pagedattn.h -- C ABI of the paged KV-cache decode path (NVIDIA B200, sm_100a).
 *
 * PagedAttention keeps each sequence's keys and values in fixed-size physical
 * blocks that may sit anywhere in one shared pool; a per-sequence block table
 * maps logical token positions to those blocks, blocks are taken as a sequence
 * grows, and several sequences may point at the same block (shared prefixes).
 * Sources: "Was ändert PagedAttention an der KV-Speicherzuweisung für LLMs?"
 * (slavadubrov.com), introduction, §"Ungenutzten Platz in Blöcken berechnen"
 * (16-token blocks, only the last block partly filled) and §"Gemeinsame Nutzung
 * erfordert mehr als Speicherzuweisung" (several requests reference one block;
 * copy-on-write); "PagedAttention et vLLM" (aiunderstanding.org), §"Plongée
 * profonde" (lookup table from logical positions to physical blocks);
 * "vLLM PagedAttention: eine Revolution für den Durchsatz bei der
 * LLM-Inferenz" (de.news.hada.io) (decoding is the memory-bandwidth-bound
 * phase); "Внутреннее устройство vLLM" (artificials.ru), paragraphs on the
 * KV-cache manager (16-token blocks) and on the padding-free super-batch
 * (per-sequence lengths instead of padding).
 *
 * Layouts (row-major, the pages leave layout to the runtime; this is the one
 * this library fixes):
 *   k_cache, v_cache  [num_blocks][num_kv_heads][block_size][head_dim]
 *   q, out            [num_seqs][num_q_heads][head_dim]
 *   k, v (new tokens) [num_tokens][num_kv_heads][head_dim]
 *   slot_mapping      int64  [num_tokens]; slot = block * block_size + offset
 *   block_tables      int32  [num_seqs][max_blocks_per_seq]
 *   seq_lens          int32  [num_seqs]   (tokens to attend, new token included)
 * Query head i reads kv head i / (num_q_heads / num_kv_heads).
 *
 * Ownership and execution: every pointer argument is device memory owned by
 * the caller (the library allocates no device memory and keeps no pointer).
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 * default stream) and return once the work is enqueued.
 *
 * Early start of the decode kernels: every decode entry point (pa_decode,
 * pa_decode_partitions, pa_decode_reduce, pa_decode_fp8 and its two steps,
 * pa_decode_multi, pa_decode_shared_prefix and its prompt-group form,
 * pa_decode_noalloc) launches its kernels with
 * programmatic stream serialization, so they may start before the previous
 * kernel in the stream has finished.  Before waiting for that kernel they
 * already read seq_lens, block_tables, q_start, the prefix groups and q (they never touch the
 * caches, out or the workspace before the wait).  This is safe whenever the
 * previous kernel in the stream did not trigger its dependents early (a kernel
 * that never executes griddepcontrol.launch_dependents /
 * cudaTriggerProgrammaticLaunchCompletion lets dependents start only when it
 * completes), and whenever those four arrays were written before such a
 * trigger.  A caller whose previous kernel writes them after an early trigger
 * must separate the two launches (an event, or any kernel without an early
 * trigger in between).  The library's own cache writes trigger early, but
 * they write only the caches, which the decode reads after the wait.  Host-side validation
 * never reads device memory.  Pointers to q, k, v, caches and out must be
 * 16-byte aligned; tables, lengths and slots naturally aligned.  The caches
 * and tables may be shared between sequences but must not overlap `out` or the
 * workspace.  The library never traps or aborts: bad device-side values (a
 * slot or block id outside the pool, an impossible length) are skipped and
 * recorded in a sticky per-device error word read by pa_get_device_error.
 */
#ifndef PAGEDATTN_H_
#define PAGEDATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define PA_OK 0
#define PA_ERR_INVALID_ARG (-1) /* null/misaligned pointer, bad sizes        */
#define PA_ERR_UNSUPPORTED (-2) /* dtype, head_dim, block size or group size */
#define PA_ERR_WORKSPACE (-3)   /* workspace missing or too small            */
#define PA_ERR_CUDA (-4)        /* a CUDA call or launch failed              */
#define PA_ERR_SCRATCH_LIMIT (-5) /* pa_decode_noalloc: sizes need more than its fixed buffer */
#define PA_ERR_OUT_OF_BLOCKS (-6) /* block manager: the pool has too few free blocks     */

/* Element types (q, caches, new k/v and out share one). */
#define PA_DTYPE_F32 0
#define PA_DTYPE_BF16 1

/* Bits of the sticky device error word. */
#define PA_DEVERR_SLOT_OOB 1u  /* cache write: slot >= num_blocks*block_size, token skipped */
#define PA_DEVERR_BLOCK_OOB 2u /* decode: table entry outside [0, num_blocks), block masked */
#define PA_DEVERR_SEQ_LEN 4u   /* decode: seq_len < 0 or beyond capacity, clamped          */
#define PA_DEVERR_TIMEOUT 8u   /* a bounded wait on an async copy gave up                  */
#define PA_DEVERR_PREFIX 16u   /* shared-prefix decode: a table does not start with the
                                  shared blocks, or a sequence is shorter than them      */
#define PA_DEVERR_Q_RANGE 32u  /* E4M3 decode: a query value outside the f16 range the
                                  kernel rounds q to (|q| > 65504, inf, NaN); the rows
                                  of that (sequence, kv head) are not meaningful        */

/*
 * Cache write (the scatter of newly computed K/V into the paged pool).
 * For every token t with slot s = slot_mapping[t] >= 0 and every kv head h:
 *   k_cache[s / block_size][h][s % block_size][:] = k[t][h][:]   (same for v)
 * Bytes are copied unchanged.  Slots < 0 are padding and write nothing; a slot
 * beyond the pool writes nothing and sets PA_DEVERR_SLOT_OOB.  Two tokens with
 * the same slot race (one of them wins).  block_size must be 16; head_dim 64
 * or 128.  Source: slavadubrov.com, introduction (logical positions mapped to
 * physical blocks); artificials.ru (16-token blocks).
 */
PA_API int pa_cache_write(const void* k, const void* v, const int64_t* slot_mapping,
                   int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                   void* k_cache, void* v_cache, int32_t num_blocks,
                   int32_t block_size, int32_t dtype, void* stream);

/*
 * FP8 KV cache, quantising cache write.  The caches hold one byte per element,
 * an FP8 E4M3 code (sign, 4 exponent bits of bias 7, 3 mantissa bits; largest
 * finite 448; S.1111.111 is NaN), with one scale per kv head and pool, so a
 * token costs half the bytes of a bf16 cache (cache quantisation as a remedy
 * when the KV data do not fit: "Was ändert PagedAttention an der
 * KV-Speicherzuweisung für LLMs?", slavadubrov.com, §"Gemeinsame Nutzung
 * erfordert mehr als Speicherzuweisung", last paragraph).  Layout as for
 * pa_cache_write with uint8 elements: k_cache[num_blocks][num_kv_heads][16][head_dim].
 * For every token t with slot s = slot_mapping[t] >= 0, kv head h and d:
 *   k_cache[s / 16][h][s % 16][d] = E4M3(float(k[t][h][d]) * k_inv_scale[h])
 * (same for v), where the product is one fp32 multiply rounded to nearest and
 * E4M3() rounds to the nearest code, ties to even, saturates magnitudes above
 * 448 to +-448 (infinities too) and gives 0x7F for NaN.  k and v are bf16
 * [num_tokens][num_kv_heads][head_dim]; k_inv_scale and v_inv_scale are fp32
 * device arrays [num_kv_heads] (the inverses of the scales pa_decode_fp8 takes).
 * Slots: as pa_cache_write (< 0 skipped, beyond the pool skipped with
 * PA_DEVERR_SLOT_OOB).  block_size 16; head_dim 64 or 128.  Pointers 16-byte
 * aligned (scales 4-byte).  Errors: PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED as
 * pa_cache_write; nothing is launched then.
 */
PA_API int pa_cache_write_fp8(const void* k, const void* v, const int64_t* slot_mapping,
                              int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                              void* k_cache, void* v_cache, int32_t num_blocks,
                              int32_t block_size, const float* k_inv_scale,
                              const float* v_inv_scale, void* stream);

/*
 * Paged decode attention over FP8 E4M3 caches (written by pa_cache_write_fp8):
 * as pa_decode with dtype BF16 (q and out bf16), where
 *   K_s[t] = decode(k_cache[block_tables[s][t / 16]][h][t % 16]) * k_scale[h]
 * (same for V with v_scale), decode() being the exact value of the code.
 * The kernel widens the codes to f16 (exact), computes q . code and P . code
 * on tensor cores (f16 in, fp32 accumulate; q rounded to f16, exact for bf16
 * values of magnitude 2^-14 .. 65504), and applies the scales in fp32.
 * k_scale and v_scale are fp32 device arrays [num_kv_heads].  Workspace: the
 * size pa_decode_workspace_size gives for the same arguments.  Same errors
 * and device error bits as pa_decode; null scales give PA_ERR_INVALID_ARG.
 */
PA_API int pa_decode_fp8(const void* q, const void* k_cache, const void* v_cache,
                         const float* k_scale, const float* v_scale,
                         const int32_t* block_tables, int32_t max_blocks_per_seq,
                         const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                         int32_t num_blocks, int32_t block_size, float scale,
                         int32_t partition_blocks, void* workspace, size_t workspace_bytes,
                         void* out, void* stream);

/*
 * The two steps of pa_decode_fp8 as separate calls (as pa_decode_partitions
 * and pa_decode_reduce are for pa_decode), so that each kernel can be timed
 * on its own; issued back to back on one stream they give pa_decode_fp8's
 * result bit for bit.  pa_decode_fp8_partitions takes pa_decode_fp8's
 * arguments and writes out[] for the single-piece (sequence, kv head) units
 * and the workspace partials for the others.  pa_decode_fp8_reduce takes
 * pa_decode_reduce's arguments (out is bf16) and merges the partials of an
 * E4M3 partition step (the warp ranges of the balanced split depend on the
 * kernel form, so the bf16 reduce must not be used on them).
 * Interface plumbing: no passage (the pages define no API); the arithmetic
 * is pa_decode_fp8's and pa_decode_reduce's.  Errors as for those calls.
 */
PA_API int pa_decode_fp8_partitions(const void* q, const void* k_cache, const void* v_cache,
                                    const float* k_scale, const float* v_scale,
                                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                                    const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t num_blocks, int32_t block_size, float scale,
                                    int32_t partition_blocks, void* workspace, size_t workspace_bytes,
                                    void* out, void* stream);
PA_API int pa_decode_fp8_reduce(const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                                int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_blocks_per_seq, int32_t block_size,
                                int32_t partition_blocks, const void* workspace,
                                size_t workspace_bytes, void* out, void* stream);

/*
 * Several new query tokens per sequence: the check step of speculative
 * decoding, or a short prefill chunk ("vLLM PagedAttention: eine Revolution
 * für den Durchsatz bei der LLM-Inferenz", de.news.hada.io, list of advanced
 * features; "Внутреннее устройство vLLM", artificials.ru, paragraphs on
 * chunked prefill and on speculative decoding).  The rows are packed without
 * padding, as in the engine's super-batch (same page, super-batch paragraph):
 * the query tokens of sequence s are rows q_start[s] .. q_start[s+1]-1
 * (int32 [num_seqs+1], q_start[num_seqs] = num_q_rows) of q and out, both
 * [num_q_rows][num_q_heads][head_dim].  They are the sequence's last n
 * positions (their K/V already in the cache), so token k attends to keys
 * 0 .. seq_lens[s] - n + k (causal among the new tokens).  Needs PA_DTYPE_BF16.
 * With group * max_q_len <= 16 the (token, head) rows of a (sequence, kv head)
 * fit one warp-level MMA tile and run in the decode kernel (the check of a few
 * drafted tokens); with more (prefill chunks of any length), tiles of up to
 * 256 rows (two halves of floor(128 / group) tokens x group heads) of one
 * sequence run on the tensor-memory kernel, reading each K/V block once per
 * tile, with the
 * keys cut into at most 16 chunks (merged by a log-sum-exp reduction) when
 * there are too few tiles to fill the device, or when the sequences are long
 * enough (chunks of at least 256 blocks) that more, shorter items even out
 * the SMs' work.  A sequence with more than
 * max_q_len or more than seq_lens[s] query tokens has the excess ignored (its
 * rows are not written) and PA_DEVERR_SEQ_LEN set.  Workspace from
 * pa_decode_multi_workspace_size (rows are query-token rows); other arguments
 * as for pa_decode.  With one query token per sequence this is pa_decode.
 */
PA_API int pa_decode_multi(const void* q, const int32_t* q_start, int32_t num_q_rows,
                           int32_t max_q_len, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                           int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                           int32_t num_blocks, int32_t block_size, float scale,
                           int32_t partition_blocks, void* workspace, size_t workspace_bytes,
                           void* out, int32_t dtype, void* stream);

/* Workspace bytes pa_decode_multi needs: the pa_decode layout with
 * num_q_rows * num_q_heads rows and as many pieces per row as either path can
 * write (the tile path's key chunks depend on the current device's SM count:
 * query the size on the device that runs the call), and for the tile path 256
 * bytes at the end for its work counter (zeroed by every call), so the size is
 * never 0. */
PA_API size_t pa_decode_multi_workspace_size(int32_t num_seqs, int32_t num_q_rows,
                                             int32_t num_q_heads, int32_t num_kv_heads,
                                             int32_t head_dim, int32_t max_seq_len,
                                             int32_t block_size, int32_t partition_blocks);

/*
 * Block copy, the device half of copy-on-write: for every i, physical block
 * dst[i] of both pools becomes a byte copy of block src[i] (all kv heads).
 * A shared, partly filled block is copied before one of its sequences writes
 * into it ("Was ändert PagedAttention an der KV-Speicherzuweisung für LLMs?",
 * slavadubrov.com, §"Gemeinsame Nutzung erfordert mehr als
 * Speicherzuweisung"; "PagedAttention et vLLM", aiunderstanding.org,
 * §"Questions fréquemment posées").  src/dst are device int32 arrays; no dst
 * may appear as another pair's src or dst in the same call (the block manager
 * below only produces fresh destinations).  Ids outside the pool skip the pair
 * and set PA_DEVERR_BLOCK_OOB.
 */
PA_API int pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* src, const int32_t* dst,
                          int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim,
                          int32_t num_blocks, int32_t block_size, int32_t dtype, void* stream);

/*
 * How the decode splits sequences, from partition_blocks:
 *   0   (auto) balanced split.  All (sequence, kv head) units form one stream
 *       of blocks and every warp of the persistent grid takes an equal share
 *       (at least 16 blocks), so long and short sequences mix without load
 *       imbalance.  A unit that spans several shares becomes several pieces.
 *   > 0 fixed partitions of that many blocks.
 *   -1  never split: one pass over each whole sequence.
 * Returns 0 for the balanced split, the partition size otherwise (a value >=
 * the blocks of max_seq_len means no split), or a negative status on bad
 * arguments.
 */
PA_API int32_t pa_decode_partition_blocks(int32_t num_seqs, int32_t num_kv_heads,
                                          int32_t max_seq_len, int32_t block_size,
                                          int32_t partition_blocks);

/*
 * Bytes of workspace pa_decode needs for these sizes (0 when no sequence of up
 * to max_seq_len tokens can be split).  Interface plumbing: the pages describe
 * no workspace (the split-K partials are this library's design).  It takes
 * num_kv_heads because the workspace ends with one piece count per
 * (sequence, kv head).  Workspace layout: P is the number of
 * pieces a unit can have at max_seq_len (fixed: ceil(nb / partition_blocks);
 * balanced: ceil(nb / 16) + 1, with nb = ceil(max_seq_len / 16)), and rows
 * r = seq * num_q_heads + q_head:
 *   float   m    [num_seqs*num_q_heads][P]    max score of the piece (natural log units)
 *   float   l    [num_seqs*num_q_heads][P]    sum of exp(score - m)
 *   float   acc  [num_seqs*num_q_heads][P][D] sum of exp(score - m) * v
 *   int32_t parts[num_seqs*num_kv_heads]      pieces of each (sequence, kv head)
 * each array starting on a 256-byte boundary.  Its contents need no
 * initialisation: every value read is written first in the same call.
 */
PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                       int32_t num_kv_heads, int32_t head_dim,
                                       int32_t max_seq_len, int32_t block_size,
                                       int32_t partition_blocks);

/*
 * Paged decode attention: for each sequence s and query head i,
 *   out[s][i] = softmax_t(scale * q[s][i] . K_s[t]) V_s,  t < seq_lens[s],
 * where K_s[t] = k_cache[block_tables[s][t / bs]][i / group][t % bs] (same for V).
 * Accumulation is fp32 (bf16 inputs: scores and P.V on tensor cores with fp32
 * accumulators); out is rounded to the input dtype (round to nearest even).  A
 * zero-length sequence gives a zero row.  Sequences are cut into pieces as
 * partition_blocks says (pa_decode_partition_blocks) and the partial results of
 * a split sequence are merged by a log-sum-exp reduction (pa_decode runs both
 * steps).
 * max_seq_len is a host-side bound on seq_lens (<= 0: max_blocks_per_seq *
 * block_size); it sizes the workspace, and longer sequences are clamped to it
 * with PA_DEVERR_SEQ_LEN set.  Table entries past a sequence's last block are
 * never read.  Supported: block_size 16, head_dim 64 or 128, dtype F32 or
 * BF16, num_q_heads / num_kv_heads <= 16.
 * Source: slavadubrov.com, introduction and §"Ungenutzten Platz in Blöcken
 * berechnen"; aiunderstanding.org, §"Plongée profonde"; artificials.ru,
 * paragraph on the padding-free super-batch.
 */
PA_API int pa_decode(const void* q, const void* k_cache, const void* v_cache,
              const int32_t* block_tables, int32_t max_blocks_per_seq,
              const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
              int32_t num_blocks, int32_t block_size, float scale,
              int32_t partition_blocks, void* workspace, size_t workspace_bytes,
              void* out, int32_t dtype, void* stream);

/*
 * First step of pa_decode alone: walks the block tables and writes out[] for
 * every (sequence, kv head) that is one piece, and the workspace partials
 * (layout above) for every piece of the others.  Same arguments as pa_decode.
 */
PA_API int pa_decode_partitions(const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, int32_t max_blocks_per_seq,
                         const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                         int32_t num_blocks, int32_t block_size, float scale,
                         int32_t partition_blocks, void* workspace, size_t workspace_bytes,
                         void* out, int32_t dtype, void* stream);

/*
 * Second step of pa_decode alone: for every (sequence, kv head) with more than
 * one piece (the count recorded in the workspace), merges the partials of its
 * query heads,
 *   M = max_p m_p,  out = sum_p e^(m_p - M) acc_p / sum_p e^(m_p - M) l_p,
 * and writes out[] in `dtype`.  Rows of single-piece units are left untouched.
 * The sizes must be those given to pa_decode_partitions.
 */
PA_API int pa_decode_reduce(const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                     int32_t max_blocks_per_seq, int32_t block_size,
                     int32_t partition_blocks, const void* workspace,
                     size_t workspace_bytes, void* out, int32_t dtype, void* stream);

/*
 * Decode for a batch whose sequences all start with the same prompt, stored
 * once: the first `shared_blocks` entries of every block table are the same
 * physical blocks (prefix caching: "Was ändert PagedAttention an der
 * KV-Speicherzuweisung für LLMs?", slavadubrov.com, §"Gemeinsame Nutzung
 * erfordert mehr als Speicherzuweisung"; "PagedAttention et vLLM",
 * aiunderstanding.org, §"Questions fréquemment posées").  Same result as
 * pa_decode, computed in three launches: each sequence's own blocks go
 * through the decode kernel; then the query rows of all sequences attend to
 * the shared blocks together, so those blocks are read once per tile of up
 * to 256 query rows of a kv head rather than once per sequence
 * (5th-generation tensor cores, accumulators in tensor memory; this launch
 * starts on the SMs the decode leaves, without waiting for the decode, and
 * completes after it); a log-sum-exp reduction merges the two.  Preconditions: every table starts with the
 * prefix blocks of table 0, and every seq_len >= shared_blocks * block_size.
 * A violation is flagged with PA_DEVERR_PREFIX (the result is then
 * meaningless for the offending sequences).  Only PA_DTYPE_BF16.  The
 * workspace is sized by pa_decode_shared_prefix_workspace_size; the other
 * arguments are those of pa_decode.  shared_blocks = 0 is plain pa_decode.
 */
PA_API int pa_decode_shared_prefix(const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* block_tables, int32_t max_blocks_per_seq,
                                   const int32_t* seq_lens, int32_t max_seq_len,
                                   int32_t shared_blocks, int32_t num_seqs, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                                   int32_t block_size, float scale, int32_t partition_blocks,
                                   void* workspace, size_t workspace_bytes, void* out,
                                   int32_t dtype, void* stream);

/*
 * Workspace bytes pa_decode_shared_prefix needs.  Layout as for pa_decode, with
 * P = min(16, shared_blocks) slots for the prefix's key chunks + the pieces the
 * private part of a sequence can have; pieces 0 .. chunks-1 of every row hold
 * the shared prefix's partials (the chunk count, at most 16, is chosen at
 * launch to fill the device) and the private pieces follow.  256 more bytes at
 * the end hold the tile kernel's work counter, which every call sets to zero
 * on its stream before the kernel runs.
 */
PA_API size_t pa_decode_shared_prefix_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                                     int32_t num_kv_heads, int32_t head_dim,
                                                     int32_t max_seq_len, int32_t shared_blocks,
                                                     int32_t block_size,
                                                     int32_t partition_blocks);

/*
 * Decode for a batch that holds several prompt groups, each stored once: the
 * sequences of group i are seq group_start[i] .. group_start[i+1]-1 (groups
 * are consecutive ranges of the batch, group_start[0] = 0 and
 * group_start[num_groups] = num_seqs), and the first group_shared_blocks[i]
 * entries of every table of group i are the same physical blocks (those of
 * the group's first sequence).  This is the general form of
 * pa_decode_shared_prefix: several system prompts in one batch, or branches
 * of a request (parallel samples, beams) that share its prompt, each group
 * with its own prefix length; a group with 0 shared blocks is decoded as by
 * pa_decode ("Was ändert PagedAttention an der KV-Speicherzuweisung für
 * LLMs?", slavadubrov.com, §"Gemeinsame Nutzung erfordert mehr als
 * Speicherzuweisung": parallel sampling and beam search share blocks;
 * "PagedAttention et vLLM", aiunderstanding.org, §"Mise en œuvre dans le monde
 * réel" and §"Questions fréquemment posées": many requests with a common
 * system prompt).  Each group's shared blocks are read once per tile of up to
 * 256 query rows of its sequences (tensor-memory kernel); each sequence's own
 * blocks go through the decode kernel; a log-sum-exp reduction merges both.
 * group_start (int32 [num_groups + 1]) and group_shared_blocks (int32
 * [num_groups]) are device arrays read like the block tables;
 * max_shared_blocks is a host bound on group_shared_blocks that sizes the
 * workspace (pa_decode_shared_prefix_groups_workspace_size).  Device checks
 * (PA_DEVERR_PREFIX, the rows of an offending group are then meaningless): the
 * groups are ordered ranges of the batch, no count exceeds max_shared_blocks,
 * every table of a group starts with its shared blocks and no sequence of a
 * group is shorter than them.  Only PA_DTYPE_BF16 (max_shared_blocks = 0:
 * plain pa_decode, any dtype).  Other arguments and errors as pa_decode.
 */
PA_API int pa_decode_shared_prefix_groups(const void* q, const void* k_cache, const void* v_cache,
                                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                                          const int32_t* seq_lens, int32_t max_seq_len,
                                          const int32_t* group_start, const int32_t* group_shared_blocks,
                                          int32_t num_groups, int32_t max_shared_blocks, int32_t num_seqs,
                                          int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                          int32_t num_blocks, int32_t block_size, float scale,
                                          int32_t partition_blocks, void* workspace, size_t workspace_bytes,
                                          void* out, int32_t dtype, void* stream);

/*
 * Workspace bytes pa_decode_shared_prefix_groups needs: the pa_decode layout
 * with P = min(16, max_shared_blocks) slots for the prefix chunks + the pieces
 * a whole sequence of max_seq_len tokens can have (a group may share nothing),
 * and 256 bytes at the end for the tile kernel's work counter (zeroed by every
 * call).
 */
PA_API size_t pa_decode_shared_prefix_groups_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                                            int32_t num_kv_heads, int32_t head_dim,
                                                            int32_t max_seq_len, int32_t max_shared_blocks,
                                                            int32_t num_groups, int32_t block_size,
                                                            int32_t partition_blocks);

/*
 * Host-side block manager: the bookkeeping that hands out physical blocks.
 * A sequence holds ceil(len / block_size) blocks, taken first-in first-out
 * from a free list (initially in ascending id order) as it grows and returned
 * when it is freed ("Was ändert PagedAttention an der KV-Speicherzuweisung
 * für LLMs?", slavadubrov.com, §"Ungenutzten Platz in Blöcken berechnen").
 * Forking shares every block of the parent (reference counts); appending to a
 * sequence whose last block is shared and partly filled first replaces that
 * block with a fresh copy, and reports the (src, dst) pair for pa_copy_blocks
 * (copy-on-write).  Full shared blocks are never written and stay shared.
 * Pure host code: no CUDA call, no device memory; thread-safe.
 */
typedef struct pa_block_manager pa_block_manager;

/* NULL on bad sizes or allocation failure. */
PA_API pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size,
                                      int32_t max_blocks_per_seq);
PA_API void pa_bm_destroy(pa_block_manager* m);
/* A new empty sequence; PA_ERR_INVALID_ARG if the id is in use. */
PA_API int pa_bm_add_sequence(pa_block_manager* m, int32_t seq);
/* `child` starts as a copy of `parent`, sharing all of its blocks. */
PA_API int pa_bm_fork(pa_block_manager* m, int32_t parent, int32_t child);
/*
 * Reserves num_tokens slots at the end of `seq` and writes them (block *
 * block_size + offset, the input of pa_cache_write) to slots_out.  If the last
 * block had to be copied first, its (src, dst) pair goes to copy_src[0] /
 * copy_dst[0] and *num_copies = 1 (else 0); run pa_copy_blocks on it before
 * writing the new tokens.  PA_ERR_OUT_OF_BLOCKS (nothing changed) when the
 * free list is too short; PA_ERR_INVALID_ARG when the sequence would exceed
 * max_blocks_per_seq.
 */
PA_API int pa_bm_append(pa_block_manager* m, int32_t seq, int32_t num_tokens, int64_t* slots_out,
                        int32_t* copy_src, int32_t* copy_dst, int32_t* num_copies);
/* Releases the sequence's blocks (those no other sequence holds go back to the free list). */
PA_API int pa_bm_free_sequence(pa_block_manager* m, int32_t seq);
PA_API int32_t pa_bm_num_free(pa_block_manager* m);
PA_API int32_t pa_bm_refcount(pa_block_manager* m, int32_t block);
/*
 * Block tables ([num_seqs][width], unused entries -1) and lengths of the given
 * sequences, ready to upload for pa_decode.
 */
PA_API int pa_bm_export_tables(pa_block_manager* m, const int32_t* seq_ids, int32_t num_seqs,
                               int32_t* tables_out, int32_t width, int32_t* lens_out);

/*
 * Reads the sticky device error word of the current device (PA_DEVERR_* bits)
 * after synchronising `stream`; clears it when `clear` is non-zero (so that a
 * caller can check one call at a time).  Interface plumbing: the pages have no
 * passage on error reporting.  Returns PA_ERR_INVALID_ARG for a null `bits`,
 * PA_ERR_CUDA if the synchronisation or the read fails.
 */
PA_API int pa_get_device_error(uint32_t* bits, int32_t clear, void* stream);

/*
 * pa_decode without any device allocation, for callers that cannot allocate
 * device memory themselves.  Examples: a plugin inside an inference engine
 * that owns every byte of device memory through its own pool and forbids
 * cudaMalloc, a runtime whose memory budget is fixed at start-up, or a
 * foreign-language caller with no binding for CUDA allocation.  The pages
 * have no counterpart: this is an interface convenience, not part of the
 * method.
 *
 * Same arguments and result as pa_decode, minus the workspace.  The split-K
 * partials live in a buffer of PA_NOALLOC_SCRATCH_BYTES (32 MiB) built into
 * the library as a static device array.  Every GPU that loads the library
 * holds that buffer until the process exits.  If the sizes need more than
 * that (pa_decode_workspace_size > PA_NOALLOC_SCRATCH_BYTES) the call returns
 * PA_ERR_SCRATCH_LIMIT and does nothing.  Use larger partitions or pa_decode
 * with your own workspace instead.
 *
 * The first call on a device looks up the buffer's device address (a
 * one-time set-up per device, done with that device current) and keeps it for
 * the life of the process.  Make that first call before any stream capture.
 * Call it with the device's primary context current (the CUDA runtime's
 * default); after cudaDeviceReset, or from another context on the same device,
 * the kept address is no longer valid, so neither is supported.  All calls share the one buffer and
 * it keeps the last call's contents.  Nothing in it needs to start at zero,
 * since each partial is written before it is read.  Calls that overlap on the
 * GPU race on that buffer (two streams, or two threads), so serialise them.
 * Calls no cudaMalloc, cudaFree or other allocating routine.
 */
PA_API int pa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, int32_t max_blocks_per_seq,
                             const int32_t* seq_lens, int32_t max_seq_len, int32_t num_seqs,
                             int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                             int32_t num_blocks, int32_t block_size, float scale,
                             int32_t partition_blocks, void* out, int32_t dtype, void* stream);

#define PA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* Human-readable text for a return code (for PA_ERR_CUDA: the last CUDA error
 * seen by the calling thread).  Interface plumbing: no passage of the pages.
 * The string is static (or thread-local for PA_ERR_CUDA); do not free it. */
PA_API const char* pa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H_ */
