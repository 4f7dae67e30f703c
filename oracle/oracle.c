/*
 * oracle.c -- plain, slow, single-threaded fp64 CPU oracle for the paged
 * KV-cache decode path.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg may load or call this code.  It
 * shares no source, header, table or helper with the CUDA library, and the
 * library never calls it.
 *
 * What it follows:
 *   - Block tables: "Was ändert PagedAttention an der KV-Speicherzuweisung für
 *     LLMs?" (slavadubrov.com), introduction: a block table maps a request's
 *     logical token positions to fixed-size physical blocks; §"Ungenutzten
 *     Platz in Blöcken berechnen": 16-token blocks, only the last block of a
 *     sequence is partly filled.  "PagedAttention et vLLM"
 *     (aiunderstanding.org), §"Plongée profonde": a lookup table maps logical
 *     token positions to physical blocks that may live anywhere.
 *   - Attention: the pages do not print the formula; the method computes
 *     ordinary attention softmax(scale * q K^T) V over the sequence's tokens,
 *     so the oracle is that definition, written out after gathering K/V into
 *     contiguous fp64 arrays.
 *
 * Conventions (the pages leave layout open -- slavadubrov.com,
 * §"Ungenutzten Platz in Blöcken berechnen": block size and layouts depend on
 * the runtime -- so this is the reading taken):
 *   cache       [num_blocks][num_kv_heads][block_size][head_dim]
 *   q, out      [num_seqs][num_q_heads][head_dim]
 *   new k / v   [num_tokens][num_kv_heads][head_dim]
 *   tables      int32 [num_seqs][max_blocks]
 *   query head i reads kv head i / (num_q_heads / num_kv_heads).
 *   dtype 0 = float32, 1 = bfloat16 (raw bits; bf16 -> fp64 is exact).
 *
 * Parity pins live in the test suite (worked 35-token example, brute-force
 * contiguous attention, library SDPA in fp64, permutation invariance, shared
 * prefix vs private copies, closed forms).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_E4M3 = 2 };

/* bf16 is the top half of an IEEE float32: widen the bits, exact. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double oracle_e4m3_decode(uint8_t c);

static double load_elem(const void* base, size_t idx, int dtype) {
    if (dtype == ORACLE_F32) return (double)((const float*)base)[idx];
    if (dtype == ORACLE_E4M3) return oracle_e4m3_decode(((const uint8_t*)base)[idx]);
    return bf16_bits_to_double(((const uint16_t*)base)[idx]);
}

static size_t elem_size(int dtype) { return dtype == ORACLE_F32 ? 4u : 2u; }

/*
 * FP8 E4M3 (the 8-bit format with 4 exponent bits of bias 7 and 3 mantissa
 * bits; no infinities; S.1111.111 is NaN; largest finite 1.75 * 2^8 = 448;
 * smallest normal 2^-6; subnormals m * 2^-9).  Written from that definition.
 */
double oracle_e4m3_decode(uint8_t c) {
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round to the nearest E4M3 value, ties to even; magnitudes above 448
 * saturate to 448; NaN gives 0x7F. */
uint8_t oracle_e4m3_encode(float y) {
    if (isnan(y)) return 0x7F;
    const uint8_t sign = signbit(y) ? 0x80 : 0x00;
    const double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);   /* a = f * 2^e with f in [0.5, 1): floor(log2 a) = e - 1 */
    int ex = e - 1;
    if (ex < -6) ex = -6; /* subnormal range shares the quantum of the lowest binade */
    const double quantum = ldexp(1.0, ex - 3);
    const double n = rint(a / quantum); /* exact division; rint rounds half to even */
    const double m = n * quantum;
    if (m == 0.0) return sign;
    if (m < ldexp(1.0, -6)) return sign | (uint8_t)(m / ldexp(1.0, -9));
    int e2;
    frexp(m, &e2);
    const int ex2 = e2 - 1;
    const int mant = (int)((m / ldexp(1.0, ex2) - 1.0) * 8.0);
    return sign | (uint8_t)(((ex2 + 7) << 3) | mant);
}

/*
 * Cache write into an FP8 E4M3 cache: every element of the new k / v (bf16)
 * is multiplied in fp32 by its kv head's inverse scale and rounded to E4M3
 * (oracle_e4m3_encode).  Slots as for oracle_cache_write.
 */
int64_t oracle_cache_write_fp8(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping,
                               int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                               uint8_t* k_cache, uint8_t* v_cache, int64_t num_blocks,
                               int32_t block_size, const float* k_inv_scale,
                               const float* v_inv_scale) {
    int64_t bad = 0;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_blocks * (int64_t)block_size) { ++bad; continue; }
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            size_t src = ((size_t)t * num_kv_heads + h) * head_dim;
            size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + off) * head_dim;
            for (int32_t d = 0; d < head_dim; ++d) {
                const float xk = (float)bf16_bits_to_double(k[src + d]);
                const float xv = (float)bf16_bits_to_double(v[src + d]);
                const float yk = xk * k_inv_scale[h];
                const float yv = xv * v_inv_scale[h];
                k_cache[dst + d] = oracle_e4m3_encode(yk);
                v_cache[dst + d] = oracle_e4m3_encode(yv);
            }
        }
    }
    return bad;
}

/*
 * Cache write: each new token t with slot s = slot_mapping[t] >= 0 lands in
 * physical block s / block_size at offset s % block_size, for every kv head.
 * Bytes are copied unchanged.  Slots < 0 are padding and write nothing.
 * Returns the number of tokens skipped because their slot lies outside the
 * pool (those write nothing).
 */
int64_t oracle_cache_write(const void* k, const void* v, const int64_t* slot_mapping,
                           int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                           int32_t dtype, void* k_cache, void* v_cache,
                           int64_t num_blocks, int32_t block_size) {
    const size_t es = elem_size(dtype);
    const size_t row = (size_t)head_dim * es;
    int64_t bad = 0;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_blocks * (int64_t)block_size) { ++bad; continue; }
        int64_t blk = slot / block_size;
        int64_t off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            size_t src = ((size_t)t * num_kv_heads + h) * row;
            size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + off) * row;
            memcpy((char*)k_cache + dst, (const char*)k + src, row);
            memcpy((char*)v_cache + dst, (const char*)v + src, row);
        }
    }
    return bad;
}

/*
 * Block copy (copy-on-write of a shared block): for every pair i, block
 * dst[i] of both pools becomes a byte copy of block src[i] (all kv heads).
 * Pairs with an id outside the pool are skipped and counted.
 */
int64_t oracle_copy_blocks(void* k_cache, void* v_cache, const int32_t* src, const int32_t* dst,
                           int64_t num_pairs, int64_t num_blocks, int64_t block_bytes) {
    int64_t bad = 0;
    for (int64_t i = 0; i < num_pairs; ++i) {
        if (src[i] < 0 || src[i] >= num_blocks || dst[i] < 0 || dst[i] >= num_blocks) { ++bad; continue; }
        memmove((char*)k_cache + (size_t)dst[i] * block_bytes, (const char*)k_cache + (size_t)src[i] * block_bytes,
                (size_t)block_bytes);
        memmove((char*)v_cache + (size_t)dst[i] * block_bytes, (const char*)v_cache + (size_t)src[i] * block_bytes,
                (size_t)block_bytes);
    }
    return bad;
}

/*
 * Gather the first `len` tokens of kv head h of sequence s through its block
 * table into contiguous [len][D] fp64 arrays.  Logical position p sits in
 * physical block table[p / block_size] at offset p % block_size.
 * Returns -1 if a table entry lies outside [0, num_blocks).
 */
static int gather_sequence(const void* k_cache, const void* v_cache, const int32_t* table,
                           int32_t len, int32_t h, int32_t num_kv_heads, int32_t head_dim,
                           int32_t block_size, int64_t num_blocks, int dtype,
                           double* K, double* V) {
    for (int32_t p = 0; p < len; ++p) {
        int32_t blk = table[p / block_size];
        int32_t off = p % block_size;
        if (blk < 0 || blk >= num_blocks) return -1;
        size_t base = (((size_t)blk * num_kv_heads + h) * block_size + off) * (size_t)head_dim;
        for (int32_t d = 0; d < head_dim; ++d) {
            K[(size_t)p * head_dim + d] = load_elem(k_cache, base + d, dtype);
            V[(size_t)p * head_dim + d] = load_elem(v_cache, base + d, dtype);
        }
    }
    return 0;
}

/*
 * Attention of one query over a contiguous token range [t0, t1) of K/V:
 *   z_t = scale * sum_d q_d K_{t,d};  M = max_t z_t;  w_t = exp(z_t - M);
 * and returns M, sum_t w_t and sum_t w_t V_t (unnormalised).
 * An empty range returns M = -inf, l = 0, acc = 0.
 */
static void attend_range(const double* qv, const double* K, const double* V, int32_t t0,
                         int32_t t1, int32_t D, double scale, double* z, double* m_out,
                         double* l_out, double* acc) {
    for (int32_t d = 0; d < D; ++d) acc[d] = 0.0;
    if (t1 <= t0) { *m_out = -INFINITY; *l_out = 0.0; return; }
    double M = -INFINITY;
    for (int32_t t = t0; t < t1; ++t) {
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d) dot += qv[d] * K[(size_t)t * D + d];
        z[t - t0] = scale * dot;
        if (z[t - t0] > M) M = z[t - t0];
    }
    double l = 0.0;
    for (int32_t t = t0; t < t1; ++t) {
        double w = exp(z[t - t0] - M);
        l += w;
        for (int32_t d = 0; d < D; ++d) acc[d] += w * V[(size_t)t * D + d];
    }
    *m_out = M;
    *l_out = l;
}

/*
 * Decode attention through block tables, fp64.  For every sequence s and
 * query head qh (or only the (sel_seq[i], sel_head[i]) pairs when sel_seq is
 * not NULL), out = softmax(scale * q K_s^T) V_s over the sequence's
 * seq_lens[s] tokens; a zero-length sequence gives a zero row.
 * out is [num_seqs][num_q_heads][D] in full mode, [nsel][D] in selected mode.
 * Returns 0, or -1 when a table entry is outside the pool, -2 on bad sizes.
 */
int oracle_paged_decode(const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, int32_t max_blocks,
                        const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                        int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                        int64_t num_blocks, int32_t dtype, double scale,
                        const int32_t* sel_seq, const int32_t* sel_head, int32_t nsel,
                        double* out) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
        return -2;
    const int32_t group = num_q_heads / num_kv_heads;
    const int32_t D = head_dim;
    int32_t max_len = 0;
    for (int32_t s = 0; s < num_seqs; ++s) {
        if (seq_lens[s] < 0 || seq_lens[s] > max_blocks * block_size) return -2;
        if (seq_lens[s] > max_len) max_len = seq_lens[s];
    }
    double* K = (double*)malloc(sizeof(double) * ((size_t)max_len * D + 1));
    double* V = (double*)malloc(sizeof(double) * ((size_t)max_len * D + 1));
    double* z = (double*)malloc(sizeof(double) * ((size_t)max_len + 1));
    double* qv = (double*)malloc(sizeof(double) * (size_t)D);
    double* acc = (double*)malloc(sizeof(double) * (size_t)D);
    int rc = 0;
    const int32_t nrows = sel_seq ? nsel : num_seqs * num_q_heads;
    int32_t gathered_s = -1, gathered_h = -1;
    for (int32_t r = 0; r < nrows && rc == 0; ++r) {
        int32_t s = sel_seq ? sel_seq[r] : r / num_q_heads;
        int32_t qh = sel_seq ? sel_head[r] : r % num_q_heads;
        double* o = out + (size_t)r * D;
        if (s < 0 || s >= num_seqs || qh < 0 || qh >= num_q_heads) { rc = -2; break; }
        int32_t h = qh / group;
        int32_t L = seq_lens[s];
        if (L == 0) { for (int32_t d = 0; d < D; ++d) o[d] = 0.0; continue; }
        if (s != gathered_s || h != gathered_h) {
            if (gather_sequence(k_cache, v_cache, block_tables + (size_t)s * max_blocks, L, h,
                                num_kv_heads, D, block_size, num_blocks, dtype, K, V)) {
                rc = -1;
                break;
            }
            gathered_s = s;
            gathered_h = h;
        }
        for (int32_t d = 0; d < D; ++d)
            qv[d] = load_elem(q, ((size_t)s * num_q_heads + qh) * D + d, dtype);
        double M, l;
        attend_range(qv, K, V, 0, L, D, scale, z, &M, &l, acc);
        for (int32_t d = 0; d < D; ++d) o[d] = acc[d] / l;
    }
    free(K); free(V); free(z); free(qv); free(acc);
    return rc;
}

/*
 * Several new query tokens per sequence (a speculative-decoding check, a small
 * prefill chunk), rows packed without padding: the query tokens of sequence s
 * are rows q_start[s] .. q_start[s+1]-1 of q / out ([rows][num_q_heads][D]).
 * They are the sequence's last n = q_start[s+1] - q_start[s] positions, so
 * token r (0-based) sits at position p = seq_lens[s] - n + r and attends to
 * keys 0 .. p (causal).  Returns 0, -1 (table entry outside the pool), -2 (bad
 * sizes, or n > seq_len).
 */
int oracle_paged_decode_multi(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, int32_t max_blocks,
                              const int32_t* seq_lens, const int32_t* q_start, int32_t num_seqs,
                              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                              int32_t block_size, int64_t num_blocks, int32_t dtype, double scale,
                              double* out) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
        return -2;
    const int32_t group = num_q_heads / num_kv_heads;
    const int32_t D = head_dim;
    int32_t max_len = 0;
    for (int32_t s = 0; s < num_seqs; ++s) {
        const int32_t n = q_start[s + 1] - q_start[s];
        if (seq_lens[s] < 0 || seq_lens[s] > max_blocks * block_size || n < 0 || n > seq_lens[s])
            return -2;
        if (seq_lens[s] > max_len) max_len = seq_lens[s];
    }
    double* K = (double*)malloc(sizeof(double) * ((size_t)max_len * D + 1));
    double* V = (double*)malloc(sizeof(double) * ((size_t)max_len * D + 1));
    double* z = (double*)malloc(sizeof(double) * ((size_t)max_len + 1));
    double* qv = (double*)malloc(sizeof(double) * (size_t)D);
    double* acc = (double*)malloc(sizeof(double) * (size_t)D);
    int rc = 0;
    for (int32_t s = 0; s < num_seqs && rc == 0; ++s) {
        const int32_t L = seq_lens[s], n = q_start[s + 1] - q_start[s];
        for (int32_t h = 0; h < num_kv_heads && rc == 0; ++h) {
            if (gather_sequence(k_cache, v_cache, block_tables + (size_t)s * max_blocks, L, h,
                                num_kv_heads, D, block_size, num_blocks, dtype, K, V)) {
                rc = -1;
                break;
            }
            for (int32_t r = 0; r < n; ++r) {
                const int32_t pos = L - n + r;
                const size_t qrow = (size_t)q_start[s] + r;
                for (int32_t i = 0; i < group; ++i) {
                    const int32_t qh = h * group + i;
                    for (int32_t d = 0; d < D; ++d)
                        qv[d] = load_elem(q, (qrow * num_q_heads + qh) * D + d, dtype);
                    double M, l;
                    attend_range(qv, K, V, 0, pos + 1, D, scale, z, &M, &l, acc);
                    double* o = out + (qrow * num_q_heads + qh) * D;
                    for (int32_t d = 0; d < D; ++d) o[d] = acc[d] / l;
                }
            }
        }
    }
    free(K); free(V); free(z); free(qv); free(acc);
    return rc;
}

/*
 * Decode over an FP8 E4M3 cache: K_s[t] = decode(code) * k_scale[h] (same for
 * V), in fp64; q is bf16.  Otherwise as oracle_paged_decode (all rows).
 */
int oracle_paged_decode_fp8(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                            const int32_t* block_tables, int32_t max_blocks,
                            const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int64_t num_blocks, const float* k_scale, const float* v_scale,
                            double scale, double* out) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
        return -2;
    const int32_t group = num_q_heads / num_kv_heads;
    const int32_t D = head_dim;
    int32_t max_len = 0;
    for (int32_t s = 0; s < num_seqs; ++s) {
        if (seq_lens[s] < 0 || seq_lens[s] > max_blocks * block_size) return -2;
        if (seq_lens[s] > max_len) max_len = seq_lens[s];
    }
    double* K = (double*)malloc(sizeof(double) * ((size_t)max_len * D + 1));
    double* V = (double*)malloc(sizeof(double) * ((size_t)max_len * D + 1));
    double* z = (double*)malloc(sizeof(double) * ((size_t)max_len + 1));
    double* qv = (double*)malloc(sizeof(double) * (size_t)D);
    double* acc = (double*)malloc(sizeof(double) * (size_t)D);
    int rc = 0;
    for (int32_t s = 0; s < num_seqs && rc == 0; ++s) {
        const int32_t L = seq_lens[s];
        for (int32_t h = 0; h < num_kv_heads && rc == 0; ++h) {
            for (int32_t i = 0; i < group; ++i) {
                double* o = out + ((size_t)s * num_q_heads + h * group + i) * D;
                for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
            }
            if (L == 0) continue;
            if (gather_sequence(k_cache, v_cache, block_tables + (size_t)s * max_blocks, L, h,
                                num_kv_heads, D, block_size, num_blocks, ORACLE_E4M3, K, V)) {
                rc = -1;
                break;
            }
            for (size_t e = 0; e < (size_t)L * D; ++e) {
                K[e] *= (double)k_scale[h];
                V[e] *= (double)v_scale[h];
            }
            for (int32_t i = 0; i < group; ++i) {
                const int32_t qh = h * group + i;
                for (int32_t d = 0; d < D; ++d)
                    qv[d] = bf16_bits_to_double(q[((size_t)s * num_q_heads + qh) * D + d]);
                double M, l;
                attend_range(qv, K, V, 0, L, D, scale, z, &M, &l, acc);
                double* o = out + ((size_t)s * num_q_heads + qh) * D;
                for (int32_t d = 0; d < D; ++d) o[d] = acc[d] / l;
            }
        }
    }
    free(K); free(V); free(z); free(qv); free(acc);
    return rc;
}

/*
 * Split-K form of the same computation, used to pin the log-sum-exp merge:
 * the tokens of each sequence are cut into partitions of partition_tokens
 * consecutive logical positions; for partition p of (s, qh) it returns
 *   m = max z over the partition, l = sum exp(z - m), acc = sum exp(z - m) V.
 * nparts[s] = ceil(len / partition_tokens).  Layout:
 *   m, l  [num_seqs][num_q_heads][max_parts]
 *   acc   [num_seqs][num_q_heads][max_parts][D]
 * Returns 0, -1 (table entry outside the pool), -2 (bad sizes / too many parts).
 */
int oracle_decode_partials(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int32_t max_blocks,
                           const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                           int64_t num_blocks, int32_t dtype, double scale,
                           int32_t partition_tokens, int32_t max_parts, double* m, double* l,
                           double* acc, int32_t* nparts) {
    if (partition_tokens <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -2;
    const int32_t group = num_q_heads / num_kv_heads;
    const int32_t D = head_dim;
    int32_t max_len = 0;
    for (int32_t s = 0; s < num_seqs; ++s) {
        if (seq_lens[s] < 0 || seq_lens[s] > max_blocks * block_size) return -2;
        if (seq_lens[s] > max_len) max_len = seq_lens[s];
        nparts[s] = (seq_lens[s] + partition_tokens - 1) / partition_tokens;
        if (nparts[s] > max_parts) return -2;
    }
    double* K = (double*)malloc(sizeof(double) * ((size_t)max_len * D + 1));
    double* V = (double*)malloc(sizeof(double) * ((size_t)max_len * D + 1));
    double* z = (double*)malloc(sizeof(double) * ((size_t)partition_tokens + 1));
    double* qv = (double*)malloc(sizeof(double) * (size_t)D);
    int rc = 0;
    for (int32_t s = 0; s < num_seqs && rc == 0; ++s) {
        int32_t L = seq_lens[s];
        for (int32_t h = 0; h < num_kv_heads && rc == 0; ++h) {
            if (gather_sequence(k_cache, v_cache, block_tables + (size_t)s * max_blocks, L, h,
                                num_kv_heads, D, block_size, num_blocks, dtype, K, V)) {
                rc = -1;
                break;
            }
            for (int32_t i = 0; i < group; ++i) {
                int32_t qh = h * group + i;
                for (int32_t d = 0; d < D; ++d)
                    qv[d] = load_elem(q, ((size_t)s * num_q_heads + qh) * D + d, dtype);
                for (int32_t p = 0; p < nparts[s]; ++p) {
                    size_t idx = ((size_t)s * num_q_heads + qh) * max_parts + p;
                    int32_t t0 = p * partition_tokens;
                    int32_t t1 = t0 + partition_tokens < L ? t0 + partition_tokens : L;
                    attend_range(qv, K, V, t0, t1, D, scale, z, &m[idx], &l[idx], acc + idx * D);
                }
            }
        }
    }
    free(K); free(V); free(z); free(qv);
    return rc;
}

/*
 * Log-sum-exp merge of per-partition results:
 *   M = max_p m_p;  out = sum_p e^{m_p - M} acc_p / sum_p e^{m_p - M} l_p.
 * A sequence with no partitions gives a zero row.
 */
void oracle_lse_merge(const double* m, const double* l, const double* acc,
                      const int32_t* nparts, int32_t num_seqs, int32_t num_q_heads,
                      int32_t head_dim, int32_t max_parts, double* out) {
    const int32_t D = head_dim;
    for (int32_t s = 0; s < num_seqs; ++s) {
        for (int32_t qh = 0; qh < num_q_heads; ++qh) {
            size_t row = (size_t)s * num_q_heads + qh;
            double* o = out + row * D;
            for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
            if (nparts[s] == 0) continue;
            double M = -INFINITY;
            for (int32_t p = 0; p < nparts[s]; ++p)
                if (m[row * max_parts + p] > M) M = m[row * max_parts + p];
            double den = 0.0;
            for (int32_t p = 0; p < nparts[s]; ++p) {
                double w = exp(m[row * max_parts + p] - M);
                den += w * l[row * max_parts + p];
                for (int32_t d = 0; d < D; ++d) o[d] += w * acc[(row * max_parts + p) * D + d];
            }
            for (int32_t d = 0; d < D; ++d) o[d] /= den;
        }
    }
}
