// block_manager.cpp -- host-side bookkeeping of the paged KV pool.
//
// The KV cache is a pool of fixed 16-token blocks.  A sequence holds
// ceil(len / 16) of them, listed in its block table; blocks are taken from a
// free list as the sequence grows and returned when it ends ("Was ändert
// PagedAttention an der KV-Speicherzuweisung für LLMs?", slavadubrov.com,
// §"Ungenutzten Platz in Blöcken berechnen").  Several sequences may hold the
// same block (a forked prompt, parallel samples, a cached prefix); a block that
// is shared and only partly filled is copied before a sequence writes into it
// (copy-on-write: same page, §"Gemeinsame Nutzung erfordert mehr als
// Speicherzuweisung"; "PagedAttention et vLLM", aiunderstanding.org,
// §"Questions fréquemment posées": copy only when a branch diverges).
//
// This file keeps that state on the host: free list (first-in first-out,
// starting in ascending id order), reference counts, and per-sequence tables
// and lengths.  It computes the slot of every appended token (the input of
// pa_cache_write) and the block copies a divergence needs (the input of
// pa_copy_blocks), and exports block tables for pa_decode.  It touches no GPU
// memory.  All entry points lock the manager, so one manager may be shared by
// threads.
#include <cstdint>
#include <deque>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedattn.h"

struct pa_block_manager {
    int32_t num_blocks;
    int32_t block_size;
    int32_t max_blocks_per_seq;
    std::deque<int32_t> free_list;
    std::vector<int32_t> ref;
    struct Seq {
        std::vector<int32_t> table;
        int32_t len = 0;
    };
    std::unordered_map<int32_t, Seq> seqs;
    std::mutex mu;
};

namespace {

int32_t take_block(pa_block_manager* m) {
    const int32_t b = m->free_list.front();
    m->free_list.pop_front();
    m->ref[b] = 1;
    return b;
}

void release_block(pa_block_manager* m, int32_t b) {
    if (--m->ref[b] == 0) m->free_list.push_back(b);
}

}  // namespace

extern "C" {

pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size, int32_t max_blocks_per_seq) {
    if (num_blocks <= 0 || block_size <= 0 || max_blocks_per_seq <= 0) return nullptr;
    pa_block_manager* m = new (std::nothrow) pa_block_manager();
    if (!m) return nullptr;
    m->num_blocks = num_blocks;
    m->block_size = block_size;
    m->max_blocks_per_seq = max_blocks_per_seq;
    m->ref.assign(static_cast<size_t>(num_blocks), 0);
    for (int32_t b = 0; b < num_blocks; ++b) m->free_list.push_back(b);
    return m;
}

void pa_bm_destroy(pa_block_manager* m) { delete m; }

int pa_bm_add_sequence(pa_block_manager* m, int32_t seq) {
    if (!m) return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(m->mu);
    if (m->seqs.count(seq)) return PA_ERR_INVALID_ARG;
    m->seqs.emplace(seq, pa_block_manager::Seq());
    return PA_OK;
}

int pa_bm_fork(pa_block_manager* m, int32_t parent, int32_t child) {
    if (!m) return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(m->mu);
    auto it = m->seqs.find(parent);
    if (it == m->seqs.end() || m->seqs.count(child)) return PA_ERR_INVALID_ARG;
    pa_block_manager::Seq s = it->second;
    for (int32_t b : s.table) ++m->ref[b];
    m->seqs.emplace(child, std::move(s));
    return PA_OK;
}

int pa_bm_append(pa_block_manager* m, int32_t seq, int32_t num_tokens, int64_t* slots_out,
                 int32_t* copy_src, int32_t* copy_dst, int32_t* num_copies) {
    if (!m || num_tokens < 0 || (num_tokens > 0 && !slots_out) || !num_copies)
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(m->mu);
    auto it = m->seqs.find(seq);
    if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
    pa_block_manager::Seq& s = it->second;
    const int64_t B = m->block_size;
    const int64_t new_len = static_cast<int64_t>(s.len) + num_tokens;
    const int64_t need_blocks = (new_len + B - 1) / B;
    if (need_blocks > m->max_blocks_per_seq) return PA_ERR_INVALID_ARG;
    const int64_t new_blocks = need_blocks - static_cast<int64_t>(s.table.size());
    // the last block is written into: copy it first if it is shared
    const bool cow = num_tokens > 0 && s.len % B != 0 && m->ref[s.table.back()] > 1;
    if (cow && (!copy_src || !copy_dst)) return PA_ERR_INVALID_ARG;
    if (new_blocks + (cow ? 1 : 0) > static_cast<int64_t>(m->free_list.size()))
        return PA_ERR_OUT_OF_BLOCKS;  // nothing changed
    *num_copies = 0;
    if (cow) {
        const int32_t old = s.table.back();
        const int32_t nb = take_block(m);
        copy_src[0] = old;
        copy_dst[0] = nb;
        *num_copies = 1;
        release_block(m, old);
        s.table.back() = nb;
    }
    for (int64_t pos = s.len; pos < new_len; ++pos) {
        const int64_t j = pos / B;
        if (j == static_cast<int64_t>(s.table.size())) s.table.push_back(take_block(m));
        slots_out[pos - s.len] = static_cast<int64_t>(s.table[j]) * B + pos % B;
    }
    s.len = static_cast<int32_t>(new_len);
    return PA_OK;
}

int pa_bm_free_sequence(pa_block_manager* m, int32_t seq) {
    if (!m) return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(m->mu);
    auto it = m->seqs.find(seq);
    if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
    for (int32_t b : it->second.table) release_block(m, b);
    m->seqs.erase(it);
    return PA_OK;
}

int32_t pa_bm_num_free(pa_block_manager* m) {
    if (!m) return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(m->mu);
    return static_cast<int32_t>(m->free_list.size());
}

int32_t pa_bm_refcount(pa_block_manager* m, int32_t block) {
    if (!m || block < 0 || block >= m->num_blocks) return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(m->mu);
    return m->ref[block];
}

int pa_bm_export_tables(pa_block_manager* m, const int32_t* seq_ids, int32_t num_seqs,
                        int32_t* tables_out, int32_t width, int32_t* lens_out) {
    if (!m || num_seqs < 0 || width <= 0 || (num_seqs > 0 && (!seq_ids || !tables_out || !lens_out)))
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(m->mu);
    for (int32_t i = 0; i < num_seqs; ++i) {
        auto it = m->seqs.find(seq_ids[i]);
        if (it == m->seqs.end() || static_cast<int32_t>(it->second.table.size()) > width)
            return PA_ERR_INVALID_ARG;
    }
    for (int32_t i = 0; i < num_seqs; ++i) {
        const pa_block_manager::Seq& s = m->seqs.find(seq_ids[i])->second;
        int32_t* row = tables_out + static_cast<size_t>(i) * width;
        const int32_t n = static_cast<int32_t>(s.table.size());
        for (int32_t j = 0; j < width; ++j) row[j] = j < n ? s.table[j] : -1;
        lens_out[i] = s.len;
    }
    return PA_OK;
}

}  // extern "C"
