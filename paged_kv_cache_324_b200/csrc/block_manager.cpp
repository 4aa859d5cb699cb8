// Host-side block manager: the bookkeeping that feeds the paged kernels.
//
// Physical blocks of the pool are handed out from a FIFO free list; each
// sequence keeps the ordered list of its blocks (its block table) and its
// length.  A sequence takes a new block only when its last one is full, so
// it holds ceil(L / B) blocks and wastes at most B - 1 slots (Ultralytics
// glossary "PagedAttention", section "How paging works").  Blocks carry
// reference counts: a fork shares every block of its parent; appending to a
// last block that other sequences also reference first gives the writer a
// private copy (a (src, dst) pair for pkv_copy_blocks), and the last holder
// writes in place (glossary, section "Sharing blocks across sequences";
// "vLLM and PagedAttention" transcript: only the partially filled shared
// block is copied, full ones stay shared).  Freeing a sequence returns the
// blocks whose count drops to zero to the back of the free list at once.

#include <cstdint>
#include <cstring>
#include <deque>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pagedkv.h"

struct pkv_block_manager {
    int num_blocks = 0;
    int block_size = 0;
    std::deque<int32_t> free_list;
    std::vector<int32_t> ref;   // per physical block
    struct Seq {
        std::vector<int32_t> blocks;
        int64_t len = 0;
    };
    std::unordered_map<int64_t, Seq> seqs;
    std::mutex mu;

    int32_t take() {
        const int32_t b = free_list.front();
        free_list.pop_front();
        ref[b] = 1;
        return b;
    }
    void release(int32_t b) {
        if (--ref[b] == 0) free_list.push_back(b);
    }
};

extern "C" pkv_block_manager* pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order) {
    if (num_blocks <= 0 || block_size <= 0) return nullptr;
    pkv_block_manager* m = new (std::nothrow) pkv_block_manager();
    if (!m) return nullptr;
    m->num_blocks = num_blocks;
    m->block_size = block_size;
    m->ref.assign(num_blocks, 0);
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
        const int32_t b = free_order ? free_order[i] : i;
        if (b < 0 || b >= num_blocks || seen[b]) {   // must be a permutation of 0..num_blocks-1
            delete m;
            return nullptr;
        }
        seen[b] = 1;
        m->free_list.push_back(b);
    }
    return m;
}

extern "C" void pkv_bm_destroy(pkv_block_manager* m) { delete m; }

extern "C" int pkv_bm_num_free(pkv_block_manager* m) {
    if (!m) return -1;
    std::lock_guard<std::mutex> g(m->mu);
    return static_cast<int>(m->free_list.size());
}

extern "C" pkv_status pkv_bm_add_sequence(pkv_block_manager* m, int64_t seq_id) {
    if (!m) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(m->mu);
    if (m->seqs.count(seq_id)) return PKV_ERR_INVALID_ARG;
    m->seqs.emplace(seq_id, pkv_block_manager::Seq{});
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_fork(pkv_block_manager* m, int64_t parent, int64_t child) {
    if (!m) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(m->mu);
    auto it = m->seqs.find(parent);
    if (it == m->seqs.end() || m->seqs.count(child)) return PKV_ERR_INVALID_ARG;
    pkv_block_manager::Seq c = it->second;
    for (int32_t b : c.blocks) ++m->ref[b];
    m->seqs.emplace(child, std::move(c));
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_append_slots(pkv_block_manager* m, const int64_t* seq_ids, int n, int64_t* slots,
                                          int64_t* pairs, int max_pairs, int* num_pairs) {
    if (!m || n < 0 || (n > 0 && (!seq_ids || !slots)) || !num_pairs || max_pairs < 0 ||
        (max_pairs > 0 && !pairs))
        return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(m->mu);
    // check everything first so that a failed call changes nothing
    size_t need_blocks = 0;
    int need_pairs = 0;
    std::unordered_map<int32_t, int> copied;   // copies already planned per shared block
    for (int i = 0; i < n; ++i) {
        auto it = m->seqs.find(seq_ids[i]);
        if (it == m->seqs.end()) return PKV_ERR_INVALID_ARG;
        for (int k = 0; k < i; ++k)
            if (seq_ids[k] == seq_ids[i]) return PKV_ERR_INVALID_ARG;   // one token per sequence per call
        const auto& s = it->second;
        if (s.len % m->block_size == 0) {
            ++need_blocks;                                   // last block full (or none): a new block
        } else {
            const int32_t last = s.blocks.back();
            if (m->ref[last] - copied[last] > 1) {           // still shared when this sequence writes
                ++copied[last];
                ++need_blocks;
                ++need_pairs;
            }
        }
    }
    if (need_blocks > m->free_list.size()) return PKV_ERR_OUT_OF_BLOCKS;
    if (need_pairs > max_pairs) return PKV_ERR_INVALID_ARG;
    int np = 0;
    for (int i = 0; i < n; ++i) {
        auto& s = m->seqs[seq_ids[i]];
        const int64_t off = s.len % m->block_size;
        if (off == 0) {
            s.blocks.push_back(m->take());
        } else {
            const int32_t last = s.blocks.back();
            if (m->ref[last] > 1) {                          // copy before write
                const int32_t fresh = m->take();
                pairs[2 * np] = last;
                pairs[2 * np + 1] = fresh;
                ++np;
                --m->ref[last];
                s.blocks.back() = fresh;
            }
        }
        slots[i] = static_cast<int64_t>(s.blocks.back()) * m->block_size + off;
        ++s.len;
    }
    *num_pairs = np;
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_free_sequence(pkv_block_manager* m, int64_t seq_id) {
    if (!m) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(m->mu);
    auto it = m->seqs.find(seq_id);
    if (it == m->seqs.end()) return PKV_ERR_INVALID_ARG;
    for (int32_t b : it->second.blocks) m->release(b);
    m->seqs.erase(it);
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_block_tables(pkv_block_manager* m, const int64_t* seq_ids, int n, int32_t* tables,
                                          int max_blocks, int32_t pad, int32_t* context_lens) {
    if (!m || n < 0 || max_blocks <= 0 || (n > 0 && (!seq_ids || !tables))) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(m->mu);
    for (int i = 0; i < n; ++i) {
        auto it = m->seqs.find(seq_ids[i]);
        if (it == m->seqs.end()) return PKV_ERR_INVALID_ARG;
        if (static_cast<int>(it->second.blocks.size()) > max_blocks) return PKV_ERR_INVALID_ARG;
    }
    for (int i = 0; i < n; ++i) {
        const auto& s = m->seqs[seq_ids[i]];
        int32_t* row = tables + static_cast<size_t>(i) * max_blocks;
        const size_t nb = s.blocks.size();
        if (nb) std::memcpy(row, s.blocks.data(), nb * sizeof(int32_t));
        for (int j = static_cast<int>(nb); j < max_blocks; ++j) row[j] = pad;
        if (context_lens) context_lens[i] = static_cast<int32_t>(s.len);
    }
    return PKV_OK;
}

extern "C" int pkv_bm_ref_count(pkv_block_manager* m, int32_t block) {
    if (!m || block < 0) return -1;
    std::lock_guard<std::mutex> g(m->mu);
    return block < m->num_blocks ? m->ref[block] : -1;
}

extern "C" int64_t pkv_bm_sequence_length(pkv_block_manager* m, int64_t seq_id) {
    if (!m) return -1;
    std::lock_guard<std::mutex> g(m->mu);
    auto it = m->seqs.find(seq_id);
    return it == m->seqs.end() ? -1 : it->second.len;
}
