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
//
// Prefix caching by block content (glossary, same section: hashing whole
// blocks extends sharing across requests, the prompt cache; "Paged Attention"
// study notes, section on prefix caching: look the prefix up by hash, then
// confirm the whole prefix matches).  A full block can be registered under a
// hash chained over its tokens and its predecessor's hash; a new sequence whose
// leading full blocks hit the cache starts with those blocks shared.  A hit is
// confirmed exactly: the block's stored tokens equal the request's and its
// stored predecessor is the block matched just before, in the same generation
// (a block's generation advances whenever it leaves the cache, so a stale
// child of a recycled block never matches).  Registered blocks whose count
// drops to zero stay cached, idle; allocation takes the free list first, then
// evicts the idle cached block released longest ago.
//
// Swapping (transcript, on preemption: a whole group of sequences leaves GPU
// memory, its KV data moved to CPU memory and brought back later): sequences
// move between two managers (a GPU pool's and a host pool's); every distinct
// block they use gets one block on the other side, and the (from, to) pairs
// drive pkv_swap_blocks.

#include <cstdint>
#include <cstring>
#include <deque>
#include <list>
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

    // prefix cache
    std::unordered_map<uint64_t, int32_t> cache;    // chained content hash -> block
    std::vector<char> cached;                       // block is registered
    std::vector<uint64_t> hash_of;
    std::vector<int32_t> parent_of;                 // block matched before it (-1: first block)
    std::vector<uint64_t> parent_gen_of;
    std::vector<uint64_t> gen;                      // advances when a block leaves the cache
    std::vector<std::vector<int32_t>> tokens_of;
    std::list<int32_t> idle;                        // cached blocks with no holder, oldest first
    std::vector<std::list<int32_t>::iterator> idle_pos;
    std::vector<char> in_idle;

    void init(int nb, int bs) {
        num_blocks = nb;
        block_size = bs;
        ref.assign(nb, 0);
        cached.assign(nb, 0);
        hash_of.assign(nb, 0);
        parent_of.assign(nb, -1);
        parent_gen_of.assign(nb, 0);
        gen.assign(nb, 0);
        tokens_of.assign(nb, {});
        idle_pos.resize(nb);
        in_idle.assign(nb, 0);
    }

    size_t available() const { return free_list.size() + idle.size(); }

    void uncache(int32_t b) {
        auto it = cache.find(hash_of[b]);
        if (it != cache.end() && it->second == b) cache.erase(it);
        cached[b] = 0;
        tokens_of[b].clear();
        ++gen[b];
    }

    // Callers check available() first.
    int32_t take() {
        int32_t b;
        if (!free_list.empty()) {
            b = free_list.front();
            free_list.pop_front();
        } else {
            b = idle.front();
            idle.pop_front();
            in_idle[b] = 0;
            uncache(b);
        }
        ref[b] = 1;
        return b;
    }

    void release(int32_t b) {
        if (--ref[b] == 0) {
            if (cached[b]) {
                idle.push_back(b);
                idle_pos[b] = std::prev(idle.end());
                in_idle[b] = 1;
            } else {
                free_list.push_back(b);
            }
        }
    }

    void acquire(int32_t b) {   // one more holder of a (possibly idle) cached block
        if (in_idle[b]) {
            idle.erase(idle_pos[b]);
            in_idle[b] = 0;
        }
        ++ref[b];
    }

    // 64-bit hash of one block's tokens chained on its predecessor's hash
    // (multiply-xorshift mixing of each 32-bit token into the running state).
    static uint64_t mix(uint64_t x) {
        x ^= x >> 33;
        x *= 0xff51afd7ed558ccdull;
        x ^= x >> 33;
        x *= 0xc4ceb9fe1a85ec53ull;
        x ^= x >> 33;
        return x;
    }
    // A cached block b holds exactly these tokens and follows block prev (-1: the first block)
    // of the same generation.
    bool confirms(int32_t b, int32_t prev, const int32_t* toks) const {
        return parent_of[b] == prev && (prev < 0 || parent_gen_of[b] == gen[prev]) &&
               std::memcmp(tokens_of[b].data(), toks, sizeof(int32_t) * block_size) == 0;
    }
    uint64_t block_hash(uint64_t parent, const int32_t* toks) const {
        uint64_t h = mix(parent ^ 0x9e3779b97f4a7c15ull);
        for (int i = 0; i < block_size; ++i) h = mix(h ^ (static_cast<uint64_t>(static_cast<uint32_t>(toks[i])) +
                                                        (static_cast<uint64_t>(i) << 32)));
        return h;
    }
};

extern "C" pkv_block_manager* pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order) {
    if (num_blocks <= 0 || block_size <= 0) return nullptr;
    pkv_block_manager* m = new (std::nothrow) pkv_block_manager();
    if (!m) return nullptr;
    try {
        m->init(num_blocks, block_size);
    } catch (...) {
        delete m;
        return nullptr;
    }
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
    return static_cast<int>(m->available());
}

extern "C" int pkv_bm_num_cached(pkv_block_manager* m) {
    if (!m) return -1;
    std::lock_guard<std::mutex> g(m->mu);
    return static_cast<int>(m->cache.size());
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
    for (int32_t b : c.blocks) m->acquire(b);
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
    if (need_blocks > m->available()) return PKV_ERR_OUT_OF_BLOCKS;
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

extern "C" pkv_status pkv_bm_append_tokens(pkv_block_manager* m, int64_t seq_id, int n, int64_t* slots,
                                           int64_t* pairs, int max_pairs, int* num_pairs) {
    if (!m || n < 0 || (n > 0 && !slots) || !num_pairs || max_pairs < 0 || (max_pairs > 0 && !pairs))
        return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(m->mu);
    auto it = m->seqs.find(seq_id);
    if (it == m->seqs.end()) return PKV_ERR_INVALID_ARG;
    auto& s = it->second;
    const int64_t B = m->block_size;
    const int64_t off = s.len % B;
    // a shared partial last block is copied once, before the first write; the tokens that do
    // not fit in the last block take ceil(rest / B) new blocks
    const bool copy = n > 0 && off != 0 && m->ref[s.blocks.back()] > 1;
    const int64_t room = off == 0 ? 0 : B - off;
    const int64_t rest = n > room ? n - room : 0;
    const size_t need = static_cast<size_t>((rest + B - 1) / B) + (copy ? 1 : 0);
    if (need > m->available()) return PKV_ERR_OUT_OF_BLOCKS;
    if (copy && max_pairs < 1) return PKV_ERR_INVALID_ARG;
    int np = 0;
    if (copy) {
        const int32_t last = s.blocks.back();
        const int32_t fresh = m->take();
        pairs[0] = last;
        pairs[1] = fresh;
        np = 1;
        --m->ref[last];
        s.blocks.back() = fresh;
    }
    for (int i = 0; i < n; ++i) {
        const int64_t o = s.len % B;
        if (o == 0) s.blocks.push_back(m->take());
        slots[i] = static_cast<int64_t>(s.blocks.back()) * B + o;
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

// ---- prefix cache ----------------------------------------------------------------

extern "C" pkv_status pkv_bm_add_sequence_cached(pkv_block_manager* m, int64_t seq_id, const int32_t* tokens,
                                                 int num_tokens, int* num_cached_tokens) {
    if (!m || num_tokens < 0 || (num_tokens > 0 && !tokens) || !num_cached_tokens) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(m->mu);
    if (m->seqs.count(seq_id)) return PKV_ERR_INVALID_ARG;
    const int B = m->block_size;
    const int max_blocks = num_tokens > 0 ? (num_tokens - 1) / B : 0;   // leave at least one token to compute
    pkv_block_manager::Seq s;
    uint64_t h = 0;
    int32_t prev = -1;
    for (int j = 0; j < max_blocks; ++j) {
        const int32_t* toks = tokens + static_cast<size_t>(j) * B;
        h = m->block_hash(h, toks);
        auto it = m->cache.find(h);
        if (it == m->cache.end()) break;
        const int32_t b = it->second;
        if (!m->confirms(b, prev, toks)) break;                // hash collision or stale entry: stop
        s.blocks.push_back(b);
        prev = b;
    }
    for (int32_t b : s.blocks) m->acquire(b);
    s.len = static_cast<int64_t>(s.blocks.size()) * B;
    *num_cached_tokens = static_cast<int>(s.len);
    m->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

extern "C" pkv_status pkv_bm_cache_sequence(pkv_block_manager* m, int64_t seq_id, const int32_t* tokens,
                                            int num_tokens) {
    if (!m || num_tokens < 0 || (num_tokens > 0 && !tokens)) return PKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(m->mu);
    auto it = m->seqs.find(seq_id);
    if (it == m->seqs.end() || num_tokens > it->second.len) return PKV_ERR_INVALID_ARG;
    const int B = m->block_size;
    const auto& s = it->second;
    uint64_t h = 0;
    int32_t prev = -1;
    for (int j = 0; j < num_tokens / B; ++j) {
        const int32_t* toks = tokens + static_cast<size_t>(j) * B;
        const int32_t b = s.blocks[j];
        h = m->block_hash(h, toks);
        if (!m->cached[b]) {
            auto hit = m->cache.find(h);
            if (hit != m->cache.end()) {
                // The same prefix already cached in another block: keep that one and chain the
                // following blocks on it, so that a lookup walking the cached chain reaches them.
                // A colliding hash whose block holds another prefix ends the registration.
                if (!m->confirms(hit->second, prev, toks)) break;
                prev = hit->second;
                continue;
            }
            m->cache.emplace(h, b);
            m->cached[b] = 1;
            m->hash_of[b] = h;
            m->parent_of[b] = prev;
            m->parent_gen_of[b] = prev >= 0 ? m->gen[prev] : 0;
            m->tokens_of[b].assign(toks, toks + B);
        }
        prev = b;
    }
    return PKV_OK;
}

// ---- swapping between two managers -------------------------------------------------

extern "C" pkv_status pkv_bm_swap(pkv_block_manager* from, pkv_block_manager* to, const int64_t* seq_ids, int n,
                                  int64_t* pairs, int max_pairs, int* num_pairs) {
    if (!from || !to || from == to || n < 0 || (n > 0 && !seq_ids) || !num_pairs || max_pairs < 0 ||
        (max_pairs > 0 && !pairs) || from->block_size != to->block_size)
        return PKV_ERR_INVALID_ARG;
    std::scoped_lock g(from->mu, to->mu);
    std::unordered_map<int32_t, int32_t> map;   // block in `from` -> block in `to`
    std::vector<int32_t> order;
    for (int i = 0; i < n; ++i) {
        auto it = from->seqs.find(seq_ids[i]);
        if (it == from->seqs.end() || to->seqs.count(seq_ids[i])) return PKV_ERR_INVALID_ARG;
        for (int k = 0; k < i; ++k)
            if (seq_ids[k] == seq_ids[i]) return PKV_ERR_INVALID_ARG;
        for (int32_t b : it->second.blocks)
            if (map.emplace(b, -1).second) order.push_back(b);
    }
    if (order.size() > to->available()) return PKV_ERR_OUT_OF_BLOCKS;
    if (static_cast<int>(order.size()) > max_pairs) return PKV_ERR_INVALID_ARG;
    for (size_t i = 0; i < order.size(); ++i) {
        const int32_t nb = to->take();
        to->ref[nb] = 0;   // counted below, once per sequence that holds it
        map[order[i]] = nb;
        pairs[2 * i] = order[i];
        pairs[2 * i + 1] = nb;
    }
    for (int i = 0; i < n; ++i) {
        auto it = from->seqs.find(seq_ids[i]);
        pkv_block_manager::Seq t;
        t.len = it->second.len;
        for (int32_t b : it->second.blocks) {
            const int32_t nb = map[b];
            ++to->ref[nb];
            t.blocks.push_back(nb);
            from->release(b);
        }
        from->seqs.erase(it);
        to->seqs.emplace(seq_ids[i], std::move(t));
    }
    *num_pairs = static_cast<int>(order.size());
    return PKV_OK;
}
