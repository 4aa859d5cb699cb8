// Host helper for shared-prefix decode: finds sequences whose block tables begin
// with the same physical blocks (a shared prompt, ref-counted -- Ultralytics
// glossary "PagedAttention", section "Sharing blocks across sequences") and packs
// them into units for pkv_paged_attn_decode_shared_prefix.

#include <algorithm>
#include <cstdint>
#include <map>
#include <vector>

#include "../../include/pagedkv.h"

extern "C" pkv_status pkv_find_shared_prefixes(const int32_t* block_tables, const int32_t* context_lens,
                                               int num_seqs, int max_blocks_per_seq, int block_size,
                                               int unit_width, int32_t* seq_prefix_len, int32_t* unit_seqs,
                                               int32_t* unit_len, int max_units, int* num_units,
                                               int* max_prefix_len) {
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || unit_width <= 0 || max_units < 0 ||
        !num_units || !max_prefix_len || (num_seqs > 0 && (!block_tables || !context_lens || !seq_prefix_len)) ||
        (max_units > 0 && (!unit_seqs || !unit_len)))
        return PKV_ERR_INVALID_ARG;
    // group sequences by their first block (sharing starts at block 0)
    std::map<int32_t, std::vector<int>> by_first;
    for (int s = 0; s < num_seqs; ++s) {
        seq_prefix_len[s] = 0;
        if (context_lens[s] >= block_size) by_first[block_tables[static_cast<size_t>(s) * max_blocks_per_seq]].push_back(s);
    }
    int nu = 0, maxp = 0;
    for (auto& kv : by_first) {
        const std::vector<int>& g = kv.second;
        if (g.size() < 2) continue;
        // common leading blocks, each full for every member
        int common = max_blocks_per_seq;
        for (int s : g) common = std::min(common, static_cast<int>(context_lens[s] / block_size));
        const int32_t* t0 = block_tables + static_cast<size_t>(g[0]) * max_blocks_per_seq;
        for (size_t i = 1; i < g.size(); ++i) {
            const int32_t* ti = block_tables + static_cast<size_t>(g[i]) * max_blocks_per_seq;
            int j = 0;
            while (j < common && ti[j] == t0[j]) ++j;
            common = j;
        }
        if (common == 0) continue;
        const int plen = common * block_size;
        for (size_t i = 0; i < g.size(); i += unit_width) {
            if (nu >= max_units) return PKV_ERR_INVALID_ARG;
            for (int m = 0; m < unit_width; ++m) {
                const size_t k = i + m;
                unit_seqs[static_cast<size_t>(nu) * unit_width + m] = k < g.size() ? g[k] : -1;
                if (k < g.size()) seq_prefix_len[g[k]] = plen;
            }
            unit_len[nu++] = plen;
        }
        maxp = std::max(maxp, plen);
    }
    *num_units = nu;
    *max_prefix_len = maxp;
    return PKV_OK;
}
