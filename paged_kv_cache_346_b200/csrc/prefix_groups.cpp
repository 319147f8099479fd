// Host-side grouping for the shared-prefix decode: sequences whose block
// tables start with the same physical blocks.
//
// Blocks shared by several sequences are the paged cache's copy-on-write
// sharing: parallel samples forked from one prompt hold the prompt's blocks
// until they write into them ("pagedattention vllm" §Copy-on-Write Sharing),
// and requests that hit the same cached prompt blocks hold those
// (§Advanced Features).  A physical block holds one set of tokens, so two
// sequences that hold the same block at the same logical position attend to
// the same keys and values there.
#include <algorithm>
#include <cstdint>
#include <map>
#include <vector>

#include "pagedkv.h"

extern "C" int pkv_decode_prefix_groups(const int32_t* block_tables, const int32_t* context_lens,
                                        int num_seqs, int max_blocks_per_seq, int block_size,
                                        int max_group_size, int min_prefix_blocks,
                                        int32_t* seq_prefix_len, int32_t* group_members,
                                        int group_capacity, int* num_groups) {
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || max_group_size < 2 ||
        max_group_size > PKV_MAX_PREFIX_GROUP || min_prefix_blocks < 1 || group_capacity < 0 ||
        !num_groups)
        return PKV_EINVAL;
    if (num_seqs > 0 && (!block_tables || !context_lens || !seq_prefix_len)) return PKV_EINVAL;
    if (group_capacity > 0 && !group_members) return PKV_EINVAL;
    *num_groups = 0;
    // full blocks of each sequence (only those can be shared by sequences of
    // different lengths); buckets by the first block, in order of first member
    std::vector<int> nfull(num_seqs);
    std::map<int32_t, std::vector<int>> bucket;
    std::vector<int32_t> first_seen;
    for (int b = 0; b < num_seqs; ++b) {
        seq_prefix_len[b] = 0;
        const int L = context_lens[b];
        nfull[b] = L > 0 ? std::min(L / block_size, max_blocks_per_seq) : 0;
        if (nfull[b] < min_prefix_blocks) continue;
        const int32_t first = block_tables[(int64_t)b * max_blocks_per_seq];
        if (first < 0) continue;  // released (sliding window) or padding
        auto& v = bucket[first];
        if (v.empty()) first_seen.push_back(first);
        v.push_back(b);
    }
    int ng = 0;
    for (int32_t first : first_seen) {
        const std::vector<int>& mem = bucket[first];
        for (size_t c0 = 0; c0 + 1 < mem.size(); c0 += max_group_size) {
            const size_t c1 = std::min(mem.size(), c0 + (size_t)max_group_size);
            // longest common run of table entries over the chunk's full blocks
            int lcp = nfull[mem[c0]];
            for (size_t i = c0 + 1; i < c1; ++i) lcp = std::min(lcp, nfull[mem[i]]);
            const int32_t* t0 = block_tables + (int64_t)mem[c0] * max_blocks_per_seq;
            for (size_t i = c0 + 1; i < c1 && lcp > 0; ++i) {
                const int32_t* ti = block_tables + (int64_t)mem[i] * max_blocks_per_seq;
                int j = 0;
                while (j < lcp && ti[j] == t0[j]) ++j;
                lcp = j;
            }
            if (lcp < min_prefix_blocks) continue;
            if (ng >= group_capacity) return PKV_EBOUNDS;
            int32_t* row = group_members + (int64_t)ng * max_group_size;
            for (int k = 0; k < max_group_size; ++k) row[k] = -1;
            for (size_t i = c0; i < c1; ++i) {
                row[i - c0] = mem[i];
                seq_prefix_len[mem[i]] = lcp * block_size;
            }
            ++ng;
        }
    }
    *num_groups = ng;
    return PKV_OK;
}
