// Host-side KV block manager: free list, reference counts, fork and
// copy-on-write ("pagedattention vllm" §Memory Management and §Copy-on-Write
// Sharing; "What is PagedAttention ..." §How it works).  The rules each
// operation follows are stated next to the declarations in pagedkv.h.
//
// Data structures: a vector used as a stack of free block ids, a reference
// count per block, and a hash map from sequence id to (block table, length,
// swapped?).  An optional host pool (its own free stack) receives the blocks
// of swapped-out sequences ("pagedattention vllm" §Memory Management:
// swapping blocks to CPU memory).  Every operation either completes or
// leaves all of it untouched.
//
// Prefix cache ("pagedattention vllm" §vLLM Integration and §Advanced
// Features: prefix caching; "PagedAttention" glossary entry: prompt caching
// lets later requests that start the same way skip that part).  A full
// prompt block is registered under (registration id of the block before it,
// its block_size token ids); a new prompt walks its full blocks and reuses
// each registered block whose key matches, so a hit means the whole prefix up
// to that block is identical.  A registered block whose count drops to zero
// is kept (evictable, least recently released first) until an allocation finds
// the free stack empty and takes it back.
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

struct pkv_alloc {
    int32_t num_blocks;
    int32_t block_size;
    int32_t num_host_blocks = 0;
    std::vector<int32_t> free_stack;       // back() is handed out next
    std::vector<int32_t> host_free_stack;  // host pool, same discipline
    std::vector<int32_t> ref;
    struct Seq {
        std::vector<int32_t> table;  // device block ids, or host ids when swapped
        int64_t len;
        bool swapped = false;
    };
    int32_t swapped_seqs = 0;
    std::unordered_map<int64_t, Seq> seqs;
    int64_t refcount_sum = 0;
    int64_t logical_tokens = 0;
    int32_t used_blocks = 0;
    int32_t shared_blocks = 0;

    // ---- prefix cache (allocated on first use)
    std::vector<int64_t> reg_id;       // per block: registration id, 0 = not registered
    std::vector<int64_t> reg_parent;   // per block: registration id of the block before it
    std::vector<int32_t> reg_tokens;   // per block: its block_size token ids
    std::unordered_multimap<uint64_t, int32_t> reg_map;  // key hash -> registered blocks
    int64_t next_reg = 1;
    int32_t cached_blocks = 0;
    // evictable registered blocks: a doubly linked list over block ids,
    // least recently released at the head
    std::vector<int32_t> ev_prev, ev_next;
    int32_t ev_head = -1, ev_tail = -1, evictable = 0;

    bool cache_on() const { return !reg_id.empty(); }
    void cache_init() {
        if (cache_on()) return;
        reg_id.assign(num_blocks, 0);
        reg_parent.assign(num_blocks, 0);
        reg_tokens.assign((size_t)num_blocks * block_size, 0);
        ev_prev.assign(num_blocks, -1);
        ev_next.assign(num_blocks, -1);
    }
    static uint64_t key_hash(int64_t parent, const int32_t* tokens, int n) {
        uint64_t h = 1469598103934665603ull;  // FNV-1a, 64 bit
        auto mix = [&](uint64_t v) {
            for (int i = 0; i < 8; ++i) {
                h ^= (v >> (8 * i)) & 0xffu;
                h *= 1099511628211ull;
            }
        };
        mix((uint64_t)parent);
        for (int i = 0; i < n; ++i) mix((uint64_t)(uint32_t)tokens[i]);
        return h;
    }
    // the registered block with this exact key, or -1
    int32_t lookup(int64_t parent, const int32_t* tokens) const {
        auto range = reg_map.equal_range(key_hash(parent, tokens, block_size));
        for (auto it = range.first; it != range.second; ++it) {
            const int32_t b = it->second;
            if (reg_parent[b] == parent &&
                std::memcmp(&reg_tokens[(size_t)b * block_size], tokens,
                            sizeof(int32_t) * block_size) == 0)
                return b;
        }
        return -1;
    }
    void ev_push(int32_t b) {
        ev_prev[b] = ev_tail;
        ev_next[b] = -1;
        if (ev_tail >= 0) ev_next[ev_tail] = b; else ev_head = b;
        ev_tail = b;
        ++evictable;
    }
    void ev_remove(int32_t b) {
        if (ev_prev[b] >= 0) ev_next[ev_prev[b]] = ev_next[b]; else ev_head = ev_next[b];
        if (ev_next[b] >= 0) ev_prev[ev_next[b]] = ev_prev[b]; else ev_tail = ev_prev[b];
        ev_prev[b] = ev_next[b] = -1;
        --evictable;
    }
    void unregister(int32_t b) {
        auto range = reg_map.equal_range(
            key_hash(reg_parent[b], &reg_tokens[(size_t)b * block_size], block_size));
        for (auto it = range.first; it != range.second; ++it)
            if (it->second == b) {
                reg_map.erase(it);
                break;
            }
        reg_id[b] = 0;
        --cached_blocks;
    }
    int64_t available() const { return (int64_t)free_stack.size() + evictable; }

    int32_t take() {
        int32_t b;
        if (!free_stack.empty()) {
            b = free_stack.back();
            free_stack.pop_back();
        } else {  // evict the least recently released cached block
            b = ev_head;
            ev_remove(b);
            unregister(b);
        }
        ref[b] = 1;
        ++used_blocks;
        ++refcount_sum;
        return b;
    }
    void add_ref(int32_t b) {
        if (ref[b] == 1) ++shared_blocks;
        ++ref[b];
        ++refcount_sum;
    }
    void drop_ref(int32_t b) {
        --ref[b];
        --refcount_sum;
        if (ref[b] == 1) --shared_blocks;
        if (ref[b] == 0) {
            --used_blocks;
            if (cache_on() && reg_id[b] != 0) ev_push(b);
            else free_stack.push_back(b);
        }
    }
};

extern "C" {

int pkv_alloc_create_swap(int num_blocks, int num_host_blocks, int block_size,
                          pkv_alloc** out) {
    if (!out || num_blocks <= 0 || num_host_blocks < 0 || block_size <= 0) return PKV_EINVAL;
    pkv_alloc* a = new (std::nothrow) pkv_alloc();
    if (!a) return PKV_ENOMEM;
    a->num_blocks = num_blocks;
    a->num_host_blocks = num_host_blocks;
    a->block_size = block_size;
    try {
        a->free_stack.resize(num_blocks);
        for (int32_t i = 0; i < num_blocks; ++i) a->free_stack[i] = num_blocks - 1 - i;
        a->host_free_stack.resize(num_host_blocks);
        for (int32_t i = 0; i < num_host_blocks; ++i)
            a->host_free_stack[i] = num_host_blocks - 1 - i;
        a->ref.assign(num_blocks, 0);
    } catch (...) {
        delete a;
        return PKV_ENOMEM;
    }
    *out = a;
    return PKV_OK;
}

int pkv_alloc_create(int num_blocks, int block_size, pkv_alloc** out) {
    return pkv_alloc_create_swap(num_blocks, 0, block_size, out);
}

void pkv_alloc_destroy(pkv_alloc* a) { delete a; }

int pkv_alloc_add_seq(pkv_alloc* a, int64_t seq_id, int num_tokens) {
    if (!a || num_tokens < 0) return PKV_EINVAL;
    if (a->seqs.count(seq_id)) return PKV_EEXIST;
    const int64_t need = ((int64_t)num_tokens + a->block_size - 1) / a->block_size;
    if (need > a->available()) return PKV_ENOMEM;
    pkv_alloc::Seq s;
    s.len = num_tokens;
    s.table.reserve(need);
    for (int64_t i = 0; i < need; ++i) s.table.push_back(a->take());
    a->logical_tokens += num_tokens;
    a->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

int pkv_alloc_fork(pkv_alloc* a, int64_t parent, int64_t child) {
    if (!a) return PKV_EINVAL;
    auto it = a->seqs.find(parent);
    if (it == a->seqs.end()) return PKV_ENOSEQ;
    if (a->seqs.count(child)) return PKV_EEXIST;
    if (it->second.swapped) return PKV_EINVAL;
    pkv_alloc::Seq s = it->second;  // copy of table and length
    for (int32_t b : s.table)
        if (b >= 0) a->add_ref(b);
    a->logical_tokens += s.len;
    a->seqs.emplace(child, std::move(s));
    return PKV_OK;
}

int pkv_alloc_append_slot(pkv_alloc* a, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                          int32_t* cow_dst) {
    if (!a || !slot || !cow_src || !cow_dst) return PKV_EINVAL;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ENOSEQ;
    pkv_alloc::Seq& s = it->second;
    if (s.swapped) return PKV_EINVAL;
    const int64_t off = s.len % a->block_size;
    int32_t src = -1, dst = -1;
    if (off == 0) {
        if (a->available() == 0) return PKV_ENOMEM;
        s.table.push_back(a->take());
    } else if (a->ref[s.table.back()] > 1) {
        if (a->available() == 0) return PKV_ENOMEM;
        dst = a->take();
        src = s.table.back();
        a->drop_ref(src);  // stays > 0: another sequence still holds it
        s.table.back() = dst;
    }
    *slot = (int64_t)s.table.back() * a->block_size + off;
    *cow_src = src;
    *cow_dst = dst;
    s.len += 1;
    a->logical_tokens += 1;
    return PKV_OK;
}

int pkv_alloc_append_slots(pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* slots,
                           int32_t* cow_pairs, int* num_cow, int* num_done) {
    if (!a || n < 0 || (n > 0 && (!seq_ids || !slots || !cow_pairs)) || !num_cow ||
        !num_done)
        return PKV_EINVAL;
    *num_cow = 0;
    *num_done = 0;
    for (int i = 0; i < n; ++i) {
        int32_t src, dst;
        int rc = pkv_alloc_append_slot(a, seq_ids[i], &slots[i], &src, &dst);
        if (rc != PKV_OK) return rc;
        if (src >= 0) {
            cow_pairs[2 * *num_cow] = src;
            cow_pairs[2 * *num_cow + 1] = dst;
            ++*num_cow;
        }
        ++*num_done;
    }
    return PKV_OK;
}

int pkv_alloc_free_seq(pkv_alloc* a, int64_t seq_id) {
    if (!a) return PKV_EINVAL;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ENOSEQ;
    if (it->second.swapped) {
        for (int32_t h : it->second.table)
            if (h >= 0) a->host_free_stack.push_back(h);
        --a->swapped_seqs;
    } else {
        for (int32_t b : it->second.table)
            if (b >= 0) a->drop_ref(b);
    }
    a->logical_tokens -= it->second.len;
    a->seqs.erase(it);
    return PKV_OK;
}

int pkv_alloc_seq_len(const pkv_alloc* a, int64_t seq_id, int* len) {
    if (!a || !len) return PKV_EINVAL;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ENOSEQ;
    *len = (int)it->second.len;
    return PKV_OK;
}

int pkv_alloc_block_table(const pkv_alloc* a, int64_t seq_id, int32_t* out, int capacity,
                          int* n_out) {
    if (!a || !n_out || capacity < 0 || (capacity > 0 && !out)) return PKV_EINVAL;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ENOSEQ;
    const auto& t = it->second.table;
    *n_out = (int)t.size();
    if ((int64_t)t.size() > capacity) return PKV_EBOUNDS;
    for (size_t i = 0; i < t.size(); ++i) out[i] = t[i];
    return PKV_OK;
}

int pkv_alloc_build_block_tables(const pkv_alloc* a, const int64_t* seq_ids, int n,
                                 int32_t* tables, int max_blocks, int32_t fill,
                                 int32_t* context_lens) {
    if (!a || n < 0 || max_blocks < 0 ||
        (n > 0 && (!seq_ids || !context_lens || (max_blocks > 0 && !tables))))
        return PKV_EINVAL;
    for (int i = 0; i < n; ++i) {  // check everything before writing anything
        auto it = a->seqs.find(seq_ids[i]);
        if (it == a->seqs.end()) return PKV_ENOSEQ;
        if (it->second.swapped) return PKV_EINVAL;
        if ((int64_t)it->second.table.size() > max_blocks) return PKV_EBOUNDS;
    }
    for (int i = 0; i < n; ++i) {
        const auto& s = a->seqs.find(seq_ids[i])->second;
        int32_t* row = tables + (int64_t)i * max_blocks;
        size_t j = 0;
        for (; j < s.table.size(); ++j) row[j] = s.table[j];
        for (; j < (size_t)max_blocks; ++j) row[j] = fill;
        context_lens[i] = (int32_t)s.len;
    }
    return PKV_OK;
}

int pkv_alloc_refcount(const pkv_alloc* a, int32_t block, int* out) {
    if (!a || !out) return PKV_EINVAL;
    if (block < 0 || block >= a->num_blocks) return PKV_EBOUNDS;
    *out = a->ref[block];
    return PKV_OK;
}

int pkv_alloc_swap_out(pkv_alloc* a, int64_t seq_id, int32_t* pairs, int capacity,
                       int* num_pairs) {
    if (!a || !num_pairs || capacity < 0 || (capacity > 0 && !pairs)) return PKV_EINVAL;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ENOSEQ;
    pkv_alloc::Seq& s = it->second;
    if (s.swapped) return PKV_EINVAL;
    int n = 0;
    for (int32_t b : s.table) n += b >= 0;  // entries released by a sliding window stay -1
    *num_pairs = n;
    if (n > capacity) return PKV_EBOUNDS;
    if (n > (int)a->host_free_stack.size()) return PKV_ENOMEM;
    int k = 0;
    for (int32_t& b : s.table) {
        if (b < 0) continue;
        const int32_t h = a->host_free_stack.back();
        a->host_free_stack.pop_back();
        pairs[2 * k] = b;
        pairs[2 * k + 1] = h;
        ++k;
        a->drop_ref(b);  // other holders keep a shared block on the device
        b = h;
    }
    s.swapped = true;
    ++a->swapped_seqs;
    return PKV_OK;
}

int pkv_alloc_swap_in(pkv_alloc* a, int64_t seq_id, int32_t* pairs, int capacity,
                      int* num_pairs) {
    if (!a || !num_pairs || capacity < 0 || (capacity > 0 && !pairs)) return PKV_EINVAL;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ENOSEQ;
    pkv_alloc::Seq& s = it->second;
    if (!s.swapped) return PKV_EINVAL;
    int n = 0;
    for (int32_t h : s.table) n += h >= 0;
    *num_pairs = n;
    if (n > capacity) return PKV_EBOUNDS;
    if (n > a->available()) return PKV_ENOMEM;
    int k = 0;
    for (int32_t& h : s.table) {
        if (h < 0) continue;
        const int32_t d = a->take();
        pairs[2 * k] = h;
        pairs[2 * k + 1] = d;
        ++k;
        a->host_free_stack.push_back(h);
        h = d;
    }
    s.swapped = false;
    --a->swapped_seqs;
    return PKV_OK;
}

int pkv_alloc_slide_window(pkv_alloc* a, int64_t seq_id, int window, int* released) {
    if (!a || !released || window <= 0) return PKV_EINVAL;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ENOSEQ;
    pkv_alloc::Seq& s = it->second;
    if (s.swapped) return PKV_EINVAL;
    *released = 0;
    // block j holds tokens [j*bs, (j+1)*bs): gone once (j+1)*bs <= len - window
    const int64_t keep_from = s.len - window;
    for (size_t j = 0; j < s.table.size() && (int64_t)(j + 1) * a->block_size <= keep_from; ++j) {
        if (s.table[j] < 0) continue;
        a->drop_ref(s.table[j]);
        s.table[j] = -1;
        ++*released;
    }
    return PKV_OK;
}

int pkv_alloc_add_seq_prefix(pkv_alloc* a, int64_t seq_id, const int32_t* tokens,
                             int num_tokens, int* cached_tokens) {
    if (!a || num_tokens < 0 || (num_tokens > 0 && !tokens) || !cached_tokens) return PKV_EINVAL;
    if (a->seqs.count(seq_id)) return PKV_EEXIST;
    try {
        a->cache_init();
    } catch (...) {
        return PKV_ENOMEM;
    }
    const int bs = a->block_size;
    const int64_t nfull = num_tokens / bs;
    const int64_t need = ((int64_t)num_tokens + bs - 1) / bs;
    // 1. the registered prefix (read only)
    std::vector<int32_t> hits;
    int64_t parent = 0, evictable_hits = 0;
    for (int64_t j = 0; j < nfull; ++j) {
        const int32_t b = a->lookup(parent, tokens + j * bs);
        if (b < 0) break;
        hits.push_back(b);
        evictable_hits += a->ref[b] == 0;
        parent = a->reg_id[b];
    }
    const int64_t fresh = need - (int64_t)hits.size();
    if (fresh > a->available() - evictable_hits) return PKV_ENOMEM;
    // 2. take the hits, then allocate (and register the full blocks among) the rest
    pkv_alloc::Seq s;
    s.len = num_tokens;
    try {
        s.table.reserve(need);
        a->reg_map.reserve(a->reg_map.size() + nfull);
    } catch (...) {
        return PKV_ENOMEM;
    }
    for (int32_t b : hits) {
        if (a->ref[b] == 0) {
            a->ev_remove(b);
            a->ref[b] = 1;
            ++a->used_blocks;
            ++a->refcount_sum;
        } else {
            a->add_ref(b);
        }
        s.table.push_back(b);
    }
    for (int64_t j = (int64_t)hits.size(); j < need; ++j) {
        const int32_t b = a->take();
        s.table.push_back(b);
        if (j < nfull) {
            const int32_t* tk = tokens + j * bs;
            a->reg_id[b] = a->next_reg++;
            a->reg_parent[b] = parent;
            std::memcpy(&a->reg_tokens[(size_t)b * bs], tk, sizeof(int32_t) * bs);
            a->reg_map.emplace(pkv_alloc::key_hash(parent, tk, bs), b);
            ++a->cached_blocks;
            parent = a->reg_id[b];
        }
    }
    *cached_tokens = (int)(hits.size() * bs);
    a->logical_tokens += num_tokens;
    a->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

int pkv_alloc_cache_stats(const pkv_alloc* a, int32_t* cached_blocks, int32_t* evictable_blocks) {
    if (!a || !cached_blocks || !evictable_blocks) return PKV_EINVAL;
    *cached_blocks = a->cached_blocks;
    *evictable_blocks = a->evictable;
    return PKV_OK;
}

int pkv_alloc_evictable_list(const pkv_alloc* a, int32_t* out, int capacity, int* n_out) {
    if (!a || !n_out || capacity < 0 || (capacity > 0 && !out)) return PKV_EINVAL;
    *n_out = a->evictable;
    if (a->evictable > capacity) return PKV_EBOUNDS;
    int k = 0;
    for (int32_t b = a->ev_head; b >= 0; b = a->ev_next[b]) out[k++] = b;
    return PKV_OK;
}

int pkv_alloc_is_swapped(const pkv_alloc* a, int64_t seq_id, int* swapped) {
    if (!a || !swapped) return PKV_EINVAL;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ENOSEQ;
    *swapped = it->second.swapped ? 1 : 0;
    return PKV_OK;
}

int pkv_alloc_stats(const pkv_alloc* a, pkv_alloc_stats_t* out) {
    if (!a || !out) return PKV_EINVAL;
    out->num_host_blocks = a->num_host_blocks;
    out->free_host_blocks = (int32_t)a->host_free_stack.size();
    out->swapped_seqs = a->swapped_seqs;
    out->num_blocks = a->num_blocks;
    out->block_size = a->block_size;
    out->free_blocks = (int32_t)a->free_stack.size();
    out->used_blocks = a->used_blocks;
    out->shared_blocks = a->shared_blocks;
    out->num_seqs = (int32_t)a->seqs.size();
    out->refcount_sum = a->refcount_sum;
    out->logical_tokens = a->logical_tokens;
    return PKV_OK;
}

int pkv_alloc_free_list(const pkv_alloc* a, int32_t* out, int capacity, int* n_out) {
    if (!a || !n_out || capacity < 0 || (capacity > 0 && !out)) return PKV_EINVAL;
    const auto& fs = a->free_stack;
    *n_out = (int)fs.size();
    if ((int64_t)fs.size() > capacity) return PKV_EBOUNDS;
    for (size_t i = 0; i < fs.size(); ++i) out[i] = fs[fs.size() - 1 - i];
    return PKV_OK;
}

}  // extern "C"
