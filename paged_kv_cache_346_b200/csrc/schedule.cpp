// Host-side schedule order for the decode: longest sequences first.
//
// CTAs are dispatched in grid order as SMs free up.  When a long partition is
// dispatched last, a few SMs keep working after all others are done; putting
// the longest sequences first leaves only short work for the end of the grid.
#include <algorithm>
#include <cstdint>
#include <numeric>
#include <vector>

#include "pagedkv.h"

extern "C" int pkv_decode_schedule_order(const int32_t* context_lens, int num_seqs,
                                         int32_t* order_out) {
    if (num_seqs < 0 || (num_seqs > 0 && (!context_lens || !order_out))) return PKV_EINVAL;
    std::iota(order_out, order_out + num_seqs, 0);
    std::stable_sort(order_out, order_out + num_seqs, [&](int32_t x, int32_t y) {
        return context_lens[x] > context_lens[y];
    });
    return PKV_OK;
}

// The decode's work list: every (sequence, partition) pair with tokens,
// longest partition first.  The partition count mirrors the kernels' span
// (decode_common.cuh seq_span without a shared prefix): attended tokens
// [lo, L), partitions from the block holding lo.
extern "C" int pkv_decode_schedule_items(const int32_t* context_lens, int num_seqs,
                                         int block_size, int partition_size,
                                         int sliding_window, int32_t* items_out,
                                         int item_capacity, int* num_items) {
    if (num_seqs < 0 || block_size <= 0 || partition_size < 64 || partition_size > 8192 ||
        partition_size % 64 != 0 || sliding_window < 0 || item_capacity < 0 || !num_items ||
        (num_seqs > 0 && !context_lens))
        return PKV_EINVAL;
    struct Item {
        int32_t len, seq, part;
    };
    std::vector<Item> v;
    v.reserve((size_t)num_seqs);
    for (int b = 0; b < num_seqs; ++b) {
        const int64_t L = context_lens[b];
        if (L < 0) return PKV_EINVAL;
        const int64_t lo = (sliding_window > 0 && L > sliding_window) ? L - sliding_window : 0;
        const int64_t base = lo - lo % block_size;
        const int64_t n = L > 0 ? (L - base + partition_size - 1) / partition_size : 1;
        for (int64_t p = 0; p < n; ++p)
            v.push_back({(int32_t)std::min<int64_t>(partition_size, L - base - p * partition_size),
                         b, (int32_t)p});
    }
    if (v.size() > (size_t)INT32_MAX) return PKV_EINVAL;
    *num_items = (int)v.size();
    if ((int64_t)v.size() > item_capacity) return PKV_EBOUNDS;
    if (!v.empty() && !items_out) return PKV_EINVAL;
    std::stable_sort(v.begin(), v.end(), [](const Item& x, const Item& y) {
        return x.len > y.len;  // ties keep (sequence, partition) order
    });
    for (size_t i = 0; i < v.size(); ++i) {
        items_out[2 * i] = v[i].seq;
        items_out[2 * i + 1] = v[i].part;
    }
    return PKV_OK;
}
