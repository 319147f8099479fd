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
