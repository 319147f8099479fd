// Host-side work plan for the planned decode: the attended tokens of every
// (sequence, KV head, tile of query heads) unit are cut into pieces of at
// most piece_tokens tokens, and the pieces are spread over a fixed number of
// persistent CTAs, largest first, each to the CTA with the least work so far
// (longest-processing-time-first list scheduling).  Every warp of a CTA
// leaves a partial softmax state per piece in its own workspace slot; the
// warp that completes a unit's count merges them.
//
// Plan layout (int32 words; the same struct the kernels read):
//   header      PKV_PLAN_HEADER_WORDS words (pkv_decode_plan_header)
//   cta_begin   [num_ctas + 1]: items of CTA c are [cta_begin[c], cta_begin[c+1])
//   items       [num_items][PKV_PLAN_ITEM_WORDS]: b, y, t0, t1, mask_lo, unit,
//               unit's first slot, unit's pieces, this piece's index, 0 ...
//               (y = KV head * head_chunks + chunk; tokens [t0, t1) of b;
//               mask_lo tokens at the start lie before a sliding window;
//               unit = its (sequence, y) in schedule order; warp w of the
//               piece's CTA writes slot first + index * warps_per_cta + w)
#include <algorithm>
#include <cstdint>
#include <numeric>
#include <queue>
#include <vector>

#include "pagedkv.h"

namespace {

int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

extern "C" int pkv_decode_plan(const int32_t* context_lens, const int32_t* seq_order,
                               int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int sliding_window, int num_ctas,
                               int piece_tokens, int32_t* plan, size_t plan_capacity,
                               pkv_decode_plan_header* info) {
    if (num_seqs < 0 || num_seqs > 65535 || num_q_heads <= 0 || num_kv_heads <= 0 ||
        (head_dim != 128 && head_dim != 256) ||
        num_q_heads % num_kv_heads != 0 || num_q_heads / num_kv_heads > 16 ||
        (block_size != 16 && block_size != 32 && block_size != 64) || sliding_window < 0 ||
        num_ctas <= 0 || num_ctas > (1 << 20) || piece_tokens < 0 ||
        (piece_tokens != 0 && (piece_tokens % 64 != 0 || piece_tokens > 8192)) || !info ||
        (num_seqs > 0 && !context_lens))
        return PKV_EINVAL;
    // the tensor-core kernels' tiles: 8 query heads (groups of up to 8), else 16
    const int G = num_q_heads / num_kv_heads;
    const int heads_per_cta = G <= 8 ? 8 : 16;
    const int head_chunks = (G + heads_per_cta - 1) / heads_per_cta;
    // warps per CTA of the planned kernel (two for one live head at head_dim
    // 128, else four); a warp takes at most 32 slices of 16 tokens of a piece
    const int warps = head_dim == 128 && G == 1 ? 2 : 4;
    const int max_piece = 32 * 16 * warps;
    if (piece_tokens > max_piece) return PKV_EINVAL;
    const int64_t units_per_seq = (int64_t)num_kv_heads * head_chunks;
    static_assert(sizeof(pkv_decode_plan_header) == PKV_PLAN_HEADER_WORDS * 4, "header words");
    // attended span of each sequence: [base, L), base block aligned
    std::vector<int32_t> order(num_seqs), base(num_seqs), lo(num_seqs);
    int64_t total = 0;
    for (int z = 0; z < num_seqs; ++z) {
        const int b = seq_order ? seq_order[z] : z;
        if (b < 0 || b >= num_seqs) return PKV_EINVAL;
        order[z] = b;
        const int L = context_lens[b];
        if (L < 0) return PKV_EINVAL;
        const int l0 = sliding_window > 0 && L > sliding_window ? L - sliding_window : 0;
        lo[b] = l0;
        base[b] = l0 - l0 % block_size;
        total += (int64_t)(L - base[b]) * units_per_seq;
    }
    // pieces: about a CTA's share, a multiple of 64 tokens (so every piece
    // starts on a block), 256 .. the kernel's largest piece
    int pt = piece_tokens;
    if (pt == 0) {
        const int64_t share = ceil_div64(total, (int64_t)num_ctas);
        pt = (int)std::min<int64_t>(max_piece, std::max<int64_t>(256, ceil_div64(share, 64) * 64));
    }
    struct Piece {
        int32_t b, y, t0, t1, mask_lo, unit, slot0, np, index;
        int64_t cost;
    };
    std::vector<Piece> pieces;
    int64_t slots = 0;
    int32_t split_units = 0, unit = 0;
    for (int z = 0; z < num_seqs; ++z) {
        const int b = order[z];
        const int L = context_lens[b];
        const int n = L - base[b];
        const int np = n > 0 ? (int)ceil_div64(n, pt) : 1;
        for (int64_t y = 0; y < units_per_seq; ++y, ++unit) {
            for (int p = 0; p < np; ++p) {
                Piece q;
                q.b = b;
                q.y = (int32_t)y;
                q.t0 = base[b] + p * pt;
                q.t1 = std::min(L, q.t0 + pt);
                q.mask_lo = p == 0 ? lo[b] - base[b] : 0;
                q.unit = unit;
                q.slot0 = (int32_t)slots;
                q.np = np;
                q.index = p;
                // cost in tokens, plus a fixed share for the piece's partial
                // state and merge
                q.cost = (int64_t)(q.t1 - q.t0) + 32;
                pieces.push_back(q);
            }
            slots += (int64_t)np * warps;
            if (np > 1) ++split_units;
        }
    }
    if (slots > INT32_MAX) return PKV_EINVAL;
    // largest first onto the least loaded CTA (ties: lower CTA index, then
    // batch order)
    std::vector<int32_t> idx(pieces.size());
    std::iota(idx.begin(), idx.end(), 0);
    std::stable_sort(idx.begin(), idx.end(),
                     [&](int32_t x, int32_t y) { return pieces[x].cost > pieces[y].cost; });
    using Slot = std::pair<int64_t, int32_t>;  // (load, cta)
    std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
    for (int32_t c = 0; c < num_ctas; ++c) heap.push({0, c});
    std::vector<int32_t> owner(pieces.size());
    int64_t max_load = 0;
    for (int32_t i : idx) {
        Slot s = heap.top();
        heap.pop();
        owner[i] = s.second;
        s.first += pieces[i].cost;
        max_load = std::max(max_load, s.first);
        heap.push(s);
    }
    const int64_t num_items = (int64_t)pieces.size();
    const size_t words = PKV_PLAN_HEADER_WORDS + (size_t)num_ctas + 1 +
                         (size_t)num_items * PKV_PLAN_ITEM_WORDS;
    if (words > (size_t)INT32_MAX) return PKV_EINVAL;
    pkv_decode_plan_header h = {};
    h.magic = PKV_PLAN_MAGIC;
    h.num_ctas = num_ctas;
    h.num_items = (int32_t)num_items;
    h.num_merges = split_units;
    h.num_slots = (int32_t)slots;
    h.num_seqs = num_seqs;
    h.num_q_heads = num_q_heads;
    h.num_kv_heads = num_kv_heads;
    h.heads_per_cta = heads_per_cta;
    h.head_chunks = head_chunks;
    h.block_size = block_size;
    h.sliding_window = sliding_window;
    h.piece_tokens = pt;
    h.words = (int32_t)words;
    h.max_cta_tokens = (int32_t)std::min<int64_t>(max_load, INT32_MAX);
    h.warps_per_cta = warps;
    *info = h;
    if (!plan) return PKV_OK;  // size query
    if (plan_capacity < words) return PKV_EBOUNDS;
    int32_t* out = plan;
    std::copy(reinterpret_cast<const int32_t*>(&h),
              reinterpret_cast<const int32_t*>(&h) + PKV_PLAN_HEADER_WORDS, out);
    int32_t* cta_begin = out + PKV_PLAN_HEADER_WORDS;
    int32_t* items = cta_begin + num_ctas + 1;
    // items grouped by CTA, each CTA's in the order they were assigned
    std::vector<int32_t> count(num_ctas + 1, 0);
    for (int32_t i : idx) ++count[owner[i] + 1];
    for (int c = 0; c < num_ctas; ++c) count[c + 1] += count[c];
    std::copy(count.begin(), count.end(), cta_begin);
    for (int32_t i : idx) {
        int32_t* it = items + (int64_t)count[owner[i]]++ * PKV_PLAN_ITEM_WORDS;
        const Piece& q = pieces[i];
        std::fill(it, it + PKV_PLAN_ITEM_WORDS, 0);
        it[0] = q.b;
        it[1] = q.y;
        it[2] = q.t0;
        it[3] = q.t1;
        it[4] = q.mask_lo;
        it[5] = q.unit;
        it[6] = q.slot0;
        it[7] = q.np;
        it[8] = q.index;
    }
    return PKV_OK;
}
