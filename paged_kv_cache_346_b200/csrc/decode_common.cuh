// Arguments and the log-sum-exp reduce shared by both decode kernels.
#pragma once

#include <cmath>

#include "context_cache.h"
#include "device_common.cuh"

namespace pkv {

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

struct DecodeArgs {
    void* out;                    // [B, Hq, D] T
    const void* q;                // [B, Hq, D] T
    const void* k_cache;          // [N, Hkv, BS, D] T
    const void* v_cache;
    const int32_t* block_tables;  // [B, max_blocks_per_seq]
    const int32_t* context_lens;  // [B]
    const int32_t* seq_order;     // [B] schedule order (CTA z takes sequence seq_order[z]), or null
    const int32_t* items;         // [num_items][2] work list: CTA z takes (sequence, partition), or null
    const float* k_scale;         // scales of E4M3 K / V pages, or null: [Hkv], or
    const float* v_scale;         // [num_blocks, Hkv] when scale_per_block
    // shared-prefix decode: tokens [0, seq_start[b]) of sequence b were
    // attended by the group pass (whole blocks shared with the other members
    // of its group); null = every sequence starts at token 0
    const int32_t* seq_start;     // [B] or null
    const int32_t* group_members; // [num_groups][group_stride] batch indices, -1 padded
    float* ws_o;                  // [B, Hq, ws_slots, D] partial outputs (normalised)
    float* ws_ml;                 // [B, Hq, ws_slots, 2] (m in log2 units, l)
    unsigned int* status;
    int num_seqs;
    int num_items;                // work-list length (items only)
    int num_q_heads;
    int num_kv_heads;
    int group;                    // Hq / Hkv
    int head_chunks;              // CTAs per KV head along the query group
    int max_blocks_per_seq;
    int num_blocks;
    int max_tokens;               // max_blocks_per_seq * BS
    int partition_size;           // tokens per partition
    int max_partitions;           // grid.x = ceil(longest attended span / partition_size)
    int ws_slots;                 // partial results per row in the workspace
    int group_stride;             // group_members row length
    int after_groups;             // launched as a programmatic dependent of the group pass
    int block_size;
    int window;                   // sliding window in tokens, 0 = attend to the whole context
    int scale_per_block;          // E4M3 scales per (block, KV head) page
    float scale_log2;             // scale * log2(e): logits are kept in base 2
};

// The sequence this CTA works on: grid z, through the schedule order when one
// is given (-1: a bad order entry, flagged once).
__device__ __forceinline__ int scheduled_seq(const DecodeArgs& a, int z, bool report) {
    if (!a.seq_order) return z;
    const int b = a.seq_order[z];
    if ((unsigned)b >= (unsigned)a.num_seqs) {
        if (report) flag(a.status, PKV_DEV_BAD_ORDER);
        return -1;
    }
    return b;
}

// The (sequence, partition) this CTA works on: with a work list, item z of
// it (grid x is 1); else grid z through the schedule order and partition
// grid x.  b = -1: a bad order entry or item (flagged by the CTA of head
// chunk 0).
struct CtaUnit {
    int b, part;
};
__device__ __forceinline__ CtaUnit cta_unit(const DecodeArgs& a, int tid) {
    if (a.items) {
        const int b = a.items[2 * blockIdx.z], part = a.items[2 * blockIdx.z + 1];
        if ((unsigned)b >= (unsigned)a.num_seqs || part < 0) {
            if (tid == 0 && blockIdx.y == 0) flag(a.status, PKV_DEV_BAD_ORDER);
            return {-1, 0};
        }
        return {b, part};
    }
    const int part = blockIdx.x;
    return {scheduled_seq(a, blockIdx.z, tid == 0 && part == 0 && blockIdx.y == 0), part};
}

// The decode grid: (partitions, KV heads x head chunks, sequences), or one
// CTA per (item, KV head x head chunk) with a work list.
__host__ __forceinline__ dim3 decode_grid(const DecodeArgs& a) {
    return a.items ? dim3(1, a.num_kv_heads * a.head_chunks, a.num_items)
                   : dim3(a.max_partitions, a.num_kv_heads * a.head_chunks, a.num_seqs);
}

// Length of sequence b as the kernels use it: negative or too long lengths
// are clamped (and flagged once, by the CTA that owns partition 0, head 0).
__device__ __forceinline__ int seq_len(const DecodeArgs& a, int b, bool report) {
    int L = a.context_lens[b];
    if (L < 0 || L > a.max_tokens) {
        if (report) flag(a.status, PKV_DEV_BAD_LEN);
        L = L < 0 ? 0 : a.max_tokens;
    }
    return L;
}

// The tokens a sequence attends to and how they are cut into partitions.
// Without a window: [0, L).  With a window of W tokens: [lo, L), lo =
// max(0, L - W) ("pagedattention vllm" §Advanced Features: sliding-window
// models keep only the recent blocks); the partitions then start at the
// block holding lo (base), and the first lo - base tokens are masked.
// With a shared prefix of S tokens (seq_start), the partitions cover [S, L)
// and their partial results take workspace slots ceil(S / P) onwards, after
// the group pass's slots of the prefix.
struct Span {
    int L;       // sequence length
    int lo;      // first attended token
    int base;    // first token of partition 0 (block aligned)
    int np;      // partitions
    int slot0;   // workspace slot of partition 0
    bool direct; // one partial result in all: written straight to out
};

__device__ __forceinline__ Span seq_span(const DecodeArgs& a, int b, bool report) {
    Span sp;
    sp.L = seq_len(a, b, report);
    sp.lo = (a.window > 0 && sp.L > a.window) ? sp.L - a.window : 0;
    sp.slot0 = 0;
    if (a.seq_start) {
        int st = a.seq_start[b];
        // the prefix must be whole blocks of the sequence, within the slots
        // the group pass has (ws_slots - max_partitions of them)
        if (st < 0 || st > sp.L || st % a.block_size != 0 ||
            (st + a.partition_size - 1) / a.partition_size > a.ws_slots - a.max_partitions) {
            if (report) flag(a.status, PKV_DEV_BAD_GROUP);
            st = 0;
        }
        sp.lo = max(sp.lo, st);
        sp.slot0 = (st + a.partition_size - 1) / a.partition_size;
    }
    sp.base = sp.lo - sp.lo % a.block_size;
    int n = (sp.L - sp.base + a.partition_size - 1) / a.partition_size;
    if (n > a.max_partitions) {
        if (report) flag(a.status, PKV_DEV_BAD_LEN);
        n = a.max_partitions;
    }
    sp.np = n;
    sp.direct = sp.slot0 == 0 && n <= 1;
    return sp;
}

// The shared prefix of a group as the group pass cuts it: tokens [0, S),
// S = seq_start of the group's first member b (whole blocks of b), in
// partitions of partition_size whose partial results take workspace slots
// 0, 1, ... of every member row.  A prefix that is not whole blocks of b or
// needs more than max_partitions (the group pass's grid) is flagged and left
// out (S = 0: the regular pass then takes the whole sequence).
__device__ __forceinline__ Span group_span(const DecodeArgs& a, int b, bool report) {
    Span sp;
    const int L = seq_len(a, b, false);
    int st = a.seq_start[b];
    if (st < 0 || st > L || st % a.block_size != 0 ||
        (st + a.partition_size - 1) / a.partition_size > a.max_partitions) {
        if (report) flag(a.status, PKV_DEV_BAD_GROUP);
        st = 0;
    }
    sp.L = st;
    sp.lo = sp.base = 0;
    sp.np = (st + a.partition_size - 1) / a.partition_size;
    sp.slot0 = 0;
    sp.direct = false;
    return sp;
}

// The table slice of a partition goes to shared memory.  For partition 0 (the
// only CTA of every sequence up to one partition long) the first entries are
// requested before the sequence length is known, so the two reads overlap
// instead of following each other; later partitions read their slice after
// the length check, since most of those CTAs find their sequence too short
// and leave at once.
struct TablePrefetch {
    int32_t v;
    bool ok;
};

__device__ __forceinline__ TablePrefetch table_prefetch(const DecodeArgs& a, int b, int part,
                                                        int blocks_per_part, int tid) {
    // Partition part starts at block part * blocks_per_part, so its table
    // slice is read alongside the length, not after it.  (With a sliding
    // window or a shared prefix the partitions start at a block known only
    // after the length is read: no early read then.)  An entry past the
    // sequence's blocks is read but never used.
    const int64_t i = (int64_t)part * blocks_per_part + tid;
    TablePrefetch pf{0, a.window == 0 && !a.seq_start && tid < blocks_per_part &&
                            i < a.max_blocks_per_seq};
    if (pf.ok) pf.v = a.block_tables[(int64_t)b * a.max_blocks_per_seq + i];
    return pf;
}

__device__ __forceinline__ void table_hoist(const DecodeArgs& a, int b, int first_block, int nblk,
                                            TablePrefetch pf, int32_t* s_tab, int tid,
                                            int nthreads) {
    const int32_t* trow = a.block_tables + (int64_t)b * a.max_blocks_per_seq + first_block;
    for (int i = tid; i < nblk; i += nthreads) {
        int32_t p = (pf.ok && i == tid) ? pf.v : trow[i];
        // an entry outside [0, num_blocks) is flagged and replaced by block 0,
        // so no page load leaves the pool (checked here, in parallel, rather
        // than by the thread that issues the copies: measured 8-10 % faster)
        if ((unsigned)p >= (unsigned)a.num_blocks) {
            flag(a.status, PKV_DEV_BAD_BLOCK);
            p = 0;
        }
        s_tab[i] = p;
    }
}

// Shared-memory layout of the warp merge at the end of a partition: per warp
// and head an accumulator row (pitch D + 4 floats, so rows written by
// different lanes fall in different banks), then m, l and the per-warp scale.
template <int D, int NH, int NW>
struct MergeArea {
    static constexpr int RP = D + 4;
    static constexpr int FLOATS = NW * NH * RP + 3 * NW * NH;
    static constexpr int BYTES = FLOATS * 4;
};

// Merge NW parked warp states (acc rows, m, l in `red`, written and
// synchronised by the caller) of nh heads and write the output rows (direct:
// the row's only partial result) or the partial (m, l, o) to the workspace.
// Tile row hh is output row row_of(hh) = sequence * Hq + head, and partial
// row part_of(hh) of the workspace (ws_o rows of D floats, ws_ml rows of 2);
// rows with row_of(hh) < 0 are skipped.  All threads of the CTA take part.
// Per head: M = max_w m_w, den = sum_w 2^(m_w - M) l_w,
// o = sum_w (2^(m_w - M) / den) acc_w.
template <typename T, int D, int NH, int NW, typename RowOf, typename PartOf>
__device__ __forceinline__ void merge_warps_and_store(const DecodeArgs& a, float* red,
                                                      RowOf row_of, PartOf part_of, int nh,
                                                      bool direct, int tid, int nthreads) {
    using A = MergeArea<D, NH, NW>;
    float* red_m = red + NW * NH * A::RP;
    float* red_l = red_m + NW * NH;
    float* red_s = red_l + NW * NH;
    T* out = reinterpret_cast<T*>(a.out);
    if constexpr (NH == 1) {
        // one head: every thread folds the NW warp states for its elements
        // (measured faster than a serial scale step plus a barrier here)
        (void)red_s;
        const int64_t row = row_of(0);
        for (int d = tid; d < D; d += nthreads) {
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w]);
            float num = 0.f, den = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = exp2f(red_m[w] - M);  // 0 for a warp with no tokens
                num = fmaf(f, red[w * A::RP + d], num);
                den = fmaf(f, red_l[w], den);
            }
            if (direct) {
                out[row * D + d] = Elem<T>::from_f32(num / den);
            } else {
                const int64_t pr = part_of(0);
                a.ws_o[pr * D + d] = num / den;
                if (d == 0) {
                    a.ws_ml[pr * 2] = M;
                    a.ws_ml[pr * 2 + 1] = den;
                }
            }
        }
        return;
    } else {
        // several heads: the per-warp scale factors of each head once, then
        // one fused multiply-add per warp and element
        if (tid < nh) {
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w * NH + tid]);
            float f[NW], den = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                f[w] = exp2f(red_m[w * NH + tid] - M);  // 0 for a warp with no tokens
                den = fmaf(f[w], red_l[w * NH + tid], den);
            }
            const float inv = 1.f / den;
#pragma unroll
            for (int w = 0; w < NW; ++w) red_s[w * NH + tid] = f[w] * inv;
            if (!direct && row_of(tid) >= 0) {
                const int64_t pr = part_of(tid);
                a.ws_ml[pr * 2] = M;
                a.ws_ml[pr * 2 + 1] = den;
            }
        }
        __syncthreads();
        for (int i = tid; i < nh * D; i += nthreads) {
            const int hh = i / D, d = i - hh * D;
            const int64_t row = row_of(hh);  // < 0: a row the group pass skips
            if (row < 0) continue;
            float o = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w)
                o = fmaf(red_s[w * NH + hh], red[(w * NH + hh) * A::RP + d], o);
            if (direct)
                out[row * D + d] = Elem<T>::from_f32(o);
            else
                a.ws_o[part_of(hh) * D + d] = o;
        }
    }
}

// A decode kernel's griddepcontrol.wait: before its first read of pages (or
// scales) and its first global write.  The regular pass after the group
// pass waits only as it leaves (GroupPassWait).
__device__ __forceinline__ void pdl_wait_before_pages(const DecodeArgs& a) {
    if (!a.after_groups) pdl_wait_primary();
}

// The regular pass of the shared-prefix decode may start while the group
// pass still runs (it is a programmatic dependent of it; neither reads the
// other's results).  The log-sum-exp reduce, a programmatic dependent of the
// regular pass, reads both: so no CTA of the regular pass leaves before the
// group pass has completed and its writes are visible.  Held by every CTA of
// the regular pass; releases at each exit.
struct GroupPassWait {
    const DecodeArgs& a;
    __device__ __forceinline__ ~GroupPassWait() {
        if (a.after_groups) pdl_wait_primary();
    }
};

// Launch a decode kernel as a programmatic dependent of the kernel before it
// in the stream: its CTAs may become resident while that kernel (the KV
// append, or the group pass) runs, and wait in griddepcontrol.wait before
// reading anything (or, after the group pass, only before they leave).
template <typename K, typename... Args>
cudaError_t launch_decode_kernel(K kernel, dim3 grid, dim3 block, int smem, cudaStream_t stream,
                                 Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// "Dynamic shared memory limit raised" bookkeeping for one kernel, per CUDA
// context (the attribute belongs to the context's copy of the module).
struct SmemAttr {
    PerContext done;
    template <typename K>
    cudaError_t ensure(K kernel, int bytes) {
        void* v = nullptr;
        return per_context_value(done, &v, [&](void** o) {
            *o = reinterpret_cast<void*>(1);
            return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        });
    }
};

}  // namespace pkv
