// The split-K merge of a decode's partitions: the log-sum-exp reduce.
//
// A sequence longer than one partition leaves one partial result per
// partition and query head: its maximum m_p (base-2 logits), its sum l_p and
// its normalised output o_p.  Merged, they give exactly the attention over
// the whole sequence ("pagedattention vllm" §Attention Computation: attention
// taken block by block equals attention over the contiguous sequence):
//   M = max_p m_p,  w_p = l_p 2^(m_p - M),  out = sum_p w_p o_p / sum_p w_p.
#pragma once

#include "decode_common.cuh"

namespace pkv {

// Two forms of the merge.  The reduce is launched as a programmatic
// dependent of the decode, and a CTA of a split row sits resident waiting
// for the decode grid: where rows have few partitions (a batch of mostly
// short sequences) that CTA must be small, so the registers-only form runs:
// one CTA of 8 warps per 8 query heads of S consecutive sequences (a warp
// per row, sequence after sequence; far fewer CTAs than rows to launch and
// retire), no dynamic shared memory.  S keeps about two CTAs per SM: a batch
// of many sequences, few of them split, launches a few hundred CTAs instead
// of one per sequence, most of which only read lengths and leave.
// Rows of many partitions (long contexts) stream their partial outputs
// through shared memory with bulk copies (48 KB per CTA, one per row); their
// waiting CTAs appear only when the decode CTAs, all split, finish their
// loops.
constexpr int kReduceRowsPerCta = 8;
constexpr int kReduceThreads = 256;
constexpr int kReduceStreamSlots = 16;  // partial results per row from which rows stream
constexpr int kReduceSms = 148;         // SMs of a B200: the small form's grid size target

// Few partitions per row: one warp merges np partial results of one row into
// out_row from registers.  Partial p's (m, l) is at ml + 2 p, its o at
// o + p * D; every lane sees every partial (so holds the whole sum) and owns
// D / 32 consecutive dimensions.  Four partials' loads are issued before the
// first is used.
template <typename T, int D>
__device__ __forceinline__ void merge_row_warp(const float* __restrict__ ml,
                                               const float* __restrict__ o, int np, T* out_row,
                                               int lane) {
    constexpr int PER_LANE = D / 32;
    float M = -INFINITY;
    for (int p = lane; p < np; p += 32) M = fmaxf(M, __ldg(ml + 2 * p));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    auto load_o = [&](int p, float (&x)[PER_LANE]) {
        const float* op = o + (int64_t)p * D + lane * PER_LANE;
        if constexpr (PER_LANE % 4 == 0) {
#pragma unroll
            for (int i = 0; i < PER_LANE; i += 4) {
                const float4 v = __ldg(reinterpret_cast<const float4*>(op + i));
                x[i] = v.x;
                x[i + 1] = v.y;
                x[i + 2] = v.z;
                x[i + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < PER_LANE; ++i) x[i] = __ldg(op + i);
        }
    };
    float num[PER_LANE];
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) num[i] = 0.f;
    float den = 0.f;
    constexpr int U = 4;
    int p = 0;
    for (; p + U <= np; p += U) {
        float pm[U], pl[U], x[U][PER_LANE];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            pm[u] = __ldg(ml + 2 * (p + u));
            pl[u] = __ldg(ml + 2 * (p + u) + 1);
            load_o(p + u, x[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float w = pl[u] * exp2f(pm[u] - M);
            den += w;
#pragma unroll
            for (int i = 0; i < PER_LANE; ++i) num[i] = fmaf(w, x[u][i], num[i]);
        }
    }
    for (; p < np; ++p) {
        float x[PER_LANE];
        load_o(p, x);
        const float w = __ldg(ml + 2 * p + 1) * exp2f(__ldg(ml + 2 * p) - M);
        den += w;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) num[i] = fmaf(w, x[i], num[i]);
    }
    const float inv = 1.f / den;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i)
        out_row[lane * PER_LANE + i] = Elem<T>::from_f32(num[i] * inv);
}

// Chunks of a row's partial outputs streamed through shared memory: CH
// partitions (16 KB) per chunk, STAGES chunks in flight.
template <int D>
struct ReduceCfg {
    static constexpr int CH = 16384 / (D * 4);
    static constexpr int STAGES = 3;
    static constexpr int CHUNK_BYTES = CH * D * 4;
    static constexpr int SMEM = 64 + STAGES * CHUNK_BYTES;  // barriers, then the ring
    static_assert(kReduceThreads % D == 0 && CH % (kReduceThreads / D) == 0, "layout");
};

// Many partitions per row: merge np partial results of one (sequence, query
// head) row into out_row.  Partial p's (m, l) is at ml + p * ml_stride, its o
// at o + p * D (one
// contiguous run of np * D floats for the row, 16-byte aligned); they were
// written by an earlier grid.  The o rows stream into shared memory in
// 16 KB bulk copies (TMA), three in flight, so a row of many partitions (a
// long context in 512-token partitions: 256, 128 KB) is read at copy-engine
// rate rather than one dependent load after another.  Thread t sums
// dimension t % D over its share (t / D) of each chunk's partitions.  A wait
// that gives up flags the status word and leaves the row unwritten.
template <typename T, int D>
__device__ __forceinline__ void merge_partials(const float* __restrict__ ml, int64_t ml_stride,
                                               const float* __restrict__ o, int np, T* out_row,
                                               unsigned int* status) {
    using C = ReduceCfg<D>;
    constexpr int NT = kReduceThreads;
    constexpr int SPLIT = NT / D;           // threads per dimension
    constexpr int PER = C::CH / SPLIT;      // partitions per thread and chunk
    extern __shared__ __align__(128) unsigned char smem_red[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem_red);
    float* ring = reinterpret_cast<float*>(smem_red + 64);
    __shared__ float s_max[NT / 32];
    __shared__ float s_part[SPLIT][D + 1];
    __shared__ int s_abort;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nchunks = (np + C::CH - 1) / C::CH;

    auto issue = [&](int c, int stage) {  // thread 0
        const int n = min(C::CH, np - c * C::CH);
        mbar_arrive_expect_tx(full + stage, (uint32_t)(n * D * 4));
        bulk_load(ring + stage * (C::CHUNK_BYTES / 4), o + (int64_t)c * C::CH * D,
                  (uint32_t)(n * D * 4), full + stage, policy_evict_first());
    };
    if (tid == 0) {
        s_abort = 0;
        for (int st = 0; st < C::STAGES; ++st) mbar_init(full + st, 1);
        fence_barrier_init();
        for (int c = 0; c < min(C::STAGES, nchunks); ++c) issue(c, c);
    }

    // M = max_p m_p while the first chunks are in flight
    float M = -INFINITY;
    for (int p = tid; p < np; p += NT) M = fmaxf(M, __ldg(ml + p * ml_stride));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    if (lane == 0) s_max[warp] = M;
    __syncthreads();  // also: the barriers are initialised
    M = s_max[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, s_max[w]);

    const int d = tid % D, part = tid / D;
    float num = 0.f, den = 0.f;
    for (int c = 0; c < nchunks; ++c) {
        const int stage = c % C::STAGES;
        if (!mbar_wait(full + stage, (uint32_t)((c / C::STAGES) & 1), status)) s_abort = 1;
        const float* ch = ring + stage * (C::CHUNK_BYTES / 4);
        const int p0 = c * C::CH;
#pragma unroll 4
        for (int j = 0; j < PER; ++j) {
            const int pc = part * PER + j;  // partition within the chunk
            const int p = p0 + pc;
            if (p < np) {
                const float w = __ldg(ml + p * ml_stride + 1) * exp2f(__ldg(ml + p * ml_stride) - M);
                den += w;
                num = fmaf(w, ch[pc * D + d], num);
            }
        }
        __syncthreads();  // every thread is done with this stage (and saw s_abort)
        if (s_abort) {
            // let the copies still in flight land (bounded) before the CTA
            // leaves: this chunk's (some thread gave up on it) and the next
            if (tid == 0) drain_ring(full, C::STAGES, c, min(nchunks, c + C::STAGES), status);
            return;
        }
        if (tid == 0 && c + C::STAGES < nchunks) issue(c + C::STAGES, stage);
    }
    s_part[part][d] = num;
    if (d == 0) s_part[part][D] = den;
    __syncthreads();
    if (tid < D) {
        float x = 0.f, total = 0.f;
#pragma unroll
        for (int q = 0; q < SPLIT; ++q) {
            x += s_part[q][tid];
            total += s_part[q][D];
        }
        out_row[tid] = Elem<T>::from_f32(x / total);
    }
}

// Merge the partitions of each (sequence, query head) row.  Rows with one
// partial result in all were written by the decode kernel and are skipped.
// Launched as a programmatic dependent of the decode kernel: the CTAs of
// sequences with one partition leave before the wait, during the decode's
// tail; the others wait for the decode grid's writes before reading.
// STREAM: one CTA per row (grid Hq x B); else one CTA per 8 query heads of
// S = ceil(B / gridDim.y) <= 32 consecutive sequences (grid ceil(Hq / 8) x
// ceil(B / S)), a warp per row.
template <typename T, int D, bool STREAM>
__global__ void __launch_bounds__(kReduceThreads, 1) lse_reduce_kernel(const DecodeArgs a) {
    // the partition count depends only on the inputs, not on the decode
    // grid's output: rows with one partial result leave before the wait
    if constexpr (STREAM) {
        const int b = blockIdx.y;
        const Span sp = seq_span(a, b, false);
        if (sp.direct) return;
        const int np = sp.slot0 + sp.np;  // the group pass's slots, then this row's partitions
        pdl_wait_primary();
        const int64_t row = (int64_t)b * a.num_q_heads + blockIdx.x;
        merge_partials<T, D>(a.ws_ml + row * a.ws_slots * 2, 2, a.ws_o + row * a.ws_slots * D,
                             np, reinterpret_cast<T*>(a.out) + row * D, a.status);
    } else if (gridDim.y == (unsigned)a.num_seqs) {  // one sequence per CTA
        const int b = blockIdx.y;
        const Span sp = seq_span(a, b, false);
        if (sp.direct) return;
        pdl_wait_primary();
        const int h = blockIdx.x * kReduceRowsPerCta + (threadIdx.x >> 5);
        if (h >= a.num_q_heads) return;
        const int64_t row = (int64_t)b * a.num_q_heads + h;
        merge_row_warp<T, D>(a.ws_ml + row * a.ws_slots * 2, a.ws_o + row * a.ws_slots * D,
                             sp.slot0 + sp.np, reinterpret_cast<T*>(a.out) + row * D,
                             threadIdx.x & 31);
    } else {
        __shared__ uint32_t s_split;  // bit j: sequence b0 + j has partial results to merge
        const int S = (a.num_seqs + gridDim.y - 1) / gridDim.y;
        const int b0 = blockIdx.y * S;
        const int lane = threadIdx.x & 31;
        if (threadIdx.x < 32) {
            const int b = b0 + lane;
            const bool split = lane < S && b < a.num_seqs && !seq_span(a, b, false).direct;
            const uint32_t m = __ballot_sync(0xffffffffu, split);
            if (lane == 0) s_split = m;
        }
        __syncthreads();
        uint32_t split = s_split;
        if (split == 0) return;
        pdl_wait_primary();
        const int h = blockIdx.x * kReduceRowsPerCta + (threadIdx.x >> 5);
        if (h >= a.num_q_heads) return;
        while (split) {
            const int b = b0 + __ffs(split) - 1;
            split &= split - 1;
            const Span sp = seq_span(a, b, false);
            const int np = sp.slot0 + sp.np;
            const int64_t row = (int64_t)b * a.num_q_heads + h;
            merge_row_warp<T, D>(a.ws_ml + row * a.ws_slots * 2, a.ws_o + row * a.ws_slots * D,
                                 np, reinterpret_cast<T*>(a.out) + row * D, lane);
        }
    }
}

// Launch the reduce after the decode kernel on the same stream, as a
// programmatic dependent launch: the streaming form when rows may hold at
// least kReduceStreamSlots partial results, else the small one.
template <typename T, int D>
cudaError_t launch_lse_reduce(const DecodeArgs& a, cudaStream_t stream) {
    const bool streamed = a.ws_slots >= kReduceStreamSlots;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kReduceThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!streamed) {
        // S sequences per CTA: about two CTAs per SM, at most 32 (one ballot)
        const int64_t hx = (a.num_q_heads + kReduceRowsPerCta - 1) / kReduceRowsPerCta;
        const int64_t per_seq = hx * (a.num_seqs > 0 ? 1 : 0);
        int S = (int)((per_seq * a.num_seqs + 2 * kReduceSms - 1) / (2 * kReduceSms));
        S = S < 1 ? 1 : (S > 32 ? 32 : S);
        const int gy = a.num_seqs > 0 ? (a.num_seqs + S - 1) / S : 1;
        cfg.gridDim = dim3((unsigned)hx, (unsigned)gy, 1);
        cfg.dynamicSmemBytes = 0;
        return cudaLaunchKernelEx(&cfg, lse_reduce_kernel<T, D, false>, a);
    }
    static SmemAttr smem_attr;
    cudaError_t e = smem_attr.ensure(lse_reduce_kernel<T, D, true>, ReduceCfg<D>::SMEM);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(a.num_q_heads, a.num_seqs, 1);
    cfg.dynamicSmemBytes = ReduceCfg<D>::SMEM;
    return cudaLaunchKernelEx(&cfg, lse_reduce_kernel<T, D, true>, a);
}

}  // namespace pkv
