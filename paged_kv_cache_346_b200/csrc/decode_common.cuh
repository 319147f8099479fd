// Arguments and the log-sum-exp reduce shared by both decode kernels.
#pragma once

#include <atomic>
#include <cmath>

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
    float* ws_o;                  // [B, Hq, max_partitions, D] partition outputs
    float* ws_ml;                 // [B, Hq, max_partitions, 2] (m in log2 units, l)
    unsigned int* status;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int group;                    // Hq / Hkv
    int head_chunks;              // CTAs per KV head along the query group
    int max_blocks_per_seq;
    int num_blocks;
    int max_tokens;               // max_blocks_per_seq * BS
    int partition_size;           // tokens per partition
    int max_partitions;           // grid.x = ceil(max_context_len / partition_size)
    float scale_log2;             // scale * log2(e): logits are kept in base 2
};

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

__device__ __forceinline__ int num_partitions(const DecodeArgs& a, int L, bool report) {
    int n = (L + a.partition_size - 1) / a.partition_size;
    if (n > a.max_partitions) {
        if (report) flag(a.status, PKV_DEV_BAD_LEN);
        n = a.max_partitions;
    }
    return n;
}

// Merge the partitions of one (sequence, query head) row: with per-partition
// maxima m_p (base-2 logits), sums l_p and normalised outputs o_p,
//   M = max_p m_p,  w_p = l_p 2^(m_p - M),  out = sum_p w_p o_p / sum_p w_p.
// One CTA of 128 threads per row; rows that fit one partition were written by
// the decode kernel and are skipped.  Launched as a programmatic dependent of
// the decode kernel: it waits for the decode grid's writes before reading.
template <typename T, int D>
__global__ void __launch_bounds__(128) lse_reduce_kernel(const DecodeArgs a) {
    constexpr int NW = 4;
    constexpr int PER_LANE = D / 32;  // floats of o per lane
    pdl_wait_primary();
    const int h = blockIdx.x;
    const int b = blockIdx.y;
    const int L = seq_len(a, b, false);
    const int np = num_partitions(a, L, false);
    if (np <= 1) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = (int64_t)b * a.num_q_heads + h;
    const float* ml = a.ws_ml + row * a.max_partitions * 2;
    const float* o = a.ws_o + row * a.max_partitions * D;

    __shared__ float s_max[NW];
    __shared__ float s_den[NW];
    __shared__ float s_num[NW][D];

    float M = -INFINITY;
    for (int p = tid; p < np; p += 128) M = fmaxf(M, ml[2 * p]);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    if (lane == 0) s_max[warp] = M;
    __syncthreads();
    M = fmaxf(fmaxf(s_max[0], s_max[1]), fmaxf(s_max[2], s_max[3]));

    float num[PER_LANE];
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) num[i] = 0.f;
    float den = 0.f;
    for (int p = warp; p < np; p += NW) {
        const float w = ml[2 * p + 1] * exp2f(ml[2 * p] - M);
        den += w;
        const float* op = o + (int64_t)p * D + lane * PER_LANE;
        if constexpr (PER_LANE % 4 == 0) {
#pragma unroll
            for (int i = 0; i < PER_LANE; i += 4) {
                const float4 x = *reinterpret_cast<const float4*>(op + i);
                num[i] = fmaf(w, x.x, num[i]);
                num[i + 1] = fmaf(w, x.y, num[i + 1]);
                num[i + 2] = fmaf(w, x.z, num[i + 2]);
                num[i + 3] = fmaf(w, x.w, num[i + 3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < PER_LANE; ++i) num[i] = fmaf(w, op[i], num[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) s_num[warp][lane * PER_LANE + i] = num[i];
    if (lane == 0) s_den[warp] = den;
    __syncthreads();
    const float total = s_den[0] + s_den[1] + s_den[2] + s_den[3];
    T* out = reinterpret_cast<T*>(a.out) + row * D;
    for (int d = tid; d < D; d += 128) {
        const float x = s_num[0][d] + s_num[1][d] + s_num[2][d] + s_num[3][d];
        out[d] = Elem<T>::from_f32(x / total);
    }
}

// Per-device "dynamic shared memory size set" bookkeeping for one kernel.
struct SmemAttr {
    std::atomic<unsigned long long> done{0};
    template <typename K>
    cudaError_t ensure(K kernel, int bytes) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        const unsigned long long bit = 1ull << (dev & 63);
        if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
        return e;
    }
};

// Launch the reduce after the decode kernel on the same stream, as a
// programmatic dependent launch.
template <typename T, int D>
cudaError_t launch_lse_reduce(const DecodeArgs& a, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.num_q_heads, a.num_seqs, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, lse_reduce_kernel<T, D>, a);
}

}  // namespace pkv
