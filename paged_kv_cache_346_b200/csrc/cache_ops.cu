// KV append (slot-mapping scatter), copy-on-write block copies and swapping.
//
// All are pure bit moves bound by HBM (or host-link) bandwidth: 16-byte vector
// loads and stores, several in flight per thread, no shared memory.
#include "cache_ops.cuh"

namespace pkv {

// 16 fp16 / bf16 values (two 16-byte vectors) -> 16 E4M3 codes of x / scale,
// the code of the float32 quotient rounded to nearest (ties to even,
// saturating at the largest finite code).
//
// Fast path: q = x * r with r = 1 / scale (float32), within 2^-23 (relative)
// of the true quotient, so the float32 quotient lies within 2^-22 of q.  The
// E4M3 rounding is monotone, so if q (1 - 2^-20) and q (1 + 2^-20) -- each
// rounded again, still bracketing it -- convert to the same code, that is
// the code of the quotient.  Otherwise (q within ~2^-20 of a rounding
// boundary between two codes: rare) the element takes the division itself.
// Scales outside [2^-100, 2^100] (where r could lose precision) always take
// the division.
template <typename Tin>
__device__ __forceinline__ uint4 quantise16(const uint4* src, float scale) {
    float f[16];
    Elem<Tin>::to_f32(src[0], f);
    Elem<Tin>::to_f32(src[1], f + 8);
    const bool fast = scale >= 0x1p-100f && scale <= 0x1p100f;
    const float r = 1.f / scale;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t x = 0;
#pragma unroll
        for (int b = 0; b < 4; b += 2) {
            const float q0 = f[4 * j + b] * r, q1 = f[4 * j + b + 1] * r;
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(
                make_float2(q0 * (1.f - 0x1p-20f), q1 * (1.f - 0x1p-20f)), __NV_SATFINITE,
                __NV_E4M3);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(
                make_float2(q0 * (1.f + 0x1p-20f), q1 * (1.f + 0x1p-20f)), __NV_SATFINITE,
                __NV_E4M3);
            uint32_t pair = lo;
            if (!fast || lo != hi) {  // near a boundary: the exact quotients
                const uint32_t c0 =
                    __nv_cvt_float_to_fp8(f[4 * j + b] / scale, __NV_SATFINITE, __NV_E4M3);
                const uint32_t c1 =
                    __nv_cvt_float_to_fp8(f[4 * j + b + 1] / scale, __NV_SATFINITE, __NV_E4M3);
                pair = c0 | (c1 << 8);
            }
            x |= (pair & 0xffffu) << (8 * b);
        }
        w[j] = x;
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// One thread per 16-byte vector of the new tokens' [T, Hkv, D] rows.
// Token t's vector r (r < H * D * e / 16) lands in its slot's row: block
// s / bs, KV head r / head_vecs, offset s % bs ("What is PagedAttention ..."
// §How it works: blocks fill as the sequence grows).
__global__ void __launch_bounds__(256) kv_append_kernel(uint4* __restrict__ kc,
                                                         uint4* __restrict__ vc,
                                                         const uint4* __restrict__ k,
                                                         const uint4* __restrict__ v,
                                                         const int64_t* __restrict__ slots,
                                                         int64_t total_vecs, int row_vecs,
                                                         int head_vecs, int num_kv_heads,
                                                         int block_size, int64_t num_slots,
                                                         unsigned int* status) {
    // the decode that usually follows waits for this grid to finish anyway:
    // let it launch (and set up) while the appends run
    pdl_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total_vecs; i += stride) {
        const int64_t t = i / row_vecs;
        const int r = (int)(i - t * row_vecs);
        const int64_t s = slots[t];
        if (s < 0) continue;  // padding token
        if (s >= num_slots) {
            if (r == 0) flag(status, PKV_DEV_BAD_SLOT);
            continue;
        }
        const int h = r / head_vecs;
        const int c = r - h * head_vecs;
        const int64_t blk = s / block_size;
        const int off = (int)(s - blk * block_size);
        const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_vecs + c;
        const uint4 kx = k[i];
        const uint4 vx = v[i];
        kc[dst] = kx;
        vc[dst] = vx;
    }
}

// Quantising append: one thread per 16 elements of the new tokens' [T, Hkv, D]
// rows (two 16-byte input vectors of fp16 / bf16, one 16-byte vector of
// codes out).  code = E4M3(x / scale[h]): a correctly rounded float32
// division, then the hardware conversion (nearest, ties to even, saturating
// at the largest finite code).
template <typename Tin>
__global__ void __launch_bounds__(256) kv_append_e4m3_kernel(
    uint4* __restrict__ kc, uint4* __restrict__ vc, const uint4* __restrict__ k,
    const uint4* __restrict__ v, const float* __restrict__ ks, const float* __restrict__ vs,
    const int64_t* __restrict__ slots, int64_t total_vecs, int row_vecs, int head_vecs,
    int num_kv_heads, int block_size, int64_t num_slots, int per_block, unsigned int* status) {
    pdl_launch_dependents();  // as kv_append_kernel
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total_vecs; i += stride) {
        const int64_t t = i / row_vecs;
        const int r = (int)(i - t * row_vecs);
        const int64_t s = slots[t];
        if (s < 0) continue;
        if (s >= num_slots) {
            if (r == 0) flag(status, PKV_DEV_BAD_SLOT);
            continue;
        }
        const int h = r / head_vecs;
        const int c = r - h * head_vecs;
        const int64_t blk = s / block_size;
        const int off = (int)(s - blk * block_size);
        const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_vecs + c;
        const int64_t si = per_block ? blk * num_kv_heads + h : h;
        kc[dst] = quantise16<Tin>(k + 2 * i, ks[si]);
        vc[dst] = quantise16<Tin>(v + 2 * i, vs[si]);
    }
}

// Whole-page moves, shared by the copy-on-write copies (within one pool) and
// swapping (between a device pool and a page-locked host pool).  Grid
// (chunks, pairs, 2): blockIdx.z picks K or V; each thread keeps UNROLL
// 16-byte loads in flight before its stores.  The source and destination
// pools may be the same buffer (different blocks), so no pointer is declared
// restrict.
template <int UNROLL>
__global__ void __launch_bounds__(256) move_pages_kernel(uint4* dk, uint4* dv, const uint4* sk,
                                                          const uint4* sv,
                                                          const int32_t* __restrict__ pairs,
                                                          int num_pairs, int64_t block_vecs,
                                                          int src_blocks, int dst_blocks,
                                                          unsigned int* status) {
    uint4* dbase = blockIdx.z ? dv : dk;
    const uint4* sbase = blockIdx.z ? sv : sk;
    for (int pr = blockIdx.y; pr < num_pairs; pr += gridDim.y) {
        const int32_t src = pairs[2 * pr];
        const int32_t dst = pairs[2 * pr + 1];
        if ((unsigned)src >= (unsigned)src_blocks || (unsigned)dst >= (unsigned)dst_blocks) {
            if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0)
                flag(status, PKV_DEV_BAD_BLOCK);
            continue;
        }
        const uint4* s = sbase + (int64_t)src * block_vecs;
        uint4* d = dbase + (int64_t)dst * block_vecs;
        const int64_t step = (int64_t)gridDim.x * blockDim.x * UNROLL;
        for (int64_t i0 = ((int64_t)blockIdx.x * blockDim.x) * UNROLL + threadIdx.x;
             i0 < block_vecs; i0 += step) {
            uint4 x[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int64_t i = i0 + (int64_t)u * blockDim.x;
                if (i < block_vecs) x[u] = s[i];
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int64_t i = i0 + (int64_t)u * blockDim.x;
                if (i < block_vecs) d[i] = x[u];
            }
        }
    }
}

template <int UNROLL>
static cudaError_t launch_move_pages(void* dk, void* dv, const void* sk, const void* sv,
                                     const int32_t* pairs, int num_pairs, int64_t block_bytes,
                                     int src_blocks, int dst_blocks, unsigned int* status,
                                     cudaStream_t stream) {
    if (num_pairs == 0) return cudaSuccess;
    const int64_t block_vecs = block_bytes / 16;
    int64_t chunks = (block_vecs + 256 * UNROLL - 1) / (256 * UNROLL);
    if (chunks > 1024) chunks = 1024;
    const int ys = num_pairs < 65535 ? num_pairs : 65535;
    dim3 grid((unsigned)chunks, (unsigned)ys, 2);
    move_pages_kernel<UNROLL><<<grid, 256, 0, stream>>>(
        static_cast<uint4*>(dk), static_cast<uint4*>(dv), static_cast<const uint4*>(sk),
        static_cast<const uint4*>(sv), pairs, num_pairs, block_vecs, src_blocks, dst_blocks,
        status);
    return cudaGetLastError();
}

cudaError_t launch_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               const int32_t* pairs, int num_pairs, int64_t block_bytes,
                               int src_blocks, int dst_blocks, unsigned int* status,
                               cudaStream_t stream) {
    // more loads in flight: one side sits behind the host link
    return launch_move_pages<8>(dst_k, dst_v, src_k, src_v, pairs, num_pairs, block_bytes,
                                src_blocks, dst_blocks, status, stream);
}

cudaError_t launch_kv_append(void* k_cache, void* v_cache, const void* k, const void* v,
                             const int64_t* slots, int num_tokens, int num_kv_heads,
                             int row_bytes_per_head, int block_size, int num_blocks,
                             unsigned int* status, cudaStream_t stream) {
    const int head_vecs = row_bytes_per_head / 16;
    const int row_vecs = head_vecs * num_kv_heads;
    const int64_t total = (int64_t)num_tokens * row_vecs;
    if (total == 0) return cudaSuccess;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    kv_append_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slots, total, row_vecs,
        head_vecs, num_kv_heads, block_size, (int64_t)num_blocks * block_size, status);
    return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs,
                               int num_pairs, int64_t block_bytes, int num_blocks,
                               unsigned int* status, cudaStream_t stream) {
    return launch_move_pages<4>(k_cache, v_cache, k_cache, v_cache, pairs, num_pairs,
                                block_bytes, num_blocks, num_blocks, status, stream);
}

cudaError_t launch_kv_append_e4m3(void* k_cache, void* v_cache, const void* k, const void* v,
                                  const float* k_scale, const float* v_scale,
                                  const int64_t* slots, int num_tokens, int num_kv_heads,
                                  int head_dim, int block_size, int num_blocks, bool bf16_in,
                                  bool per_block, unsigned int* status, cudaStream_t stream) {
    const int head_vecs = head_dim / 16;
    const int row_vecs = head_vecs * num_kv_heads;
    const int64_t total = (int64_t)num_tokens * row_vecs;
    if (total == 0) return cudaSuccess;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    auto kern = bf16_in ? kv_append_e4m3_kernel<__nv_bfloat16> : kv_append_e4m3_kernel<__half>;
    kern<<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), k_scale, v_scale, slots,
        total, row_vecs, head_vecs, num_kv_heads, block_size, (int64_t)num_blocks * block_size,
        per_block ? 1 : 0, status);
    return cudaGetLastError();
}

}  // namespace pkv
