// Tensor-core paged decode over E4M3 pages: instantiations.
#include "decode_stream_e4m3.cuh"

namespace pkv {

// CTA shape: 2 warps when the CTAs are many and short-lived relative to
// their start-up -- one live head (MHA) or partitions of at most 512 tokens;
// else 4 warps.  Measured on B200 (E4M3 pages, head_dim 128, bs 16, per-warp
// rings of 4 stages, 12 warps per SM): the 2-warp shape is 6 % faster on the
// MHA layer and 10-15 % faster with 512-token partitions, and on the GQA
// batch with 4096-token partitions 26 % slower (its longest partitions, at
// half the warps each, become the tail).
//
// 8-head tiles at head_dim 128 take 3-stage rings and 128 registers, so
// eight 2-warp or four 4-warp CTAs share an SM (16 warps): 1-9 % faster than
// 4-stage rings at 12 warps per SM, by workload.  16-head tiles and head_dim
// 256 keep 4 stages.
template <typename T>
static cudaError_t dispatch_mma_e4m3(const DecodeArgs& a, int head_dim, int block_size, int nh,
                                     cudaStream_t stream) {
    const bool two = head_dim == 128 && (a.group == 1 || a.partition_size <= 512);
    if (two) {
#define PKV_MMA8_TWO(BS_, NH_)                                        \
    if (block_size == BS_ && nh == NH_)                               \
        return launch_decode_mma_e4m3<T, 128, BS_, NH_, 2, NH_ == 8 ? 3 : 0>(a, stream);
        PKV_MMA8_TWO(16, 8) PKV_MMA8_TWO(16, 16) PKV_MMA8_TWO(32, 8) PKV_MMA8_TWO(32, 16)
        PKV_MMA8_TWO(64, 8) PKV_MMA8_TWO(64, 16)
#undef PKV_MMA8_TWO
    }
#define PKV_MMA8_CASE(D_, BS_, NH_)                                   \
    if (head_dim == D_ && block_size == BS_ && nh == NH_)             \
        return launch_decode_mma_e4m3<T, D_, BS_, NH_, 4, (D_ == 128 && NH_ == 8) ? 3 : 0>(a, stream);
#define PKV_MMA8_NH(D_, BS_) PKV_MMA8_CASE(D_, BS_, 8) PKV_MMA8_CASE(D_, BS_, 16)
#define PKV_MMA8_BS(D_) PKV_MMA8_NH(D_, 16) PKV_MMA8_NH(D_, 32) PKV_MMA8_NH(D_, 64)
    PKV_MMA8_BS(128)
    PKV_MMA8_BS(256)
#undef PKV_MMA8_BS
#undef PKV_MMA8_NH
#undef PKV_MMA8_CASE
    return cudaErrorInvalidValue;
}

cudaError_t decode_mma_e4m3_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                cudaStream_t stream) {
    return dispatch_mma_e4m3<__half>(a, head_dim, block_size, hg, stream);
}
cudaError_t decode_mma_e4m3_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                 cudaStream_t stream) {
    return dispatch_mma_e4m3<__nv_bfloat16>(a, head_dim, block_size, hg, stream);
}

// The planned decode: the same CTA shapes and ring depths as the regular
// grid's (2 warps for one live head at head_dim 128, else 4; 3-stage rings
// for 8-head tiles at head_dim 128).
template <typename T, int D, int BS, int NH, int NW, int STAGES>
static cudaError_t launch_stream(const DecodeArgs& a, int ctas, int* occupancy,
                                 cudaStream_t stream) {
    using S = StreamCfg<D, BS, NW, STAGES>;
    static SmemAttr attr[2];
    auto kern = a.scale_per_block ? decode_stream_e4m3_kernel<T, D, BS, NH, NW, STAGES, true>
                                  : decode_stream_e4m3_kernel<T, D, BS, NH, NW, STAGES, false>;
    cudaError_t e = attr[a.scale_per_block ? 1 : 0].ensure(kern, S::SMEM);
    if (e != cudaSuccess) return e;
    if (occupancy)
        return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, kern, NW * 32, S::SMEM);
    const int64_t rows = (int64_t)a.num_blocks * a.num_kv_heads * BS;
    CUtensorMap tk, tv;
    e = make_cache_tensor_map(&tk, a.k_cache, 1, false, D, rows, 16);
    if (e != cudaSuccess) return e;
    e = make_cache_tensor_map(&tv, a.v_cache, 1, false, D, rows, 16);
    if (e != cudaSuccess) return e;
    kern<<<ctas, NW * 32, S::SMEM, stream>>>(a, tk, tv);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t dispatch_stream(const DecodeArgs& a, int head_dim, int block_size, int nh,
                                   int nw, int ctas, int* occupancy, cudaStream_t stream) {
#define PKV_ST_CASE(D_, BS_, NH_, NW_)                                                  \
    if (head_dim == D_ && block_size == BS_ && nh == NH_ && nw == NW_)                  \
        return launch_stream<T, D_, BS_, NH_, NW_, (D_ == 128 && NH_ == 8) ? 3 : 0>(a, ctas, \
                                                                                occupancy, stream);
#define PKV_ST_NH(D_, BS_, NW_) PKV_ST_CASE(D_, BS_, 8, NW_) PKV_ST_CASE(D_, BS_, 16, NW_)
#define PKV_ST_BS(D_, NW_) PKV_ST_NH(D_, 16, NW_) PKV_ST_NH(D_, 32, NW_) PKV_ST_NH(D_, 64, NW_)
    PKV_ST_BS(128, 2)
    PKV_ST_BS(128, 4)
    PKV_ST_BS(256, 4)
#undef PKV_ST_BS
#undef PKV_ST_NH
#undef PKV_ST_CASE
    return cudaErrorInvalidValue;
}

cudaError_t decode_stream_e4m3(const DecodeArgs& a, bool bf16, int head_dim, int block_size,
                               int hg, int nw, int planned_ctas, int* occupancy,
                               cudaStream_t stream) {
    return bf16 ? dispatch_stream<__nv_bfloat16>(a, head_dim, block_size, hg, nw, planned_ctas,
                                                 occupancy, stream)
                : dispatch_stream<__half>(a, head_dim, block_size, hg, nw, planned_ctas,
                                          occupancy, stream);
}

}  // namespace pkv
