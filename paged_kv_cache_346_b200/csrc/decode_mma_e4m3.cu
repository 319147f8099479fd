// Tensor-core paged decode over E4M3 pages: instantiations.
#include "decode_mma_e4m3.cuh"

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

}  // namespace pkv
