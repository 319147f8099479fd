// Tensor-core paged decode over E4M3 pages: instantiations.
#include "decode_mma_e4m3.cuh"

namespace pkv {

// CTA shape: 2 warps x 4 stages (6 CTAs per SM) when the CTAs are many and
// short-lived relative to their start-up -- one live head (MHA) or
// partitions of at most 512 tokens; else 4 warps x 3 stages (3 CTAs per SM).
// Measured on B200 (E4M3 pages, head_dim 128, bs 16): the 2-warp shape is
// 5 % faster on the MHA layer and 7-14 % faster with 512-token partitions,
// 3-14 % slower on GQA and long contexts with 2048-token partitions.  It
// needs a 32-token stage of whole blocks: block sizes 16 and 32.
template <typename T>
static cudaError_t dispatch_mma_e4m3(const DecodeArgs& a, int head_dim, int block_size, int nh,
                                     cudaStream_t stream) {
    const bool two = head_dim == 128 && block_size <= 32 &&
                     (a.group == 1 || a.partition_size <= 512);
    if (two) {
        if (block_size == 16 && nh == 8) return launch_decode_mma_e4m3<T, 128, 16, 8, 2, 4>(a, stream);
        if (block_size == 16 && nh == 16) return launch_decode_mma_e4m3<T, 128, 16, 16, 2, 4>(a, stream);
        if (block_size == 32 && nh == 8) return launch_decode_mma_e4m3<T, 128, 32, 8, 2, 4>(a, stream);
        if (block_size == 32 && nh == 16) return launch_decode_mma_e4m3<T, 128, 32, 16, 2, 4>(a, stream);
    }
#define PKV_MMA8_CASE(D_, BS_, NH_)                                   \
    if (head_dim == D_ && block_size == BS_ && nh == NH_)             \
        return launch_decode_mma_e4m3<T, D_, BS_, NH_>(a, stream);
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
