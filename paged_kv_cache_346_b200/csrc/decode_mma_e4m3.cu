// Tensor-core paged decode over E4M3 pages: instantiations.
#include "decode_mma_e4m3.cuh"

namespace pkv {

template <typename T>
static cudaError_t dispatch_mma_e4m3(const DecodeArgs& a, int head_dim, int block_size, int nh,
                                     cudaStream_t stream) {
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
