// Group pass of the shared-prefix decode (tensor cores, fp16 / bf16 pages):
// instantiations.
#include "decode_mma.cuh"

namespace pkv {

template <typename T>
static cudaError_t dispatch_mma_groups(const DecodeArgs& a, int head_dim, int block_size, int nh,
                                       int num_groups, cudaStream_t stream) {
#define PKV_MMAG_CASE(D_, BS_, NH_)                                   \
    if (head_dim == D_ && block_size == BS_ && nh == NH_)             \
        return launch_decode_mma_groups<T, D_, BS_, NH_>(a, num_groups, stream);
#define PKV_MMAG_NH(D_, BS_) PKV_MMAG_CASE(D_, BS_, 8) PKV_MMAG_CASE(D_, BS_, 16)
#define PKV_MMAG_BS(D_) PKV_MMAG_NH(D_, 16) PKV_MMAG_NH(D_, 32) PKV_MMAG_NH(D_, 64)
    PKV_MMAG_BS(64)
    PKV_MMAG_BS(128)
    PKV_MMAG_BS(256)
#undef PKV_MMAG_BS
#undef PKV_MMAG_NH
#undef PKV_MMAG_CASE
    return cudaErrorInvalidValue;
}

cudaError_t decode_mma_groups_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                  int num_groups, cudaStream_t stream) {
    return dispatch_mma_groups<__half>(a, head_dim, block_size, hg, num_groups, stream);
}
cudaError_t decode_mma_groups_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                   int num_groups, cudaStream_t stream) {
    return dispatch_mma_groups<__nv_bfloat16>(a, head_dim, block_size, hg, num_groups, stream);
}

}  // namespace pkv
