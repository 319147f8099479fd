// CUDA-core paged decode instantiations for __nv_bfloat16 caches.
#include "decode_dispatch.cuh"

namespace pkv {
cudaError_t decode_simt_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                            cudaStream_t stream) {
    return dispatch_decode_simt<__nv_bfloat16>(a, head_dim, block_size, hg, stream);
}
}  // namespace pkv
