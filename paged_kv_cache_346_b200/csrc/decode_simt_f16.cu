// CUDA-core paged decode instantiations for __half caches.
#include "decode_dispatch.cuh"

namespace pkv {
cudaError_t decode_simt_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                            cudaStream_t stream) {
    return dispatch_decode_simt<__half>(a, head_dim, block_size, hg, stream);
}
}  // namespace pkv
