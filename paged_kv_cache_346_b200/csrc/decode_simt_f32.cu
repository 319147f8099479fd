// CUDA-core paged decode instantiations for float caches.
#include "decode_dispatch.cuh"

namespace pkv {
cudaError_t decode_simt_f32(const DecodeArgs& a, int head_dim, int block_size, int hg,
                            cudaStream_t stream) {
    return dispatch_decode_simt<float>(a, head_dim, block_size, hg, stream);
}
}  // namespace pkv
