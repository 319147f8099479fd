// CUDA-core paged decode instantiations for E4M3 pages with __nv_bfloat16 q / out.
#include "decode_dispatch.cuh"

namespace pkv {
cudaError_t decode_simt_e4m3_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                  cudaStream_t stream) {
    return dispatch_decode_simt<__nv_bfloat16, E4M3>(a, head_dim, block_size, hg, stream);
}
}  // namespace pkv
