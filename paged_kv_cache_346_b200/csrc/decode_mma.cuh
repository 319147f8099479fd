// Tensor-core paged decode (query groups of 4..16 heads, f16 / bf16 caches).
#pragma once

#include "decode_common.cuh"

namespace pkv {

constexpr bool kMmaBuilt = false;

cudaError_t decode_mma_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                           cudaStream_t stream);
cudaError_t decode_mma_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                            cudaStream_t stream);

}  // namespace pkv
