#include "decode_mma.cuh"

namespace pkv {
cudaError_t decode_mma_f16(const DecodeArgs&, int, int, int, cudaStream_t) {
    return cudaErrorInvalidValue;
}
cudaError_t decode_mma_bf16(const DecodeArgs&, int, int, int, cudaStream_t) {
    return cudaErrorInvalidValue;
}
}  // namespace pkv
