// Template dispatch of the CUDA-core decode kernel over (head_dim, block_size,
// heads per CTA) for one element type.  Each element type is instantiated in
// its own translation unit so the builds run in parallel.
#pragma once

#include "decode_simt.cuh"

namespace pkv {

// TC: the page element type (T, or E4M3 pages with T = fp16/bf16 q and out).
template <typename T, typename TC = T>
cudaError_t dispatch_decode_simt(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                 cudaStream_t stream) {
#define PKV_SIMT_CASE(D_, BS_, HG_)                                   \
    if (head_dim == D_ && block_size == BS_ && hg == HG_)             \
        return launch_decode_simt<T, D_, BS_, HG_, 4, 0, TC>(a, stream);
// E4M3 pages stop at 2 heads per CTA: 16 values per 16-byte chunk double the
// q and accumulator registers, and 4 heads would spill.
#define PKV_SIMT_HG(D_, BS_)                                 \
    PKV_SIMT_CASE(D_, BS_, 1) PKV_SIMT_CASE(D_, BS_, 2)     \
    if constexpr (Elem<TC>::kBytes >= 2) { PKV_SIMT_CASE(D_, BS_, 4) }
#define PKV_SIMT_BS(D_) PKV_SIMT_HG(D_, 16) PKV_SIMT_HG(D_, 32) PKV_SIMT_HG(D_, 64)
    if constexpr (Elem<TC>::kBytes >= 2) {  // rows of at least 128 bytes
        PKV_SIMT_BS(64)
    }
    PKV_SIMT_BS(128)
    if constexpr (Elem<TC>::kBytes <= 2) {  // 1 KB float32 rows would not fit two stages
        PKV_SIMT_BS(256)
    }
#undef PKV_SIMT_BS
#undef PKV_SIMT_HG
#undef PKV_SIMT_CASE
    return cudaErrorInvalidValue;
}

cudaError_t decode_simt_f32(const DecodeArgs& a, int head_dim, int block_size, int hg,
                            cudaStream_t stream);
cudaError_t decode_simt_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                            cudaStream_t stream);
cudaError_t decode_simt_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                             cudaStream_t stream);
// E4M3 pages; q and out fp16 / bf16
cudaError_t decode_simt_e4m3_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                 cudaStream_t stream);
cudaError_t decode_simt_e4m3_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                  cudaStream_t stream);

}  // namespace pkv
