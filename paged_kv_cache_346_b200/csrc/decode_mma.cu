// Tensor-core paged decode: instantiations and the tensor-map encoder.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "decode_mma.cuh"

namespace pkv {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

// The pool viewed as a 2-D tensor: `rows` = num_blocks * Hkv * BS rows of
// head_dim elements (2 bytes: f16 / bf16, 1 byte: E4M3 codes as uint8); boxes
// of 128 bytes x box_rows rows, 128-byte swizzle (the layout the kernels'
// ldmatrix addressing assumes).
cudaError_t make_cache_tensor_map(CUtensorMap* map, const void* base, int dtype_bytes,
                                  bool bf16, int head_dim, int64_t rows, int box_rows) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return cudaErrorNotSupported;
    const cuuint64_t gdim[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)head_dim * dtype_bytes};
    const cuuint32_t box[2] = {128u / (cuuint32_t)dtype_bytes, (cuuint32_t)box_rows};
    const cuuint32_t estride[2] = {1u, 1u};
    const CUtensorMapDataType dt = dtype_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : bf16           ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (dtype_bytes != 1 && dtype_bytes != 2) return cudaErrorInvalidValue;
    const CUresult r = g_encode(
        map, dt, 2,
        const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t dispatch_mma(const DecodeArgs& a, int head_dim, int block_size, int nh,
                                cudaStream_t stream) {
#define PKV_MMA_CASE(D_, BS_, NH_)                                    \
    if (head_dim == D_ && block_size == BS_ && nh == NH_)             \
        return launch_decode_mma<T, D_, BS_, NH_>(a, stream);
#define PKV_MMA_NH(D_, BS_) PKV_MMA_CASE(D_, BS_, 8) PKV_MMA_CASE(D_, BS_, 16)
#define PKV_MMA_BS(D_) PKV_MMA_NH(D_, 16) PKV_MMA_NH(D_, 32) PKV_MMA_NH(D_, 64)
    PKV_MMA_BS(64)
    PKV_MMA_BS(128)
    PKV_MMA_BS(256)
#undef PKV_MMA_BS
#undef PKV_MMA_NH
#undef PKV_MMA_CASE
    return cudaErrorInvalidValue;
}

cudaError_t decode_mma_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                           cudaStream_t stream) {
    return dispatch_mma<__half>(a, head_dim, block_size, hg, stream);
}
cudaError_t decode_mma_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                            cudaStream_t stream) {
    return dispatch_mma<__nv_bfloat16>(a, head_dim, block_size, hg, stream);
}

}  // namespace pkv
