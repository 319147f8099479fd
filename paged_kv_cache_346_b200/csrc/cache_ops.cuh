// Launchers of the KV append and block copy kernels.
#pragma once

#include "device_common.cuh"

namespace pkv {

// row_bytes_per_head = head_dim * element size (a multiple of 16).
cudaError_t launch_kv_append(void* k_cache, void* v_cache, const void* k, const void* v,
                             const int64_t* slots, int num_tokens, int num_kv_heads,
                             int row_bytes_per_head, int block_size, int num_blocks,
                             unsigned int* status, cudaStream_t stream);

// E4M3 pages from fp16 (bf16_in false) or bf16 rows; head_dim a multiple of 16.
cudaError_t launch_kv_append_e4m3(void* k_cache, void* v_cache, const void* k, const void* v,
                                  const float* k_scale, const float* v_scale,
                                  const int64_t* slots, int num_tokens, int num_kv_heads,
                                  int head_dim, int block_size, int num_blocks, bool bf16_in,
                                  bool per_block, unsigned int* status, cudaStream_t stream);

// block_bytes = num_kv_heads * block_size * head_dim * element size.
cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs,
                               int num_pairs, int64_t block_bytes, int num_blocks,
                               unsigned int* status, cudaStream_t stream);

// Pages between two pools (device or page-locked host, as device views).
cudaError_t launch_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               const int32_t* pairs, int num_pairs, int64_t block_bytes,
                               int src_blocks, int dst_blocks, unsigned int* status,
                               cudaStream_t stream);

// One thread waits (bounded by `limit` clock cycles) on an mbarrier that
// nothing completes, flags PKV_DEV_TIMEOUT and returns (selftest.cu).
cudaError_t launch_wait_timeout(long long limit, unsigned int* status, cudaStream_t stream);

}  // namespace pkv
