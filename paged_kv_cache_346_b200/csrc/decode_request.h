// One decode call as the host sees it, and the plan the host checks derive
// from it (partitioning, kernel choice, workspace size).  Shared by the
// entry points in abi.cu and decode_static_ws.cu, so both validate arguments
// and size the workspace the same way before anything is launched.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "pagedkv.h"

namespace pkv {

struct DecodeRequest {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const float* k_scale;         // E4M3 pages only
    const float* v_scale;
    int scale_per_block;
    bool e4m3;                    // pages hold E4M3 codes; dtype is that of q and out
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* seq_order;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int head_dim;
    int block_size;
    int max_blocks_per_seq;
    int num_blocks;
    int max_context_len;
    float scale;
    int sliding_window;
    pkv_dtype dtype;
    int partition_size;           // 0 = the default for the shape
    pkv_kernel kernel;
    const int32_t* items = nullptr;  // work list (pairs sequence, partition) instead of seq_order
    int num_items = 0;
};

struct DecodePlan {
    bool empty;                   // num_seqs == 0: nothing to launch
    int span;                     // longest attended span in tokens
    int partition_size;           // tokens per partition, resolved
    int max_partitions;           // ceil(span / partition_size), at least 1
    bool use_mma;                 // tensor-core kernel
    int heads_per_cta;            // query heads of one CTA's tile
    int head_chunks;              // CTAs per KV head along the query group
    size_t workspace_bytes;       // scratch the call needs (0: none)
};

// Host-side checks of every argument; fills the plan.  Returns PKV_OK,
// PKV_EINVAL or PKV_EUNSUPPORTED; nothing is launched.
int plan_decode(const DecodeRequest& r, DecodePlan* plan);

// Launches the decode the plan describes, with `workspace` (at least plan.workspace_bytes
// of device memory, 16-byte aligned, when that is non-zero; checked).
int run_decode(const DecodeRequest& r, const DecodePlan& plan, void* workspace,
               size_t workspace_bytes, cudaStream_t stream);

}  // namespace pkv
