// Paged decode with a library-owned, statically sized workspace.
//
// pkv_paged_attention_decode needs device scratch for sequences that span more
// than one partition, and expects the caller to allocate it.  Some callers
// cannot allocate device memory at all: a plugin inside a host application
// that owns every byte of the device and forbids cudaMalloc, or a serving
// loop that must never hit cudaMalloc's implicit device synchronisation.  This
// entry point gives them the same decode with the scratch taken from a fixed
// array compiled into the library.
//
// The array is a file-scope __device__ variable, so every GPU that loads this
// library's device code holds PKV_STATIC_WORKSPACE_BYTES of it until the
// process exits.  On the host its name is only a handle: its device address
// is looked up with cudaGetSymbolAddress on the first call made in each CUDA
// context (normally a device's primary context), with that context current,
// and that address is what the kernels receive.
#include <cstdint>

#include <cuda_runtime.h>

#include "context_cache.h"
#include "decode_request.h"
#include "pagedkv.h"

namespace {

static __device__ __align__(256) unsigned char g_static_workspace[PKV_STATIC_WORKSPACE_BYTES];

pkv::PerContext g_static_workspace_addr;

// Device address of the array in the current context (looked up on first use
// in each context, with that context current).
int static_workspace_address(void** out) {
    const cudaError_t e = pkv::per_context_value(g_static_workspace_addr, out, [](void** o) {
        return cudaGetSymbolAddress(o, g_static_workspace);
    });
    return e == cudaSuccess && *out ? PKV_OK : PKV_ECUDA;
}

}  // namespace

extern "C" int pkv_paged_attention_decode_static_ws(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* seq_order,
    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
    int sliding_window, pkv_dtype dtype, int partition_size, pkv_kernel kernel,
    pkv_stream_t stream) {
    // the regular entry point's argument checks and partitioning, first, so a
    // bad argument gets the same status here as there
    const pkv::DecodeRequest r{out, q, k_cache, v_cache, nullptr, nullptr, 0, false,
                               block_tables, context_lens, seq_order, num_seqs, num_q_heads,
                               num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                               max_context_len, scale, sliding_window, dtype, partition_size,
                               kernel};
    pkv::DecodePlan plan;
    int rc = pkv::plan_decode(r, &plan);
    if (rc != PKV_OK || plan.empty) return rc;
    if (plan.workspace_bytes > (size_t)PKV_STATIC_WORKSPACE_BYTES) return PKV_EBOUNDS;
    void* ws = nullptr;
    if (plan.workspace_bytes > 0) {
        rc = static_workspace_address(&ws);
        if (rc != PKV_OK) return rc;
    }
    // Nothing in the workspace has to start at zero: every entry the merge
    // reads is written earlier in the same call.
    return pkv::run_decode(r, plan, ws, ws ? (size_t)PKV_STATIC_WORKSPACE_BYTES : 0,
                           reinterpret_cast<cudaStream_t>(stream));
}
