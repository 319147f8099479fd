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
// is looked up once per device with cudaGetSymbolAddress (with that device
// current) on the first call made on that device, and that address is what
// the kernels receive.
#include <atomic>
#include <cstdint>

#include <cuda_runtime.h>

#include "pagedkv.h"

namespace {

static __device__ __align__(256) unsigned char g_static_workspace[PKV_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_static_workspace_addr[kMaxDevices];

// Device address of the array on the current device (set up on first use).
int static_workspace_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return PKV_ECUDA;
    void* p = g_static_workspace_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return PKV_ECUDA;
        g_static_workspace_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return PKV_OK;
}

}  // namespace

extern "C" int pkv_paged_attention_decode_static_ws(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* seq_order,
    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
    int sliding_window, pkv_dtype dtype, int partition_size, pkv_kernel kernel,
    pkv_stream_t stream) {
    const int64_t span = sliding_window > 0 && (int64_t)sliding_window + block_size - 1 <
                                                   (int64_t)max_context_len
                             ? (int64_t)sliding_window + block_size - 1
                             : (int64_t)max_context_len;
    const size_t need = pkv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                  (int)span, partition_size);
    if (need > (size_t)PKV_STATIC_WORKSPACE_BYTES) return PKV_EBOUNDS;
    void* ws = nullptr;
    if (need > 0) {
        const int rc = static_workspace_address(&ws);
        if (rc != PKV_OK) return rc;
    }
    // Everything else -- argument checks, kernels, results -- is the regular
    // entry point's.  Nothing in the workspace has to start at zero: every
    // entry the merge reads is written earlier in the same call.
    return pkv_paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens,
                                      seq_order, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                      max_blocks_per_seq, num_blocks, max_context_len, scale,
                                      sliding_window, dtype, partition_size, ws,
                                      ws ? (size_t)PKV_STATIC_WORKSPACE_BYTES : 0, kernel, stream);
}
