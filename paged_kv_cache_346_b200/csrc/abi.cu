// The C ABI of pagedkv (declared in include/pagedkv.h): host-side argument
// checks, kernel selection and launches.  No call here allocates device
// memory or synchronises, except pkv_device_status.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>

#include <nvtx3/nvToolsExt.h>

#include "cache_ops.cuh"
#include "decode_dispatch.cuh"
#include "decode_mma.cuh"
#include "decode_mma_e4m3.cuh"

namespace pkv {

// The device status word (one per device), read by pkv_device_status.
__device__ unsigned int g_status_word;

// An NVTX range around each call that launches device work, so a timeline
// (ncu, Nsight Systems) shows the library's calls by name.  Header-only NVTX:
// without a tool attached a range costs a few nanoseconds.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

namespace {

constexpr int kMaxDevices = 64;
std::atomic<unsigned int*> g_status_ptr[kMaxDevices];

// Device address of the status word on the current device, looked up once
// per device (the host-side symbol is only a handle, never a device address).
cudaError_t status_word(unsigned int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    unsigned int* p = g_status_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_status_word);
        if (e != cudaSuccess) return e;
        g_status_ptr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
}

int elem_size(pkv_dtype dt) {
    switch (dt) {
        case PKV_F32: return 4;
        case PKV_F16: return 2;
        case PKV_BF16: return 2;
        case PKV_E4M3: return 1;
    }
    return 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

// The address a kernel on the current device can use for p: device memory of
// this device, managed memory, or page-locked host memory (through its mapped
// view).  Pageable host memory and other devices' memory are refused.
bool device_view(const void* p, void** out) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();  // clear the error this query leaves behind
        return false;
    }
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    switch (at.type) {
        case cudaMemoryTypeDevice:
            if (at.device != dev) return false;
            *out = at.devicePointer ? at.devicePointer : const_cast<void*>(p);
            return true;
        case cudaMemoryTypeManaged:
            *out = at.devicePointer ? at.devicePointer : const_cast<void*>(p);
            return true;
        case cudaMemoryTypeHost:
            if (!at.devicePointer) return false;
            *out = at.devicePointer;
            return true;
        default:
            return false;
    }
}

constexpr int kNumSMs = 148;


// The decode behind both entry points.  e4m3: the pages hold E4M3 codes with
// per-KV-head scales and dtype is the type of q and out.
int decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                const float* k_scale, const float* v_scale, int scale_per_block, bool e4m3,
                const int32_t* block_tables, const int32_t* context_lens,
                const int32_t* seq_order, int num_seqs, int num_q_heads, int num_kv_heads,
                int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                int max_context_len, float scale, int sliding_window, pkv_dtype dtype,
                int partition_size, void* workspace, size_t workspace_bytes, pkv_kernel kernel,
                pkv_stream_t stream) {
    // ---- host-side checks (nothing has been launched if these fail)
    const int es = elem_size(dtype);
    if (dtype == PKV_E4M3 || (e4m3 && dtype == PKV_F32)) return PKV_EINVAL;
    if (es == 0 || num_seqs < 0 || num_seqs > 65535 || num_q_heads <= 0 || num_kv_heads <= 0 ||
        num_q_heads % num_kv_heads != 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
        max_context_len < 0 || (int64_t)max_context_len > (int64_t)max_blocks_per_seq * block_size ||
        !std::isfinite(scale) || sliding_window < 0 || partition_size < 0 ||
        (partition_size != 0 && (partition_size % 64 != 0 || partition_size > 8192)))
        return PKV_EINVAL;
    if (kernel != PKV_KERNEL_AUTO && kernel != PKV_KERNEL_SIMT && kernel != PKV_KERNEL_MMA)
        return PKV_EINVAL;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PKV_EUNSUPPORTED;
    if (block_size != 16 && block_size != 32 && block_size != 64) return PKV_EUNSUPPORTED;
    if (dtype == PKV_F32 && head_dim == 256) return PKV_EUNSUPPORTED;
    if (e4m3 && head_dim == 64) return PKV_EUNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_EINVAL;
    if (e4m3 && (!k_scale || !v_scale || (scale_per_block != 0 && scale_per_block != 1)))
        return PKV_EINVAL;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_EINVAL;

    const int G = num_q_heads / num_kv_heads;
    // longest span a sequence attends to: with a window, at most the window
    // plus the part of its first block ahead of it
    const int span = sliding_window > 0
                         ? (int)std::min<int64_t>(max_context_len,
                                                  (int64_t)sliding_window + block_size - 1)
                         : max_context_len;
    const int P = partition_size ? partition_size
                                 : pkv_decode_default_partition(num_seqs, num_kv_heads, span);
    const int np = span > 0 ? ceil_div(span, P) : 1;
    if (np > 1) {
        const size_t need = pkv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads,
                                                      head_dim, span, P);
        if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PKV_EINVAL;
    }

    // the tensor-core kernel addresses the pool as one 2-D tensor of
    // num_blocks * Hkv * block_size rows with 32-bit TMA coordinates
    const bool mma_fits = dtype != PKV_F32 && G <= 16 &&
                          (int64_t)num_blocks * num_kv_heads * block_size < (1ll << 31);
    bool use_mma;
    if (kernel == PKV_KERNEL_MMA) {
        if (!kMmaBuilt || !mma_fits) return PKV_EUNSUPPORTED;
        use_mma = true;
    } else if (kernel == PKV_KERNEL_SIMT) {
        use_mma = false;
    } else {
        // E4M3 pages: the tensor cores for every group size (the conversions
        // would bound the CUDA-core kernel below the memory roofline)
        use_mma = kMmaBuilt && mma_fits && (G >= 4 || e4m3);
    }
    const int hg = use_mma ? (G <= 8 ? 8 : 16)
                           : (G % 4 == 0 && !e4m3 ? 4 : (G % 2 == 0 ? 2 : 1));
    const int head_chunks = (G + hg - 1) / hg;
    if ((int64_t)num_kv_heads * head_chunks > 65535) return PKV_EUNSUPPORTED;

    DecodeArgs a;
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.seq_order = seq_order;
    a.k_scale = e4m3 ? k_scale : nullptr;
    a.v_scale = e4m3 ? v_scale : nullptr;
    a.scale_per_block = e4m3 ? scale_per_block : 0;
    a.ws_o = static_cast<float*>(workspace);
    a.ws_ml = np > 1 ? a.ws_o + (int64_t)num_seqs * num_q_heads * np * head_dim : nullptr;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.group = G;
    a.head_chunks = head_chunks;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.max_tokens = max_blocks_per_seq * block_size;
    a.partition_size = P;
    a.max_partitions = np;
    a.block_size = block_size;
    a.window = sliding_window;
    a.scale_log2 = scale * 1.4426950408889634f;
    if (status_word(&a.status) != cudaSuccess) return PKV_ECUDA;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (e4m3 && use_mma) {
        e = dtype == PKV_F16 ? decode_mma_e4m3_f16(a, head_dim, block_size, hg, s)
                             : decode_mma_e4m3_bf16(a, head_dim, block_size, hg, s);
    } else if (e4m3) {
        e = dtype == PKV_F16 ? decode_simt_e4m3_f16(a, head_dim, block_size, hg, s)
                             : decode_simt_e4m3_bf16(a, head_dim, block_size, hg, s);
    } else if (use_mma) {
        e = dtype == PKV_F16 ? decode_mma_f16(a, head_dim, block_size, hg, s)
                             : decode_mma_bf16(a, head_dim, block_size, hg, s);
    } else {
        switch (dtype) {
            case PKV_F32: e = decode_simt_f32(a, head_dim, block_size, hg, s); break;
            case PKV_F16: e = decode_simt_f16(a, head_dim, block_size, hg, s); break;
            default: e = decode_simt_bf16(a, head_dim, block_size, hg, s); break;
        }
    }
    if (e == cudaErrorInvalidValue) return PKV_EUNSUPPORTED;
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" {

const char* pkv_status_string(int status) {
    switch (status) {
        case PKV_OK: return "ok";
        case PKV_EINVAL: return "invalid argument";
        case PKV_ENOMEM: return "no free block";
        case PKV_ENOSEQ: return "unknown sequence";
        case PKV_EEXIST: return "sequence exists";
        case PKV_EBOUNDS: return "index out of range";
        case PKV_ECUDA: return "CUDA error";
        case PKV_EUNSUPPORTED: return "unsupported configuration";
    }
    return "unknown status";
}

int pkv_version(void) { return 10000; }

int pkv_decode_has_kernel(pkv_kernel kernel) {
    return kernel == PKV_KERNEL_AUTO || kernel == PKV_KERNEL_SIMT ||
           (kernel == PKV_KERNEL_MMA && kMmaBuilt);
}

int pkv_decode_default_partition(int num_seqs, int num_kv_heads, int max_context_len) {
    // Partitions long enough that a CTA's start-up (table slice, first
    // stages) and the split-K merge are small against its streaming time:
    // 4096 tokens when there are many (sequence, KV head) units -- a batch of
    // many sequences, whose CTAs are plentiful and of mixed length -- else
    // 2048, so a few very long sequences still give enough CTAs to balance.
    // Measured on B200 with the longest sequences scheduled first (seq_order):
    // on the GQA batch (2048 units) 4096 beats 2048 by 5 % (bf16) and 9 %
    // (E4M3); on the long-context batch (64 units) 2048 beats 4096 by 2-7 %
    // and 1024 by 0-2 %.  Small batches get shorter partitions so the grid
    // still fills every SM (3 CTAs each) about twice.
    const int64_t units = (int64_t)(num_seqs > 0 ? num_seqs : 1) * (num_kv_heads > 0 ? num_kv_heads : 1);
    int p = units >= 1024 ? 4096 : 2048;
    while (p > 64 && units * ceil_div(max_context_len > 0 ? max_context_len : 1, p) < 6 * kNumSMs)
        p /= 2;
    return p;
}

size_t pkv_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_context_len, int partition_size) {
    if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
        partition_size < 0)
        return 0;
    const int p = partition_size ? partition_size
                                 : pkv_decode_default_partition(num_seqs, num_kv_heads,
                                                                max_context_len);
    const int64_t np = ceil_div(max_context_len, p);
    if (np <= 1) return 0;
    return (size_t)num_seqs * num_q_heads * np * (head_dim + 2) * sizeof(float);
}


int pkv_paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, const int32_t* context_lens,
                               const int32_t* seq_order, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int num_blocks, int max_context_len,
                               float scale, int sliding_window, pkv_dtype dtype,
                               int partition_size, void* workspace, size_t workspace_bytes,
                               pkv_kernel kernel, pkv_stream_t stream) {
    NvtxRange range("pkv_paged_attention_decode");
    return pkv::decode_impl(out, q, k_cache, v_cache, nullptr, nullptr, 0, false, block_tables,
                            context_lens, seq_order, num_seqs, num_q_heads, num_kv_heads,
                            head_dim, block_size, max_blocks_per_seq, num_blocks,
                            max_context_len, scale, sliding_window, dtype, partition_size,
                            workspace, workspace_bytes, kernel, stream);
}

int pkv_paged_attention_decode_e4m3(void* out, const void* q, const void* k_cache,
                                    const void* v_cache, const float* k_scale,
                                    const float* v_scale, int scale_per_block,
                                    const int32_t* block_tables,
                                    const int32_t* context_lens, const int32_t* seq_order,
                                    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int max_blocks_per_seq, int num_blocks,
                                    int max_context_len, float scale, int sliding_window,
                                    pkv_dtype dtype, int partition_size, void* workspace,
                                    size_t workspace_bytes, pkv_kernel kernel,
                                    pkv_stream_t stream) {
    NvtxRange range("pkv_paged_attention_decode_e4m3");
    return pkv::decode_impl(out, q, k_cache, v_cache, k_scale, v_scale, scale_per_block, true,
                            block_tables,
                            context_lens, seq_order, num_seqs, num_q_heads, num_kv_heads,
                            head_dim, block_size, max_blocks_per_seq, num_blocks,
                            max_context_len, scale, sliding_window, dtype, partition_size,
                            workspace, workspace_bytes, kernel, stream);
}

int pkv_kv_cache_append(void* k_cache, void* v_cache, const void* k, const void* v,
                        const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                        int head_dim, int block_size, int num_blocks, pkv_dtype dtype,
                        pkv_stream_t stream) {
    NvtxRange range("pkv_kv_cache_append");
    const int es = elem_size(dtype);
    if (es == 0 || num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || (head_dim * es) % 16 != 0)
        return PKV_EINVAL;
    if (num_tokens == 0) return PKV_OK;
    if (!k_cache || !v_cache || !k || !v || !slot_mapping) return PKV_EINVAL;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v))
        return PKV_EINVAL;
    unsigned int* st;
    if (status_word(&st) != cudaSuccess) return PKV_ECUDA;
    cudaError_t e = launch_kv_append(k_cache, v_cache, k, v, slot_mapping, num_tokens,
                                     num_kv_heads, head_dim * es, block_size, num_blocks, st,
                                     reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int pkv_kv_cache_append_e4m3(void* k_cache, void* v_cache, const void* k, const void* v,
                             const float* k_scale, const float* v_scale, int scale_per_block,
                             const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int num_blocks, pkv_dtype in_dtype,
                             pkv_stream_t stream) {
    NvtxRange range("pkv_kv_cache_append_e4m3");
    if ((in_dtype != PKV_F16 && in_dtype != PKV_BF16) || num_tokens < 0 || num_kv_heads <= 0 ||
        head_dim <= 0 || head_dim % 16 != 0 || block_size <= 0 || num_blocks <= 0 ||
        (scale_per_block != 0 && scale_per_block != 1))
        return PKV_EINVAL;
    if (num_tokens == 0) return PKV_OK;
    if (!k_cache || !v_cache || !k || !v || !slot_mapping || !k_scale || !v_scale)
        return PKV_EINVAL;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k) || !aligned16(v))
        return PKV_EINVAL;
    unsigned int* st;
    if (status_word(&st) != cudaSuccess) return PKV_ECUDA;
    cudaError_t e = launch_kv_append_e4m3(k_cache, v_cache, k, v, k_scale, v_scale, slot_mapping,
                                          num_tokens, num_kv_heads, head_dim, block_size,
                                          num_blocks, in_dtype == PKV_BF16, scale_per_block != 0,
                                          st,
                                          reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int pkv_copy_blocks(void* k_cache, void* v_cache, const int32_t* block_pairs, int num_pairs,
                    int num_kv_heads, int head_dim, int block_size, int num_blocks,
                    pkv_dtype dtype, pkv_stream_t stream) {
    NvtxRange range("pkv_copy_blocks");
    const int es = elem_size(dtype);
    if (es == 0 || num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0)
        return PKV_EINVAL;
    const int64_t block_bytes = (int64_t)num_kv_heads * block_size * head_dim * es;
    if (block_bytes % 16 != 0) return PKV_EINVAL;
    if (num_pairs == 0) return PKV_OK;
    if (!k_cache || !v_cache || !block_pairs) return PKV_EINVAL;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return PKV_EINVAL;
    unsigned int* st;
    if (status_word(&st) != cudaSuccess) return PKV_ECUDA;
    cudaError_t e = launch_copy_blocks(k_cache, v_cache, block_pairs, num_pairs, block_bytes,
                                       num_blocks, st, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int pkv_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                    const int32_t* block_pairs, int num_pairs, int src_num_blocks,
                    int dst_num_blocks, int num_kv_heads, int head_dim, int block_size,
                    pkv_dtype dtype, pkv_stream_t stream) {
    NvtxRange range("pkv_swap_blocks");
    const int es = elem_size(dtype);
    if (es == 0 || num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0 ||
        num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return PKV_EINVAL;
    const int64_t block_bytes = (int64_t)num_kv_heads * block_size * head_dim * es;
    if (block_bytes % 16 != 0) return PKV_EINVAL;
    if (num_pairs == 0) return PKV_OK;
    if (!dst_k || !dst_v || !src_k || !src_v || !block_pairs) return PKV_EINVAL;
    void *dk, *dv, *sk, *sv, *pp;
    if (!device_view(dst_k, &dk) || !device_view(dst_v, &dv) || !device_view(src_k, &sk) ||
        !device_view(src_v, &sv) || !device_view(block_pairs, &pp))
        return PKV_EINVAL;
    if (!aligned16(dk) || !aligned16(dv) || !aligned16(sk) || !aligned16(sv)) return PKV_EINVAL;
    unsigned int* st;
    if (status_word(&st) != cudaSuccess) return PKV_ECUDA;
    cudaError_t e = launch_swap_blocks(dk, dv, sk, sv, static_cast<const int32_t*>(pp), num_pairs,
                                       block_bytes, src_num_blocks, dst_num_blocks, st,
                                       reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int pkv_debug_wait_timeout(long long limit_cycles, pkv_stream_t stream) {
    if (limit_cycles < 1 || limit_cycles > kWaitCycles) return PKV_EINVAL;
    unsigned int* st;
    if (status_word(&st) != cudaSuccess) return PKV_ECUDA;
    cudaError_t e = launch_wait_timeout(limit_cycles, st, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

int pkv_device_status(unsigned int* flags, int clear) {
    if (!flags) return PKV_EINVAL;
    if (cudaDeviceSynchronize() != cudaSuccess) return PKV_ECUDA;
    if (cudaMemcpyFromSymbol(flags, g_status_word, sizeof(unsigned int)) != cudaSuccess)
        return PKV_ECUDA;
    if (clear) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero)) != cudaSuccess)
            return PKV_ECUDA;
    }
    return PKV_OK;
}

}  // extern "C"
