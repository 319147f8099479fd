// The C ABI of pagedkv (declared in include/pagedkv.h): host-side argument
// checks, kernel selection and launches.  No call here allocates device
// memory or synchronises, except pkv_device_status.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>

#include <nvtx3/nvToolsExt.h>

#include "cache_ops.cuh"
#include "context_cache.h"
#include "decode_request.h"
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
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
std::once_flag g_ctx_once;
}  // namespace

cudaError_t current_context_id(unsigned long long* id) {
    std::call_once(g_ctx_once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    if (!g_ctx_get_current || !g_ctx_get_id) return cudaErrorNotSupported;
    CUcontext c = nullptr;
    if (g_ctx_get_current(&c) != CUDA_SUCCESS) return cudaErrorUnknown;
    *id = 0;
    if (c && g_ctx_get_id(c, id) != CUDA_SUCCESS) return cudaErrorUnknown;
    return cudaSuccess;
}

namespace {

PerContext g_status_addr;

// Device address of the status word in the current context, looked up once
// per context (the host-side symbol is only a handle, never a device address).
cudaError_t status_word(unsigned int** out) {
    void* p = nullptr;
    const cudaError_t e = per_context_value(g_status_addr, &p, [](void** o) {
        return cudaGetSymbolAddress(o, g_status_word);
    });
    *out = static_cast<unsigned int*>(p);
    return e;
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


}  // namespace

int plan_decode(const DecodeRequest& r, DecodePlan* plan) {
    const int es = elem_size(r.dtype);
    if (r.dtype == PKV_E4M3 || (r.e4m3 && r.dtype == PKV_F32)) return PKV_EINVAL;
    if (es == 0 || r.num_seqs < 0 || r.num_seqs > 65535 || r.num_q_heads <= 0 ||
        r.num_kv_heads <= 0 || r.num_q_heads % r.num_kv_heads != 0 ||
        r.max_blocks_per_seq <= 0 || r.num_blocks <= 0 || r.max_context_len < 0 ||
        (int64_t)r.max_context_len > (int64_t)r.max_blocks_per_seq * r.block_size ||
        !std::isfinite(r.scale) || r.sliding_window < 0 || r.partition_size < 0 ||
        (r.partition_size != 0 && (r.partition_size % 64 != 0 || r.partition_size > 8192)))
        return PKV_EINVAL;
    if (r.kernel != PKV_KERNEL_AUTO && r.kernel != PKV_KERNEL_SIMT && r.kernel != PKV_KERNEL_MMA)
        return PKV_EINVAL;
    // a work list: cut with an explicit partition size, instead of a schedule order
    if (r.items && (r.seq_order || r.partition_size == 0 ||
                    (r.num_seqs > 0 && (r.num_items < 1 || r.num_items > 65535))))
        return PKV_EINVAL;
    if (r.head_dim != 64 && r.head_dim != 128 && r.head_dim != 256) return PKV_EUNSUPPORTED;
    if (r.block_size != 16 && r.block_size != 32 && r.block_size != 64) return PKV_EUNSUPPORTED;
    if (r.dtype == PKV_F32 && r.head_dim == 256) return PKV_EUNSUPPORTED;
    if (r.e4m3 && r.head_dim == 64) return PKV_EUNSUPPORTED;
    plan->empty = r.num_seqs == 0;
    if (plan->empty) return PKV_OK;
    if (!r.out || !r.q || !r.k_cache || !r.v_cache || !r.block_tables || !r.context_lens)
        return PKV_EINVAL;
    if (r.e4m3 && (!r.k_scale || !r.v_scale || (r.scale_per_block != 0 && r.scale_per_block != 1)))
        return PKV_EINVAL;
    if (!aligned16(r.out) || !aligned16(r.q) || !aligned16(r.k_cache) || !aligned16(r.v_cache))
        return PKV_EINVAL;

    const int G = r.num_q_heads / r.num_kv_heads;
    // longest span a sequence attends to: with a window, at most the window
    // plus the part of its first block ahead of it
    plan->span = r.sliding_window > 0
                     ? (int)std::min<int64_t>(r.max_context_len,
                                              (int64_t)r.sliding_window + r.block_size - 1)
                     : r.max_context_len;
    plan->partition_size = r.partition_size ? r.partition_size
                                            : pkv_decode_default_partition(
                                                  r.num_seqs, r.num_kv_heads, plan->span);
    plan->max_partitions = plan->span > 0 ? ceil_div(plan->span, plan->partition_size) : 1;
    plan->workspace_bytes =
        plan->max_partitions > 1
            ? pkv_decode_workspace_size(r.num_seqs, r.num_q_heads, r.num_kv_heads, r.head_dim,
                                        plan->span, plan->partition_size)
            : 0;

    // the tensor-core kernel addresses the pool as one 2-D tensor of
    // num_blocks * Hkv * block_size rows with 32-bit TMA coordinates
    const bool mma_fits = r.dtype != PKV_F32 && G <= 16 &&
                          (int64_t)r.num_blocks * r.num_kv_heads * r.block_size < (1ll << 31);
    if (r.kernel == PKV_KERNEL_MMA) {
        if (!kMmaBuilt || !mma_fits) return PKV_EUNSUPPORTED;
        plan->use_mma = true;
    } else if (r.kernel == PKV_KERNEL_SIMT) {
        plan->use_mma = false;
    } else {
        // E4M3 pages: the tensor cores for every group size (the conversions
        // would bound the CUDA-core kernel below the memory roofline)
        plan->use_mma = kMmaBuilt && mma_fits && (G >= 4 || r.e4m3);
    }
    plan->heads_per_cta = plan->use_mma ? (G <= 8 ? 8 : 16)
                                        : (G % 4 == 0 && !r.e4m3 ? 4 : (G % 2 == 0 ? 2 : 1));
    plan->head_chunks = (G + plan->heads_per_cta - 1) / plan->heads_per_cta;
    if ((int64_t)r.num_kv_heads * plan->head_chunks > 65535) return PKV_EUNSUPPORTED;
    return PKV_OK;
}

namespace {

// Kernel arguments of a checked decode call whose workspace rows hold ws_slots
// partial results.
DecodeArgs decode_args(const DecodeRequest& r, const DecodePlan& plan, void* workspace,
                       int ws_slots) {
    DecodeArgs a;
    a.out = r.out;
    a.q = r.q;
    a.k_cache = r.k_cache;
    a.v_cache = r.v_cache;
    a.block_tables = r.block_tables;
    a.context_lens = r.context_lens;
    a.seq_order = r.seq_order;
    a.items = r.items;
    a.num_items = r.items ? r.num_items : 0;
    a.k_scale = r.e4m3 ? r.k_scale : nullptr;
    a.v_scale = r.e4m3 ? r.v_scale : nullptr;
    a.scale_per_block = r.e4m3 ? r.scale_per_block : 0;
    a.seq_start = nullptr;
    a.group_members = nullptr;
    a.group_stride = 0;
    a.after_groups = 0;
    a.ws_slots = ws_slots;
    a.ws_o = static_cast<float*>(workspace);
    a.ws_ml = ws_slots > 1
                  ? a.ws_o + (int64_t)r.num_seqs * r.num_q_heads * ws_slots * r.head_dim
                  : nullptr;
    a.num_seqs = r.num_seqs;
    a.num_q_heads = r.num_q_heads;
    a.num_kv_heads = r.num_kv_heads;
    a.group = r.num_q_heads / r.num_kv_heads;
    a.head_chunks = plan.head_chunks;
    a.max_blocks_per_seq = r.max_blocks_per_seq;
    a.num_blocks = r.num_blocks;
    a.max_tokens = r.max_blocks_per_seq * r.block_size;
    a.partition_size = plan.partition_size;
    a.max_partitions = plan.max_partitions;
    a.block_size = r.block_size;
    a.window = r.sliding_window;
    a.scale_log2 = r.scale * 1.4426950408889634f;
    a.status = nullptr;
    return a;
}

// The partition kernel the plan chose (and the reduce when rows merge).
int launch_decode_kernels(const DecodeRequest& r, const DecodePlan& plan, const DecodeArgs& a,
                   cudaStream_t s) {
    const int D = r.head_dim, bs = r.block_size, hg = plan.heads_per_cta;
    cudaError_t e;
    if (r.e4m3 && plan.use_mma) {
        e = r.dtype == PKV_F16 ? decode_mma_e4m3_f16(a, D, bs, hg, s)
                               : decode_mma_e4m3_bf16(a, D, bs, hg, s);
    } else if (r.e4m3) {
        e = r.dtype == PKV_F16 ? decode_simt_e4m3_f16(a, D, bs, hg, s)
                               : decode_simt_e4m3_bf16(a, D, bs, hg, s);
    } else if (plan.use_mma) {
        e = r.dtype == PKV_F16 ? decode_mma_f16(a, D, bs, hg, s) : decode_mma_bf16(a, D, bs, hg, s);
    } else {
        switch (r.dtype) {
            case PKV_F32: e = decode_simt_f32(a, D, bs, hg, s); break;
            case PKV_F16: e = decode_simt_f16(a, D, bs, hg, s); break;
            default: e = decode_simt_bf16(a, D, bs, hg, s); break;
        }
    }
    if (e == cudaErrorInvalidValue) return PKV_EUNSUPPORTED;
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

}  // namespace

int run_decode(const DecodeRequest& r, const DecodePlan& plan, void* workspace,
               size_t workspace_bytes, cudaStream_t s) {
    if (plan.empty) return PKV_OK;
    if (plan.workspace_bytes > 0 &&
        (!workspace || workspace_bytes < plan.workspace_bytes || !aligned16(workspace)))
        return PKV_EINVAL;
    DecodeArgs a = decode_args(r, plan, workspace, plan.max_partitions);
    if (status_word(&a.status) != cudaSuccess) return PKV_ECUDA;
    return launch_decode_kernels(r, plan, a, s);
}

namespace {

// Workspace slots per row of the shared-prefix decode: the prefix's
// partitions, then the rest's.
int prefix_slots(int max_prefix_len, int partition_size) {
    return max_prefix_len > 0 ? ceil_div(max_prefix_len, partition_size) : 0;
}

int prefix_groups_impl(const DecodeRequest& r, const int32_t* seq_prefix_len,
                       const int32_t* group_members, int num_groups, int max_group_size,
                       int max_prefix_len, void* workspace, size_t workspace_bytes,
                       cudaStream_t s) {
    if (r.sliding_window != 0 || (r.dtype != PKV_F16 && r.dtype != PKV_BF16 &&
                                  r.dtype != PKV_F32))
        return PKV_EINVAL;
    if (num_groups < 0 || num_groups > 65535 || max_group_size < 1 ||
        max_group_size > PKV_MAX_PREFIX_GROUP || max_prefix_len < 0 ||
        max_prefix_len % std::max(r.block_size, 1) != 0 || max_prefix_len > r.max_context_len)
        return PKV_EINVAL;
    DecodePlan plan;
    int rc = plan_decode(r, &plan);
    if (rc != PKV_OK || plan.empty) return rc;
    if (r.dtype == PKV_F32) return PKV_EUNSUPPORTED;  // the group pass is fp16 / bf16
    if (!seq_prefix_len || (num_groups > 0 && !group_members)) return PKV_EINVAL;
    const int G = r.num_q_heads / r.num_kv_heads;
    const int pslots = prefix_slots(max_prefix_len, plan.partition_size);
    const int ws_slots = pslots + plan.max_partitions;
    const size_t need = ws_slots > 1 ? (size_t)r.num_seqs * r.num_q_heads * ws_slots *
                                           (r.head_dim + 2) * sizeof(float)
                                     : 0;
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
        return PKV_EINVAL;
    // the group pass: tiles of 8 or 16 (member, head) rows on the tensor cores
    const bool groups = num_groups > 0 && pslots > 0;
    const int rows = max_group_size * G;
    const int nh = rows <= 8 ? 8 : 16;
    const int chunks = ceil_div(rows, nh);
    if (groups && (!kMmaBuilt || G > 16 ||
                   (int64_t)r.num_blocks * r.num_kv_heads * r.block_size >= (1ll << 31) ||
                   (int64_t)r.num_kv_heads * chunks > 65535))
        return PKV_EUNSUPPORTED;

    DecodeArgs a = decode_args(r, plan, workspace, ws_slots);
    if (status_word(&a.status) != cudaSuccess) return PKV_ECUDA;
    a.seq_start = seq_prefix_len;
    if (groups) {
        DecodeArgs ag = a;
        ag.seq_order = nullptr;
        ag.group_members = group_members;
        ag.group_stride = max_group_size;
        ag.head_chunks = chunks;
        ag.max_partitions = pslots;
        const cudaError_t e =
            r.dtype == PKV_F16
                ? decode_mma_groups_f16(ag, r.head_dim, r.block_size, nh, num_groups, s)
                : decode_mma_groups_bf16(ag, r.head_dim, r.block_size, nh, num_groups, s);
        if (e == cudaErrorInvalidValue) return PKV_EUNSUPPORTED;
        if (e != cudaSuccess) return PKV_ECUDA;
        a.after_groups = 1;  // overlap the regular pass with the group pass's last wave
    }
    return launch_decode_kernels(r, plan, a, s);
}

// The decode behind both caller-workspace entry points.
int decode_impl(const DecodeRequest& r, void* workspace, size_t workspace_bytes,
                pkv_stream_t stream) {
    DecodePlan plan;
    const int rc = plan_decode(r, &plan);
    if (rc != PKV_OK) return rc;
    return run_decode(r, plan, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
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
    // and 1024 by 0-2 %.  Over the work list (no CTAs without tokens) 4096
    // still leads on the GQA batch: E4M3 pages 83.9, 85.2, 85.3, 87.0,
    // 89.3 us at 4096, 3072, 2560, 2048, 1536 tokens; bf16 134.0 to 140.6 us.  Small batches get shorter partitions so the grid
    // still fills every SM (3 CTAs each) about twice.
    //
    // Little work in all (a grid under one wave of 3 CTAs per SM even at
    // 2048 tokens, e.g. a few sequences behind a sliding window): one wave of
    // CTAs as long as that allows, so each SM slot pays the start-up once.
    // Measured on B200, long contexts behind a 4096-token window (64 units):
    // 768 and 1024 tokens 11-12 % faster than 256 and 512, 2048 26 % slower.
    const int64_t units = (int64_t)(num_seqs > 0 ? num_seqs : 1) * (num_kv_heads > 0 ? num_kv_heads : 1);
    const int64_t len = max_context_len > 0 ? max_context_len : 1;
    const int64_t slots = 3 * kNumSMs;
    if (units * ceil_div(len, 2048) <= slots) {
        int q = 64;
        while (q < 2048 && units * ceil_div(len, q) > slots) q += 64;
        return q;
    }
    int p = units >= 1024 ? 4096 : 2048;
    while (p > 64 && units * ceil_div(len, p) < 6 * kNumSMs) p /= 2;
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
    const DecodeRequest r{out, q, k_cache, v_cache, nullptr, nullptr, 0, false, block_tables,
                          context_lens, seq_order, num_seqs, num_q_heads, num_kv_heads,
                          head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len,
                          scale, sliding_window, dtype, partition_size, kernel};
    return pkv::decode_impl(r, workspace, workspace_bytes, stream);
}

int pkv_paged_attention_decode_items(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* items,
    int num_items, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int num_blocks, int max_context_len, float scale, int sliding_window,
    pkv_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
    pkv_kernel kernel, pkv_stream_t stream) {
    NvtxRange range("pkv_paged_attention_decode_items");
    if (!items && num_seqs > 0) return PKV_EINVAL;
    DecodeRequest r{out, q, k_cache, v_cache, nullptr, nullptr, 0, false, block_tables,
                    context_lens, nullptr, num_seqs, num_q_heads, num_kv_heads,
                    head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len,
                    scale, sliding_window, dtype, partition_size, kernel};
    r.items = items;
    r.num_items = num_items;
    return pkv::decode_impl(r, workspace, workspace_bytes, stream);
}

int pkv_paged_attention_decode_e4m3_items(
    void* out, const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
    const float* v_scale, int scale_per_block, const int32_t* block_tables,
    const int32_t* context_lens, const int32_t* items, int num_items, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
    int num_blocks, int max_context_len, float scale, int sliding_window, pkv_dtype dtype,
    int partition_size, void* workspace, size_t workspace_bytes, pkv_kernel kernel,
    pkv_stream_t stream) {
    NvtxRange range("pkv_paged_attention_decode_e4m3_items");
    if (!items && num_seqs > 0) return PKV_EINVAL;
    DecodeRequest r{out, q, k_cache, v_cache, k_scale, v_scale, scale_per_block, true,
                    block_tables, context_lens, nullptr, num_seqs, num_q_heads,
                    num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                    max_context_len, scale, sliding_window, dtype, partition_size, kernel};
    r.items = items;
    r.num_items = num_items;
    return pkv::decode_impl(r, workspace, workspace_bytes, stream);
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
    const DecodeRequest r{out, q, k_cache, v_cache, k_scale, v_scale, scale_per_block, true,
                          block_tables, context_lens, seq_order, num_seqs, num_q_heads,
                          num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                          max_context_len, scale, sliding_window, dtype, partition_size, kernel};
    return pkv::decode_impl(r, workspace, workspace_bytes, stream);
}

size_t pkv_decode_prefix_groups_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                               int head_dim, int max_context_len,
                                               int max_prefix_len, int partition_size) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        max_context_len < 0 || max_prefix_len < 0 || max_prefix_len > max_context_len ||
        partition_size < 0)
        return 0;
    const int p = partition_size ? partition_size
                                 : pkv_decode_default_partition(num_seqs, num_kv_heads,
                                                                max_context_len);
    const int64_t slots = pkv::prefix_slots(max_prefix_len, p) +
                          (max_context_len > 0 ? ceil_div(max_context_len, p) : 1);
    if (slots <= 1) return 0;
    return (size_t)num_seqs * num_q_heads * slots * (head_dim + 2) * sizeof(float);
}

int pkv_paged_attention_decode_prefix_groups(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* seq_order,
    const int32_t* seq_prefix_len, const int32_t* group_members, int num_groups,
    int max_group_size, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int max_blocks_per_seq, int num_blocks, int max_context_len,
    int max_prefix_len, float scale, pkv_dtype dtype, int partition_size, void* workspace,
    size_t workspace_bytes, pkv_kernel kernel, pkv_stream_t stream) {
    NvtxRange range("pkv_paged_attention_decode_prefix_groups");
    const DecodeRequest r{out, q, k_cache, v_cache, nullptr, nullptr, 0, false, block_tables,
                          context_lens, seq_order, num_seqs, num_q_heads, num_kv_heads,
                          head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len,
                          scale, 0, dtype, partition_size, kernel};
    return pkv::prefix_groups_impl(r, seq_prefix_len, group_members, num_groups, max_group_size,
                                   max_prefix_len, workspace, workspace_bytes,
                                   reinterpret_cast<cudaStream_t>(stream));
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
