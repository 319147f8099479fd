/*
 * pagedkv -- PagedAttention decode for NVIDIA B200 (sm_100a), C ABI.
 *
 * What the library does, in the pages' terms:
 *   A sequence's key/value cache is stored in fixed-size blocks of
 *   `block_size` tokens (16 by default in vLLM) that sit anywhere in a
 *   physical pool; a per-sequence block table maps logical block i to a
 *   physical block, like an OS page table ("What is PagedAttention ..."
 *   §How it works; lastdictionary "PagedAttention"; "pagedattention vllm"
 *   §PagedAttention Design).  The attention kernel reads keys and values
 *   through that table and computes the same result as attention over a
 *   contiguous cache ("pagedattention vllm" §Attention Computation).
 *   Blocks are handed out on demand from a free list, shared between
 *   sequences with a common prefix under reference counts, and copied before
 *   a sequence writes into a shared one ("pagedattention vllm"
 *   §Copy-on-Write Sharing, §Memory Management).
 *
 * Layouts (all row-major, contiguous):
 *   q, out          [num_seqs, num_q_heads, head_dim]           dtype
 *   k_cache,v_cache [num_blocks, num_kv_heads, block_size, head_dim] dtype
 *   block_tables    int32 [num_seqs, max_blocks_per_seq]; entry i of row b is
 *                   the physical block holding tokens [i*bs, (i+1)*bs) of
 *                   sequence b; entries past ceil(len/bs) are never read.
 *                   4-byte entries, as the pages size the table
 *                   ("pagedattention vllm" §Implementation Details).
 *   context_lens    int32 [num_seqs]
 *   k, v (append)   [num_tokens, num_kv_heads, head_dim]        dtype
 *   slot_mapping    int64 [num_tokens]; slot = block * block_size + offset,
 *                   negative = padding token, nothing written
 *   block_pairs     int32 [num_pairs][2] = (src, dst)
 * Query head h reads KV head h / (num_q_heads / num_kv_heads).
 *
 * Conventions:
 *   - Device calls take device pointers, enqueue work on `stream` and return
 *     without synchronising.  The caller owns all memory; device calls never
 *     allocate.  Pointers must not alias (K and V are separate buffers).
 *   - Every call returns a pkv_status.  Arguments are checked on the host
 *     before anything is launched (PKV_EINVAL / PKV_EUNSUPPORTED); a failed
 *     launch gives PKV_ECUDA.
 *   - Data the host cannot see (table entries, lengths, slots, pairs) is
 *     checked on the device: an access that would leave its buffer is not
 *     made, and a bit is set in the device status word
 *     (pkv_device_status).  Results of such a call are unspecified.
 *   - The allocator (pkv_alloc_*) is host-only and not thread-safe: one
 *     caller at a time per allocator.
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA stream type (identical to cudaStream_t); NULL = legacy default. */
typedef struct CUstream_st* pkv_stream_t;

typedef enum {
    PKV_OK = 0,
    PKV_EINVAL = -1,       /* bad argument (host-side check) */
    PKV_ENOMEM = -2,       /* allocator: no free block */
    PKV_ENOSEQ = -3,       /* allocator: unknown sequence id */
    PKV_EEXIST = -4,       /* allocator: sequence id already present */
    PKV_EBOUNDS = -5,      /* an index out of range */
    PKV_ECUDA = -6,        /* a CUDA runtime call or launch failed */
    PKV_EUNSUPPORTED = -7  /* valid but not built (e.g. head_dim 96) */
} pkv_status;

/* Element types.  PKV_E4M3: FP8 codes (1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits; largest finite value 448, code 0x7F / 0xFF = NaN), the
 * storage of quantised KV pages; the cache operations move them as bytes and
 * the decode reads them through pkv_paged_attention_decode_e4m3. */
typedef enum { PKV_F32 = 0, PKV_F16 = 1, PKV_BF16 = 2, PKV_E4M3 = 3 } pkv_dtype;

/* Decode kernel choice.  AUTO takes the tensor-core kernel for 16-bit caches
 * with a query group of 4 to 16 heads per KV head and for E4M3 pages with a
 * group of at most 16, else the CUDA-core one. */
typedef enum { PKV_KERNEL_AUTO = 0, PKV_KERNEL_SIMT = 1, PKV_KERNEL_MMA = 2 } pkv_kernel;

/* Device status bits (pkv_device_status) */
#define PKV_DEV_BAD_BLOCK 1u    /* a table entry or copy pair outside [0, num_blocks) */
#define PKV_DEV_BAD_LEN 2u      /* a context length < 0 or past the caller's bounds */
#define PKV_DEV_BAD_SLOT 4u     /* a slot at or past num_blocks * block_size */
#define PKV_DEV_TIMEOUT 8u      /* a bounded wait inside a kernel gave up */
#define PKV_DEV_BAD_ORDER 16u   /* a seq_order entry outside [0, num_seqs), or a bad work item */
#define PKV_DEV_DRAIN_TIMEOUT 32u /* after a wait gave up, a copy still had not landed
                                     when the kernel's block left (see below) */
#define PKV_DEV_BAD_GROUP 64u   /* a shared-prefix group whose members disagree
                                   (prefix length, table entries) */
/*
 * After PKV_DEV_TIMEOUT the outputs of that call are lost (the blocks whose
 * wait gave up wrote nothing).  With PKV_DEV_DRAIN_TIMEOUT as well, a page
 * copy may have landed in shared memory after its block left, i.e. in a
 * later block's: treat every result computed on the device since the flag
 * was last cleared as lost, this call's and those of kernels that ran beside
 * it.  Neither happens with valid inputs on a healthy device.
 */

/* Name of a status code. */
PKV_API const char* pkv_status_string(int status);

/* ABI version: major * 10000 + minor * 100 + patch. */
PKV_API int pkv_version(void);

/* 1 if the library was compiled with decode kernel `kernel`, else 0. */
PKV_API int pkv_decode_has_kernel(pkv_kernel kernel);

/*
 * Partition size the decode uses when `partition_size` is 0, for this shape
 * (max_context_len: the longest span attended, i.e. at most the window plus
 * block_size - 1 under a sliding window).  When even 2048-token partitions
 * give at most 3 CTAs per SM (148 SMs), the smallest multiple of 64 that
 * keeps the grid within that one wave.  Otherwise 4096 tokens when
 * num_seqs * num_kv_heads >= 1024, else 2048, halved while the grid would
 * hold fewer than ~6 CTAs per SM.  Tuned with a longest-first seq_order;
 * without one, shorter partitions can be faster when lengths are very uneven.
 */
PKV_API int pkv_decode_default_partition(int num_seqs, int num_kv_heads, int max_context_len);

/*
 * Bytes of device workspace pkv_paged_attention_decode needs: float32 partial
 * results (m, l and the normalised output of each partition) for sequences
 * longer than one partition.  0 when max_context_len fits one partition.
 * partition_size 0 = pkv_decode_default_partition(num_seqs, num_kv_heads,
 * max_context_len).  Returns 0 for invalid sizes.
 */
PKV_API size_t pkv_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                                 int head_dim, int max_context_len, int partition_size);

/*
 * Paged decode attention: for every sequence b and query head h,
 *   out[b,h,:] = softmax_t(scale * q[b,h,:] . k_t) weighted sum of v_t,
 * over the tokens t < context_lens[b] (the last sliding_window of them when
 * sliding_window > 0), k_t and v_t read from the physical
 * block block_tables[b][t / block_size] at offset t % block_size
 * ("pagedattention vllm" §Attention Computation: gather physical blocks,
 * compute as if contiguous).  A sequence with length 0 gets a zero row.
 *
 * The context of each sequence is cut into partitions of `partition_size`
 * tokens; one CTA takes one (sequence, KV head, partition) with a tile of
 * that KV head's query heads (up to 4 on the CUDA cores, 8 or 16 on the
 * tensor cores); sequences longer than one partition are merged by a
 * log-sum-exp reduce over the workspace.  Accumulation is float32;
 * `out` is written in `dtype` (round to nearest even).
 *
 * Arguments:
 *   out, q, k_cache, v_cache, block_tables, context_lens: device pointers,
 *       layouts above; k_cache and v_cache 16-byte aligned.
 *   num_q_heads % num_kv_heads == 0; head_dim in {64, 128, 256};
 *   block_size in {16, 32, 64}; dtype f32, f16 or bf16.
 *   seq_order: NULL, or a device int32 permutation of [0, num_seqs): the
 *       order in which sequences are scheduled onto the GPU.  It changes no
 *       result (every row is computed the same way), only the timing: with
 *       the longest sequences first (pkv_decode_schedule_order) the grid
 *       ends without a tail of long partitions.  An entry outside
 *       [0, num_seqs) is skipped and flagged (PKV_DEV_BAD_ORDER); a repeated
 *       entry leaves some row unwritten.
 *   max_context_len: host-side upper bound of context_lens, and
 *       <= max_blocks_per_seq * block_size.
 *   sliding_window: 0 to attend to the whole context, else W > 0: sequence
 *       b attends only to its last W tokens, [max(0, L_b - W), L_b)
 *       ("pagedattention vllm" §Advanced Features: sliding-window models
 *       cache only recent blocks).  Table entries of blocks that lie wholly
 *       before the window are never read (they may be -1 once released,
 *       pkv_alloc_slide_window).  The workspace is then sized with
 *       max_context_len = min(max_context_len, W + block_size - 1).
 *   partition_size: 0 for the default, else a multiple of 64 in [64, 8192].
 *   workspace: device memory of at least pkv_decode_workspace_size(...)
 *       bytes, 16-byte aligned; may be NULL when that size is 0.
 *   kernel: PKV_KERNEL_AUTO, or force one kernel (for measurements);
 *       PKV_KERNEL_MMA needs f16/bf16 and a group of at most 16 heads.
 * Returns PKV_OK, PKV_EINVAL, PKV_EUNSUPPORTED or PKV_ECUDA.
 */
PKV_API int pkv_paged_attention_decode(void* out, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* block_tables,
                               const int32_t* context_lens, const int32_t* seq_order,
                               int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int max_blocks_per_seq, int num_blocks,
                               int max_context_len, float scale, int sliding_window,
                               pkv_dtype dtype, int partition_size, void* workspace,
                               size_t workspace_bytes, pkv_kernel kernel,
                               pkv_stream_t stream);

/*
 * Paged decode attention over FP8 E4M3 pages ("pagedattention vllm"
 * §Comparison with Alternatives: the paged layout combines with a quantised
 * cache).  Page element x of KV head g in physical block n stands for the
 * value E4M3(x) * k_scale[g] (keys) or E4M3(x) * v_scale[g] (values) -- or,
 * with scale_per_block = 1, k_scale[n * Hkv + g] and v_scale[n * Hkv + g],
 * one scale per page -- and the result is pkv_paged_attention_decode's over
 * those values:
 *   out[b,h,:] = softmax_t(scale * q[b,h,:] . (k_scale * E4M3(k_t)))
 *                weighted sum of v_scale * E4M3(v_t),   g = h / (Hq/Hkv).
 * Each code is widened exactly (every E4M3 value is a binary16 value).  The
 * tensor-core kernel (AUTO for groups of at most 16 heads) multiplies fp16
 * operands with fp32 accumulation: q enters it scaled by a power of two that
 * puts max |q| of the CTA's heads in [2^14, 2^15) (exact unless an element
 * falls below the fp16 normal range there), each softmax weight p enters as
 * two fp16 terms, hi = fp16(p) and lo = fp16(p - hi) (about 22 significant
 * bits, so the weights' rounding stays far below the fp16 / bf16 output
 * tolerance whatever the values' magnitudes), and the logits are multiplied
 * by scale * k_scale (and the power of two) in fp32.
 * The CUDA-core kernel works in fp32 throughout, k_scale folded into q and
 * v_scale into the accumulator (per page: into that page's logits and
 * weights).  The tensor-core kernel keeps each warp's P.V sums in units of a
 * reference V scale vref: a page whose v_scale lies in [vref, 128 vref]
 * enters with its weights times v_scale / vref (then at most 2^15, still an
 * fp16 hi + lo pair with p's precision), any other page first moves vref to
 * its v_scale / 8 and rescales the fp32 sums; the output is multiplied by
 * vref.  The sums stay in fp32 range for the per-page V scales of a KV head
 * within a factor 2^80 of one another, each at least 2^-120 (the kernel
 * takes 8 / v_scale in fp32).
 *
 * Arguments as pkv_paged_attention_decode, plus:
 *   k_cache, v_cache: device E4M3 codes [num_blocks, Hkv, block_size, head_dim].
 *   k_scale, v_scale: device float32 [num_kv_heads] (scale_per_block 0) or
 *       [num_blocks][num_kv_heads] (scale_per_block 1), finite and > 0 (not
 *       checked on the device: the caller's quantisation scales).
 *   dtype: PKV_F16 or PKV_BF16, the type of q and out.
 *   head_dim in {128, 256} (a page row must be at least 128 bytes).
 *   kernel: PKV_KERNEL_AUTO, SIMT or MMA (MMA: groups of at most 16 heads).
 *   The workspace is sized as for the 16-bit decode
 *   (pkv_decode_workspace_size).
 * Returns PKV_OK, PKV_EINVAL, PKV_EUNSUPPORTED or PKV_ECUDA.
 */
PKV_API int pkv_paged_attention_decode_e4m3(
    void* out, const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
    const float* v_scale, int scale_per_block, const int32_t* block_tables,
    const int32_t* context_lens,
    const int32_t* seq_order, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
    int sliding_window, pkv_dtype dtype, int partition_size, void* workspace,
    size_t workspace_bytes, pkv_kernel kernel, pkv_stream_t stream);

/*
 * Size of the workspace compiled into the library for
 * pkv_paged_attention_decode_static_ws: 64 MiB per GPU.
 */
#define PKV_STATIC_WORKSPACE_BYTES (64u * 1024u * 1024u)

/*
 * pkv_paged_attention_decode for callers that cannot allocate device memory.
 * The pages have no counterpart of this call: it exists for callers such as a
 * plugin inside a host application that owns all device memory and forbids
 * cudaMalloc, or a serving loop that must not take cudaMalloc's implicit
 * device synchronisation.  Same arguments, checks, kernels and results as
 * pkv_paged_attention_decode, minus the workspace: the partition scratch comes
 * from a fixed array of PKV_STATIC_WORKSPACE_BYTES inside the library, which
 * every GPU that loads the library's device code holds until the process
 * exits.  The call itself allocates nothing.
 *
 *   - Returns PKV_EBOUNDS, before launching anything, when the shape needs
 *     more scratch than that (pkv_decode_workspace_size(...) >
 *     PKV_STATIC_WORKSPACE_BYTES), e.g. far longer contexts or bigger
 *     batches; use pkv_paged_attention_decode with a caller workspace then.
 *   - The first call in a CUDA context (normally a device's primary context)
 *     looks up the array's device address there (cudaGetSymbolAddress, with
 *     that context current) and keeps it for that context; make that first
 *     call before any stream capture begins.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents.  Nothing in it needs to start at zero, but calls that can
 *     overlap on the GPU (different streams, no ordering between them) race
 *     on it: order them, or use the caller-workspace entry point.
 */
PKV_API int pkv_paged_attention_decode_static_ws(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* seq_order,
    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
    int sliding_window, pkv_dtype dtype, int partition_size, pkv_kernel kernel,
    pkv_stream_t stream);

/* Largest shared-prefix group (sequences) of the shared-prefix decode. */
#define PKV_MAX_PREFIX_GROUP 64

/*
 * Shared-prefix decode: pkv_paged_attention_decode's result, computed so that
 * a prefix of blocks held by several sequences is read from memory once for
 * all of them.  Sequences that hold the same physical blocks for their first
 * S tokens share those keys and values: parallel samples forked from one
 * prompt keep the prompt's blocks until they write into them
 * ("pagedattention vllm" §Copy-on-Write Sharing), and requests that hit the
 * same cached prompt blocks hold those (§Advanced Features, prefix caching).
 *   - A group is up to PKV_MAX_PREFIX_GROUP sequences whose tables agree on
 *     their first S / block_size entries (S a positive multiple of
 *     block_size, at most each member's length); seq_prefix_len[b] = S for
 *     its members, 0 for sequences in no group (pkv_decode_prefix_groups
 *     finds the groups of a batch from its tables).
 *   - The group pass runs on the tensor cores: one CTA per (prefix partition,
 *     KV head, chunk of up to 16 rows) of a group, whose rows are the
 *     members' query heads of that KV head, so each prefix page is read once
 *     and feeds every member's heads, as a query group shares its KV head.
 *   - The regular pass takes tokens [S, L_b) of every sequence ([0, L_b)
 *     outside groups) with the usual kernel choice; the log-sum-exp reduce
 *     merges the prefix's partial results with the rest's.
 * The summation order differs from pkv_paged_attention_decode's, so results
 * agree within rounding, not bit for bit.
 *
 * Arguments as pkv_paged_attention_decode (dtype PKV_F16 or PKV_BF16,
 * sliding_window 0, query groups of at most 16 heads per KV head), plus:
 *   seq_prefix_len: device int32 [num_seqs].
 *   group_members: device int32 [num_groups][max_group_size]: batch indices
 *       of each group's members, -1 after the last; a sequence is in at most
 *       one group.  May be NULL when num_groups is 0.
 *   num_groups >= 0; 1 <= max_group_size <= PKV_MAX_PREFIX_GROUP.
 *   max_prefix_len: host-side bound of seq_prefix_len, a multiple of
 *       block_size, <= max_context_len.
 *   workspace: pkv_decode_prefix_groups_workspace_size(...) bytes, 16-byte
 *       aligned (NULL when that is 0).
 * A member whose prefix length differs from its group's first member's, a
 * member whose table differs from the first member's over the prefix, or a
 * prefix that is not whole blocks of its sequence sets PKV_DEV_BAD_GROUP
 * (results unspecified); a sequence with seq_prefix_len > 0 that is in no
 * group is not detected (its result is unspecified).
 * Returns PKV_OK, PKV_EINVAL, PKV_EUNSUPPORTED or PKV_ECUDA.
 */
PKV_API int pkv_paged_attention_decode_prefix_groups(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* seq_order,
    const int32_t* seq_prefix_len, const int32_t* group_members, int num_groups,
    int max_group_size, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
    int block_size, int max_blocks_per_seq, int num_blocks, int max_context_len,
    int max_prefix_len, float scale, pkv_dtype dtype, int partition_size, void* workspace,
    size_t workspace_bytes, pkv_kernel kernel, pkv_stream_t stream);

/*
 * Workspace bytes of pkv_paged_attention_decode_prefix_groups: float32
 * partial results of ceil(max_prefix_len / P) prefix partitions and
 * ceil(max_context_len / P) further partitions per (sequence, query head);
 * partition_size 0 = pkv_decode_default_partition(num_seqs, num_kv_heads,
 * max_context_len).  0 when no row needs a merge; 0 for invalid sizes.
 */
PKV_API size_t pkv_decode_prefix_groups_workspace_size(int num_seqs, int num_q_heads,
                                                       int num_kv_heads, int head_dim,
                                                       int max_context_len, int max_prefix_len,
                                                       int partition_size);

/*
 * Host helper: the shared-prefix groups of a batch, from its host block
 * tables and lengths.  Sequences are bucketed by the physical block of their
 * first full block; each bucket, in batch order, is cut into groups of at
 * most max_group_size (2 .. PKV_MAX_PREFIX_GROUP) members, and a group's
 * prefix is the longest run of table entries all its members share over
 * their full blocks.  Groups whose prefix has fewer than min_prefix_blocks
 * (>= 1) blocks, and single sequences, are left out.
 *   seq_prefix_len: [num_seqs] out: the prefix tokens (0 outside groups).
 *   group_members: [group_capacity][max_group_size] out, -1 padded; a
 *       capacity of num_seqs / 2 always suffices.
 *   *num_groups: out.
 * Returns PKV_OK, PKV_EINVAL or PKV_EBOUNDS (capacity too small; the outputs
 * are then incomplete).
 */
PKV_API int pkv_decode_prefix_groups(const int32_t* block_tables, const int32_t* context_lens,
                                     int num_seqs, int max_blocks_per_seq, int block_size,
                                     int max_group_size, int min_prefix_blocks,
                                     int32_t* seq_prefix_len, int32_t* group_members,
                                     int group_capacity, int* num_groups);

/*
 * Host helper: order_out[0..n) = the sequence indices sorted by decreasing
 * context length (ties by index), for the seq_order argument of the decode.
 * context_lens is a host array.  Returns PKV_OK or PKV_EINVAL.
 */
PKV_API int pkv_decode_schedule_order(const int32_t* context_lens, int num_seqs,
                                      int32_t* order_out);

/*
 * Host helper: the work list of a decode -- every (sequence, partition) pair
 * that has tokens to attend, longest partition first (ties by sequence, then
 * partition), for pkv_paged_attention_decode_items and
 * pkv_paged_attention_decode_e4m3_items.  Sequence b of length L (host
 * context_lens) attends to [lo, L), lo = max(0, L - sliding_window) with a
 * window (else 0); its partitions of partition_size tokens start at the
 * block holding lo, so it has ceil((L - lo + lo % block_size) /
 * partition_size) of them, and one (empty: the zero row) when L is 0.
 * items_out receives 2 int32 per pair, (sequence, partition); *num_items
 * their number.  partition_size must be the decode's (a multiple of 64 in
 * [64, 8192]: resolve a default with pkv_decode_default_partition).
 * Returns PKV_OK, PKV_EINVAL (bad sizes, a negative length) or PKV_EBOUNDS
 * (more pairs than item_capacity; *num_items then holds the number needed).
 */
PKV_API int pkv_decode_schedule_items(const int32_t* context_lens, int num_seqs, int block_size,
                                      int partition_size, int sliding_window,
                                      int32_t* items_out, int item_capacity, int* num_items);

/*
 * pkv_paged_attention_decode over a work list instead of a schedule order:
 * one CTA per (item, KV head) -- no CTA for a partition a sequence does not
 * have, and partitions in the list's order (pkv_decode_schedule_items:
 * longest first).  items: device int32 pairs (sequence, partition),
 * num_items of them, 1 <= num_items <= 65535; partition_size: the one the
 * list was cut with (> 0).  Every partition a sequence has must be listed
 * once (else rows stay unwritten or partial); an item whose sequence is
 * outside [0, num_seqs) or whose partition is negative is skipped and
 * flagged (PKV_DEV_BAD_ORDER), one past the sequence's partitions is
 * skipped.  Results equal pkv_paged_attention_decode's with the same
 * partition_size, bit for bit.  The other arguments and the workspace are
 * as there.
 */
PKV_API int pkv_paged_attention_decode_items(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* items,
    int num_items, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
    int max_blocks_per_seq, int num_blocks, int max_context_len, float scale, int sliding_window,
    pkv_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
    pkv_kernel kernel, pkv_stream_t stream);

/* pkv_paged_attention_decode_e4m3 over a work list (as above). */
PKV_API int pkv_paged_attention_decode_e4m3_items(
    void* out, const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
    const float* v_scale, int scale_per_block, const int32_t* block_tables,
    const int32_t* context_lens, const int32_t* items, int num_items, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
    int num_blocks, int max_context_len, float scale, int sliding_window, pkv_dtype dtype,
    int partition_size, void* workspace, size_t workspace_bytes, pkv_kernel kernel,
    pkv_stream_t stream);

/*
 * KV append: the key and value of each new token go into the slot the block
 * manager gave it ("What is PagedAttention ..." §How it works: blocks are
 * filled as the answer grows):
 *   k_cache[s / bs, h, s % bs, :] = k[t, h, :], same for v, s = slot_mapping[t];
 * s < 0 writes nothing.  Two tokens with the same non-negative slot in one
 * call leave that slot undefined.  A slot >= num_blocks * block_size is
 * skipped and flagged (PKV_DEV_BAD_SLOT).  Bit copy; any head_dim with
 * head_dim * element size a multiple of 16 bytes.
 */
PKV_API int pkv_kv_cache_append(void* k_cache, void* v_cache, const void* k, const void* v,
                        const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                        int head_dim, int block_size, int num_blocks, pkv_dtype dtype,
                        pkv_stream_t stream);

/*
 * KV append into E4M3 pages: as pkv_kv_cache_append, but each element is
 * quantised on the way in:
 *   k_cache[s / bs, h, s % bs, d] = E4M3(k[t, h, d] / k_scale[h]),
 * same for v with v_scale; with scale_per_block = 1 the scale is that of the
 * page the slot lies in, k_scale[(s / bs) * Hkv + h] (set before the block's
 * first token).  The division is a float32 division (correctly
 * rounded), the code the nearest E4M3 value (ties to even), magnitudes
 * beyond 448 saturate to 448 and NaN stays NaN.
 *   k, v: device [num_tokens, Hkv, head_dim] in in_dtype (PKV_F16 or PKV_BF16),
 *       16-byte aligned; head_dim a multiple of 16.
 *   k_scale, v_scale: device float32 [num_kv_heads] or, with
 *       scale_per_block = 1, [num_blocks][num_kv_heads].
 *   k_cache, v_cache: device E4M3 codes, 16-byte aligned.
 * Slots as pkv_kv_cache_append (negative skipped, past the pool flagged
 * PKV_DEV_BAD_SLOT).  Returns PKV_OK, PKV_EINVAL or PKV_ECUDA.
 */
PKV_API int pkv_kv_cache_append_e4m3(void* k_cache, void* v_cache, const void* k, const void* v,
                                     const float* k_scale, const float* v_scale,
                                     int scale_per_block, const int64_t* slot_mapping,
                                     int num_tokens,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int num_blocks, pkv_dtype in_dtype, pkv_stream_t stream);

/*
 * Copy-on-write block copies ("pagedattention vllm" §Copy-on-Write Sharing:
 * a shared block is copied before a sequence modifies it): for each pair,
 * k_cache[dst] = k_cache[src] and v_cache[dst] = v_cache[src], the whole block
 * (all heads, all slots).  block_pairs: device int32 [num_pairs][2].
 * A dst must not appear twice nor also be a src in the same call.  Pairs with
 * an id outside [0, num_blocks) are skipped and flagged (PKV_DEV_BAD_BLOCK).
 */
PKV_API int pkv_copy_blocks(void* k_cache, void* v_cache, const int32_t* block_pairs,
                    int num_pairs, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, pkv_dtype dtype, pkv_stream_t stream);

/*
 * Swap pages between two pools, one of which may be page-locked host memory
 * (cudaHostAlloc / cudaHostRegister, e.g. torch's pin_memory): for each pair,
 * dst_k[dst] = src_k[src] and dst_v[dst] = src_v[src], whole blocks of
 * num_kv_heads x block_size x head_dim elements ("pagedattention vllm"
 * §Memory Management: swapping).  One kernel moves all pairs, reading or
 * writing the host pool directly over the host link.  Pools are checked on
 * the host: pageable host memory is refused (PKV_EINVAL), since the GPU
 * cannot reach it.  block_pairs: int32 [num_pairs][2] (src, dst) in device or
 * page-locked host memory; pairs outside their pools are skipped and flagged
 * (PKV_DEV_BAD_BLOCK).
 */
PKV_API int pkv_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                            const int32_t* block_pairs, int num_pairs, int src_num_blocks,
                            int dst_num_blocks, int num_kv_heads, int head_dim, int block_size,
                            pkv_dtype dtype, pkv_stream_t stream);

/*
 * Reads (and with clear != 0, resets) the device status word of the current
 * device: an OR of PKV_DEV_* bits set by earlier calls.  Synchronises the
 * device.
 */
PKV_API int pkv_device_status(unsigned int* flags, int clear);

/*
 * Failure-detection self-test.  Every wait inside the decode kernels (for a
 * page copy to land) is bounded: after ~2 s it gives up, sets
 * PKV_DEV_TIMEOUT, lets its own copies still in flight land (again bounded)
 * and leaves, so a broken input or a lost copy ends the kernel with a status
 * the host reads instead of a hung GPU.  This launches one thread that makes
 * the same bounded wait on a barrier that nothing completes, giving up after
 * limit_cycles clock cycles (1 .. 4e9; ~0.5 ms per 1e6 at 2 GHz); afterwards
 * pkv_device_status reports PKV_DEV_TIMEOUT and the device stays usable.
 * Returns PKV_OK, PKV_EINVAL or PKV_ECUDA.
 */
PKV_API int pkv_debug_wait_timeout(long long limit_cycles, pkv_stream_t stream);

/* ------------------------------------------------------------------------
 * Host block allocator ("pagedattention vllm" §Memory Management: a free list,
 * allocate on demand, free when the sequence completes; §Copy-on-Write
 * Sharing: reference counts, free at zero, copy before writing a shared
 * block).  Rules:
 *   - the free list is a stack; a new allocator pops 0, 1, 2, ...;
 *   - add_seq(n) takes ceil(n / block_size) blocks in logical order, or none;
 *   - append_slot: a full (or absent) last block -> take a new block; a
 *     shared last block (count > 1) -> take a block dst, report (last, dst)
 *     for pkv_copy_blocks, drop one reference to last and use dst; the sole
 *     holder writes in place.  Returns the token's slot;
 *   - fork(parent, child): child gets the parent's table and length, every
 *     block one more reference;
 *   - free_seq: drop one reference per table entry in logical order, push
 *     each block that reaches zero;
 *   - a failed call changes nothing.
 * ------------------------------------------------------------------------ */
typedef struct pkv_alloc pkv_alloc;

typedef struct {
    int32_t num_blocks;
    int32_t block_size;
    int32_t free_blocks;
    int32_t used_blocks;     /* blocks with a reference count > 0 */
    int32_t shared_blocks;   /* blocks with a reference count > 1 */
    int32_t num_seqs;
    int64_t refcount_sum;    /* = block-table entries of the resident sequences */
    int64_t logical_tokens;  /* sum of sequence lengths (resident and swapped) */
    int32_t num_host_blocks;
    int32_t free_host_blocks;
    int32_t swapped_seqs;
    int32_t reserved;
} pkv_alloc_stats_t;

/* num_blocks > 0, block_size > 0.  *out = new allocator (free with destroy). */
PKV_API int pkv_alloc_create(int num_blocks, int block_size, pkv_alloc** out);
/* The same with a host pool of num_host_blocks >= 0 blocks for swapping. */
PKV_API int pkv_alloc_create_swap(int num_blocks, int num_host_blocks, int block_size,
                                  pkv_alloc** out);
PKV_API void pkv_alloc_destroy(pkv_alloc* a);
/* New sequence holding num_tokens >= 0 tokens. */
PKV_API int pkv_alloc_add_seq(pkv_alloc* a, int64_t seq_id, int num_tokens);
PKV_API int pkv_alloc_fork(pkv_alloc* a, int64_t parent, int64_t child);
/* One more token for seq_id: *slot gets its slot; *cow_src / *cow_dst get the
 * block copy to run first, or -1 / -1. */
PKV_API int pkv_alloc_append_slot(pkv_alloc* a, int64_t seq_id, int64_t* slot,
                          int32_t* cow_src, int32_t* cow_dst);
/* append_slot for n sequences in order.  slots[i] gets sequence i's slot;
 * cow_pairs ([n][2] capacity) gets the copies in order, *num_cow their
 * count.  Stops at the first failure: *num_done sequences were appended. */
PKV_API int pkv_alloc_append_slots(pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* slots,
                           int32_t* cow_pairs, int* num_cow, int* num_done);
PKV_API int pkv_alloc_free_seq(pkv_alloc* a, int64_t seq_id);
PKV_API int pkv_alloc_seq_len(const pkv_alloc* a, int64_t seq_id, int* len);
/* Copies seq_id's table to out (capacity entries); *n_out = its length.
 * PKV_EBOUNDS (and nothing copied) when capacity is too small. */
PKV_API int pkv_alloc_block_table(const pkv_alloc* a, int64_t seq_id, int32_t* out,
                          int capacity, int* n_out);
/* Batch tables for a decode call: row i of tables ([n][max_blocks]) gets the
 * table of seq_ids[i], padded with `fill`; context_lens[i] its length. */
PKV_API int pkv_alloc_build_block_tables(const pkv_alloc* a, const int64_t* seq_ids, int n,
                                 int32_t* tables, int max_blocks, int32_t fill,
                                 int32_t* context_lens);
PKV_API int pkv_alloc_refcount(const pkv_alloc* a, int32_t block, int* out);
PKV_API int pkv_alloc_stats(const pkv_alloc* a, pkv_alloc_stats_t* out);
/* Free blocks in the order they will be handed out. */
PKV_API int pkv_alloc_free_list(const pkv_alloc* a, int32_t* out, int capacity, int* n_out);

/*
 * Swapping ("pagedattention vllm" §Memory Management: blocks can be swapped
 * to CPU memory, trading latency for capacity).  swap_out moves a resident
 * sequence to the host pool: for each table entry in logical order it takes a
 * host block (LIFO free stack, a new pool pops 0, 1, 2, ...), reports the pair
 * (device block, host block) and drops one reference to the device block
 * (a block other sequences still share stays on the device); the table then
 * holds host block ids.  swap_in does the reverse: one new device block per
 * entry, pairs (host block, device block), host blocks pushed back in logical
 * order.  Run pkv_swap_blocks on the pairs, in stream order, before the
 * device blocks are reused.  A swapped sequence cannot be appended to,
 * forked or put in a decode batch (PKV_EINVAL) until swapped in.
 * pairs: host int32 [capacity][2]; *num_pairs = table length (PKV_EBOUNDS
 * and nothing done when it exceeds capacity); PKV_ENOMEM when the target
 * pool lacks free blocks.
 */
PKV_API int pkv_alloc_swap_out(pkv_alloc* a, int64_t seq_id, int32_t* pairs, int capacity,
                               int* num_pairs);
PKV_API int pkv_alloc_swap_in(pkv_alloc* a, int64_t seq_id, int32_t* pairs, int capacity,
                              int* num_pairs);
PKV_API int pkv_alloc_is_swapped(const pkv_alloc* a, int64_t seq_id, int* swapped);

/*
 * Sliding window ("pagedattention vllm" §Advanced Features: with sliding-window
 * attention only recent blocks are kept): every block of resident sequence
 * seq_id that lies wholly before its last `window` tokens ((j+1) * block_size
 * <= len - window) drops one reference (freed at zero) and its table entry
 * becomes -1; the length is unchanged.  *released = entries released by this
 * call.  Entries that are -1 are skipped by fork, free, swap and the decode
 * with the same or a smaller window.  window <= 0 -> PKV_EINVAL.
 */
PKV_API int pkv_alloc_slide_window(pkv_alloc* a, int64_t seq_id, int window, int* released);

/*
 * Prefix cache ("pagedattention vllm" §vLLM Integration and §Advanced
 * Features: automatic prefix caching shares common prompt starts across
 * requests; "PagedAttention" glossary entry: prompt caching lets later
 * requests that begin the same way skip that work).
 *
 * pkv_alloc_add_seq_prefix adds sequence seq_id for a prompt of num_tokens
 * token ids (host int32).  Full block j of the prompt (tokens [j*bs, (j+1)*bs))
 * has the key (registration id of block j-1, or 0 for j = 0; its bs token
 * ids).  For j = 0, 1, ... while a registered block has block j's key, the
 * sequence takes that block (one more reference; an evictable block comes
 * back); the first miss ends the walk, so a hit always means the whole prompt
 * up to that block is identical.  The remaining blocks are taken in logical
 * order (as pkv_alloc_add_seq) and each full one is registered under its key
 * with the next registration id; the partial last block is never registered.
 * *cached_tokens = hits * block_size: the prompt tokens whose K/V are already
 * in the pool (the caller computes and appends only the rest).  All or nothing
 * (PKV_ENOMEM, PKV_EEXIST).
 *
 * A registered block whose reference count reaches zero (any release:
 * free_seq, a copy-on-write source, swap_out, slide_window) is kept with its
 * contents on the evictable list, least recently released first, instead of
 * the free stack.  Every allocation pops the free stack and, only when it is
 * empty, evicts the head of the evictable list (unregistering it); capacity
 * checks count both.  Registered blocks are always full prompt blocks, so no
 * append ever writes into one.  pkv_alloc_free_list lists the free stack only.
 */
PKV_API int pkv_alloc_add_seq_prefix(pkv_alloc* a, int64_t seq_id, const int32_t* tokens,
                                     int num_tokens, int* cached_tokens);
/* Registered blocks (in use or evictable) and evictable blocks. */
PKV_API int pkv_alloc_cache_stats(const pkv_alloc* a, int32_t* cached_blocks,
                                  int32_t* evictable_blocks);
/* Evictable blocks, next to be evicted first. */
PKV_API int pkv_alloc_evictable_list(const pkv_alloc* a, int32_t* out, int capacity, int* n_out);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */
