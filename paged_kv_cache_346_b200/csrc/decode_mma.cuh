// Paged decode attention on the tensor cores, for query groups of 4 to 16
// heads per KV head with fp16 / bf16 caches.
//
// With G query heads sharing one KV head ("Paged Attention" glossary,
// systemdesign.academy: grouped-query attention lets several heads share one
// set of keys and values), each K/V page feeds G dot products per token: for
// G >= 4 the two products of a CTA's tile are small dense contractions,
//   S[t, h] = sum_d K[t, d] Q[h, d]   8-head tiles  (M = tokens, N = heads, K = dims)
//   S^T[h, t] = sum_d Q[h, d] K[t, d] 16-head tiles (M = heads, N = tokens, K = dims)
//   O^T[d, h] = sum_t V[t, d] P[h, t]               (M = dims, N = heads, K = tokens)
// done with mma.sync m16n8k16 (fp16/bf16 inputs, fp32 accumulation).  With
// 8 heads, S puts the warp's 16 tokens in M (an S^T tile would leave half of
// M empty): one MMA per 16-dim step; one movmatrix.trans per 8 tokens turns
// the rounded P into the B fragment of P^T.  A 16-head tile's S^T
// accumulator already has that layout.  P never leaves registers.
//
// Pages are staged with 2-D tiled TMA (cp.async.bulk.tensor) over the cache
// viewed as [N * Hkv * BS rows, D columns], boxes of 64 columns x 16 rows,
// 128-byte swizzle: row r of a box keeps its 16-byte chunk c at position
// c ^ (r % 8), so the ldmatrix reads of 8 rows at one column hit 8 different
// bank groups.  Each warp streams its own 16-token slices through a private
// ring of stages (its lane 0 issues the copies): it copies a slice's
// fragments into registers, refills that stage at once and then does the
// math, with no CTA barrier until the final merge.  Everything else (table
// hoist, per-warp online softmax, warp merge, split-K workspace) mirrors the
// CUDA-core kernel.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "decode_common.cuh"
#include "lse_reduce.cuh"

namespace pkv {

constexpr bool kMmaBuilt = true;

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// transpose an 8 x 8 matrix of 16-bit values held in the mma fragment layout
// (lane (g, t4): row g, columns 2 t4 and 2 t4 + 1)
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t r;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}

template <typename T>
struct Mma;

template <>
struct Mma<__half> {
    __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
            "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    // round a pair to the mma input type; lo goes to the low half
    __device__ __forceinline__ static uint32_t pack(float lo, float hi, float& rlo, float& rhi) {
        __half2 h = __floats2half2_rn(lo, hi);
        float2 f = __half22float2(h);
        rlo = f.x;
        rhi = f.y;
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

template <>
struct Mma<__nv_bfloat16> {
    __device__ __forceinline__ static void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
            "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    __device__ __forceinline__ static uint32_t pack(float lo, float hi, float& rlo, float& rhi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        float2 f = __bfloat1622float2(h);
        rlo = f.x;
        rhi = f.y;
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

// Every warp streams its own 16-token slices through a private ring of
// STAGES stages (STAGES_ = 0: as many as fit 64 KB per CTA, at least 2), one
// 16-row TMA box per 64 columns of K and of V per slice, issued by the warp's
// lane 0: no barrier ties the warps together until the final merge.
template <int D, int BS, int NW, int STAGES_ = 0>
struct MmaCfg {
    static constexpr int TILE = 16 * NW;          // tokens per round of all warps
    static constexpr int NX = D / 64;             // 64-column boxes per row
    static constexpr int BOX_BYTES = 16 * 128;    // one box: 16 rows x 128 bytes
    static constexpr int SLICE_BYTES = 16 * D * 2;  // one warp's 16 tokens of K (or V)
    static constexpr int FIT = 65536 / (NW * 2 * SLICE_BYTES);
    static constexpr int STAGES = STAGES_ ? STAGES_ : (FIT >= 4 ? 4 : (FIT >= 2 ? FIT : 2));
    static constexpr int WARP_RING = STAGES * 2 * SLICE_BYTES;
    static constexpr int RING_BYTES = NW * WARP_RING;
    static_assert(BS % 16 == 0, "16-token slices");

    static int smem_bytes(int partition_size) {
        return 1024 + round_up(partition_size / BS * 4, 128) + 1024 + RING_BYTES;
    }
};

// NH = 8 or 16 query heads per CTA (the M rows of the QK product / the N
// columns of the PV product); heads past the group are zero rows.
//
// GROUPS: the group pass of the shared-prefix decode.  Sequences that hold
// the same physical blocks for their first S tokens (parallel samples forked
// from one prompt, requests that hit the same cached prompt blocks: "pagedattention
// vllm" §Copy-on-Write Sharing, §Advanced Features) form a group; one CTA
// takes (prefix partition, KV head, chunk of tile rows) of group blockIdx.z,
// whose tile rows are the (member, query head) pairs of that KV head,
// member-major, so every page of the shared prefix is read once for all
// members and feeds all their heads, as a query group shares its KV head's
// pages.  The prefix's partial results go to workspace slots [0, ceil(S/P))
// of each member row; the regular pass starts those sequences at token S and
// the log-sum-exp reduce merges both.
template <typename T, int D, int BS, int NH, int NW, int STAGES_, bool GROUPS = false>
__global__ void __launch_bounds__(NW * 32, (D <= 128 && NH == 8) ? 3 : 1)
    decode_mma_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
    using C = MmaCfg<D, BS, NW, STAGES_>;
    using M = Mma<T>;
    constexpr int TILE = C::TILE, NX = C::NX, BOX_BYTES = C::BOX_BYTES;
    constexpr int SLICE_BYTES = C::SLICE_BYTES, WARP_RING = C::WARP_RING;
    constexpr int STAGES = C::STAGES;
    constexpr int KSTEPS = D / 16;   // k-steps of the QK product, m-tiles of PV
    constexpr int RB = NH / 8;       // 8-head row blocks
    // Hold the warp's K/V fragments in registers and release the stage before
    // the math, when that keeps three CTAs per SM within the register file.
    constexpr bool EARLY = D <= 128 && NH == 8;

    extern __shared__ __align__(1024) unsigned char smem_mma[];
    __shared__ int s_abort;
    __shared__ int64_t s_row[GROUPS ? NH : 1];  // group pass: tile row -> sequence * Hq + head
    const GroupPassWait group_pass_wait{a};
    // Launched as a programmatic dependent of the kernel before it (usually
    // the KV append): the schedule, lengths and table (which that kernel does
    // not write) are read before griddepcontrol.wait, so the start-up of the
    // first wave overlaps it; the pages are read, and anything is written,
    // only after it (pdl_wait_before_pages).  The group pass waits first:
    // it releases its own dependent (the regular pass) as it starts.
    if (GROUPS) pdl_wait_before_pages(a);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int kvh = blockIdx.y / a.head_chunks;
    const int hc = blockIdx.y - kvh * a.head_chunks;
    // (sequence, partition): the group pass takes partition grid x of group z
    const CtaUnit unit = GROUPS ? CtaUnit{0, (int)blockIdx.x} : cta_unit(a, tid);
    const int part = unit.part;
    const int h0 = kvh * a.group + hc * NH;
    const bool reporter = (tid == 0 && part == 0 && blockIdx.y == 0);
    int b, nh, nmem = 0;
    const int32_t* members = nullptr;
    TablePrefetch pf{0, false};
    Span sp;
    if constexpr (GROUPS) {
        pdl_launch_dependents();  // the regular pass may start beside this grid
        members = a.group_members + (int64_t)blockIdx.z * a.group_stride;
        while (nmem < a.group_stride && members[nmem] >= 0) ++nmem;
        b = nmem > 0 ? members[0] : -1;
        if ((unsigned)b >= (unsigned)a.num_seqs) {
            if (nmem > 0 && reporter) flag(a.status, PKV_DEV_BAD_GROUP);
            return;
        }
        nh = min(NH, nmem * a.group - hc * NH);
        if (nh <= 0) return;
        sp = group_span(a, b, reporter);
        if (tid < NH) {  // this chunk's rows; a member with another prefix is flagged, skipped
            const int r = hc * NH + tid;
            int64_t row = -1;
            if (r < nmem * a.group) {
                const int m = members[r / a.group];
                if ((unsigned)m < (unsigned)a.num_seqs && a.seq_start[m] == sp.L)
                    row = (int64_t)m * a.num_q_heads + kvh * a.group + r % a.group;
                else if (r % a.group == 0)
                    flag(a.status, PKV_DEV_BAD_GROUP);
            }
            s_row[tid] = row;
        }
    } else {
        nh = min(NH, a.group - hc * NH);
        b = unit.b;
        if (b < 0) return;
        pf = table_prefetch(a, b, part, a.partition_size / BS, tid);
        sp = seq_span(a, b, reporter);
    }
    const int L = sp.L, np = sp.np;
    T* out = reinterpret_cast<T*>(a.out);
    if (L == 0) {
        if (!GROUPS && part == 0) {
            pdl_wait_before_pages(a);
            for (int i = tid; i < nh * D; i += NW * 32)
                out[((int64_t)b * a.num_q_heads + h0 + i / D) * D + i % D] = Elem<T>::from_f32(0.f);
        }
        return;
    }
    if (part >= np) return;
    // A sequence that fits one partition needs no merge: release the reduce
    // grid at once (it starts when every CTA of this grid has released it or
    // left, and its rows of one partition leave without waiting).  CTAs of
    // split sequences release it after their loop, so a grid of mostly split
    // sequences keeps the reduce from taking SM slots while it streams.
    if (sp.direct) pdl_launch_dependents();

    const int P = a.partition_size;
    const int t0 = sp.base + part * P;
    const int ntok = min(L, t0 + P) - t0;
    const int mask_lo = part == 0 ? sp.lo - sp.base : 0;  // tokens ahead of the window
    const int nblk = (ntok + BS - 1) / BS;
    // this warp's slices: tokens [k * TILE + warp * 16, + 16), k < nslices
    const int nslices = ntok > warp * 16 ? (ntok - warp * 16 + TILE - 1) / TILE : 0;

    uint64_t* full = reinterpret_cast<uint64_t*>(smem_mma);  // [NW][STAGES]
    int32_t* s_tab = reinterpret_cast<int32_t*>(smem_mma + 1024);
    unsigned char* s_kv;
    {
        const uint32_t base = smem_u32(smem_mma + 1024 + round_up(P / BS * 4, 128));
        const uint32_t aligned = (base + 1023u) & ~1023u;  // 128-byte swizzle: 1 KB atoms
        s_kv = smem_mma + 1024 + round_up(P / BS * 4, 128) + (aligned - base);
    }

    table_hoist(a, b, t0 / BS, nblk, pf, s_tab, tid, NW * 32);
    if (tid == 0) {
        s_abort = 0;
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmk)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv)) : "memory");
#pragma unroll
        for (int s = 0; s < NW * STAGES; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncthreads();

    const uint64_t pol = policy_evict_first();
    // this warp's ring and barriers, recomputed where used (no long-lived
    // 64-bit pointers next to the fragment registers)
    const uint32_t ring_s = smem_u32(s_kv) + (uint32_t)(warp * WARP_RING);
    auto issue = [&](int k, int stage) {  // this warp's slice k (lane 0 only)
        const int tok = k * TILE + warp * 16;
        const int y = (s_tab[tok / BS] * a.num_kv_heads + kvh) * BS + tok % BS;
        uint64_t* bar = full + warp * STAGES + stage;
        mbar_arrive_expect_tx(bar, (uint32_t)(2 * SLICE_BYTES));
        unsigned char* kd = s_kv + warp * WARP_RING + stage * 2 * SLICE_BYTES;
#pragma unroll
        for (int x = 0; x < NX; ++x) {
            tma_load_2d(kd + x * BOX_BYTES, &tmk, x * 64, y, bar, pol);
            tma_load_2d(kd + SLICE_BYTES + x * BOX_BYTES, &tmv, x * 64, y, bar, pol);
        }
    };
    if (!GROUPS) pdl_wait_before_pages(a);
    if (lane == 0) {
        const int pre = min(STAGES, nslices);
        for (int s = 0; s < pre; ++s) issue(s, s);
    }
    if constexpr (GROUPS) {
        // every member must hold the first member's blocks (else flagged; the
        // result then reads the first member's)
        const int32_t* t_first = a.block_tables + (int64_t)b * a.max_blocks_per_seq + t0 / BS;
        for (int i = tid; i < nblk * (nmem - 1); i += NW * 32) {
            const int m = members[1 + i / nblk];
            if ((unsigned)m < (unsigned)a.num_seqs &&
                a.block_tables[(int64_t)m * a.max_blocks_per_seq + t0 / BS + i % nblk] !=
                    t_first[i % nblk])
                flag(a.status, PKV_DEV_BAD_GROUP);
        }
    }

    // Q: dims 2 t4, 2 t4 + 1 (lo) and 8 + 2 t4, + 1 (hi) of a 16-dim step for
    // head g (and g + 8) -- the B column g of an 8-head tile's S, the A rows
    // g, g + 8 of a 16-head tile's S^T.
    constexpr int QR = NH == 8 ? 1 : 2;
    uint32_t qa[KSTEPS][2 * QR];  // [lo g, (lo g + 8,) hi g, (hi g + 8)]
    {
        const T* qb = reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.num_q_heads + h0) * D;
        const T* qr[QR];
#pragma unroll
        for (int r = 0; r < QR; ++r) {  // r = 0: head g, r = 1: head g + 8
            const int hh = g + 8 * r;
            if constexpr (GROUPS)
                qr[r] = s_row[hh] >= 0 ? reinterpret_cast<const T*>(a.q) + s_row[hh] * D : nullptr;
            else
                qr[r] = hh < nh ? qb + hh * D : nullptr;
        }
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
#pragma unroll
            for (int r = 0; r < QR; ++r) {
                uint32_t lo = 0, hi = 0;
                if (qr[r]) {
                    lo = *reinterpret_cast<const uint32_t*>(qr[r] + ks * 16 + 2 * t4);
                    hi = *reinterpret_cast<const uint32_t*>(qr[r] + ks * 16 + 8 + 2 * t4);
                }
                qa[ks][r] = lo;
                qa[ks][QR + r] = hi;
            }
        }
    }

    // softmax state: 8-head tiles keep it for heads 2 t4, 2 t4 + 1 (the S
    // columns of this lane; l per lane, summed at the end), 16-head tiles
    // for heads g + 8 rb (the S^T rows; l summed every slice)
    constexpr int MS = NH == 8 ? 2 : RB;
    float m[MS], l[MS];
#pragma unroll
    for (int j = 0; j < MS; ++j) {
        m[j] = -INFINITY;
        l[j] = 0.f;
    }
    float o[KSTEPS][RB][4];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb)
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[mt][rb][i] = 0.f;

    // ldmatrix row addresses: lane -> (token within the warp's 16, chunk parity)
    const int lrow = (lane >> 4) * 8 + (lane & 7);
    const int lchunk = (lane >> 3) & 1;

    const int swz = lrow & 7;

    for (int it = 0; it < nslices; ++it) {
        const int stage = it % STAGES;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(full + warp * STAGES + stage,
                                                          (uint32_t)((it / STAGES) & 1), a.status));
        if (!ok) {
            s_abort = 1;
            // let this warp's copies still in flight land (bounded) before
            // the CTA leaves
            if (lane == 0)
                drain_ring(full + warp * STAGES, STAGES, it, min(nslices, it + STAGES), a.status);
            break;
        }
        const int wvalid = ntok - (it * TILE + warp * 16);
        const int wlo = mask_lo - (it * TILE + warp * 16);
        const bool work = wlo < 16 && wlo < wvalid;
        const uint32_t kbase = ring_s + (uint32_t)(stage * 2 * SLICE_BYTES + lrow * 128);
        auto kaddr = [&](int ks) {
            const int chunk = ks * 2 + lchunk;  // 16-byte chunk of the row
            return kbase + (chunk >> 3) * BOX_BYTES + (((chunk & 7) ^ swz) << 4);
        };
        // EARLY: copy the warp's K and V fragments into registers, so the
        // stage goes back to the producer before the math runs
        uint32_t kf[EARLY ? KSTEPS : 1][4], vf[EARLY ? KSTEPS : 1][4];
        if (EARLY && work) {
#pragma unroll
            for (int ks = 0; ks < (EARLY ? KSTEPS : 1); ++ks) {
                ldsm_x4(kaddr(ks), kf[ks]);
                ldsm_x4_trans(kaddr(ks) + SLICE_BYTES, vf[ks]);
            }
        }
        auto math = [&]() {
            auto kfrag = [&](int ks, uint32_t (&kb)[4]) {
                // kb: token g dims 2 t4 (+1), token g dims 8 + 2 t4 (+1),
                // token g + 8 dims 2 t4 (+1), token g + 8 dims 8 + 2 t4 (+1)
                if constexpr (EARLY) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) kb[i] = kf[ks < (EARLY ? KSTEPS : 1) ? ks : 0][i];
                } else {
                    ldsm_x4(kaddr(ks), kb);
                }
            };
            // P enters the MMA in T.  bf16 keeps 8 significant bits, too few
            // for the weights: P = hi + lo, two bf16 terms (~16 bits), and
            // two P.V products.  fp16's 11 bits are kept as one term.
            constexpr bool SPLIT = std::is_same<T, __nv_bfloat16>::value;
            uint32_t pb[RB][2], pl[RB][2];
            float alpha_c[RB][2];
            // 2^x: the hardware approximation where the fragments sit in
            // registers (8-head tiles, head_dim <= 128); the other tiles keep
            // exp2f, which there holds the register count
            auto ex2 = [](float x) {
                if constexpr (EARLY)
                    return ex2_approx(x);
                else
                    return exp2f(x);
            };
            if constexpr (NH == 8) {
                // S = K Q^T: A rows = tokens g, g + 8, B column = head g
                float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    uint32_t kb[4];
                    kfrag(ks, kb);
                    const uint32_t ka[4] = {kb[0], kb[2], kb[1], kb[3]};
                    M::run(s, ka, qa[ks][0], qa[ks][1]);
                }
                // lane (g, t4): s[0], s[1] = token g, heads 2 t4, 2 t4 + 1;
                // s[2], s[3] = token g + 8; logits in base 2, masked past the
                // sequence end
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tok = g + 8 * (i >> 1);
                    s[i] = (tok >= wlo && tok < wvalid) ? s[i] * a.scale_log2 : -INFINITY;
                }
                float mnew[2], p[4], pr[4];
#pragma unroll
                for (int j = 0; j < 2; ++j) {  // head 2 t4 + j: its tokens sit on the 8 lanes of t4
                    float mx = fmaxf(s[j], s[2 + j]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    mnew[j] = fmaxf(m[j], mx);
                    alpha_c[0][j] = ex2(m[j] - mnew[j]);
                    m[j] = mnew[j];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) p[i] = ex2(s[i] - mnew[i & 1]);
                const uint32_t h0p = M::pack(p[0], p[1], pr[0], pr[1]);
                const uint32_t h1p = M::pack(p[2], p[3], pr[2], pr[3]);
                // P (tokens x heads) -> P^T fragments: head g, tokens 2 t4,
                // 2 t4 + 1 of 0-7, then of 8-15
                pb[0][0] = movmatrix_trans(h0p);
                pb[0][1] = movmatrix_trans(h1p);
                if constexpr (SPLIT) {
                    float r[4];
                    const uint32_t l0p = M::pack(p[0] - pr[0], p[1] - pr[1], r[0], r[1]);
                    const uint32_t l1p = M::pack(p[2] - pr[2], p[3] - pr[3], r[2], r[3]);
                    pl[0][0] = movmatrix_trans(l0p);
                    pl[0][1] = movmatrix_trans(l1p);
                    // the weights P.V uses, hi + lo; with the fragments in
                    // registers the row sums take p itself, within 2^-18 p
#pragma unroll
                    for (int i = 0; i < 4; ++i) pr[i] = EARLY ? p[i] : pr[i] + r[i];
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) l[j] = l[j] * alpha_c[0][j] + (pr[j] + pr[2 + j]);
            } else {
                // S^T = Q K^T: two n-tiles of 8 tokens
                float s[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) s[nt][i] = 0.f;
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    uint32_t kb[4];
                    kfrag(ks, kb);
                    M::run(s[0], qa[ks], kb[0], kb[1]);
                    M::run(s[1], qa[ks], kb[2], kb[3]);
                }
                // logits in base 2, masked past the sequence end
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int tok = nt * 8 + 2 * t4 + (i & 1);
                        s[nt][i] = (tok >= wlo && tok < wvalid) ? s[nt][i] * a.scale_log2 : -INFINITY;
                    }
#pragma unroll
                for (int rb = 0; rb < RB; ++rb) {
                    const int i0 = 2 * rb;  // s[nt][i0], s[nt][i0 + 1]: head g + 8 rb
                    float mx = fmaxf(fmaxf(s[0][i0], s[0][i0 + 1]), fmaxf(s[1][i0], s[1][i0 + 1]));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    const float mnew = fmaxf(m[rb], mx);
                    const float alpha = exp2f(m[rb] - mnew);
                    float p[2][2], pr[2][2];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        p[nt][0] = exp2f(s[nt][i0] - mnew);
                        p[nt][1] = exp2f(s[nt][i0 + 1] - mnew);
                        pb[rb][nt] = M::pack(p[nt][0], p[nt][1], pr[nt][0], pr[nt][1]);
                        if constexpr (SPLIT) {
                            float r0, r1;
                            pl[rb][nt] = M::pack(p[nt][0] - pr[nt][0], p[nt][1] - pr[nt][1], r0, r1);
                            pr[nt][0] += r0;  // the weights P.V uses, hi + lo
                            pr[nt][1] += r1;
                        }
                    }
                    float ps = (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
                    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
                    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
                    l[rb] = l[rb] * alpha + ps;
                    m[rb] = mnew;
                    // O^T columns of this thread are heads 2 t4, 2 t4 + 1 (+ 8 rb)
                    alpha_c[rb][0] = __shfl_sync(0xffffffffu, alpha, (2 * t4) * 4);
                    alpha_c[rb][1] = __shfl_sync(0xffffffffu, alpha, (2 * t4 + 1) * 4);
                }
            }
            // O^T += V^T P^T
            const bool partial = wvalid < 16 || wlo > 0;
            if constexpr (EARLY) {
                // the fragments are in registers: zero the values of masked
                // tokens once (registers 0, 1: tokens 2 t4, 2 t4 + 1, low and
                // high half; 2, 3: the same + 8), so the loop has no branch
                if (partial) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int tk = 8 * j + 2 * t4;
                        const uint32_t keep =
                            (tk >= wlo && tk < wvalid ? 0x0000ffffu : 0u) |
                            (tk + 1 >= wlo && tk + 1 < wvalid ? 0xffff0000u : 0u);
#pragma unroll
                        for (int ks = 0; ks < (EARLY ? KSTEPS : 1); ++ks) {
                            vf[ks][2 * j] &= keep;
                            vf[ks][2 * j + 1] &= keep;
                        }
                    }
                }
            }
#pragma unroll
            for (int mt = 0; mt < KSTEPS; ++mt) {
                uint32_t va[4];
                if constexpr (EARLY) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) va[i] = vf[mt < (EARLY ? KSTEPS : 1) ? mt : 0][i];
                } else {
                    ldsm_x4_trans(kaddr(mt) + SLICE_BYTES, va);
                }
                if (!EARLY && partial) {
                    // zero values of masked tokens (0 * NaN would poison)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int tk = (i >> 1) * 8 + 2 * t4;
                        const uint32_t keep =
                            (tk >= wlo && tk < wvalid ? 0x0000ffffu : 0u) |
                            (tk + 1 >= wlo && tk + 1 < wvalid ? 0xffff0000u : 0u);
                        va[i] &= keep;
                    }
                }
#pragma unroll
                for (int rb = 0; rb < RB; ++rb) {
                    o[mt][rb][0] *= alpha_c[rb][0];
                    o[mt][rb][1] *= alpha_c[rb][1];
                    o[mt][rb][2] *= alpha_c[rb][0];
                    o[mt][rb][3] *= alpha_c[rb][1];
                    M::run(o[mt][rb], va, pb[rb][0], pb[rb][1]);
                    if constexpr (SPLIT) M::run(o[mt][rb], va, pl[rb][0], pl[rb][1]);
                }
            }
        };
        if (!EARLY && work) math();
        __syncwarp();  // the warp's reads of the stage are done: refill it
        if (lane == 0 && it + STAGES < nslices) issue(it + STAGES, stage);
        if (EARLY && work) math();
    }
    __syncthreads();  // every warp is out of its ring (or gave up)
    if (s_abort) return;
    if (!sp.direct) pdl_launch_dependents();

    // merge the warps (padded rows: lanes of one store hit distinct banks)
    using A = MergeArea<D, NH, NW>;
    static_assert(A::BYTES <= C::RING_BYTES, "merge area");
    float* red = reinterpret_cast<float*>(s_kv);
    float* red_m = red + NW * NH * A::RP;
    float* red_l = red_m + NW * NH;
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
        for (int rb = 0; rb < RB; ++rb)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int head = 8 * rb + 2 * t4 + (i & 1);
                const int dim = mt * 16 + g + 8 * (i >> 1);
                red[(warp * NH + head) * A::RP + dim] = o[mt][rb][i];
            }
    if constexpr (NH == 8) {  // heads 2 t4 + j, l summed over the lanes of one t4
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            l[j] += __shfl_xor_sync(0xffffffffu, l[j], 4);
            l[j] += __shfl_xor_sync(0xffffffffu, l[j], 8);
            l[j] += __shfl_xor_sync(0xffffffffu, l[j], 16);
        }
        if (g == 0) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                red_m[warp * NH + 2 * t4 + j] = m[j];
                red_l[warp * NH + 2 * t4 + j] = l[j];
            }
        }
    } else if (t4 == 0) {
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) {
            red_m[warp * NH + g + 8 * rb] = m[rb];
            red_l[warp * NH + g + 8 * rb] = l[rb];
        }
    }
    __syncthreads();
    if constexpr (GROUPS)
        merge_warps_and_store<T, D, NH, NW>(
            a, red, [&](int hh) { return s_row[hh]; },
            [&](int hh) { return s_row[hh] * a.ws_slots + part; }, nh, false, tid, NW * 32);
    else
        merge_warps_and_store<T, D, NH, NW>(
            a, red, [&](int hh) { return (int64_t)b * a.num_q_heads + h0 + hh; },
            [&](int hh) {
                return ((int64_t)b * a.num_q_heads + h0 + hh) * a.ws_slots + sp.slot0 + part;
            },
            nh, sp.direct, tid, NW * 32);
}

// Host side: tensor maps over the K and V pools, launch, optional reduce.
cudaError_t make_cache_tensor_map(CUtensorMap* map, const void* base, int dtype_bytes,
                                  bool bf16, int head_dim, int64_t rows, int box_rows);

template <typename T, int D, int BS, int NH, int NW = 4, int STAGES = 0>
cudaError_t launch_decode_mma(const DecodeArgs& a, cudaStream_t stream) {
    using C = MmaCfg<D, BS, NW, STAGES>;
    static SmemAttr attr;
    auto kern = decode_mma_kernel<T, D, BS, NH, NW, STAGES>;
    cudaError_t e = attr.ensure(kern, C::smem_bytes(8192));
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)a.num_blocks * a.num_kv_heads * BS;
    CUtensorMap tk, tv;
    const bool bf = std::is_same<T, __nv_bfloat16>::value;
    e = make_cache_tensor_map(&tk, a.k_cache, 2, bf, D, rows, 16);
    if (e != cudaSuccess) return e;
    e = make_cache_tensor_map(&tv, a.v_cache, 2, bf, D, rows, 16);
    if (e != cudaSuccess) return e;
    const dim3 grid = decode_grid(a);
    e = launch_decode_kernel(kern, grid, dim3(NW * 32), C::smem_bytes(a.partition_size), stream,
                             a, tk, tv);
    if (e != cudaSuccess || a.ws_slots <= 1) return e;
    return launch_lse_reduce<T, D>(a, stream);
}

// The group pass of the shared-prefix decode: grid (prefix partitions,
// Hkv x row chunks, groups); writes workspace slots only (the reduce runs
// after the regular pass).
template <typename T, int D, int BS, int NH, int NW = 4, int STAGES = 0>
cudaError_t launch_decode_mma_groups(const DecodeArgs& a, int num_groups, cudaStream_t stream) {
    using C = MmaCfg<D, BS, NW, STAGES>;
    static SmemAttr attr;
    auto kern = decode_mma_kernel<T, D, BS, NH, NW, STAGES, true>;
    cudaError_t e = attr.ensure(kern, C::smem_bytes(8192));
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)a.num_blocks * a.num_kv_heads * BS;
    CUtensorMap tk, tv;
    const bool bf = std::is_same<T, __nv_bfloat16>::value;
    e = make_cache_tensor_map(&tk, a.k_cache, 2, bf, D, rows, 16);
    if (e != cudaSuccess) return e;
    e = make_cache_tensor_map(&tv, a.v_cache, 2, bf, D, rows, 16);
    if (e != cudaSuccess) return e;
    dim3 grid(a.max_partitions, a.num_kv_heads * a.head_chunks, num_groups);
    kern<<<grid, NW * 32, C::smem_bytes(a.partition_size), stream>>>(a, tk, tv);
    return cudaGetLastError();
}

cudaError_t decode_mma_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                           cudaStream_t stream);
cudaError_t decode_mma_groups_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                  int num_groups, cudaStream_t stream);
cudaError_t decode_mma_groups_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                   int num_groups, cudaStream_t stream);
cudaError_t decode_mma_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                            cudaStream_t stream);

}  // namespace pkv
