// Paged decode attention on the CUDA cores.
//
// One CTA takes one (partition of a sequence's context, KV head, slice of HG
// query heads of that KV head's group).  The steps follow "pagedattention vllm"
// §Attention Computation: translate each logical block to its physical block
// through the table, load the physical block, compute attention over the
// gathered tokens as if they were contiguous.
//
//   1. The table entries of the partition are read once, coalesced, into
//      shared memory (4-byte entries, "pagedattention vllm" §Implementation
//      Details).
//   2. Every warp streams its own 16-token slices (tokens [16w, 16w + 16) of
//      each round of TILE = 16 * NW tokens) through a private ring of STAGES
//      shared-memory stages: its lane 0 issues 1-D bulk copies (TMA,
//      cp.async.bulk) of the slice's 16 contiguous rows of a (block, KV head)
//      page for K and for V, completing on the stage's mbarrier.  The warp
//      copies the slice into registers, refills that stage at once and then
//      does the math; no barrier ties the warps together until the merge.
//   3. Warp w takes tokens [16w, 16w + 16) of each round.  QK: 8 lanes per
//      token, each with D/8 dims of q (float32, pre-scaled by scale*log2 e) in
//      registers; 3 xor-shuffles finish each dot product.  Tokens past the
//      sequence end get a logit of -inf and their values are never read, so
//      whatever sits in the unused slots of the last block cannot leak in.
//   4. Per-warp online softmax in base 2: running max m, sum l, accumulator
//      rescaled by 2^(m_old - m_new).
//   5. PV: LPV lanes per token read one 16-byte chunk of v each; the weights
//      go through a 16-entry per-warp shared array.
//   6. The NW per-warp (m, l, acc) are merged in shared memory; a one-partition
//      sequence writes out directly, a longer one writes (m, l, acc / l) to the
//      workspace for the log-sum-exp reduce.
#pragma once

#include <type_traits>

#include "decode_common.cuh"
#include "lse_reduce.cuh"

namespace pkv {

// Stage count: the most stages (2..4) whose ring still lets three CTAs share
// an SM (<= 72 KB).  Measured on B200 for the 40-head fp16 layer: three
// CTAs of 2 x 32 KB stages stream at 6.4 TB/s where two CTAs of 3 stages
// reach 5.2 TB/s -- more independent CTAs per SM hide the DRAM latency and
// the per-CTA start-up better than deeper rings.
template <int ROW_BYTES, int NW>
struct SimtStages {
    static constexpr int kTile = 16 * NW;
    static constexpr int kStageBytes = 2 * kTile * ROW_BYTES;  // K + V
    static constexpr int kBudget = 73728;
    static constexpr int kStages =
        kBudget / kStageBytes >= 4 ? 4 : (kBudget / kStageBytes >= 3 ? 3 : 2);
};

// STAGES_ = 0 picks the stage count by SimtStages (stages per warp ring; the
// CTA's rings together hold what one CTA-wide ring of that depth would).
// TC is the page element type: T itself, or E4M3 codes with T = fp16/bf16
// for q and out.
template <typename T, int D, int BS, int HG, int NW, int STAGES_ = 0, typename TC = T>
struct SimtCfg {
    static constexpr int ROW = D * Elem<TC>::kBytes;
    static constexpr int CPR = ROW / 16;
    static constexpr int EPC = Elem<TC>::kPerVec;
    static constexpr int TILE = 16 * NW;
    static constexpr int SLICE_BYTES = 16 * ROW;    // one warp's 16 tokens of K (or V)
    static constexpr int STAGE_BYTES = TILE * ROW;  // all warps' slices of one stage
    static constexpr int STAGES = STAGES_ ? STAGES_ : SimtStages<ROW, NW>::kStages;
    static constexpr int WARP_RING = STAGES * 2 * SLICE_BYTES;
    static constexpr int CPL = CPR / 8;
    static constexpr int LPV = CPR < 32 ? CPR : 32;
    static constexpr int TPV = 32 / LPV;
    static constexpr int CPV = CPR / LPV;
    static constexpr int THREADS = NW * 32;
    static_assert(BS % 16 == 0, "16-token slices of whole rows");
    static_assert(CPR % 8 == 0, "rows of at least 128 bytes");

    static int smem_bytes(int partition_size) {
        return 256 + round_up(partition_size / BS * 4, 128) + STAGES * 2 * STAGE_BYTES;
    }
};

// One consumer warp's share of a partition: its q slice, online-softmax state
// and accumulator, and the per-stage work on its 16 tokens.
template <typename T, int D, int HG, typename C, typename TC = T>
struct SimtWarp {
    using E = Elem<TC>;   // pages
    using EQ = Elem<T>;   // q and out
    static constexpr int ROW = C::ROW, EPC = C::EPC, CPL = C::CPL, LPV = C::LPV;
    static constexpr int TPV = C::TPV, CPV = C::CPV;
    static constexpr int NTV = 16 / TPV;  // tokens per lane in P.V
    // Copy the warp's share of a stage into registers and release the stage
    // before the math (EARLY), when that fits the register budget of three
    // CTAs per SM; otherwise read from the stage and release it afterwards.
    static constexpr bool EARLY = ROW <= 256 && (HG == 1 || ROW <= 128);
    static constexpr int KR = EARLY ? CPL : 1, NV = EARLY ? NTV : 1, VC = EARLY ? CPV : 1;

    float qf[HG][CPL][EPC];
    float m[HG], l[HG], acc[HG][CPV][EPC];
    uint4 kr[4][KR];      // this lane's K chunks of the warp's 16 tokens (EARLY)
    uint4 vr[NV][VC];     // and its V chunks
    const unsigned char* Kp;  // the stage rows otherwise
    const unsigned char* Vp;
    int lane, grp, sub, lv, tv;

    __device__ __forceinline__ uint4 kchunk(int r, int i) const {
        if constexpr (EARLY) return kr[r][i];
        else return *reinterpret_cast<const uint4*>(Kp + (r * 4 + grp) * ROW + (sub + 8 * i) * 16);
    }
    __device__ __forceinline__ uint4 vchunk(int j, int c) const {
        if constexpr (EARLY) return vr[j][c];
        else return *reinterpret_cast<const uint4*>(Vp + (tv + j * TPV) * ROW + (lv + c * LPV) * 16);
    }

    // qscale: scale * log2(e), times the K pages' scale for quantised pages
    __device__ __forceinline__ void init(const T* qb, int nh, float qscale, int lane_) {
        lane = lane_;
        grp = lane >> 3;
        sub = lane & 7;
        lv = lane % LPV;
        tv = lane / LPV;
        constexpr int QV = EPC / EQ::kPerVec;  // 16-byte q vectors per page chunk
#pragma unroll
        for (int hh = 0; hh < HG; ++hh) {
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                if (hh < nh) {
#pragma unroll
                    for (int u = 0; u < QV; ++u) {
                        const uint4 v = *reinterpret_cast<const uint4*>(
                            qb + hh * D + (sub + 8 * i) * EPC + u * EQ::kPerVec);
                        EQ::to_f32(v, qf[hh][i] + u * EQ::kPerVec);
                    }
#pragma unroll
                    for (int e = 0; e < EPC; ++e) qf[hh][i][e] *= qscale;
                } else {
#pragma unroll
                    for (int e = 0; e < EPC; ++e) qf[hh][i][e] = 0.f;
                }
            }
            m[hh] = -INFINITY;
            l[hh] = 0.f;
#pragma unroll
            for (int c = 0; c < CPV; ++c)
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[hh][c][e] = 0.f;
        }
    }

    // Copy this lane's share of the warp's 16 tokens (rows of ROW bytes at Kw /
    // Vw) into registers, so the stage can be refilled before the math runs.
    __device__ __forceinline__ void fetch(const unsigned char* Kw, const unsigned char* Vw) {
        Kp = Kw;
        Vp = Vw;
        if constexpr (EARLY) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int i = 0; i < CPL; ++i)
                    kr[r][i] = *reinterpret_cast<const uint4*>(Kw + (r * 4 + grp) * ROW + (sub + 8 * i) * 16);
#pragma unroll
            for (int j = 0; j < NTV; ++j)
#pragma unroll
                for (int c = 0; c < CPV; ++c)
                    vr[j][c] = *reinterpret_cast<const uint4*>(Vw + (tv + j * TPV) * ROW + (lv + c * LPV) * 16);
        }
    }

    // The fetched 16 tokens; tokens [wlo, wvalid) of them are attended to
    // (before wlo: ahead of a sliding window; from wvalid: past the end).
    // s_p: this warp's [HG][16] weight scratch.  E4M3 pages with a scale per
    // page: kts multiplies the logits and vts the weights of the V sum (the
    // row sum l keeps the plain weights).
    __device__ __forceinline__ void compute(int wlo, int wvalid, float (*s_p)[16],
                                            float kts = 1.f, float vts = 1.f) {
        constexpr bool Q8 = std::is_same<TC, E4M3>::value;
        float s[HG][4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int tok = r * 4 + grp;
            float d[HG];
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) d[hh] = 0.f;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                float kf[EPC];
                E::to_f32(kchunk(r, i), kf);
#pragma unroll
                for (int hh = 0; hh < HG; ++hh)
#pragma unroll
                    for (int e = 0; e < EPC; ++e) d[hh] = fmaf(qf[hh][i][e], kf[e], d[hh]);
            }
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) {
                d[hh] += __shfl_xor_sync(0xffffffffu, d[hh], 1);
                d[hh] += __shfl_xor_sync(0xffffffffu, d[hh], 2);
                d[hh] += __shfl_xor_sync(0xffffffffu, d[hh], 4);
                s[hh][r] = (tok >= wlo && tok < wvalid) ? (Q8 ? d[hh] * kts : d[hh]) : -INFINITY;
            }
        }
#pragma unroll
        for (int hh = 0; hh < HG; ++hh) {
            float mx = fmaxf(fmaxf(s[hh][0], s[hh][1]), fmaxf(s[hh][2], s[hh][3]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mnew = fmaxf(m[hh], mx);  // finite: one token is attended to
            const float alpha = exp2f(m[hh] - mnew);
            float ps = 0.f;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                s[hh][r] = exp2f(s[hh][r] - mnew);
                ps += s[hh][r];
            }
            ps += __shfl_xor_sync(0xffffffffu, ps, 8);
            ps += __shfl_xor_sync(0xffffffffu, ps, 16);
            l[hh] = l[hh] * alpha + ps;
            m[hh] = mnew;
#pragma unroll
            for (int c = 0; c < CPV; ++c)
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[hh][c][e] *= alpha;
            if (sub == 0) {
#pragma unroll
                for (int r = 0; r < 4; ++r) s_p[hh][r * 4 + grp] = Q8 ? s[hh][r] * vts : s[hh][r];
            }
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < NTV; ++j) {
            const int t = tv + j * TPV;
            if (t >= wlo && t < wvalid) {  // masked values are never used (they may be NaN)
#pragma unroll
                for (int c = 0; c < CPV; ++c) {
                    float vf[EPC];
                    E::to_f32(vchunk(j, c), vf);
#pragma unroll
                    for (int hh = 0; hh < HG; ++hh) {
                        const float p = s_p[hh][t];
#pragma unroll
                        for (int e = 0; e < EPC; ++e) acc[hh][c][e] = fmaf(p, vf[e], acc[hh][c][e]);
                    }
                }
            }
        }
        __syncwarp();
    }

    // Fold the token lanes together and park (m, l, acc) in the merge area.
    // vscale: the V pages' scale for quantised pages (else 1)
    template <int NW>
    __device__ __forceinline__ void park(int warp, float* red, float vscale) {
        using A = MergeArea<D, HG, NW>;
        float* red_m = red + NW * HG * A::RP;
        float* red_l = red_m + NW * HG;
        if (vscale != 1.f) {
#pragma unroll
            for (int hh = 0; hh < HG; ++hh)
#pragma unroll
                for (int c = 0; c < CPV; ++c)
#pragma unroll
                    for (int e = 0; e < EPC; ++e) acc[hh][c][e] *= vscale;
        }
#pragma unroll
        for (int msk = LPV; msk < 32; msk <<= 1)
#pragma unroll
            for (int hh = 0; hh < HG; ++hh)
#pragma unroll
                for (int c = 0; c < CPV; ++c)
#pragma unroll
                    for (int e = 0; e < EPC; ++e)
                        acc[hh][c][e] += __shfl_xor_sync(0xffffffffu, acc[hh][c][e], msk);
        if (tv == 0) {
#pragma unroll
            for (int hh = 0; hh < HG; ++hh)
#pragma unroll
                for (int c = 0; c < CPV; ++c)
#pragma unroll
                    for (int e = 0; e < EPC; e += 4)
                        *reinterpret_cast<float4*>(red + (warp * HG + hh) * A::RP +
                                                   (lv + c * LPV) * EPC + e) =
                            make_float4(acc[hh][c][e], acc[hh][c][e + 1], acc[hh][c][e + 2],
                                        acc[hh][c][e + 3]);
        }
        if (lane == 0) {
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) {
                red_m[warp * HG + hh] = m[hh];
                red_l[warp * HG + hh] = l[hh];
            }
        }
    }
};

template <typename T, int D, int BS, int HG, int NW, int STAGES_, typename TC>
__global__ void __launch_bounds__(SimtCfg<T, D, BS, HG, NW, STAGES_, TC>::THREADS,
                                  SimtCfg<T, D, BS, HG, NW, STAGES_, TC>::ROW <= 256 ? 3 : 1)
    decode_simt_kernel(const DecodeArgs a) {
    using C = SimtCfg<T, D, BS, HG, NW, STAGES_, TC>;
    using E = Elem<T>;
    constexpr int ROW = C::ROW, TILE = C::TILE, SLICE_BYTES = C::SLICE_BYTES;
    constexpr int STAGE_BYTES = C::STAGE_BYTES, WARP_RING = C::WARP_RING;
    constexpr int STAGES = C::STAGES, THREADS = C::THREADS;

    extern __shared__ __align__(128) unsigned char smem_simt[];
    __shared__ float s_p[NW][HG][16];
    __shared__ volatile int s_abort;
    const GroupPassWait group_pass_wait{a};
    // Launched as a programmatic dependent of the kernel before it (usually
    // the KV append): the schedule, lengths and table (which that kernel does
    // not write) are read before griddepcontrol.wait, so the start-up of the
    // first wave overlaps it; the pages are read, and anything is written,
    // only after it (pdl_wait_before_pages).

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kvh = blockIdx.y / a.head_chunks;
    const int hc = blockIdx.y - kvh * a.head_chunks;
    const CtaUnit unit = cta_unit(a, tid);  // (sequence, partition)
    const int part = unit.part;
    const int h0 = kvh * a.group + hc * HG;
    const int nh = min(HG, a.group - hc * HG);
    const bool reporter = (tid == 0 && part == 0 && blockIdx.y == 0);
    const int b = unit.b;
    if (b < 0) return;

    const TablePrefetch pf = table_prefetch(a, b, part, a.partition_size / BS, tid);
    const Span sp = seq_span(a, b, reporter);
    const int L = sp.L, np = sp.np;
    if (L == 0) {  // empty sequence: a zero row
        if (part == 0) {
            pdl_wait_before_pages(a);
            T* out = reinterpret_cast<T*>(a.out);
            for (int i = tid; i < nh * D; i += THREADS)
                out[((int64_t)b * a.num_q_heads + h0 + i / D) * D + i % D] = E::from_f32(0.f);
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

    uint64_t* full = reinterpret_cast<uint64_t*>(smem_simt);  // [NW][STAGES]
    int32_t* s_tab = reinterpret_cast<int32_t*>(smem_simt + 256);
    unsigned char* s_kv = smem_simt + 256 + round_up(P / BS * 4, 128);
    static_assert(NW * STAGES * 8 <= 256, "barriers");

    // 1. table slice -> shared memory
    table_hoist(a, b, t0 / BS, nblk, pf, s_tab, tid, THREADS);
    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < NW * STAGES; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncthreads();

    // 2. this warp's ring: lane 0 issues the copies of slice k into a stage
    const unsigned char* kbase = reinterpret_cast<const unsigned char*>(a.k_cache);
    const unsigned char* vbase = reinterpret_cast<const unsigned char*>(a.v_cache);
    const uint64_t pol = policy_evict_first();
    auto issue = [&](int k, int stage) {
        const int tok = k * TILE + warp * 16;
        const int64_t off =
            (((int64_t)s_tab[tok / BS] * a.num_kv_heads + kvh) * BS + tok % BS) * ROW;
        uint64_t* bar = full + warp * STAGES + stage;
        unsigned char* kd = s_kv + warp * WARP_RING + stage * 2 * SLICE_BYTES;
        mbar_arrive_expect_tx(bar, (uint32_t)(2 * SLICE_BYTES));
        bulk_load(kd, kbase + off, SLICE_BYTES, bar, pol);
        bulk_load(kd + SLICE_BYTES, vbase + off, SLICE_BYTES, bar, pol);
    };
    pdl_wait_before_pages(a);
    if (lane == 0) {
        const int pre = min(STAGES, nslices);
        for (int s = 0; s < pre; ++s) issue(s, s);
    }

    float* red = reinterpret_cast<float*>(s_kv);  // merge area, once the rings are drained
    static_assert(MergeArea<D, HG, NW>::BYTES <= STAGES * 2 * STAGE_BYTES, "merge area");

    // 3.-5. the warps
    SimtWarp<T, D, HG, C, TC> W;
    W.init(reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.num_q_heads + h0) * D, nh,
           a.k_scale && !a.scale_per_block ? a.scale_log2 * a.k_scale[kvh] : a.scale_log2,
           lane);
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
        const int wvalid = ntok - (it * TILE + warp * 16);  // tokens this warp owns
        const int wlo = mask_lo - (it * TILE + warp * 16);
        const bool work = wlo < 16 && wlo < wvalid;
        if (work) {
            const unsigned char* Kw = s_kv + warp * WARP_RING + stage * 2 * SLICE_BYTES;
            W.fetch(Kw, Kw + SLICE_BYTES);
        }
        float kts = 1.f, vts = 1.f;  // page scales of this warp's tokens (per-page mode)
        if (a.scale_per_block && work) {
            const int64_t si =
                (int64_t)s_tab[(it * TILE + warp * 16) / BS] * a.num_kv_heads + kvh;
            kts = a.k_scale[si];
            vts = a.v_scale[si];
        }
        if (!W.EARLY && work) W.compute(wlo, wvalid, s_p[warp], kts, vts);
        // the slice is in registers (or used): refill its stage
        __syncwarp();
        if (lane == 0 && it + STAGES < nslices) issue(it + STAGES, stage);
        if (W.EARLY && work) W.compute(wlo, wvalid, s_p[warp], kts, vts);
    }
    __syncthreads();  // every warp is out of its ring (or gave up)
    if (s_abort) return;
    if (!sp.direct) pdl_launch_dependents();

    // 6. merge the warps
    W.template park<NW>(warp, red, a.v_scale && !a.scale_per_block ? a.v_scale[kvh] : 1.f);
    __syncthreads();
    merge_warps_and_store<T, D, HG, NW>(
        a, red, [&](int hh) { return (int64_t)b * a.num_q_heads + h0 + hh; },
        [&](int hh) { return ((int64_t)b * a.num_q_heads + h0 + hh) * a.ws_slots + sp.slot0 + part; },
        nh, sp.direct, tid, NW * 32);
}

template <typename T, int D, int BS, int HG, int NW = 4, int STAGES = 0, typename TC = T>
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t stream) {
    using C = SimtCfg<T, D, BS, HG, NW, STAGES, TC>;
    static SmemAttr attr;
    const int smem_simt = C::smem_bytes(a.partition_size);
    auto kern = decode_simt_kernel<T, D, BS, HG, NW, STAGES, TC>;
    cudaError_t e = attr.ensure(kern, C::smem_bytes(8192));
    if (e != cudaSuccess) return e;
    const dim3 grid = decode_grid(a);
    e = launch_decode_kernel(kern, grid, dim3(C::THREADS), smem_simt, stream, a);
    if (e != cudaSuccess || a.ws_slots <= 1) return e;
    return launch_lse_reduce<T, D>(a, stream);
}

}  // namespace pkv
