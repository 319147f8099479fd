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
//   2. One thread issues 1-D bulk copies (TMA, cp.async.bulk) of whole
//      (block, KV head) pages -- BS x D contiguous elements each for K and for
//      V -- into a ring of STAGES shared-memory stages of TILE = 16 * NW tokens,
//      completing on an mbarrier per stage.  Each warp first copies its part
//      of a stage into registers; the stage is refilled (copy of stage
//      i + STAGES) as soon as every warp has done so, before the math runs.
//   3. Warp w takes tokens [16w, 16w + 16) of each stage.  QK: 8 lanes per
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

// STAGES_ = 0 picks the stage count by SimtStages; WS = true adds a
// producer warp that re-arms each stage as soon as the consumer warps have
// released it (per-stage "empty" mbarriers) instead of a CTA-wide barrier.
// TC is the page element type: T itself, or E4M3 codes with T = fp16/bf16
// for q and out.
template <typename T, int D, int BS, int HG, int NW, int STAGES_ = 0, bool WS = false,
          typename TC = T>
struct SimtCfg {
    static constexpr int ROW = D * Elem<TC>::kBytes;
    static constexpr int CPR = ROW / 16;
    static constexpr int EPC = Elem<TC>::kPerVec;
    static constexpr int TILE = 16 * NW;
    static constexpr int BPT = TILE / BS;
    static constexpr int BLK_BYTES = BS * ROW;
    static constexpr int STAGE_BYTES = TILE * ROW;  // one of K / V
    static constexpr int STAGES = STAGES_ ? STAGES_ : SimtStages<ROW, NW>::kStages;
    static constexpr int CPL = CPR / 8;
    static constexpr int LPV = CPR < 32 ? CPR : 32;
    static constexpr int TPV = 32 / LPV;
    static constexpr int CPV = CPR / LPV;
    static constexpr int THREADS = (NW + (WS ? 1 : 0)) * 32;
    static_assert(TILE % BS == 0, "a stage holds whole blocks");
    static_assert(CPR % 8 == 0, "rows of at least 128 bytes");

    static int smem_bytes(int partition_size) {
        return 128 + round_up(partition_size / BS * 4, 128) + STAGES * 2 * STAGE_BYTES;
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

template <typename T, int D, int BS, int HG, int NW, int STAGES_, bool WS, typename TC>
__global__ void __launch_bounds__(SimtCfg<T, D, BS, HG, NW, STAGES_, WS, TC>::THREADS,
                                  SimtCfg<T, D, BS, HG, NW, STAGES_, WS, TC>::ROW <= 256 ? 3 : 1)
    decode_simt_kernel(const DecodeArgs a) {
    using C = SimtCfg<T, D, BS, HG, NW, STAGES_, WS, TC>;
    using E = Elem<T>;
    constexpr int ROW = C::ROW, TILE = C::TILE, BPT = C::BPT;
    constexpr int BLK_BYTES = C::BLK_BYTES, STAGE_BYTES = C::STAGE_BYTES;
    constexpr int STAGES = C::STAGES, THREADS = C::THREADS;

    extern __shared__ __align__(128) unsigned char smem_simt[];
    __shared__ float s_p[NW][HG][16];
    __shared__ volatile int s_abort;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kvh = blockIdx.y / a.head_chunks;
    const int hc = blockIdx.y - kvh * a.head_chunks;
    const int part = blockIdx.x;
    const int h0 = kvh * a.group + hc * HG;
    const int nh = min(HG, a.group - hc * HG);
    const bool reporter = (tid == 0 && part == 0 && blockIdx.y == 0);
    const int b = scheduled_seq(a, blockIdx.z, reporter);
    if (b < 0) return;

    const TablePrefetch pf = table_prefetch(a, b, part, a.partition_size / BS, tid);
    const Span sp = seq_span(a, b, reporter);
    const int L = sp.L, np = sp.np;
    if (L == 0) {  // empty sequence: a zero row
        if (part == 0) {
            T* out = reinterpret_cast<T*>(a.out);
            for (int i = tid; i < nh * D; i += THREADS)
                out[((int64_t)b * a.num_q_heads + h0 + i / D) * D + i % D] = E::from_f32(0.f);
        }
        return;
    }
    if (part >= np) return;

    const int P = a.partition_size;
    const int t0 = sp.base + part * P;
    const int ntok = min(L, t0 + P) - t0;
    const int mask_lo = part == 0 ? sp.lo - sp.base : 0;  // tokens ahead of the window
    const int ntiles = (ntok + TILE - 1) / TILE;
    const int nblk = (ntok + BS - 1) / BS;

    uint64_t* full = reinterpret_cast<uint64_t*>(smem_simt);
    uint64_t* empty = full + STAGES;  // WS only
    int32_t* s_tab = reinterpret_cast<int32_t*>(smem_simt + 128);
    unsigned char* s_kv = smem_simt + 128 + round_up(P / BS * 4, 128);

    // 1. table slice -> shared memory
    table_hoist(a, b, t0 / BS, nblk, pf, s_tab, tid, THREADS);
    if (tid == 0) {
        s_abort = 0;
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            if (WS) mbar_init(&empty[s], NW);
        }
        fence_barrier_init();
    }
    __syncthreads();

    const unsigned char* kbase = reinterpret_cast<const unsigned char*>(a.k_cache);
    const unsigned char* vbase = reinterpret_cast<const unsigned char*>(a.v_cache);
    auto issue = [&](int tile, int stage, uint64_t pol) {
        const int jb = tile * BPT;
        const int je = min(nblk, jb + BPT);
        mbar_arrive_expect_tx(&full[stage], (uint32_t)((je - jb) * BLK_BYTES * 2));
        unsigned char* kd = s_kv + stage * 2 * STAGE_BYTES;
        unsigned char* vd = kd + STAGE_BYTES;
        for (int j = jb; j < je; ++j) {
            const int64_t off = ((int64_t)s_tab[j] * a.num_kv_heads + kvh) * BLK_BYTES;
            bulk_load(kd + (j - jb) * BLK_BYTES, kbase + off, BLK_BYTES, &full[stage], pol);
            bulk_load(vd + (j - jb) * BLK_BYTES, vbase + off, BLK_BYTES, &full[stage], pol);
        }
    };

    float* red = reinterpret_cast<float*>(s_kv);  // merge area, after the last stage
    static_assert(MergeArea<D, HG, NW>::BYTES <= STAGES * 2 * STAGE_BYTES, "merge area");

    if (WS && warp == NW) {
        // 2. producer warp: keep every stage loaded as soon as it is released
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            for (int it = 0; it < ntiles; ++it) {
                const int stage = it % STAGES;
                if (it >= STAGES &&
                    !mbar_wait(&empty[stage], (uint32_t)(((it / STAGES) - 1) & 1), a.status)) {
                    s_abort = 1;
                    break;
                }
                if (s_abort) break;
                issue(it, stage, pol);
            }
        }
        __syncthreads();  // matches the consumers' barrier before the merge
        if (s_abort) return;
        pdl_launch_dependents();
        __syncthreads();
        merge_warps_and_store<T, D, HG, NW>(a, red, b, h0, nh, part, np, tid, THREADS);
        return;
    }

    if (!WS && tid == 0) {
        const uint64_t pol = policy_evict_first();
        const int pre = min(STAGES, ntiles);
        for (int s = 0; s < pre; ++s) issue(s, s, pol);
    }

    // 3.-5. consumer warps
    SimtWarp<T, D, HG, C, TC> W;
    W.init(reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.num_q_heads + h0) * D, nh,
           a.k_scale && !a.scale_per_block ? a.scale_log2 * a.k_scale[kvh] : a.scale_log2,
           lane);
    const uint64_t pol = WS ? 0 : policy_evict_first();
    int it_stop = ntiles;  // the tile a timed-out wait stopped at
    for (int it = 0; it < ntiles; ++it) {
        const int stage = it % STAGES;
        if (!mbar_wait(&full[stage], (uint32_t)((it / STAGES) & 1), a.status)) s_abort = 1;
        if (WS && s_abort) break;
        const int wvalid = ntok - (it * TILE + warp * 16);  // tokens this warp owns
        const int wlo = mask_lo - (it * TILE + warp * 16);
        const bool work = wvalid > 0 && wlo < 16 && wlo < wvalid;
        if (!s_abort && work) {
            const unsigned char* Kw = s_kv + stage * 2 * STAGE_BYTES + warp * 16 * ROW;
            W.fetch(Kw, Kw + STAGE_BYTES);
        }
        float kts = 1.f, vts = 1.f;  // page scales of this warp's tokens (per-page mode)
        if (a.scale_per_block && work) {
            const int64_t si =
                (int64_t)s_tab[(it * TILE + warp * 16) / BS] * a.num_kv_heads + kvh;
            kts = a.k_scale[si];
            vts = a.v_scale[si];
        }
        if (!W.EARLY && !s_abort && work) W.compute(wlo, wvalid, s_p[warp], kts, vts);
        // the stage's data is in registers (or used): hand the stage back
        if (WS) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
        } else {
            __syncthreads();
            if (s_abort) {
                it_stop = it;
                break;
            }
            if (tid == 0 && it + STAGES < ntiles) issue(it + STAGES, stage, pol);
        }
        if (W.EARLY && work) W.compute(wlo, wvalid, s_p[warp], kts, vts);
    }
    if (WS) __syncthreads();  // producer and consumers: every stage consumed
    if (s_abort) {
        // let the copies still in flight land (bounded) before the CTA leaves
        if (!WS && tid == 0)
            for (int k = it_stop; k < min(ntiles, it_stop + STAGES); ++k)
                mbar_wait(&full[k % STAGES], (uint32_t)((k / STAGES) & 1), a.status);
        return;
    }
    if (!WS) pdl_launch_dependents();

    // 6. merge the warps
    W.template park<NW>(warp, red, a.v_scale && !a.scale_per_block ? a.v_scale[kvh] : 1.f);
    __syncthreads();
    merge_warps_and_store<T, D, HG, NW>(a, red, b, h0, nh, part, np, tid, WS ? THREADS : NW * 32);
}

template <typename T, int D, int BS, int HG, int NW = 4, int STAGES = 0, bool WS = false,
          typename TC = T>
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t stream) {
    using C = SimtCfg<T, D, BS, HG, NW, STAGES, WS, TC>;
    static SmemAttr attr;
    const int smem_simt = C::smem_bytes(a.partition_size);
    auto kern = decode_simt_kernel<T, D, BS, HG, NW, STAGES, WS, TC>;
    cudaError_t e = attr.ensure(kern, C::smem_bytes(8192));
    if (e != cudaSuccess) return e;
    dim3 grid(a.max_partitions, a.num_kv_heads * a.head_chunks, a.num_seqs);
    kern<<<grid, C::THREADS, smem_simt, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.max_partitions <= 1) return e;
    return launch_lse_reduce<T, D>(a, stream);
}

}  // namespace pkv
