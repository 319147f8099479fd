// The planned decode over E4M3 pages: persistent CTAs whose warps stream the
// pieces of a host plan without ever waiting for each other.
//
// A per-CTA timeline of the regular grid (one CTA per sequence, KV head and
// partition) showed a quarter of the CTA slot time spent in each CTA's set-up
// (length, table slice, first pages, one after the other) and merge, the
// kernel as long as its longest partition, and shorter partitions losing to
// the CTAs that find their sequence too short.  Here a host plan
// (pkv_decode_plan) cuts every (sequence, KV head, tile of query heads) unit
// into pieces and spreads them over the CTAs, and every warp of a CTA walks
// the CTA's pieces on its own:
//   * warp w takes slices w, w + NW, ... (16 tokens each) of every piece, so
//     its ring streams from one piece into the next with no gap: its lane 0
//     issues the next piece's first pages while the warp still works on the
//     current piece;
//   * the next piece's descriptor and this warp's table entries for it are
//     fetched with cp.async one piece ahead (two for the descriptor);
//   * at the end of a piece the warp writes its partial softmax state (m, l
//     and the unnormalised sum of p v) to a workspace slot -- a few KB that
//     stay in L2 -- and counts itself in at the unit's counter; the warp that
//     completes the count merges all of the unit's partial states and writes
//     the output rows, then sets the counter back to zero.
// No CTA barrier and no shared merge area: the warps never wait for each
// other, and a unit cut into several pieces (on several CTAs) is merged the
// same way, so no reduce kernel runs after the grid.
//
// Plan item (PKV_PLAN_ITEM_WORDS int32 words): b, y (KV head * head_chunks +
// tile), t0, t1, mask_lo, unit, first slot of the unit, the unit's pieces,
// this piece's index in the unit.  Warp w's partial state of piece p of a
// unit is slot unit_slot0 + p * NW + w: ws_ml [slot][NH][2] (m, l) and ws_o
// [slot][NH][D]; a.plan_counts [units] int32 counters, zero between calls.
#pragma once

#include "decode_mma_e4m3.cuh"

namespace pkv {

__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Shared memory of a CTA: the ring barriers, then per warp 3 descriptors and
// 2 table buffers, then the rings (1 KB aligned for the 128-byte swizzle).
template <int D, int BS, int NW, int STAGES_>
struct StreamCfg {
    using C = MmaE4m3Cfg<D, BS, NW, STAGES_>;
    static constexpr int TAB = 32;  // table entries per warp and piece: 32 slices
    static constexpr int META = NW * (3 * PKV_PLAN_ITEM_WORDS + 2 * TAB) * 4;
    static constexpr int HEAD = 128 + META;  // the rings follow, 1 KB aligned at run time
    static constexpr int SMEM = HEAD + 1024 + C::RING_BYTES;
    static constexpr int MAX_PIECE = TAB * 16 * NW;  // tokens of the largest piece
};

template <typename T, int D, int BS, int NH, int NW, int STAGES_, bool PPB>
__global__ void __launch_bounds__(NW * 32, E4m3MinBlocks<D, NH, NW, STAGES_>::value)
    decode_stream_e4m3_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                              const __grid_constant__ CUtensorMap tmv) {
    using C = MmaE4m3Cfg<D, BS, NW, STAGES_>;
    using S = StreamCfg<D, BS, NW, STAGES_>;
    constexpr int NX = C::NX, BOX_BYTES = C::BOX_BYTES;
    constexpr int SLICE_BYTES = C::SLICE_BYTES, WARP_RING = C::WARP_RING;
    constexpr int STAGES = C::STAGES;
    constexpr int KSTEPS = D / 16, KP = KSTEPS / 2, RB = NH / 8;
    constexpr int IW = PKV_PLAN_ITEM_WORDS;
    constexpr bool EARLY = D <= 128 && NH == 8;
    constexpr int MS = NH == 8 ? 2 : RB;
    constexpr int QR = NH == 16 ? 4 : 2;

    extern __shared__ __align__(1024) unsigned char smem_st[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem_st) + warp * STAGES;
    int32_t* desc = reinterpret_cast<int32_t*>(smem_st + 128) +
                    warp * (3 * IW + 2 * S::TAB);            // [3][IW]
    int32_t* tabs = desc + 3 * IW;                            // [2][TAB]
    unsigned char* ring;
    {
        const uint32_t base = smem_u32(smem_st + S::HEAD);
        const uint32_t aligned = (base + 1023u) & ~1023u;  // 128-byte swizzle: 1 KB atoms
        ring = smem_st + S::HEAD + (aligned - base) + warp * WARP_RING;
    }
    const uint32_t ring_s = smem_u32(ring);

    const int i0 = a.plan_cta[blockIdx.x];
    const int n = a.plan_cta[blockIdx.x + 1] - i0;  // this CTA's pieces
    const int units = a.num_seqs * a.num_kv_heads * a.head_chunks;

    if (lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmk)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv)) : "memory");
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }

    // -- descriptors and table entries (device data: every field is checked) --
    // A piece this warp cannot use is "dead": no slices, no partial state, and
    // flagged; its unit is then never completed (its rows stay unwritten).
    auto fetch_desc = [&](int i) {  // cp.async of piece i's descriptor
        if (i < n && lane < IW) cp_async4(desc + (i % 3) * IW + lane, a.plan_items + (int64_t)(i0 + i) * IW + lane);
    };
    // ntok of piece i, or -1 when its descriptor is not valid here
    auto piece_tokens = [&](int i) -> int {
        const int32_t* d = desc + (i % 3) * IW;
        const int b = d[0], y = d[1], t0 = d[2], t1 = d[3], ml = d[4], unit = d[5], slot0 = d[6],
                  np = d[7], pi = d[8];
        if ((unsigned)b >= (unsigned)a.num_seqs ||
            (unsigned)y >= (unsigned)(a.num_kv_heads * a.head_chunks) || t0 < 0 || t0 % BS != 0 ||
            t1 < t0 || t1 - t0 > S::MAX_PIECE || ml < 0 || ml > t1 - t0 ||
            (unsigned)unit >= (unsigned)units || np < 1 || pi < 0 || pi >= np || slot0 < 0 ||
            (int64_t)slot0 + (int64_t)np * NW > a.ws_slots || t1 > a.max_tokens)
            return -1;
        return t1 - t0;
    };
    auto warp_slices = [&](int ntok) {  // this warp's slices of a piece of ntok tokens
        return ntok > warp * 16 ? (ntok - warp * 16 + 16 * NW - 1) / (16 * NW) : 0;
    };
    // cp.async of this warp's table entries for piece i (its descriptor landed)
    auto fetch_tab = [&](int i, int ntok) {
        if (i >= n || ntok <= 0) return;
        const int32_t* d = desc + (i % 3) * IW;
        const int32_t* trow = a.block_tables + (int64_t)d[0] * a.max_blocks_per_seq + d[2] / BS;
        if (lane < warp_slices(ntok)) cp_async4(tabs + (i & 1) * S::TAB + lane, trow + (warp + NW * lane) * 16 / BS);
    };

    // -- the producer: lane 0 issues slice pj of piece pi into ring position pgk --
    // Pieces up to open_i have their table here; their slices for this warp
    // and their KV head are kept for the two pieces the producer can be in
    // (by parity).
    const uint64_t pol = policy_evict_first();
    int pi = 0, pj = 0, pgk = 0, open_i = -1;
    int ns_p[2] = {0, 0}, kvh_p[2] = {0, 0};
    auto set_open = [&](int i, int ntok) {  // piece i's table is here
        const int ns = ntok > 0 ? warp_slices(ntok) : 0;
        const int kv = desc[(i % 3) * IW + 1] / a.head_chunks;
        if (i & 1) {
            ns_p[1] = ns;
            kvh_p[1] = kv;
        } else {
            ns_p[0] = ns;
            kvh_p[0] = kv;
        }
        open_i = i;
    };
    int ci = 0;         // the piece the consumer works on
    int ntok_next = 0;  // tokens of piece ci + 1 (-1: dead)
    auto open_next = [&]() {  // wait for piece ci + 1's table (all lanes)
        cp_async_wait_all();
        __syncwarp();
        set_open(ci + 1, ntok_next);
    };
    // issue while a stage is free and the next slice lies in a piece whose
    // table is here (the producer waits at piece ci + 2)
    auto top_up = [&](int gk) {
        while (pgk - gk < STAGES && pi < n) {
            if (pi > open_i) {
                if (pi == ci + 1) open_next();
                else return;
            }
            const int ns = (pi & 1) ? ns_p[1] : ns_p[0];
            if (pj >= ns) {  // on to the next piece
                ++pi;
                pj = 0;
                continue;
            }
            if (lane == 0) {
                int32_t blk = tabs[(pi & 1) * S::TAB + pj];
                if ((unsigned)blk >= (unsigned)a.num_blocks) {
                    flag(a.status, PKV_DEV_BAD_BLOCK);
                    blk = 0;
                }
                const int kv = (pi & 1) ? kvh_p[1] : kvh_p[0];
                const int tok = (warp + NW * pj) * 16;
                const int yrow = (blk * a.num_kv_heads + kv) * BS + tok % BS;
                const int stage = pgk % STAGES;
                mbar_arrive_expect_tx(&full[stage], (uint32_t)(2 * SLICE_BYTES));
                unsigned char* kd = ring + stage * 2 * SLICE_BYTES;
#pragma unroll
                for (int x = 0; x < NX; ++x) {
                    tma_load_2d(kd + x * BOX_BYTES, &tmk, x * 128, yrow, &full[stage], pol);
                    tma_load_2d(kd + SLICE_BYTES + x * BOX_BYTES, &tmv, x * 128, yrow,
                                &full[stage], pol);
                }
            }
            ++pj;
            ++pgk;
        }
    };

    // prologue: descriptors of pieces 0, 1 (2 comes at piece 0's start), the
    // table of piece 0
    fetch_desc(0);
    fetch_desc(1);
    cp_async_wait_all();
    __syncwarp();
    int ntok_cur = n > 0 ? piece_tokens(0) : 0;
    if (ntok_cur < 0 && lane == 0) flag(a.status, PKV_DEV_BAD_PLAN);
    fetch_tab(0, ntok_cur);
    cp_async_wait_all();
    __syncwarp();
    if (n > 0) set_open(0, ntok_cur);

    // ldmatrix.x4 row addresses (see decode_mma_e4m3_kernel)
    const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int lchunk = lane >> 4;
    const int swz = lrow & 7;
    int gk = 0;  // ring position of the consumer

    for (; ci < n; ++ci) {
        // the descriptor of piece ci + 1 landed with the last wait; fetch its
        // table and the descriptor of ci + 2 (one cp.async group)
        ntok_next = ci + 1 < n ? piece_tokens(ci + 1) : 0;
        if (ntok_next < 0 && lane == 0) flag(a.status, PKV_DEV_BAD_PLAN);
        fetch_tab(ci + 1, ntok_next);
        fetch_desc(ci + 2);
        const int32_t* d = desc + (ci % 3) * IW;
        const int b = d[0], y = d[1], t0 = d[2], mask_lo = d[4], unit = d[5], slot0 = d[6],
                  np = d[7], pidx = d[8];
        const int ntok = ntok_cur;  // -1: a dead piece
        const int kvh = y / a.head_chunks, hc = y - kvh * a.head_chunks;
        const int h0 = kvh * a.group + hc * NH;
        const int nh = min(NH, a.group - hc * NH);
        const int ns = ntok > 0 ? warp_slices(ntok) : 0;
        const int32_t* tab_cur = tabs + (ci & 1) * S::TAB;

        uint32_t qa[KSTEPS][QR];
        float qmul = 0.f;
        if (ns > 0) {
            const T* qb = reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.num_q_heads + h0) * D;
            qmul = e4m3_prepare_q<T, D, NH>(
                [&](int hh) { return hh < nh ? qb + hh * D : nullptr; },
                a.scale_log2 * (PPB ? 1.f : a.k_scale[kvh]), qa, g, t4);
        }
        float m[MS], l[MS], o[KSTEPS][RB][4];
#pragma unroll
        for (int j = 0; j < MS; ++j) {
            m[j] = -INFINITY;
            l[j] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
            for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                for (int i = 0; i < 4; ++i) o[mt][rb][i] = 0.f;

        for (int j = 0; j < ns; ++j) {
            top_up(gk);
            const int stage = gk % STAGES;
            const bool ok = __all_sync(0xffffffffu,
                                       mbar_wait(&full[stage], (uint32_t)((gk / STAGES) & 1),
                                                 a.status));
            if (!ok) {  // a copy never landed: drain what this warp issued, then leave
                if (lane == 0) drain_ring(full, STAGES, gk, pgk, a.status);
                return;
            }
            const int tok = (warp + NW * j) * 16;  // the slice's first token in the piece
            const int wvalid = ntok - tok;
            const int wlo = mask_lo - tok;
            const bool work = wlo < 16 && wlo < wvalid;
            const uint32_t kbase = ring_s + (uint32_t)(stage * 2 * SLICE_BYTES + lrow * 128);
            float kmul = qmul, vmul = 1.f;
            if (PPB && work) {
                const int64_t si = (int64_t)tab_cur[j] * a.num_kv_heads + kvh;
                if ((unsigned)tab_cur[j] < (unsigned)a.num_blocks) {
                    kmul = qmul * a.k_scale[si];
                    vmul = a.v_scale[si];
                }
            }
            auto addr = [&](int kp) {
                const int chunk = 2 * kp + lchunk;
                return kbase + (chunk >> 3) * BOX_BYTES + (((chunk & 7) ^ swz) << 4);
            };
            uint32_t kf[EARLY ? KP : 1][4], vf[EARLY ? KP : 1][4];
            if (EARLY && work) {
#pragma unroll
                for (int kp = 0; kp < (EARLY ? KP : 1); ++kp) {
                    ldsm_x4(addr(kp), kf[kp]);
                    ldsm_x4_trans(addr(kp) + SLICE_BYTES, vf[kp]);
                }
            }
            if (!EARLY && work)
                e4m3_slice_math<D, NH, PPB, EARLY>(qa, m, l, o, kf, vf, addr, wvalid, wlo, kmul,
                                                   vmul, g, t4);
            __syncwarp();  // the warp's reads of the stage are done: it is free
            ++gk;
            top_up(gk);
            if (EARLY && work)
                e4m3_slice_math<D, NH, PPB, EARLY>(qa, m, l, o, kf, vf, addr, wvalid, wlo, kmul,
                                                   vmul, g, t4);
        }
        if (open_i < ci + 1 && ci + 1 < n) open_next();
        ntok_cur = ntok_next;
        if (ntok < 0) continue;  // a dead piece (flagged): no state to hand on

        // -- this warp's partial state of the piece -> its slot --
        const int64_t slot = (int64_t)slot0 + (int64_t)pidx * NW + warp;
        float* po = a.ws_o + slot * NH * D;
        float* pml = a.ws_ml + slot * NH * 2;
        const float vs_out = PPB ? 1.f : a.v_scale[kvh];
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
            for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int head = 8 * rb + 2 * t4 + (i & 1);
                    const int dim = mt * 16 + 2 * g + (i >> 1);
                    po[head * D + dim] = o[mt][rb][i] * vs_out;
                }
        if constexpr (NH == 8) {  // heads 2 t4 + j, summed over the lanes of one t4
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                l[j] += __shfl_xor_sync(0xffffffffu, l[j], 4);
                l[j] += __shfl_xor_sync(0xffffffffu, l[j], 8);
                l[j] += __shfl_xor_sync(0xffffffffu, l[j], 16);
            }
            if (g == 0)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    pml[(2 * t4 + j) * 2] = m[j];
                    pml[(2 * t4 + j) * 2 + 1] = l[j];
                }
        } else {  // heads g + 8 rb, summed over the lanes of one g
#pragma unroll
            for (int rb = 0; rb < RB; ++rb) {
                l[rb] += __shfl_xor_sync(0xffffffffu, l[rb], 1);
                l[rb] += __shfl_xor_sync(0xffffffffu, l[rb], 2);
            }
            if (t4 == 0)
#pragma unroll
                for (int rb = 0; rb < RB; ++rb) {
                    pml[(g + 8 * rb) * 2] = m[rb];
                    pml[(g + 8 * rb) * 2 + 1] = l[rb];
                }
        }
        __threadfence();
        __syncwarp();
        int done = 0;
        if (lane == 0) done = atomicAdd(a.plan_counts + unit, 1) + 1;
        done = __shfl_sync(0xffffffffu, done, 0);
        if (done != np * NW) continue;

        // -- the last of the unit's warps: merge its partial states --
        __threadfence();
        const int nparts = np * NW;
        const float* mlu = a.ws_ml + (int64_t)slot0 * NH * 2;
        const float* ou = a.ws_o + (int64_t)slot0 * NH * D;
        T* out = reinterpret_cast<T*>(a.out) + ((int64_t)b * a.num_q_heads + h0) * D;
        // lane: heads hh = lane % NH ... every (head, 4 dims) pair in turn
        constexpr int PAIRS = NH * D / 4;
        for (int pq = lane; pq < PAIRS; pq += 32) {
            const int hh = pq / (D / 4), d4 = (pq % (D / 4)) * 4;
            if (hh >= nh) continue;
            float M = -INFINITY;
            for (int p = 0; p < nparts; ++p) M = fmaxf(M, __ldcg(mlu + ((int64_t)p * NH + hh) * 2));
            float den = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (M != -INFINITY) {
                for (int p = 0; p < nparts; ++p) {
                    const float mp = __ldcg(mlu + ((int64_t)p * NH + hh) * 2);
                    const float f = exp2f(mp - M);  // 0 for a warp with no tokens
                    den = fmaf(f, __ldcg(mlu + ((int64_t)p * NH + hh) * 2 + 1), den);
                    const float4 x =
                        __ldcg(reinterpret_cast<const float4*>(ou + ((int64_t)p * NH + hh) * D + d4));
                    acc[0] = fmaf(f, x.x, acc[0]);
                    acc[1] = fmaf(f, x.y, acc[1]);
                    acc[2] = fmaf(f, x.z, acc[2]);
                    acc[3] = fmaf(f, x.w, acc[3]);
                }
            }
            const float inv = den > 0.f ? 1.f / den : 0.f;  // an empty sequence: zeros
#pragma unroll
            for (int k = 0; k < 4; ++k) out[hh * D + d4 + k] = Elem<T>::from_f32(acc[k] * inv);
        }
        if (lane == 0) a.plan_counts[unit] = 0;  // ready for the next call
    }
    // every issued copy has been consumed (the producer never runs past the
    // CTA's last piece)
}

}  // namespace pkv
