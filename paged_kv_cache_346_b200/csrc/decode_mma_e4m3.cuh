// Paged decode attention over FP8 E4M3 pages on the tensor cores.
//
// The same two contractions as the 16-bit tensor-core kernel,
//   S[h, t] = sum_d Q[h, d] K[t, d]        O^T[d, h] = sum_t V[t, d] P[h, t],
// with mma.sync m16n8k16 in fp16 (fp32 accumulation).  A tile of 8 heads
// computes S as K Q^T (M = the slice's 16 tokens, N = 8 heads: one MMA per
// 16-dim step, where an 8-head S^T tile fills half of M); a 16-head tile
// computes S^T as Q K^T (M = heads, N = tokens).  The pages stay one
// byte per element all the way into the registers: ldmatrix moves 16-byte
// rows of codes, and each register of four codes becomes two f16x2 operand
// registers with the hardware E4M3 -> f16x2 conversion (exact: every E4M3
// value is an f16 value).  Quantised pages are the paged layout combined with
// a compressed cache ("pagedattention vllm" §Comparison with Alternatives).
//
// Operand layouts (the contraction order is free, so the byte layout that
// ldmatrix delivers is kept and the other operand is arranged to match):
//   * K: ldmatrix (non-transposed) hands lane (g, t4) the codes
//     K[t = g][4 t4 .. 4 t4 + 3] of a 16-dim step (and of t = g + 8).  The low
//     pair serves logical k = 2 t4, 2 t4 + 1, the high pair k = 2 t4 + 8, + 9,
//     so Q's fragment (B columns of an 8-head tile, A rows of a 16-head tile)
//     takes dims 4 t4, 4 t4 + 1 and 4 t4 + 2, 4 t4 + 3 at those positions.
//     An 8-head tile's S accumulator gives lane (g, t4) tokens g, g + 8 of
//     heads 2 t4, 2 t4 + 1; after rounding to fp16, one movmatrix.trans per 8
//     tokens turns it into P^T's B fragment (head g, tokens 2 t4, 2 t4 + 1).
//     A 16-head tile's S^T accumulator is already that fragment.
//   * V^T as the A operand of O^T: ldmatrix.trans on 2-byte units hands lane
//     (g, t4) the codes V[2 t4][2 g], V[2 t4][2 g + 1], V[2 t4 + 1][2 g],
//     V[2 t4 + 1][2 g + 1].  One byte permute makes the token pairs of dims
//     2 g and 2 g + 1: A rows g and g + 8 of an m-tile are dims 2 g and 2 g + 1
//     of its 16, and the tokens (k) keep their natural order.
//
// q (fp16 or bf16) enters the fp16 MMA multiplied by a power of two 2^e that
// puts its largest magnitude in [2^14, 2^15) (exact for every value that stays
// an f16 normal); the logits are multiplied back by scale * log2(e) *
// k_scale * 2^-e in fp32, and the output by v_scale.  With a scale per page,
// a warp's 16-token slice lies in one block: its logits take that page's
// k_scale, and the warp keeps its P.V sums in units of a reference V scale
// vref.  A page whose v_scale lies in [vref, 128 vref] enters with its
// weights times v_scale / vref (then at most 2^15: still an fp16 hi + lo
// pair, no less precise than p itself); any other page first moves vref to
// its v_scale / 8 and rescales the fp32 sums, as a rise of the reference max
// does.  The warp's output is multiplied by vref.
//
// Each softmax weight p (fp32) enters the P.V product as two fp16 terms,
// hi = fp16(p) and lo = fp16(p - hi), in two MMAs on the same V fragment: one
// fp16 term keeps 11 significant bits, and the output error it leaves,
// ~2^-11 times the largest |v|, exceeds the fp16 / bf16 tolerance once values
// are large (e.g. per-page V scales spread over decades); hi + lo keeps ~22.
// The row sums l add the fp32 weights themselves: p - (hi + lo) is the
// rounding of the remainder, at most 2^-23 p + 2^-25 (the second term only
// where p is below fp16's normal range), so the normaliser differs from the
// sum of the weights the products used by less than 2^-23 of it plus 2^-25
// per token, against l >= 1 (the reference max's own token has p = 1).
#pragma once

#include "decode_mma.cuh"

namespace pkv {

// Every warp streams its own 16-token slices through a private ring of
// STAGES stages (STAGES_ = 0: 4), one 16-row TMA box
// per 128 columns of K and of V per slice, issued by the warp's lane 0, so no
// barrier ties the warps together until the final merge.  Measured on B200
// against one ring shared by the CTA (refilled after a CTA barrier by one
// thread): +20 % on the MHA layer, +15 % on the GQA batch, +24-32 % on long
// contexts.
template <int D, int BS, int NW, int STAGES_ = 0>
struct MmaE4m3Cfg {
    static constexpr int TILE = 16 * NW;          // tokens per round of all warps
    static constexpr int NX = D / 128;            // 128-column boxes per row
    static constexpr int BOX_BYTES = 16 * 128;    // one box: 16 rows x 128 bytes
    static constexpr int SLICE_BYTES = 16 * D;    // one warp's 16 tokens of K (or V)
    static constexpr int STAGES = STAGES_ ? STAGES_ : 4;
    static constexpr int WARP_RING = STAGES * 2 * SLICE_BYTES;
    static constexpr int RING_BYTES = NW * WARP_RING;
    static_assert(BS % 16 == 0 && D % 128 == 0, "16-token slices of 128-byte rows");

    static int smem_bytes(int partition_size) {
        // barriers, table slice, slack to the ring's 1 KB (swizzle atom) alignment
        return 128 + round_up(partition_size / BS * 4, 128) + 1024 + RING_BYTES;
    }
};

// four E4M3 codes (bytes 0..3) -> f16x2 of bytes 0, 1 (lo) and of bytes 2, 3
// (hi); the lower byte of each pair goes to the lower half
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// d += A B, fp16 operands given as separate registers (a constant 0 for an
// all-zero row block lets the compiler use the zero register)
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t byte_perm(uint32_t x, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(x), "r"(sel));
    return r;
}

// a pair rounded to f16x2 (lo in the low half)
__device__ __forceinline__ uint32_t f16x2_rn(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// CTAs per SM the register allocation is held to.  8-head tiles at head_dim
// 128 fit 128 registers without spills, so with 3-stage rings (whose shared
// memory then also fits) four 4-warp or eight 2-warp CTAs share an SM: 16
// warps instead of 12 to cover the issue latency of the conversions and the
// softmax.  Otherwise three CTAs (8-head tiles) or one.
template <int D, int NH, int NW, int STAGES_>
struct E4m3MinBlocks {
    static constexpr int value =
        (D <= 128 && NH == 8) ? (D == 128 && STAGES_ == 3 ? 16 / NW : 3) : 1;
};

// q (fp16 or bf16) as the fp16 MMA operand: rows g (and g + 8 when NH is 16)
// of the tile, qrow(hh) giving head hh's row (nullptr: a zero row), dims in
// the order ldmatrix delivers the K codes (k = 2 t4 + j -> dim 4 t4 + j,
// k = 2 t4 + 8 + j -> dim 4 t4 + 2 + j), scaled by the power of two 2^e that
// puts the tile's largest |q| in [2^14, 2^15).  Returns the logits'
// multiplier, mul * 2^-e.  All 32 lanes take part.
template <typename T, int D, int NH, typename QRow>
__device__ __forceinline__ float e4m3_prepare_q(QRow qrow, float mul,
                                                uint32_t (&qa)[D / 16][NH == 16 ? 4 : 2], int g,
                                                int t4) {
    constexpr int KSTEPS = D / 16;
    float qf[KSTEPS][2][4];
    float mx = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const T* row = qrow(g + 8 * r);
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                qf[ks][r][j] = row ? Elem<T>::load1(row + ks * 16 + 4 * t4 + j) : 0.f;
                mx = fmaxf(mx, fabsf(qf[ks][r][j]));
            }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    // 2^e with mx * 2^e in [2^14, 2^15): e = 141 - biased exponent of mx
    const int be = (__float_as_int(mx) >> 23) & 0xff;
    int e = be == 0 ? 0 : 141 - be;
    e = max(-126, min(126, e));
    const float up = __int_as_float((127 + e) << 23);
    const float down = __int_as_float((127 - e) << 23);
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const __half2 lo = __floats2half2_rn(qf[ks][r][0] * up, qf[ks][r][1] * up);
            const __half2 hi = __floats2half2_rn(qf[ks][r][2] * up, qf[ks][r][3] * up);
            if (NH == 16 || r == 0) {
                // NH 16: qa = a0a1, a2a3, a4a5, a6a7; NH 8: qa = a0a1, a4a5
                qa[ks][NH == 16 ? r : 0] = *reinterpret_cast<const uint32_t*>(&lo);
                qa[ks][NH == 16 ? 2 + r : 1] = *reinterpret_cast<const uint32_t*>(&hi);
            }
        }
    return mul * down;
}

// One warp's work on one 16-token slice of K and V (codes in its ring stage,
// or already in kf / vf with EARLY): the logits, the online softmax against
// the lazy reference max, and O^T += V^T P^T with P as fp16 hi + lo.  The
// state (m, l, o) is the warp's; addr(kp) is the ldmatrix address of chunk
// pair kp of the slice's K rows (V rows: + 16 D bytes); tokens outside
// [wlo, wvalid) of the slice are masked.  PPB: the weights enter P.V times
// pmul, the page's V scale over the warp's reference (in [1, 128], so p pmul
// is at most 2^15), while l sums the weights themselves.
template <int D, int NH, bool PPB, bool EARLY, typename Addr>
__device__ __forceinline__ void e4m3_slice_math(
    const uint32_t (&qa)[D / 16][NH == 16 ? 4 : 2], float (&m)[NH == 8 ? 2 : NH / 8],
    float (&l)[NH == 8 ? 2 : NH / 8], float (&o)[D / 16][NH / 8][4],
    const uint32_t (&kf)[EARLY ? D / 32 : 1][4], uint32_t (&vf)[EARLY ? D / 32 : 1][4],
    Addr addr, int wvalid, int wlo, float kmul, float pmul, int g, int t4) {
    using M = Mma<__half>;
    constexpr int KSTEPS = D / 16, KP = KSTEPS / 2, RB = NH / 8;
    constexpr int SLICE_BYTES = 16 * D;
    (void)pmul;
    (void)SLICE_BYTES;
    const bool partial = wvalid < 16 || wlo > 0;
    bool grew;               // the reference max moved: rescale o
    float alpha_c[RB][2];    // rescale factors of o's columns 2 t4, 2 t4 + 1
    uint32_t pb[RB][2];      // P^T as the B operand: tokens 0-7, 8-15 (fp16 hi)
    uint32_t pl[RB][2];      // the fp16 remainders p - hi, same layout (lo)
    auto kcodes = [&](int kp, uint32_t (&kc)[4]) {
        if constexpr (EARLY) {
#pragma unroll
            for (int i = 0; i < 4; ++i) kc[i] = kf[kp < (EARLY ? KP : 1) ? kp : 0][i];
        } else {
            ldsm_x4(addr(kp), kc);
        }
    };
    if constexpr (NH == 8) {
        // S[t, h] = K Q^T with the slice's 16 tokens as M and the 8
        // heads as N: one MMA per 16-dim step (an 8-head S^T tile
        // would fill half of M).  K codes of tokens g / g + 8 are the
        // A rows, q the B columns; two accumulator sets (even / odd
        // steps) make two short dependency chains.
        float s[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kp = 0; kp < KP; ++kp) {
            uint32_t kc[4];
            kcodes(kp, kc);
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // k-step 2 kp + h
                uint32_t k0, k1, k2, k3;
                e4m3x4_to_f16x2(kc[2 * h], k0, k1);      // token g
                e4m3x4_to_f16x2(kc[2 * h + 1], k2, k3);  // token g + 8
                const uint32_t* q4 = qa[2 * kp + h];
                mma_f16(h ? s2 : s, k0, k2, k1, k3, q4[0], q4[1]);
            }
        }
        // lane (g, t4): s[0], s[1] = token g, heads 2 t4, 2 t4 + 1;
        // s[2], s[3] = token g + 8
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            s[i] = (s[i] + s2[i]) * kmul;
            const int tok = g + 8 * (i >> 1);
            if (partial && (tok < wlo || tok >= wvalid)) s[i] = -INFINITY;
        }
        // lazy reference max per head (see below); a head's tokens
        // are spread over the 8 lanes of one t4
        bool up = false;
        float tmax[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            tmax[j] = fmaxf(s[j], s[2 + j]);
            up |= tmax[j] > m[j] + 8.f;
        }
        grew = __any_sync(0xffffffffu, up);
        if (grew) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float mx = tmax[j];
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float mnew = fmaxf(m[j], mx);
                const float alpha = ex2_approx(m[j] - mnew);
                l[j] *= alpha;
                m[j] = mnew;
                alpha_c[0][j] = alpha;
            }
        }
        float p[4], pr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = ex2_approx(s[i] - m[i & 1]);
        l[0] += p[0] + p[2];
        l[1] += p[1] + p[3];
        if constexpr (PPB) {
#pragma unroll
            for (int i = 0; i < 4; ++i) p[i] *= pmul;
        }
        const uint32_t p0 = M::pack(p[0], p[1], pr[0], pr[1]);
        const uint32_t p1 = M::pack(p[2], p[3], pr[2], pr[3]);
        const uint32_t r0 = f16x2_rn(p[0] - pr[0], p[1] - pr[1]);
        const uint32_t r1 = f16x2_rn(p[2] - pr[2], p[3] - pr[3]);
        // P (tokens x heads) -> P^T fragments: lane (g, t4) gets head
        // g, tokens 2 t4, 2 t4 + 1 (of 0-7, then of 8-15)
        pb[0][0] = movmatrix_trans(p0);
        pb[0][1] = movmatrix_trans(p1);
        pl[0][0] = movmatrix_trans(r0);
        pl[0][1] = movmatrix_trans(r1);
    } else {
        // 16-head tiles: S^T[h, t] = Q K^T, heads as M, the slice's
        // tokens as N (two n-tiles), two accumulator sets
        float s[2][4], s2[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) s[nt][i] = s2[nt][i] = 0.f;
#pragma unroll
        for (int kp = 0; kp < KP; ++kp) {
            uint32_t kc[4];
            kcodes(kp, kc);
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // k-step 2 kp + h
                uint32_t b0, b1, b2, b3;
                e4m3x4_to_f16x2(kc[2 * h], b0, b1);      // tokens 0-7
                e4m3x4_to_f16x2(kc[2 * h + 1], b2, b3);  // tokens 8-15
                const uint32_t* q4 = qa[2 * kp + h];
                mma_f16(h ? s2[0] : s[0], q4[0], q4[1], q4[2], q4[3], b0, b1);
                mma_f16(h ? s2[1] : s[1], q4[0], q4[1], q4[2], q4[3], b2, b3);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) s[nt][i] = (s[nt][i] + s2[nt][i]) * kmul;
        if (partial) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tok = nt * 8 + 2 * t4 + (i & 1);
                    if (tok < wlo || tok >= wvalid) s[nt][i] = -INFINITY;
                }
        }
        // Softmax against a reference max m that moves only when a
        // logit exceeds it by more than 2^8 (then p <= 256 fits fp16
        // and the accumulators are rescaled); l is kept per lane (this
        // lane's tokens) and summed over the head's lanes at the end.
        // The result is the same softmax: every p and l of a head
        // shares m.
        bool up = false;
        float tmax[RB];
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) {
            const int i0 = 2 * rb;
            tmax[rb] = fmaxf(fmaxf(s[0][i0], s[0][i0 + 1]), fmaxf(s[1][i0], s[1][i0 + 1]));
            up |= tmax[rb] > m[rb] + 8.f;
        }
        grew = __any_sync(0xffffffffu, up);
        if (grew) {
#pragma unroll
            for (int rb = 0; rb < RB; ++rb) {
                float mx = tmax[rb];
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float mnew = fmaxf(m[rb], mx);
                const float alpha = ex2_approx(m[rb] - mnew);
                l[rb] *= alpha;
                m[rb] = mnew;
                alpha_c[rb][0] = __shfl_sync(0xffffffffu, alpha, (2 * t4) * 4);
                alpha_c[rb][1] = __shfl_sync(0xffffffffu, alpha, (2 * t4 + 1) * 4);
            }
        }
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) {
            const int i0 = 2 * rb;
            float ps[2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float p0 = ex2_approx(s[nt][i0] - m[rb]);
                float p1 = ex2_approx(s[nt][i0 + 1] - m[rb]);
                ps[nt] = p0 + p1;
                if constexpr (PPB) {
                    p0 *= pmul;
                    p1 *= pmul;
                }
                float h0, h1;
                pb[rb][nt] = M::pack(p0, p1, h0, h1);
                pl[rb][nt] = f16x2_rn(p0 - h0, p1 - h1);
            }
            l[rb] += ps[0] + ps[1];
        }
    }
    // The rescale and the masking sit outside the P.V loop, which then has
    // no branch and schedules as one block.
    if (grew) {
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
            for (int rb = 0; rb < RB; ++rb) {
                o[mt][rb][0] *= alpha_c[rb][0];
                o[mt][rb][1] *= alpha_c[rb][1];
                o[mt][rb][2] *= alpha_c[rb][0];
                o[mt][rb][3] *= alpha_c[rb][1];
            }
    }
    // Codes of masked tokens become 0 (0 * NaN would poison the sum).  Code
    // register 2 h of a pair holds tokens 2 t4 (bytes 0, 1) and 2 t4 + 1
    // (bytes 2, 3), register 2 h + 1 the same tokens + 8.
    uint32_t keep[2] = {~0u, ~0u};
    if (partial) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int tk = 8 * j + 2 * t4;
            keep[j] = (tk >= wlo && tk < wvalid ? 0x0000ffffu : 0u) |
                      (tk + 1 >= wlo && tk + 1 < wvalid ? 0xffff0000u : 0u);
        }
        if constexpr (EARLY) {
#pragma unroll
            for (int kp = 0; kp < (EARLY ? KP : 1); ++kp)
#pragma unroll
                for (int i = 0; i < 4; ++i) vf[kp][i] &= keep[i & 1];
        }
    }
#pragma unroll
    for (int kp = 0; kp < KP; ++kp) {
        uint32_t vc[4];
        if constexpr (EARLY) {
#pragma unroll
            for (int i = 0; i < 4; ++i) vc[i] = vf[kp < (EARLY ? KP : 1) ? kp : 0][i];
        } else {
            ldsm_x4_trans(addr(kp) + SLICE_BYTES, vc);
#pragma unroll
            for (int i = 0; i < 4; ++i) vc[i] &= keep[i & 1];
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // m-tile 2 kp + h
            const int mt = 2 * kp + h;
            uint32_t va[4];
            // (V[r0][2g], V[r0][2g+1], V[r1][2g], V[r1][2g+1]) ->
            // (V[r0][2g], V[r1][2g] | V[r0][2g+1], V[r1][2g+1])
            e4m3x4_to_f16x2(byte_perm(vc[2 * h], 0x3120u), va[0], va[1]);
            e4m3x4_to_f16x2(byte_perm(vc[2 * h + 1], 0x3120u), va[2], va[3]);
#pragma unroll
            for (int rb = 0; rb < RB; ++rb) {
                mma_f16(o[mt][rb], va[0], va[1], va[2], va[3], pb[rb][0], pb[rb][1]);
                mma_f16(o[mt][rb], va[0], va[1], va[2], va[3], pl[rb][0], pl[rb][1]);
            }
        }
    }
}

// PPB: a scale per page (a.scale_per_block), a compile-time choice so the
// per-head path carries no per-slice scale code.
template <typename T, int D, int BS, int NH, int NW, int STAGES_, bool PPB>
__global__ void __launch_bounds__(NW * 32, E4m3MinBlocks<D, NH, NW, STAGES_>::value)
    decode_mma_e4m3_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                           const __grid_constant__ CUtensorMap tmv) {
    using C = MmaE4m3Cfg<D, BS, NW, STAGES_>;
    using M = Mma<__half>;
    constexpr int TILE = C::TILE, NX = C::NX, BOX_BYTES = C::BOX_BYTES;
    constexpr int SLICE_BYTES = C::SLICE_BYTES, WARP_RING = C::WARP_RING;
    constexpr int STAGES = C::STAGES;
    constexpr int KSTEPS = D / 16;   // k-steps of QK, m-tiles of PV (one 16-byte chunk each)
    constexpr int KP = KSTEPS / 2;   // ldmatrix.x4 loads per warp tile (two chunks each)
    constexpr int RB = NH / 8;
    constexpr bool EARLY = D <= 128 && NH == 8;

    extern __shared__ __align__(1024) unsigned char smem_mma8[];
    __shared__ int s_abort;
    // Launched as a programmatic dependent of the kernel before it (usually
    // the KV append): the schedule, lengths and table (which that kernel does
    // not write) are read before griddepcontrol.wait, so the start-up of the
    // first wave overlaps it; the pages and scales are read, and anything is
    // written, only after it (pdl_wait_before_pages).

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int kvh = blockIdx.y / a.head_chunks;
    const int hc = blockIdx.y - kvh * a.head_chunks;
    const CtaUnit unit = cta_unit(a, tid);  // (sequence, partition)
    const int part = unit.part;
    const int h0 = kvh * a.group + hc * NH;
    const int nh = min(NH, a.group - hc * NH);
    const bool reporter = (tid == 0 && part == 0 && blockIdx.y == 0);
    const int b = unit.b;
    if (b < 0) return;

    const TablePrefetch pf = table_prefetch(a, b, part, a.partition_size / BS, tid);
    const Span sp = seq_span(a, b, reporter);
    const int L = sp.L, np = sp.np;
    T* out = reinterpret_cast<T*>(a.out);
    if (L == 0) {
        if (part == 0) {
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
    const int mask_lo = part == 0 ? sp.lo - sp.base : 0;
    const int nblk = (ntok + BS - 1) / BS;
    // this warp's slices: tokens [k * TILE + warp * 16, + 16), k < nslices
    const int nslices = ntok > warp * 16 ? (ntok - warp * 16 + TILE - 1) / TILE : 0;

    uint64_t* full = reinterpret_cast<uint64_t*>(smem_mma8);  // [NW][STAGES]
    static_assert(NW * STAGES * 8 <= 128, "barriers");
    int32_t* s_tab = reinterpret_cast<int32_t*>(smem_mma8 + 128);
    unsigned char* s_kv;
    {
        const uint32_t base = smem_u32(smem_mma8 + 128 + round_up(P / BS * 4, 128));
        const uint32_t aligned = (base + 1023u) & ~1023u;  // 128-byte swizzle: 1 KB atoms
        s_kv = smem_mma8 + 128 + round_up(P / BS * 4, 128) + (aligned - base);
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
            tma_load_2d(kd + x * BOX_BYTES, &tmk, x * 128, y, bar, pol);
            tma_load_2d(kd + SLICE_BYTES + x * BOX_BYTES, &tmv, x * 128, y, bar, pol);
        }
    };
    pdl_wait_before_pages(a);
    if (lane == 0) {
        const int pre = min(STAGES, nslices);
        for (int s = 0; s < pre; ++s) issue(s, s);
    }

    // Q as the A operand (rows = heads g, g + 8), dims in the order the K
    // codes arrive (e4m3_prepare_q)
    constexpr int QR = NH == 16 ? 4 : 2;
    uint32_t qa[KSTEPS][QR];
    const T* qb = reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.num_q_heads + h0) * D;
    // logits multiplier: scale * log2(e) * k_scale * 2^-e
    const float qmul = e4m3_prepare_q<T, D, NH>(
        [&](int hh) { return hh < nh ? qb + hh * D : nullptr; },
        a.scale_log2 * (PPB ? 1.f : a.k_scale[kvh]), qa, g, t4);

    // softmax state: 8-head tiles keep it for heads 2 t4, 2 t4 + 1 (the S
    // columns of this lane), 16-head tiles for heads g + 8 rb (its S^T rows)
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

    // ldmatrix.x4 row addresses: matrices (tokens 0-7, chunk c), (tokens 8-15,
    // chunk c), (tokens 0-7, chunk c + 1), (tokens 8-15, chunk c + 1)
    const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int lchunk = lane >> 4;
    const int swz = lrow & 7;

    // the output's V scale: the KV head's, or (per-page scales) the warp's
    // reference vref: o holds the P.V sums in units of vref, a page whose
    // scale v lies in [vref, 128 vref] enters with its weights times v / vref,
    // and any other page first moves vref to v / 8, rescaling o
    const float vs_out = PPB ? 1.f : a.v_scale[kvh];
    float vref = 0.f, inv_vref = 0.f;

    int stage = 0;       // it % STAGES
    uint32_t phase = 0;  // (it / STAGES) & 1
    // per-page mode: the scales of the warp's first slice.  Scale indices
    // are 32-bit: table entries are checked against the pool, whose
    // num_blocks * Hkv * block_size rows this kernel's tensor maps address
    // with 32-bit coordinates.
    float ks_next = 1.f, vs_next = 1.f;
    if (PPB && EARLY && nslices > 0) {
        const uint32_t si =
            (uint32_t)s_tab[(warp * 16) / BS] * (uint32_t)a.num_kv_heads + (uint32_t)kvh;
        ks_next = a.k_scale[si];
        vs_next = a.v_scale[si];
    }
    for (int it = 0; it < nslices; ++it) {
        const bool ok =
            __all_sync(0xffffffffu, mbar_wait(full + warp * STAGES + stage, phase, a.status));
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
        // this slice's page scales (per-page mode): logits and P.V multipliers;
        // with 8-head tiles at head_dim <= 128 loaded one slice ahead (their
        // latency hides behind a slice's math; elsewhere that spills)
        float kmul = qmul, vmul = 1.f;
        if constexpr (PPB && EARLY) {
            kmul = qmul * ks_next;
            vmul = vs_next;
            if (it + 1 < nslices) {
                const uint32_t si = (uint32_t)s_tab[((it + 1) * TILE + warp * 16) / BS] *
                                        (uint32_t)a.num_kv_heads +
                                    (uint32_t)kvh;
                ks_next = a.k_scale[si];
                vs_next = a.v_scale[si];
            }
        } else if (PPB && work) {
            const uint32_t si = (uint32_t)s_tab[(it * TILE + warp * 16) / BS] *
                                    (uint32_t)a.num_kv_heads +
                                (uint32_t)kvh;
            kmul = qmul * a.k_scale[si];
            vmul = a.v_scale[si];
        }
        float pmul = 1.f;  // per-page: this page's v_scale / vref
        if (PPB && work) {
            pmul = vmul * inv_vref;
            if (!(pmul >= 1.f && pmul <= 128.f)) {  // warp-uniform, rare
                const float vnew = vmul * 0.125f;
                const float f = vref / vnew;  // 0 for the warp's first page (o = 0)
#pragma unroll
                for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
                    for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                        for (int i = 0; i < 4; ++i) o[mt][rb][i] *= f;
                vref = vnew;
                inv_vref = 8.f / vmul;
                pmul = vmul * inv_vref;
            }
        }
        auto addr = [&](int kp) {  // chunk pair kp: chunks 2 kp, 2 kp + 1
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
        auto math = [&]() {
            e4m3_slice_math<D, NH, PPB, EARLY>(qa, m, l, o, kf, vf, addr, wvalid, wlo, kmul, pmul,
                                               g, t4);
        };
        if (!EARLY && work) math();
        __syncwarp();  // the warp's reads of the stage are done: refill it
        if (lane == 0 && it + STAGES < nslices) issue(it + STAGES, stage);
        if (EARLY && work) math();
        if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
        }
    }
    __syncthreads();  // every warp is out of its ring (or gave up)
    if (s_abort) return;
    if (!sp.direct) pdl_launch_dependents();

    // merge the warps; A rows g, g + 8 of m-tile mt are dims 16 mt + 2 g, + 1
    using A = MergeArea<D, NH, NW>;
    static_assert(A::BYTES <= C::RING_BYTES, "merge area");
    float* red = reinterpret_cast<float*>(s_kv);
    float* red_m = red + NW * NH * A::RP;
    float* red_l = red_m + NW * NH;
    const float vs = PPB ? vref : vs_out;
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
        for (int rb = 0; rb < RB; ++rb)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int head = 8 * rb + 2 * t4 + (i & 1);
                const int dim = mt * 16 + 2 * g + (i >> 1);
                red[(warp * NH + head) * A::RP + dim] = o[mt][rb][i] * vs;
            }
    if constexpr (NH == 8) {  // heads 2 t4 + j, summed over the lanes of one t4
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
    } else {  // heads g + 8 rb, summed over the lanes of one g
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) {
            l[rb] += __shfl_xor_sync(0xffffffffu, l[rb], 1);
            l[rb] += __shfl_xor_sync(0xffffffffu, l[rb], 2);
        }
        if (t4 == 0) {
#pragma unroll
            for (int rb = 0; rb < RB; ++rb) {
                red_m[warp * NH + g + 8 * rb] = m[rb];
                red_l[warp * NH + g + 8 * rb] = l[rb];
            }
        }
    }
    __syncthreads();
    merge_warps_and_store<T, D, NH, NW>(
        a, red, [&](int hh) { return (int64_t)b * a.num_q_heads + h0 + hh; },
        [&](int hh) {
            return ((int64_t)b * a.num_q_heads + h0 + hh) * a.ws_slots + sp.slot0 + part;
        },
        nh, sp.direct, tid, NW * 32);
}

template <typename T, int D, int BS, int NH, int NW = 4, int STAGES = 0>
cudaError_t launch_decode_mma_e4m3(const DecodeArgs& a, cudaStream_t stream) {
    using C = MmaE4m3Cfg<D, BS, NW, STAGES>;
    static SmemAttr attr[2];  // one per kernel variant
    auto kern = a.scale_per_block ? decode_mma_e4m3_kernel<T, D, BS, NH, NW, STAGES, true>
                                  : decode_mma_e4m3_kernel<T, D, BS, NH, NW, STAGES, false>;
    cudaError_t e = attr[a.scale_per_block ? 1 : 0].ensure(kern, C::smem_bytes(8192));
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)a.num_blocks * a.num_kv_heads * BS;
    CUtensorMap tk, tv;
    e = make_cache_tensor_map(&tk, a.k_cache, 1, false, D, rows, 16);
    if (e != cudaSuccess) return e;
    e = make_cache_tensor_map(&tv, a.v_cache, 1, false, D, rows, 16);
    if (e != cudaSuccess) return e;
    const dim3 grid = decode_grid(a);
    e = launch_decode_kernel(kern, grid, dim3(NW * 32), C::smem_bytes(a.partition_size), stream,
                             a, tk, tv);
    if (e != cudaSuccess || a.ws_slots <= 1) return e;
    return launch_lse_reduce<T, D>(a, stream);
}

cudaError_t decode_mma_e4m3_f16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                cudaStream_t stream);
cudaError_t decode_mma_e4m3_bf16(const DecodeArgs& a, int head_dim, int block_size, int hg,
                                 cudaStream_t stream);
}  // namespace pkv
