/*
 * CPU oracle for paged decode attention, float64.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library links or calls this file;
 * only the tests, the smoke check and the benchmark's CPU-baseline leg load it.
 * It shares no code, header or constant with the CUDA path.
 *
 * What it computes is the plain definition the pages give:
 *   - each sequence's keys and values live in fixed-size blocks spread over a
 *     physical pool, and a per-sequence block table maps logical block i to a
 *     physical block ("What is PagedAttention ..." §How it works;
 *     "pagedattention vllm" §PagedAttention Design, Block Table);
 *   - attention reads them through that table, translating each position to a
 *     physical block, and computes exactly what attention over a contiguous
 *     cache computes ("pagedattention vllm" §Attention Computation: block-wise
 *     attention, address translation; systemdesign.academy "Paged Attention"
 *     FAQ answer on whether the model's results change: they do not).
 *
 * So, for sequence b and query head h (G = Hq / Hkv query heads share KV head
 * g = h / G), with L = context_lens[b]:
 *     k_t = K[table[b][t / bs], g, t % bs, :]   (same for v_t), lo <= t < L
 *     s_t = scale * sum_d q[b,h,d] k_t[d]
 *     out[b,h,:] = sum_t exp(s_t - max s) v_t / sum_t exp(s_t - max s)
 * in float64, plain loops, no blocking and no online rescaling.  L = 0 gives a
 * zero row.  Quantised caches (FP8 E4M3 codes) hold code * scale, with one
 * scale per KV head for K and one for V, or one per (physical block, KV head)
 * page (paging combines with quantisation: "pagedattention vllm"
 * §Comparison with Alternatives).
 * lo = 0, or with a sliding window of W tokens lo = max(0, L - W):
 * only the last W tokens are attended to ("pagedattention vllm" §Advanced
 * Features: sliding-window models keep only recent blocks).  The inputs are decoded bit by bit from their storage type
 * (float32, IEEE binary16, bfloat16) by this file's own decoders.
 *
 * OpenMP spreads the independent (b, h) rows over host threads; each row's
 * arithmetic is the sequential loop above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { O_F32 = 0, O_F16 = 1, O_BF16 = 2, O_E4M3 = 3 };

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits */
double pkvo_decode_f16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (ex == 0) {
        v = ldexp((double)man, -24);                 /* zero / subnormal */
    } else if (ex == 31) {
        v = man ? NAN : INFINITY;
    } else {
        v = ldexp(1.0 + (double)man / 1024.0, ex - 15);
    }
    return sign ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits */
double pkvo_decode_bf16(uint16_t b) {
    int sign = (b >> 15) & 1;
    int ex = (b >> 7) & 0xff;
    int man = b & 0x7f;
    double v;
    if (ex == 0) {
        v = ldexp((double)man, -133);                /* 2^(1-127) * man/128 */
    } else if (ex == 255) {
        v = man ? NAN : INFINITY;
    } else {
        v = ldexp(1.0 + (double)man / 128.0, ex - 127);
    }
    return sign ? -v : v;
}

/* IEEE 754 binary32: 1 sign bit, 8 exponent bits (bias 127), 23 fraction bits */
double pkvo_decode_f32(uint32_t u) {
    int sign = (u >> 31) & 1;
    int ex = (u >> 23) & 0xff;
    uint32_t man = u & 0x7fffff;
    double v;
    if (ex == 0) {
        v = ldexp((double)man, -149);
    } else if (ex == 255) {
        v = man ? NAN : INFINITY;
    } else {
        v = ldexp(1.0 + (double)man / 8388608.0, ex - 127);
    }
    return sign ? -v : v;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign bit, 4 exponent bits (bias 7), 3
 * fraction bits; no infinities, S.1111.111 is NaN. */
double pkvo_decode_e4m3(uint8_t c) {
    int sign = (c >> 7) & 1;
    int ex = (c >> 3) & 0xf;
    int man = c & 0x7;
    double v;
    if (ex == 0) {
        v = ldexp((double)man, -9);                  /* 2^(1-7) * man/8 */
    } else if (ex == 15 && man == 7) {
        v = NAN;
    } else {
        v = ldexp(1.0 + (double)man / 8.0, ex - 7);
    }
    return sign ? -v : v;
}

static double load_elem(const void* base, int64_t idx, int dtype) {
    if (dtype == O_E4M3) {
        uint8_t c;
        memcpy(&c, (const char*)base + idx, 1);
        return pkvo_decode_e4m3(c);
    }
    if (dtype == O_F32) {
        uint32_t u;
        memcpy(&u, (const char*)base + 4 * idx, 4);
        return pkvo_decode_f32(u);
    }
    uint16_t h;
    memcpy(&h, (const char*)base + 2 * idx, 2);
    return dtype == O_F16 ? pkvo_decode_f16(h) : pkvo_decode_bf16(h);
}

void pkvo_decode_array(int dtype, const void* src, double* dst, int64_t n) {
    for (int64_t i = 0; i < n; ++i) dst[i] = load_elem(src, i, dtype);
}

/* One (b, h) row.  Returns 0, or -1 when a table entry the row needs is not a
 * valid pool index. */
static int decode_row(double* out_row, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int b, int h, int num_q_heads,
                      int num_kv_heads, int head_dim, int block_size,
                      int max_blocks_per_seq, int64_t num_blocks, double scale,
                      int window, int dtype, int kv_dtype, const float* k_scale,
                      const float* v_scale, int scale_per_block,
                      double* s /* scratch, >= L + head_dim */) {
    const int G = num_q_heads / num_kv_heads;
    const int g = h / G;
    const int L = context_lens[b];
    const int lo = (window > 0 && L > window) ? L - window : 0;
    const int D = head_dim;
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    if (L <= 0) return 0;

    /* the query row, decoded once */
    double* qrow = s + L;
    const int64_t q_off = ((int64_t)b * num_q_heads + h) * D;
    for (int d = 0; d < D; ++d) qrow[d] = load_elem(q, q_off + d, dtype);

    /* logits, gathered through the block table */
    for (int t = lo; t < L; ++t) {
        int32_t phys = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
        if (phys < 0 || phys >= num_blocks) return -1;
        int64_t k_off = (((int64_t)phys * num_kv_heads + g) * block_size + t % block_size) * D;
        /* quantised pages: value = code * scale of the KV head (or of the page) */
        const int64_t si = scale_per_block ? (int64_t)phys * num_kv_heads + g : g;
        const double ks = k_scale ? (double)k_scale[si] : 1.0;
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += qrow[d] * (load_elem(k_cache, k_off + d, kv_dtype) * ks);
        s[t] = scale * acc;
    }
    double m = s[lo];
    for (int t = lo + 1; t < L; ++t)
        if (s[t] > m) m = s[t];
    double denom = 0.0;
    for (int t = lo; t < L; ++t) {
        double w = exp(s[t] - m);
        denom += w;
        int32_t phys = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];
        int64_t v_off = (((int64_t)phys * num_kv_heads + g) * block_size + t % block_size) * D;
        const int64_t si = scale_per_block ? (int64_t)phys * num_kv_heads + g : g;
        const double vs = v_scale ? (double)v_scale[si] : 1.0;
        for (int d = 0; d < D; ++d)
            out_row[d] += w * (load_elem(v_cache, v_off + d, kv_dtype) * vs);
    }
    for (int d = 0; d < D; ++d) out_row[d] /= denom;
    return 0;
}

/*
 * out: float64 [num_rows, head_dim] when rows != NULL (rows = num_rows pairs
 *      (b, h)), else float64 [num_seqs, num_q_heads, head_dim].
 * Returns 0, -1 on a bad table entry, -2 on bad sizes.
 */
int pkvo_paged_decode(double* out, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int num_seqs, int num_q_heads,
                      int num_kv_heads, int head_dim, int block_size,
                      int max_blocks_per_seq, int64_t num_blocks, double scale,
                      int window, int dtype, int kv_dtype, const float* k_scale,
                      const float* v_scale, int scale_per_block, const int32_t* rows,
                      int64_t num_rows, int num_threads) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_q_heads % num_kv_heads != 0)
        return -2;
    int max_len = 0;
    for (int b = 0; b < num_seqs; ++b)
        if (context_lens[b] > max_len) max_len = context_lens[b];
    if (max_len > (int64_t)max_blocks_per_seq * block_size) return -2;
    const int64_t n = rows ? num_rows : (int64_t)num_seqs * num_q_heads;
    int err = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#endif
#pragma omp parallel reduction(| : err)
    {
        double* s = (double*)malloc(sizeof(double) * ((size_t)max_len + (size_t)head_dim));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n; ++i) {
            int b, h;
            if (rows) {
                b = rows[2 * i];
                h = rows[2 * i + 1];
            } else {
                b = (int)(i / num_q_heads);
                h = (int)(i % num_q_heads);
            }
            if (b < 0 || b >= num_seqs || h < 0 || h >= num_q_heads) {
                err |= 2;
                continue;
            }
            if (decode_row(out + i * head_dim, q, k_cache, v_cache, block_tables,
                           context_lens, b, h, num_q_heads, num_kv_heads, head_dim,
                           block_size, max_blocks_per_seq, num_blocks, scale, window, dtype,
                           kv_dtype, k_scale, v_scale, scale_per_block, s))
                err |= 1;
        }
        free(s);
    }
    return err ? -1 : 0;
}

int pkvo_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
