/*
 * attn_oracle.c -- plain fp64 eager attention on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is
 * checked against.  Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load it.  It shares no code, header or constant with
 * the CUDA library, and the CUDA library never calls it.
 *
 * What it computes (the plain definition; every step is written out):
 *
 *   For each batch b, query head h, and query row i, with the KV head
 *   g = h / G, G = Hq / Hkv (a run of G consecutive query heads shares one KV
 *   head -- the grouped-query definition on the NVIDIA attention-optimisation
 *   page, "Parameter one: group size"):
 *
 *     s_ij  = scale * sum_d q[b,h,i,d] * k[b,g,j,d]      for visible j
 *     s_ij  = -inf                                        for masked j
 *     m_i   = max_j s_ij
 *     l_i   = sum_j exp(s_ij - m_i)
 *     O_i   = sum_j exp(s_ij - m_i) * v[b,g,j,:] / l_i
 *     LSE_i = m_i + ln(l_i)
 *
 *   Visible keys (the causal-alignment section of the SDPA / FlashAttention
 *   selection guide, with its numpy demonstration):
 *     prefill, causal     : j <= i + (Lk - Lq)   (bottom-right alignment)
 *     prefill, not causal : every j < Lk
 *     decode              : every j < seqlens[b] (one new query row sees the
 *                           whole cache, so no mask is needed)
 *
 *   A row with no visible key has O = 0 and LSE = -inf (the pages are silent
 *   on this case; this is the convention the library documents).
 *
 *   Like the eager implementation described on the same guide ("eager
 *   attention memory"), each query row first fills its whole row of the score
 *   table, masked cells included, then takes the softmax of that row in full
 *   precision and mixes V with it.  Nothing is tiled, fused or reordered.
 *
 * Inputs may be fp64, fp32 or bf16 bit patterns (uint16); every element is
 * widened to fp64 before use.  bf16 -> fp32 is exact by definition (a bf16
 * number is the upper half of an IEEE binary32 word), and fp32 -> fp64 is
 * exact.  All arithmetic is fp64.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC attn_oracle.c -o libattn_oracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F64 = 0, ORACLE_F32 = 1, ORACLE_BF16 = 2 };

/* Read element i of an array of the given element type, widened to fp64. */
static double load_elem(const void* base, int dtype, size_t i) {
    if (dtype == ORACLE_F64) return ((const double*)base)[i];
    if (dtype == ORACLE_F32) return (double)((const float*)base)[i];
    /* bf16: the 16 stored bits are the high half of a binary32 word. */
    uint32_t word = ((uint32_t)((const uint16_t*)base)[i]) << 16;
    float f;
    memcpy(&f, &word, sizeof f);
    return (double)f;
}

/*
 * One query row against one KV head.
 *   q_off       : element offset of the query row (D elements)
 *   kv_off      : element offset of key/value row 0 of this KV head
 *   n_keys      : number of key rows that exist (length of the score row)
 *   last_vis    : keys 0..last_vis are visible, the rest are masked
 *   score       : scratch, n_keys doubles (the row of the score table)
 *   out_row     : D doubles
 *   lse_out     : one double
 *   probs_row   : n_keys doubles or NULL (the softmax weights; 0 when masked)
 */
static void eager_row(const void* q, const void* k, const void* v, int dtype,
                      size_t q_off, size_t kv_off, int n_keys, int D,
                      double scale, long last_vis, double* score,
                      double* out_row, double* lse_out, double* probs_row) {
    /* the full row of the score table, masked cells = -inf */
    for (int j = 0; j < n_keys; ++j) {
        if ((long)j > last_vis) {
            score[j] = -INFINITY;
            continue;
        }
        double dot = 0.0;
        size_t k_off = kv_off + (size_t)j * (size_t)D;
        for (int d = 0; d < D; ++d)
            dot += load_elem(q, dtype, q_off + d) * load_elem(k, dtype, k_off + d);
        score[j] = scale * dot;
    }
    /* row max over the table row */
    double m = -INFINITY;
    for (int j = 0; j < n_keys; ++j)
        if (score[j] > m) m = score[j];
    if (m == -INFINITY) { /* no visible key */
        for (int d = 0; d < D; ++d) out_row[d] = 0.0;
        *lse_out = -INFINITY;
        if (probs_row)
            for (int j = 0; j < n_keys; ++j) probs_row[j] = 0.0;
        return;
    }
    /* exponentials and their sum */
    double l = 0.0;
    for (int j = 0; j < n_keys; ++j) {
        score[j] = (score[j] == -INFINITY) ? 0.0 : exp(score[j] - m);
        l += score[j];
    }
    /* O = sum_j exp(s_j - m) v_j / l */
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    for (int j = 0; j < n_keys; ++j) {
        if (score[j] == 0.0) continue;
        size_t v_off = kv_off + (size_t)j * (size_t)D;
        for (int d = 0; d < D; ++d)
            out_row[d] += score[j] * load_elem(v, dtype, v_off + d);
    }
    for (int d = 0; d < D; ++d) out_row[d] /= l;
    *lse_out = m + log(l);
    if (probs_row)
        for (int j = 0; j < n_keys; ++j) probs_row[j] = score[j] / l;
}

static int set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Number of threads the oracle will use for a given request (0 = default). */
int oracle_num_threads(int nthreads) { return set_threads(nthreads); }

/*
 * Prefill (and chunked prefill): Q [B,Hq,Lq,D], K/V [B,Hkv,Lk,D].
 * rows / n_rows select which query positions to evaluate (rows == NULL means
 * all Lq of them, in order).  Outputs are laid out over the selected rows:
 *   out   [B,Hq,n_rows,D]  (fp64)
 *   lse   [B,Hq,n_rows]    (fp64)
 *   probs [B,Hq,n_rows,Lk] (fp64) or NULL
 * Returns 0 on success, -1 on bad arguments, -2 if scratch allocation fails.
 */
int oracle_attn_prefill(const void* q, const void* k, const void* v, int dtype,
                        int B, int Hq, int Hkv, int Lq, int Lk, int D,
                        double scale, int is_causal,
                        const int32_t* rows, int n_rows,
                        double* out, double* lse, double* probs, int nthreads) {
    if (!q || !k || !v || !out || !lse) return -1;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Lq < 0 || Lk < 0 || D <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (dtype < ORACLE_F64 || dtype > ORACLE_BF16) return -1;
    if (!rows) n_rows = Lq;
    if (n_rows < 0) return -1;
    for (int r = 0; rows && r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= Lq) return -1;
    const int G = Hq / Hkv;
    const long total = (long)B * Hq * n_rows;
    int failed = 0;
    set_threads(nthreads);
#pragma omp parallel
    {
        double* score = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        if (!score) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (long t = 0; t < total; ++t) {
            if (!score) continue;
            int r = (int)(t % n_rows);
            int h = (int)((t / n_rows) % Hq);
            int b = (int)(t / ((long)n_rows * Hq));
            int i = rows ? rows[r] : r;
            int g = h / G;
            size_t q_off = (((size_t)b * Hq + h) * (size_t)Lq + (size_t)i) * (size_t)D;
            size_t kv_off = ((size_t)b * Hkv + g) * (size_t)Lk * (size_t)D;
            long last_vis = is_causal ? (long)i + (long)Lk - (long)Lq : (long)Lk - 1;
            double* probs_row = probs ? probs + (size_t)t * (size_t)Lk : NULL;
            eager_row(q, k, v, dtype, q_off, kv_off, Lk, D, scale, last_vis, score,
                      out + (size_t)t * (size_t)D, lse + t, probs_row);
        }
        free(score);
    }
    return failed ? -2 : 0;
}

/*
 * Decode: one new query row per sequence against a KV cache.
 *   q       [B,Hq,D]
 *   k_cache [B,Hkv,Lmax,D], v_cache [B,Hkv,Lmax,D]
 *   seqlens [B]  -- cache rows 0..seqlens[b]-1 are valid; the rest are never
 *                   read (they may hold anything, NaN included)
 *   out [B,Hq,D], lse [B,Hq]   (fp64)
 */
int oracle_attn_decode(const void* q, const void* k_cache, const void* v_cache, int dtype,
                       const int32_t* seqlens, int B, int Hq, int Hkv, int Lmax, int D,
                       double scale, double* out, double* lse, int nthreads) {
    if (!q || !k_cache || !v_cache || !seqlens || !out || !lse) return -1;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Lmax < 0 || D <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (dtype < ORACLE_F64 || dtype > ORACLE_BF16) return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Lmax) return -1;
    const int G = Hq / Hkv;
    const long total = (long)B * Hq;
    int failed = 0;
    set_threads(nthreads);
#pragma omp parallel
    {
        double* score = (double*)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        if (!score) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long t = 0; t < total; ++t) {
            if (!score) continue;
            int h = (int)(t % Hq);
            int b = (int)(t / Hq);
            int g = h / G;
            size_t q_off = ((size_t)b * Hq + h) * (size_t)D;
            size_t kv_off = ((size_t)b * Hkv + g) * (size_t)Lmax * (size_t)D;
            /* only the seqlens[b] valid rows form the score row */
            eager_row(q, k_cache, v_cache, dtype, q_off, kv_off, seqlens[b], D, scale,
                      (long)seqlens[b] - 1, score, out + (size_t)t * (size_t)D, lse + t, NULL);
        }
        free(score);
    }
    return failed ? -2 : 0;
}

/*
 * 8-bit KV caches (the library's attn_decode_kv8).  The pages only name the
 * q8_0 cache type (the llama.cpp server configuration on the "Attention
 * Slack" page) and define no format; the two formats here are written from
 * their published definitions:
 *
 *   FP8 E4M3 (OCP 8-bit floating point, E4M3): bit 7 sign, bits 6-3 exponent
 *   e with bias 7, bits 2-0 mantissa m.
 *     e = 0          : (-1)^s * m * 2^-9            (subnormal, and +-0)
 *     e = 15, m = 7  : NaN                          (no infinities)
 *     otherwise      : (-1)^s * (1 + m / 8) * 2^(e - 7)
 *   Dequantised element [b,g,r,d] = k_scale[g] * value(code) (one fp32 scale
 *   per KV head).
 *
 *   q8_0: int8 codes (two's complement) with one scale per 32 consecutive
 *   values of a row, the scale an IEEE binary16 number: bit 15 sign, bits
 *   14-10 exponent e with bias 15, bits 9-0 mantissa m.
 *     e = 0          : (-1)^s * m * 2^-24
 *     e = 31         : +-inf (m = 0) or NaN
 *     otherwise      : (-1)^s * (1 + m / 1024) * 2^(e - 15)
 *   Dequantised element [b,g,r,d] = scale[b,g,r,d / 32] * code.
 */
double oracle_e4m3_value(uint8_t code) {
    const int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

double oracle_f16_value(uint16_t bits) {
    const int s = bits >> 15, e = (bits >> 10) & 31, m = bits & 1023;
    double v;
    if (e == 31) return m ? NAN : (s ? -INFINITY : INFINITY);
    if (e == 0)
        v = ldexp((double)m, -24);
    else
        v = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -v : v;
}

enum { ORACLE_KV_E4M3 = 1, ORACLE_KV_Q8_0 = 2 };

/*
 * codes [B,Hkv,L,D] (uint8) -> out [B,Hkv,L,D] fp64.
 *   fmt E4M3: scales = float [Hkv]
 *   fmt Q8_0: scales = binary16 bit patterns [B,Hkv,L,D/32]  (D % 32 == 0)
 */
int oracle_dequant_kv8(const uint8_t* codes, int fmt, const void* scales, int B, int Hkv, int L, int D,
                       double* out) {
    if (!codes || !scales || !out || B < 0 || Hkv <= 0 || L < 0 || D <= 0) return -1;
    if (fmt != ORACLE_KV_E4M3 && fmt != ORACLE_KV_Q8_0) return -1;
    if (fmt == ORACLE_KV_Q8_0 && D % 32 != 0) return -1;
    for (long bg = 0; bg < (long)B * Hkv; ++bg) {
        const int g = (int)(bg % Hkv);
        for (long r = 0; r < L; ++r) {
            const size_t row = ((size_t)bg * (size_t)L + (size_t)r) * (size_t)D;
            for (int d = 0; d < D; ++d) {
                if (fmt == ORACLE_KV_E4M3) {
                    out[row + d] = (double)((const float*)scales)[g] * oracle_e4m3_value(codes[row + d]);
                } else {
                    const size_t srow = ((size_t)bg * (size_t)L + (size_t)r) * (size_t)(D / 32);
                    const double sc = oracle_f16_value(((const uint16_t*)scales)[srow + d / 32]);
                    out[row + d] = sc * (double)(int8_t)codes[row + d];
                }
            }
        }
    }
    return 0;
}

/* n elements of the given type (fp64, fp32 or bf16 bits) widened to fp64. */
int oracle_widen(const void* x, int dtype, size_t n, double* out) {
    if ((!x && n) || (!out && n) || dtype < ORACLE_F64 || dtype > ORACLE_BF16) return -1;
    for (size_t i = 0; i < n; ++i) out[i] = load_elem(x, dtype, i);
    return 0;
}
