/*
 * oracle.c -- plain, slow, fp64 CPU oracle for exact scaled dot-product attention.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may load this library. The CUDA product path never calls it, and the two share no code.
 *
 * What it computes, and the passage each step follows:
 *   - O_i = sum_j softmax_j(q_i . k_j * scale) v_j, one query head at a time
 *     ("attention-transformers", Q "How does self-attention work in a transformer?";
 *      "Transformer Attention Mechanism Interview Deep Dive", "Scaled dot-product attention").
 *   - Masks enter as -inf on the logits before the softmax
 *     ("Transformer Attention Mechanism Interview Deep Dive", "Causal masking").
 *     Causal: key j visible to query i iff j <= i. Sliding window of width w (always together
 *     with causal): j in [i-w+1, i] ("attention-transformers", Q "What is sparse / sliding-window
 *     attention?").
 *   - Grouped-query attention: query head h reads K/V head floor(h / (Hq/Hkv))
 *     ("Transformer Complexity, Inference Optimization, GQA and FlashAttention", Part 3).
 *   - RoPE: pairs (2i, 2i+1) of q and k are rotated counter-clockwise by pos * base^(-2i/D)
 *     ("attention-transformers", Q "How does Rotary Position Embedding (RoPE) work?").
 *     The rotated values are rounded to bf16 with round-to-nearest-even, because the tensor
 *     cores that consume them take bf16 operands.
 *   - The saved row statistic is LSE_i = m_i + ln(l_i), natural log of the scaled scores
 *     ("Why is attention O(n^2), how does FlashAttention help, ...", "Deep dive: FlashAttention":
 *     the backward pass recomputes from the saved m and l).
 *   - Paged decode gathers a sequence's cached keys/values through its block table in logical
 *     order ("Self-Attention Complexity, FlashAttention, PagedAttention, and RoPE in Code",
 *     Part 3: fixed-size blocks and block tables) and computes the single query row at the
 *     sequence's last position over all seq_len cached tokens.
 *   - Position variants of the prefill: half-split RoPE pairs (i, i + D/2) instead of (2i, 2i+1)
 *     (the pages' "each 2D subspace" allows either pairing); Position Interpolation divides
 *     positions by a factor; NTK-aware scaling multiplies the base by factor^(D/(D-2)), which
 *     leaves the highest frequency unchanged and divides the lowest by the factor
 *     ("attention-transformers", Q "What are NTK-aware RoPE scaling and YaRN?"); ALiBi subtracts
 *     m_h (i - j) from the logit of query i and key j, with a per-head slope m_h
 *     ("attention-transformers", Q "How does ALiBi encode position?").
 *   - A decode step appends the new tokens first: their keys, rotated at their positions, and
 *     their values go into the slots the block table gives (same Part 3; the rotation of the
 *     RoPE question above), then each new token's query, rotated at its position, attends
 *     causally to the cache -- the last rows of causal attention over the whole sequence.
 *
 * The score row of every query is materialised in full (masked entries hold -inf), then
 * max, exp, sum, the weighted sum of V and the logsumexp are taken -- the plain definition,
 * with no tiling and no online rescaling.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_INDEX 2
#define ORACLE_ERR_NOMEM 3

/* bf16 bit pattern -> its exact value. A bf16 number is the top 16 bits of an IEEE binary32. */
static double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 (8 significant bits, exponent range of binary32), ties to
 * even, in one step (no intermediate rounding to binary32). Returns the bf16 bit pattern. */
uint16_t oracle_round_bf16(double x) {
    if (isnan(x)) return 0x7FC0u;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double ax = fabs(x);
    if (ax == 0.0) return sign;
    /* Largest finite bf16 is (2 - 2^-7) * 2^127; halfway to the next binade rounds to inf
     * because the largest mantissa is odd. */
    const double max_finite = ldexp(2.0 - ldexp(1.0, -7), 127);
    const double overflow_edge = ldexp(2.0 - ldexp(1.0, -8), 127);
    if (ax >= overflow_edge) return (uint16_t)(sign | 0x7F80u);
    int ex;
    frexp(ax, &ex);                 /* ax in [2^(ex-1), 2^ex) */
    int qexp = ex - 8;              /* quantum of an 8-significant-bit number in that binade */
    if (qexp < -133) qexp = -133;   /* subnormal quantum of binary32/bf16 */
    double r = nearbyint(ldexp(ax, -qexp));   /* default rounding mode: to nearest, ties even */
    double y = ldexp(r, qexp);
    if (y > max_finite) return (uint16_t)(sign | 0x7F80u);
    float yf = (float)y;            /* exact: y has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &yf, sizeof u);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFFu));
}

/* RoPE on one head vector x[0..D) at position pos, pairs (2i, 2i+1), angle pos * base^(-2i/D),
 * counter-clockwise: (x0 cos - x1 sin, x0 sin + x1 cos). Result rounded to bf16, returned as
 * exact doubles. base <= 0 means no rotation (values passed through exactly). */
static void rope_row(const uint16_t* x, int D, long pos, double base, double* out) {
    if (base <= 0.0) {
        for (int d = 0; d < D; ++d) out[d] = bf16_value(x[d]);
        return;
    }
    for (int i = 0; i < D / 2; ++i) {
        double theta = pow(base, -2.0 * (double)i / (double)D);
        double angle = (double)pos * theta;
        double c = cos(angle), s = sin(angle);
        double x0 = bf16_value(x[2 * i]), x1 = bf16_value(x[2 * i + 1]);
        out[2 * i] = bf16_value(oracle_round_bf16(x0 * c - x1 * s));
        out[2 * i + 1] = bf16_value(oracle_round_bf16(x0 * s + x1 * c));
    }
}

/* Exposed for the pins: rotate n_rows rows of length D; row r sits at position pos[r]. */
/* RoPE with a choice of pairing and scaling: pairs (2i, 2i+1) (half_split = 0) or (i, i + D/2)
 * (half_split = 1); the angle of pair i at position pos is (pos / pos_scale) * b^(-2i/D) with
 * b = base * ntk_factor^(D/(D-2)). Rotated values are rounded to bf16. */
static void rope_row_ex(const uint16_t* x, int D, long pos, double base, int half_split, double pos_scale,
                        double ntk_factor, double* out) {
    if (base <= 0.0) {
        for (int d = 0; d < D; ++d) out[d] = bf16_value(x[d]);
        return;
    }
    const double b = base * pow(ntk_factor, (double)D / (double)(D - 2));
    for (int i = 0; i < D / 2; ++i) {
        const double theta = pow(b, -2.0 * (double)i / (double)D);
        const double angle = ((double)pos / pos_scale) * theta;
        const double c = cos(angle), sn = sin(angle);
        const int a0 = half_split ? i : 2 * i;
        const int a1 = half_split ? i + D / 2 : 2 * i + 1;
        const double x0 = bf16_value(x[a0]), x1 = bf16_value(x[a1]);
        out[a0] = bf16_value(oracle_round_bf16(x0 * c - x1 * sn));
        out[a1] = bf16_value(oracle_round_bf16(x0 * sn + x1 * c));
    }
}

int oracle_rope_bf16_ex(const uint16_t* x, const int64_t* pos, int64_t n_rows, int D, double base, int half_split,
                        double pos_scale, double ntk_factor, uint16_t* out) {
    if (!x || !pos || !out || D <= 0 || (D % 2) != 0 || n_rows < 0 || !(pos_scale > 0.0) || !(ntk_factor > 0.0))
        return ORACLE_ERR_ARG;
    double* tmp = (double*)malloc(sizeof(double) * (size_t)D);
    if (!tmp) return ORACLE_ERR_NOMEM;
    for (int64_t r = 0; r < n_rows; ++r) {
        rope_row_ex(x + r * D, D, (long)pos[r], base, half_split, pos_scale, ntk_factor, tmp);
        for (int d = 0; d < D; ++d) out[r * D + d] = oracle_round_bf16(tmp[d]);
    }
    free(tmp);
    return ORACLE_OK;
}

int oracle_rope_bf16(const uint16_t* x, const int64_t* pos, int64_t n_rows, int D, double base,
                     uint16_t* out) {
    if (!x || !pos || !out || D <= 0 || (D % 2) != 0 || n_rows < 0) return ORACLE_ERR_ARG;
    double* tmp = (double*)malloc(sizeof(double) * (size_t)D);
    if (!tmp) return ORACLE_ERR_NOMEM;
    for (int64_t r = 0; r < n_rows; ++r) {
        rope_row(x + r * D, D, (long)pos[r], base, tmp);
        for (int d = 0; d < D; ++d) out[r * D + d] = oracle_round_bf16(tmp[d]);
    }
    free(tmp);
    return ORACLE_OK;
}

/* One query row against keys/values already converted to doubles.
 * q[D]; kk, vv: [N, D]; writes o[D] and *lse. Masked keys get score -inf. */
static void attend_row(const double* q, const double* kk, const double* vv, int N, int D,
                       long i, int causal, int window, double scale, double alibi_slope, double* s_row,
                       double* o, double* lse) {
    for (int j = 0; j < N; ++j) {
        int visible = 1;
        if (causal && j > i) visible = 0;
        if (window > 0 && (long)j < i - window + 1) visible = 0;
        if (!visible) {
            s_row[j] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += q[d] * kk[(size_t)j * D + d];
        s_row[j] = acc * scale;
        if (alibi_slope != 0.0) s_row[j] -= alibi_slope * (double)(i - j);
    }
    double m = -INFINITY;
    for (int j = 0; j < N; ++j)
        if (s_row[j] > m) m = s_row[j];
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (m == -INFINITY) { /* no visible key: defined as O = 0, LSE = -inf */
        *lse = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int j = 0; j < N; ++j) {
        double p = exp(s_row[j] - m); /* exp(-inf) == 0 for masked keys */
        s_row[j] = p;
        l += p;
    }
    for (int j = 0; j < N; ++j) {
        double p = s_row[j];
        if (p == 0.0) continue;
        const double* vj = vv + (size_t)j * D;
        for (int d = 0; d < D; ++d) o[d] += p * vj[d];
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    *lse = m + log(l);
}

/*
 * Prefill attention. q: bf16 [B, Hq, N, D]; k, v: bf16 [B, Hkv, N, D] (contiguous).
 * rows: NULL for every row, else n_rows flat row ids ((b*Hq + h)*N + i).
 * o: [n_rows, D] (or [B*Hq*N, D]); lse: [n_rows] (or [B*Hq*N]). Query i sits at position i.
 */
/*
 * Prefill attention with position variants: rope_half_split, rope_pos_scale, rope_ntk_factor as in
 * rope_row_ex (0, 1, 1: the plain interleaved RoPE), alibi_slopes: NULL or [Hq] slopes m_h.
 */
int oracle_attention_pos(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq, int Hkv, int N,
                         int D, int causal, int window, double rope_base, int rope_half_split, double rope_pos_scale,
                         double rope_ntk_factor, const double* alibi_slopes, double scale, const int64_t* rows,
                         int64_t n_rows, double* o, double* lse, int nthreads) {
    if (!q || !k || !v || !o || !lse) return ORACLE_ERR_ARG;
    if (!(rope_pos_scale > 0.0) || !(rope_ntk_factor > 0.0)) return ORACLE_ERR_ARG;
    const int plain_rope = !rope_half_split && rope_pos_scale == 1.0 && rope_ntk_factor == 1.0;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || D <= 0 || Hq % Hkv != 0) return ORACLE_ERR_ARG;
    if (window > 0 && !causal) return ORACLE_ERR_ARG;
    if (rope_base > 0.0 && (D % 2) != 0) return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq * N;
    if (rows == NULL) n_rows = total;
    for (int64_t r = 0; rows && r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return ORACLE_ERR_INDEX;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    double* kk = (double*)malloc(sizeof(double) * (size_t)N * D);
    double* vv = (double*)malloc(sizeof(double) * (size_t)N * D);
    if (!kk || !vv) {
        free(kk);
        free(vv);
        return ORACLE_ERR_NOMEM;
    }
    int status = ORACLE_OK;
    /* One K/V head at a time: rotate its keys once, then every requested query row that
     * reads it. */
    for (int b = 0; b < B && status == ORACLE_OK; ++b) {
        for (int g = 0; g < Hkv && status == ORACLE_OK; ++g) {
            int needed = 0;
            for (int64_t r = 0; r < n_rows && !needed; ++r) {
                int64_t id = rows ? rows[r] : r;
                int rb = (int)(id / ((int64_t)Hq * N));
                int rh = (int)((id / N) % Hq);
                if (rb == b && rh / G == g) needed = 1;
            }
            if (!needed) continue;
            const size_t kv_off = ((size_t)b * Hkv + g) * (size_t)N * D;
#pragma omp parallel for schedule(static)
            for (int j = 0; j < N; ++j) {
                if (plain_rope)
                    rope_row(k + kv_off + (size_t)j * D, D, j, rope_base, kk + (size_t)j * D);
                else
                    rope_row_ex(k + kv_off + (size_t)j * D, D, j, rope_base, rope_half_split, rope_pos_scale,
                                rope_ntk_factor, kk + (size_t)j * D);
                for (int d = 0; d < D; ++d) vv[(size_t)j * D + d] = bf16_value(v[kv_off + (size_t)j * D + d]);
            }
#pragma omp parallel
            {
                double* s_row = (double*)malloc(sizeof(double) * (size_t)N);
                double* qq = (double*)malloc(sizeof(double) * (size_t)D);
                if (!s_row || !qq) {
#pragma omp atomic write
                    status = ORACLE_ERR_NOMEM;
                } else {
#pragma omp for schedule(dynamic, 16)
                    for (int64_t r = 0; r < n_rows; ++r) {
                        int64_t id = rows ? rows[r] : r;
                        int rb = (int)(id / ((int64_t)Hq * N));
                        int rh = (int)((id / N) % Hq);
                        long i = (long)(id % N);
                        if (rb != b || rh / G != g) continue;
                        if (plain_rope)
                            rope_row(q + (size_t)id * D, D, i, rope_base, qq);
                        else
                            rope_row_ex(q + (size_t)id * D, D, i, rope_base, rope_half_split, rope_pos_scale,
                                        rope_ntk_factor, qq);
                        attend_row(qq, kk, vv, N, D, i, causal, window, scale,
                                   alibi_slopes ? alibi_slopes[rh] : 0.0, s_row, o + (size_t)r * D, lse + r);
                    }
                }
                free(s_row);
                free(qq);
            }
        }
    }
    free(kk);
    free(vv);
    return status;
}

int oracle_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                     int Hkv, int N, int D, int causal, int window, double rope_base,
                     double scale, const int64_t* rows, int64_t n_rows, double* o, double* lse,
                     int nthreads) {
    return oracle_attention_pos(q, k, v, B, Hq, Hkv, N, D, causal, window, rope_base, 0, 1.0, 1.0, NULL, scale,
                                rows, n_rows, o, lse, nthreads);
}

/*
 * Paged decode: one query token per sequence, attending to all seq_lens[s] cached tokens.
 * q: bf16 [S, Hq, D] (taken as already rotated); k_pages, v_pages: bf16
 * [num_pages, Hkv, page_size, D]; block_table: [S, max_blocks]; seq_lens: [S].
 * Token t of sequence s lives in page block_table[s][t / page_size], slot t % page_size.
 * o: [S, Hq, D]; lse: [S, Hq].
 */
int oracle_decode_paged(const uint16_t* q, const uint16_t* k_pages, const uint16_t* v_pages,
                        const int32_t* block_table, const int32_t* seq_lens, int S,
                        int max_blocks, int num_pages, int page_size, int Hq, int Hkv, int D,
                        double scale, double* o, double* lse, int nthreads) {
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o || !lse) return ORACLE_ERR_ARG;
    if (S <= 0 || max_blocks <= 0 || num_pages <= 0 || page_size <= 0 || Hq <= 0 || Hkv <= 0 ||
        D <= 0 || Hq % Hkv != 0)
        return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    for (int s = 0; s < S; ++s) {
        int len = seq_lens[s];
        if (len < 1 || (int64_t)len > (int64_t)max_blocks * page_size) return ORACLE_ERR_INDEX;
        int pages = (len + page_size - 1) / page_size;
        for (int p = 0; p < pages; ++p) {
            int32_t pg = block_table[(size_t)s * max_blocks + p];
            if (pg < 0 || pg >= num_pages) return ORACLE_ERR_INDEX;
        }
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int sg = 0; sg < S * Hkv; ++sg) {
        int s = sg / Hkv, g = sg % Hkv;
        int len = seq_lens[s];
        double* kk = (double*)malloc(sizeof(double) * (size_t)len * D);
        double* vv = (double*)malloc(sizeof(double) * (size_t)len * D);
        double* s_row = (double*)malloc(sizeof(double) * (size_t)len);
        double* qq = (double*)malloc(sizeof(double) * (size_t)D);
        if (!kk || !vv || !s_row || !qq) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        } else {
            for (int t = 0; t < len; ++t) {
                int32_t pg = block_table[(size_t)s * max_blocks + t / page_size];
                size_t base = (((size_t)pg * Hkv + g) * page_size + (size_t)(t % page_size)) * D;
                for (int d = 0; d < D; ++d) {
                    kk[(size_t)t * D + d] = bf16_value(k_pages[base + d]);
                    vv[(size_t)t * D + d] = bf16_value(v_pages[base + d]);
                }
            }
            for (int hh = 0; hh < G; ++hh) {
                int h = g * G + hh;
                for (int d = 0; d < D; ++d) qq[d] = bf16_value(q[((size_t)s * Hq + h) * D + d]);
                /* the query is the sequence's last token: position len-1, causal over the cache */
                attend_row(qq, kk, vv, len, D, (long)len - 1, 1, 0, scale, 0.0, s_row,
                           o + ((size_t)s * Hq + h) * D, lse + (size_t)s * Hq + h);
            }
        }
        free(kk);
        free(vv);
        free(s_row);
        free(qq);
    }
    return status;
}

/*
 * Decode step over a paged cache: append, then attend. q: bf16 [S, T, Hq, D] as given (rotated
 * here when rope_base > 0); k_new, v_new: bf16 [S, T, Hkv, D] or both NULL (the cache already
 * holds the new tokens). seq_lens count the T new tokens, which sit at positions len-T .. len-1.
 * k_pages, v_pages [num_pages, Hkv, page_size, D] are updated in place: the key of new token t
 * rotated at its position and rounded to bf16, the value as given. Sequences are appended in
 * order; slots written by two sequences are the caller's error. o: [S, T, Hq, D]; lse: [S, T, Hq].
 */
int oracle_decode_step(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pages,
                       uint16_t* v_pages, const int32_t* block_table, const int32_t* seq_lens, int S, int T,
                       int max_blocks, int num_pages, int page_size, int Hq, int Hkv, int D, double rope_base,
                       double scale, double* o, double* lse, int nthreads) {
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o || !lse) return ORACLE_ERR_ARG;
    if ((k_new == NULL) != (v_new == NULL)) return ORACLE_ERR_ARG;
    if (S <= 0 || T <= 0 || max_blocks <= 0 || num_pages <= 0 || page_size <= 0 || Hq <= 0 || Hkv <= 0 ||
        D <= 0 || (D % 2) != 0 || Hq % Hkv != 0)
        return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    for (int s = 0; s < S; ++s) {
        int len = seq_lens[s];
        if (len < T || (int64_t)len > (int64_t)max_blocks * page_size) return ORACLE_ERR_INDEX;
        int pages = (len + page_size - 1) / page_size;
        for (int p = 0; p < pages; ++p) {
            int32_t pg = block_table[(size_t)s * max_blocks + p];
            if (pg < 0 || pg >= num_pages) return ORACLE_ERR_INDEX;
        }
    }
    double* tmp = (double*)malloc(sizeof(double) * (size_t)D);
    if (!tmp) return ORACLE_ERR_NOMEM;
    if (k_new != NULL) {
        for (int s = 0; s < S; ++s) {
            for (int t = 0; t < T; ++t) {
                long pos = (long)seq_lens[s] - T + t;
                int32_t pg = block_table[(size_t)s * max_blocks + pos / page_size];
                for (int g = 0; g < Hkv; ++g) {
                    size_t src = (((size_t)s * T + t) * Hkv + g) * D;
                    size_t dst = (((size_t)pg * Hkv + g) * page_size + (size_t)(pos % page_size)) * D;
                    rope_row(k_new + src, D, pos, rope_base, tmp);
                    for (int d = 0; d < D; ++d) {
                        k_pages[dst + d] = oracle_round_bf16(tmp[d]);
                        v_pages[dst + d] = v_new[src + d];
                    }
                }
            }
        }
    }
    free(tmp);
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int sg = 0; sg < S * Hkv; ++sg) {
        int s = sg / Hkv, g = sg % Hkv;
        int len = seq_lens[s];
        double* kk = (double*)malloc(sizeof(double) * (size_t)len * D);
        double* vv = (double*)malloc(sizeof(double) * (size_t)len * D);
        double* s_row = (double*)malloc(sizeof(double) * (size_t)len);
        double* qq = (double*)malloc(sizeof(double) * (size_t)D);
        if (!kk || !vv || !s_row || !qq) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        } else {
            for (int t = 0; t < len; ++t) {
                int32_t pg = block_table[(size_t)s * max_blocks + t / page_size];
                size_t base = (((size_t)pg * Hkv + g) * page_size + (size_t)(t % page_size)) * D;
                for (int d = 0; d < D; ++d) {
                    kk[(size_t)t * D + d] = bf16_value(k_pages[base + d]);
                    vv[(size_t)t * D + d] = bf16_value(v_pages[base + d]);
                }
            }
            for (int t = 0; t < T; ++t) {
                long pos = (long)len - T + t;
                for (int hh = 0; hh < G; ++hh) {
                    int h = g * G + hh;
                    size_t row = ((size_t)s * T + t) * Hq + h;
                    rope_row(q + row * D, D, pos, rope_base, qq);
                    attend_row(qq, kk, vv, len, D, pos, 1, 0, scale, 0.0, s_row, o + row * D, lse + row);
                }
            }
        }
        free(kk);
        free(vv);
        free(s_row);
        free(qq);
    }
    return status;
}

/*
 * FP8 e4m3 (the "fn" encoding: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no
 * infinities, S.1111.111 is NaN) to its exact value: exponent field 0 gives the subnormals
 * m * 2^-9, otherwise (1 + m/8) * 2^(e-7). FP8 attention of the pages ("Why is attention O(n^2),
 * ...": newer hardware, FP8) is exact attention on these values times their per-tensor scales.
 */
void oracle_e4m3_to_f64(const uint8_t* x, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) {
        const int sign = x[i] >> 7, e = (x[i] >> 3) & 15, m = x[i] & 7;
        double v;
        if (e == 15 && m == 7)
            v = NAN;
        else if (e == 0)
            v = ldexp((double)m, -9);
        else
            v = ldexp(1.0 + (double)m / 8.0, e - 7);
        out[i] = sign ? -v : v;
    }
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Vector form of oracle_round_bf16, for the pins. */
void oracle_round_bf16_array(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_bf16(x[i]);
}

/* ============================================================================ backward
 * Gradients of the scalar L = sum_{b,h,i,d} O[b,h,i,d] * dO[b,h,i,d] with respect to q, k, v,
 * for the same attention as oracle_attention ("Self-Attention Complexity, FlashAttention,
 * PagedAttention, and RoPE in Code", Part 2: the backward pass; "Why is attention O(n^2), how does
 * FlashAttention help, ...", "Deep dive: FlashAttention": it recomputes the scores from the saved
 * statistics instead of storing P). Per query row i, with P_i the softmax row over the visible
 * keys (written out plainly by the chain rule):
 *   dV_j += P_ij dO_i                         dP_ij = dO_i . v_j
 *   dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik)   dq_i  = scale * sum_j dS_ij k_j
 *   dk_j += scale * dS_ij q_i
 * where q, k are the rotated vectors. The rotation is linear, so the gradient of the unrotated
 * vector is the rotated-back gradient: rotate by -angle. Rounding the rotated values to bf16 is
 * treated as the identity in the gradient.
 */

/* Rotate a fp64 row by +angle (forward) or -angle (inverse, the transpose); optional bf16 rounding. */
static void rope_row_f64(const double* x, int D, long pos, double base, int inverse, int round_to_bf16,
                         double* out) {
    if (base <= 0.0) {
        for (int d = 0; d < D; ++d) out[d] = x[d];
        return;
    }
    for (int i = 0; i < D / 2; ++i) {
        double theta = pow(base, -2.0 * (double)i / (double)D);
        double angle = (double)pos * theta;
        double c = cos(angle), s = inverse ? -sin(angle) : sin(angle);
        double y0 = x[2 * i] * c - x[2 * i + 1] * s;
        double y1 = x[2 * i] * s + x[2 * i + 1] * c;
        if (round_to_bf16) {
            y0 = bf16_value(oracle_round_bf16(y0));
            y1 = bf16_value(oracle_round_bf16(y1));
        }
        out[2 * i] = y0;
        out[2 * i + 1] = y1;
    }
}

/* Forward on fp64 inputs (every row), for the finite-difference and autograd pins. */
int oracle_attention_f64(const double* q, const double* k, const double* v, int B, int Hq, int Hkv, int N,
                         int D, int causal, int window, double rope_base, double scale, int round_rotated,
                         double* o, double* lse) {
    if (!q || !k || !v || !o || !lse) return ORACLE_ERR_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || D <= 0 || Hq % Hkv != 0) return ORACLE_ERR_ARG;
    if (window > 0 && !causal) return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    double* kk = (double*)malloc(sizeof(double) * (size_t)N * D);
    double* s_row = (double*)malloc(sizeof(double) * (size_t)N);
    double* qq = (double*)malloc(sizeof(double) * (size_t)D);
    if (!kk || !s_row || !qq) {
        free(kk); free(s_row); free(qq);
        return ORACLE_ERR_NOMEM;
    }
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g) {
            const size_t kv_off = ((size_t)b * Hkv + g) * (size_t)N * D;
            for (int j = 0; j < N; ++j)
                rope_row_f64(k + kv_off + (size_t)j * D, D, j, rope_base, 0, round_rotated, kk + (size_t)j * D);
            for (int hh = 0; hh < G; ++hh) {
                const int h = g * G + hh;
                for (int i = 0; i < N; ++i) {
                    const size_t row = ((size_t)b * Hq + h) * N + i;
                    rope_row_f64(q + row * D, D, i, rope_base, 0, round_rotated, qq);
                    attend_row(qq, kk, v + kv_off, N, D, i, causal, window, scale, 0.0, s_row, o + row * D, lse + row);
                }
            }
        }
    free(kk); free(s_row); free(qq);
    return ORACLE_OK;
}

/* Backward on fp64 inputs. dq: [B,Hq,N,D]; dk, dv: [B,Hkv,N,D]. */
int oracle_attention_bwd_f64(const double* q, const double* k, const double* v, const double* dout, int B,
                             int Hq, int Hkv, int N, int D, int causal, int window, double rope_base,
                             double scale, int round_rotated, double* dq, double* dk, double* dv,
                             int nthreads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return ORACLE_ERR_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || D <= 0 || Hq % Hkv != 0) return ORACLE_ERR_ARG;
    if (window > 0 && !causal) return ORACLE_ERR_ARG;
    if (rope_base > 0.0 && (D % 2) != 0) return ORACLE_ERR_ARG;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const int G = Hq / Hkv;
    const size_t ND = (size_t)N * D;
    double* kk = (double*)malloc(sizeof(double) * ND);
    double* dk_rot = (double*)malloc(sizeof(double) * ND);
    if (!kk || !dk_rot) {
        free(kk); free(dk_rot);
        return ORACLE_ERR_NOMEM;
    }
    int status = ORACLE_OK;
    for (int b = 0; b < B && status == ORACLE_OK; ++b)
        for (int g = 0; g < Hkv && status == ORACLE_OK; ++g) {
            const size_t kv_off = ((size_t)b * Hkv + g) * ND;
            const double* vv = v + kv_off;
            for (int j = 0; j < N; ++j)
                rope_row_f64(k + kv_off + (size_t)j * D, D, j, rope_base, 0, round_rotated, kk + (size_t)j * D);
            for (size_t e = 0; e < ND; ++e) dk_rot[e] = 0.0, dv[kv_off + e] = 0.0;
            /* per-thread accumulators, summed in thread order afterwards (a fixed static schedule
             * makes the result reproducible for a given thread count) */
#ifdef _OPENMP
            const int n_thr = omp_get_max_threads();
#else
            const int n_thr = 1;
#endif
            double* acc_dk = (double*)calloc((size_t)n_thr * ND, sizeof(double));
            double* acc_dv = (double*)calloc((size_t)n_thr * ND, sizeof(double));
            if (!acc_dk || !acc_dv) {
                free(acc_dk); free(acc_dv);
                status = ORACLE_ERR_NOMEM;
                break;
            }
#pragma omp parallel num_threads(n_thr)
            {
#ifdef _OPENMP
                const int tid = omp_get_thread_num();
#else
                const int tid = 0;
#endif
                double* s_row = (double*)malloc(sizeof(double) * (size_t)N);
                double* dp = (double*)malloc(sizeof(double) * (size_t)N);
                double* qq = (double*)malloc(sizeof(double) * (size_t)D);
                double* dqr = (double*)malloc(sizeof(double) * (size_t)D);
                double* o_row = (double*)malloc(sizeof(double) * (size_t)D);
                double* my_dk = acc_dk + (size_t)tid * ND;
                double* my_dv = acc_dv + (size_t)tid * ND;
                if (!s_row || !dp || !qq || !dqr || !o_row) {
#pragma omp atomic write
                    status = ORACLE_ERR_NOMEM;
                } else {
#pragma omp for schedule(static)
                    for (int r = 0; r < G * N; ++r) {
                        const int h = g * G + r / N, i = r % N;
                        const size_t row = ((size_t)b * Hq + h) * N + i;
                        const double* dO = dout + row * D;
                        double lse_i;
                        rope_row_f64(q + row * D, D, i, rope_base, 0, round_rotated, qq);
                        attend_row(qq, kk, vv, N, D, i, causal, window, scale, 0.0, s_row, o_row, &lse_i);
                        /* attend_row leaves exp(s_ij - m_i) in s_row; P_ij is that over its row sum */
                        double lsum = 0.0;
                        for (int j = 0; j < N; ++j) lsum += s_row[j];
                        for (int j = 0; j < N; ++j) s_row[j] /= lsum;
                        double dsum = 0.0;
                        for (int j = 0; j < N; ++j) {
                            dp[j] = 0.0;
                            if (s_row[j] == 0.0) continue;
                            for (int d = 0; d < D; ++d) dp[j] += dO[d] * vv[(size_t)j * D + d];
                            dsum += s_row[j] * dp[j];
                        }
                        for (int d = 0; d < D; ++d) dqr[d] = 0.0;
                        for (int j = 0; j < N; ++j) {
                            const double p = s_row[j];
                            if (p == 0.0) continue;
                            const double ds = p * (dp[j] - dsum);
                            for (int d = 0; d < D; ++d) {
                                dqr[d] += scale * ds * kk[(size_t)j * D + d];
                                my_dk[(size_t)j * D + d] += scale * ds * qq[d];
                                my_dv[(size_t)j * D + d] += p * dO[d];
                            }
                        }
                        rope_row_f64(dqr, D, i, rope_base, 1, 0, dq + row * D);
                    }
                }
                free(s_row); free(dp); free(qq); free(dqr); free(o_row);
            }
            for (int t = 0; t < n_thr; ++t)
                for (size_t e = 0; e < ND; ++e) {
                    dk_rot[e] += acc_dk[(size_t)t * ND + e];
                    dv[kv_off + e] += acc_dv[(size_t)t * ND + e];
                }
            free(acc_dk); free(acc_dv);
            for (int j = 0; j < N; ++j)
                rope_row_f64(dk_rot + (size_t)j * D, D, j, rope_base, 1, 0, dk + kv_off + (size_t)j * D);
        }
    free(kk); free(dk_rot);
    return status;
}

/* Backward on bf16 inputs (the GPU's bits), rotated values rounded to bf16 as in the forward. */
/*
 * dq of selected query rows only (bf16 inputs, rotated values rounded to bf16 as in the forward):
 * the same steps as oracle_attention_bwd_f64 for one row -- its full score row, P, dP_ij = dO_i . v_j,
 * D_i = sum_j P_ij dP_ij, dS = P (dP - D_i), dq_i = scale sum_j dS_ij k_j rotated back -- which
 * needs only that row, so rows of large problems can be checked one by one.
 * rows: flat ids ((b*Hq + h)*N + i); dq: [n_rows, D].
 */
int oracle_attention_bwd_dq_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                                 int B, int Hq, int Hkv, int N, int D, int causal, int window, double rope_base,
                                 double scale, const int64_t* rows, int64_t n_rows, double* dq, int nthreads) {
    if (!q || !k || !v || !dout || !rows || !dq) return ORACLE_ERR_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || D <= 0 || Hq % Hkv != 0) return ORACLE_ERR_ARG;
    if (window > 0 && !causal) return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq * N;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return ORACLE_ERR_INDEX;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const size_t ND = (size_t)N * D;
    double* kk = (double*)malloc(sizeof(double) * ND);
    double* vv = (double*)malloc(sizeof(double) * ND);
    if (!kk || !vv) {
        free(kk); free(vv);
        return ORACLE_ERR_NOMEM;
    }
    int status = ORACLE_OK;
    for (int b = 0; b < B && status == ORACLE_OK; ++b)
        for (int g = 0; g < Hkv && status == ORACLE_OK; ++g) {
            int needed = 0;
            for (int64_t r = 0; r < n_rows && !needed; ++r) {
                const int rb = (int)(rows[r] / ((int64_t)Hq * N)), rh = (int)((rows[r] / N) % Hq);
                if (rb == b && rh / G == g) needed = 1;
            }
            if (!needed) continue;
            const size_t kv_off = ((size_t)b * Hkv + g) * ND;
#pragma omp parallel for schedule(static)
            for (int j = 0; j < N; ++j) {
                double tmp[512];
                for (int d = 0; d < D; ++d) tmp[d] = bf16_value(k[kv_off + (size_t)j * D + d]);
                rope_row_f64(tmp, D, j, rope_base, 0, 1, kk + (size_t)j * D);
                for (int d = 0; d < D; ++d) vv[(size_t)j * D + d] = bf16_value(v[kv_off + (size_t)j * D + d]);
            }
#pragma omp parallel
            {
                double* s_row = (double*)malloc(sizeof(double) * (size_t)N);
                double* dp = (double*)malloc(sizeof(double) * (size_t)N);
                double* buf = (double*)malloc(sizeof(double) * (size_t)D * 4);
                if (!s_row || !dp || !buf) {
#pragma omp atomic write
                    status = ORACLE_ERR_NOMEM;
                } else {
                    double *qq = buf, *dqr = buf + D, *o_row = buf + 2 * D, *dO = buf + 3 * D;
#pragma omp for schedule(dynamic, 1)
                    for (int64_t r = 0; r < n_rows; ++r) {
                        const int64_t id = rows[r];
                        const int rb = (int)(id / ((int64_t)Hq * N)), rh = (int)((id / N) % Hq);
                        const long i = (long)(id % N);
                        if (rb != b || rh / G != g) continue;
                        double lse_i;
                        for (int d = 0; d < D; ++d) {
                            dqr[d] = bf16_value(q[(size_t)id * D + d]);
                            dO[d] = bf16_value(dout[(size_t)id * D + d]);
                        }
                        rope_row_f64(dqr, D, i, rope_base, 0, 1, qq);
                        attend_row(qq, kk, vv, N, D, i, causal, window, scale, 0.0, s_row, o_row, &lse_i);
                        double lsum = 0.0;
                        for (int j = 0; j < N; ++j) lsum += s_row[j];
                        for (int j = 0; j < N; ++j) s_row[j] /= lsum;
                        double dsum = 0.0;
                        for (int j = 0; j < N; ++j) {
                            dp[j] = 0.0;
                            if (s_row[j] == 0.0) continue;
                            for (int d = 0; d < D; ++d) dp[j] += dO[d] * vv[(size_t)j * D + d];
                            dsum += s_row[j] * dp[j];
                        }
                        for (int d = 0; d < D; ++d) dqr[d] = 0.0;
                        for (int j = 0; j < N; ++j) {
                            const double pj = s_row[j];
                            if (pj == 0.0) continue;
                            const double ds = pj * (dp[j] - dsum);
                            for (int d = 0; d < D; ++d) dqr[d] += scale * ds * kk[(size_t)j * D + d];
                        }
                        rope_row_f64(dqr, D, i, rope_base, 1, 0, dq + (size_t)r * D);
                    }
                }
                free(s_row); free(dp); free(buf);
            }
        }
    free(kk); free(vv);
    return status;
}

int oracle_attention_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout, int B,
                         int Hq, int Hkv, int N, int D, int causal, int window, double rope_base, double scale,
                         double* dq, double* dk, double* dv, int nthreads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return ORACLE_ERR_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || D <= 0 || Hq % Hkv != 0) return ORACLE_ERR_ARG;
    const size_t nq = (size_t)B * Hq * N * D, nk = (size_t)B * Hkv * N * D;
    double* qd = (double*)malloc(sizeof(double) * nq);
    double* dod = (double*)malloc(sizeof(double) * nq);
    double* kd = (double*)malloc(sizeof(double) * nk);
    double* vd = (double*)malloc(sizeof(double) * nk);
    int st = ORACLE_ERR_NOMEM;
    if (qd && dod && kd && vd) {
        for (size_t e = 0; e < nq; ++e) qd[e] = bf16_value(q[e]), dod[e] = bf16_value(dout[e]);
        for (size_t e = 0; e < nk; ++e) kd[e] = bf16_value(k[e]), vd[e] = bf16_value(v[e]);
        st = oracle_attention_bwd_f64(qd, kd, vd, dod, B, Hq, Hkv, N, D, causal, window, rope_base, scale, 1,
                                      dq, dk, dv, nthreads);
    }
    free(qd); free(dod); free(kd); free(vd);
    return st;
}
