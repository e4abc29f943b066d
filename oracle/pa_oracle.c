/*
 * Paged KV-cache append and paged decode attention: fp64 CPU ORACLE.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
 * leg may.  It shares no code, header, helper or constant with the CUDA
 * library: it is a plain, slow restatement of what the pages define.
 *
 * What the pages define, and where:
 *  - "vLLM — PagedAttention으로 LLM 추론 성능을 2~4배 끌어올린 서빙 엔진" (dev.to),
 *    section "PagedAttention — OS 가상 메모리에서 영감": the KV cache is cut into
 *    fixed-size blocks (pages); physical and logical blocks are kept apart so
 *    that non-contiguous physical memory is used as if it were contiguous.
 *    Here: logical token j of a sequence lives in physical block
 *    table[j / Bs] at offset j % Bs (oracle_slot, gather_sequence).
 *  - same page, section "KV Cache가 왜 병목인가": each generated token's
 *    self-attention reads the Key and Value of every previous token, which is
 *    why they are cached (oracle_paged_decode reads all L cached tokens), and
 *    the cache size is 2 (K and V) x layers x heads x head_dim x tokens x
 *    bytes per element (oracle_kv_bytes).
 *  - "[Hacker News 요약] ... Tiny-vLLM ..." (aisleshub), section
 *    "고성능 추론을 위한 고급 최적화 기법": attention is the basic formula of
 *    "Attention is all you need" (softmax(q K^T * scale) V), the KV cache keeps
 *    K/V projections of previous tokens, grouped-query attention lets several
 *    query heads share one K/V head, and a causal mask lets a token see only
 *    earlier tokens.  With one decode query at the last position the mask
 *    keeps every cached token.
 *  - Readings where the pages are silent (stated, not derived): the pool is
 *    laid out [num_blocks][num_kv_heads][block_size][head_dim]; query head h
 *    reads kv head h / (Hq / Hkv) (contiguous groups); a sequence with no
 *    cached token outputs zeros; a negative slot means "do not write"; a slot
 *    past the pool is not written either.
 *
 * Everything is computed in double.  bf16 inputs are widened exactly
 * (bits << 16 is the float with the same value; float -> double is exact).
 * Sums run in logical token order, so the result does not depend on where the
 * blocks physically are.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- bf16 (8-bit exponent, 7-bit mantissa: the upper half of an IEEE float) ---- */
double oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ---- KV size accounting: 2 (K and V) x layers x heads x head_dim x tokens x bytes ---- */
int64_t oracle_kv_bytes(int64_t layers, int64_t kv_heads, int64_t head_dim, int64_t tokens,
                        int64_t bytes_per_element) {
    return 2 * layers * kv_heads * head_dim * tokens * bytes_per_element;
}

/* ---- logical -> physical: the slot of logical position p in a sequence's table ---- */
int64_t oracle_slot(const int32_t* table_row, int64_t position, int64_t block_size) {
    const int64_t logical_block = position / block_size;
    const int64_t offset = position % block_size;
    return (int64_t)table_row[logical_block] * block_size + offset;
}

/* slots for the newest token of each sequence (position = length - 1) */
void oracle_slot_mapping(const int32_t* block_tables, int64_t max_blocks_per_seq,
                         const int32_t* lengths_after_append, int64_t num_seqs,
                         int64_t block_size, int64_t* slots) {
    for (int64_t b = 0; b < num_seqs; ++b) {
        const int64_t p = (int64_t)lengths_after_append[b] - 1;
        slots[b] = p < 0 ? -1 : oracle_slot(block_tables + b * max_blocks_per_seq, p, block_size);
    }
}

/* grouped-query attention: query head h reads kv head h / (Hq / Hkv) */
static int64_t kv_head_of(int64_t h, int64_t num_q_heads, int64_t num_kv_heads) {
    return h / (num_q_heads / num_kv_heads);
}

/* element index of (block, kv head, offset, d) in the [N][Hkv][Bs][D] pool */
static int64_t pool_index(int64_t block, int64_t kv_head, int64_t offset, int64_t d,
                          int64_t num_kv_heads, int64_t block_size, int64_t head_dim) {
    return ((block * num_kv_heads + kv_head) * block_size + offset) * head_dim + d;
}

/* ---- KV append: write token t's K/V rows into slot slot_mapping[t] ---- */
void oracle_append_kv(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping,
                      int64_t num_tokens, int64_t num_kv_heads, int64_t head_dim,
                      int64_t block_size, int64_t num_blocks, uint16_t* k_cache,
                      uint16_t* v_cache) {
    for (int64_t t = 0; t < num_tokens; ++t) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0 || slot >= num_blocks * block_size) continue;
        const int64_t block = slot / block_size;
        const int64_t offset = slot % block_size;
        for (int64_t h = 0; h < num_kv_heads; ++h) {
            for (int64_t d = 0; d < head_dim; ++d) {
                const int64_t dst = pool_index(block, h, offset, d, num_kv_heads, block_size, head_dim);
                const int64_t src = (t * num_kv_heads + h) * head_dim + d;
                k_cache[dst] = k[src];
                v_cache[dst] = v[src];
            }
        }
    }
}

/* Gather logical tokens [0, L) of one sequence and kv head into contiguous fp64 rows. */
static void gather_sequence(const uint16_t* cache, const int32_t* table_row, int64_t L,
                            int64_t kv_head, int64_t num_kv_heads, int64_t block_size,
                            int64_t head_dim, double* rows) {
    for (int64_t j = 0; j < L; ++j) {
        const int64_t slot = oracle_slot(table_row, j, block_size);
        const int64_t block = slot / block_size;
        const int64_t offset = slot % block_size;
        for (int64_t d = 0; d < head_dim; ++d) {
            rows[j * head_dim + d] = oracle_bf16_to_double(
                cache[pool_index(block, kv_head, offset, d, num_kv_heads, block_size, head_dim)]);
        }
    }
}

/*
 * Textbook attention of one query over contiguous rows [t0, t1):
 *   s_j = scale * sum_d q_d K_jd,  m = max_j s_j,  e_j = exp(s_j - m),  Z = sum_j e_j,
 *   p_j = e_j / Z,  o_d = sum_j p_j V_jd,  lse = m + ln Z.
 * Writes o (head_dim values), returns lse; *psum = sum_j p_j.
 */
static double attend(const double* qd, const double* K, const double* V, int64_t t0, int64_t t1,
                     int64_t head_dim, double scale, double* s, double* o, double* psum) {
    double m = -INFINITY;
    for (int64_t j = t0; j < t1; ++j) {
        double dot = 0.0;
        for (int64_t d = 0; d < head_dim; ++d) dot += qd[d] * K[j * head_dim + d];
        s[j - t0] = scale * dot;
        if (s[j - t0] > m) m = s[j - t0];
    }
    double Z = 0.0;
    for (int64_t j = t0; j < t1; ++j) Z += exp(s[j - t0] - m);
    double total = 0.0;
    for (int64_t d = 0; d < head_dim; ++d) o[d] = 0.0;
    for (int64_t j = t0; j < t1; ++j) {
        const double p = exp(s[j - t0] - m) / Z;
        total += p;
        for (int64_t d = 0; d < head_dim; ++d) o[d] += p * V[j * head_dim + d];
    }
    if (psum) *psum = total;
    return m + log(Z);
}

static int g_threads = 0; /* 0: OpenMP default */

void oracle_set_num_threads(int n) { g_threads = n; }

int oracle_num_threads(void) {
#ifdef _OPENMP
    return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Paged decode attention.
 *   q            [B][Hq][D] bf16 bits        block_tables [B][MB] int32
 *   k/v_cache    [N][Hkv][Bs][D] bf16 bits   context_lens [B] int32 (tokens attended)
 *   out          [B][Hq][D] double           weight_sums  [B][Hq] double or NULL
 * For each sequence b and query head h: gather the L = context_lens[b] cached
 * tokens of kv head h / (Hq/Hkv) into contiguous rows, then attend.
 * Work is spread over (sequence, kv head) pairs so one gather serves the query
 * heads that read that kv head; each output's arithmetic is the same serial
 * loop whatever the thread count.
 */
int oracle_paged_decode(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                        const int32_t* block_tables, const int32_t* context_lens,
                        int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                        int64_t head_dim, int64_t block_size, int64_t max_blocks_per_seq,
                        double scale, double* out, double* weight_sums) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
    const int64_t pairs = num_seqs * num_kv_heads;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(oracle_num_threads())
    for (int64_t pair = 0; pair < pairs; ++pair) {
        const int64_t b = pair / num_kv_heads;
        const int64_t kvh = pair % num_kv_heads;
        const int64_t L = context_lens[b];
        const int32_t* table_row = block_tables + b * max_blocks_per_seq;
        for (int64_t h = 0; h < num_q_heads; ++h) {
            if (kv_head_of(h, num_q_heads, num_kv_heads) != kvh) continue;
            double* o = out + (b * num_q_heads + h) * head_dim;
            for (int64_t d = 0; d < head_dim; ++d) o[d] = 0.0;
            if (weight_sums) weight_sums[b * num_q_heads + h] = 0.0;
        }
        if (L <= 0) continue;
        double* K = (double*)malloc(sizeof(double) * (size_t)(L * head_dim));
        double* V = (double*)malloc(sizeof(double) * (size_t)(L * head_dim));
        double* s = (double*)malloc(sizeof(double) * (size_t)L);
        double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
        if (!K || !V || !s || !qd) {
#pragma omp atomic write
            failed = 1;
        } else {
            gather_sequence(k_cache, table_row, L, kvh, num_kv_heads, block_size, head_dim, K);
            gather_sequence(v_cache, table_row, L, kvh, num_kv_heads, block_size, head_dim, V);
            for (int64_t h = 0; h < num_q_heads; ++h) {
                if (kv_head_of(h, num_q_heads, num_kv_heads) != kvh) continue;
                for (int64_t d = 0; d < head_dim; ++d)
                    qd[d] = oracle_bf16_to_double(q[(b * num_q_heads + h) * head_dim + d]);
                attend(qd, K, V, 0, L, head_dim, scale, s,
                       out + (b * num_q_heads + h) * head_dim,
                       weight_sums ? weight_sums + b * num_q_heads + h : NULL);
            }
        }
        free(K);
        free(V);
        free(s);
        free(qd);
    }
    return failed ? -2 : 0;
}

/*
 * Partial attention of every (sequence, query head) over the logical token
 * range [t0, min(t1, L)): normalised output o [B][Hq][D] and its natural-log
 * log-sum-exp lse [B][Hq] (-inf and o = 0 when the range is empty).  This is
 * the state a split of the context produces before the splits are merged.
 */
int oracle_paged_decode_partial(const uint16_t* q, const uint16_t* k_cache,
                                const uint16_t* v_cache, const int32_t* block_tables,
                                const int32_t* context_lens, int64_t num_seqs,
                                int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                                int64_t block_size, int64_t max_blocks_per_seq, double scale,
                                int64_t t0, int64_t t1, double* o_out, double* lse_out) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(oracle_num_threads())
    for (int64_t pair = 0; pair < num_seqs * num_kv_heads; ++pair) {
        const int64_t b = pair / num_kv_heads;
        const int64_t kvh = pair % num_kv_heads;
        const int64_t L = context_lens[b];
        const int64_t hi = t1 < L ? t1 : L;
        for (int64_t h = 0; h < num_q_heads; ++h) {
            if (kv_head_of(h, num_q_heads, num_kv_heads) != kvh) continue;
            for (int64_t d = 0; d < head_dim; ++d) o_out[(b * num_q_heads + h) * head_dim + d] = 0.0;
            lse_out[b * num_q_heads + h] = -INFINITY;
        }
        if (hi <= t0) continue;
        double* K = (double*)malloc(sizeof(double) * (size_t)(hi * head_dim));
        double* V = (double*)malloc(sizeof(double) * (size_t)(hi * head_dim));
        double* s = (double*)malloc(sizeof(double) * (size_t)(hi - t0));
        double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
        if (!K || !V || !s || !qd) {
#pragma omp atomic write
            failed = 1;
        } else {
            const int32_t* table_row = block_tables + b * max_blocks_per_seq;
            gather_sequence(k_cache, table_row, hi, kvh, num_kv_heads, block_size, head_dim, K);
            gather_sequence(v_cache, table_row, hi, kvh, num_kv_heads, block_size, head_dim, V);
            for (int64_t h = 0; h < num_q_heads; ++h) {
                if (kv_head_of(h, num_q_heads, num_kv_heads) != kvh) continue;
                for (int64_t d = 0; d < head_dim; ++d)
                    qd[d] = oracle_bf16_to_double(q[(b * num_q_heads + h) * head_dim + d]);
                lse_out[b * num_q_heads + h] =
                    attend(qd, K, V, t0, hi, head_dim, scale, s,
                           o_out + (b * num_q_heads + h) * head_dim, NULL);
            }
        }
        free(K);
        free(V);
        free(s);
        free(qd);
    }
    return failed ? -2 : 0;
}

/*
 * Merge S partial states of one query: each split s covers a disjoint token
 * range with normalised output o_s and lse_s = ln sum_{j in s} exp(score_j).
 * Softmax over the union: weight of split s is exp(lse_s - M) with
 * M = max_s lse_s; out = sum_s w_s o_s / sum_s w_s.  Splits with lse = -inf
 * (empty) get weight 0; if all are empty the output is zero.
 */
void oracle_merge_partials(const double* o, const double* lse, int64_t num_splits,
                           int64_t head_dim, double* out) {
    double M = -INFINITY;
    for (int64_t s = 0; s < num_splits; ++s)
        if (lse[s] > M) M = lse[s];
    for (int64_t d = 0; d < head_dim; ++d) out[d] = 0.0;
    if (M == -INFINITY) return;
    double W = 0.0;
    for (int64_t s = 0; s < num_splits; ++s) {
        const double w = exp(lse[s] - M);
        W += w;
        for (int64_t d = 0; d < head_dim; ++d) out[d] += w * o[s * head_dim + d];
    }
    for (int64_t d = 0; d < head_dim; ++d) out[d] /= W;
}

/*
 * ---- RoPE (rotary position embedding) ----
 * "[Hacker News 요약] ... Tiny-vLLM ..." (aisleshub), section "핵심 LLM 연산의 CUDA
 * 커널 구현", names RoPE among the per-layer operations of the Llama 3.2 1B model
 * it targets, and gives no formula.  Reading (stated, not derived): RoFormer's
 * rotation in the rotate-half pairing, with the caller's frequency base theta.
 * For i < D/2, the pair (x[i], x[i + D/2]) of each head of a token at
 * position p turns by the angle a_i = p * theta^(-2i/D):
 *   y[i]       = x[i] cos a_i - x[i + D/2] sin a_i
 *   y[i + D/2] = x[i] sin a_i + x[i + D/2] cos a_i
 * x: [T][H][D] bf16, pos: [T]; out: [T][H][D] double, unrounded.
 */
void oracle_rope(const uint16_t* x, int64_t T, int64_t H, int64_t D, const int32_t* pos,
                 double theta, double* out) {
    const int64_t half = D / 2;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t h = 0; h < H; ++h) {
            const uint16_t* xr = x + (t * H + h) * D;
            double* yr = out + (t * H + h) * D;
            for (int64_t i = 0; i < half; ++i) {
                const double a = (double)pos[t] * pow(theta, -2.0 * (double)i / (double)D);
                const double c = cos(a), s = sin(a);
                const double x1 = oracle_bf16_to_double(xr[i]);
                const double x2 = oracle_bf16_to_double(xr[i + half]);
                yr[i] = x1 * c - x2 * s;
                yr[i + half] = x1 * s + x2 * c;
            }
        }
}

/*
 * Round to the nearest bf16, ties to even (the format q and the caches are
 * stored in).  With |x| in [2^(e-1), 2^e), a normal bf16 there is a multiple
 * of 2^(e-8); below 2^-126 the subnormals are multiples of 2^-133.  Scaling by
 * a power of two is exact, and rint() rounds half to even, so
 * y = rint(x / q) * q is the correctly rounded value; past the largest finite
 * bf16 it becomes infinity.  y is then exact in float, whose upper 16 bits are
 * the bf16.
 */
void oracle_round_bf16(const double* x, int64_t n, uint16_t* out) {
    const double max_bf16 = (2.0 - ldexp(1.0, -7)) * ldexp(1.0, 127);
    for (int64_t k = 0; k < n; ++k) {
        double v = x[k];
        uint32_t u;
        if (isnan(v)) {
            out[k] = 0x7FC0;
            continue;
        }
        if (v != 0.0 && isfinite(v)) {
            int e;
            frexp(v, &e);                          /* |v| in [2^(e-1), 2^e) */
            const int qexp = e - 8 > -133 ? e - 8 : -133;
            v = ldexp(rint(ldexp(v, -qexp)), qexp);
            if (fabs(v) > max_bf16) v = v > 0 ? INFINITY : -INFINITY;
        }
        const float f = (float)v;                 /* exact: v is a bf16 value */
        memcpy(&u, &f, sizeof u);
        out[k] = (uint16_t)(u >> 16);
    }
}

/*
 * ---- FP8 KV cache (e4m3) ----
 * "[Hacker News 요약] ... Tiny-vLLM ..." (aisleshub), section "향후 전망", names
 * FP8 among the data types to support next, with no format or scale scheme.
 * Reading (stated, not derived): the OCP 8-bit floating-point E4M3 format --
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
 * exponent and mantissa all ones = NaN, largest finite 448, subnormals
 * m * 2^-9 -- with one scale per cache tensor.  A bf16 value x is stored as
 * code = e4m3(y), y = float(x) * float(1/scale) formed in float (that
 * product decides the code, so both sides take it in float), rounded to
 * nearest even with values past +-448 saturating to +-448; it reads back as
 * value(code) * scale.
 */
double oracle_e4m3_to_double(uint8_t code) {
    const int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);                          /* subnormal: m/8 * 2^(1-7) */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

uint8_t oracle_e4m3_from_float(float y) {
    if (isnan(y)) return 0x7F;
    const uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7E;                     /* saturate: S.1111.110 = 448 */
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                                           /* a in [2^(e-1), 2^e) */
    const int qexp = e - 4 > -9 ? e - 4 : -9;               /* 3 mantissa bits; subnormal quantum 2^-9 */
    a = ldexp(rint(ldexp(a, -qexp)), qexp);                 /* nearest, ties to even */
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);                                          /* a in [2^(e2-1), 2^e2) */
    const int E = e2 - 1 + 7;
    if (E >= 1) {
        const int m = (int)(ldexp(a, -(e2 - 1)) * 8.0 - 8.0);
        return sign | (uint8_t)(E << 3) | (uint8_t)m;
    }
    return sign | (uint8_t)(int)ldexp(a, 9);
}

/* codes of n bf16 values: e4m3(float(x) * inv_scale) */
void oracle_quantize_e4m3(const uint16_t* x, int64_t n, float inv_scale, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u = ((uint32_t)x[i]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        volatile float y = f * inv_scale;                   /* one float multiply, rounded */
        out[i] = oracle_e4m3_from_float(y);
    }
}

/* Append of e4m3 codes (already quantized rows) into u8 pools: same slots as oracle_append_kv. */
void oracle_append_kv_e4m3(const uint8_t* k, const uint8_t* v, const int64_t* slot_mapping,
                           int64_t num_tokens, int64_t num_kv_heads, int64_t head_dim,
                           int64_t block_size, int64_t num_blocks, uint8_t* k_cache,
                           uint8_t* v_cache) {
    for (int64_t t = 0; t < num_tokens; ++t) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0 || slot >= num_blocks * block_size) continue;
        const int64_t block = slot / block_size, offset = slot % block_size;
        for (int64_t h = 0; h < num_kv_heads; ++h)
            for (int64_t d = 0; d < head_dim; ++d) {
                const int64_t dst = pool_index(block, h, offset, d, num_kv_heads, block_size, head_dim);
                const int64_t src = (t * num_kv_heads + h) * head_dim + d;
                k_cache[dst] = k[src];
                v_cache[dst] = v[src];
            }
    }
}

static void gather_sequence_e4m3(const uint8_t* cache, double cache_scale, const int32_t* table_row,
                                 int64_t L, int64_t kv_head, int64_t num_kv_heads,
                                 int64_t block_size, int64_t head_dim, double* rows) {
    for (int64_t j = 0; j < L; ++j) {
        const int64_t slot = oracle_slot(table_row, j, block_size);
        const int64_t block = slot / block_size;
        const int64_t offset = slot % block_size;
        for (int64_t d = 0; d < head_dim; ++d)
            rows[j * head_dim + d] = cache_scale * oracle_e4m3_to_double(
                cache[pool_index(block, kv_head, offset, d, num_kv_heads, block_size, head_dim)]);
    }
}

/* oracle_paged_decode over e4m3 pools: K and V values are code values times their scale. */
int oracle_paged_decode_e4m3(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                             double k_scale, double v_scale, const int32_t* block_tables,
                             const int32_t* context_lens, int64_t num_seqs, int64_t num_q_heads,
                             int64_t num_kv_heads, int64_t head_dim, int64_t block_size,
                             int64_t max_blocks_per_seq, double scale, double* out) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
    const int64_t pairs = num_seqs * num_kv_heads;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(oracle_num_threads())
    for (int64_t pair = 0; pair < pairs; ++pair) {
        const int64_t b = pair / num_kv_heads, kvh = pair % num_kv_heads;
        const int64_t L = context_lens[b];
        const int32_t* table_row = block_tables + b * max_blocks_per_seq;
        for (int64_t h = 0; h < num_q_heads; ++h) {
            if (kv_head_of(h, num_q_heads, num_kv_heads) != kvh) continue;
            double* o = out + (b * num_q_heads + h) * head_dim;
            for (int64_t d = 0; d < head_dim; ++d) o[d] = 0.0;
        }
        if (L <= 0) continue;
        double* K = (double*)malloc(sizeof(double) * (size_t)(L * head_dim));
        double* V = (double*)malloc(sizeof(double) * (size_t)(L * head_dim));
        double* s = (double*)malloc(sizeof(double) * (size_t)L);
        double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
        if (!K || !V || !s || !qd) {
#pragma omp atomic write
            failed = 1;
        } else {
            gather_sequence_e4m3(k_cache, k_scale, table_row, L, kvh, num_kv_heads, block_size, head_dim, K);
            gather_sequence_e4m3(v_cache, v_scale, table_row, L, kvh, num_kv_heads, block_size, head_dim, V);
            for (int64_t h = 0; h < num_q_heads; ++h) {
                if (kv_head_of(h, num_q_heads, num_kv_heads) != kvh) continue;
                for (int64_t d = 0; d < head_dim; ++d)
                    qd[d] = oracle_bf16_to_double(q[(b * num_q_heads + h) * head_dim + d]);
                attend(qd, K, V, 0, L, head_dim, scale, s, out + (b * num_q_heads + h) * head_dim, NULL);
            }
        }
        free(K);
        free(V);
        free(s);
        free(qd);
    }
    return failed ? -2 : 0;
}

/*
 * ---- paged prefill (chunked prefill) ----
 * "Nano-vLLM로 배우는 vLLM 추론 엔진 작동 원리 한눈에 정리" (tilnote.io), section
 * "Prefill vs Decode: 추론이 '한 번에 읽고, 한 글자씩 쓴다'": prefill processes the
 * whole input at once; the Tiny-vLLM summary page, section "고성능 추론을 위한 고급
 * 최적화 기법", fixes the attention formula and the causal mask (a token sees only
 * itself and earlier tokens).  Reading: sequence b holds context_lens[b] = L
 * tokens in the paged cache after this step's append, the last Tq of them are
 * this step's queries (q rows cu_q[b] .. cu_q[b+1]-1, positions L-Tq .. L-1),
 * and the query at position p attends to cache tokens 0..p.
 *   q   [total_q][Hq][D] bf16      out [total_q][Hq][D] double
 */
int oracle_paged_prefill(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                         const int32_t* block_tables, const int32_t* cu_q, const int32_t* context_lens,
                         int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads, int64_t head_dim,
                         int64_t block_size, int64_t max_blocks_per_seq, double scale, double* out) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
    const int64_t pairs = num_seqs * num_kv_heads;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(oracle_num_threads())
    for (int64_t pair = 0; pair < pairs; ++pair) {
        const int64_t b = pair / num_kv_heads, kvh = pair % num_kv_heads;
        const int64_t L = context_lens[b];
        const int64_t q0 = cu_q[b], Tq = cu_q[b + 1] - cu_q[b];
        if (Tq <= 0) continue;
        if (Tq > L) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        const int32_t* table_row = block_tables + b * max_blocks_per_seq;
        double* K = (double*)malloc(sizeof(double) * (size_t)(L * head_dim));
        double* V = (double*)malloc(sizeof(double) * (size_t)(L * head_dim));
        double* s = (double*)malloc(sizeof(double) * (size_t)L);
        double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
        if (!K || !V || !s || !qd) {
#pragma omp atomic write
            failed = 1;
        } else {
            gather_sequence(k_cache, table_row, L, kvh, num_kv_heads, block_size, head_dim, K);
            gather_sequence(v_cache, table_row, L, kvh, num_kv_heads, block_size, head_dim, V);
            for (int64_t i = 0; i < Tq; ++i) {
                const int64_t pos = L - Tq + i;             /* the query's position */
                for (int64_t h = 0; h < num_q_heads; ++h) {
                    if (kv_head_of(h, num_q_heads, num_kv_heads) != kvh) continue;
                    const int64_t row = (q0 + i) * num_q_heads + h;
                    for (int64_t d = 0; d < head_dim; ++d) qd[d] = oracle_bf16_to_double(q[row * head_dim + d]);
                    attend(qd, K, V, 0, pos + 1, head_dim, scale, s, out + row * head_dim, NULL);
                }
            }
        }
        free(K);
        free(V);
        free(s);
        free(qd);
    }
    return failed ? -2 : 0;
}
