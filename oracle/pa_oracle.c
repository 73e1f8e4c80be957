/*
 * pa_oracle.c -- plain, slow, fp64 CPU oracle for the paged decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product links, loads or calls this
 * file; only the tests, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Pages cited (titles as printed on them):
 *   P1  "大模型部署中的PagedAttention：KV Cache显存管理突破"  (PagedAttention in LLM
 *       deployment: KV-cache memory management), blog.csdn.net
 *   P2  "大模型推理优化：KV Cache与PagedAttention技术详解"  (LLM inference
 *       optimisation: KV cache and PagedAttention explained), intelliparadigm.com
 *   P3  "LLM 推理中的 PageAttention 实现原理：虚拟内存管理在 KV Cache 中的创新应用"
 *       (How PageAttention works in LLM inference), dpshk.com
 *
 * What is computed, and where it comes from:
 *   - Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V            (P1 §1, first formula)
 *     taken as ONE softmax over all of a sequence's tokens in logical order.  The
 *     per-block sum of separately normalised softmaxes printed next to it (P1 §1,
 *     second formula; P1 §2 paged_attention sketch) is not normalised and is not
 *     the definition used here.  The scale is a caller parameter; 1/sqrt(d_k) is
 *     the value callers pass.
 *   - token index -> (physical block, offset) = (table[idx / B], idx % B)
 *                                        (P3 §三, BlockTable::get_physical_location)
 *   - blocks needed for n tokens = ceil(n / B)  (P3 §三, BlockTable::num_required_blocks)
 *   - KV bytes = 2 * seq_len * layers * heads * head_dim * dtype_size   (P2 §2.2)
 *   - writing the step's new K/V into the cache comes before attending over all
 *     t tokens                                                     (P2 §2.1, decode steps 3-5)
 *
 * Cache layout (a reading: the pages fix blocks of B tokens, P1 §1 and P3 §一, a
 * per-block tensor of (block_size, d_model), P1 §2, and a cache of
 * [seq_len, num_heads, head_dim], P2 §2.1, but not the order inside a block):
 *   cache[num_blocks][block_size][num_kv_heads][head_dim], element (slot, h, i)
 *   at ((slot * num_kv_heads + h) * head_dim + i), slot = phys * block_size + off.
 *
 * Values arrive as raw IEEE binary16 / bfloat16 bit patterns and are widened to
 * double exactly, by the formats' definitions, below.
 *
 * PA_ORACLE_MUTANT (compile-time) plants one known mistake; the test suite builds
 * each mutant and checks that some pin catches it.  The default build has none.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef PA_ORACLE_MUTANT
#define PA_ORACLE_MUTANT 0
#endif

#define ORACLE_F16 0
#define ORACLE_BF16 1

/* ---------------------------------------------------------------- formats */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double pa_oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
#if PA_ORACLE_MUTANT == 7
    const int bias_fix = 24; /* planted: exponent bias off by one */
#else
    const int bias_fix = 25; /* 15 (bias) + 10 (fraction bits) */
#endif
    if (e == 0)
        v = ldexp((double)m, -24); /* subnormal: m * 2^(1 - 15 - 10) */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - bias_fix);
    return sign ? -v : v;
}

/* bfloat16: the upper half of an IEEE binary32 -- 1 sign, 8 exponent (bias 127),
 * 7 fraction bits. */
double pa_oracle_bf16_to_double(uint16_t b) {
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int m = b & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)m, -133); /* subnormal: m * 2^(1 - 127 - 7) */
    else if (e == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + m), e - 134); /* (1 + m/2^7) * 2^(e - 127) */
    return sign ? -v : v;
}

static double widen(uint16_t bits, int dtype) {
    return dtype == ORACLE_BF16 ? pa_oracle_bf16_to_double(bits) : pa_oracle_half_to_double(bits);
}

/* OCP FP8 E4M3 ("e4m3fn"): 1 sign, 4 exponent bits (bias 7), 3 fraction bits, no
 * infinities, S.1111.111 is NaN; largest finite magnitude 448. */
double pa_oracle_e4m3_to_double(uint8_t b) {
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xf;
    int m = b & 7;
    double v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -9); /* subnormal: m/8 * 2^(1-7) */
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Nearest E4M3 code to x, ties to even; finite magnitudes at or beyond 448 and
 * infinities saturate to +-448; NaN gives the NaN code. */
uint8_t pa_oracle_e4m3_from_float(float x) {
    if (isnan(x)) return 0x7f;
    const int sign = signbit(x) ? 0x80 : 0;
    const double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7e);
    int e2;
    frexp(a, &e2); /* a = f * 2^e2, f in [0.5, 1): floor(log2 a) = e2 - 1 */
    const int subnormal = a < ldexp(1.0, -6);
    const double quantum = subnormal ? ldexp(1.0, -9) : ldexp(1.0, e2 - 1 - 3);
#if PA_ORACLE_MUTANT == 11
    double n = trunc(a / quantum); /* planted: rounds toward zero */
#else
    double n = rint(a / quantum); /* the division is exact; rint rounds half to even */
#endif
    int code;
    if (subnormal) {
        code = (int)n; /* n == 8 is the smallest normal, whose code is 0x08 as well */
    } else {
        int E = e2 - 1 + 7;
        if (n >= 16.0) { /* rounded up into the next binade */
            ++E;
            n = 8.0;
        }
        code = (E << 3) | ((int)n - 8);
    }
    return (uint8_t)(sign | code);
}

/* ---------------------------------------------------------- slot arithmetic */

/* P3 §三, BlockTable::num_required_blocks: ceil(n / B). */
int64_t pa_oracle_num_required_blocks(int64_t num_tokens, int64_t block_size) {
#if PA_ORACLE_MUTANT == 10
    return num_tokens / block_size; /* planted: floor instead of ceil */
#else
    return (num_tokens + block_size - 1) / block_size;
#endif
}

/* P3 §三, BlockTable::get_physical_location: (table[idx / B], idx % B), or
 * "none" (returns -1) when the table has no entry for that logical block. */
int pa_oracle_physical_location(const int32_t* table, int64_t num_entries, int64_t token_idx,
                                int64_t block_size, int64_t* phys, int64_t* offset) {
    int64_t logical = token_idx / block_size;
    if (token_idx < 0 || logical >= num_entries) return -1;
    *phys = table[logical];
    *offset = token_idx % block_size;
    return 0;
}

/* P2 §2.2: memory = 2 x seq_len x num_layers x num_heads x head_dim x dtype_size. */
int64_t pa_oracle_kv_bytes(int64_t seq_len, int64_t num_layers, int64_t num_heads, int64_t head_dim,
                           int64_t dtype_size) {
    return 2 * seq_len * num_layers * num_heads * head_dim * dtype_size;
}

/* Slot of each sequence's newest token.  context_lens count the new token (P2
 * §2.1: the step's K/V is appended, then attention runs over all t tokens), so the
 * new token sits at position len-1: slot = table[(len-1)/B]*B + (len-1)%B.  A
 * sequence with len 0 has no new token: slot -1.  Returns 0, or -1 when a table
 * entry is missing. */
int pa_oracle_slot_mapping(const int32_t* tables, int max_blocks_per_seq, const int32_t* context_lens,
                           int num_seqs, int block_size, int64_t* slots) {
    for (int s = 0; s < num_seqs; ++s) {
        int64_t len = context_lens[s];
        if (len <= 0) {
            slots[s] = -1;
            continue;
        }
#if PA_ORACLE_MUTANT == 9
        int64_t pos = len; /* planted: position of the token after the new one */
#else
        int64_t pos = len - 1;
#endif
        int64_t phys, off;
        if (pa_oracle_physical_location(tables + (int64_t)s * max_blocks_per_seq, max_blocks_per_seq, pos,
                                        block_size, &phys, &off) != 0)
            return -1;
        slots[s] = phys * block_size + off;
    }
    return 0;
}

/* --------------------------------------------------------- cache write (K1) */

/* For token i and kv head h: cache[slot[i]][h][:] = k[i][h][:] (and v alike),
 * bit for bit.  Slots outside [0, num_blocks*block_size) are skipped; the return
 * value counts them. */
int pa_oracle_reshape_and_cache(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping,
                                uint16_t* k_cache, uint16_t* v_cache, int num_tokens, int num_kv_heads,
                                int head_dim, int block_size, int num_blocks) {
    int skipped = 0;
    int64_t num_slots = (int64_t)num_blocks * block_size;
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0 || slot >= num_slots) {
            ++skipped;
            continue;
        }
#if PA_ORACLE_MUTANT == 8
        slot = (slot + 1) % num_slots; /* planted: writes the neighbouring slot */
#endif
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t src = ((int64_t)i * num_kv_heads + h) * head_dim;
            int64_t dst = (slot * num_kv_heads + h) * head_dim;
            memcpy(k_cache + dst, k + src, sizeof(uint16_t) * (size_t)head_dim);
            memcpy(v_cache + dst, v + src, sizeof(uint16_t) * (size_t)head_dim);
        }
    }
    return skipped;
}

/* The cache write into an fp8 cache: each element of k (v) is widened to fp32,
 * divided by k_scale (v_scale) in fp32 (IEEE, round to nearest) and stored as the
 * nearest E4M3 code (saturating).  Slots outside [0, num_blocks*block_size) are
 * skipped; the return value counts them. */
int pa_oracle_reshape_and_cache_fp8(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping,
                                    uint8_t* k_cache, uint8_t* v_cache, int num_tokens, int num_kv_heads,
                                    int head_dim, int block_size, int num_blocks, int dtype, float k_scale,
                                    float v_scale) {
    int skipped = 0;
    int64_t num_slots = (int64_t)num_blocks * block_size;
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0 || slot >= num_slots) {
            ++skipped;
            continue;
        }
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t src = ((int64_t)i * num_kv_heads + h) * head_dim;
            int64_t dst = (slot * num_kv_heads + h) * head_dim;
            for (int j = 0; j < head_dim; ++j) {
                const float kx = (float)widen(k[src + j], dtype) / k_scale;
                const float vx = (float)widen(v[src + j], dtype) / v_scale;
                k_cache[dst + j] = pa_oracle_e4m3_from_float(kx);
                v_cache[dst + j] = pa_oracle_e4m3_from_float(vx);
            }
        }
    }
    return skipped;
}

/* ------------------------------------------------------ whole-block copies */

/* For each pair (src, dst): the dst block of both caches becomes a copy of the
 * src block (block_size * num_kv_heads * head_dim elements), bit for bit.  Pairs
 * with an id outside [0, num_blocks) are skipped; the return value counts them. */
int pa_oracle_copy_blocks(uint16_t* k_cache, uint16_t* v_cache, const int32_t* pairs, int num_pairs,
                          int num_blocks, int block_size, int num_kv_heads, int head_dim) {
    int skipped = 0;
    const int64_t per_block = (int64_t)block_size * num_kv_heads * head_dim;
    for (int i = 0; i < num_pairs; ++i) {
        const int32_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            ++skipped;
            continue;
        }
        memmove(k_cache + dst * per_block, k_cache + src * per_block, sizeof(uint16_t) * (size_t)per_block);
        memmove(v_cache + dst * per_block, v_cache + src * per_block, sizeof(uint16_t) * (size_t)per_block);
    }
    return skipped;
}

/* ------------------------------------------------------------- decode (K2+K3) */

typedef struct {
    const uint16_t *q, *k_cache, *v_cache;
    const uint8_t *k8, *v8; /* fp8 caches (k_cache / v_cache unused then) */
    double k_scale, v_scale;
    const int32_t *tables, *context_lens;
    double scale;
    int num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype;
    const int32_t* pairs; /* NULL: every (s, h) in order; else npairs (s, h) pairs */
    int npairs;
    double* out;
    int nthreads;
    int error; /* set by workers: 1 bad argument / table entry */
} decode_job;

typedef struct {
    decode_job* job;
    int tid;
} worker_arg;

/* Prefill: query rows come from a packed [T][H][d] array; query row i of sequence
 * s sits at absolute position context_lens[s] - n_s + i and attends to tokens
 * 0..position (causal). */
typedef struct {
    decode_job base;       /* caches, tables, lengths, scale, shapes (q unused) */
    const uint16_t* q;     /* [T][H][d] */
    const int32_t* query_start; /* [S + 1] */
    int total_queries;
} prefill_job;

/* Value of cache element `idx`: a 16-bit element widened, or an fp8 code times its scale. */
static double kval(const decode_job* j, int64_t idx) {
    return j->k8 ? pa_oracle_e4m3_to_double(j->k8[idx]) * j->k_scale : widen(j->k_cache[idx], j->dtype);
}
static double vval(const decode_job* j, int64_t idx) {
    return j->v8 ? pa_oracle_e4m3_to_double(j->v8[idx]) * j->v_scale : widen(j->v_cache[idx], j->dtype);
}

/* Element offset of (token slot, kv head, 0) in the cache layout above. */
static int64_t cache_row(const decode_job* j, int64_t phys, int64_t off, int kv_head) {
#if PA_ORACLE_MUTANT == 3
    /* planted: heads outside tokens inside a block ([NB][Hk][B][d]) */
    return ((phys * j->num_kv_heads + kv_head) * j->block_size + off) * j->head_dim;
#else
    return ((phys * j->block_size + off) * j->num_kv_heads + kv_head) * j->head_dim;
#endif
}

static int attend(const decode_job* j, int s, int h, const uint16_t* qrow, int64_t len, double* out, double* qd,
                  double* x);

static int decode_one(const decode_job* j, int s, int h, double* out, double* qd, double* x) {
    const int64_t len = j->context_lens[s];
    if (len < 0 || len > (int64_t)j->max_blocks_per_seq * j->block_size) return 1;
    return attend(j, s, h, j->q + ((int64_t)s * j->num_heads + h) * j->head_dim, len, out, qd, x);
}

/* Attention of one query row (query head h of sequence s) over the sequence's
 * first `len` tokens:
 *   x_t = scale * sum_i q_i K_t,i                for t = 0..len-1 (logical order)
 *   out = sum_t exp(x_t - M) V_t / sum_t exp(x_t - M),   M = max_t x_t
 * M only keeps exp() in range; any constant gives the same value in exact math. */
static int attend(const decode_job* j, int s, int h, const uint16_t* qrow, int64_t len, double* out, double* qd,
                  double* x) {
    const int d = j->head_dim, bs = j->block_size;
    const int group = j->num_heads / j->num_kv_heads;
#if PA_ORACLE_MUTANT == 4
    const int kv_head = h % j->num_kv_heads; /* planted: interleaved GQA groups */
    (void)group;
#else
    const int kv_head = h / group; /* contiguous groups of `group` query heads */
#endif
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    if (len == 0) return 0; /* empty context: zeros */

    for (int i = 0; i < d; ++i) qd[i] = widen(qrow[i], j->dtype);

    const int32_t* table = j->tables + (int64_t)s * j->max_blocks_per_seq;
    for (int64_t t = 0; t < len; ++t) {
        int64_t phys, off;
        if (pa_oracle_physical_location(table, j->max_blocks_per_seq, t, bs, &phys, &off) != 0) return 1;
#if PA_ORACLE_MUTANT == 2
        off = (t + 1) % bs; /* planted: off-by-one offset inside the block */
#endif
        if (phys < 0 || phys >= j->num_blocks) return 1;
        const int64_t krow = cache_row(j, phys, off, kv_head);
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += qd[i] * kval(j, krow + i);
#if PA_ORACLE_MUTANT == 1
        x[t] = dot; /* planted: scale dropped */
#else
        x[t] = j->scale * dot;
#endif
    }

#if PA_ORACLE_MUTANT == 5
    /* planted: the per-block formula -- a softmax inside each block, summed */
    for (int64_t b0 = 0; b0 < len; b0 += bs) {
        int64_t b1 = b0 + bs < len ? b0 + bs : len;
        double m = -INFINITY, den = 0.0;
        for (int64_t t = b0; t < b1; ++t) m = x[t] > m ? x[t] : m;
        for (int64_t t = b0; t < b1; ++t) den += exp(x[t] - m);
        for (int64_t t = b0; t < b1; ++t) {
            int64_t phys, off;
            pa_oracle_physical_location(table, j->max_blocks_per_seq, t, bs, &phys, &off);
            const int64_t vrow = cache_row(j, phys, off, kv_head);
            double w = exp(x[t] - m) / den;
            for (int i = 0; i < d; ++i) out[i] += w * vval(j, vrow + i);
        }
    }
    return 0;
#else
    double m = -INFINITY;
    for (int64_t t = 0; t < len; ++t) m = x[t] > m ? x[t] : m;
    double den = 0.0;
    for (int64_t t = 0; t < len; ++t) {
        int64_t phys, off;
        pa_oracle_physical_location(table, j->max_blocks_per_seq, t, bs, &phys, &off);
#if PA_ORACLE_MUTANT == 2
        off = (t + 1) % bs;
#endif
        const int64_t vrow = cache_row(j, phys, off, kv_head);
        double w = exp(x[t] - m);
        den += w;
        for (int i = 0; i < d; ++i) out[i] += w * vval(j, vrow + i);
    }
#if PA_ORACLE_MUTANT == 6
    (void)den; /* planted: the softmax denominator is left out */
#else
    for (int i = 0; i < d; ++i) out[i] /= den;
#endif
    return 0;
#endif
}

static void* decode_worker(void* p) {
    worker_arg* a = (worker_arg*)p;
    decode_job* j = a->job;
    const int d = j->head_dim;
    int64_t max_len = (int64_t)j->max_blocks_per_seq * j->block_size;
    double* qd = (double*)malloc(sizeof(double) * (size_t)d);
    double* x = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
    if (!qd || !x) {
        j->error = 2;
        free(qd);
        free(x);
        return NULL;
    }
    int total = j->pairs ? j->npairs : j->num_seqs * j->num_heads;
    for (int w = a->tid; w < total; w += j->nthreads) {
        int s, h;
        if (j->pairs) {
            s = j->pairs[2 * w];
            h = j->pairs[2 * w + 1];
        } else {
            s = w / j->num_heads;
            h = w % j->num_heads;
        }
        if (s < 0 || s >= j->num_seqs || h < 0 || h >= j->num_heads ||
            decode_one(j, s, h, j->out + (int64_t)w * d, qd, x) != 0)
            j->error = 1;
    }
    free(qd);
    free(x);
    return NULL;
}

static int run_decode(decode_job* job) {
    int nthreads = job->nthreads;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    worker_arg* args = (worker_arg*)malloc(sizeof(worker_arg) * (size_t)nthreads);
    if (!th || !args) {
        free(th);
        free(args);
        return 2;
    }
    for (int t = 0; t < nthreads; ++t) {
        args[t].job = job;
        args[t].tid = t;
        if (t > 0) pthread_create(&th[t], NULL, decode_worker, &args[t]);
    }
    decode_worker(&args[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(args);
    return job->error;
}

static int bad_sizes(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                     int max_blocks_per_seq, int dtype) {
    return num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
           head_dim <= 0 || block_size <= 0 || num_blocks < 0 || max_blocks_per_seq < 0 ||
           (dtype != ORACLE_F16 && dtype != ORACLE_BF16);
}

/* Decode attention for every (s, h) (pairs == NULL, out is [S][H][d]) or for the
 * listed (s, h) pairs (out is [npairs][d]).  Returns 0, 1 on a bad argument or an
 * out-of-range table entry / length, 2 on allocation failure. */
int pa_oracle_decode(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                     const int32_t* block_tables, const int32_t* context_lens, double scale, int num_seqs,
                     int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                     int max_blocks_per_seq, int dtype, const int32_t* pairs, int npairs, double* out,
                     int nthreads) {
    if (bad_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype))
        return 1;
    decode_job job = {q, k_cache, v_cache, NULL, NULL, 1.0, 1.0, block_tables, context_lens, scale, num_seqs,
                      num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype,
                      pairs, npairs, out, nthreads < 1 ? 1 : nthreads, 0};
    return run_decode(&job);
}

/* The same over fp8 caches: K = code * k_scale, V = code * v_scale, exactly. */
int pa_oracle_decode_fp8(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                         const int32_t* block_tables, const int32_t* context_lens, double scale, double k_scale,
                         double v_scale, int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, int max_blocks_per_seq, int dtype, const int32_t* pairs, int npairs,
                         double* out, int nthreads) {
    if (bad_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype))
        return 1;
    decode_job job = {q, NULL, NULL, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale,
                      num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                      dtype, pairs, npairs, out, nthreads < 1 ? 1 : nthreads, 0};
    return run_decode(&job);
}

static void* prefill_worker(void* p) {
    worker_arg* a = (worker_arg*)p;
    prefill_job* pj = (prefill_job*)a->job;
    decode_job* j = &pj->base;
    const int d = j->head_dim;
    int64_t max_len = (int64_t)j->max_blocks_per_seq * j->block_size;
    double* qd = (double*)malloc(sizeof(double) * (size_t)d);
    double* x = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
    if (!qd || !x) {
        j->error = 2;
        free(qd);
        free(x);
        return NULL;
    }
    const int64_t rows = (int64_t)pj->total_queries * j->num_heads;
    for (int64_t w = a->tid; w < rows; w += j->nthreads) {
        const int64_t qi = w / j->num_heads;
        const int h = (int)(w % j->num_heads);
        int s = 0;  /* the sequence owning packed query row qi */
        while (s < j->num_seqs && pj->query_start[s + 1] <= qi) ++s;
        if (s >= j->num_seqs) {
            j->error = 1;
            continue;
        }
        const int64_t n = pj->query_start[s + 1] - pj->query_start[s];
        const int64_t len = j->context_lens[s];
        const int64_t pos = len - n + (qi - pj->query_start[s]); /* absolute position of this query */
        if (len > max_len || pos < 0) {
            j->error = 1;
            continue;
        }
#if PA_ORACLE_MUTANT == 12
        const int64_t nvis = pos + 2 < len ? pos + 2 : len; /* planted: sees one token past its position */
#else
        const int64_t nvis = pos + 1; /* tokens 0 .. pos */
#endif
        if (attend(j, s, h, pj->q + (qi * j->num_heads + h) * d, nvis, j->out + w * d, qd, x) != 0)
            j->error = 1;
    }
    free(qd);
    free(x);
    return NULL;
}

/* Prefill attention: out[i][h] for every packed query row i (of T) and head h,
 * causal over the paged cache (which already holds the chunk's own K/V).  Query
 * rows of sequence s are rows query_start[s] .. query_start[s+1]-1.  out is
 * [T][H][d].  Returns 0, 1 on a bad argument, 2 on allocation failure. */
int pa_oracle_prefill(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                      const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
                      double scale, int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, int max_blocks_per_seq, int dtype, double* out, int nthreads) {
    if (bad_sizes(num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype))
        return 1;
    for (int s = 0; s < num_seqs; ++s)
        if (query_start[s + 1] < query_start[s]) return 1;
    prefill_job pj;
    decode_job base = {NULL, k_cache, v_cache, NULL, NULL, 1.0, 1.0, block_tables, context_lens, scale, num_seqs,
                       num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype,
                       NULL, 0, out, nthreads < 1 ? 1 : nthreads, 0};
    pj.base = base;
    pj.q = q;
    pj.query_start = query_start;
    pj.total_queries = query_start[num_seqs];
    int n = pj.base.nthreads;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n);
    worker_arg* args = (worker_arg*)malloc(sizeof(worker_arg) * (size_t)n);
    if (!th || !args) {
        free(th);
        free(args);
        return 2;
    }
    for (int t = 0; t < n; ++t) {
        args[t].job = (decode_job*)&pj;
        args[t].tid = t;
        if (t > 0) pthread_create(&th[t], NULL, prefill_worker, &args[t]);
    }
    prefill_worker(&args[0]);
    for (int t = 1; t < n; ++t) pthread_join(th[t], NULL);
    free(th);
    free(args);
    return pj.base.error;
}

/* Build-time identification for the tests: which mistake (0 = none) is planted. */
int pa_oracle_mutant_id(void) { return PA_ORACLE_MUTANT; }
