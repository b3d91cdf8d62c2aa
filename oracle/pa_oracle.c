/*
 * pa_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU restatement of what the paged-KV hot
 * path computes, in fp64.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path and includes nothing from it.
 *
 * Sources (pages cited by title and section):
 *  [P1] "LLM inference optimization: KV cache & PagedAttention"
 *       (carlstack.gravito.dev)
 *  [P2] "vLLM explained" (jackchen890311.github.io)
 *
 * What is computed:
 *  - attention:   out = softmax(q . K^T * scale) . V           [P1] §二, the
 *                 Attention(Q,K,V) formula;
 *  - paging:      token t of a sequence lives in physical block
 *                 block_table[t / B] at offset t % B, blocks of B = 16 tokens,
 *                 not contiguous                                 [P1] §三.1,
 *                 [P2] "PagedAttention：用分頁管理 KV cache";
 *  - paging leaves the math unchanged, so the oracle gathers K/V in LOGICAL
 *    order and then evaluates the plain definition           [P2] "兩層實作";
 *  - chunked prefill: a chunk of new queries at absolute positions H..H+L-1
 *    attends causally to the paged history and to itself     [P1] §六.2,
 *    [P2] "附錄與延伸" (Chunked Prefill);
 *  - FP8 KV cache: one byte per element                      [P2] "Block 的大小
 *    怎麼決定" (FP8 1 byte); element value = E4M3 value x per-tensor scale;
 *  - slot write of new K/V and copy-on-write block copy     [P1] §三.2,
 *    [P2] "帶來的好處" (copy-on-write).
 *
 * Number formats are decoded from their published definitions: IEEE 754
 * binary16 and binary32, bfloat16 (the upper half of binary32) and OCP 8-bit
 * floating point E4M3 ("FN": bias 7, no infinities, S.1111.111 is NaN,
 * largest finite 448).  Encoding to E4M3 is round-to-nearest-even with
 * saturation to +-448 (the "satfinite" reading of a quantiser that must not
 * produce NaN from finite input).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2, ORC_E4M3 = 3 };

/* ------------------------------------------------------------------------ */
/* number formats                                                           */
/* ------------------------------------------------------------------------ */

double orc_f16_to_f64(uint16_t h) {
    int s = h >> 15, e = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24); /* subnormal: m/2^10 * 2^-14 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -v : v;
}

double orc_bf16_to_f64(uint16_t b) {
    int s = b >> 15, e = (b >> 7) & 0xff, m = b & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)m, -133); /* subnormal: m/2^7 * 2^-126 */
    else if (e == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1.0 + m / 128.0, e - 127);
    return s ? -v : v;
}

double orc_f32_to_f64(uint32_t w) {
    int s = w >> 31, e = (w >> 23) & 0xff;
    uint32_t m = w & 0x7fffff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -149); /* subnormal: m/2^23 * 2^-126 */
    else if (e == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1.0 + m / 8388608.0, e - 127);
    return s ? -v : v;
}

double orc_e4m3_to_f64(uint8_t x) {
    int s = x >> 7, e = (x >> 3) & 0xf, m = x & 0x7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9); /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round x to the nearest multiple of 2^q, ties to the even multiple. */
static double round_to_quantum(double x, int q) {
    double r = ldexp(x, -q); /* exact: scaling by a power of two */
    double fl = floor(r);
    double frac = r - fl;    /* exact for |r| < 2^52 */
    double n;
    if (frac > 0.5)
        n = fl + 1.0;
    else if (frac < 0.5)
        n = fl;
    else
        n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    return ldexp(n, q);
}

/* Round a finite x to a binary format with p significand bits (implicit bit
 * included) and smallest normal exponent emin; no range limit applied. */
static double round_to_format(double x, int p, int emin) {
    if (x == 0.0 || isnan(x) || isinf(x))
        return x;
    int e;
    frexp(fabs(x), &e); /* |x| = f * 2^e, f in [0.5, 1) -> leading bit 2^(e-1) */
    int lead = e - 1;
    if (lead < emin)
        lead = emin;
    return round_to_quantum(x, lead - (p - 1));
}

/* E4M3 code of a float, round-to-nearest-even, saturating to +-448. */
uint8_t orc_f32_to_e4m3_satfinite(float xf) {
    double x = (double)xf;
    if (isnan(x))
        return 0x7f;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double r = round_to_format(fabs(x), 4, -6);
    if (r > 448.0)
        r = 448.0;
    if (r == 0.0)
        return sign;
    int e;
    frexp(r, &e);
    int lead = e - 1;
    if (lead < -6) { /* subnormal: r = m * 2^-9 */
        int m = (int)ldexp(r, 9);
        return sign | (uint8_t)m;
    }
    int m = (int)(ldexp(r, -lead) * 8.0) - 8; /* r = (1 + m/8) 2^lead */
    return sign | (uint8_t)(((lead + 7) << 3) | m);
}

/* bfloat16 / binary16 codes of a double, round-to-nearest-even, overflow to
 * infinity; used by tests to compare in the output dtype. */
uint16_t orc_f64_to_bf16(double x) {
    if (isnan(x))
        return 0x7fc0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double r = round_to_format(fabs(x), 8, -126);
    if (r == 0.0)
        return sign;
    if (r >= ldexp(1.0, 128) || isinf(r))
        return sign | 0x7f80;
    int e;
    frexp(r, &e);
    int lead = e - 1;
    if (lead < -126)
        return sign | (uint16_t)ldexp(r, 133);
    int m = (int)(ldexp(r, -lead) * 128.0) - 128;
    return sign | (uint16_t)(((lead + 127) << 7) | m);
}

uint16_t orc_f64_to_f16(double x) {
    if (isnan(x))
        return 0x7e00;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double r = round_to_format(fabs(x), 11, -14);
    if (r == 0.0)
        return sign;
    if (r >= 65520.0 || isinf(r)) /* above max finite 65504 after rounding */
        return sign | 0x7c00;
    int e;
    frexp(r, &e);
    int lead = e - 1;
    if (lead < -14)
        return sign | (uint16_t)ldexp(r, 24);
    int m = (int)(ldexp(r, -lead) * 1024.0) - 1024;
    return sign | (uint16_t)(((lead + 15) << 10) | m);
}

static int elem_bytes(int dt) {
    switch (dt) {
    case ORC_F32: return 4;
    case ORC_F16: return 2;
    case ORC_BF16: return 2;
    case ORC_E4M3: return 1;
    }
    return 0;
}

/* value of element i of a raw array of dtype dt */
static double load_elem(const void* base, int dt, int64_t i) {
    const uint8_t* p = (const uint8_t*)base;
    switch (dt) {
    case ORC_F32: {
        uint32_t w;
        memcpy(&w, p + 4 * i, 4);
        return orc_f32_to_f64(w);
    }
    case ORC_F16: {
        uint16_t h;
        memcpy(&h, p + 2 * i, 2);
        return orc_f16_to_f64(h);
    }
    case ORC_BF16: {
        uint16_t b;
        memcpy(&b, p + 2 * i, 2);
        return orc_bf16_to_f64(b);
    }
    case ORC_E4M3:
        return orc_e4m3_to_f64(p[i]);
    }
    return NAN;
}

/* ------------------------------------------------------------------------ */
/* attention over a paged cache                                             */
/* ------------------------------------------------------------------------ */

typedef struct {
    /* shared description of one call */
    const void *q, *k_pool, *v_pool;
    int q_dtype, kv_dtype;
    const int32_t* block_tables;
    const int32_t* context_lens;   /* decode: per sequence; prefill: per chunk */
    const int32_t* query_start_loc; /* prefill only, [n_units + 1] */
    double scale, k_scale, v_scale;
    int n_units;                    /* sequences (decode) or chunks (prefill) */
    int n_q, n_kv, d, block_size, max_blocks, num_blocks;
    double* out;
    /* work distribution */
    int next;
    int bad;
    pthread_mutex_t lock;
} orc_job;

/* Address (element index) of K/V element [token t][dim i] for kv head h of a
 * sequence whose block table row is bt: the token lives in physical block
 * bt[t / B] at offset t % B; pools are [num_blocks][n_kv][B][d]. */
static int64_t paged_index(const orc_job* J, const int32_t* bt, int t, int h, int i, int* ok) {
    int32_t blk = bt[t / J->block_size];
    if (blk < 0 || blk >= J->num_blocks) {
        *ok = 0;
        return 0;
    }
    return (((int64_t)blk * J->n_kv + h) * J->block_size + (t % J->block_size)) * J->d + i;
}

/* One query row attending to the first n_keys tokens of a paged sequence:
 * out[i] = sum_t w_t v_t[i] / sum_t w_t with w_t = exp(s_t - max_s),
 * s_t = scale * sum_i q[i] k_t[i].  K and V are first gathered in logical
 * order (token 0 .. n_keys-1); element values are the stored value, times the
 * per-tensor scale for E4M3. */
static int attend_one(const orc_job* J, const int32_t* bt, int kvh, int64_t q_off,
                      int n_keys, double* out_row) {
    const int d = J->d;
    double kmul = (J->kv_dtype == ORC_E4M3) ? J->k_scale : 1.0;
    double vmul = (J->kv_dtype == ORC_E4M3) ? J->v_scale : 1.0;
    if (n_keys <= 0) {
        for (int i = 0; i < d; i++) out_row[i] = 0.0;
        return 1;
    }
    double* q = malloc(sizeof(double) * d);
    double* K = malloc(sizeof(double) * (size_t)n_keys * d);
    double* V = malloc(sizeof(double) * (size_t)n_keys * d);
    double* s = malloc(sizeof(double) * (size_t)n_keys);
    int ok = 1;
    for (int i = 0; i < d; i++) q[i] = load_elem(J->q, J->q_dtype, q_off + i);
    for (int t = 0; t < n_keys && ok; t++)
        for (int i = 0; i < d; i++) {
            int64_t idx = paged_index(J, bt, t, kvh, i, &ok);
            if (!ok) break;
            K[(size_t)t * d + i] = load_elem(J->k_pool, J->kv_dtype, idx) * kmul;
            V[(size_t)t * d + i] = load_elem(J->v_pool, J->kv_dtype, idx) * vmul;
        }
    if (ok) {
        double m = -INFINITY;
        for (int t = 0; t < n_keys; t++) {
            double acc = 0.0;
            for (int i = 0; i < d; i++) acc += q[i] * K[(size_t)t * d + i];
            s[t] = J->scale * acc;
            if (s[t] > m) m = s[t];
        }
        double l = 0.0;
        for (int i = 0; i < d; i++) out_row[i] = 0.0;
        for (int t = 0; t < n_keys; t++) {
            double w = exp(s[t] - m);
            l += w;
            for (int i = 0; i < d; i++) out_row[i] += w * V[(size_t)t * d + i];
        }
        for (int i = 0; i < d; i++) out_row[i] /= l;
    } else {
        for (int i = 0; i < d; i++) out_row[i] = NAN;
    }
    free(q);
    free(K);
    free(V);
    free(s);
    return ok;
}

/* decode: unit u = (sequence, kv head); every q head of the group attends to
 * all context_lens[seq] tokens.  q head h reads kv head h / (n_q / n_kv). */
static int decode_unit(orc_job* J, int u) {
    int seq = u / J->n_kv, kvh = u % J->n_kv;
    int group = J->n_q / J->n_kv;
    const int32_t* bt = J->block_tables + (int64_t)seq * J->max_blocks;
    int ctx = J->context_lens[seq];
    int ok = 1;
    for (int g = 0; g < group; g++) {
        int h = kvh * group + g;
        int64_t row = (int64_t)seq * J->n_q + h;
        ok &= attend_one(J, bt, kvh, row * J->d, ctx, J->out + row * J->d);
    }
    return ok;
}

/* prefill: unit u = (chunk, kv head).  Chunk c owns query rows
 * query_start_loc[c] .. query_start_loc[c+1]-1 (L rows) and its sequence holds
 * context_lens[c] tokens including the chunk, so the history is
 * H = context_lens[c] - L.  Query i of the chunk sits at absolute position
 * H + i and attends to keys 0 .. H + i (causal). */
static int prefill_unit(orc_job* J, int u) {
    int c = u / J->n_kv, kvh = u % J->n_kv;
    int group = J->n_q / J->n_kv;
    const int32_t* bt = J->block_tables + (int64_t)c * J->max_blocks;
    int q0 = J->query_start_loc[c], q1 = J->query_start_loc[c + 1];
    int L = q1 - q0;
    int H = J->context_lens[c] - L;
    int ok = 1;
    if (H < 0) return 0;
    for (int i = 0; i < L; i++)
        for (int g = 0; g < group; g++) {
            int h = kvh * group + g;
            int64_t row = (int64_t)(q0 + i) * J->n_q + h;
            ok &= attend_one(J, bt, kvh, row * J->d, H + i + 1, J->out + row * J->d);
        }
    return ok;
}

typedef int (*unit_fn)(orc_job*, int);
typedef struct {
    orc_job* J;
    unit_fn fn;
} worker_arg;

static void* worker(void* p) {
    worker_arg* a = (worker_arg*)p;
    orc_job* J = a->J;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int u = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->n_units * J->n_kv) break;
        if (!a->fn(J, u)) {
            pthread_mutex_lock(&J->lock);
            J->bad++;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

static int run_units(orc_job* J, unit_fn fn, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    J->next = 0;
    J->bad = 0;
    pthread_mutex_init(&J->lock, NULL);
    worker_arg a = {J, fn};
    if (nthreads == 1) {
        worker(&a);
    } else {
        pthread_t* th = malloc(sizeof(pthread_t) * nthreads);
        for (int i = 0; i < nthreads; i++) pthread_create(&th[i], NULL, worker, &a);
        for (int i = 0; i < nthreads; i++) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J->lock);
    return J->bad;
}

/* Decode attention over the paged cache.  Shapes: q [num_seqs][n_q][d];
 * pools [num_blocks][n_kv][block_size][d]; block_tables [num_seqs][max_blocks];
 * out [num_seqs][n_q][d] (double).  Returns the number of (seq, kv head)
 * units that met an out-of-range block id (their rows are NaN). */
int orc_paged_decode(double* out, const void* q, int q_dtype, const void* k_pool,
                     const void* v_pool, int kv_dtype, const int32_t* block_tables,
                     const int32_t* context_lens, double scale, double k_scale,
                     double v_scale, int num_seqs, int n_q, int n_kv, int d,
                     int block_size, int max_blocks, int num_blocks, int nthreads) {
    orc_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k_pool = k_pool; J.v_pool = v_pool;
    J.q_dtype = q_dtype; J.kv_dtype = kv_dtype;
    J.block_tables = block_tables; J.context_lens = context_lens;
    J.scale = scale; J.k_scale = k_scale; J.v_scale = v_scale;
    J.n_units = num_seqs; J.n_q = n_q; J.n_kv = n_kv; J.d = d;
    J.block_size = block_size; J.max_blocks = max_blocks; J.num_blocks = num_blocks;
    J.out = out;
    return run_units(&J, decode_unit, nthreads);
}

/* Chunked prefill over the paged cache.  q [total_q][n_q][d]; out likewise. */
int orc_paged_prefill(double* out, const void* q, int q_dtype, const void* k_pool,
                      const void* v_pool, int kv_dtype, const int32_t* block_tables,
                      const int32_t* query_start_loc, const int32_t* context_lens,
                      double scale, double k_scale, double v_scale, int n_chunks, int n_q,
                      int n_kv, int d, int block_size, int max_blocks, int num_blocks,
                      int nthreads) {
    orc_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k_pool = k_pool; J.v_pool = v_pool;
    J.q_dtype = q_dtype; J.kv_dtype = kv_dtype;
    J.block_tables = block_tables; J.context_lens = context_lens;
    J.query_start_loc = query_start_loc;
    J.scale = scale; J.k_scale = k_scale; J.v_scale = v_scale;
    J.n_units = n_chunks; J.n_q = n_q; J.n_kv = n_kv; J.d = d;
    J.block_size = block_size; J.max_blocks = max_blocks; J.num_blocks = num_blocks;
    J.out = out;
    return run_units(&J, prefill_unit, nthreads);
}

/* ------------------------------------------------------------------------ */
/* slot write and block copy                                                */
/* ------------------------------------------------------------------------ */

/* Write new K/V rows into their slots.  key/value [num_tokens][n_kv][d] of
 * src_dtype; pools [num_blocks][n_kv][B][d] of cache_dtype.  slot s < 0 means
 * "no slot" (skip); otherwise block s / B, offset s % B.  If the cache dtype
 * equals the source dtype the bytes are copied; if the cache is E4M3 each
 * element is divided by its per-tensor scale in binary32 (the precision the
 * quantised code is decided in) and rounded to E4M3 (nearest-even,
 * saturating).  Returns the number of tokens whose slot was out of range
 * (those are skipped). */
int orc_reshape_and_cache(void* k_pool, void* v_pool, const void* key, const void* value,
                          const int64_t* slot_mapping, int num_tokens, int n_kv, int d,
                          int block_size, int num_blocks, int src_dtype, int cache_dtype,
                          float k_scale, float v_scale) {
    int bad = 0;
    int sb = elem_bytes(src_dtype), cb = elem_bytes(cache_dtype);
    for (int t = 0; t < num_tokens; t++) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t blk = slot / block_size, off = slot % block_size;
        if (blk >= num_blocks) {
            bad++;
            continue;
        }
        for (int h = 0; h < n_kv; h++)
            for (int i = 0; i < d; i++) {
                int64_t src = ((int64_t)t * n_kv + h) * d + i;
                int64_t dst = ((blk * n_kv + h) * block_size + off) * d + i;
                if (cache_dtype == src_dtype) {
                    memcpy((uint8_t*)k_pool + dst * cb, (const uint8_t*)key + src * sb, sb);
                    memcpy((uint8_t*)v_pool + dst * cb, (const uint8_t*)value + src * sb, sb);
                } else if (cache_dtype == ORC_E4M3) {
                    float kx = (float)load_elem(key, src_dtype, src);   /* exact */
                    float vx = (float)load_elem(value, src_dtype, src); /* exact */
                    float kq = kx / k_scale;
                    float vq = vx / v_scale;
                    ((uint8_t*)k_pool)[dst] = orc_f32_to_e4m3_satfinite(kq);
                    ((uint8_t*)v_pool)[dst] = orc_f32_to_e4m3_satfinite(vq);
                } else {
                    return -1;
                }
            }
    }
    return bad;
}

/* Copy whole blocks (all kv heads, K and V): for each pair (src, dst) the dst
 * block's bytes become the src block's bytes.  Returns the number of pairs
 * skipped because an id was out of range. */
int orc_copy_blocks(void* k_pool, void* v_pool, const int64_t* pairs, int n_pairs, int n_kv,
                    int d, int block_size, int num_blocks, int dtype) {
    int bad = 0;
    size_t bytes = (size_t)n_kv * block_size * d * elem_bytes(dtype);
    for (int p = 0; p < n_pairs; p++) {
        int64_t s = pairs[2 * p], t = pairs[2 * p + 1];
        if (s < 0 || s >= num_blocks || t < 0 || t >= num_blocks) {
            bad++;
            continue;
        }
        memmove((uint8_t*)k_pool + t * bytes, (uint8_t*)k_pool + s * bytes, bytes);
        memmove((uint8_t*)v_pool + t * bytes, (uint8_t*)v_pool + s * bytes, bytes);
    }
    return bad;
}

/* Swap: copy whole blocks between two pools -- a GPU pool and a host pool,
 * in either direction -- when a preempted request's KV cache is moved out
 * and back ("vLLM explained", the table in "KV cache 什麼時候可以被覆蓋": when
 * memory runs short, preempt by recomputation or by swapping to the CPU).
 * For each pair (src, dst), block dst of the destination pools becomes a
 * byte copy of block src of the source pools.  Pairs with an id out of range
 * are skipped and counted. */
int orc_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                    const int64_t* pairs, int n_pairs, int n_kv, int d, int block_size,
                    int src_num_blocks, int dst_num_blocks, int dtype) {
    int bad = 0;
    size_t bytes = (size_t)n_kv * block_size * d * elem_bytes(dtype);
    for (int p = 0; p < n_pairs; p++) {
        int64_t s = pairs[2 * p], t = pairs[2 * p + 1];
        if (s < 0 || s >= src_num_blocks || t < 0 || t >= dst_num_blocks) {
            bad++;
            continue;
        }
        memcpy((uint8_t*)dst_k + t * bytes, (const uint8_t*)src_k + s * bytes, bytes);
        memcpy((uint8_t*)dst_v + t * bytes, (const uint8_t*)src_v + s * bytes, bytes);
    }
    return bad;
}

/* ------------------------------------------------------------------------ */
/* array forms of the format routines (for exhaustive tests)                */
/* ------------------------------------------------------------------------ */

void orc_decode_array(int dtype, const void* src, double* dst, int64_t n) {
    for (int64_t i = 0; i < n; i++) dst[i] = load_elem(src, dtype, i);
}

void orc_encode_e4m3_array(const float* src, uint8_t* dst, int64_t n) {
    for (int64_t i = 0; i < n; i++) dst[i] = orc_f32_to_e4m3_satfinite(src[i]);
}

void orc_encode_bf16_array(const double* src, uint16_t* dst, int64_t n) {
    for (int64_t i = 0; i < n; i++) dst[i] = orc_f64_to_bf16(src[i]);
}

void orc_encode_f16_array(const double* src, uint16_t* dst, int64_t n) {
    for (int64_t i = 0; i < n; i++) dst[i] = orc_f64_to_f16(src[i]);
}
