/*
 * oracle/mla_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU restatement of MLA decode attention over a
 * paged latent KV cache, and of the split-KV work partition. Only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg may load this library; the
 * product path (the CUDA library and its Python binding) never calls it and shares
 * no code, header, table or constant with it.
 *
 * Sources (the pages are scraped web articles; the attention formula itself is
 * written on none of them, so the plain reading is used and stated below):
 *   [INFRA] "Deep analysis of the DeepSeek Infra open-source releases"
 *           (jingzhunhuoke.net/55333.html), section "DAY1 FlashMLA":
 *             - glossary: MLA is DeepSeek-V2's attention that replaces GQA; FlashMLA is
 *               a FlashAttention-style CUDA kernel for it;
 *             - feature (2): the KV cache is cut into blocks of 64 tokens;
 *             - feature (4): the kernel runs "Gemm1" (scores) then "Gemm2" (weighted
 *               values) over the same loaded Q/K/V;
 *             - feature (5): inputs of very different lengths are load-balanced.
 *   Task statement of this library: keys are the full 576-d latent vectors, values are
 *   their first 512 dims, one latent per token shared by all heads, `scale` applied to
 *   q.k before the softmax, fp32-or-better softmax, `out[b,s_q,h_q,512]`,
 *   `lse[b,h_q,s_q]` (natural log).
 *
 * Precision: every product and sum is taken in double from exactly up-converted
 * bf16 inputs; the outputs are doubles (never rounded to bf16 here).
 *
 * The fp8 cache (oracle_decode_fp8) holds, per token, 512 latent dims as OCP E4M3 bytes
 * and the 64 rotary dims as bf16; a latent byte x stands for kv_scale * e4m3(x). Keys
 * and values are those dequantized vectors; everything after that is the same
 * attention, in double.
 *
 * Sparse mode (oracle_decode_sparse): query row (b, t, h) attends only to the keys at the
 * positions listed for query token t of sequence b (shared by its heads); entries outside the
 * sequence are no key. Pinned in tests/test_oracle_sparse.py (the full list in order is the
 * dense decode bit for bit; list order and invalid entries change nothing; one key, no key;
 * a library SDPA over the gathered keys).
 *
 * Parity pins (see tests/test_oracle*.py): dense non-paged brute force through a
 * library softmax-attention routine, single-token sequences, block-permutation
 * invariance, lse against a library log-sum-exp, q = 0 closed form, NaN-poisoned
 * tails, causal reduction to shorter non-causal sequences, and a hand-worked
 * partition example for the metadata.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_D_QK 576 /* 512 latent + 64 rotary dims: the whole vector is the key */
#define OR_D_V 512  /* the value is the first 512 dims of the same vector      */
#define OR_BLK 64   /* tokens per cache block [INFRA, DAY1 FlashMLA, feature (2)] */

/* bf16 -> double, exact: a bf16 is the top half of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point (OFP8), format E4M3, exactly: bit 7 sign, bits 6..3
 * exponent field E (bias 7), bits 2..0 mantissa M. E = 0: (M / 8) * 2^-6
 * (subnormal; M = 0 is a signed zero). E = 15 and M = 7: NaN. Otherwise
 * (1 + M / 8) * 2^(E - 7); the largest finite magnitude is 1.75 * 2^8 = 448. There
 * are no infinities. */
static double e4m3_to_double(uint8_t x) {
    const int sign = x >> 7, e = (x >> 3) & 15, m = x & 7;
    double v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* ------------------------------------------------------------------------- */
/* Work partition (split-KV metadata), written out by brute force over every  */
/* (sequence, block) pair.                                                    */
/*                                                                            */
/* Reading of [INFRA, DAY1 FlashMLA, feature (5)] ("dynamic load balancing of  */
/* inputs of different length"; the page defers the details to the code):     */
/* lay the sequences end to end on a line of work units; sequence i with       */
/* w_i = ceil(n_i/64) > 0 blocks occupies C "start-up" units followed by one   */
/* unit per block (sequences with no tokens occupy nothing). With U units in   */
/* all and P parts, T = max(1, ceil(U/P)); a block at unit u belongs to part   */
/* floor(u/T). Each part is a contiguous run of (sequence, block) pairs; a     */
/* sequence whose blocks fall into k > 1 parts is computed as k pieces whose    */
/* partial results are merged afterwards.                                     */
/*                                                                            */
/* Output layout per part p (8 int32): begin_seq, begin_blk, end_seq (inclusive),*/
/* end_blk (exclusive, within end_seq), index of the part's first piece within  */
/* its sequence, 0, 0, 0. An empty part is {0, 0, -1, 0, 0, 0, 0, 0}.          */
/* num_splits_cum[0] = 0, num_splits_cum[i+1] = num_splits_cum[i] + (number of   */
/* parts that hold blocks of sequence i).                                     */
/* Returns 0, or -1 on bad arguments.                                          */
/* ------------------------------------------------------------------------- */
int oracle_metadata(const int32_t *seqlens, int batch, int num_parts, int fixed_cost,
                    int32_t *tile_meta, int32_t *num_splits_cum) {
    if (batch < 0 || num_parts < 1 || fixed_cost < 0 || !tile_meta || !num_splits_cum)
        return -1;
    if (batch > 0 && !seqlens) return -1;

    /* total units U */
    int64_t U = 0;
    for (int i = 0; i < batch; ++i) {
        int64_t n = seqlens[i] > 0 ? seqlens[i] : 0;
        int64_t w = (n + OR_BLK - 1) / OR_BLK;
        if (w > 0) U += fixed_cost + w;
    }
    int64_t T = (U + num_parts - 1) / num_parts;
    if (T < 1) T = 1;

    for (int p = 0; p < num_parts; ++p) {
        int32_t *m = tile_meta + 8 * (size_t)p;
        m[0] = 0; m[1] = 0; m[2] = -1; m[3] = 0; m[4] = 0; m[5] = 0; m[6] = 0; m[7] = 0;
    }
    char *seen = (char *)calloc((size_t)num_parts, 1);
    if (!seen) return -1;

    num_splits_cum[0] = 0;
    int64_t unit = 0; /* unit position of the current sequence's first unit */
    for (int i = 0; i < batch; ++i) {
        int64_t n = seqlens[i] > 0 ? seqlens[i] : 0;
        int64_t w = (n + OR_BLK - 1) / OR_BLK;
        int parts_of_seq = 0;
        int64_t prev_part = -1, first_part = -1;
        if (w > 0) {
            for (int64_t k = 0; k < w; ++k) {
                int64_t u = unit + fixed_cost + k;
                int64_t p = u / T;
                int32_t *m = tile_meta + 8 * (size_t)p;
                if (first_part < 0) first_part = p;
                if (p != prev_part) {
                    ++parts_of_seq;
                    prev_part = p;
                }
                if (!seen[p]) { /* first block of this part, in walk order */
                    seen[p] = 1;
                    m[0] = i;
                    m[1] = (int32_t)k;
                    m[4] = (int32_t)(p - first_part);
                }
                m[2] = i;              /* last block seen so far in this part */
                m[3] = (int32_t)(k + 1);
            }
            unit += fixed_cost + w;
        }
        num_splits_cum[i + 1] = num_splits_cum[i] + parts_of_seq;
    }
    free(seen);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Decode attention.                                                           */
/*                                                                            */
/* For batch b, query token t in [0, s_q), head h:                             */
/*   n = seqlens[b]; visible keys V = causal ? clamp(n - s_q + t + 1, 0, n) : n */
/*   key j (j < V) = kv_cache[block_table[b][j / 64]][j % 64][0][0:576]         */
/*   s_j = scale * sum_{d<576} q[b][t][h][d] * key_j[d]                          */
/*   lse[b][h][t] = log(sum_j exp(s_j))   (taken as m + log sum exp(s_j - m))   */
/*   out[b][t][h][d] = sum_j exp(s_j - lse) * key_j[d],  d < 512                 */
/*   V == 0: out = 0, lse = -inf.                                              */
/* The causal reading (task statement: "causal masking between the query       */
/* tokens"): the s_q query tokens are the last s_q tokens of the sequence, so  */
/* query t sees keys 0 .. n - s_q + t.                                          */
/* Only the first ceil(V/64) block-table entries of a row are read; the other */
/* entries and the cache rows past V are never touched.                        */
/* ------------------------------------------------------------------------- */
#define OR_F8_REC 640 /* fp8 cache: bytes per token (512 E4M3 + 64 bf16) */

typedef struct {
    const uint16_t *q, *kv;
    const uint8_t *kv8; /* fp8 cache (kv == NULL), with its latent scale */
    double kv_scale;
    double f8val[256];  /* fp8 cache: kv_scale * e4m3_to_double(code) for every code (the same values,
                           computed once instead of once per element) */
    int64_t num_blocks;
    const int32_t *block_table;
    int64_t bt_stride;
    const int32_t *seqlens;
    int batch, s_q, h_q, causal;
    double scale;
    double *out, *lse;
    const int32_t *tasks; /* optional list of (b, t, h) triples */
    const int32_t *indices; /* sparse mode: int32[b, s_q, topk] key positions (NULL: dense) */
    int topk;
    int64_t ntasks;
    int64_t next;         /* shared work counter */
    pthread_mutex_t lock;
    int error;
} dec_job;

/* The 576 dims of cache row `row` (physical block * 64 + slot) as doubles. */
static void load_key(const dec_job *J, int64_t row, double *k) {
    if (J->kv) {
        const uint16_t *src = J->kv + (size_t)row * OR_D_QK;
        for (int d = 0; d < OR_D_QK; ++d) k[d] = bf16_bits_to_double(src[d]);
    } else {
        const uint8_t *src = J->kv8 + (size_t)row * OR_F8_REC;
        for (int d = 0; d < OR_D_V; ++d) k[d] = J->f8val[src[d]];
        for (int d = OR_D_V; d < OR_D_QK; ++d) {
            const uint8_t *r = src + OR_D_V + 2 * (d - OR_D_V); /* little-endian bf16 */
            k[d] = bf16_bits_to_double((uint16_t)(r[0] | (r[1] << 8)));
        }
    }
}

static int one_row(dec_job *J, int b, int t, int h, double *scores, double *acc) {
    const int rows = J->s_q * J->h_q;
    const int r = t * J->h_q + h;
    double *o = J->out + ((size_t)b * rows + r) * OR_D_V;
    double *lse = J->lse + ((size_t)b * J->h_q + h) * J->s_q + t;
    const uint16_t *qrow = J->q + ((size_t)b * rows + r) * OR_D_QK;

    int64_t n = J->seqlens[b] > 0 ? J->seqlens[b] : 0;
    int64_t V = n;
    const int32_t *list = NULL; /* sparse mode: key i of this row is token list[i] (skipped unless in [0, n)) */
    if (J->indices) {
        list = J->indices + ((size_t)b * J->s_q + t) * J->topk;
        V = J->topk;
    } else if (J->causal) {
        V = n - J->s_q + t + 1;
        if (V < 0) V = 0;
        if (V > n) V = n;
    }
    if (V == 0) {
        for (int d = 0; d < OR_D_V; ++d) o[d] = 0.0;
        *lse = -INFINITY;
        return 0;
    }
    double qd[OR_D_QK];
    for (int d = 0; d < OR_D_QK; ++d) qd[d] = bf16_bits_to_double(qrow[d]);

    double m = -INFINITY, key[OR_D_QK];
    for (int64_t j = 0; j < V; ++j) {
        const int64_t pos = list ? (int64_t)list[j] : j;
        if (pos < 0 || pos >= n) { /* sparse mode: an entry outside the sequence is no key */
            scores[j] = -INFINITY;
            continue;
        }
        int32_t phys = J->block_table[(size_t)b * J->bt_stride + pos / OR_BLK];
        if (phys < 0 || phys >= J->num_blocks) return -1;
        load_key(J, (int64_t)phys * OR_BLK + pos % OR_BLK, key);
        double dot = 0.0;
        for (int d = 0; d < OR_D_QK; ++d) dot += qd[d] * key[d];
        scores[j] = J->scale * dot;
        if (scores[j] > m) m = scores[j];
    }
    if (m == -INFINITY) { /* no valid key */
        for (int d = 0; d < OR_D_V; ++d) o[d] = 0.0;
        *lse = -INFINITY;
        return 0;
    }
    double sum = 0.0;
    for (int64_t j = 0; j < V; ++j) sum += exp(scores[j] - m);
    double L = m + log(sum);
    for (int d = 0; d < OR_D_V; ++d) acc[d] = 0.0;
    for (int64_t j = 0; j < V; ++j) {
        if (scores[j] == -INFINITY) continue;
        const int64_t pos = list ? (int64_t)list[j] : j;
        int32_t phys = J->block_table[(size_t)b * J->bt_stride + pos / OR_BLK];
        load_key(J, (int64_t)phys * OR_BLK + pos % OR_BLK, key); /* the value is its first 512 dims */
        double p = exp(scores[j] - L);
        for (int d = 0; d < OR_D_V; ++d) acc[d] += p * key[d];
    }
    for (int d = 0; d < OR_D_V; ++d) o[d] = acc[d];
    *lse = L;
    return 0;
}

static void *dec_worker(void *arg) {
    dec_job *J = (dec_job *)arg;
    int64_t maxlen = J->indices ? J->topk : 0;
    for (int b = 0; b < J->batch; ++b)
        if (J->seqlens[b] > maxlen) maxlen = J->seqlens[b];
    double *scores = (double *)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
    double *acc = (double *)malloc(sizeof(double) * OR_D_V);
    if (!scores || !acc) {
        pthread_mutex_lock(&J->lock);
        J->error = -2;
        pthread_mutex_unlock(&J->lock);
        free(scores);
        free(acc);
        return NULL;
    }
    const int64_t total = J->tasks ? J->ntasks : (int64_t)J->batch * J->s_q * J->h_q;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t i = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (i >= total) break;
        int b, t, h;
        if (J->tasks) {
            b = J->tasks[3 * i];
            t = J->tasks[3 * i + 1];
            h = J->tasks[3 * i + 2];
            if (b < 0 || b >= J->batch || t < 0 || t >= J->s_q || h < 0 || h >= J->h_q) {
                pthread_mutex_lock(&J->lock);
                J->error = -1;
                pthread_mutex_unlock(&J->lock);
                continue;
            }
        } else {
            b = (int)(i / ((int64_t)J->s_q * J->h_q));
            int64_t rem = i % ((int64_t)J->s_q * J->h_q);
            t = (int)(rem / J->h_q);
            h = (int)(rem % J->h_q);
        }
        if (one_row(J, b, t, h, scores, acc) != 0) {
            pthread_mutex_lock(&J->lock);
            J->error = -3;
            pthread_mutex_unlock(&J->lock);
        }
    }
    free(scores);
    free(acc);
    return NULL;
}

/*
 * Computes out (double[b, s_q, h_q, 512]) and lse (double[b, h_q, s_q]) for every
 * row, or, when `tasks` is non-NULL, only for the listed (b, t, h) triples (the other
 * entries of out/lse are left untouched). Uses `nthreads` POSIX threads (>= 1).
 * Returns 0; -1 bad arguments; -2 out of memory; -3 a block-table entry that must be
 * read is outside [0, num_blocks).
 */
static int run_decode(const uint16_t *q, const uint16_t *kv_cache, const uint8_t *kv8, double kv_scale,
                      int64_t num_blocks, const int32_t *block_table, int64_t bt_stride,
                      const int32_t *seqlens, int batch, int s_q, int h_q, double scale, int causal,
                      double *out, double *lse, const int32_t *tasks, int64_t ntasks, int nthreads) {
    if (!q || (!kv_cache && !kv8) || !block_table || !seqlens || !out || !lse) return -1;
    if (batch < 0 || s_q < 1 || h_q < 1 || nthreads < 1 || num_blocks < 0) return -1;
    if (tasks && ntasks < 0) return -1;
    for (int b = 0; b < batch; ++b) {
        int64_t n = seqlens[b] > 0 ? seqlens[b] : 0;
        if ((n + OR_BLK - 1) / OR_BLK > bt_stride) return -1;
    }
    dec_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.kv = kv_cache; J.kv8 = kv8; J.kv_scale = kv_scale; J.num_blocks = num_blocks; J.block_table = block_table;
    J.bt_stride = bt_stride; J.seqlens = seqlens; J.batch = batch; J.s_q = s_q;
    J.h_q = h_q; J.causal = causal; J.scale = scale; J.out = out; J.lse = lse;
    J.tasks = tasks; J.ntasks = ntasks; J.next = 0; J.error = 0;
    if (kv8)
        for (int c = 0; c < 256; ++c) J.f8val[c] = kv_scale * e4m3_to_double((uint8_t)c);
    pthread_mutex_init(&J.lock, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -2;
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, dec_worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) dec_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return J.error;
}

int oracle_decode(const uint16_t *q, const uint16_t *kv_cache, int64_t num_blocks,
                  const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                  int batch, int s_q, int h_q, double scale, int causal, double *out,
                  double *lse, const int32_t *tasks, int64_t ntasks, int nthreads) {
    if (!kv_cache) return -1;
    return run_decode(q, kv_cache, NULL, 0.0, num_blocks, block_table, bt_stride, seqlens, batch, s_q,
                      h_q, scale, causal, out, lse, tasks, ntasks, nthreads);
}

/*
 * The same attention over the fp8 cache: kv8 is uint8[num_blocks, 64, 640], per token
 * 512 E4M3 latent bytes (value kv_scale * e4m3(byte)) then 64 bf16 rotary dims
 * (little-endian). Arguments and return codes as oracle_decode.
 */
int oracle_decode_fp8(const uint16_t *q, const uint8_t *kv8, double kv_scale, int64_t num_blocks,
                      const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                      int batch, int s_q, int h_q, double scale, int causal, double *out,
                      double *lse, const int32_t *tasks, int64_t ntasks, int nthreads) {
    if (!kv8) return -1;
    return run_decode(q, NULL, kv8, kv_scale, num_blocks, block_table, bt_stride, seqlens, batch, s_q,
                      h_q, scale, causal, out, lse, tasks, ntasks, nthreads);
}

/* E4M3 byte -> double, for the tests that pin the decoding itself. */
void oracle_e4m3_decode(const uint8_t *x, int64_t n, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_to_double(x[i]);
}

/* ------------------------------------------------------------------------- */
/* Appending new tokens to the paged cache (the step that precedes decode).     */
/*                                                                            */
/* Token t of sequence b's new tokens goes to position p = seqlens[b] + t of   */
/* the sequence: cache row block_table[b][p / 64] * 64 + p % 64. bf16 cache:   */
/* the 576 bf16 values are copied. fp8 cache: each latent value x (bf16,      */
/* exactly a float) is multiplied by inv_scale in fp32 and written as the E4M3 */
/* code of the product, rounded to nearest (ties to even) and saturated to    */
/* +-448 (infinities too); NaN stays NaN; the rotary dims are copied as bf16.  */
/* Returns 0, or -1 when a row would land outside the table or the cache.      */
/* ------------------------------------------------------------------------- */

/* fp32 -> E4M3 code, round to nearest even, saturating (OCP OFP8 E4M3, see e4m3_to_double). */
static uint8_t e4m3_from_float(float v) {
    uint32_t u;
    memcpy(&u, &v, sizeof u);
    const uint8_t sign = (uint8_t)((u >> 31) << 7);
    if (isnan(v)) return (uint8_t)(sign | 0x7F);
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    /* the spacing of E4M3 values around a: 2^-9 below 2^-6 (subnormals), else 2^(e - 3) */
    int e;
    frexp(a, &e);          /* a = f * 2^e, f in [0.5, 1): the leading bit is 2^(e-1) */
    int lead = e - 1;      /* a in [2^lead, 2^(lead+1)) */
    if (lead < -6) lead = -6;
    const double quantum = ldexp(1.0, lead - 3);
    double q = a / quantum; /* exact: a power-of-two scaling */
    double fl = floor(q), rem = q - fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
    const double r = fl * quantum; /* the rounded magnitude; may step up to the next binade */
    if (r >= 448.0) return (uint8_t)(sign | 0x7E);
    if (r == 0.0) return sign;
    int re;
    frexp(r, &re);
    int rlead = re - 1;
    if (rlead < -6) { /* subnormal: r = m * 2^-9 */
        const int m = (int)(r / ldexp(1.0, -9));
        return (uint8_t)(sign | m);
    }
    const int E = rlead + 7;
    const int m = (int)((r / ldexp(1.0, rlead) - 1.0) * 8.0);
    return (uint8_t)(sign | (E << 3) | m);
}

void oracle_e4m3_encode(const float *x, int64_t n, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_from_float(x[i]);
}

static int append_rows(const uint16_t *new_kv, int n_new, uint16_t *kv, uint8_t *kv8, float inv_scale,
                       int64_t num_blocks, const int32_t *block_table, int64_t bt_stride,
                       const int32_t *seqlens, int batch) {
    if (!new_kv || (!kv && !kv8) || !block_table || !seqlens || n_new < 0 || batch < 0) return -1;
    for (int b = 0; b < batch; ++b) {
        for (int t = 0; t < n_new; ++t) {
            const int64_t pos = (int64_t)(seqlens[b] > 0 ? seqlens[b] : 0) + t;
            if (pos / OR_BLK >= bt_stride) return -1;
            const int32_t phys = block_table[(size_t)b * bt_stride + pos / OR_BLK];
            if (phys < 0 || phys >= num_blocks) return -1;
            const int64_t row = (int64_t)phys * OR_BLK + pos % OR_BLK;
            const uint16_t *src = new_kv + ((size_t)b * n_new + t) * OR_D_QK;
            if (kv) {
                memcpy(kv + (size_t)row * OR_D_QK, src, OR_D_QK * sizeof(uint16_t));
            } else {
                uint8_t *dst = kv8 + (size_t)row * OR_F8_REC;
                for (int d = 0; d < OR_D_V; ++d) {
                    const float x = (float)bf16_bits_to_double(src[d]);
                    dst[d] = e4m3_from_float(x * inv_scale); /* one fp32 multiply, then the rounding */
                }
                for (int d = OR_D_V; d < OR_D_QK; ++d) {
                    dst[OR_D_V + 2 * (d - OR_D_V)] = (uint8_t)(src[d] & 0xFF);
                    dst[OR_D_V + 2 * (d - OR_D_V) + 1] = (uint8_t)(src[d] >> 8);
                }
            }
        }
    }
    return 0;
}

int oracle_append(const uint16_t *new_kv, int n_new, uint16_t *kv_cache, int64_t num_blocks,
                  const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens, int batch) {
    if (!kv_cache) return -1;
    return append_rows(new_kv, n_new, kv_cache, NULL, 0.f, num_blocks, block_table, bt_stride, seqlens, batch);
}

int oracle_append_fp8(const uint16_t *new_kv, int n_new, uint8_t *kv8, float inv_scale, int64_t num_blocks,
                      const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens, int batch) {
    if (!kv8) return -1;
    return append_rows(new_kv, n_new, NULL, kv8, inv_scale, num_blocks, block_table, bt_stride, seqlens, batch);
}

/*
 * Sparse mode: query row (b, t, h) attends only to the keys at the positions
 * indices[b][t][0 .. topk) of sequence b (shared by every head of that query token). An entry
 * outside [0, seqlens[b]) is no key; an entry listed twice counts twice; a row with no valid
 * entry gives out = 0, lse = -inf. No causal mask (the list decides). bf16 cache; other
 * arguments and return codes as oracle_decode.
 */
int oracle_decode_sparse(const uint16_t *q, const uint16_t *kv_cache, int64_t num_blocks,
                         const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                         const int32_t *indices, int topk, int batch, int s_q, int h_q, double scale,
                         double *out, double *lse, int nthreads) {
    if (!q || !kv_cache || !block_table || !seqlens || !indices || !out || !lse) return -1;
    if (batch < 0 || s_q < 1 || h_q < 1 || nthreads < 1 || num_blocks < 0 || topk < 0) return -1;
    for (int b = 0; b < batch; ++b) {
        int64_t n = seqlens[b] > 0 ? seqlens[b] : 0;
        if ((n + OR_BLK - 1) / OR_BLK > bt_stride) return -1;
    }
    dec_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.kv = kv_cache; J.num_blocks = num_blocks; J.block_table = block_table;
    J.bt_stride = bt_stride; J.seqlens = seqlens; J.batch = batch; J.s_q = s_q; J.h_q = h_q;
    J.causal = 0; J.scale = scale; J.out = out; J.lse = lse; J.indices = indices; J.topk = topk;
    pthread_mutex_init(&J.lock, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -2;
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, dec_worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) dec_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return J.error;
}

