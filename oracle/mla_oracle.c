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
typedef struct {
    const uint16_t *q, *kv;
    int64_t num_blocks;
    const int32_t *block_table;
    int64_t bt_stride;
    const int32_t *seqlens;
    int batch, s_q, h_q, causal;
    double scale;
    double *out, *lse;
    const int32_t *tasks; /* optional list of (b, t, h) triples */
    int64_t ntasks;
    int64_t next;         /* shared work counter */
    pthread_mutex_t lock;
    int error;
} dec_job;

static int one_row(dec_job *J, int b, int t, int h, double *scores, double *acc) {
    const int rows = J->s_q * J->h_q;
    const int r = t * J->h_q + h;
    double *o = J->out + ((size_t)b * rows + r) * OR_D_V;
    double *lse = J->lse + ((size_t)b * J->h_q + h) * J->s_q + t;
    const uint16_t *qrow = J->q + ((size_t)b * rows + r) * OR_D_QK;

    int64_t n = J->seqlens[b] > 0 ? J->seqlens[b] : 0;
    int64_t V = n;
    if (J->causal) {
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

    double m = -INFINITY;
    for (int64_t j = 0; j < V; ++j) {
        int32_t phys = J->block_table[(size_t)b * J->bt_stride + j / OR_BLK];
        if (phys < 0 || phys >= J->num_blocks) return -1;
        const uint16_t *key = J->kv + ((size_t)phys * OR_BLK + (size_t)(j % OR_BLK)) * OR_D_QK;
        double dot = 0.0;
        for (int d = 0; d < OR_D_QK; ++d) dot += qd[d] * bf16_bits_to_double(key[d]);
        scores[j] = J->scale * dot;
        if (scores[j] > m) m = scores[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j < V; ++j) sum += exp(scores[j] - m);
    double L = m + log(sum);
    for (int d = 0; d < OR_D_V; ++d) acc[d] = 0.0;
    for (int64_t j = 0; j < V; ++j) {
        int32_t phys = J->block_table[(size_t)b * J->bt_stride + j / OR_BLK];
        const uint16_t *val = J->kv + ((size_t)phys * OR_BLK + (size_t)(j % OR_BLK)) * OR_D_QK;
        double p = exp(scores[j] - L);
        for (int d = 0; d < OR_D_V; ++d) acc[d] += p * bf16_bits_to_double(val[d]);
    }
    for (int d = 0; d < OR_D_V; ++d) o[d] = acc[d];
    *lse = L;
    return 0;
}

static void *dec_worker(void *arg) {
    dec_job *J = (dec_job *)arg;
    int64_t maxlen = 0;
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
int oracle_decode(const uint16_t *q, const uint16_t *kv_cache, int64_t num_blocks,
                  const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                  int batch, int s_q, int h_q, double scale, int causal, double *out,
                  double *lse, const int32_t *tasks, int64_t ntasks, int nthreads) {
    if (!q || !kv_cache || !block_table || !seqlens || !out || !lse) return -1;
    if (batch < 0 || s_q < 1 || h_q < 1 || nthreads < 1 || num_blocks < 0) return -1;
    if (tasks && ntasks < 0) return -1;
    for (int b = 0; b < batch; ++b) {
        int64_t n = seqlens[b] > 0 ? seqlens[b] : 0;
        if ((n + OR_BLK - 1) / OR_BLK > bt_stride) return -1;
    }
    dec_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.kv = kv_cache; J.num_blocks = num_blocks; J.block_table = block_table;
    J.bt_stride = bt_stride; J.seqlens = seqlens; J.batch = batch; J.s_q = s_q;
    J.h_q = h_q; J.causal = causal; J.scale = scale; J.out = out; J.lse = lse;
    J.tasks = tasks; J.ntasks = ntasks; J.next = 0; J.error = 0;
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
