/*
 * mla.h -- C ABI of the B200 (sm_100a) MLA decode-attention library.
 *
 * What is computed. Multi-head Latent Attention (MLA) decoding over a paged latent
 * KV cache. MLA is the attention of DeepSeek-V2 that replaces GQA, and FlashMLA is a
 * FlashAttention-style CUDA kernel for it ("Deep analysis of the DeepSeek Infra
 * open-source releases", jingzhunhuoke.net/55333.html, section "DAY1 FlashMLA",
 * glossary). Every query head attends over ONE shared 576-d latent vector per token
 * (512 compressed dims + 64 rotary dims). The key is the whole 576-d vector, the value
 * is its first 512 dims. The cache is stored in blocks of 64 tokens (same section,
 * feature (2)) addressed through a per-sequence block table. For batch b, query token
 * t, head h (row r = t*h_q + h):
 *     n  = seqlens[b]
 *     V  = causal ? clamp(n - s_q + t + 1, 0, n) : n        (visible keys)
 *     k_j = kv_cache[block_table[b*bt_stride + j/64]][j%64][0][0:576],  j < V
 *     s_j = scale * <q[b][t][h][:], k_j>
 *     lse[b][h][t]       = log(sum_j exp(s_j))               (natural log)
 *     out[b][t][h][0:512] = sum_j exp(s_j - lse) * k_j[0:512]
 *     V == 0  ->  out = 0, lse = -inf
 * The pages do not write this formula out; it is the standard scaled-softmax reading.
 * The query tokens of one sequence are its last s_q tokens under causal masking.
 *
 * How. Two steps on the caller's stream:
 *   1. mla_get_metadata: a length-aware split of all (sequence, 64-token block) work
 *      into `num_parts` contiguous parts (same section, feature (5): inputs of very
 *      different lengths are load-balanced). A sequence that spans k > 1 parts is
 *      computed as k pieces.
 *   2. mla_decode: a persistent kernel walks each part (one 2-CTA cluster per part and
 *      group of 128 query rows): TMA gathers of block-table-addressed KV tiles into a
 *      shared-memory ring, QK^T ("Gemm1") and PV ("Gemm2") as tcgen05 MMAs with TMEM
 *      accumulators (same section, feature (4)), an fp32 online softmax; pieces of
 *      split sequences leave fp32 partial outputs + lse in the workspace, and a
 *      combine kernel merges them by log-sum-exp.
 * Around it: mla_decode_fp8 reads an FP8 (E4M3) latent cache instead; mla_decode_sparse
 * attends each query token to a list of cache positions (top-k) instead of its whole
 * sequence; mla_append_kv / mla_append_kv_fp8 write new tokens into the cache;
 * mla_head_gemm computes the per-head projections on either side (the absorbed q_nope W_UK
 * and o_latent W_UV); mla_decode_host and mla_decode_noalloc are conveniences over
 * mla_decode.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers unless the name says host. All device buffers are
 *     owned by the caller; the library allocates no device memory. It keeps only a
 *     small host-side cache of TMA descriptors keyed by (kv_cache, num_blocks, format).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     asynchronous unless stated; nothing is synchronised implicitly.
 *   - Inputs are never written (the cache appends write the cache, their output). Arguments
 *     are validated on the host BEFORE any launch;
 *     an invalid call returns a non-zero mla_status and launches nothing.
 *   - Kernels never trap. A block-table entry outside [0, num_blocks) or a pipeline
 *     wait that exceeds its iteration bound, or a row outside the decode's numeric range
 *     (MLA_ERR_RANGE), sets a per-device error word; the affected outputs are then
 *     unspecified. mla_check_status() reports and clears it.
 *   - Thread safety: calls on different streams may run concurrently; the TMA
 *     descriptor cache is guarded by a mutex.
 */
#ifndef MLA_DECODE_B200_MLA_H_
#define MLA_DECODE_B200_MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_D_QK 576          /* key width: 512 latent + 64 rotary dims        */
#define MLA_D_V 512           /* value width: the first 512 dims of the key    */
#define MLA_BLOCK_TOKENS 64   /* tokens per cache block                        */
#define MLA_TILE_META_INTS 8  /* int32 per part in tile_meta                   */
#define MLA_MAX_ROWS 1024     /* max s_q * h_q per call                        */
#define MLA_MAX_BATCH 65536   /* max batch per call                            */
#define MLA_FP8_RECORD_BYTES 640 /* fp8 cache: bytes per token (512 E4M3 + 64 bf16) */

typedef enum mla_status {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, size out of range        */
    MLA_ERR_UNSUPPORTED = 2, /* device is not sm_100 / shape not supported        */
    MLA_ERR_WORKSPACE = 3,   /* workspace smaller than mla_workspace_bytes()      */
    MLA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed                 */
    MLA_ERR_TIMEOUT = 5,     /* a device pipeline wait hit its bound (reported by mla_check_status) */
    MLA_ERR_BOUNDS = 6,      /* a block-table entry outside [0, num_blocks) was needed */
    MLA_ERR_RANGE = 7        /* a value outside the range of an internal fp16 form: an fp8-cache
                                query value, or a row's partial-score factors (see mla_decode);
                                reported by mla_check_status */
} mla_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *mla_status_string(int status);

/*
 * Default number of parts for the decode kernel on `device`: one part per 2-SM cluster
 * per group of 128 query rows, i.e. floor(SMs / 2) / ceil(s_q*h_q / 128), at least 1.
 * Host only (queries the SM count). Returns MLA_OK and writes *num_parts.
 */
int mla_default_num_parts(int device, int h_q, int s_q, int *num_parts);

/* Default per-piece start-up cost, in 64-token-block units, used by the partition. */
int mla_default_fixed_cost(int h_q, int s_q);

/*
 * Bytes of device workspace mla_decode needs: fp32 partial outputs, lse and two precision
 * bounds (see mla_decode) for at most batch + num_parts - 1 pieces of s_q*h_q rows each:
 *     (batch + num_parts) * s_q * h_q * (512 + 3) * 4, rounded up to 256.
 * Returns 0 for invalid sizes. Host only.
 */
size_t mla_workspace_bytes(int batch, int s_q, int h_q, int num_parts);

/*
 * Split-KV metadata ("tile-scheduler metadata").
 *   seqlens     int32[batch]                  device, read only (negative = 0)
 *   tile_meta   int32[num_parts * 8]          device, written: per part
 *               {begin_seq, begin_blk, end_seq (inclusive), end_blk (exclusive),
 *                index of the part's first piece within its sequence, 0, 0, 0};
 *               an empty part is {0, 0, -1, 0, 0, 0, 0, 0}
 *   num_splits  int32[batch + 1]              device, written: num_splits[0] = 0,
 *               num_splits[i+1] - num_splits[i] = pieces of sequence i (0 if n_i <= 0)
 *   fixed_cost  start-up cost of a sequence in block units (>= 0)
 * Rule: sequence i with w_i = ceil(n_i/64) > 0 blocks occupies fixed_cost + w_i units on a
 * line of work units (start-up first, then its blocks, sequences in order); with U units
 * in all, T = max(1, ceil(U/num_parts)) and the block at unit u belongs to part u / T.
 * One single-CTA launch; h_q and s_q are validated but do not change the result.
 */
int mla_get_metadata(const int32_t *seqlens, int batch, int h_q, int s_q, int num_parts,
                     int fixed_cost, int32_t *tile_meta, int32_t *num_splits, void *stream);

/*
 * Decode attention (split kernel + combine kernel on `stream`).
 *   q            bf16[batch, s_q, h_q, 576]      contiguous, 16-byte aligned
 *   kv_cache     bf16[num_blocks, 64, 1, 576]    contiguous, 16-byte aligned
 *   block_table  int32[batch, bt_stride]          entry j of row b = physical block of
 *                tokens [64j, 64j+64) of sequence b; only the first ceil(n_b/64) entries
 *                are read; others may hold anything (e.g. -1)
 *   seqlens      int32[batch]                     tokens in each sequence (<= 64*bt_stride)
 *   tile_meta, num_splits, num_parts, as produced by mla_get_metadata for these seqlens
 *   scale        multiplies q.k before the softmax (finite, >= 0: the kernel takes the row
 *                maximum of the raw scores and scales it afterwards)
 *   causal       0/1, masking between the s_q query tokens (see top of file)
 *   out          bf16[batch, s_q, h_q, 512]       written (round to nearest even)
 *   lse          fp32[batch, h_q, s_q]            written (natural log; -inf if no key)
 *   workspace    >= mla_workspace_bytes(batch, s_q, h_q, num_parts) bytes, 256-aligned;
 *                contents on entry are ignored
 * Requires an sm_100 device (B200). 1 <= s_q*h_q <= MLA_MAX_ROWS.
 * Precision: the two SMs that share a row exchange, per token, the square root of its share of
 * the softmax from their halves of q.k as fp16, relative to each SM's own partial maximum over 32
 * tokens. That is exact to 2^-10 while a token's partial score is within ~58 octaves (about 40 in
 * natural-log units of scale * q.k) of that maximum. A row whose dominant keys fall outside that
 * range (its two partial maxima, from different keys, overstate its true maximum by ~50 octaves
 * or more: far from attention at scale 192^-0.5, possible with very large scores) may lose
 * precision in out and lse; when a bound on the error that the exchange's subnormal range adds to
 * its softmax sum exceeds 2^-11 of the sum, the kernel sets MLA_ERR_RANGE, which mla_check_status
 * reports. Results are then unspecified for that row.
 */
int mla_decode(const void *q, const void *kv_cache, int64_t num_blocks,
               const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
               const int32_t *tile_meta, const int32_t *num_splits, int num_parts, int batch,
               int s_q, int h_q, float scale, int causal, void *out, float *lse,
               void *workspace, size_t workspace_bytes, void *stream);

/* The two launches of mla_decode, separately (same arguments and rules). The split
 * kernel writes `out`/`lse` of every sequence held by one piece and the workspace
 * partials of the others; the combine kernel then finishes the split sequences and
 * the sequences with no tokens. Both must run, in this order, on the same stream. */
int mla_decode_split(const void *q, const void *kv_cache, int64_t num_blocks,
                     const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                     const int32_t *tile_meta, const int32_t *num_splits, int num_parts,
                     int batch, int s_q, int h_q, float scale, int causal, void *out,
                     float *lse, void *workspace, size_t workspace_bytes, void *stream);
int mla_decode_combine(const int32_t *num_splits, int num_parts, int batch, int s_q, int h_q,
                       void *out, float *lse, const void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * The same decode over an FP8 latent cache. The pages name FP8 precision as a tuning option for
 * more throughput ("Playing DeepSeek on the cloud, part 5: ... FlashMLA accelerating
 * DeepSeek-V2-Lite inference", section 4 "developer practice", item 2 "monitoring and tuning"),
 * and FP8 as the data type DeepEP dispatches natively ("Deep analysis of the DeepSeek Infra
 * open-source releases", DAY2 DeepEP, project feature 3); neither fixes a cache format, so this
 * one is the library's own:
 *   kv_cache_fp8  uint8[num_blocks, 64, 1, MLA_FP8_RECORD_BYTES], 16-byte aligned; per token
 *                 bytes [0, 512) are the 512 latent dims as OCP E4M3 (1 sign, 4 exponent bits
 *                 with bias 7, 3 mantissa bits; no infinities), and bytes [512, 640) are the 64
 *                 rotary dims as little-endian bf16
 *   kv_scale      latent byte x stands for kv_scale * e4m3(x) (one scale for the whole cache;
 *                 finite, in [2^-64, 2^64]); the rotary dims are not scaled
 * Keys are the dequantized 576-d vectors and values their first 512 dims; all other arguments,
 * outputs, the workspace and the two-kernel split are as for mla_decode.
 * How it computes: the latent query dims are multiplied by kv_scale / 2^floor(log2 kv_scale) and
 * rounded to fp16 (a relative error of at most 2^-11 per element; every E4M3 value is an fp16
 * number, so the cache side is exact), the products and sums are fp32, the probabilities P are
 * rounded to fp16 for P.V. A query value that does not fit fp16 after that multiplication (or is
 * not finite) sets MLA_ERR_RANGE, which mla_check_status reports; the results are then undefined.
 */
int mla_decode_fp8(const void *q, const void *kv_cache_fp8, int64_t num_blocks, float kv_scale,
                   const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                   const int32_t *tile_meta, const int32_t *num_splits, int num_parts, int batch,
                   int s_q, int h_q, float scale, int causal, void *out, float *lse, void *workspace,
                   size_t workspace_bytes, void *stream);
/* The split kernel alone (mla_decode_combine finishes, as for mla_decode_split). */
int mla_decode_split_fp8(const void *q, const void *kv_cache_fp8, int64_t num_blocks, float kv_scale,
                         const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                         const int32_t *tile_meta, const int32_t *num_splits, int num_parts,
                         int batch, int s_q, int h_q, float scale, int causal, void *out,
                         float *lse, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Sparse decode over the bf16 cache: every query token attends to a list of cache positions
 * instead of its whole sequence. The pages recommend a sparse attention mode for sequences over 8K
 * tokens ("Playing DeepSeek on the cloud, part 5: ... FlashMLA accelerating DeepSeek-V2-Lite
 * inference", section 4 "developer practice", item 2 "monitoring and tuning") without saying what is
 * sparse; this library's reading: row (b, t, h) attends only to the keys at the positions
 * indices[b, t, 0..topk), shared by the h_q heads of that token.
 *   indices   int32[batch, s_q, topk], 4-byte aligned: positions within sequence b. An entry outside
 *             [0, seqlens[b]) is no key (e.g. -1 padding); an entry listed twice counts twice; order
 *             does not matter. No causal mask applies (the list decides). A row with no key gets
 *             out = 0, lse = -inf.
 *   topk      1 <= topk <= 2^24
 *   tile_meta, num_splits, num_parts: from mla_get_metadata_sparse with the same batch, s_q, h_q,
 *             topk (the work units are the batch * s_q query tokens, each with topk keys)
 *   workspace >= mla_workspace_bytes(batch * s_q, 1, h_q, num_parts) bytes, 256-aligned
 * All other arguments, outputs, precision and status rules are those of mla_decode (q, out and lse
 * have the same shapes; 1 <= batch * s_q <= MLA_MAX_BATCH, 1 <= h_q <= MLA_MAX_ROWS). A position whose
 * block-table entry lies outside [0, num_blocks) (or past bt_stride) is treated as no key and
 * reported as MLA_ERR_BOUNDS by mla_check_status. Launches the split and combine kernels on
 * `stream`; allocates nothing.
 */
int mla_get_metadata_sparse(int batch, int s_q, int h_q, int topk, int num_parts, int fixed_cost,
                            int32_t *tile_meta, int32_t *num_splits, void *stream);
int mla_decode_sparse(const void *q, const void *kv_cache, int64_t num_blocks, const int32_t *block_table,
                      int64_t bt_stride, const int32_t *seqlens, const int32_t *indices, int topk,
                      const int32_t *tile_meta, const int32_t *num_splits, int num_parts, int batch, int s_q,
                      int h_q, float scale, void *out, float *lse, void *workspace, size_t workspace_bytes,
                      void *stream);

/*
 * Appending new tokens to the paged cache, the step that precedes decode. Token t of sequence b's
 * new tokens goes to position p = seqlens[b] + t of that sequence, i.e. cache row
 * block_table[b][p / 64] * 64 + p % 64 ("Deep analysis of the DeepSeek Infra open-source releases",
 * DAY1 FlashMLA, feature (2): 64-token blocks).
 *   new_kv       bf16[batch, n_new, 576], contiguous, 16-byte aligned: the new tokens' latent vectors
 *   kv_cache     bf16[num_blocks, 64, 1, 576] (mla_append_kv) or uint8[num_blocks, 64, 1, 640]
 *                (mla_append_kv_fp8), 16-byte aligned; written in place
 *   block_table  int32[batch, bt_stride]; the entries for the new positions must already be set
 *   seqlens      int32[batch]: the lengths BEFORE the append (the caller adds n_new afterwards)
 *   kv_scale     fp8 only: the cache's latent scale; each latent value x is stored as the E4M3 code
 *                of x * (1 / kv_scale) (one fp32 multiply), rounded to nearest even and saturated
 *                to +-448; the rotary dims are stored as bf16
 * Asynchronous on `stream`; allocates nothing. n_new = 0 is a no-op. A new row whose table entry is
 * past bt_stride or outside [0, num_blocks) is skipped and reported as MLA_ERR_BOUNDS by
 * mla_check_status. Returns MLA_ERR_INVALID_ARG for null or misaligned pointers or sizes out of
 * range (and a non-finite or non-positive kv_scale), MLA_ERR_UNSUPPORTED without an sm_100 device,
 * MLA_ERR_CUDA if the launch fails, else MLA_OK.
 */
int mla_append_kv(const void *new_kv, int n_new, void *kv_cache, int64_t num_blocks, const int32_t *block_table,
                  int64_t bt_stride, const int32_t *seqlens, int batch, void *stream);
int mla_append_kv_fp8(const void *new_kv, int n_new, void *kv_cache_fp8, int64_t num_blocks, float kv_scale,
                      const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens, int batch,
                      void *stream);

/*
 * The per-head projections on either side of decode attention, as GEMMs on the tensor cores: for
 * every head h, Y_h (m x n) = X_h (m x k) W_h (k x n) in bf16 with fp32 accumulation, rounded to
 * bf16 (nearest even). With the up-projections absorbed into the query and the output ("Deep
 * analysis of the DeepSeek Infra open-source releases", DAY1 FlashMLA: the kernel works on the
 * latent vectors; feature (4)), the query side is q_latent = q_nope W_UK (k 128, n 512, written
 * straight into the first 512 dims of q's rows) and the output side is o = o_latent W_UV
 * (k 512, n 128).
 *   x   bf16; row r of X_h starts at x + r * ldx + h * x_head_stride (elements)
 *   w   bf16[heads, k, n], contiguous (W_h row-major)
 *   y   bf16; row r of Y_h starts at y + r * ldy + h * y_head_stride; written
 * k and n are multiples of 64; ldx, x_head_stride, ldy, y_head_stride multiples of 8 (16-byte rows);
 * the head blocks lie inside a row ((heads - 1) * stride + width <= ld); pointers 16-byte aligned.
 * Asynchronous on `stream`; allocates nothing. Returns MLA_ERR_INVALID_ARG for arguments outside
 * these rules, MLA_ERR_UNSUPPORTED without an sm_100 device, MLA_ERR_CUDA if a CUDA call fails, else
 * MLA_OK; a pipeline wait past its bound is reported as MLA_ERR_TIMEOUT by mla_check_status.
 */
int mla_head_gemm(const void *x, int64_t ldx, int64_t x_head_stride, const void *w, void *y, int64_t ldy,
                  int64_t y_head_stride, int m, int n, int k, int heads, void *stream);

/*
 * End-to-end call on HOST buffers: copies the inputs host->device, runs metadata +
 * decode, copies out/lse device->host, and synchronises `stream` before returning.
 * Host buffers should be pinned for the copies to be asynchronous. `dev` holds the
 * caller-allocated device buffers, each at least as large as the host one
 * (workspace: mla_workspace_bytes). Uses num_parts = dev->num_parts and
 * fixed_cost = dev->fixed_cost.
 */
typedef struct mla_device_buffers {
    void *q;             /* bf16[batch, s_q, h_q, 576]    */
    void *kv_cache;      /* bf16[num_blocks, 64, 1, 576]  */
    int32_t *block_table;/* int32[batch, bt_stride]       */
    int32_t *seqlens;    /* int32[batch]                  */
    int32_t *tile_meta;  /* int32[num_parts * 8]          */
    int32_t *num_splits; /* int32[batch + 1]              */
    void *out;           /* bf16[batch, s_q, h_q, 512]    */
    float *lse;          /* fp32[batch, h_q, s_q]         */
    void *workspace;
    size_t workspace_bytes;
    int num_parts;
    int fixed_cost;
} mla_device_buffers;

int mla_decode_host(const void *q_host, const void *kv_cache_host, int64_t num_blocks,
                    const int32_t *block_table_host, int64_t bt_stride,
                    const int32_t *seqlens_host, int batch, int s_q, int h_q, float scale,
                    int causal, void *out_host, float *lse_host,
                    const mla_device_buffers *dev, void *stream);
/* The same over the fp8 cache (mla_decode_fp8): kv_cache_fp8_host is uint8[num_blocks, 64, 1,
 * MLA_FP8_RECORD_BYTES] and dev->kv_cache a device buffer of that size. */
int mla_decode_host_fp8(const void *q_host, const void *kv_cache_fp8_host, int64_t num_blocks, float kv_scale,
                        const int32_t *block_table_host, int64_t bt_stride, const int32_t *seqlens_host,
                        int batch, int s_q, int h_q, float scale, int causal, void *out_host, float *lse_host,
                        const mla_device_buffers *dev, void *stream);

/*
 * Decode for callers that cannot allocate device memory (no counterpart on the pages: this
 * is a library convenience). Same arguments, rules and results as mla_decode, without the
 * workspace: the fp32 partials of split sequences go to a fixed scratch array of
 * MLA_NOALLOC_SCRATCH_BYTES that is part of the library's device image (every GPU that
 * loads the library holds it until the process exits). For callers whose memory comes from
 * a fixed pool, or whose serving path may not call cudaMalloc (a late allocation can fail
 * or synchronise), this call allocates nothing: no cudaMalloc, cudaFree or allocating
 * library routine.
 *   - Returns MLA_ERR_WORKSPACE, launching nothing, when mla_workspace_bytes(batch, s_q, h_q,
 *     num_parts) exceeds MLA_NOALLOC_SCRATCH_BYTES (reduce num_parts or the batch).
 *   - The first call on each device (and the first after a device reset, which reloads the
 *     library's module) looks up the scratch array's device address (cudaGetSymbolAddress)
 *     with that device current; make that first call before any stream capture.
 *   - Every call on a device shares the one scratch array, which keeps the last call's
 *     contents (none of which must start at zero): calls that overlap on the GPU, e.g. on
 *     two streams, race on it and must be serialised by the caller.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (16u << 20)
int mla_decode_noalloc(const void *q, const void *kv_cache, int64_t num_blocks,
                       const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                       const int32_t *tile_meta, const int32_t *num_splits, int num_parts,
                       int batch, int s_q, int h_q, float scale, int causal, void *out, float *lse,
                       void *stream);

/*
 * Synchronises `stream`, then reads and clears this device's error word.
 * Returns MLA_OK, MLA_ERR_BOUNDS, MLA_ERR_TIMEOUT, MLA_ERR_RANGE (in that order of priority
 * when several bits are set), or MLA_ERR_CUDA if a CUDA call
 * (including an earlier asynchronous launch) failed.
 */
int mla_check_status(void *stream);

/* Number of kernel launches made by this process through the library so far (host
 * counter; used to report how many of the library's kernels a benchmark ran). */
int64_t mla_launch_count(void);

/* Name and description of the last CUDA error that a call of this library saw (a failed
 * launch, or an earlier asynchronous fault reported by mla_check_status), for the message that
 * goes with MLA_ERR_CUDA; "no error" if there was none. Host only; the string is static. */
const char *mla_last_cuda_error(void);

/*
 * Test of the failure path of the kernels' bounded waits (the pages have no counterpart; it
 * exists so that the timeout path can be exercised without a fault). Launches, on `stream`,
 * one CTA that waits, with the decode kernel's own wait primitive, on an mbarrier that nothing
 * completes, for at most `spin_cycles` SM clock cycles (1e5 .. 4e9). The wait then gives up and
 * raises the timeout bit of the device error word, so the next mla_check_status returns
 * MLA_ERR_TIMEOUT. Returns MLA_ERR_INVALID_ARG for a bound outside the range, MLA_ERR_UNSUPPORTED
 * without an sm_100 device, MLA_ERR_CUDA if the launch fails, else MLA_OK. Allocates nothing.
 */
int mla_selftest_wait_timeout(int64_t spin_cycles, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_B200_MLA_H_ */
