// common.cuh -- device-side helpers shared by the library's kernels (not by any test code).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

constexpr int kDqk = 576;        // key width: 512 latent + 64 rotary dims
constexpr int kDv = 512;         // value width: first 512 dims of the key
constexpr int kBlk = 64;         // tokens per cache block
constexpr int kMetaInts = 8;     // int32 per part in tile_meta

// Per-device error word (bit flags), read and cleared by mla_check_status().
constexpr unsigned kErrBounds = 1u;   // a needed block-table entry was outside [0, num_blocks)
constexpr unsigned kErrTimeout = 2u;  // a pipeline wait hit its iteration bound
constexpr unsigned kErrRange = 4u;    // fp8 cache: a query value outside the range of its fp16 form
// Defined here: the library is one translation unit (csrc/mla_lib.cu).
__device__ unsigned int g_error_word = 0;

__device__ __forceinline__ void raise_error(unsigned bit) { atomicOr(&g_error_word, bit); }

// Parameters shared by the split kernels (one struct, passed by value).
struct DecodeParams {
    const __nv_bfloat16 *q;        // [b, s_q, h_q, 576]
    const __nv_bfloat16 *kv;       // [nblk, 64, 576]
    const int32_t *block_table;    // [b, bt_stride]
    const int32_t *seqlens;        // [b]
    const int32_t *tile_meta;      // [num_parts, 8]
    const int32_t *num_splits;     // [b + 1] (cumulative)
    __nv_bfloat16 *out;            // [b, s_q, h_q, 512]
    float *lse;                    // [b, h_q, s_q]
    float *o_part;                 // [slots, rows, 512]
    float *lse_part;               // [slots, rows]
    float *lost_part;              // [slots, rows, 2]: per CTA half, a bound on the error that the pair
                                   // exchange's subnormal range added to the piece's softmax sum, over that sum
    // sparse mode: work unit (sequence) u is query token u % sp_sq of sequence u / sp_sq, with s_q = 1
    // and causal = 0; its keys are the cache positions indices[u, 0..topk) (entries outside
    // [0, seqlens[u / sp_sq]) are no key)
    const int32_t *indices;        // [b * sp_sq, topk], or null (dense)
    int topk, sp_sq;
    int64_t num_blocks;
    int64_t bt_stride;
    int batch, s_q, h_q, rows, num_parts;
    int causal;
    int out_v8;                    // `out` is 32-byte aligned: the epilogue may use 32-byte stores
    float scale;                   // softmax scale
    float scale_log2;              // scale * log2(e) (fp8 cache: also times 2^-k, see q_rope_mul)
    // fp8 cache only: a latent byte x stands for kv_scale * e4m3(x), kv_scale = q_lat_mul * 2^-k with
    // q_lat_mul in [1, 2), and the kernel's fp16 form of it is e4m3(x) * 2^-8; the latent query dims
    // are multiplied by q_lat_mul, the rotary ones by q_rope_mul = 2^(k-8), the output by
    // v_scale = kv_scale * 2^8.
    float v_scale, q_lat_mul, q_rope_mul;
};

// Visible keys of query token t in a sequence of n tokens (causal: the s_q query
// tokens are the sequence's last s_q tokens).
__device__ __forceinline__ int visible_keys(int n, int s_q, int t, int causal) {
    if (n < 0) n = 0;
    if (!causal) return n;
    int v = n - s_q + t + 1;
    return v < 0 ? 0 : (v > n ? n : v);
}

// ceil(n / 64) without forming n + 63 (which overflows for n near INT32_MAX)
__device__ __forceinline__ int num_blocks_of(int n) { return n > 0 ? (n - 1) / kBlk + 1 : 0; }

}  // namespace mla
