// combine.cu -- merges the partial results of sequences computed as several pieces.
//
// A piece s of a sequence leaves, per query row, o_s = (sum_j e^{s_j} v_j) / (sum_j e^{s_j})
// over its keys and lse_s = log(sum_j e^{s_j}). The whole-sequence result is
//   lse = log(sum_s e^{lse_s}),   out = sum_s e^{lse_s - lse} o_s
// (the split-KV reading of "Deep analysis of the DeepSeek Infra open-source releases",
// DAY1 FlashMLA, feature (5); the merge is exact up to rounding). Pieces with no visible
// key carry lse_s = -inf and weight 0; if every piece of a row is empty the row gets
// out = 0, lse = -inf. Sequences with no tokens at all (no piece) are written here too.
//
// Each piece also leaves, per CTA half, a bound on the error that the split kernel's pair exchange
// added to its softmax sum through fp16 subnormals, relative to that sum. The row's bound is the
// pieces' weighted by e^{lse_s - lse}; above 2^-11 the row is reported (MLA_ERR_RANGE).
//
// One warp per (sequence, row); each lane owns 16 of the 512 output dims (four float4),
// so every partial row is read as one coalesced 2 KB segment. Sequences of up to four pieces
// (nearly all) load everything in one go; longer ones walk their pieces.
#include "common.cuh"

namespace mla {

constexpr int kCombineWarps = 8;
constexpr int kFastPieces = 4;

__device__ __forceinline__ void store_row(__nv_bfloat16 *orow, float *lrow, const float (&acc)[16], float L, int lane) {
    uint4 packed[2];
    uint32_t *pw = reinterpret_cast<uint32_t *>(packed);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        __nv_bfloat162 two = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
        pw[k] = *reinterpret_cast<uint32_t *>(&two);
    }
    reinterpret_cast<uint4 *>(orow)[0] = packed[0];
    reinterpret_cast<uint4 *>(orow)[1] = packed[1];
    if (lane == 0) *lrow = L;
}

// Rows of sequences with 0..kFastPieces pieces: the pieces' lse and this lane's 16 dims of each
// partial row are loaded at once, then merged from registers.
__device__ __forceinline__ float lost_of(const float *__restrict__ lost_part, size_t slot) {
    return fmaxf(lost_part[2 * slot], lost_part[2 * slot + 1]);  // the worse of the two CTA halves
}

__device__ __forceinline__ void combine_few(int ns, int s0, int rows, int r, int lane, __nv_bfloat16 *orow, float *lrow,
                                            const float *__restrict__ o_part, const float *__restrict__ lse_part,
                                            const float *__restrict__ lost_part) {
    float ls[kFastPieces], lost[kFastPieces];
    float4 v[kFastPieces][4];
#pragma unroll
    for (int s = 0; s < kFastPieces; ++s) {
        if (s < ns) {
            const size_t slot = (size_t)(s0 + s) * rows + r;
            ls[s] = lse_part[slot];
            lost[s] = lost_of(lost_part, slot);
            const float4 *src = reinterpret_cast<const float4 *>(o_part + slot * kDv + lane * 16);
#pragma unroll
            for (int k = 0; k < 4; ++k) v[s][k] = src[k];
        } else {
            ls[s] = -INFINITY;
            lost[s] = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) v[s][k] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    float m = ls[0];
#pragma unroll
    for (int s = 1; s < kFastPieces; ++s) m = fmaxf(m, ls[s]);
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.f;
    if (m == -INFINITY) {  // no piece, or no visible key in any piece
        store_row(orow, lrow, acc, -INFINITY, lane);
        return;
    }
    float sum = 0.f;
#pragma unroll
    for (int s = 0; s < kFastPieces; ++s) sum += expf(ls[s] - m);  // empty pieces: e^-inf = 0
    const float L = m + logf(sum);
    float lost_row = 0.f;
#pragma unroll
    for (int s = 0; s < kFastPieces; ++s) {
        const float wgt = expf(ls[s] - L);
        if (wgt == 0.f) continue;  // empty piece (its o is 0) or negligible weight
        lost_row = fmaf(wgt, lost[s], lost_row);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc[4 * k + 0] += wgt * v[s][k].x;
            acc[4 * k + 1] += wgt * v[s][k].y;
            acc[4 * k + 2] += wgt * v[s][k].z;
            acc[4 * k + 3] += wgt * v[s][k].w;
        }
    }
    if (lane == 0 && lost_row > 0x1p-11f) raise_error(kErrRange);
    store_row(orow, lrow, acc, L, lane);
}

__global__ void __launch_bounds__(kCombineWarps * 32)
combine_kernel(const int32_t *__restrict__ num_splits, int batch, int num_parts, int s_q, int h_q, int sp_sq,
               __nv_bfloat16 *__restrict__ out, float *__restrict__ lse,
               const float *__restrict__ o_part, const float *__restrict__ lse_part,
               const float *__restrict__ lost_part) {
    const int rows = s_q * h_q;
    const int b = blockIdx.x;
    const int r = blockIdx.y * kCombineWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (b >= batch || r >= rows) return;
    const int s0 = num_splits[b], s1 = num_splits[b + 1];
    const int ns = s1 - s0;
    if (ns == 1) return;  // written directly by the split kernel
    if (ns < 0 || s0 < 0 || s1 > batch + num_parts) {  // malformed metadata
        if (lane == 0) raise_error(kErrBounds);
        return;
    }
    const int t = r / h_q, h = r % h_q;
    __nv_bfloat16 *orow = out + ((size_t)b * rows + r) * kDv + lane * 16;
    // sparse mode (sp_sq > 0): work unit b is query token b % sp_sq of sequence b / sp_sq
    float *lrow = sp_sq > 0 ? lse + ((size_t)(b / sp_sq) * h_q + h) * sp_sq + b % sp_sq
                            : lse + ((size_t)b * h_q + h) * s_q + t;
    if (ns <= kFastPieces) {  // common case: every load issued before any arithmetic (one memory round trip)
        combine_few(ns, s0, rows, r, lane, orow, lrow, o_part, lse_part, lost_part);
        return;
    }

    float m = -INFINITY;
    for (int s = lane; s < ns; s += 32) m = fmaxf(m, lse_part[(size_t)(s0 + s) * rows + r]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

    if (ns == 0 || m == -INFINITY) {
        uint4 z = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4 *>(orow)[0] = z;
        reinterpret_cast<uint4 *>(orow)[1] = z;
        if (lane == 0) *lrow = -INFINITY;
        return;
    }
    float sum = 0.f;
    for (int s = lane; s < ns; s += 32) sum += expf(lse_part[(size_t)(s0 + s) * rows + r] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float L = m + logf(sum);

    float lost_row = 0.f;
    for (int s = lane; s < ns; s += 32) {
        const size_t slot = (size_t)(s0 + s) * rows + r;
        const float wgt = expf(lse_part[slot] - L);
        if (wgt != 0.f) lost_row = fmaf(wgt, lost_of(lost_part, slot), lost_row);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lost_row += __shfl_xor_sync(0xffffffffu, lost_row, o);
    if (lane == 0 && lost_row > 0x1p-11f) raise_error(kErrRange);

    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.f;
    for (int s = 0; s < ns; ++s) {
        const size_t slot = (size_t)(s0 + s) * rows + r;
        const float wgt = expf(lse_part[slot] - L);
        if (wgt == 0.f) continue;  // empty piece (its o is 0) or negligible weight
        const float4 *src = reinterpret_cast<const float4 *>(o_part + slot * kDv + lane * 16);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float4 v = src[k];
            acc[4 * k + 0] += wgt * v.x;
            acc[4 * k + 1] += wgt * v.y;
            acc[4 * k + 2] += wgt * v.z;
            acc[4 * k + 3] += wgt * v.w;
        }
    }
    store_row(orow, lrow, acc, L, lane);
}

cudaError_t launch_combine(const int32_t *num_splits, int batch, int num_parts, int s_q, int h_q, int sp_sq,
                           __nv_bfloat16 *out, float *lse, const float *o_part,
                           const float *lse_part, const float *lost_part, cudaStream_t stream) {
    const int rows = s_q * h_q;
    dim3 grid(batch, (rows + kCombineWarps - 1) / kCombineWarps);
    combine_kernel<<<grid, kCombineWarps * 32, 0, stream>>>(num_splits, batch, num_parts, s_q, h_q, sp_sq, out, lse,
                                                           o_part, lse_part, lost_part);
    return cudaGetLastError();
}

}  // namespace mla
