// append.cu -- writing new tokens' 576-d latent vectors into the paged cache, the step that precedes
// decode attention. Token t of sequence b's new tokens goes to position p = seqlens[b] + t of that
// sequence: cache row block_table[b][p / 64] * 64 + p % 64 ("Deep analysis of the DeepSeek Infra
// open-source releases", DAY1 FlashMLA, feature (2): the cache is kept in 64-token blocks).
//  * bf16 cache: the row is copied.
//  * fp8 cache (640-byte records): each latent value is multiplied by 1 / kv_scale in fp32 and stored
//    as its E4M3 code, rounded to nearest even and saturated to +-448; the 64 rotary dims are copied
//    as bf16.
// One warp per new row; a row whose block-table entry is missing or outside [0, num_blocks) sets the
// device error word (kErrBounds) and is skipped.
#include <cuda_fp8.h>

#include "common.cuh"

namespace mla {
namespace {

constexpr int kAppendWarps = 8;
constexpr int kF8Record = 640;  // fp8 cache: bytes per token (512 E4M3 latent + 64 bf16 rotary)

template <bool F8>
__global__ void __launch_bounds__(32 * kAppendWarps)
    append_kernel(const __nv_bfloat16 *__restrict__ new_kv, int n_new, uint8_t *__restrict__ kv, int64_t num_blocks,
                  const int32_t *__restrict__ block_table, int64_t bt_stride, const int32_t *__restrict__ seqlens,
                  int batch, float inv_scale) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (int64_t)batch * n_new) return;
    const int b = (int)(w / n_new), t = (int)(w % n_new);
    const int64_t pos = (int64_t)max(seqlens[b], 0) + t;
    const int64_t bi = pos / kBlk;
    const int32_t phys = bi < bt_stride ? block_table[(size_t)b * bt_stride + bi] : -1;
    if (phys < 0 || (int64_t)phys >= num_blocks) {
        if (lane == 0) raise_error(kErrBounds);
        return;
    }
    const int64_t row = (int64_t)phys * kBlk + pos % kBlk;
    const uint4 *src = reinterpret_cast<const uint4 *>(new_kv + (size_t)w * kDqk);  // 72 chunks of 8 bf16
    if constexpr (!F8) {
        uint4 *dst = reinterpret_cast<uint4 *>(kv + row * (int64_t)(kDqk * 2));
        for (int c = lane; c < kDqk / 8; c += 32) dst[c] = src[c];
    } else {
        uint8_t *rec = kv + row * (int64_t)kF8Record;
        for (int c = lane; c < kDv / 8; c += 32) {  // 8 latent values per chunk -> 8 E4M3 bytes
            const uint4 x = src[c];
            const uint32_t wv[4] = {x.x, x.y, x.z, x.w};
            uint32_t out[2];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float lo = __uint_as_float(wv[i] << 16) * inv_scale;
                const float hi = __uint_as_float(wv[i] & 0xffff0000u) * inv_scale;
                const uint32_t two = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
                if (i & 1)
                    out[i >> 1] |= two << 16;
                else
                    out[i >> 1] = two;
            }
            reinterpret_cast<uint2 *>(rec)[c] = make_uint2(out[0], out[1]);
        }
        if (lane < (kDqk - kDv) / 8) reinterpret_cast<uint4 *>(rec + kDv)[lane] = src[kDv / 8 + lane];
    }
}

}  // namespace

cudaError_t launch_append(const __nv_bfloat16 *new_kv, int n_new, void *kv, int64_t num_blocks,
                          const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens, int batch,
                          bool fp8, float inv_scale, cudaStream_t stream) {
    const int64_t rows = (int64_t)batch * n_new;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kAppendWarps - 1) / kAppendWarps);
    if (fp8)
        append_kernel<true><<<grid, 32 * kAppendWarps, 0, stream>>>(new_kv, n_new, static_cast<uint8_t *>(kv),
                                                                   num_blocks, block_table, bt_stride, seqlens,
                                                                   batch, inv_scale);
    else
        append_kernel<false><<<grid, 32 * kAppendWarps, 0, stream>>>(new_kv, n_new, static_cast<uint8_t *>(kv),
                                                                    num_blocks, block_table, bt_stride, seqlens,
                                                                    batch, inv_scale);
    return cudaGetLastError();
}

}  // namespace mla
