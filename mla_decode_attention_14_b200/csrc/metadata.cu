// metadata.cu -- length-aware split-KV work partition on the device.
//
// "Deep analysis of the DeepSeek Infra open-source releases" (jingzhunhuoke.net/55333.html),
// DAY1 FlashMLA, feature (5): inputs of very different lengths are load-balanced (the page
// gives no algorithm), and feature (2): the cache is cut into 64-token blocks.
//
// Rule (the library's reading): sequences lie end to end on a line of work units; sequence
// i with w_i = ceil(n_i/64) > 0 blocks occupies C start-up units and then one unit per
// block; empty sequences occupy nothing. With U units in all and P parts,
// T = max(1, ceil(U/P)) and the block at unit u belongs to part floor(u/T). So every part
// is a contiguous run of (sequence, block) pairs and its work is at most T + C units.
//
// Sparse mode gives every work unit the same length (its index list); `seqlens` is then null
// and `uniform_n` that length.
//
// This kernel derives each part's bounds in closed form from the prefix sums of the
// per-sequence costs: one CTA, a chunked block-wide scan over the sequences, and each
// sequence writes the begin/end fields of the parts its blocks touch (every field is
// written by exactly one thread).
#include "common.cuh"

namespace mla {

constexpr int kMetaThreads = 1024;

template <typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T *warp_sums, T *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    T x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        T s = lane < nw ? warp_sums[lane] : T(0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            T y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < nw) warp_sums[lane] = s;  // inclusive prefix of warp totals
    }
    __syncthreads();
    T warp_prefix = warp > 0 ? warp_sums[warp - 1] : T(0);
    *total = warp_sums[(blockDim.x >> 5) - 1];
    __syncthreads();
    return warp_prefix + x - v;
}

__global__ void __launch_bounds__(kMetaThreads)
metadata_kernel(const int32_t *__restrict__ seqlens, int uniform_n, int batch, int num_parts, int C,
                int32_t *__restrict__ tile_meta, int32_t *__restrict__ num_splits) {
    __shared__ int64_t warp_sums64[32];
    __shared__ int32_t warp_sums32[32];
    __shared__ int64_t red[32];

    // empty parts first
    for (int p = threadIdx.x; p < num_parts; p += blockDim.x) {
        int32_t *m = tile_meta + (size_t)p * kMetaInts;
        m[0] = 0; m[1] = 0; m[2] = -1; m[3] = 0; m[4] = 0; m[5] = 0; m[6] = 0; m[7] = 0;
    }

    // pass 1: total units U
    int64_t local = 0;
    for (int i = threadIdx.x; i < batch; i += blockDim.x) {
        int w = num_blocks_of(seqlens ? seqlens[i] : uniform_n);
        if (w > 0) local += (int64_t)C + w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = local;
    __syncthreads();
    int64_t U = 0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) U += red[k];
    int64_t T = (U + num_parts - 1) / num_parts;
    if (T < 1) T = 1;
    __syncthreads();  // parts initialised before any sequence writes into them

    // pass 2: prefix of costs -> part bounds; prefix of piece counts -> num_splits
    if (threadIdx.x == 0) num_splits[0] = 0;
    int64_t carry_units = 0;
    int32_t carry_splits = 0;
    for (int base = 0; base < batch; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int w = i < batch ? num_blocks_of(seqlens ? seqlens[i] : uniform_n) : 0;
        const int64_t cost = w > 0 ? (int64_t)C + w : 0;
        int64_t chunk_units;
        const int64_t pre = carry_units + block_exclusive_scan<int64_t>(cost, warp_sums64, &chunk_units);
        int32_t splits = 0;
        if (w > 0) {
            const int64_t u0 = pre + C;            // unit of block 0
            const int64_t u1 = u0 + w - 1;         // unit of the last block
            const int64_t first = u0 / T, last = u1 / T;
            splits = (int32_t)(last - first + 1);
            const bool begins_first = (pre == 0) || ((pre - 1) / T < first);
            const bool ends_last = (u1 + 1 == U) || ((u1 + 1 + C) / T > last);
            for (int64_t q = first; q <= last; ++q) {
                int32_t *m = tile_meta + (size_t)q * kMetaInts;
                if (q > first || begins_first) {
                    m[0] = i;
                    m[1] = (int32_t)(q > first ? q * T - u0 : 0);
                    m[4] = (int32_t)(q - first);
                }
                if (q < last || ends_last) {
                    m[2] = i;
                    m[3] = (int32_t)(q < last ? (q + 1) * T - u0 : w);
                }
            }
        }
        int32_t chunk_splits;
        const int32_t spre = carry_splits + block_exclusive_scan<int32_t>(splits, warp_sums32, &chunk_splits);
        if (i < batch) num_splits[i + 1] = spre + splits;
        carry_units += chunk_units;
        carry_splits += chunk_splits;
    }
}

cudaError_t launch_metadata(const int32_t *seqlens, int uniform_n, int batch, int num_parts, int fixed_cost,
                            int32_t *tile_meta, int32_t *num_splits, cudaStream_t stream) {
    metadata_kernel<<<1, kMetaThreads, 0, stream>>>(seqlens, uniform_n, batch, num_parts, fixed_cost,
                                                    tile_meta, num_splits);
    return cudaGetLastError();
}

}  // namespace mla
