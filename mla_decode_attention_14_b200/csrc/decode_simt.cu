// decode_simt.cu -- CUDA-core split kernel: the bring-up path that fixes the work
// partition, partial-buffer layout and masking semantics the tensor-core kernel shares.
//
// One CTA per (part, group of 16 query rows), 8 warps, 2 rows per warp. For each piece of
// its part the CTA stages every 64-token block ("Deep analysis of the DeepSeek Infra
// open-source releases", DAY1 FlashMLA, feature (2)) in shared memory through the block
// table, scores it against the rows' 576-d queries ("Gemm1"), updates a running max and
// sum (online softmax, fp32), and accumulates the weighted 512-d values ("Gemm2").
#include "common.cuh"

namespace mla {

constexpr int kSimtRows = 16;
constexpr int kSimtThreads = 256;
constexpr int kRowPad = kDqk + 8;  // bf16 per staged key row: 1168 B, conflict-free 16 B reads

struct SimtSmem {
    __nv_bfloat16 kv[kBlk][kRowPad];
    float q[kSimtRows][kDqk];
};

__global__ void __launch_bounds__(kSimtThreads)
decode_simt_kernel(DecodeParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem &sm = *reinterpret_cast<SimtSmem *>(smem_raw);
    const int part = blockIdx.x;
    const int row0 = blockIdx.y * kSimtRows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t *meta = p.tile_meta + (size_t)part * kMetaInts;
    const int begin_seq = meta[0], begin_blk = meta[1], end_seq = meta[2], end_blk = meta[3];
    const int first_piece = meta[4];
    if (end_seq >= begin_seq && (begin_seq < 0 || end_seq >= p.batch)) {  // malformed metadata
        if (threadIdx.x == 0) raise_error(kErrBounds);
        return;
    }

    for (int seq = begin_seq; seq <= end_seq; ++seq) {
        const int n = p.seqlens[seq] > 0 ? p.seqlens[seq] : 0;
        const int wblk = num_blocks_of(n);
        const int lo = seq == begin_seq ? begin_blk : 0;
        const int hi = seq == end_seq ? end_blk : wblk;
        if (hi <= lo) continue;
        const int piece = seq == begin_seq ? first_piece : 0;
        const int nsplit = p.num_splits[seq + 1] - p.num_splits[seq];
        const int slot = p.num_splits[seq] + piece;
        if (nsplit > 1 && (slot < 0 || slot >= p.batch + p.num_parts)) {
            if (threadIdx.x == 0) raise_error(kErrBounds);
            continue;
        }

        __syncthreads();  // previous piece done with sm.q
        for (int e = threadIdx.x; e < kSimtRows * kDqk; e += blockDim.x) {
            const int rr = e / kDqk, d = e % kDqk;
            const int r = row0 + rr;
            sm.q[rr][d] = r < p.rows ? __bfloat162float(p.q[((size_t)seq * p.rows + r) * kDqk + d]) : 0.f;
        }

        float m[2], l[2], o[2][16];
        int vis[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int r = row0 + warp * 2 + k;
            m[k] = -INFINITY;
            l[k] = 0.f;
            vis[k] = r < p.rows ? visible_keys(n, p.s_q, r / p.h_q, p.causal) : 0;
#pragma unroll
            for (int d = 0; d < 16; ++d) o[k][d] = 0.f;
        }

        for (int blk = lo; blk < hi; ++blk) {
            int phys = blk < p.bt_stride ? p.block_table[(size_t)seq * p.bt_stride + blk] : -1;
            const bool ok = phys >= 0 && phys < p.num_blocks;
            if (!ok) {
                if (threadIdx.x == 0) raise_error(kErrBounds);
                phys = 0;
            }
            const int valid = min(kBlk, n - blk * kBlk);  // tokens of this block inside the sequence
            __syncthreads();  // previous block done with sm.kv
            const uint4 *src = reinterpret_cast<const uint4 *>(p.kv + (size_t)phys * kBlk * kDqk);
            for (int e = threadIdx.x; e < kBlk * (kDqk / 8); e += blockDim.x) {
                const int tok = e / (kDqk / 8), c = e % (kDqk / 8);
                uint4 v = (ok && tok < valid) ? src[e] : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(&sm.kv[tok][c * 8]) = v;
            }
            __syncthreads();

#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int rr = warp * 2 + k;
                float s[2];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int tok = lane + 32 * h2;
                    float acc = 0.f;
                    for (int c = 0; c < kDqk / 8; ++c) {
                        uint4 raw = *reinterpret_cast<const uint4 *>(&sm.kv[tok][c * 8]);
                        const __nv_bfloat162 *kb = reinterpret_cast<const __nv_bfloat162 *>(&raw);
                        const float4 qa = *reinterpret_cast<const float4 *>(&sm.q[rr][c * 8]);
                        const float4 qb = *reinterpret_cast<const float4 *>(&sm.q[rr][c * 8 + 4]);
                        float2 k0 = __bfloat1622float2(kb[0]), k1 = __bfloat1622float2(kb[1]);
                        float2 k2 = __bfloat1622float2(kb[2]), k3 = __bfloat1622float2(kb[3]);
                        acc += qa.x * k0.x + qa.y * k0.y + qa.z * k1.x + qa.w * k1.y;
                        acc += qb.x * k2.x + qb.y * k2.y + qb.z * k3.x + qb.w * k3.y;
                    }
                    const int key = blk * kBlk + tok;
                    s[h2] = key < vis[k] ? acc * p.scale_log2 : -INFINITY;  // log2 domain
                }
                float bm = fmaxf(s[0], s[1]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
                const float m_new = fmaxf(m[k], bm);
                if (m_new == -INFINITY) continue;  // nothing visible yet for this row
                const float alpha = exp2f(m[k] - m_new);  // m[k] = -inf -> 0
                const float p0 = exp2f(s[0] - m_new), p1 = exp2f(s[1] - m_new);
                float ps = p0 + p1;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
                l[k] = l[k] * alpha + ps;
                m[k] = m_new;
#pragma unroll
                for (int d = 0; d < 16; ++d) o[k][d] *= alpha;
                for (int j = 0; j < kBlk; ++j) {
                    const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
                    if (pj == 0.f) continue;
                    const uint4 *vrow = reinterpret_cast<const uint4 *>(&sm.kv[j][lane * 16]);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint4 raw = vrow[c];
                        const __nv_bfloat162 *vb = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            float2 v = __bfloat1622float2(vb[e2]);
                            o[k][c * 8 + 2 * e2] += pj * v.x;
                            o[k][c * 8 + 2 * e2 + 1] += pj * v.y;
                        }
                    }
                }
            }
        }

        // epilogue: normalise; whole sequence -> out/lse, piece of a split sequence -> partials
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int r = row0 + warp * 2 + k;
            if (r >= p.rows) continue;
            const bool empty = !(l[k] > 0.f);
            const float inv = empty ? 0.f : 1.f / l[k];
            const float lse_val = empty ? -INFINITY : (m[k] + log2f(l[k])) * 0.69314718055994530942f;
            if (nsplit == 1) {
                __nv_bfloat16 *orow = p.out + ((size_t)seq * p.rows + r) * kDv + lane * 16;
                uint4 packed[2];
                uint32_t *pw = reinterpret_cast<uint32_t *>(packed);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    __nv_bfloat162 two = __floats2bfloat162_rn(o[k][2 * e] * inv, o[k][2 * e + 1] * inv);
                    pw[e] = *reinterpret_cast<uint32_t *>(&two);
                }
                reinterpret_cast<uint4 *>(orow)[0] = packed[0];
                reinterpret_cast<uint4 *>(orow)[1] = packed[1];
                if (lane == 0) {
                    const int t = r / p.h_q, h = r % p.h_q;
                    p.lse[((size_t)seq * p.h_q + h) * p.s_q + t] = lse_val;
                }
            } else {
                float4 *dst = reinterpret_cast<float4 *>(p.o_part + ((size_t)slot * p.rows + r) * kDv + lane * 16);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    dst[c] = make_float4(o[k][4 * c] * inv, o[k][4 * c + 1] * inv, o[k][4 * c + 2] * inv,
                                         o[k][4 * c + 3] * inv);
                if (lane == 0) p.lse_part[(size_t)slot * p.rows + r] = lse_val;
            }
        }
    }
}

cudaError_t launch_decode_simt(const DecodeParams &p, cudaStream_t stream) {
    const size_t smem = sizeof(SimtSmem);
    cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.num_parts, (p.rows + kSimtRows - 1) / kSimtRows);
    decode_simt_kernel<<<grid, kSimtThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace mla
