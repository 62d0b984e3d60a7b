// decode_sm100.cu -- the B200 (sm_100a) split kernel of MLA decode attention.
//
// What it computes (per query row r of sequence b, over that sequence's visible keys j):
// S_j = scale * <q_r, k_j> over all 576 latent+rotary dims ("Gemm1"), an fp32 online softmax,
// and O = sum_j softmax_j * k_j[0:512] ("Gemm2"). "Deep analysis of the DeepSeek Infra
// open-source releases" (jingzhunhuoke.net/55333.html), DAY1 FlashMLA: the cache is kept in
// 64-token blocks (feature (2)), the kernel streams each block once and runs Gemm1 then Gemm2
// on it (feature (4)), and lengths are load-balanced over the SMs (feature (5)).
//
// How (B200 design; the pages' Hopper design is prior art only):
//  * One 2-CTA cluster per (work part, group of 128 query rows); 74 clusters fill the 148 SMs.
//    The fp32 accumulator O for 128 rows x 512 value dims is 256 KB -- all of one SM's tensor
//    memory -- so each CTA of the pair owns HALF of the value dims (O: 128 lanes x 256 columns
//    of TMEM) and streams only the cache columns it needs: CTA h loads latent dims
//    [256h, 256h+256) and rotary dims [512+32h, 512+32h+32), i.e. exactly half of every
//    block (36,864 bytes); the pair together reads each block once.
//  * Gemm1 is split along its 576-long contraction: CTA h computes the partial scores over its
//    288 dims (18 tcgen05 MMAs, M=128 rows, N=64 tokens, K=16, A = this half of Q held in
//    TMEM, B = the K tile in shared memory). The two partial score tiles (128 x 64 fp32) are
//    swapped through distributed shared memory (st.async completing on the receiver's
//    mbarrier); both CTAs add them in the same order and so hold bit-identical scores.
//  * Softmax warps (one thread per query row = one TMEM lane) apply the scale, masks (tail
//    and causal), an online max with lazy rescaling (O is rescaled only when the running max
//    grows by more than 2^8), write P (bf16) into TMEM and release Gemm2.
//  * Gemm2: 4 MMAs (M=128, N=256, K=16 tokens each) with A = P from TMEM and B = the value
//    half of the same shared-memory tile read MN-major -- the block is loaded once for both
//    GEMMs.
//  * Warp roles: warp 0 lane 0 = TMA producer (4-stage ring, block-table gather, L2
//    evict-first); warp 1 = MMA warp (lane 0 issues; the warp owns the TMEM allocation and
//    zeroes the cache rows past a sequence's end before any MMA reads them, so undefined
//    tail contents never reach the result); warps 4-7 = softmax, correction and epilogue
//    (warps 2-3 idle: the softmax warps must sit in TMEM lane quarters 0-3).
//  * Pieces of split sequences leave fp32 partial O and lse in the workspace for the combine
//    kernel; whole sequences are written straight to bf16 out / fp32 lse.
// Every wait is bounded; a timeout sets the device error word and the CTA exits cleanly.
#include "common.cuh"
#include "sm100_ptx.cuh"

namespace mla {
using namespace sm100;

namespace dec {
constexpr int kStages = 4;
constexpr int kThreads = 256;
constexpr int kBoxBytes = kBlk * 128;                      // 64 tokens x 64 bf16 (128-byte swizzle)
constexpr int kRopeBoxBytes = kBlk * 64;                   // 64 tokens x 32 bf16 (64-byte swizzle)
constexpr int kStageBytes = 4 * kBoxBytes + kRopeBoxBytes;  // 36,864: half of one cache block
constexpr int kXchgFloats = 128 * 64;                      // partial score tile of one block
constexpr float kRescaleThreshold = 8.0f;                  // log2 units: rescale O when max grows > 2^8

// TMEM column map (512 columns allocated, 128 lanes = 128 query rows)
constexpr uint32_t kTmemO = 0;    // 256 fp32: O for this CTA's 256 value dims
constexpr uint32_t kTmemS = 256;  // 64 fp32: partial scores of the current block
constexpr uint32_t kTmemQ = 320;  // 144 x (2 bf16): this CTA's 288 query dims
constexpr uint32_t kTmemP = 464;  // 32 x (2 bf16): probabilities of the current block
constexpr uint32_t kTmemCols = 512;

struct __align__(1024) Smem {
    uint8_t stage[kStages][kStageBytes];
    float4 xchg[2][16][128];  // [slot][4-column group][row]: partial scores written by the peer CTA
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full, s_free, p_full, p_free, o_full, o_free, q_full, mma_done;
    uint64_t xfull[2];
    uint32_t tmem_base;
    int abort;
};

struct Piece {
    int seq, lo, hi, n, nsplit, slot;
};

// Walks the non-empty pieces of one part (all roles walk the same list independently).
struct Cursor {
    int seq, begin_seq, begin_blk, end_seq, end_blk, first_piece;
    __device__ void init(const int32_t *meta, int batch) {
        begin_seq = meta[0];
        begin_blk = meta[1];
        end_seq = meta[2];
        end_blk = meta[3];
        first_piece = meta[4];
        if (end_seq >= begin_seq && (begin_seq < 0 || end_seq >= batch)) end_seq = begin_seq - 1;  // malformed
        seq = begin_seq;
    }
    __device__ bool next(const DecodeParams &p, Piece &pc) {
        while (seq <= end_seq) {
            const int s = seq++;
            const int n = max(p.seqlens[s], 0);
            const int w = num_blocks_of(n);
            const int lo = s == begin_seq ? max(begin_blk, 0) : 0;
            const int hi = s == end_seq ? min(end_blk, w) : w;
            if (hi <= lo) continue;
            pc.seq = s;
            pc.lo = lo;
            pc.hi = hi;
            pc.n = n;
            pc.nsplit = p.num_splits[s + 1] - p.num_splits[s];
            pc.slot = p.num_splits[s] + (s == begin_seq ? first_piece : 0);
            if (pc.nsplit > 1 && (pc.slot < 0 || pc.slot >= p.batch + p.num_parts)) continue;  // malformed
            return true;
        }
        return false;
    }
};

__device__ __forceinline__ bool is_tail_block(const Piece &pc, int blk) {
    return blk == num_blocks_of(pc.n) - 1 && (pc.n % kBlk) != 0;
}

// ---------------------------------------------------------------- TMA producer (1 thread)
__device__ void producer(Smem &sm, const DecodeParams &p, const CUtensorMap *map_lat, const CUtensorMap *map_rope,
                         const int32_t *meta, uint32_t half) {
    const uint64_t policy = l2_evict_first_policy();
    Cursor cur;
    cur.init(meta, p.batch);
    Piece pc;
    int gidx = 0;
    bool bad_block = false;
    while (cur.next(p, pc)) {
        for (int blk = pc.lo; blk < pc.hi; ++blk, ++gidx) {
            const int s = gidx % kStages, fill = gidx / kStages;
            if (fill > 0 && !mbar_wait(&sm.kv_empty[s], (fill - 1) & 1, &sm.abort)) goto drain;
            const int phys = blk < p.bt_stride ? __ldg(&p.block_table[(size_t)pc.seq * p.bt_stride + blk]) : -1;
            if (phys < 0 || (int64_t)phys >= p.num_blocks) {
                bad_block = true;
                mbar_arrive(&sm.kv_full[s]);  // consumers run on stale data; the error word reports it
                continue;
            }
            mbar_arrive_expect_tx(&sm.kv_full[s], kStageBytes);
            const int y = phys * kBlk;
            uint8_t *dst = sm.stage[s];
#pragma unroll
            for (int b = 0; b < 4; ++b)
                tma_load_2d(dst + b * kBoxBytes, map_lat, 256 * (int)half + 64 * b, y, &sm.kv_full[s], policy);
            tma_load_2d(dst + 4 * kBoxBytes, map_rope, 512 + 32 * (int)half, y, &sm.kv_full[s], policy);
        }
    }
drain:
    if (bad_block) raise_error(kErrBounds);
    // every load still in flight must land before the CTA may exit
    for (int k = max(0, gidx - kStages); k < gidx; ++k) {
        const long long t0 = clock64();
        while (!mbar_test(&sm.kv_full[k % kStages], (k / kStages) & 1) && clock64() - t0 < kSpinCycles) {
        }
    }
}

// ---------------------------------------------------------------- MMA warp
// Lane 0 waits on the barriers and issues every tcgen05 MMA/commit; the whole warp zeroes
// the cache rows past a sequence's end in that sequence's last block (undefined contents --
// possibly NaN -- must not reach Gemm2 even with zero probabilities) before lane 0 issues.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort, int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, abort);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ void zero_tail_rows(uint8_t *st, int valid, int lane) {
    const int zr = kBlk - valid;
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int e = lane; e < 4 * zr * 8; e += 32) {  // four 128-byte-swizzled boxes: 8 chunks per row
        const int b = e / (zr * 8), rem = e % (zr * 8);
        *reinterpret_cast<uint4 *>(st + b * kBoxBytes + (valid + rem / 8) * 128 + (rem % 8) * 16) = z;
    }
    for (int e = lane; e < zr * 4; e += 32)  // rotary box: 4 chunks per 64-byte row
        *reinterpret_cast<uint4 *>(st + 4 * kBoxBytes + (valid + e / 4) * 64 + (e % 4) * 16) = z;
    fence_proxy_async_smem();  // generic-proxy writes visible to the tensor core
    __syncwarp();
}

__device__ void mma_warp(Smem &sm, const DecodeParams &p, const int32_t *meta, uint32_t tmem) {
    constexpr uint32_t id1 = idesc_bf16_f32(128, 64, 0);   // S = Q K^T: K-major B
    constexpr uint32_t id2 = idesc_bf16_f32(128, 256, 1);  // O += P V: MN-major B
    const int lane = threadIdx.x & 31;
    Cursor cur;
    cur.init(meta, p.batch);
    Piece pc;
    int gidx = 0, piece_k = 0;
    volatile int *abort = &sm.abort;

    // O += P_b V_b for block b (global index); first == first block of its piece
    auto gemm2 = [&](int b, bool first) -> bool {
        if (!warp_wait(&sm.p_full, b & 1, abort, lane)) return false;
        if (first && piece_k > 0 && !warp_wait(&sm.o_free, (piece_k - 1) & 1, abort, lane)) return false;
        if (lane == 0) {
            tc_fence_after();
            const uint32_t st = smem_addr(sm.stage[b % kStages]);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts(tmem + kTmemO, tmem + kTmemP + 8 * kk, smem_desc(st + kk * 2048, 4 * 2048, 1024, 2), id2,
                       (!first || kk > 0) ? 1u : 0u);
            mma_commit(&sm.p_free);
            mma_commit(&sm.kv_empty[b % kStages]);
        }
        __syncwarp();
        return true;
    };

    while (cur.next(p, pc)) {
        if (!warp_wait(&sm.q_full, piece_k & 1, abort, lane)) goto done;
        {
            const int nb = pc.hi - pc.lo;
            for (int j = 0; j < nb; ++j, ++gidx) {
                const int s = gidx % kStages;
                if (!warp_wait(&sm.kv_full[s], (gidx / kStages) & 1, abort, lane)) goto done;
                if (is_tail_block(pc, pc.lo + j)) zero_tail_rows(sm.stage[s], pc.n - (pc.lo + j) * kBlk, lane);
                if (gidx > 0 && !warp_wait(&sm.s_free, (gidx - 1) & 1, abort, lane)) goto done;
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t st = smem_addr(sm.stage[s]);
#pragma unroll
                    for (int k = 0; k < 18; ++k) {
                        const uint64_t bd = k < 16 ? smem_desc(st + (k >> 2) * kBoxBytes + (k & 3) * 32, 16, 1024, 2)
                                                   : smem_desc(st + 4 * kBoxBytes + (k - 16) * 32, 16, 512, 4);
                        mma_ts(tmem + kTmemS, tmem + kTmemQ + 8 * k, bd, id1, k > 0 ? 1u : 0u);
                    }
                    mma_commit(&sm.s_full);
                }
                __syncwarp();
                if (j > 0 && !gemm2(gidx - 1, j == 1)) goto done;
            }
            if (!gemm2(gidx - 1, nb == 1)) goto done;
            if (lane == 0) mma_commit(&sm.o_full);
            __syncwarp();
            ++piece_k;
        }
    }
done:
    // all issued MMAs complete before teardown (bounded; independent of the abort flag)
    if (lane == 0) {
        mma_commit(&sm.mma_done);
        const long long t0 = clock64();
        while (!mbar_test(&sm.mma_done, 0) && clock64() - t0 < kSpinCycles) {
        }
    }
    __syncwarp();
}

// ---------------------------------------------------------------- softmax / epilogue (warps 4-7)
__device__ __forceinline__ void load_q(const DecodeParams &p, const Piece &pc, int r, bool row_ok, uint32_t half,
                                       uint32_t taddr) {
    const uint4 *qrow = reinterpret_cast<const uint4 *>(p.q + ((size_t)pc.seq * p.rows + (row_ok ? r : 0)) * kDqk);
#pragma unroll 1
    for (int c16 = 0; c16 < 9; ++c16) {  // 9 x 16 columns = 288 bf16 (256 latent + 32 rotary)
        uint32_t w[16];
        const int off = c16 < 8 ? (256 * (int)half + 32 * c16) / 8 : (512 + 32 * (int)half) / 8;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 x = row_ok ? __ldg(qrow + off + v) : make_uint4(0, 0, 0, 0);
            w[4 * v + 0] = x.x;
            w[4 * v + 1] = x.y;
            w[4 * v + 2] = x.z;
            w[4 * v + 3] = x.w;
        }
        tmem_st16(taddr + 16 * c16, w);
    }
    tmem_wait_st();
}

__device__ void softmax_role(Smem &sm, const DecodeParams &p, const int32_t *meta, uint32_t tmem, uint32_t half,
                             int group) {
    const int i = threadIdx.x - 128;  // row within the group == TMEM lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int r = group * 128 + i;
    const bool row_ok = r < p.rows;
    const bool warp_ok = group * 128 + wq * 32 < p.rows;
    const int nvalid_warps = min(4, (p.rows - group * 128 + 31) / 32);
    const uint32_t xbytes = (uint32_t)nvalid_warps * 32 * 16 * 16;
    const int t_q = row_ok ? r / p.h_q : 0, h_idx = row_ok ? r % p.h_q : 0;
    const uint32_t peer = half ^ 1u;
    const uint32_t xchg_peer = map_to_rank(&sm.xchg[0][0][0], peer);
    const uint32_t xfull_peer0 = map_to_rank(&sm.xfull[0], peer);
    volatile int *abort = &sm.abort;
    const float sl2 = p.scale_log2;

    Cursor cur;
    cur.init(meta, p.batch);
    Piece pc;
    bool have = cur.next(p, pc);
    if (have) {
        if (warp_ok) load_q(p, pc, r, row_ok, half, tmem + kTmemQ + lane_off);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.q_full);
    }
    int gidx = 0, piece_k = 0;
    while (have) {
        const Piece cp = pc;
        const int vis = row_ok ? visible_keys(cp.n, p.s_q, t_q, p.causal) : 0;
        float m_ref = -INFINITY, l = 0.f;
        const int nb = cp.hi - cp.lo;
        for (int j = 0; j < nb; ++j, ++gidx) {
            const int slot = gidx & 1;
            if (threadIdx.x == 128) mbar_arrive_expect_tx(&sm.xfull[slot], xbytes);
            if (!mbar_wait(&sm.s_full, gidx & 1, abort)) return;
            tc_fence_after();
            uint32_t sv[64];
            if (warp_ok) {
                uint32_t (&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
                uint32_t (&b)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
                tmem_ld32(tmem + kTmemS + lane_off, a);
                tmem_ld32(tmem + kTmemS + lane_off + 32, b);
                tmem_wait_ld();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.s_free);
            // swap partial scores with the peer CTA
            if (warp_ok) {
                const uint32_t dst = xchg_peer + (uint32_t)((slot * 16) * 128 + i) * 16;
                const uint32_t bar = xfull_peer0 + slot * 8;
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4)
                    st_async_v4(dst + c4 * 128 * 16, __uint_as_float(sv[4 * c4]), __uint_as_float(sv[4 * c4 + 1]),
                                __uint_as_float(sv[4 * c4 + 2]), __uint_as_float(sv[4 * c4 + 3]), bar);
            }
            if (!mbar_wait_cluster(&sm.xfull[slot], (gidx >> 1) & 1, abort)) return;
            bool need = false;
            float alpha = 1.f;
            uint32_t pk[32];
            if (warp_ok) {
                const int key0 = (cp.lo + j) * kBlk;
                float s[64];
                float mb = -INFINITY;
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const float4 o = sm.xchg[slot][c4][i];
                    const float po[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 4 * c4 + e;
                        const float v = (__uint_as_float(sv[c]) + po[e]) * sl2;
                        s[c] = key0 + c < vis ? v : -INFINITY;
                        mb = fmaxf(mb, s[c]);
                    }
                }
                if (j == 0) {
                    m_ref = mb;
                } else if (mb > m_ref + kRescaleThreshold) {
                    if (m_ref == -INFINITY) {
                        m_ref = mb;  // nothing accumulated yet (O and l are zero)
                    } else {
                        alpha = exp2f(m_ref - mb);
                        m_ref = mb;
                        l *= alpha;
                        need = true;
                    }
                }
                float sum = 0.f;
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const float p0 = m_ref == -INFINITY ? 0.f : exp2f(s[c] - m_ref);
                    const float p1 = m_ref == -INFINITY ? 0.f : exp2f(s[c + 1] - m_ref);
                    sum += p0 + p1;
                    __nv_bfloat162 two = __floats2bfloat162_rn(p0, p1);
                    pk[c >> 1] = *reinterpret_cast<uint32_t *>(&two);
                }
                l += sum;
            }
            // P buffer and O are free once Gemm2 of the previous block has completed
            if (gidx > 0 && !mbar_wait(&sm.p_free, (gidx - 1) & 1, abort)) return;
            tc_fence_after();
            if (warp_ok) {
                if (__any_sync(0xffffffffu, need)) {
                    const float a = need ? alpha : 1.f;
#pragma unroll 1
                    for (int c = 0; c < 8; ++c) {
                        uint32_t v[32];
                        tmem_ld32(tmem + kTmemO + lane_off + 32 * c, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * a);
                        tmem_st32(tmem + kTmemO + lane_off + 32 * c, v);
                    }
                }
                tmem_st32(tmem + kTmemP + lane_off, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full);
        }
        // the last Gemm1 of this piece has completed: Q may be replaced by the next piece's
        have = cur.next(p, pc);
        if (have) {
            if (warp_ok) load_q(p, pc, r, row_ok, half, tmem + kTmemQ + lane_off);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_full);
        }
        // epilogue of piece cp
        if (!mbar_wait(&sm.o_full, piece_k & 1, abort)) return;
        tc_fence_after();
        if (warp_ok) {
            const bool empty = !(l > 0.f);
            const float inv = empty ? 0.f : 1.f / l;
            const float lse = empty ? -INFINITY : (m_ref + log2f(l)) * 0.69314718055994530942f;
            const bool whole = cp.nsplit == 1;
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + kTmemO + lane_off + 32 * c, v);
                tmem_wait_ld();
                if (!row_ok) continue;
                if (whole) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((size_t)cp.seq * p.rows + r) * kDv +
                                                           256 * half + 32 * c);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 two = __floats2bfloat162_rn(__uint_as_float(v[8 * q4 + 2 * e]) * inv,
                                                                       __uint_as_float(v[8 * q4 + 2 * e + 1]) * inv);
                            w[e] = *reinterpret_cast<uint32_t *>(&two);
                        }
                        dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(p.o_part + ((size_t)cp.slot * p.rows + r) * kDv +
                                                             256 * half + 32 * c);
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        dst[q4] = make_float4(__uint_as_float(v[4 * q4]) * inv, __uint_as_float(v[4 * q4 + 1]) * inv,
                                              __uint_as_float(v[4 * q4 + 2]) * inv,
                                              __uint_as_float(v[4 * q4 + 3]) * inv);
                }
            }
            if (row_ok && half == 0) {
                if (whole)
                    p.lse[((size_t)cp.seq * p.h_q + h_idx) * p.s_q + t_q] = lse;
                else
                    p.lse_part[(size_t)cp.slot * p.rows + r] = lse;
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.o_free);
        ++piece_k;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
decode_sm100_kernel(const __grid_constant__ CUtensorMap map_lat, const __grid_constant__ CUtensorMap map_rope,
                    const DecodeParams p, const int groups) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t half = cluster_ctarank();
    const int cluster = blockIdx.x >> 1;
    const int part = cluster / groups, group = cluster % groups;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t *meta = p.tile_meta + (size_t)part * kMetaInts;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.kv_full[s], 1);
            mbar_init(&sm.kv_empty[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.s_free, 4);
        mbar_init(&sm.p_full, 4);
        mbar_init(&sm.p_free, 1);
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.o_free, 4);
        mbar_init(&sm.q_full, 4);
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.xfull[0], 1);
        mbar_init(&sm.xfull[1], 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&map_lat);
        prefetch_tensormap(&map_rope);
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();  // the peer's barriers exist before any exchange targets them
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        if (lane == 0) producer(sm, p, &map_lat, &map_rope, meta, half);
    } else if (warp == 1) {
        mma_warp(sm, p, meta, tmem);
    } else if (warp >= 4) {
        softmax_role(sm, p, meta, tmem, half, group);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && sm.abort) raise_error(kErrTimeout);
    cluster_sync();  // the peer no longer writes into this CTA's shared memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}
}  // namespace dec

size_t decode_sm100_smem_bytes() { return sizeof(dec::Smem) + 1024; }

cudaError_t launch_decode_sm100(const DecodeParams &p, const CUtensorMap &map_lat, const CUtensorMap &map_rope,
                                cudaStream_t stream) {
    const int groups = (p.rows + 127) / 128;
    const size_t smem = decode_sm100_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(dec::decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * p.num_parts * groups, 1, 1);
    cfg.blockDim = dim3(dec::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, dec::decode_sm100_kernel, map_lat, map_rope, p, groups);
}

}  // namespace mla
