// head_gemm.cu -- the per-head projections on either side of decode attention, as GEMMs on the
// tcgen05 tensor cores: for every head h, Y_h (m x n) = X_h (m x k) W_h (k x n), bf16 in, fp32
// accumulated in tensor memory, bf16 out (round to nearest even). With the up-projections absorbed
// ("Deep analysis of the DeepSeek Infra open-source releases", DAY1 FlashMLA: the kernel is fed
// latent queries and its latent outputs are projected afterwards, feature (4) "Gemm" context), the
// query side is q_latent = q_nope W_UK (k 128, n 512) and the output side o = o_latent W_UV
// (k 512, n 128).
//
// One CTA per (128-row tile, head, 256-column tile): TMA brings 64-wide k-chunks of X (K-major,
// 128-byte swizzle) and of W (read MN-major: boxes of 64 k-rows x 64 columns) into a 2-stage
// mbarrier ring; one thread issues 4 MMAs (M 128, N <= 256, K 16) per chunk into a TMEM
// accumulator; the four warps then read one row each per lane and store bf16. Rows past m are
// zero-filled by TMA and not stored. Every wait is bounded.
#include "common.cuh"
#include "sm100_ptx.cuh"

namespace mla {
using namespace sm100;

namespace hg {
constexpr int kM = 128, kKc = 64, kStages = 2, kMaxN = 256;
constexpr int kABytes = kM * kKc * 2;  // 16 KB: 128 rows x 64 k
constexpr int kBBox = kKc * 64 * 2;     // 8 KB: 64 k-rows x 64 columns

struct __align__(1024) Smem {
    uint8_t a[kStages][kABytes];
    uint8_t b[kStages][(kMaxN / 64) * kBBox];
    uint64_t full[kStages], empty[kStages], done;
    uint32_t tmem_base;
    int abort;
};

struct Params {
    __nv_bfloat16 *y;
    int64_t ldy, y_head;  // elements
    int64_t x_head;       // elements: column of head h's X_h within a row of X
    int m, n, k, heads;
    int y_v8;             // y, ldy and y_head allow 32-byte stores (else 16-byte ones)
};

__global__ void __launch_bounds__(128, 1)
head_gemm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int ntiles = (p.n + kMaxN - 1) / kMaxN;
    const int nt = blockIdx.x % ntiles, h = (blockIdx.x / ntiles) % p.heads, mt = blockIdx.x / (ntiles * p.heads);
    const int n0 = nt * kMaxN, NT = min(kMaxN, p.n - n0), m0 = mt * kM;
    const uint32_t cols = NT <= 64 ? 64u : (NT <= 128 ? 128u : 256u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunks = p.k / kKc;

    if (warp == 1) tmem_alloc(&sm.tmem_base, cols);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.done, 1);
        sm.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&map_x);
        prefetch_tensormap(&map_w);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0 && lane == 0) {  // TMA producer
        const uint64_t policy = l2_evict_first_policy();
        int issued = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            if (c >= kStages && !mbar_wait(&sm.empty[s], (c / kStages - 1) & 1, &sm.abort)) break;
            mbar_arrive_expect_tx(&sm.full[s], kABytes + (NT / 64) * kBBox);
            tma_load_2d(sm.a[s], &map_x, (int)(h * p.x_head) + c * kKc, m0, &sm.full[s], policy);
            for (int j = 0; j < NT / 64; ++j)
                tma_load_2d(sm.b[s] + j * kBBox, &map_w, n0 + 64 * j, h * p.k + c * kKc, &sm.full[s], policy);
            issued = c + 1;
        }
        // every load still in flight must land before the CTA may exit
        for (int c = max(0, issued - kStages); c < issued; ++c) {
            const long long t0 = clock64();
            while (!mbar_sleep_test(&sm.full[c % kStages], (c / kStages) & 1) && clock64() - t0 < kSpinCycles) {
            }
        }
    } else if (warp == 1 && lane == 0) {  // MMA issuer
        const uint32_t idesc = idesc_bf16_f32(kM, NT, 1);  // A K-major, B MN-major
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c % kStages;
            ok = mbar_wait(&sm.full[s], (c / kStages) & 1, &sm.abort);
            if (!ok) break;
            tc_fence_after();
            const uint64_t ad = smem_desc(smem_addr(sm.a[s]), 16, 1024, 2);
            const uint64_t bd = smem_desc(smem_addr(sm.b[s]), kBBox, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < kKc / 16; ++kk)  // A: +32 bytes per k-step; B: +16 rows of 128 bytes
                mma_ss(tmem, ad + 2 * kk, bd + 128 * kk, idesc, (c > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&sm.empty[s]);
        }
        mma_commit(&sm.done);  // every MMA this thread issued has completed (also on the error path)
    }
    __syncwarp();
    // epilogue: lane = row of the tile; warp w reads TMEM lanes [32w, 32w + 32)
    const bool ok = mbar_wait(&sm.done, 0, &sm.abort);
    tc_fence_after();
    const int r = m0 + warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    if (ok) {
        for (int c16 = 0; c16 < NT / 16; ++c16) {
            uint32_t v[16];
            tmem_ld16(tmem + lane_off + 16 * c16, v);
            tmem_wait_ld();
            if (r < p.m && !sm.abort) {
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    __nv_bfloat162 two = __floats2bfloat162_rn(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                    w[j] = *reinterpret_cast<uint32_t *>(&two);
                }
                // each lane writes its own row, so the number of stores sets the epilogue's time
                __nv_bfloat16 *dst = p.y + (int64_t)r * p.ldy + h * p.y_head + n0 + 16 * c16;
                if (p.y_v8) {
                    st_global_v8(dst, w);
                } else {
                    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    reinterpret_cast<uint4 *>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && sm.abort) raise_error(kErrTimeout);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, cols);
    }
}
}  // namespace hg

size_t head_gemm_smem_bytes() { return sizeof(hg::Smem) + 1024; }

cudaError_t launch_head_gemm(const CUtensorMap &map_x, const CUtensorMap &map_w, __nv_bfloat16 *y, int64_t ldy,
                             int64_t y_head, int64_t x_head, int m, int n, int k, int heads, cudaStream_t stream) {
    hg::Params p;
    p.y = y;
    p.ldy = ldy;
    p.y_head = y_head;
    p.x_head = x_head;
    p.m = m;
    p.n = n;
    p.k = k;
    p.heads = heads;
    p.y_v8 = (reinterpret_cast<uintptr_t>(y) % 32) == 0 && (ldy * 2) % 32 == 0 && (y_head * 2) % 32 == 0;
    const size_t smem = head_gemm_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(hg::head_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)((m + hg::kM - 1) / hg::kM) * heads * ((n + hg::kMaxN - 1) / hg::kMaxN);
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    hg::head_gemm_kernel<<<(unsigned)grid, 128, smem, stream>>>(map_x, map_w, p);
    return cudaGetLastError();
}

}  // namespace mla
