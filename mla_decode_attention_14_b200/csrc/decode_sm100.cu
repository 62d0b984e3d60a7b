// decode_sm100.cu -- the B200 (sm_100a) split kernel of MLA decode attention.
//
// What it computes (per query row r of sequence b, over that sequence's visible keys j):
// S_j = scale * <q_r, k_j> over all 576 latent+rotary dims ("Gemm1"), an online softmax in
// fp32, and O = sum_j softmax_j * k_j[0:512] ("Gemm2"). "Deep analysis of the DeepSeek Infra
// open-source releases" (jingzhunhuoke.net/55333.html), DAY1 FlashMLA: the cache is kept in
// 64-token blocks (feature (2)), the kernel streams each block once and runs Gemm1 then Gemm2
// on it (feature (4)), and lengths are load-balanced over the SMs (feature (5)).
//
// How (B200 design; the pages' Hopper design is prior art only):
//  * One 2-CTA cluster per (work part, group of 128 query rows); 74 clusters fill the 148 SMs.
//    The fp32 accumulator O for 128 rows x 512 value dims is 256 KB -- all of one SM's tensor
//    memory -- so each CTA of the pair owns HALF of the value dims (O: 128 lanes x 256 columns
//    of TMEM) and streams only the cache columns it needs: CTA h loads latent dims
//    [256h, 256h+256) and rotary dims [512+32h, 512+32h+32), i.e. exactly half of every block
//    (36,864 bytes); the pair together reads each block once.
//  * Gemm1 is split along its 576-long contraction: CTA h computes the partial scores over its
//    288 dims (18 tcgen05 MMAs, M=128 rows, N=64 tokens, into one accumulator; the latent part
//    of Q is the A operand in TMEM, the rotary part in shared memory).
//  * The pair combines the partial scores multiplicatively: 2^(s0 + s1 - m) =
//    2^(s0 - m0) * 2^(s1 - m1) * 2^(m0 + m1 - m). Each CTA computes, for its own partial with
//    its own row offset m, R = 2^((s - m)/2 + 15) -- the square root of its factor, scaled --
//    keeps it in fp32, and sends it to the peer as fp16 together with m in fp32: st.async
//    stores into the peer's 2-slot receive ring complete on the peer's mbarrier. R lies in
//    [0, 2^15] and is normal in fp16 while s - m >= -58, so the exchange keeps a relative
//    precision of 2^-10 (once squared) over 58 octaves of partial score whatever the score
//    magnitude (rows whose two partial maxima overstate the true maximum by up to ~34 octaves
//    lose nothing), and the traffic is half that of fp32 scores. A row that goes past that range
//    is not lost silently: the softmax warps bound the error that subnormal peer factors add to
//    its sum and set the range bit of the device error word when it exceeds 2^-11 of the sum. The link between the two SMs
//    moves only about 20 bytes per cycle, so the stores are spread over the softmax warps'
//    compute.
//  * Eight softmax warps: warp w serves TMEM lane quarter w&3 (32 query rows) and one half of
//    every block's tokens; the two halves of a row agree on an upper bound of the block max
//    through shared memory, so both take the same lazy-rescaling decisions (O is rescaled only
//    when the running max grows by more than 2^8). P = (R_own R_peer)^2 2^(m0 + m1 - m - 60) goes
//    to TMEM as two bf16 terms (hi = P with its low 16 bits cleared, lo = the exact remainder
//    with its low 16 bits cleared; hi + lo is within 2^-14 of P), so P's rounding does not add
//    to the bf16 output rounding.
//  * Issuing a tcgen05 MMA occupies the issuing thread for about 70 cycles, so Gemm1 and Gemm2
//    have their own issuing warps and the tensor core runs both at once. The softmax warps read
//    the scores of block g+1 before they finish block g, so Gemm1 of block g+2 runs while
//    Gemm2 of block g waits for P.
//  * Gemm2: 8 MMAs (M=128, N=256, K=16 tokens; A = P_hi then P_lo from TMEM, B = the value half
//    of the same cache tile read MN-major): the block is loaded once for both GEMMs.
//  * Warp roles: warp 0 lane 0 = TMA producer (5-stage ring, block-table gather, L2
//    evict-first); warp 1 issues Gemm1 and owns the TMEM allocation; warp 3 issues Gemm2 and
//    zeroes the cache rows past a sequence's end before Gemm2 reads them, so undefined tail
//    contents never reach the result; warps 4-11 = softmax, correction and epilogue (a warp may
//    only touch TMEM lane quarter w & 3). Warpgroup 0 hands registers to the softmax warps.
//  * Pieces of split sequences leave fp32 partial O and lse in the workspace for the combine
//    kernel; whole sequences are written straight to bf16 out / fp32 lse.
//  * The two softmax warps of an SM sub-partition move in lockstep (the per-row barrier) and
//    share its issue slots, so their instruction count sets the pace: the per-token-pair
//    arithmetic uses the packed f32x2 instructions and block maxima the three-input max.
//  * The same kernel, instantiated with F8 = true, reads an FP8 latent cache (640-byte token
//    records: 512 E4M3 latent bytes, 64 bf16 rotary dims): TMA loads the E4M3 boxes into the
//    upper half of each stage, four converter warps (warps 4-7) expand them in place to the fp16
//    layout above, Gemm1's latent MMAs and Gemm2 run in fp16, and P is a single fp16 term set
//    against the exact block max; the softmax warps are then warps 8-15.
// Every wait is bounded; a timeout sets the device error word and the CTA exits cleanly.
#include <cuda_fp16.h>

#include "common.cuh"
#include "schedule.cuh"
#include "sm100_ptx.cuh"

namespace mla {
using namespace sm100;

namespace dec {
constexpr int kStages = 5;
constexpr int kSoftWarps = 8;                     // two per SM sub-partition
// bf16 cache: warpgroup 0 = TMA producer, Gemm1 issuer, (idle), Gemm2 issuer; softmax from warp 4.
// fp8 cache: warpgroup 1 = four converter warps (one per SM sub-partition); softmax from warp 8.
// sparse mode (bf16 cache): warpgroup 1 = four gather warps; softmax from warp 8.
constexpr int kConvWarps = 4;
template <bool F8, bool SP = false> constexpr int first_soft_warp() { return (F8 || SP) ? 4 + kConvWarps : 4; }
template <bool F8, bool SP = false> constexpr int num_threads() {
    return 32 * (first_soft_warp<F8, SP>() + kSoftWarps);  // 384 / 512
}
constexpr int kTq = 2;                            // token halves per block
constexpr int kTokPer = kBlk / kTq;               // 32 tokens per softmax thread
// Register split (setmaxnreg): the launch gives 168 per thread (384 x 168 = 64,512); warpgroup 0
// drops to 96 and the two softmax warpgroups rise to 200: 128 x 96 + 256 x 200 = 63,488 <= 64,512.
// fp8 and sparse: 512 x 128 = 65,536 at launch; the control and converter (gather) warpgroups drop
// to 56: 2 x 128 x 56 + 256 x 200 = 65,536.
constexpr uint32_t kRegsControl = 96, kRegsSoftmax = 200, kRegsSmall = 56;
constexpr int kBoxBytes = kBlk * 128;                      // 64 tokens x 64 bf16 (128-byte swizzle)
constexpr int kRopeBoxBytes = kBlk * 64;                   // 64 tokens x 32 bf16 (64-byte swizzle)
constexpr int kStageBytes = 4 * kBoxBytes + kRopeBoxBytes;  // 36,864: half of one cache block
// fp8 cache (640-byte token records: 512 E4M3 latent bytes, then 64 bf16 rotary dims): the same
// stages. TMA puts the two 64-token x 128-byte E4M3 latent boxes (128-byte swizzle) where fp16
// boxes 2 and 3 go and the rotary box where it always goes; the converter warps then expand the
// latent in place into the four fp16 boxes, so both GEMMs read the bf16 layout (in fp16).
constexpr int kRawBoxBytes = kBlk * 128;                 // 64 tokens x 128 E4M3
constexpr int kF8LoadBytes = 2 * kRawBoxBytes + kRopeBoxBytes;  // 20,480 loaded per stage
constexpr int kRopeOffset = 4 * kBoxBytes;
constexpr float kRescaleThreshold = 8.0f;                  // log2 units: rescale O when max grows > 2^8
// The pair exchanges R = 2^((s - m) / 2 + 15), the square root of a factor, in fp16: R <= 2^15
// (< 65504), normal (full 11-bit precision) while s - m >= -58 and subnormal down to -78, so the
// exchange spans 58 octaves of score range at a relative precision of 2^-10 once squared (a
// factor sent directly would span only 29). P = (R_own R_peer)^2 2^(m0 + m1 - m_ref - 60).
constexpr float kXScaleLog2 = 15.0f;

// TMEM column map (512 columns allocated, 128 lanes = 128 query rows)
constexpr uint32_t kTmemO = 0;     // 256 fp32: O for this CTA's 256 value dims
constexpr uint32_t kTmemQ = 256;   // 128 x (2 bf16): this CTA's 256 latent query dims
constexpr uint32_t kTmemS = 384;   // 64 fp32: partial scores of a block
constexpr uint32_t kTmemPhi = 448; // 32 x (2 bf16): P with its low 16 bits cleared (the A operand of Gemm2);
                                   // fp8 cache: P as fp16 (the only term)
constexpr uint32_t kTmemPlo = 480; // 32 x (2 bf16): the remainder, likewise (bf16 cache only)
constexpr uint32_t kTmemCols = 512;
constexpr int kXchgEBytes = 2 * kBlk * 128 * 2;    // two slots of 128 rows x 64 fp16 factors
constexpr int kXchgOffBytes = 2 * kTq * 128 * 4;   // two slots of 128 rows x 2 fp32 offsets

struct __align__(1024) Smem {
    uint8_t stage[kStages][kStageBytes];  // KV ring
    uint4 xchg[(kXchgEBytes + kXchgOffBytes) / 16];  // peer factors R (fp16) [slot][token half][16 B][row]
                                                     // + row offsets (fp32) [slot][token half][row]
    float xmax[2][kTq][128];  // per-row exchange between the two token halves (block max bound; sums)
    uint8_t q_rope[128 * 64];             // rotary query dims [128 rows x 32], K-major, 64-byte swizzle
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t conv_full[kStages];  // fp8 cache: the stage's latent is in fp16
    uint64_t vmask[kStages];      // sparse mode: bit j = token j of the stage is a key
    uint64_t s_full, s_free, p_full, p_free, o_full, o_free, q_full, mma_done;
    uint64_t xfull[2];  // receive slots filled by the peer
    uint32_t tmem_base;
    int abort;
};

static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory (with 1 KB for alignment) must fit 227 KB");

// Walks the blocks of one part in order, with piece boundaries (SP: sparse mode).
template <bool SP = false>
struct BlockWalker {
    Cursor<SP> cur;
    Piece pc;
    int blk, piece_k;
    bool live;
    __device__ void init(const int32_t *meta, const DecodeParams &p) {
        cur.init(meta, p.batch);
        live = cur.next(p, pc);
        blk = live ? pc.lo : 0;
        piece_k = 0;
    }
    __device__ bool first() const { return blk == pc.lo; }
    __device__ bool last() const { return blk == pc.hi - 1; }
    __device__ bool tail() const { return blk == num_blocks_of(pc.n) - 1 && (pc.n % kBlk) != 0; }
    __device__ void advance(const DecodeParams &p) {
        if (blk + 1 < pc.hi) {
            ++blk;
            return;
        }
        live = cur.next(p, pc);
        if (live) {
            blk = pc.lo;
            ++piece_k;
        }
    }
};

// ---------------------------------------------------------------- TMA producer (1 thread)
template <bool F8>
__device__ void producer(Smem &sm, const DecodeParams &p, const CUtensorMap *map_lat, const CUtensorMap *map_rope,
                         const int32_t *meta, uint32_t half) {
    const uint64_t policy = l2_evict_first_policy();
    BlockWalker<> w;
    w.init(meta, p);
    int gidx = 0;
    bool bad_block = false;
    for (; w.live; w.advance(p), ++gidx) {
        const int s = gidx % kStages, fill = gidx / kStages;
        if (fill > 0 && !mbar_wait(&sm.kv_empty[s], (fill - 1) & 1, &sm.abort)) break;
        const int phys = w.blk < p.bt_stride ? __ldg(&p.block_table[(size_t)w.pc.seq * p.bt_stride + w.blk]) : -1;
        if (phys < 0 || (int64_t)phys >= p.num_blocks) {
            bad_block = true;
            mbar_arrive(&sm.kv_full[s]);  // consumers run on stale data; the error word reports it
            continue;
        }
        mbar_arrive_expect_tx(&sm.kv_full[s], F8 ? kF8LoadBytes : kStageBytes);
        const int y = phys * kBlk;
        uint8_t *dst = sm.stage[s];
        // the latent boxes of this half in ONE 3-D operation (an SM's TMA unit works through about one
        // operation at a time, so few large ones keep the stream at HBM speed), then the rotary box
        if constexpr (F8)  // coordinates: bytes of the record (latent), bf16 elements (rotary)
            tma_load_3d(dst + 2 * kBoxBytes, map_lat, 0, y, 2 * (int)half, &sm.kv_full[s], policy);
        else
            tma_load_3d(dst, map_lat, 0, y, 4 * (int)half, &sm.kv_full[s], policy);
        tma_load_2d(dst + kRopeOffset, map_rope, (F8 ? 256 : 512) + 32 * (int)half, y, &sm.kv_full[s], policy);
    }
    if (bad_block) raise_error(kErrBounds);
    // every load still in flight must land before the CTA may exit
    for (int k = max(0, gidx - kStages); k < gidx; ++k) {
        const long long t0 = clock64();
        while (!mbar_sleep_test(&sm.kv_full[k % kStages], (k / kStages) & 1) && clock64() - t0 < kSpinCycles) {
        }
    }
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort, int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, abort);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// ---------------------------------------------------------------- sparse mode: gather producers (4 warps)
// Block k of work unit u holds the keys listed at indices[u, 64k .. 64k+64). Gather warp h (warps
// 4-7) takes the block's tokens [16h, 16h + 16); its lane l < 16 resolves entry 16h + l: a position
// inside [0, seqlens[b]) is a key, read from cache row block_table[b, pos / 64] * 64 + pos % 64;
// anything else (or a list shorter than the block) is no key, copied as zeros. Then, token by
// token, the warp's 32 lanes copy this CTA's 512-byte latent half of the row, one 16-byte chunk
// each (one coalesced 512-byte read), and lanes 0-3 its 64-byte rotary half, with 16-byte
// asynchronous copies into the positions the stage's 128-byte (latent) and 64-byte (rotary)
// swizzles give them -- the layout the MMA descriptors read, which a TMA box cannot produce for
// single rows. Each warp stores its quarter of the stage's validity mask before its lane 0 arrives on
// kv_full, and each lane's copies complete on kv_full too (4 x 33 arrivals per fill).
// A warp keeps only ~9 KB of such copies in flight (measured: ~6k cycles to issue one block's
// 36 KB from one warp, ~3.5k from two), so the copies are split over a warpgroup. Resolving an entry takes two
// dependent loads (list, then block table), so the walk is pipelined: while block g is copied, the
// block-table entry of block g+1 and the list entry (and sequence length) of block g+2 are in flight.
constexpr int kGatherWarps = 4;
constexpr int kGatherTok = kBlk / kGatherWarps;  // 16 tokens of each block per gather warp
constexpr uint32_t kSparseFullArrivals = kGatherWarps * 33;

struct GatherAhead {  // this lane's list entry of one block, loaded ahead
    int pos, n, b;
};

__device__ __forceinline__ void gather_load_list(const DecodeParams &p, const BlockWalker<true> &w, int e_off,
                                                 GatherAhead &a) {
    a.b = w.live ? w.pc.seq / p.sp_sq : 0;
    a.n = w.live ? max(__ldg(&p.seqlens[a.b]), 0) : 0;
    const int e = w.blk * kBlk + e_off;  // e_off < 0: this lane has no entry
    a.pos = w.live && e_off >= 0 && e < p.topk ? __ldg(&p.indices[(size_t)w.pc.seq * p.topk + e]) : -1;
}

// the cache row (physical block * 64 + slot) of the entry, or -1
__device__ __forceinline__ int gather_resolve(const DecodeParams &p, const GatherAhead &a, bool &bad_entry) {
    const int pos = a.pos;
    if (pos < 0 || pos >= a.n) return -1;
    const int blk = pos / kBlk;
    const int phys = blk < p.bt_stride ? __ldg(&p.block_table[(size_t)a.b * p.bt_stride + blk]) : -1;
    if (phys >= 0 && (int64_t)phys < p.num_blocks) return phys * kBlk + pos % kBlk;
    bad_entry = true;  // reported; the entry is treated as no key
    return -1;
}

__device__ void gather_producer(Smem &sm, const DecodeParams &p, const int32_t *meta, uint32_t half, int gw) {
    const int lane = threadIdx.x & 31;
    const int t0 = kGatherTok * gw;  // this warp's tokens of each block
    const int e_off = lane < kGatherTok ? t0 + lane : -1;  // lanes past the warp's tokens resolve nothing
    volatile int *abort = &sm.abort;
    const char *kv = reinterpret_cast<const char *>(p.kv);
    bool bad_entry = false;
    // w: the block being copied; w2: two blocks ahead (its list entries are loaded)
    BlockWalker<true> w, w2;
    w.init(meta, p);
    w2 = w;
    GatherAhead a1, a2;  // list entries of blocks g+1 and g+2
    gather_load_list(p, w, e_off, a1);
    int row = gather_resolve(p, a1, bad_entry);  // block g
    if (w2.live) w2.advance(p);
    gather_load_list(p, w2, e_off, a1);
    if (w2.live) w2.advance(p);
    int gidx = 0;
    for (; w.live; w.advance(p), ++gidx) {
        gather_load_list(p, w2, e_off, a2);  // block g+2
        if (w2.live) w2.advance(p);
        const int s = gidx % kStages, fill = gidx / kStages;
        if (fill > 0 && !warp_wait(&sm.kv_empty[s], (fill - 1) & 1, abort, lane)) break;
        const uint32_t mask = __ballot_sync(0xffffffffu, row >= 0) & ((1u << kGatherTok) - 1);
        const uint32_t dst = smem_addr(sm.stage[s]);
#pragma unroll 4
        for (int k = 0; k < kGatherTok; ++k) {
            const int t = t0 + k;
            const int r = __shfl_sync(0xffffffffu, row, k);
            const uint32_t bytes = r >= 0 ? 16u : 0u;  // 0: the chunk is zero-filled, nothing is read
            const char *src = kv + (size_t)(r >= 0 ? r : 0) * (kDqk * 2);
            // latent chunk `lane` of this half: dims 256 half + 8 lane, box lane / 8, chunk lane % 8
            cp_async_16(dst + (lane >> 3) * kBoxBytes + t * 128 + (((lane & 7) ^ (t & 7)) << 4),
                        src + (256 * half + 8 * lane) * 2, bytes);
            if (lane < 4)  // rotary chunk `lane`: dims 512 + 32 half + 8 lane (64-byte swizzle)
                cp_async_16(dst + kRopeOffset + t * 64 + ((lane ^ ((t >> 1) & 3)) << 4),
                            src + (512 + 32 * half + 8 * lane) * 2, bytes);
        }
        if (lane == 0) {
            reinterpret_cast<uint16_t *>(&sm.vmask[s])[gw] = (uint16_t)mask;  // bits 16 gw .. 16 gw + 15
            mbar_arrive(&sm.kv_full[s]);
        }
        cp_async_mbar_arrive_noinc(&sm.kv_full[s]);
        row = gather_resolve(p, a1, bad_entry);  // block g+1
        a1 = a2;
    }
    if (bad_entry) raise_error(kErrBounds);
    cp_async_wait_all();  // every copy lands before the CTA may exit
}

// ---------------------------------------------------------------- MMA issuing warps

// Zero the cache rows past a sequence's end in its last block (undefined contents -- possibly
// NaN -- must not reach Gemm2 even with zero probabilities).
__device__ void zero_tail_rows(uint8_t *st, int valid, int lane) {
    const int zr = kBlk - valid;
    const uint4 z = make_uint4(0, 0, 0, 0);
    // (whole rows are zeroed, so the swizzle, a permutation within each row, does not matter; shifts,
    // not divisions: this runs on Gemm2's issuing warp right before the last block's MMAs)
    for (int e = lane; e < zr * 8; e += 32) {  // chunk e % 8 of tail row e / 8 in each of the four boxes
        const int off = (valid + (e >> 3)) * 128 + ((e & 7) << 4);
#pragma unroll
        for (int b = 0; b < 4; ++b) *reinterpret_cast<uint4 *>(st + b * kBoxBytes + off) = z;
    }
    for (int e = lane; e < zr * 4; e += 32)  // rotary box: 4 chunks per 64-byte row
        *reinterpret_cast<uint4 *>(st + 4 * kBoxBytes + (valid + (e >> 2)) * 64 + ((e & 3) << 4)) = z;
    fence_proxy_async_smem();  // generic-proxy writes visible to the tensor core
    __syncwarp();
}

// fp8 cache, warps 4-7: the latent half of every block from E4M3 to fp16 bit patterns, in place,
// into the layout the MMA descriptors read (the bf16 stage's four 128-byte-swizzled boxes of 64
// tokens x 64 dims). Raw box 0 (in fp16 box 2's place) becomes boxes 0-1; after a barrier of the four
// warps, raw box 1 (in box 3's place) becomes boxes 2-3: every row of box 3 is written by the
// instruction that read the same row of raw box 1, so the expansion never overwrites unread bytes.
// The E4M3 byte s.eeee.mmm placed as the fp16 pattern s.0eeee.mmm0000000 is the fp16 number
// e4m3 * 2^-8 -- exactly, subnormals included (both formats put the subnormal point at exponent
// field 0) -- so the conversion is four integer operations per pair of values (byte permute, mask,
// shift, merge); the 2^-8 is folded into the score and output scales. (The hardware e4m3x2 -> f16x2
// conversion took ~8k cycles per block on one warp.) Rows past a sequence's end are written as
// zeros, so undefined tail contents never reach Gemm2. Lane mapping: each group of 8 lanes takes
// 16-byte chunks 0-3 of one row of a row pair and chunks 4-7 of the other row, so the group's reads
// (one chunk each) and writes (two chunks each) fall on 8 distinct bank groups.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_scaled(uint32_t w, uint32_t sel) {
    const uint32_t t = __byte_perm(w, 0u, sel);  // the two bytes at bits 8-15 and 24-31
    return (t & 0x80008000u) | ((t & 0x7f007f00u) >> 1);
}

constexpr int kConvBarrier = 5;  // named barrier of the four converter warps (1-4: softmax row pairs)

__device__ void convert_warp(Smem &sm, const DecodeParams &p, const int32_t *meta) {
    const int lane = threadIdx.x & 31, cw = (threadIdx.x >> 5) & (kConvWarps - 1);
    const int u = lane & 7, hp = (lane >> 3) & 1, pq = lane >> 4;  // chunk, half of the pair, pair of the step
    const int k0 = 2 * (u & 3);                                     // first fp16 chunk of the box row
    volatile int *abort = &sm.abort;
    BlockWalker<> w;
    w.init(meta, p);
    for (int g = 0; w.live; w.advance(p), ++g) {
        const int s = g % kStages;
        if (!warp_wait(&sm.kv_full[s], (g / kStages) & 1, abort, lane)) break;
        const int valid = w.tail() ? w.pc.n - w.blk * kBlk : kBlk;
        uint8_t *dst = sm.stage[s];
#pragma unroll 1
        for (int bx = 0; bx < 2; ++bx) {  // raw box bx: 32 row pairs, 4 steps of 2 pairs per warp
            if (bx == 1) named_bar_sync(kConvBarrier, 32 * kConvWarps);  // raw box 0 read by all four warps
#pragma unroll
            for (int it = 16 * bx + cw; it < 16 * bx + 16; it += kConvWarps) {
                const int pi = 2 * it + pq;  // row pair over both raw boxes: 2 x 32 pairs
                const int row = 2 * (pi & 31) + ((u >> 2) ^ hp), sw = row & 7;
                uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
                if (row < valid) {
                    const uint4 x =
                        *reinterpret_cast<const uint4 *>(dst + (2 + bx) * kBoxBytes + row * 128 + ((u ^ sw) << 4));
                    // bytes 0,1 -> word 0; bytes 2,3 -> word 1 (little-endian: the lower dim in the low half)
                    lo = make_uint4(e4m3x2_to_f16x2_scaled(x.x, 0x1404u), e4m3x2_to_f16x2_scaled(x.x, 0x3424u),
                                    e4m3x2_to_f16x2_scaled(x.y, 0x1404u), e4m3x2_to_f16x2_scaled(x.y, 0x3424u));
                    hi = make_uint4(e4m3x2_to_f16x2_scaled(x.z, 0x1404u), e4m3x2_to_f16x2_scaled(x.z, 0x3424u),
                                    e4m3x2_to_f16x2_scaled(x.w, 0x1404u), e4m3x2_to_f16x2_scaled(x.w, 0x3424u));
                }
                uint8_t *o = dst + (2 * bx + (u >> 2)) * kBoxBytes + row * 128;
                *reinterpret_cast<uint4 *>(o + ((k0 ^ sw) << 4)) = lo;
                *reinterpret_cast<uint4 *>(o + (((k0 + 1) ^ sw) << 4)) = hi;
            }
        }
        fence_proxy_async_smem();  // generic-proxy writes visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.conv_full[s]);  // one arrival per converter warp
    }
}

// Issuing one tcgen05 MMA occupies the issuing thread for about 70 cycles whatever its size, so
// Gemm1 and Gemm2 are issued by two warps: the tensor core takes MMAs from both at once.

// Gemm1 of every block into S (partial scores over this CTA's 288 dims): 18 MMAs into one
// accumulator; the next block's Gemm1 may start as soon as the softmax warps have read S.
// fp8 cache: the 16 latent MMAs are fp16 x fp16 (Q converted on load, K from the converted
// buffer), the 2 rotary MMAs stay bf16 x bf16 from the raw stage; both accumulate in fp32.
template <bool F8, bool SP>
__device__ void gemm1_warp(Smem &sm, const DecodeParams &p, const int32_t *meta, uint32_t tmem) {
    constexpr uint32_t id1 = idesc_bf16_f32(128, 64, 0);  // S = Q K^T: K-major B
    constexpr uint32_t id1_lat = F8 ? idesc_f16_f32(128, 64, 0) : id1;
    const int lane = threadIdx.x & 31;
    volatile int *abort = &sm.abort;
    BlockWalker<SP> w;
    w.init(meta, p);
    for (int g = 0; w.live; w.advance(p), ++g) {
        if (w.first() && !warp_wait(&sm.q_full, w.piece_k & 1, abort, lane)) break;
        const int s = g % kStages;
        if (!warp_wait(F8 ? &sm.conv_full[s] : &sm.kv_full[s], (g / kStages) & 1, abort, lane)) break;
        if (g > 0 && !warp_wait(&sm.s_free, (g - 1) & 1, abort, lane)) break;
        if (lane == 0) {
            if constexpr (SP) fence_proxy_async_smem();  // the gathered stage (generic-proxy copies) to the tensor core
            tc_fence_after();
            // descriptors: one base each, then constant offsets (address field is in 16-byte units)
            const uint64_t kd = smem_desc(smem_addr(sm.stage[s]), 16, 1024, 2);
            const uint64_t rd = smem_desc(smem_addr(sm.stage[s]) + kRopeOffset, 16, 512, 4);
            const uint64_t qd = smem_desc(smem_addr(sm.q_rope), 16, 512, 4);
#pragma unroll
            for (int k = 0; k < 16; ++k)  // latent k-steps, A (Q) from TMEM
                mma_ts(tmem + kTmemS, tmem + kTmemQ + 8 * k, kd + (uint64_t)(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4),
                       id1_lat, k > 0 ? 1u : 0u);
#pragma unroll
            for (int c = 0; c < 2; ++c)  // rotary k-steps, A from shared memory
                mma_ss(tmem + kTmemS, qd + 2 * c, rd + 2 * c, id1, 1u);
            mma_commit(&sm.s_full);
        }
        __syncwarp();
    }
}

// Gemm2 of every block, O (+)= (P_hi + P_lo) V, once the softmax warps have written P.
// fp8 cache: O (+)= P V with P and V in fp16, 4 MMAs.
template <bool F8, bool SP>
__device__ void gemm2_warp(Smem &sm, const DecodeParams &p, const int32_t *meta, uint32_t tmem) {
    constexpr uint32_t id2 = F8 ? idesc_f16_f32(128, 256, 1) : idesc_bf16_f32(128, 256, 1);  // MN-major B
    constexpr int kTerms = F8 ? 1 : 2;
    const int lane = threadIdx.x & 31;
    volatile int *abort = &sm.abort;
    BlockWalker<SP> w;
    w.init(meta, p);
    for (int g = 0; w.live; w.advance(p), ++g) {
        if (!warp_wait(&sm.p_full, g & 1, abort, lane)) break;
        if (w.first() && w.piece_k > 0 && !warp_wait(&sm.o_free, (w.piece_k - 1) & 1, abort, lane)) break;
        const int s = g % kStages;
        // P of block g exists, so Gemm1 of block g has completed and its tile may be edited (the fp8
        // path's converter has already zeroed the tail rows)
        // (sparse mode: entries that are no key were copied as zeros)
        if (!F8 && !SP && w.tail()) zero_tail_rows(sm.stage[s], w.pc.n - w.blk * kBlk, lane);
        if (lane == 0) {
            if constexpr (SP) fence_proxy_async_smem();
            tc_fence_after();
            const uint64_t vd = smem_desc(smem_addr(sm.stage[s]), 4 * 2048, 1024, 2);
            const bool first = w.first();
#pragma unroll
            for (int hl = 0; hl < kTerms; ++hl)  // P_hi, then P_lo, A from TMEM
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tmem + kTmemO, tmem + (hl ? kTmemPlo : kTmemPhi) + 8 * kk, vd + 128 * kk, id2,
                           (!first || hl > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&sm.p_free);
            mma_commit(&sm.kv_empty[s]);
            if (w.last()) mma_commit(&sm.o_full);
        }
        __syncwarp();
    }
}

// Every MMA an issuing warp started completes before teardown (bounded; independent of the abort flag).
__device__ void drain_mmas(Smem &sm) {
    if ((threadIdx.x & 31) == 0) {
        mma_commit(&sm.mma_done);
        const long long t0 = clock64();
        while (!mbar_sleep_test(&sm.mma_done, 0) && clock64() - t0 < kSpinCycles) {
        }
    }
    __syncwarp();
}

// ---------------------------------------------------------------- softmax / epilogue (warps 4-11)
// Eight warps: warp w handles TMEM lane quarter (w & 3) -- 32 query rows -- and token half
// th = (w - 4) >> 2 of every block (tokens [32 th, 32 th + 32)); for O it owns columns
// [128 th, 128 th + 128). One thread = one (row, token half).
struct SoftCtx {
    const DecodeParams *p;
    uint32_t tmem, lane_off, half, xchg_peer, xfull_peer0;
    int i, lane, r, th;
    bool row_ok, warp_ok;
};

// fp8 cache: a bf16 pair times `mul` as an fp16 pair (round to nearest); flags values past the fp16
// range (or not finite).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v, float mul, bool &bad) {
    const float a = __uint_as_float(v << 16) * mul, b = __uint_as_float(v & 0xffff0000u) * mul;
    bad |= !(fabsf(a) <= 65504.f) || !(fabsf(b) <= 65504.f);
    __half2 two = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&two);
}
// A bf16 pair times a power of two (exact unless it leaves the range; flags overflow).
__device__ __forceinline__ uint32_t bf16x2_pow2(uint32_t v, float pow2, bool &bad) {
    const float a = __uint_as_float(v << 16) * pow2, b = __uint_as_float(v & 0xffff0000u) * pow2;
    bad |= !(fabsf(a) <= 3.0e38f) || !(fabsf(b) <= 3.0e38f);
    return (__float_as_uint(a) >> 16) | (__float_as_uint(b) & 0xffff0000u);
}

// Q of piece `pc`: latent half -> TMEM (this warp's lanes, its 64 of the 128 columns),
// rotary half -> shared memory (its 2 of the 4 16-byte chunks of the row).
// fp8 cache, with the latent scale written as mu 2^-k (mu in [1, 2)): the latent dims go to TMEM
// as fp16(q mu) and the rotary dims as q 2^(k-8) (exact), matching the converted cache's e4m3 2^-8,
// so that the accumulated score is 2^(k-8) times s / scale; the kernel's score scale carries 2^-(k-8).
template <bool F8>
__device__ __forceinline__ void load_q(Smem &sm, const SoftCtx &c, const Piece &pc) {
    if (c.warp_ok) {
        const DecodeParams &p = *c.p;
        bool bad = false;
        const uint4 *qrow =
            reinterpret_cast<const uint4 *>(p.q + ((size_t)pc.seq * p.rows + (c.row_ok ? c.r : 0)) * kDqk);
#pragma unroll 1
        for (int c16 = 4 * c.th; c16 < 4 * c.th + 4; ++c16) {  // 16 columns = 32 latent bf16 each
            uint32_t w[16];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 x = c.row_ok ? __ldg(qrow + (256 * (int)c.half + 32 * c16) / 8 + v) : make_uint4(0, 0, 0, 0);
                w[4 * v + 0] = x.x;
                w[4 * v + 1] = x.y;
                w[4 * v + 2] = x.z;
                w[4 * v + 3] = x.w;
            }
            if constexpr (F8) {
#pragma unroll
                for (int k = 0; k < 16; ++k) w[k] = bf16x2_to_f16x2(w[k], p.q_lat_mul, bad);
            }
            tmem_st16(c.tmem + kTmemQ + c.lane_off + 16 * c16, w);
        }
#pragma unroll
        for (int v = 2 * c.th; v < 2 * c.th + 2; ++v) {  // rotary dims: 16-byte chunks, 64-byte swizzle
            uint4 x = c.row_ok ? __ldg(qrow + (512 + 32 * (int)c.half) / 8 + v) : make_uint4(0, 0, 0, 0);
            if constexpr (F8)
                x = make_uint4(bf16x2_pow2(x.x, p.q_rope_mul, bad), bf16x2_pow2(x.y, p.q_rope_mul, bad),
                               bf16x2_pow2(x.z, p.q_rope_mul, bad), bf16x2_pow2(x.w, p.q_rope_mul, bad));
            *reinterpret_cast<uint4 *>(sm.q_rope + c.i * 64 + ((v ^ ((c.i >> 1) & 3)) * 16)) = x;
        }
        if (F8 && bad) raise_error(kErrRange);
        tmem_wait_st();
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&sm.q_full);
}

// Brings this thread's part of piece `pc`'s query row into L2 ahead of load_q (its 256 bytes of latent
// dims and 32 bytes of rotary dims): load_q's four dependent rounds of loads then hit L2.
__device__ __forceinline__ void prefetch_q(const SoftCtx &c, const Piece &pc) {
    if (!c.row_ok) return;
    const DecodeParams &p = *c.p;
    const char *row = reinterpret_cast<const char *>(p.q + ((size_t)pc.seq * p.rows + c.r) * kDqk);
    prefetch_l2(row + 2 * (256 * (int)c.half + 128 * c.th));
    prefetch_l2(row + 2 * (256 * (int)c.half + 128 * c.th) + 128);
    prefetch_l2(row + 2 * (512 + 32 * (int)c.half + 16 * c.th));
}

// Own partial scores of block g for this thread's 32 tokens (raw, unscaled); keys at or past `vis`
// become -inf. The accumulators are released as soon as the scores are in registers.
// Sparse mode: keys are the stage's validity mask bits instead (then `nvalid` holds this thread's
// 32 bits of it); the mask was stored before the producer's arrival on kv_full, which this thread
// waits for itself (it completed before Gemm1, and the stage is not refilled before Gemm2 of this
// block, which needs this thread's P).
template <bool SP>
__device__ __forceinline__ bool load_raw(Smem &sm, const SoftCtx &c, int g, int key0, int vis, float (&s)[kTokPer],
                                         int &nvalid) {
    if (!mbar_wait(&sm.s_full, g & 1, &sm.abort)) return false;
    tc_fence_after();
    {
        uint32_t a[32];
        tmem_ld32(c.tmem + kTmemS + c.lane_off + kTokPer * c.th, a);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kTokPer; ++j) s[j] = __uint_as_float(a[j]);
    }
    tc_fence_before();
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&sm.s_free);
    if constexpr (SP) {
        const int st = g % kStages;
        if (!mbar_wait(&sm.kv_full[st], (g / kStages) & 1, &sm.abort)) return false;
        const uint32_t m = (uint32_t)(sm.vmask[st] >> (kTokPer * c.th));
        nvalid = (int)m;
#pragma unroll
        for (int j = 0; j < kTokPer; ++j) s[j] = (m >> j) & 1u ? s[j] : -INFINITY;
    } else {
        const int k0 = key0 + kTokPer * c.th;
        nvalid = min(max(vis - k0, 0), kTokPer);  // the valid tokens are a prefix of the thread's 32
        if (k0 + kTokPer > vis) {  // the sequence ends (or the causal limit falls) inside these tokens
#pragma unroll
            for (int j = 0; j < kTokPer; ++j) s[j] = k0 + j < vis ? s[j] : -INFINITY;
        }
    }
    return true;
}

// R (fp16) and m (fp32) of block g into the peer CTA's receive slot g % 2 (the first block of a
// part; later blocks are sent from the softmax loop as their exponentials are computed).
__device__ __forceinline__ void send_factors(const SoftCtx &c, int g, const float (&e)[kTokPer], float m_own) {
    if (!c.warp_ok) return;
    const int slot = g & 1;
    const uint32_t base = c.xchg_peer + (uint32_t)(((slot * kTq + c.th) * 4) * 128 + c.i) * 16;
    const uint32_t bar = c.xfull_peer0 + slot * 8;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            __half2 two = __floats2half2_rn(e[8 * c4 + 2 * q], e[8 * c4 + 2 * q + 1]);
            w[q] = *reinterpret_cast<uint32_t *>(&two);
        }
        st_async_v4_b32(base + c4 * 128 * 16, w[0], w[1], w[2], w[3], bar);
    }
    // the row offset travels in the offsets area of the same slot
    const uint32_t offa = c.xchg_peer + (uint32_t)kXchgEBytes + (uint32_t)((slot * kTq + c.th) * 128 + c.i) * 4;
    st_async_b32(offa, __float_as_uint(m_own), bar);
}

// R = 2^((s * scale_log2 - m) / 2 + 15) in place with m = max_j s_j * scale_log2 (log2 units); R
// is in [0, 2^15], 0 for masked tokens.
__device__ __forceinline__ float exps_in_place(float (&s)[kTokPer], float sl2) {
    float t[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) t[j] = fmaxf(s[j], s[j + 16]);
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
    const bool none = t[0] == -INFINITY;
    const float m = none ? -INFINITY : t[0] * sl2;  // sl2 > 0, so the max commutes with the scaling
    const float off = none ? 0.f : kXScaleLog2 - 0.5f * m;
    const float hsl2 = 0.5f * sl2;
#pragma unroll
    for (int j = 0; j < kTokPer; ++j) s[j] = ex2_approx(fmaf(s[j], hsl2, off));
    return m;
}

// Range of the exchange. A peer factor R' below 2^-14 is an fp16 subnormal (or 0) with an absolute
// error up to 2^-25, i.e. a relative error up to 2^-25 / R' where a normal one has 2^-11. The part of
// its token's P = (R_own R' fh)^2 past normal precision is then at most R_own^2 fh^2 R' (2^-24 -
// 2^-10 R') = P (2^-24 / R' - 2^-10), and R_own^2 fh^2 2^-50 <= fh^2 2^-20 when R' = 0 (R_own <=
// 2^15). Non-negative fp16 numbers order like their bit patterns, so the u16x2 minimum of a thread's
// 32 factors (`mn`, per token parity) shows whether any is below 2^-14 (valid tokens of rows whose
// partial maxima overstate the true maximum by ~58 octaves or more; masked tokens carry R' = 0).
// Only then is the bound summed (the warp votes, so that it branches once).
// The bound above for tokens 8 c4 .. 8 c4 + 7 of this thread (those below `nv` are valid; sparse
// mode: those whose bit is set in `nv`), in units of l. `w4`: their peer factors (fp16 pairs); `pk`/`pl`: P as stored for Gemm2 (bf16 hi/lo pairs;
// fp8 cache: fp16 pairs in `pk`).
template <bool F8, bool SP>
__device__ __forceinline__ float range_excess8(const uint32_t (&w4)[4], int c4, const uint32_t (&pk)[kTokPer / 2],
                                               const uint32_t (&pl)[kTokPer / 2], int nv, float fh) {
    float sq = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int j = 8 * c4 + k, sh = 16 * (k & 1);
        const uint32_t hb = (w4[k >> 1] >> sh) & 0xffffu;
        const bool key = SP ? (((uint32_t)nv >> j) & 1u) != 0u : j < nv;
        if (hb >= 0x400u || !key) continue;  // normal, or a masked token
        const float rp = __half2float(__ushort_as_half((unsigned short)hb));
        float pj;
        if constexpr (F8) {
            pj = __half2float(__ushort_as_half((unsigned short)(pk[j >> 1] >> sh)));
        } else {  // hi + lo, each a bf16 (the top half of an fp32)
            pj = __uint_as_float(((pk[j >> 1] >> sh) & 0xffffu) << 16) +
                 __uint_as_float(((pl[j >> 1] >> sh) & 0xffffu) << 16);
        }
        sq += rp > 0.f ? pj * (0x1p-24f / rp - 0x1p-10f) : 0x1p-20f * fh * fh;
    }
    return sq;
}

template <bool F8, bool SP>
__device__ void softmax_role(Smem &sm, const DecodeParams &p, const int32_t *meta, uint32_t tmem, uint32_t half,
                             int group) {
    SoftCtx c;
    c.p = &p;
    c.tmem = tmem;
    c.half = half;
    const int warp = threadIdx.x >> 5;
    const int wq = warp & 3;
    c.th = (warp - first_soft_warp<F8, SP>()) >> 2;
    c.lane = threadIdx.x & 31;
    c.i = wq * 32 + c.lane;  // row within the group == TMEM lane
    c.lane_off = (uint32_t)(wq * 32) << 16;
    c.r = group * 128 + c.i;
    c.row_ok = c.r < p.rows;
    c.warp_ok = group * 128 + wq * 32 < p.rows;
    const uint32_t peer = half ^ 1u;
    c.xchg_peer = map_to_rank(&sm.xchg[0], peer);
    c.xfull_peer0 = map_to_rank(&sm.xfull[0], peer);
    const uint32_t xchg_peer = c.xchg_peer, xfull_peer0 = c.xfull_peer0;
    const int nvalid_warps = min(4, (p.rows - group * 128 + 31) / 32);
    const uint32_t xbytes = (uint32_t)nvalid_warps * kTq * 32 * (2 * kTokPer + 4);  // R (fp16) + offset
    const int t_q = c.row_ok ? c.r / p.h_q : 0, h_idx = c.row_ok ? c.r % p.h_q : 0;
    const float sl2 = p.scale_log2;
    volatile int *abort = &sm.abort;
    const uint4 *xe = sm.xchg;
    const float *xo = reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(sm.xchg) + kXchgEBytes);
    const int bar_id = 1 + wq;  // the two warps of these 32 rows

    // w walks one block ahead of the block being finished; of that block only a few facts are kept
    BlockWalker<SP> w;
    w.init(meta, p);
    if (!w.live) return;
    load_q<F8>(sm, c, w.pc);
    if constexpr (!F8) {  // (measured: the fp8 kernel ran 12% slower with these prefetches in its loop)
        Cursor<SP> tmp = w.cur;
        Piece nx;
        if (tmp.next(p, nx)) prefetch_q(c, nx);
    }
    int vis = c.row_ok ? visible_keys(w.pc.n, p.s_q, t_q, p.causal) : 0;
    float e_own[kTokPer], m_own;
    int nv_own;  // valid tokens of the block being finished, among this thread's 32
    if (!load_raw<SP>(sm, c, 0, w.blk * kBlk, vis, e_own, nv_own)) return;
    m_own = exps_in_place(e_own, sl2);
    send_factors(c, 0, e_own, m_own);
    if (w.last()) {  // the next piece's Q may replace this one once its last Gemm1 is done
        Cursor<SP> tmp = w.cur;
        Piece nx;
        if (tmp.next(p, nx)) load_q<F8>(sm, c, nx);
    }
    float m_ref = -INFINITY, l = 0.f;
    float lost = 0.f;  // bound on the part of l past normal precision from subnormal peer factors (scale of l)
    for (int g = 0; w.live; ++g) {
        const bool a_first = w.first(), a_last = w.last();
        const int a_piece_k = w.piece_k, a_seq = w.pc.seq, a_nsplit = w.pc.nsplit, a_slot = w.pc.slot;
        w.advance(p);
        const bool nx_live = w.live;
        // raw scores of block g+1 first: the accumulators are free for Gemm1 of block g+2 early, and
        // the peer's factors of block g arrive meanwhile
        float snx[kTokPer];
        int nv_nx = 0;
        if (nx_live) {
            if (w.first()) {  // block g+1 starts a piece: its query was loaded; warm the next piece's
                vis = c.row_ok ? visible_keys(w.pc.n, p.s_q, t_q, p.causal) : 0;
                if constexpr (!F8) {
                    Cursor<SP> tmp = w.cur;
                    Piece nx;
                    if (tmp.next(p, nx)) prefetch_q(c, nx);
                }
            }
            if (!load_raw<SP>(sm, c, g + 1, w.blk * kBlk, vis, snx, nv_nx)) return;
            if (w.last()) {
                Cursor<SP> tmp = w.cur;
                Piece nx;
                if (tmp.next(p, nx)) load_q<F8>(sm, c, nx);
            }
        } else {
#pragma unroll
            for (int j = 0; j < kTokPer; ++j) snx[j] = -INFINITY;
        }
        // peer factors of block g (slot g % 2)
        const int slot = g & 1;
        if (threadIdx.x == 32 * first_soft_warp<F8, SP>()) mbar_arrive_expect_tx(&sm.xfull[slot], xbytes);
        if (!mbar_wait_cluster(&sm.xfull[slot], (g >> 1) & 1, abort)) return;
        const float m_peer = c.warp_ok ? xo[(slot * kTq + c.th) * 128 + c.i] : -INFINITY;
        const float mbu_half = m_own + m_peer;
        uint32_t ep[kTokPer / 2];  // the peer's factors, fp16 pairs
        uint32_t mn = 0xffffffffu;  // their minimum per token parity (non-negative fp16 order like their bits)
        float mbu;                 // the block's row max (both token halves), shared by the two warps of a row
        if constexpr (F8) {
            // exact: t_j = R_own R_peer = 2^((s_j - m_own - m_peer) / 2 + 30) in place of R_own, and
            // the max of t gives the max of s. fp16 P needs it: an upper bound that overstates the
            // max by o octaves would leave P below 2^-o, where fp16 loses precision.
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const uint4 v = xe[((slot * kTq + c.th) * 4 + c4) * 128 + c.i];
                ep[4 * c4] = v.x;
                ep[4 * c4 + 1] = v.y;
                ep[4 * c4 + 2] = v.z;
                ep[4 * c4 + 3] = v.w;
            }
#pragma unroll
            for (int j = 0; j < kTokPer; j += 2) {
                const float2 e2 = __half22float2(*reinterpret_cast<const __half2 *>(&ep[j >> 1]));
                unpack2(mul2(pack2(e_own[j], e_own[j + 1]), pack2(e2.x, e2.y)), e_own[j], e_own[j + 1]);
            }
            const float tmax = max32(e_own);
            const float mx_half =
                (tmax > 0.f && mbu_half != -INFINITY) ? 2.f * (__log2f(tmax) - 2.f * kXScaleLog2) + mbu_half : -INFINITY;
            sm.xmax[g & 1][c.th][c.i] = mx_half;
            named_bar_sync(bar_id, 64);
            mbu = fmaxf(mx_half, sm.xmax[g & 1][c.th ^ 1][c.i]);
        } else {
            // an upper bound of the block's row max
            sm.xmax[g & 1][c.th][c.i] = mbu_half;
            named_bar_sync(bar_id, 64);
            mbu = fmaxf(mbu_half, sm.xmax[g & 1][c.th ^ 1][c.i]);
        }
        bool need = false;
        float alpha = 1.f;
        if (a_first) {
            m_ref = mbu;
            l = 0.f;
            lost = 0.f;
        } else if (mbu > m_ref + kRescaleThreshold) {
            if (m_ref == -INFINITY) {
                m_ref = mbu;  // nothing accumulated yet (O and l are zero)
            } else {
                alpha = ex2_approx(m_ref - mbu);
                m_ref = mbu;
                l *= alpha;
                lost *= alpha;
                need = true;
            }
        }
        if constexpr (!F8) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const uint4 v = xe[((slot * kTq + c.th) * 4 + c4) * 128 + c.i];
                ep[4 * c4] = v.x;
                ep[4 * c4 + 1] = v.y;
                ep[4 * c4 + 2] = v.z;
                ep[4 * c4 + 3] = v.w;
            }
        }
        // One straight-line region: P of block g (FMA and ALU work), the exponentials of block g+1
        // (MUFU work) and their stores into the peer (distributed shared memory, ~20 bytes per
        // cycle), spread over the region so that the three overlap. Sending block g+1 here is safe
        // with two receive slots: the peer sent block g (which has arrived) only after it had read
        // slot (g - 1) % 2 = (g + 1) % 2.
        // P = 2^(s0 + s1 - m_ref) in two bf16 terms: hi = P with its low 16 bits cleared, lo = the
        // (exact) remainder with its low 16 bits cleared; hi + lo is within 2^-14 of P.
        // P = (t fh)^2 with t = R_own R_peer and fh = 2^((mbu_half - m_ref) / 2 - 30), the square root
        // of the block's factor: fh stays a normal fp32 number down to mbu_half - m_ref = -192, where P
        // itself is below 2^-126, so no block that can matter is flushed. The exponent is capped at 64,
        // reached only when the fp8 path's exact row max lies more than ~190 octaves below the sum of
        // the partial maxima (a row the range check below reports).
        const bool none = m_ref == -INFINITY || mbu_half == -INFINITY;
        const float fh = none ? 0.f : ex2_approx(fminf(0.5f * (mbu_half - m_ref) - 2.f * kXScaleLog2, 64.f));
        float m_nx, off_nx;
        {
            const float smax = max32(snx);
            const bool nx_none = smax == -INFINITY;
            m_nx = nx_none ? -INFINITY : smax * sl2;  // sl2 > 0, so the max commutes with the scaling
            off_nx = nx_none ? 0.f : kXScaleLog2 - 0.5f * m_nx;
        }
        const bool send = nx_live && c.warp_ok;
        const int nslot = (g + 1) & 1;
        const uint32_t xbase = xchg_peer + (uint32_t)(((nslot * kTq + c.th) * 4) * 128 + c.i) * 16;
        const uint32_t xbar = xfull_peer0 + nslot * 8;
        // The arithmetic runs on token pairs with the packed f32x2 instructions (two fp32 lanes per
        // instruction, each rounded as its scalar form would be).
        uint32_t pk[kTokPer / 2], pl[kTokPer / 2];
        f32x2 su[4] = {0ull, 0ull, 0ull, 0ull};  // two lanes of partial row sums each (0 is +0, +0)
        const f32x2 ffh = pack2(fh, fh), hsl2 = pack2(0.5f * sl2, 0.5f * sl2), offnx = pack2(off_nx, off_nx);
        const f32x2 minus1 = pack2(-1.f, -1.f);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t wv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j = 8 * c4 + 2 * q;
                // R of block g+1: 2^((s * scale_log2 - m) / 2 + 15), in [0, 2^15], 0 for masked tokens
                float x0, x1;
                unpack2(fma2(pack2(snx[j], snx[j + 1]), hsl2, offnx), x0, x1);
                snx[j] = ex2_approx(x0);
                snx[j + 1] = ex2_approx(x1);
                __half2 two = __floats2half2_rn(snx[j], snx[j + 1]);
                wv[q] = *reinterpret_cast<uint32_t *>(&two);
                mn = min_u16x2(mn, ep[j >> 1]);
                // P of block g
                if constexpr (F8) {  // e_own holds t = R_own R_peer; P in fp16 (round to nearest)
                    const f32x2 tf = mul2(pack2(e_own[j], e_own[j + 1]), ffh);
                    const f32x2 pp = mul2(tf, tf);
                    su[q] = add2(su[q], pp);
                    float p0, p1;
                    unpack2(pp, p0, p1);
                    __half2 ph = __floats2half2_rn(p0, p1);
                    pk[j >> 1] = *reinterpret_cast<uint32_t *>(&ph);
                } else {
                    const float2 e2 = __half22float2(*reinterpret_cast<const __half2 *>(&ep[j >> 1]));
                    const f32x2 tf = mul2(mul2(pack2(e_own[j], e_own[j + 1]), pack2(e2.x, e2.y)), ffh);
                    const f32x2 pp = mul2(tf, tf);
                    su[q] = add2(su[q], pp);
                    float p0, p1;
                    unpack2(pp, p0, p1);
                    const uint32_t u0 = __float_as_uint(p0), u1 = __float_as_uint(p1);
                    // lo = P - hi, exact (hi is P with its low 16 bits cleared)
                    float r0, r1;
                    unpack2(fma2(pack2(__uint_as_float(u0 & 0xffff0000u), __uint_as_float(u1 & 0xffff0000u)), minus1, pp),
                            r0, r1);
                    pk[j >> 1] = __byte_perm(u0, u1, 0x7632);
                    pl[j >> 1] = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
                }
            }
            if (send) st_async_v4_b32(xbase + c4 * 128 * 16, wv[0], wv[1], wv[2], wv[3], xbar);
        }
        // Range of the exchange (see range_excess8). bf16 cache: the bound is summed here, with R'
        // read again from the receive slot 16 bytes at a time (the peer refills that slot only after
        // it has the row offset of block g+1, sent below), so the factors need not stay in registers.
        const bool suspect = fh > 0.f && ((mn & 0xffffu) < 0x400u || (mn >> 16) < 0x400u);
        if constexpr (!F8) {
            if (__any_sync(0xffffffffu, suspect) && suspect) {
                float sq = 0.f;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint4 v = xe[((slot * kTq + c.th) * 4 + c4) * 128 + c.i];
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                    sq += range_excess8<F8, SP>(w4, c4, pk, pl, nv_own, fh);
                }
                lost += sq;
            }
        }
        if (send)  // the row offset travels in the offsets area of the same slot
            st_async_b32(xchg_peer + (uint32_t)kXchgEBytes + (uint32_t)((nslot * kTq + c.th) * 128 + c.i) * 4,
                         __float_as_uint(m_nx), xbar);
        {
            float a0, a1;
            unpack2(add2(add2(su[0], su[1]), add2(su[2], su[3])), a0, a1);
            l += a0 + a1;
        }
        // the P tile and O are free once Gemm2 of block g-1 has completed
        if (g > 0 && !mbar_wait(&sm.p_free, (g - 1) & 1, abort)) return;
        tc_fence_after();
        if (c.warp_ok && __any_sync(0xffffffffu, need)) {
            const float a = need ? alpha : 1.f;
#pragma unroll 1
            for (int q = 0; q < 8; ++q) {
                uint32_t v[16];
                tmem_ld16(tmem + kTmemO + c.lane_off + 128 * c.th + 16 * q, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * a);
                tmem_st16(tmem + kTmemO + c.lane_off + 128 * c.th + 16 * q, v);
            }
            tmem_wait_st();
        }
        // this thread's 32 tokens of row i in both P regions of TMEM (bf16 pairs, lane = row)
        tmem_st16(tmem + kTmemPhi + c.lane_off + 16 * c.th, pk);
        if constexpr (!F8) tmem_st16(tmem + kTmemPlo + c.lane_off + 16 * c.th, pl);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (c.lane == 0) mbar_arrive(&sm.p_full);
        // fp8 cache: the range bound once Gemm2 has its operand, from the factors still in registers
        if constexpr (F8) {
            if (__any_sync(0xffffffffu, suspect) && suspect) {
                float sq = 0.f;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint32_t w4[4] = {ep[4 * c4], ep[4 * c4 + 1], ep[4 * c4 + 2], ep[4 * c4 + 3]};
                    sq += range_excess8<F8, SP>(w4, c4, pk, pl, nv_own, fh);
                }
                lost += sq;
            }
        }

        if (a_last) {  // epilogue of this piece: the two token halves' sums, then this warp's O columns
            // the sums travel in the other parity's row-max slots, which nobody reads until block g+1,
            // the loss bounds in this parity's, which both warps of the row have read by now
            sm.xmax[(g + 1) & 1][c.th][c.i] = l;
            sm.xmax[g & 1][c.th][c.i] = lost;
            named_bar_sync(bar_id, 64);
            const float l_row = l + sm.xmax[(g + 1) & 1][c.th ^ 1][c.i];
            const float lost_row = lost + sm.xmax[g & 1][c.th ^ 1][c.i];
            named_bar_sync(bar_id, 64);  // both sums read before block g+1 reuses the slots
            // Range of the exchange: a whole row is reported here when the bound exceeds 2^-11 of its
            // sum; a piece leaves bound / sum for the combine, which weighs the pieces of the row.
            if (c.row_ok && c.th == 0) {
                if (a_nsplit == 1 || !(l_row > 0.f)) {
                    if (lost_row > 0x1p-11f * l_row) raise_error(kErrRange);
                    if (a_nsplit != 1) p.lost_part[((size_t)a_slot * p.rows + c.r) * 2 + half] = 0.f;
                } else {
                    p.lost_part[((size_t)a_slot * p.rows + c.r) * 2 + half] = lost_row / l_row;
                }
            }
            if (!mbar_wait(&sm.o_full, a_piece_k & 1, abort)) return;
            tc_fence_after();
            if (c.warp_ok) {
                const bool empty = !(l_row > 0.f);
                const float inv = empty ? 0.f : (F8 ? p.v_scale / l_row : 1.f / l_row);
                const bool whole = a_nsplit == 1;
#pragma unroll 1
                for (int q = 0; q < 8; ++q) {
                    uint32_t v[16];
                    const int col = 128 * c.th + 16 * q;
                    tmem_ld16(tmem + kTmemO + c.lane_off + col, v);
                    tmem_wait_ld();
                    if (!c.row_ok) continue;
                    // 32-byte stores: each lane writes its own row, so a warp's store touches 32 rows and
                    // the number of stores, not their width, sets the epilogue's time
                    if (whole) {
                        uint32_t wv[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            __nv_bfloat162 two = __floats2bfloat162_rn(__uint_as_float(v[2 * j]) * inv,
                                                                       __uint_as_float(v[2 * j + 1]) * inv);
                            wv[j] = *reinterpret_cast<uint32_t *>(&two);
                        }
                        __nv_bfloat16 *dst = p.out + ((size_t)a_seq * p.rows + c.r) * kDv + 256 * half + col;
                        if (p.out_v8) {
                            st_global_v8(dst, wv);
                        } else {  // `out` only 16-byte aligned
                            reinterpret_cast<uint4 *>(dst)[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                            reinterpret_cast<uint4 *>(dst)[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
                        }
                    } else {
                        float *dst = p.o_part + ((size_t)a_slot * p.rows + c.r) * kDv + 256 * half + col;
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * inv);
                        st_global_v8(dst, v);
                        st_global_v8(dst + 8, v + 8);
                    }
                }
                if (c.row_ok && half == 0 && c.th == 0) {
                    const float lse = empty ? -INFINITY : (m_ref + log2f(l_row)) * 0.69314718055994530942f;
                    if (whole)
                        p.lse[SP ? ((size_t)(a_seq / p.sp_sq) * p.h_q + h_idx) * p.sp_sq + a_seq % p.sp_sq
                                 : ((size_t)a_seq * p.h_q + h_idx) * p.s_q + t_q] = lse;
                    else
                        p.lse_part[(size_t)a_slot * p.rows + c.r] = lse;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (c.lane == 0) mbar_arrive(&sm.o_free);
        }
        if (nx_live) {
#pragma unroll
            for (int j = 0; j < kTokPer; ++j) e_own[j] = snx[j];
            m_own = m_nx;
            nv_own = nv_nx;
        }
    }
}

template <bool F8, bool SP>
__global__ void __launch_bounds__(num_threads<F8, SP>(), 1)
decode_sm100_kernel(const __grid_constant__ CUtensorMap map_lat, const __grid_constant__ CUtensorMap map_rope,
                    const DecodeParams p, const int groups) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t half = cluster_ctarank();
    const int cluster = blockIdx.x >> 1;
    const int part = cluster / groups, group = cluster % groups;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t *meta = p.tile_meta + (size_t)part * kMetaInts;

    if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);  // whole (converged) warp
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.kv_full[s], SP ? kSparseFullArrivals : 1);  // sparse: the gather warps' copies + masks
            mbar_init(&sm.kv_empty[s], 1);
            mbar_init(&sm.conv_full[s], kConvWarps);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.s_free, kSoftWarps);
        mbar_init(&sm.p_full, kSoftWarps);
        mbar_init(&sm.p_free, 1);
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.o_free, kSoftWarps);
        mbar_init(&sm.q_full, kSoftWarps);
        mbar_init(&sm.mma_done, 2);
        mbar_init(&sm.xfull[0], 1);
        mbar_init(&sm.xfull[1], 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (!SP && warp == 0 && lane == 0) {
        prefetch_tensormap(&map_lat);
        prefetch_tensormap(&map_rope);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();  // the peer's barriers exist before any exchange targets them
    const uint32_t tmem = sm.tmem_base;

    if ((F8 || SP) && warp >= 4 && warp < first_soft_warp<F8, SP>()) {
        setmaxnreg_dec<kRegsSmall>();
        if constexpr (SP)
            gather_producer(sm, p, meta, half, warp - 4);
        else
            convert_warp(sm, p, meta);
    } else if (warp < 4) {
        setmaxnreg_dec<(F8 || SP) ? kRegsSmall : kRegsControl>();
        if (SP && warp == 0) {
            // sparse: warpgroup 1 gathers; warp 0 has nothing to do
        } else if (warp == 0) {
            if (lane == 0) producer<F8>(sm, p, &map_lat, &map_rope, meta, half);
        } else {
            if (warp == 3) {
                gemm2_warp<F8, SP>(sm, p, meta, tmem);
                drain_mmas(sm);
            } else if (warp == 1) {
                gemm1_warp<F8, SP>(sm, p, meta, tmem);
                drain_mmas(sm);
            }
        }
    } else {
        setmaxnreg_inc<kRegsSoftmax>();
        softmax_role<F8, SP>(sm, p, meta, tmem, half, group);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && sm.abort) raise_error(kErrTimeout);
    cluster_sync();  // the peer no longer writes into this CTA's shared memory
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}
}  // namespace dec

size_t decode_sm100_smem_bytes() { return sizeof(dec::Smem) + 1024; }

// sparse (p.indices set) runs the bf16-cache kernel with the gather producer; the maps are then unused.
cudaError_t launch_decode_sm100(const DecodeParams &p, const CUtensorMap &map_lat, const CUtensorMap &map_rope,
                                bool fp8, cudaStream_t stream) {
    const int groups = (p.rows + 127) / 128;
    const size_t smem = decode_sm100_smem_bytes();
    const bool sparse = p.indices != nullptr;
    if (fp8 && sparse) return cudaErrorInvalidValue;
    auto kernel = fp8 ? dec::decode_sm100_kernel<true, false>
                      : (sparse ? dec::decode_sm100_kernel<false, true> : dec::decode_sm100_kernel<false, false>);
    const int threads = fp8 ? dec::num_threads<true>() : (sparse ? dec::num_threads<false, true>() : dec::num_threads<false>());
    // setmaxnreg redistributes the registers the block was launched with: the warpgroups' shares must
    // fit in what the compiler gave the kernel, or the raising warps would wait forever
    const int need = (fp8 || sparse) ? 2 * 128 * (int)dec::kRegsSmall + 256 * (int)dec::kRegsSoftmax
                                     : 128 * (int)dec::kRegsControl + 256 * (int)dec::kRegsSoftmax;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * threads < need) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * p.num_parts * groups, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, map_lat, map_rope, p, groups);
}

}  // namespace mla
