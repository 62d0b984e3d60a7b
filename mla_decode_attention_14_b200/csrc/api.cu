// api.cu -- host side of the C ABI declared in include/mla.h: argument validation,
// workspace layout, device checks, kernel launches and the device error word.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>

#include "../../include/mla.h"
#include "common.cuh"

namespace mla {

cudaError_t launch_metadata(const int32_t *seqlens, int uniform_n, int batch, int num_parts, int fixed_cost,
                            int32_t *tile_meta, int32_t *num_splits, cudaStream_t stream);
cudaError_t launch_combine(const int32_t *num_splits, int batch, int num_parts, int s_q, int h_q, int sp_sq,
                           __nv_bfloat16 *out, float *lse, const float *o_part,
                           const float *lse_part, const float *lost_part, cudaStream_t stream);
cudaError_t launch_decode_sm100(const DecodeParams &p, const CUtensorMap &map_lat, const CUtensorMap &map_rope,
                                bool fp8, cudaStream_t stream);
cudaError_t launch_head_gemm(const CUtensorMap &map_x, const CUtensorMap &map_w, __nv_bfloat16 *y, int64_t ldy,
                             int64_t y_head, int64_t x_head, int m, int n, int k, int heads, cudaStream_t stream);
cudaError_t launch_append(const __nv_bfloat16 *new_kv, int n_new, void *kv, int64_t num_blocks,
                          const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens, int batch,
                          bool fp8, float inv_scale, cudaStream_t stream);

static std::atomic<int64_t> g_launches{0};
static std::atomic<int> g_last_cuda_error{0};  // cudaError_t of the last failing CUDA call

// MLA_OK for cudaSuccess; otherwise remembers the error (see mla_last_cuda_error) -> MLA_ERR_CUDA.
static int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return 0;
    g_last_cuda_error.store((int)e, std::memory_order_relaxed);
    return MLA_ERR_CUDA;
}

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_dev_ok[kMaxDevices];  // 0 unknown, 1 sm_100, 2 not sm_100

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The kernels are built for sm_100a only: refuse other devices before launching.
int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    int st = g_dev_ok[dev].load(std::memory_order_relaxed);
    if (st == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return MLA_ERR_CUDA;
        st = (major == 10 && minor == 0) ? 1 : 2;
        g_dev_ok[dev].store(st, std::memory_order_relaxed);
    }
    return st == 1 ? MLA_OK : MLA_ERR_UNSUPPORTED;
}

// ---- TMA descriptors of the paged cache for the exchange kernel. "latent": the cache viewed as
// [boxes][rows][box] -- bf16: [9][num_blocks * 64][64 dims], fp8: [5][num_blocks * 64][128 bytes]
// (E4M3, uint8 view) -- so that ONE operation brings a CTA's 4 bf16 (2 E4M3) latent boxes of
// 64 tokens x 128 bytes with the 128-byte swizzle; "rope": 64 tokens x 32 bf16 dims with the
// 64-byte swizzle over a 2-D bf16 view [rows, 288] (bf16) or [rows, 320] (fp8 records).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

struct MapEntry {
    const void *kv;
    int64_t num_blocks;
    int device, fp8;
    CUtensorMap lat, rope;
};
constexpr int kMapCache = 16;
MapEntry g_maps[kMapCache];
int g_maps_used = 0, g_maps_next = 0;
std::mutex g_maps_mu;

int cache_maps(const void *kv, int64_t num_blocks, int fp8, CUtensorMap *lat, CUtensorMap *rope) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_maps_mu);
    for (int k = 0; k < g_maps_used; ++k) {
        if (g_maps[k].kv == kv && g_maps[k].num_blocks == num_blocks && g_maps[k].device == dev &&
            g_maps[k].fp8 == fp8) {
            *lat = g_maps[k].lat;
            *rope = g_maps[k].rope;
            return MLA_OK;
        }
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    MapEntry e;
    e.kv = kv;
    e.num_blocks = num_blocks;
    e.device = dev;
    e.fp8 = fp8;
    const cuuint64_t rows = (cuuint64_t)num_blocks * MLA_BLOCK_TOKENS;
    const cuuint64_t rec = fp8 ? (cuuint64_t)MLA_FP8_RECORD_BYTES : (cuuint64_t)MLA_D_QK * 2;
    cuuint64_t dims[2] = {rec / 2, rows};  // bf16 view (rotary boxes)
    cuuint64_t strides[1] = {rec};
    cuuint64_t dims3[3] = {fp8 ? 128u : 64u, rows, fp8 ? 4u : 9u}, strides3[2] = {rec, 128};
    cuuint32_t box3[3] = {fp8 ? 128u : 64u, 64, fp8 ? 2u : 4u}, estr3[3] = {1, 1, 1};
    cuuint32_t box_rope[2] = {32, 64}, estr[2] = {1, 1};
    if (enc(&e.lat, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(kv),
            dims3, strides3, box3, estr3, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MLA_ERR_CUDA;
    if (enc(&e.rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(kv), dims, strides, box_rope, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MLA_ERR_CUDA;
    g_maps[g_maps_next] = e;
    g_maps_next = (g_maps_next + 1) % kMapCache;
    if (g_maps_used < kMapCache) ++g_maps_used;
    *lat = e.lat;
    *rope = e.rope;
    return MLA_OK;
}

int shape_ok(int batch, int s_q, int h_q) {
    if (batch < 1 || batch > MLA_MAX_BATCH) return 0;
    if (s_q < 1 || h_q < 1) return 0;
    if ((int64_t)s_q * h_q > MLA_MAX_ROWS) return 0;
    return 1;
}

// Sparse mode: batch * s_q work units of h_q rows each (every row of a unit shares its index list).
int sparse_shape_ok(int batch, int s_q, int h_q, int topk) {
    if (batch < 1 || s_q < 1 || h_q < 1 || topk < 1 || topk > (1 << 24)) return 0;
    if ((int64_t)batch * s_q > (1 << 24)) return 0;
    return shape_ok(batch * s_q, 1, h_q);
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout: fp32 o_part[(batch + num_parts) * rows * 512], then fp32
// lse_part[(batch + num_parts) * rows], then fp32 lost_part[(batch + num_parts) * rows * 2].
size_t opart_bytes(int batch, int rows, int num_parts) {
    return (size_t)(batch + num_parts) * rows * MLA_D_V * sizeof(float);
}
size_t lsepart_bytes(int batch, int rows, int num_parts) { return (size_t)(batch + num_parts) * rows * sizeof(float); }

int validate_decode(const void *q, const void *kv, int64_t num_blocks, const int32_t *bt,
                    int64_t bt_stride, const int32_t *seqlens, const int32_t *tile_meta,
                    const int32_t *num_splits, int num_parts, int batch, int s_q, int h_q,
                    float scale, int causal, const void *out, const float *lse,
                    const void *ws, size_t ws_bytes) {
    if (!q || !kv || !bt || !seqlens || !tile_meta || !num_splits || !out || !lse || !ws)
        return MLA_ERR_INVALID_ARG;
    if (!shape_ok(batch, s_q, h_q)) return MLA_ERR_INVALID_ARG;
    if (num_parts < 1 || num_parts > 65535) return MLA_ERR_INVALID_ARG;
    if (num_blocks < 1 || num_blocks > (int64_t)(INT32_MAX / MLA_BLOCK_TOKENS)) return MLA_ERR_INVALID_ARG;
    if (bt_stride < 1 || bt_stride > (int64_t)INT32_MAX) return MLA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale >= 0.f)) return MLA_ERR_INVALID_ARG;  // the max commutes with scale >= 0
    if (causal != 0 && causal != 1) return MLA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
        !aligned(ws, 256) || !aligned(bt, 4) || !aligned(seqlens, 4) || !aligned(tile_meta, 4) ||
        !aligned(num_splits, 4))
        return MLA_ERR_INVALID_ARG;
    if (ws_bytes < mla_workspace_bytes(batch, s_q, h_q, num_parts)) return MLA_ERR_WORKSPACE;
    return MLA_OK;
}

DecodeParams make_params(const void *q, const void *kv, int64_t num_blocks, const int32_t *bt,
                         int64_t bt_stride, const int32_t *seqlens, const int32_t *tile_meta,
                         const int32_t *num_splits, int num_parts, int batch, int s_q, int h_q,
                         float scale, int causal, void *out, float *lse, void *ws) {
    DecodeParams p;
    const int rows = s_q * h_q;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.kv = static_cast<const __nv_bfloat16 *>(kv);
    p.block_table = bt;
    p.seqlens = seqlens;
    p.tile_meta = tile_meta;
    p.num_splits = num_splits;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.o_part = static_cast<float *>(ws);
    p.lse_part = reinterpret_cast<float *>(static_cast<char *>(ws) + opart_bytes(batch, rows, num_parts));
    p.lost_part = reinterpret_cast<float *>(static_cast<char *>(ws) + opart_bytes(batch, rows, num_parts) +
                                            lsepart_bytes(batch, rows, num_parts));
    p.num_blocks = num_blocks;
    p.bt_stride = bt_stride;
    p.batch = batch;
    p.s_q = s_q;
    p.h_q = h_q;
    p.rows = rows;
    p.num_parts = num_parts;
    p.causal = causal;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.v_scale = 1.f;
    p.q_lat_mul = 1.f;
    p.q_rope_mul = 1.f;
    p.out_v8 = (reinterpret_cast<uintptr_t>(out) & 31) == 0;
    p.indices = nullptr;  // dense
    p.topk = 0;
    p.sp_sq = 0;
    return p;
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" {

const char *mla_status_string(int status) {
    switch (status) {
        case MLA_OK: return "MLA_OK";
        case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: invalid argument";
        case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: device or shape not supported";
        case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace too small";
        case MLA_ERR_CUDA: return "MLA_ERR_CUDA: a CUDA call failed";
        case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT: a device pipeline wait hit its bound";
        case MLA_ERR_BOUNDS: return "MLA_ERR_BOUNDS: block-table entry out of range";
        case MLA_ERR_RANGE: return "MLA_ERR_RANGE: a query value is outside the range of its fp16 form (fp8 cache)";
        default: return "MLA: unknown status";
    }
}

int mla_default_num_parts(int device, int h_q, int s_q, int *num_parts) {
    if (!num_parts || h_q < 1 || s_q < 1 || (int64_t)h_q * s_q > MLA_MAX_ROWS) return MLA_ERR_INVALID_ARG;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return MLA_ERR_CUDA;
    const int groups = (h_q * s_q + 127) / 128;
    int parts = (sms / 2) / groups;
    *num_parts = parts < 1 ? 1 : parts;
    return MLA_OK;
}

// Measured on a B200 (whole step: metadata + split + combine) once a piece's start had been made
// cheap (the next piece's query prefetched into L2, 32-byte epilogue stores, tail zeroing without
// divisions): start-up costs of 3 / 5 / 10 blocks gave 0.273 / 0.277 / 0.303 ms for 128 query rows
// (U[1024, 8192] lengths), 0.152 / 0.141 / 0.148 ms for 64 rows with lognormal lengths and
// 0.119 / 0.121 / 0.126 ms for 16 rows: a piece's start (Q load, pipeline fill, partial writes, one
// more combine input) now costs about as much as five blocks of steady-state work.
int mla_default_fixed_cost(int h_q, int s_q) {
    (void)h_q;
    (void)s_q;
    return 5;
}

size_t mla_workspace_bytes(int batch, int s_q, int h_q, int num_parts) {
    if (!shape_ok(batch, s_q, h_q) || num_parts < 1) return 0;
    const int rows = s_q * h_q;
    size_t b = opart_bytes(batch, rows, num_parts) + 3 * lsepart_bytes(batch, rows, num_parts);
    return round_up(b, 256);
}

int mla_get_metadata(const int32_t *seqlens, int batch, int h_q, int s_q, int num_parts,
                     int fixed_cost, int32_t *tile_meta, int32_t *num_splits, void *stream) {
    if (!seqlens || !tile_meta || !num_splits) return MLA_ERR_INVALID_ARG;
    if (!shape_ok(batch, s_q, h_q) || num_parts < 1 || num_parts > 65535 || fixed_cost < 0 ||
        fixed_cost > (1 << 20))
        return MLA_ERR_INVALID_ARG;
    if (!aligned(seqlens, 4) || !aligned(tile_meta, 4) || !aligned(num_splits, 4)) return MLA_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc != MLA_OK) return rc;
    cudaError_t e = launch_metadata(seqlens, 0, batch, num_parts, fixed_cost, tile_meta, num_splits,
                                    static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(e);
}

int mla_decode_split(const void *q, const void *kv_cache, int64_t num_blocks,
                     const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                     const int32_t *tile_meta, const int32_t *num_splits, int num_parts,
                     int batch, int s_q, int h_q, float scale, int causal, void *out,
                     float *lse, void *workspace, size_t workspace_bytes, void *stream) {
    int rc = validate_decode(q, kv_cache, num_blocks, block_table, bt_stride, seqlens, tile_meta,
                             num_splits, num_parts, batch, s_q, h_q, scale, causal, out, lse,
                             workspace, workspace_bytes);
    if (rc != MLA_OK) return rc;
    rc = check_device();
    if (rc != MLA_OK) return rc;
    DecodeParams p = make_params(q, kv_cache, num_blocks, block_table, bt_stride, seqlens, tile_meta,
                                 num_splits, num_parts, batch, s_q, h_q, scale, causal, out, lse,
                                 workspace);
    CUtensorMap map_lat, map_rope;
    rc = cache_maps(kv_cache, num_blocks, 0, &map_lat, &map_rope);
    if (rc != MLA_OK) return rc;
    cudaError_t e = launch_decode_sm100(p, map_lat, map_rope, false, static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(e);
}

int mla_decode_split_fp8(const void *q, const void *kv_cache_fp8, int64_t num_blocks, float kv_scale,
                         const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                         const int32_t *tile_meta, const int32_t *num_splits, int num_parts, int batch,
                         int s_q, int h_q, float scale, int causal, void *out, float *lse, void *workspace,
                         size_t workspace_bytes, void *stream) {
    int rc = validate_decode(q, kv_cache_fp8, num_blocks, block_table, bt_stride, seqlens, tile_meta,
                             num_splits, num_parts, batch, s_q, h_q, scale, causal, out, lse,
                             workspace, workspace_bytes);
    if (rc != MLA_OK) return rc;
    // kv_scale = mu 2^-k with mu in [1, 2): frexp gives kv_scale = f 2^e, f in [0.5, 1). The kernel's
    // fp16 form of a latent byte is e4m3 * 2^-8, so the latent side carries mu 2^-8 = kv_scale 2^(k-8):
    // the rotary query dims are multiplied by 2^(k-8) to match, the scores by 2^-(k-8), the output by
    // kv_scale 2^8.
    if (!std::isfinite(kv_scale) || !(kv_scale > 0.f)) return MLA_ERR_INVALID_ARG;
    int e2 = 0;
    const float f = std::frexp(kv_scale, &e2);
    const int k = 1 - e2;
    if (k < -64 || k > 64) return MLA_ERR_INVALID_ARG;
    const float sl2 = scale * 1.4426950408889634f * std::ldexp(1.f, 8 - k);
    if (!std::isfinite(sl2)) return MLA_ERR_INVALID_ARG;
    rc = check_device();
    if (rc != MLA_OK) return rc;
    DecodeParams p = make_params(q, kv_cache_fp8, num_blocks, block_table, bt_stride, seqlens, tile_meta,
                                 num_splits, num_parts, batch, s_q, h_q, scale, causal, out, lse,
                                 workspace);
    p.scale_log2 = sl2;
    p.v_scale = kv_scale * 256.f;
    p.q_lat_mul = 2.f * f;
    p.q_rope_mul = std::ldexp(1.f, k - 8);
    CUtensorMap map_lat, map_rope;
    rc = cache_maps(kv_cache_fp8, num_blocks, 1, &map_lat, &map_rope);
    if (rc != MLA_OK) return rc;
    cudaError_t e = launch_decode_sm100(p, map_lat, map_rope, true, static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(e);
}

int mla_decode_combine(const int32_t *num_splits, int num_parts, int batch, int s_q, int h_q,
                       void *out, float *lse, const void *workspace, size_t workspace_bytes,
                       void *stream) {
    if (!num_splits || !out || !lse || !workspace) return MLA_ERR_INVALID_ARG;
    if (!shape_ok(batch, s_q, h_q) || num_parts < 1 || num_parts > 65535) return MLA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(lse, 4) || !aligned(workspace, 256) || !aligned(num_splits, 4))
        return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < mla_workspace_bytes(batch, s_q, h_q, num_parts)) return MLA_ERR_WORKSPACE;
    int rc = check_device();
    if (rc != MLA_OK) return rc;
    const int rows = s_q * h_q;
    const float *o_part = static_cast<const float *>(workspace);
    const float *lse_part = reinterpret_cast<const float *>(static_cast<const char *>(workspace) +
                                                            opart_bytes(batch, rows, num_parts));
    const float *lost_part = lse_part + lsepart_bytes(batch, rows, num_parts) / sizeof(float);
    cudaError_t e = launch_combine(num_splits, batch, num_parts, s_q, h_q, 0, static_cast<__nv_bfloat16 *>(out),
                                   lse, o_part, lse_part, lost_part, static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(e);
}

int mla_decode(const void *q, const void *kv_cache, int64_t num_blocks,
               const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
               const int32_t *tile_meta, const int32_t *num_splits, int num_parts, int batch,
               int s_q, int h_q, float scale, int causal, void *out, float *lse,
               void *workspace, size_t workspace_bytes, void *stream) {
    int rc = mla_decode_split(q, kv_cache, num_blocks, block_table, bt_stride, seqlens, tile_meta,
                              num_splits, num_parts, batch, s_q, h_q, scale, causal, out, lse,
                              workspace, workspace_bytes, stream);
    if (rc != MLA_OK) return rc;
    return mla_decode_combine(num_splits, num_parts, batch, s_q, h_q, out, lse, workspace,
                              workspace_bytes, stream);
}

int mla_decode_fp8(const void *q, const void *kv_cache_fp8, int64_t num_blocks, float kv_scale,
                   const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                   const int32_t *tile_meta, const int32_t *num_splits, int num_parts, int batch, int s_q,
                   int h_q, float scale, int causal, void *out, float *lse, void *workspace,
                   size_t workspace_bytes, void *stream) {
    int rc = mla_decode_split_fp8(q, kv_cache_fp8, num_blocks, kv_scale, block_table, bt_stride, seqlens,
                                  tile_meta, num_splits, num_parts, batch, s_q, h_q, scale, causal, out, lse,
                                  workspace, workspace_bytes, stream);
    if (rc != MLA_OK) return rc;
    return mla_decode_combine(num_splits, num_parts, batch, s_q, h_q, out, lse, workspace,
                              workspace_bytes, stream);
}

int mla_get_metadata_sparse(int batch, int s_q, int h_q, int topk, int num_parts, int fixed_cost,
                            int32_t *tile_meta, int32_t *num_splits, void *stream) {
    if (!tile_meta || !num_splits) return MLA_ERR_INVALID_ARG;
    if (!sparse_shape_ok(batch, s_q, h_q, topk) || num_parts < 1 || num_parts > 65535 || fixed_cost < 0 ||
        fixed_cost > (1 << 20))
        return MLA_ERR_INVALID_ARG;
    if (!aligned(tile_meta, 4) || !aligned(num_splits, 4)) return MLA_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc != MLA_OK) return rc;
    cudaError_t e = launch_metadata(nullptr, topk, batch * s_q, num_parts, fixed_cost, tile_meta, num_splits,
                                    static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(e);
}

int mla_decode_sparse(const void *q, const void *kv_cache, int64_t num_blocks, const int32_t *block_table,
                      int64_t bt_stride, const int32_t *seqlens, const int32_t *indices, int topk,
                      const int32_t *tile_meta, const int32_t *num_splits, int num_parts, int batch, int s_q,
                      int h_q, float scale, void *out, float *lse, void *workspace, size_t workspace_bytes,
                      void *stream) {
    if (!indices || !aligned(indices, 4)) return MLA_ERR_INVALID_ARG;
    if (!sparse_shape_ok(batch, s_q, h_q, topk)) return MLA_ERR_INVALID_ARG;
    const int units = batch * s_q;  // one work unit per (sequence, query token), s_q = 1 each
    // the dense checks with the work-unit shape; seqlens has `batch` entries, read only by the kernel
    int rc = validate_decode(q, kv_cache, num_blocks, block_table, bt_stride, seqlens, tile_meta, num_splits,
                             num_parts, units, 1, h_q, scale, 0, out, lse, workspace, workspace_bytes);
    if (rc != MLA_OK) return rc;
    rc = check_device();
    if (rc != MLA_OK) return rc;
    DecodeParams p = make_params(q, kv_cache, num_blocks, block_table, bt_stride, seqlens, tile_meta, num_splits,
                                 num_parts, units, 1, h_q, scale, 0, out, lse, workspace);
    p.indices = indices;
    p.topk = topk;
    p.sp_sq = s_q;
    CUtensorMap unused;
    std::memset(&unused, 0, sizeof(unused));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_decode_sm100(p, unused, unused, false, st);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) return cuda_status(e);
    const float *lost_part = p.lse_part + lsepart_bytes(units, h_q, num_parts) / sizeof(float);
    e = launch_combine(num_splits, units, num_parts, 1, h_q, s_q, static_cast<__nv_bfloat16 *>(out), lse, p.o_part,
                       p.lse_part, lost_part, st);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(e);
}

static int append_common(const void *new_kv, int n_new, void *kv, int64_t num_blocks, const int32_t *block_table,
                         int64_t bt_stride, const int32_t *seqlens, int batch, bool fp8, float inv_scale,
                         void *stream) {
    if (!new_kv || !kv || !block_table || !seqlens) return MLA_ERR_INVALID_ARG;
    if (batch < 1 || batch > MLA_MAX_BATCH || n_new < 0 || n_new > (1 << 20)) return MLA_ERR_INVALID_ARG;
    if (num_blocks < 1 || num_blocks > (int64_t)(INT32_MAX / MLA_BLOCK_TOKENS)) return MLA_ERR_INVALID_ARG;
    if (bt_stride < 1 || bt_stride > (int64_t)INT32_MAX) return MLA_ERR_INVALID_ARG;
    if (!aligned(new_kv, 16) || !aligned(kv, 16) || !aligned(block_table, 4) || !aligned(seqlens, 4))
        return MLA_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc != MLA_OK) return rc;
    cudaError_t e = launch_append(static_cast<const __nv_bfloat16 *>(new_kv), n_new, kv, num_blocks, block_table,
                                  bt_stride, seqlens, batch, fp8, inv_scale, static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(n_new > 0 ? 1 : 0, std::memory_order_relaxed);
    return cuda_status(e);
}

int mla_append_kv(const void *new_kv, int n_new, void *kv_cache, int64_t num_blocks, const int32_t *block_table,
                  int64_t bt_stride, const int32_t *seqlens, int batch, void *stream) {
    return append_common(new_kv, n_new, kv_cache, num_blocks, block_table, bt_stride, seqlens, batch, false, 0.f,
                         stream);
}

int mla_append_kv_fp8(const void *new_kv, int n_new, void *kv_cache_fp8, int64_t num_blocks, float kv_scale,
                      const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens, int batch,
                      void *stream) {
    if (!std::isfinite(kv_scale) || !(kv_scale > 0.f)) return MLA_ERR_INVALID_ARG;
    const float inv = 1.f / kv_scale;
    if (!std::isfinite(inv)) return MLA_ERR_INVALID_ARG;
    return append_common(new_kv, n_new, kv_cache_fp8, num_blocks, block_table, bt_stride, seqlens, batch, true, inv,
                         stream);
}

int mla_head_gemm(const void *x, int64_t ldx, int64_t x_head_stride, const void *w, void *y, int64_t ldy,
                  int64_t y_head_stride, int m, int n, int k, int heads, void *stream) {
    if (!x || !w || !y) return MLA_ERR_INVALID_ARG;
    if (m < 1 || m > (1 << 24) || heads < 1 || heads > 4096) return MLA_ERR_INVALID_ARG;
    if (k < 64 || k > 65536 || k % 64 != 0 || n < 64 || n > 65536 || n % 64 != 0) return MLA_ERR_INVALID_ARG;
    if (ldx % 8 || x_head_stride % 8 || ldy % 8 || y_head_stride % 8 || x_head_stride < 0 || y_head_stride < 0)
        return MLA_ERR_INVALID_ARG;  // rows and head blocks start on 16-byte boundaries
    const int64_t x_cols = (int64_t)(heads - 1) * x_head_stride + k;
    if (ldx < x_cols || ldy < (int64_t)(heads - 1) * y_head_stride + n || x_cols > INT32_MAX)
        return MLA_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 16)) return MLA_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc != MLA_OK) return rc;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    CUtensorMap map_x, map_w;
    cuuint64_t dx[2] = {(cuuint64_t)x_cols, (cuuint64_t)m}, sx[1] = {(cuuint64_t)ldx * 2};
    cuuint64_t dw[2] = {(cuuint64_t)n, (cuuint64_t)heads * k}, sw[1] = {(cuuint64_t)n * 2};
    cuuint32_t bx[2] = {64, 128}, bw[2] = {64, 64}, estr[2] = {1, 1};
    if (enc(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dx, sx, bx, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        enc(&map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(w), dw, sw, bw, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MLA_ERR_CUDA;
    cudaError_t e = launch_head_gemm(map_x, map_w, static_cast<__nv_bfloat16 *>(y), ldy, y_head_stride, x_head_stride,
                                     m, n, k, heads, static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_status(e);
}

static int decode_host_common(const void *q_host, const void *kv_cache_host, int64_t num_blocks, bool fp8,
                              float kv_scale, const int32_t *block_table_host, int64_t bt_stride,
                              const int32_t *seqlens_host, int batch, int s_q, int h_q, float scale, int causal,
                              void *out_host, float *lse_host, const mla_device_buffers *dev, void *stream) {
    if (!q_host || !kv_cache_host || !block_table_host || !seqlens_host || !out_host || !lse_host || !dev)
        return MLA_ERR_INVALID_ARG;
    if (!shape_ok(batch, s_q, h_q) || num_blocks < 1 || bt_stride < 1) return MLA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int rows = s_q * h_q;
    const size_t q_bytes = (size_t)batch * rows * MLA_D_QK * 2;
    const size_t kv_bytes =
        (size_t)num_blocks * MLA_BLOCK_TOKENS * (fp8 ? (size_t)MLA_FP8_RECORD_BYTES : (size_t)MLA_D_QK * 2);
    const size_t bt_bytes = (size_t)batch * bt_stride * sizeof(int32_t);
    const size_t sl_bytes = (size_t)batch * sizeof(int32_t);
    const size_t out_bytes = (size_t)batch * rows * MLA_D_V * 2;
    const size_t lse_bytes = (size_t)batch * rows * sizeof(float);
    if (!dev->q || !dev->kv_cache || !dev->block_table || !dev->seqlens || !dev->tile_meta ||
        !dev->num_splits || !dev->out || !dev->lse || !dev->workspace)
        return MLA_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc != MLA_OK) return rc;
    if ((rc = cuda_status(cudaMemcpyAsync(dev->q, q_host, q_bytes, cudaMemcpyHostToDevice, st))) != MLA_OK ||
        (rc = cuda_status(cudaMemcpyAsync(dev->kv_cache, kv_cache_host, kv_bytes, cudaMemcpyHostToDevice, st))) != MLA_OK ||
        (rc = cuda_status(cudaMemcpyAsync(dev->block_table, block_table_host, bt_bytes, cudaMemcpyHostToDevice, st))) !=
            MLA_OK ||
        (rc = cuda_status(cudaMemcpyAsync(dev->seqlens, seqlens_host, sl_bytes, cudaMemcpyHostToDevice, st))) != MLA_OK)
        return rc;
    rc = mla_get_metadata(dev->seqlens, batch, h_q, s_q, dev->num_parts, dev->fixed_cost, dev->tile_meta,
                          dev->num_splits, stream);
    if (rc != MLA_OK) return rc;
    if (fp8)
        rc = mla_decode_fp8(dev->q, dev->kv_cache, num_blocks, kv_scale, dev->block_table, bt_stride, dev->seqlens,
                            dev->tile_meta, dev->num_splits, dev->num_parts, batch, s_q, h_q, scale, causal,
                            dev->out, dev->lse, dev->workspace, dev->workspace_bytes, stream);
    else
        rc = mla_decode(dev->q, dev->kv_cache, num_blocks, dev->block_table, bt_stride, dev->seqlens,
                        dev->tile_meta, dev->num_splits, dev->num_parts, batch, s_q, h_q, scale, causal,
                        dev->out, dev->lse, dev->workspace, dev->workspace_bytes, stream);
    if (rc != MLA_OK) return rc;
    if ((rc = cuda_status(cudaMemcpyAsync(out_host, dev->out, out_bytes, cudaMemcpyDeviceToHost, st))) != MLA_OK ||
        (rc = cuda_status(cudaMemcpyAsync(lse_host, dev->lse, lse_bytes, cudaMemcpyDeviceToHost, st))) != MLA_OK)
        return rc;
    return cuda_status(cudaStreamSynchronize(st));
}

int mla_decode_host(const void *q_host, const void *kv_cache_host, int64_t num_blocks,
                    const int32_t *block_table_host, int64_t bt_stride,
                    const int32_t *seqlens_host, int batch, int s_q, int h_q, float scale,
                    int causal, void *out_host, float *lse_host,
                    const mla_device_buffers *dev, void *stream) {
    return decode_host_common(q_host, kv_cache_host, num_blocks, false, 0.f, block_table_host, bt_stride,
                              seqlens_host, batch, s_q, h_q, scale, causal, out_host, lse_host, dev, stream);
}

int mla_decode_host_fp8(const void *q_host, const void *kv_cache_fp8_host, int64_t num_blocks, float kv_scale,
                        const int32_t *block_table_host, int64_t bt_stride, const int32_t *seqlens_host,
                        int batch, int s_q, int h_q, float scale, int causal, void *out_host, float *lse_host,
                        const mla_device_buffers *dev, void *stream) {
    return decode_host_common(q_host, kv_cache_fp8_host, num_blocks, true, kv_scale, block_table_host, bt_stride,
                              seqlens_host, batch, s_q, h_q, scale, causal, out_host, lse_host, dev, stream);
}

int mla_check_status(void *stream) {
    int rc = cuda_status(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    if (rc == MLA_OK) rc = cuda_status(cudaGetLastError());
    if (rc != MLA_OK) return rc;
    unsigned int word = 0, zero = 0;
    if ((rc = cuda_status(cudaMemcpyFromSymbol(&word, g_error_word, sizeof word))) != MLA_OK) return rc;
    if (word != 0 && (rc = cuda_status(cudaMemcpyToSymbol(g_error_word, &zero, sizeof zero))) != MLA_OK) return rc;
    if (word & kErrBounds) return MLA_ERR_BOUNDS;
    if (word & kErrTimeout) return MLA_ERR_TIMEOUT;
    if (word & kErrRange) return MLA_ERR_RANGE;
    return MLA_OK;
}

int64_t mla_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *mla_last_cuda_error(void) {
    const int e = g_last_cuda_error.load(std::memory_order_relaxed);
    return e == 0 ? "no error" : cudaGetErrorString((cudaError_t)e);
}

}  // extern "C"
