// api.cu -- host side of the C ABI declared in include/mla.h: argument validation,
// workspace layout, device checks, kernel launches and the device error word.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/mla.h"
#include "common.cuh"

namespace mla {

cudaError_t launch_metadata(const int32_t *seqlens, int batch, int num_parts, int fixed_cost,
                            int32_t *tile_meta, int32_t *num_splits, cudaStream_t stream);
cudaError_t launch_combine(const int32_t *num_splits, int batch, int num_parts, int s_q, int h_q,
                           __nv_bfloat16 *out, float *lse, const float *o_part,
                           const float *lse_part, cudaStream_t stream);
cudaError_t launch_decode_simt(const DecodeParams &p, cudaStream_t stream);

static std::atomic<int64_t> g_launches{0};

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

int shape_ok(int batch, int s_q, int h_q) {
    if (batch < 1 || batch > MLA_MAX_BATCH) return 0;
    if (s_q < 1 || h_q < 1) return 0;
    if ((int64_t)s_q * h_q > MLA_MAX_ROWS) return 0;
    return 1;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout: fp32 o_part[(batch + num_parts) * rows * 512], then fp32
// lse_part[(batch + num_parts) * rows].
size_t opart_bytes(int batch, int rows, int num_parts) {
    return (size_t)(batch + num_parts) * rows * MLA_D_V * sizeof(float);
}

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
    if (!std::isfinite(scale)) return MLA_ERR_INVALID_ARG;
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

int mla_default_fixed_cost(int h_q, int s_q) {
    (void)h_q;
    (void)s_q;
    return 5;
}

size_t mla_workspace_bytes(int batch, int s_q, int h_q, int num_parts) {
    if (!shape_ok(batch, s_q, h_q) || num_parts < 1) return 0;
    const int rows = s_q * h_q;
    size_t b = opart_bytes(batch, rows, num_parts) + (size_t)(batch + num_parts) * rows * sizeof(float);
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
    cudaError_t e = launch_metadata(seqlens, batch, num_parts, fixed_cost, tile_meta, num_splits,
                                    static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
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
    cudaError_t e = launch_decode_simt(p, static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
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
    cudaError_t e = launch_combine(num_splits, batch, num_parts, s_q, h_q, static_cast<__nv_bfloat16 *>(out), lse,
                                   o_part, lse_part, static_cast<cudaStream_t>(stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
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

int mla_decode_host(const void *q_host, const void *kv_cache_host, int64_t num_blocks,
                    const int32_t *block_table_host, int64_t bt_stride,
                    const int32_t *seqlens_host, int batch, int s_q, int h_q, float scale,
                    int causal, void *out_host, float *lse_host,
                    const mla_device_buffers *dev, void *stream) {
    if (!q_host || !kv_cache_host || !block_table_host || !seqlens_host || !out_host || !lse_host || !dev)
        return MLA_ERR_INVALID_ARG;
    if (!shape_ok(batch, s_q, h_q) || num_blocks < 1 || bt_stride < 1) return MLA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int rows = s_q * h_q;
    const size_t q_bytes = (size_t)batch * rows * MLA_D_QK * 2;
    const size_t kv_bytes = (size_t)num_blocks * MLA_BLOCK_TOKENS * MLA_D_QK * 2;
    const size_t bt_bytes = (size_t)batch * bt_stride * sizeof(int32_t);
    const size_t sl_bytes = (size_t)batch * sizeof(int32_t);
    const size_t out_bytes = (size_t)batch * rows * MLA_D_V * 2;
    const size_t lse_bytes = (size_t)batch * rows * sizeof(float);
    if (!dev->q || !dev->kv_cache || !dev->block_table || !dev->seqlens || !dev->tile_meta ||
        !dev->num_splits || !dev->out || !dev->lse || !dev->workspace)
        return MLA_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc != MLA_OK) return rc;
    if (cudaMemcpyAsync(dev->q, q_host, q_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(dev->kv_cache, kv_cache_host, kv_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(dev->block_table, block_table_host, bt_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(dev->seqlens, seqlens_host, sl_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MLA_ERR_CUDA;
    rc = mla_get_metadata(dev->seqlens, batch, h_q, s_q, dev->num_parts, dev->fixed_cost, dev->tile_meta,
                          dev->num_splits, stream);
    if (rc != MLA_OK) return rc;
    rc = mla_decode(dev->q, dev->kv_cache, num_blocks, dev->block_table, bt_stride, dev->seqlens,
                    dev->tile_meta, dev->num_splits, dev->num_parts, batch, s_q, h_q, scale, causal,
                    dev->out, dev->lse, dev->workspace, dev->workspace_bytes, stream);
    if (rc != MLA_OK) return rc;
    if (cudaMemcpyAsync(out_host, dev->out, out_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(lse_host, dev->lse, lse_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MLA_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_check_status(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof word) != cudaSuccess) return MLA_ERR_CUDA;
    if (word != 0 && cudaMemcpyToSymbol(g_error_word, &zero, sizeof zero) != cudaSuccess) return MLA_ERR_CUDA;
    if (word & kErrBounds) return MLA_ERR_BOUNDS;
    if (word & kErrTimeout) return MLA_ERR_TIMEOUT;
    return MLA_OK;
}

int64_t mla_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
