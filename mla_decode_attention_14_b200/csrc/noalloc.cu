// noalloc.cu -- decode entry point for callers that cannot allocate device memory.
//
// mla_decode needs a caller-provided workspace for the fp32 partial outputs of sequences
// that are split across several work parts. Some callers cannot call cudaMalloc (or any
// allocating routine) at the point where they decode -- for instance a host runtime that
// owns a fixed memory pool and forbids allocation on its serving path, or code running where
// a late allocation could fail or stall the stream. mla_decode_noalloc runs the same two
// kernels with that workspace taken from the fixed-size array below, which lives in the
// library's device image: every GPU that loads the library holds it until the process exits.
#include <mutex>

namespace mla {
namespace {

// Partial outputs and lse of split pieces: at most kNoAllocScratchBytes per call.
constexpr size_t kNoAllocScratchBytes = (size_t)MLA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device. In host code the array's name is only a
// host-side stand-in, so the address must come from cudaGetSymbolAddress, called with that device
// current. It is cached together with the ID of the context it was looked up in: a device reset
// (or any new primary context) reloads the module, and the next call then looks the address up
// again instead of launching kernels on a stale one.
struct ScratchEntry {
    void *ptr;
    unsigned long long ctx_id;
};
ScratchEntry g_noalloc[kMaxDevices] = {};
std::mutex g_noalloc_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// ID of the current context (unique for the process's lifetime), or 0 if it cannot be read.
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

int noalloc_scratch(void **ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    const unsigned long long ctx = current_ctx_id();  // 0 before the runtime has made a context current
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc[dev].ptr || ctx == 0 || g_noalloc[dev].ctx_id != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
        g_noalloc[dev].ptr = p;
        g_noalloc[dev].ctx_id = current_ctx_id();  // the look-up made the device's context current
    }
    *ptr = g_noalloc[dev].ptr;
    return MLA_OK;
}

}  // namespace
}  // namespace mla

extern "C" int mla_decode_noalloc(const void *q, const void *kv_cache, int64_t num_blocks,
                                  const int32_t *block_table, int64_t bt_stride, const int32_t *seqlens,
                                  const int32_t *tile_meta, const int32_t *num_splits, int num_parts,
                                  int batch, int s_q, int h_q, float scale, int causal, void *out,
                                  float *lse, void *stream) {
    using namespace mla;
    if (!shape_ok(batch, s_q, h_q) || num_parts < 1 || num_parts > 65535) return MLA_ERR_INVALID_ARG;
    const size_t need = mla_workspace_bytes(batch, s_q, h_q, num_parts);
    if (need == 0 || need > kNoAllocScratchBytes) return MLA_ERR_WORKSPACE;  // beyond the fixed scratch
    // Argument checks first (a stand-in workspace pointer: nothing is dereferenced on the host).
    int rc = validate_decode(q, kv_cache, num_blocks, block_table, bt_stride, seqlens, tile_meta, num_splits,
                             num_parts, batch, s_q, h_q, scale, causal, out, lse,
                             reinterpret_cast<const void *>((uintptr_t)256), need);
    if (rc != MLA_OK) return rc;
    rc = check_device();
    if (rc != MLA_OK) return rc;
    void *scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc != MLA_OK) return rc;
    // Nothing in the scratch has to start at zero: every partial the combine kernel reads is
    // written earlier in the same call by the split kernel.
    return mla_decode(q, kv_cache, num_blocks, block_table, bt_stride, seqlens, tile_meta, num_splits, num_parts,
                      batch, s_q, h_q, scale, causal, out, lse, scratch, kNoAllocScratchBytes, stream);
}
