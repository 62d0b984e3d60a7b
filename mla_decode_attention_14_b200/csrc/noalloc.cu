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
// host-side stand-in, so the address must come from cudaGetSymbolAddress, called once per
// device with that device current.
void *g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

int noalloc_scratch(void **ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
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
