// csa_decode_index_topk_noalloc: the decode indexer + top-k with its score scratch in a
// fixed, library-owned device array instead of a caller-provided workspace.
//
// For callers that cannot allocate device memory themselves -- for example code running
// inside a host framework or serving engine that owns every device allocation and hands
// out no scratch, or a plugin that is not allowed to call cudaMalloc.  The scratch is a
// file-scope device array of kMaxScores fp32 values (8 MiB); every GPU that loads the
// library holds it until the process exits.
//
// Host code must not use the array's name as a device address (in host code it is only a
// stand-in): the first call on each device, with that device current, resolves the real
// address once with cudaGetSymbolAddress and keeps it.  That first call should therefore
// come before any stream capture.  All calls share the one array, which keeps the last
// call's contents: calls whose work overlaps on the GPU (other streams, other host
// threads) race on it.  Nothing in it has to start at zero -- every score the top-k reads
// is written earlier in the same call.
#include <mutex>

#include "internal.cuh"

namespace hcsa {
namespace {

constexpr int64_t kMaxScores = (int64_t)1 << 21;   // 8 MiB of fp32

static __device__ __align__(256) float g_noalloc_scores[kMaxScores];

std::mutex g_setup_mu;
float *g_scores_ptr[64];

// Device address of the scratch array on the current device (resolved once per device).
hcsa_status scratch_for_current_device(float **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HCSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scores_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scores) != cudaSuccess || !p) return HCSA_ERR_CUDA;
        g_scores_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_scores_ptr[dev];
    return HCSA_OK;
}

}  // namespace
}  // namespace hcsa

using namespace hcsa;

extern "C" hcsa_status csa_decode_index_topk_noalloc(const hcsa_params *p, const hcsa_cache *cache,
                                                     const int32_t *pos, const void *qi, int64_t ld_qi,
                                                     const void *w, int64_t ld_w, int32_t *sel, void *stream) {
    // malformed requests get the same answer as from csa_decode_index_topk, whatever their size
    const hcsa_status v = check_decode_index_topk_args(p, cache, pos, qi, ld_qi, w, ld_w, sel);
    if (v != HCSA_OK) return v;
    // the scores of all B sequences must fit the fixed scratch array
    const size_t need = hcsa_workspace_bytes(p, HCSA_OP_CSA_DECODE_INDEX_TOPK);
    if (need > sizeof(g_noalloc_scores)) return HCSA_ERR_WORKSPACE;
    float *scratch = nullptr;
    hcsa_status s = scratch_for_current_device(&scratch);
    if (s != HCSA_OK) return s;
    return csa_decode_index_topk(p, cache, pos, qi, ld_qi, w, ld_w, sel, scratch, need, stream);
}
