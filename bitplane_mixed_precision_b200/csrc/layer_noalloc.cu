// pmoe_moe_layer_fwd_noalloc: the MoE layer call for callers that cannot
// allocate device memory, with the scratch space in a fixed array that lives
// in the library's own device image (see include/pmoe.h).
#include <mutex>

#include "common.h"
#include "layer.cuh"

namespace pmoe {

// Scratch of the allocation-free layer call: enough for the workspace of
// pmoe_moe_layer_fwd up to this size (pmoe_layer_workspace_bytes). Every GPU
// that loads the library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = 8u << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[128] = {};
}

// Device address of the scratch array on the current device; looked up once
// per device (the host-side symbol is only a stand-in for it) and kept for the
// life of the process, so the library is not to be used across a reset of the
// device (cudaDeviceReset).
static pmoe_status noalloc_scratch(void **out)
{
    int dev = 0;
    PMOE_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 128)
        return PMOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        PMOE_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
        if (p == nullptr)
            return PMOE_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return PMOE_OK;
}

} // namespace pmoe

using namespace pmoe;

extern "C" size_t pmoe_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" pmoe_status pmoe_noalloc_layer_error(int *code, int *detail, pmoe_stream stream)
{
    if (!code)
        return PMOE_ERR_INVALID_ARG;
    void *ws = nullptr;
    PMOE_TRY(noalloc_scratch(&ws));
    // the error record is the first words of the array, as in a workspace (pmoe_layer_error)
    int f[8];
    PMOE_CUDA(cudaMemcpyAsync(f, ws, sizeof(f), cudaMemcpyDeviceToHost, (cudaStream_t)stream));
    PMOE_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
    *code = f[0];
    if (detail)
        *detail = f[4];
    return PMOE_OK;
}

extern "C" pmoe_status pmoe_moe_layer_fwd_noalloc(const pmoe_layer *L, const uint16_t *x, const int32_t *ids,
                                                  const float *w, const uint8_t *depth, int T, int k, float *y,
                                                  pmoe_stream stream)
{
    PMOE_TRY(check_layer(L, T, k));
    if (T == 0)
        return PMOE_OK;
    if (!x || !ids || !w || !depth || !y || !aligned(x, 8))
        return PMOE_ERR_INVALID_ARG;
    size_t need = 0;
    carve_layer_ws(nullptr, T, k, L->H, L->I, &need);
    if (need > kNoAllocScratchBytes)
        return PMOE_ERR_WORKSPACE;
    void *ws = nullptr;
    PMOE_TRY(noalloc_scratch(&ws));
    // every counter and flag the kernels read is reset by the prep kernel of each call
    return launch_layer(L, nullptr, nullptr, x, const_cast<int32_t *>(ids), const_cast<float *>(w),
                        const_cast<uint8_t *>(depth), T, k, 0, y, ws, kNoAllocScratchBytes, (cudaStream_t)stream);
}
