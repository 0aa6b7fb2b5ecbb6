// Host-side helpers shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/pmoe.h"

namespace pmoe {

void set_cuda_error(cudaError_t e);

// Records a CUDA failure and returns PMOE_ERR_CUDA, or PMOE_OK.
inline pmoe_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess)
        return PMOE_OK;
    set_cuda_error(e);
    return PMOE_ERR_CUDA;
}

inline pmoe_status launch_status() { return cuda_status(cudaGetLastError()); }

#define PMOE_TRY(expr)                                                                             \
    do {                                                                                           \
        pmoe_status _s = (expr);                                                                   \
        if (_s != PMOE_OK)                                                                         \
            return _s;                                                                             \
    } while (0)

#define PMOE_CUDA(expr) PMOE_TRY(::pmoe::cuda_status(expr))

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Gaussian helpers (host, double): own implementations, see format.cu.
double norm_ppf(double p);
void tree_codebook(float *cb510);
void quantile_thresholds(double *t256);

// Device-side budget rule shared by host and device selection code.
inline int select_budget(int k, float avg_bits)
{
    double b = (double)avg_bits * (double)k + 1e-4;
    int B = (int)b;
    if ((double)B > b)
        B -= 1;
    if (B < k)
        B = k;
    if (B > 8 * k)
        B = 8 * k;
    return B;
}

constexpr int kNumSMs = 148;

} // namespace pmoe
