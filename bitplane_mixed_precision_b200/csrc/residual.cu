// Residual stream between stacked MoE layers: r += y, x = bf16(r / rms(r)).
// Not part of the PagedMoE method itself; it chains the layers of a decode
// step so that each layer's input comes from the previous layer's output.
#include <cuda_bf16.h>

#include "common.h"

namespace pmoe {

namespace {

constexpr int kResThreads = 256;

// One block per token; every thread sums its own elements in order, then a
// fixed shared-memory tree: the result does not depend on timing.
__global__ void __launch_bounds__(kResThreads) residual_norm_kernel(float *__restrict__ r,
                                                                   const float *__restrict__ y, int H,
                                                                   uint16_t *__restrict__ x)
{
    __shared__ float part[kResThreads];
    const int t = blockIdx.x, tid = threadIdx.x;
    float *rt = r + (int64_t)t * H;
    float ss = 0.0f;
    for (int i = 4 * tid; i < H; i += 4 * kResThreads) {
        float4 v = *reinterpret_cast<const float4 *>(rt + i);
        if (y != nullptr) {
            const float4 d = *reinterpret_cast<const float4 *>(y + (int64_t)t * H + i);
            v.x += d.x;
            v.y += d.y;
            v.z += d.z;
            v.w += d.w;
            *reinterpret_cast<float4 *>(rt + i) = v;
        }
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
    }
    part[tid] = ss;
    __syncthreads();
    for (int s = kResThreads / 2; s > 0; s >>= 1) {
        if (tid < s)
            part[tid] += part[tid + s];
        __syncthreads();
    }
    const float ms = part[0] / (float)H;
    const float inv = ms > 0.0f ? 1.0f / sqrtf(ms) : 0.0f;
    for (int i = 4 * tid; i < H; i += 4 * kResThreads) {
        const float4 v = *reinterpret_cast<const float4 *>(rt + i);
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x * inv, v.y * inv);
        const __nv_bfloat162 b = __floats2bfloat162_rn(v.z * inv, v.w * inv);
        uint2 o;
        o.x = *reinterpret_cast<const uint32_t *>(&a);
        o.y = *reinterpret_cast<const uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(x + (int64_t)t * H + i) = o;
    }
}

} // namespace
} // namespace pmoe

using namespace pmoe;

extern "C" pmoe_status pmoe_residual_norm(float *r, const float *y, int T, int H, uint16_t *x, pmoe_stream stream)
{
    if (!r || !x || T < 0 || H <= 0 || H % 4 || !aligned(r, 16) || (y && !aligned(y, 16)) || !aligned(x, 8))
        return PMOE_ERR_INVALID_ARG;
    if (T == 0)
        return PMOE_OK;
    residual_norm_kernel<<<T, kResThreads, 0, (cudaStream_t)stream>>>(r, y, H, x);
    return launch_status();
}
