// Routing (top-k + softmax, PagedMoE transcript cue 4) and prefix selection
// (greedy bit allocation on w^2 * E_e(b), transcript cues 29-31).
#include <cmath>
#include "common.h"
#include "dev.cuh"
#include "route.cuh"

namespace pmoe {

// ---------------------------------------------------------------- host selection

// Greedy: all experts start at 1 bit; B-k times the largest w*s*2^-b (ties to
// the lower slot, 8-bit experts skipped) gets one more bit.
static void select_host(const float *w, const int32_t *ids, const float *sens, int T, int k,
                        float avg_bits, uint8_t *depth)
{
    const int B = select_budget(k, avg_bits);
    float v[32];
    int b[32];
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < k; ++i) {
            v[i] = w[t * k + i] * sens[ids[t * k + i]];
            b[i] = 1;
        }
        for (int step = k; step < B; ++step) {
            int best = -1;
            float bp = 0.0f;
            for (int i = 0; i < k; ++i) {
                if (b[i] >= 8)
                    continue;
                const float pr = ldexpf(v[i], -b[i]);
                if (best < 0 || pr > bp) {
                    best = i;
                    bp = pr;
                }
            }
            if (best < 0)
                break;
            b[best] += 1;
        }
        for (int i = 0; i < k; ++i)
            depth[t * k + i] = (uint8_t)b[i];
    }
}

// ---------------------------------------------------------------- device kernels

// One warp (block) per token, its logits staged in shared memory; see
// route.cuh for the device functions.
__global__ void route_kernel(const float *__restrict__ logits, int T, int E, int k,
                             int32_t *__restrict__ ids, float *__restrict__ w)
{
    extern __shared__ float stage[];
    const int warp = blockIdx.x;
    if (warp >= T)
        return;
    int id;
    float wt;
    if (E <= 512)
        dev::route_token_reg<16>(logits + (int64_t)warp * E, E, k, id, wt);
    else
        dev::route_token(logits + (int64_t)warp * E, E, k, stage, id, wt);
    const int lane = threadIdx.x & 31;
    if (lane < k) {
        ids[warp * k + lane] = id;
        w[warp * k + lane] = wt;
    }
}

__global__ void select_kernel(const float *__restrict__ w, const int32_t *__restrict__ ids,
                              const float *__restrict__ sens, int T, int k, int B,
                              uint8_t *__restrict__ depth)
{
    __shared__ float prio[4][7 * 32];
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (warp >= T)
        return;
    const int lane = threadIdx.x & 31;
    float v = 0.0f;
    if (lane < k)
        v = __fmul_rn(w[warp * k + lane], sens[ids[warp * k + lane]]);
    const int b = dev::select_token(v, k, B, prio[(threadIdx.x >> 5) & 3]);
    if (lane < k)
        depth[warp * k + lane] = (uint8_t)b;
}

} // namespace pmoe

using namespace pmoe;

extern "C" {

pmoe_status pmoe_route(const float *logits, int T, int E, int k, int32_t *ids, float *w,
                       pmoe_stream stream)
{
    if (!logits || !ids || !w || T < 0 || k < 1 || k > 32 || E < k || E > 4096)
        return PMOE_ERR_INVALID_ARG;
    if (T == 0)
        return PMOE_OK;
    route_kernel<<<T, 32, (size_t)E * sizeof(float), (cudaStream_t)stream>>>(logits, T, E, k, ids, w);
    return launch_status();
}

pmoe_status pmoe_select_prefix_cache_aware(const float *w, const int32_t *ids, const float *sens,
                                           const uint8_t *resident, int T, int k, int fetch_budget,
                                           uint8_t *depth)
{
    if (!w || !ids || !sens || !resident || !depth || T < 0 || k < 1 || k > 32 || fetch_budget < 0)
        return PMOE_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t) {
        float v[32];
        int b[32], fetched = 0;
        for (int i = 0; i < k; ++i) {
            const int r = resident[t * k + i] < 8 ? resident[t * k + i] : 8;
            v[i] = w[t * k + i] * sens[ids[t * k + i]];
            b[i] = r > 0 ? r : 1; // resident planes are free; the first plane is always needed
            fetched += (r == 0) ? 1 : 0;
        }
        for (; fetched < fetch_budget; ++fetched) {
            int best = -1;
            float bp = 0.0f;
            for (int i = 0; i < k; ++i) {
                if (b[i] >= 8)
                    continue;
                const float pr = ldexpf(v[i], -b[i]);
                if (best < 0 || pr > bp) {
                    best = i;
                    bp = pr;
                }
            }
            if (best < 0)
                break;
            b[best] += 1;
        }
        for (int i = 0; i < k; ++i)
            depth[t * k + i] = (uint8_t)b[i];
    }
    return PMOE_OK;
}

pmoe_status pmoe_select_prefix_cache_aware_matched(const float *w, const int32_t *ids, const float *sens,
                                                   const uint8_t *resident, int T, int k, float avg_bits,
                                                   uint8_t *depth, double *surrogate)
{
    if (!w || !ids || !sens || !resident || !depth || T < 0 || k < 1 || k > 32 || !(avg_bits == avg_bits))
        return PMOE_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t) {
        const float *wt = w + (int64_t)t * k;
        const int32_t *it = ids + (int64_t)t * k;
        const uint8_t *rt = resident + (int64_t)t * k;
        uint8_t plain[32];
        select_host(wt, it, sens, 1, k, avg_bits, plain);
        // the budget: planes the cache-oblivious depths would fetch for this token
        int fetch = 0;
        for (int i = 0; i < k; ++i)
            fetch += plain[i] > rt[i] ? plain[i] - rt[i] : 0;
        PMOE_TRY(pmoe_select_prefix_cache_aware(wt, it, sens, rt, 1, k, fetch, depth + (int64_t)t * k));
        if (surrogate) {
            for (int i = 0; i < k; ++i) {
                const double v = (double)wt[i] * (double)sens[it[i]];
                surrogate[0] += v * v * std::ldexp(1.0, -2 * plain[i]);
                surrogate[1] += v * v * std::ldexp(1.0, -2 * depth[(int64_t)t * k + i]);
            }
        }
    }
    return PMOE_OK;
}

pmoe_status pmoe_select_prefix(const float *w, const int32_t *ids, const float *sens, int T, int k,
                               float avg_bits, uint8_t *depth, int on_device, pmoe_stream stream)
{
    if (!w || !ids || !sens || !depth || T < 0 || k < 1 || k > 32 || !(avg_bits == avg_bits))
        return PMOE_ERR_INVALID_ARG;
    if (T == 0)
        return PMOE_OK;
    if (!on_device) {
        select_host(w, ids, sens, T, k, avg_bits, depth);
        return PMOE_OK;
    }
    const int B = select_budget(k, avg_bits);
    const int blocks = (T + 3) / 4;
    select_kernel<<<blocks, 128, 0, (cudaStream_t)stream>>>(w, ids, sens, T, k, B, depth);
    return launch_status();
}

} // extern "C"
