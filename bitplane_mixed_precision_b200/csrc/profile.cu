// Offline error profiles of experts (PagedMoE transcript cues 29-31): the
// relative output error of an expert at each depth, its isotonic repair, and
// prefix selection from the resulting per-expert table.
#include <algorithm>
#include <cstring>
#include <vector>

#include "common.h"
#include "route.cuh"

namespace pmoe {

namespace {

constexpr int kErrThreads = 256;

// err[0] = mean over tokens of ||y_t - ref_t||^2 / ||ref_t||^2 (double sums in a fixed order).
__global__ void __launch_bounds__(kErrThreads) relative_error_kernel(const float *__restrict__ y,
                                                                    const float *__restrict__ ref, int T, int H,
                                                                    float *__restrict__ err)
{
    __shared__ double sd[kErrThreads], sr[kErrThreads];
    double acc = 0.0;
    for (int t = 0; t < T; ++t) {
        double d2 = 0.0, r2 = 0.0;
        for (int i = threadIdx.x; i < H; i += kErrThreads) {
            const double r = ref[(int64_t)t * H + i], d = (double)y[(int64_t)t * H + i] - r;
            d2 = fma(d, d, d2);
            r2 = fma(r, r, r2);
        }
        sd[threadIdx.x] = d2;
        sr[threadIdx.x] = r2;
        __syncthreads();
        for (int s = kErrThreads / 2; s > 0; s >>= 1) {
            if (threadIdx.x < s) {
                sd[threadIdx.x] += sd[threadIdx.x + s];
                sr[threadIdx.x] += sr[threadIdx.x + s];
            }
            __syncthreads();
        }
        if (threadIdx.x == 0)
            acc += sr[0] > 0.0 ? sd[0] / sr[0] : 0.0;
        __syncthreads();
    }
    if (threadIdx.x == 0)
        err[0] = (float)(acc / (double)T);
}

inline uint32_t order_key(float f)
{
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Least-squares non-increasing fit of g[0..n) (pool adjacent violators, equal weights).
void nonincreasing_fit(double *g, int n)
{
    std::vector<double> val;
    std::vector<int> cnt;
    for (int i = 0; i < n; ++i) {
        val.push_back(g[i]);
        cnt.push_back(1);
        while (val.size() > 1 && val[val.size() - 2] < val.back()) {
            const size_t j = val.size() - 2;
            val[j] = (val[j] * cnt[j] + val.back() * cnt.back()) / (cnt[j] + cnt.back());
            cnt[j] += cnt.back();
            val.pop_back();
            cnt.pop_back();
        }
    }
    int i = 0;
    for (size_t j = 0; j < val.size(); ++j)
        for (int c = 0; c < cnt[j]; ++c)
            g[i++] = val[j];
}

// One warp per token: greedy bits by w^2 * (E(b) - E(b+1)) in float, ties to the lower slot.
__global__ void select_table_kernel(const float *__restrict__ w, const int32_t *__restrict__ ids,
                                    const float *__restrict__ table, int T, int k, int B,
                                    uint8_t *__restrict__ depth)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= T)
        return;
    float wi = 0.0f;
    const float *E = nullptr;
    if (lane < k) {
        wi = w[warp * k + lane];
        E = table + (int64_t)ids[warp * k + lane] * 8;
    }
    int b = 1;
    for (int step = k; step < B; ++step) {
        const bool ok = lane < k && b < 8;
        const float pr = ok ? __fmul_rn(__fmul_rn(wi, wi), __fsub_rn(E[b - 1], E[b])) : 0.0f;
        const uint32_t key = ok ? dev::ord_key(pr) : 0u;
        const uint32_t gmax = __reduce_max_sync(0xffffffffu, key);
        const unsigned tied = __ballot_sync(0xffffffffu, ok && key == gmax);
        if (tied == 0u)
            break;
        if (lane == __ffs(tied) - 1)
            b += 1;
    }
    if (lane < k)
        depth[warp * k + lane] = (uint8_t)b;
}

} // namespace
} // namespace pmoe

using namespace pmoe;

extern "C" {

pmoe_status pmoe_relative_error(const float *y, const float *ref, int T, int H, float *err, pmoe_stream stream)
{
    if (!y || !ref || !err || T <= 0 || H <= 0)
        return PMOE_ERR_INVALID_ARG;
    relative_error_kernel<<<1, kErrThreads, 0, (cudaStream_t)stream>>>(y, ref, T, H, err);
    return launch_status();
}

pmoe_status pmoe_profile_repair(const float *raw, int n, float *table)
{
    if (!raw || !table || n < 0)
        return PMOE_ERR_INVALID_ARG;
    for (int e = 0; e < n; ++e) {
        const float *E = raw + (int64_t)e * 8;
        double g[7];
        for (int b = 0; b < 7; ++b)
            g[b] = (double)E[b] - (double)E[b + 1];
        nonincreasing_fit(g, 7);
        double acc = E[7];
        float *out = table + (int64_t)e * 8;
        out[7] = E[7];
        for (int b = 6; b >= 0; --b) {
            acc += g[b] > 0.0 ? g[b] : 0.0;
            out[b] = (float)acc;
        }
    }
    return PMOE_OK;
}

pmoe_status pmoe_select_prefix_table(const float *w, const int32_t *ids, const float *table, int T, int k,
                                     float avg_bits, uint8_t *depth, int on_device, pmoe_stream stream)
{
    if (!w || !ids || !table || !depth || T < 0 || k < 1 || k > 32 || !(avg_bits == avg_bits))
        return PMOE_ERR_INVALID_ARG;
    if (T == 0)
        return PMOE_OK;
    const int B = select_budget(k, avg_bits);
    if (on_device) {
        select_table_kernel<<<(T + 3) / 4, 128, 0, (cudaStream_t)stream>>>(w, ids, table, T, k, B, depth);
        return launch_status();
    }
    for (int t = 0; t < T; ++t) {
        int b[32];
        for (int i = 0; i < k; ++i)
            b[i] = 1;
        for (int step = k; step < B; ++step) {
            int best = -1;
            float bp = 0.0f;
            for (int i = 0; i < k; ++i) {
                if (b[i] >= 8)
                    continue;
                const float wi = w[t * k + i];
                const float *E = table + (int64_t)ids[t * k + i] * 8;
                const float gain = E[b[i] - 1] - E[b[i]];
                const float pr = (wi * wi) * gain;
                // the device's key order (-0 below +0)
                if (best < 0 || order_key(pr) > order_key(bp)) {
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

} // extern "C"
