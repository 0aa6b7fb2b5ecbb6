// Warp-level routing and prefix selection for one token.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace pmoe {
namespace dev {

// Order-preserving map of float to uint32 (larger float -> larger key, > 0);
// -0 and +0 are equal logits and get the same key (a tie, to the lower id).
__device__ __forceinline__ uint32_t ord_key(float f)
{
    uint32_t u = __float_as_uint(f);
    u = (u == 0x80000000u) ? 0u : u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of l[0..E) (ties to the lower id), descending, and softmax over the k
// (PagedMoE transcript cue 4: k experts, weights summing to one). Executed by
// a full warp; lane s < k receives slot s. Lane c holds ids c, c+32, ...
// stage: E floats of shared memory for this warp; the logits are copied there
// once so that the rescans after each pick read shared memory.
__device__ __forceinline__ void route_token(const float *__restrict__ l, int E, int k, float *stage, int &id_out,
                                            float &w_out)
{
    const int lane = threadIdx.x & 31;
    for (int j = lane; j < E; j += 32)
        stage[j] = __ldg(l + j);
    __syncwarp();
    // a picked id is overwritten with the bit pattern whose key is 0 (never picked)
    auto local_best = [&](uint32_t &bk, int &bj) {
        bk = 0u;
        bj = -1;
        for (int j = 0; lane + 32 * j < E; ++j) {
            const uint32_t key = ord_key(stage[lane + 32 * j]);
            if (key > bk) {
                bk = key;
                bj = j;
            }
        }
    };
    uint32_t bk;
    int bj;
    local_best(bk, bj);
    int my_id = 0;
    for (int s = 0; s < k; ++s) {
        const uint32_t gmax = __reduce_max_sync(0xffffffffu, bk);
        const unsigned cand = (bj >= 0 && bk == gmax) ? (unsigned)(lane + 32 * bj) : 0x7fffffffu;
        const unsigned win = __reduce_min_sync(0xffffffffu, cand);
        if (lane == s)
            my_id = (int)win;
        if (lane == (int)(win & 31u)) {
            stage[win] = __uint_as_float(0xffffffffu);
            local_best(bk, bj);
        }
    }
    const float my_l = (lane < k) ? __ldg(l + my_id) : 0.0f;
    __syncwarp();
    const double l0 = (double)__shfl_sync(0xffffffffu, my_l, 0);
    const double e = (lane < k) ? exp((double)my_l - l0) : 0.0;
    double sum = 0.0;
    for (int s = 0; s < k; ++s)
        sum = __dadd_rn(sum, __shfl_sync(0xffffffffu, e, s));
    id_out = my_id;
    w_out = (lane < k) ? __double2float_rn(__ddiv_rn(e, sum)) : 0.0f;
}

// route_token for E <= 32*NPL with the logits' keys in registers (NPL per lane,
// every index compile-time): the same picks, ties and weights.
template <int NPL>
__device__ __forceinline__ void route_token_reg(const float *__restrict__ l, int E, int k, int &id_out, float &w_out)
{
    const int lane = threadIdx.x & 31;
    uint32_t key[NPL];
#pragma unroll
    for (int j = 0; j < NPL; ++j)
        key[j] = (lane + 32 * j < E) ? ord_key(__ldg(l + lane + 32 * j)) : 0u;
    uint32_t bk;
    int bj;
    auto local_best = [&]() {
        bk = 0u;
        bj = -1;
#pragma unroll
        for (int j = 0; j < NPL; ++j)
            if (key[j] > bk) {
                bk = key[j];
                bj = j;
            }
    };
    local_best();
    int my_id = 0;
    for (int s = 0; s < k; ++s) {
        const uint32_t gmax = __reduce_max_sync(0xffffffffu, bk);
        const unsigned cand = (bj >= 0 && bk == gmax) ? (unsigned)(lane + 32 * bj) : 0x7fffffffu;
        const unsigned win = __reduce_min_sync(0xffffffffu, cand);
        if (lane == s)
            my_id = (int)win;
        if (lane == (int)(win & 31u)) {
            const int jw = (int)(win >> 5);
#pragma unroll
            for (int j = 0; j < NPL; ++j)
                if (j == jw)
                    key[j] = 0u;
            local_best();
        }
    }
    const float my_l = (lane < k) ? __ldg(l + my_id) : 0.0f;
    const double l0 = (double)__shfl_sync(0xffffffffu, my_l, 0);
    const double e = (lane < k) ? exp((double)my_l - l0) : 0.0;
    double sum = 0.0;
    for (int s = 0; s < k; ++s)
        sum = __dadd_rn(sum, __shfl_sync(0xffffffffu, e, s));
    id_out = my_id;
    w_out = (lane < k) ? __double2float_rn(__ddiv_rn(e, sum)) : 0.0f;
}

// Greedy prefix selection for one token (transcript cue 29): lane i < k holds
// v_i = w_i * s_{e_i}; B - k rounds grant one bit to the largest v_i * 2^-b_i
// (exact ldexp; ties to the lower slot; 8-bit slots skipped). Returns b_i.
__device__ __forceinline__ int select_token(float v, int k, int B, float * /*unused scratch*/)
{
    const int lane = threadIdx.x & 31;
    int b = 1;
    for (int step = k; step < B; ++step) {
        const bool ok = lane < k && b < 8;
        const uint32_t key = ok ? __float_as_uint(ldexpf(v, -b)) : 0u;
        const uint32_t gmax = __reduce_max_sync(0xffffffffu, ok ? key : 0u);
        const unsigned tied = __ballot_sync(0xffffffffu, ok && key == gmax);
        if (tied == 0u)
            break;
        if (lane == __ffs(tied) - 1)
            b += 1;
    }
    return b;
}

} // namespace dev
} // namespace pmoe
