// Materialise-then-multiply ablation (PagedMoE transcript cue 37; arxivlens
// Results: direct prefix execution against materialising full-precision
// experts). The depth-b prefix of every selected expert is decoded to a bf16
// matrix in HBM (scale * C rounded to bf16), then plain GEMVs run on it.
#include <cuda_bf16.h>

#include "common.h"
#include "dev.cuh"
#include "layer.cuh"

namespace pmoe {

static inline size_t al256m(size_t x) { return (x + 255) & ~(size_t)255; }

struct MatWs {
    __nv_bfloat16 *wmat; // [pairs][3][H*I]
    float *h;            // [pairs][I]
    float *part;         // [pairs][H]
};

static MatWs carve_mat_ws(void *ws, int T, int k, int H, int I, size_t *bytes)
{
    const size_t P = (size_t)T * k;
    size_t off = 0;
    const size_t o_w = off;
    off = al256m(off + P * 3 * (size_t)H * I * 2);
    const size_t o_h = off;
    off = al256m(off + P * I * 4);
    const size_t o_p = off;
    off = al256m(off + P * (size_t)H * 4);
    if (bytes)
        *bytes = off;
    MatWs M{};
    if (ws) {
        char *b = static_cast<char *>(ws);
        M.wmat = reinterpret_cast<__nv_bfloat16 *>(b + o_w);
        M.h = reinterpret_cast<float *>(b + o_h);
        M.part = reinterpret_cast<float *>(b + o_p);
    }
    return M;
}

// One warp per (pair, matrix, tile): decode the prefix and write bf16 weights.
template <int B>
__device__ void decode_tile_bf16(const uint32_t *const *base, int64_t tix, const float *srow_base,
                                 int srow_len, int G, const float *C, int R, int Q, int Kdim,
                                 __nv_bfloat16 *dst)
{
    const int lane = threadIdx.x & 31;
    uint32_t w[8][2];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        w[p][0] = w[p][1] = 0u;
        if (p < B) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(base[p] + tix * 64 + 2 * lane));
            w[p][0] = v.x;
            w[p][1] = v.y;
        }
    }
    uint8_t idx[8][8];
    dev::prefix_indices<B>(w, idx);
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            int row, col;
            dev::tile_coord(lane, q, j, row, col);
            const int n = 16 * R + row, kk = 128 * Q + col;
            const float v = __ldg(srow_base + (int64_t)n * srow_len + kk / G) * __ldg(C + idx[q][j]);
            dst[(int64_t)n * Kdim + kk] = __float2bfloat16_rn(v);
        }
}

__global__ void materialise_kernel(pmoe_layer L, const int32_t *__restrict__ ids,
                                   const uint8_t *__restrict__ depth, int P, MatWs M, int *err)
{
    const int H = L.H, I = L.I, G = L.G;
    const int64_t tiles_per_mat = (int64_t)(H / 128) * (I / 16); // same count for all three
    const int64_t gw = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (gw >= (int64_t)P * 3 * tiles_per_mat)
        return;
    const int pair = (int)(gw / (3 * tiles_per_mat));
    const int m = (int)((gw / tiles_per_mat) % 3);
    const int64_t tix = gw % tiles_per_mat;
    const int e = ids[pair], b = depth[pair];
    const int Kdim = (m == 2) ? I : H;
    const int ktiles = Kdim / 128;
    const int R = (int)(tix / ktiles), Q = (int)(tix % ktiles);
    const int64_t mat_words = (int64_t)H * I / 32;
    const uint32_t *base[8];
    for (int p = 0; p < 8; ++p) {
        base[p] = nullptr;
        if (p < b) {
            const int slot = L.slot_of[e * 8 + p];
            if (slot < 0) {
                *err = 2;
                return;
            }
            base[p] = L.pool + (int64_t)slot * L.slot_words + m * mat_words;
        }
    }
    const int64_t escale = (int64_t)e * (2 * (int64_t)I * (H / G) + (int64_t)H * (I / G));
    const float *sb = L.scales + escale + (int64_t)m * I * (H / G);
    const int srow_len = Kdim / G;
    const float *C = L.codebooks + ((int64_t)e * 3 + m) * 510 + ((1 << b) - 2);
    __nv_bfloat16 *dst = M.wmat + ((int64_t)pair * 3 + m) * (int64_t)H * I;
    switch (b) {
    case 1: decode_tile_bf16<1>(base, tix, sb, srow_len, G, C, R, Q, Kdim, dst); break;
    case 2: decode_tile_bf16<2>(base, tix, sb, srow_len, G, C, R, Q, Kdim, dst); break;
    case 3: decode_tile_bf16<3>(base, tix, sb, srow_len, G, C, R, Q, Kdim, dst); break;
    case 4: decode_tile_bf16<4>(base, tix, sb, srow_len, G, C, R, Q, Kdim, dst); break;
    case 5: decode_tile_bf16<5>(base, tix, sb, srow_len, G, C, R, Q, Kdim, dst); break;
    case 6: decode_tile_bf16<6>(base, tix, sb, srow_len, G, C, R, Q, Kdim, dst); break;
    case 7: decode_tile_bf16<7>(base, tix, sb, srow_len, G, C, R, Q, Kdim, dst); break;
    default: decode_tile_bf16<8>(base, tix, sb, srow_len, G, C, R, Q, Kdim, dst); break;
    }
}

// One warp per output row: dot of a bf16 row (K values) with a vector.
template <bool XBF16>
__device__ __forceinline__ float row_dot(const __nv_bfloat16 *row, const void *x, int K)
{
    const int lane = threadIdx.x & 31;
    float s = 0.0f;
    for (int c = 8 * lane; c < K; c += 256) {
        const uint4 wv = __ldg(reinterpret_cast<const uint4 *>(row + c));
        const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float w0 = __uint_as_float(ws[i] << 16), w1 = __uint_as_float(ws[i] & 0xffff0000u);
            float x0, x1;
            if (XBF16) {
                const uint32_t xv = __ldg(reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(x) + c + 2 * i));
                x0 = __uint_as_float(xv << 16);
                x1 = __uint_as_float(xv & 0xffff0000u);
            } else {
                const float2 xv = __ldg(reinterpret_cast<const float2 *>(static_cast<const float *>(x) + c + 2 * i));
                x0 = xv.x;
                x1 = xv.y;
            }
            s = __fmaf_rn(w0, x0, s);
            s = __fmaf_rn(w1, x1, s);
        }
    }
    return dev::warp_sum(s);
}

__global__ void mat_gateup_kernel(const uint16_t *__restrict__ x, int P, int k, int H, int I, MatWs M)
{
    const int64_t gw = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (gw >= (int64_t)P * I)
        return;
    const int pair = (int)(gw / I), r = (int)(gw % I);
    const uint16_t *xt = x + (int64_t)(pair / k) * H;
    const __nv_bfloat16 *Wg = M.wmat + (int64_t)pair * 3 * H * I;
    const float g = row_dot<true>(Wg + (int64_t)r * H, xt, H);
    const float u = row_dot<true>(Wg + (int64_t)H * I + (int64_t)r * H, xt, H);
    if ((threadIdx.x & 31) == 0)
        M.h[(int64_t)pair * I + r] = g / (1.0f + expf(-g)) * u;
}

__global__ void mat_down_kernel(int P, int H, int I, MatWs M)
{
    const int64_t gw = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (gw >= (int64_t)P * H)
        return;
    const int pair = (int)(gw / H), r = (int)(gw % H);
    const __nv_bfloat16 *Wd = M.wmat + ((int64_t)pair * 3 + 2) * H * I;
    const float v = row_dot<false>(Wd + (int64_t)r * I, M.h + (int64_t)pair * I, I);
    if ((threadIdx.x & 31) == 0)
        M.part[(int64_t)pair * H + r] = v;
}

__global__ void mat_combine_kernel(const float *__restrict__ w, int T, int k, int H, MatWs M,
                                   float *__restrict__ y)
{
    const int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (n >= (int64_t)T * H)
        return;
    const int t = (int)(n / H), c = (int)(n % H);
    float s = 0.0f;
    for (int i = 0; i < k; ++i)
        s = __fmaf_rn(w[t * k + i], M.part[(int64_t)(t * k + i) * H + c], s);
    y[n] = s;
}

} // namespace pmoe

using namespace pmoe;

extern "C" {

size_t pmoe_materialise_workspace_bytes(int T, int k, int E, int H, int I)
{
    (void)E;
    if (T < 0 || k < 1 || H <= 0 || I <= 0)
        return 0;
    size_t b = 0;
    carve_mat_ws(nullptr, T, k, H, I, &b);
    return b + 256; // + error word
}

pmoe_status pmoe_materialise_layer_fwd(const pmoe_layer *L, const uint16_t *x, const int32_t *ids,
                                       const float *w, const uint8_t *depth, int T, int k,
                                       float *y, void *ws, size_t ws_bytes, pmoe_stream stream)
{
    PMOE_TRY(check_layer(L, T, k));
    if (T == 0)
        return PMOE_OK;
    if (!x || !ids || !w || !depth || !y || !ws || !aligned(x, 16) || !aligned(ws, 256) ||
        L->H % 256 || L->I % 256)
        return PMOE_ERR_INVALID_ARG;
    size_t need = 0;
    carve_mat_ws(nullptr, T, k, L->H, L->I, &need);
    if (ws_bytes < need + 256)
        return PMOE_ERR_WORKSPACE;
    MatWs M = carve_mat_ws(ws, T, k, L->H, L->I, nullptr);
    int *err = reinterpret_cast<int *>(static_cast<char *>(ws) + need);
    cudaStream_t st = (cudaStream_t)stream;
    const int P = T * k;
    PMOE_CUDA(cudaMemsetAsync(err, 0, 4, st));
    const int64_t warps = (int64_t)P * 3 * (L->H / 128) * (L->I / 16);
    materialise_kernel<<<(unsigned)((warps + 3) / 4), 128, 0, st>>>(*L, ids, depth, P, M, err);
    PMOE_TRY(launch_status());
    const int64_t wa = (int64_t)P * L->I;
    mat_gateup_kernel<<<(unsigned)((wa + 7) / 8), 256, 0, st>>>(x, P, k, L->H, L->I, M);
    PMOE_TRY(launch_status());
    const int64_t wb = (int64_t)P * L->H;
    mat_down_kernel<<<(unsigned)((wb + 7) / 8), 256, 0, st>>>(P, L->H, L->I, M);
    PMOE_TRY(launch_status());
    const int64_t n = (int64_t)T * L->H;
    mat_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(w, T, k, L->H, M, y);
    return launch_status();
}

} // extern "C"
