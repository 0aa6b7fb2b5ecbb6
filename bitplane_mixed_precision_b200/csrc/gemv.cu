// pmoe_expert_gemv: one expert matrix times one vector, decoding the depth-b
// bitplane prefix in registers (PagedMoE transcript cue 37; arxivlens
// Methodology: cached prefixes executed without materialising full-precision
// weights).
#include <cuda_bf16.h>

#include "common.h"
#include "dev.cuh"
#include "xfrag.cuh"

namespace pmoe {

// One CTA of 4 warps per 16-row strip; warps take the strip's 128-column tiles
// round robin and reduce through shared memory at the end.
template <int B, int GS, bool XBF16>
__global__ void __launch_bounds__(128) gemv_kernel(pmoe_matrix m, const void *__restrict__ x,
                                                   float *__restrict__ y)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int K = m.K, ktiles = K / 128, ng = K / m.G;
    uint32_t *xf = reinterpret_cast<uint32_t *>(smem);                     // [K/32][24]
    int *xe = reinterpret_cast<int *>(xf + (K / 32) * dev::kFragWords);     // [K/128]
    uint32_t *big = reinterpret_cast<uint32_t *>(xe + ktiles);        // [256] for B >= 5
    float *red = reinterpret_cast<float *>(big + 256);                // [4][16]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int R = blockIdx.x;

    for (int Q = warp; Q < ktiles; Q += 4)
        dev::make_xfrag_tile<XBF16>(x, Q, xf, xe);
    dev::RegTab tab;
    dev::build_tab(m.codebook, B, tab, (B >= 5 && warp == 0) ? big : nullptr);
    __syncthreads();

    const int g = lane >> 2, t = lane & 3;
    // B column g: byte part g of x for g < 3, zero otherwise (xfrag.cuh)
    const bool fz = g >= 3;
    const float lf = dev::combine24_lane_factor(t);
    float acc0 = 0.0f, acc1 = 0.0f;
    const float *srow0 = m.scales + (int64_t)(16 * R + g) * ng;
    const float *srow1 = srow0 + 8 * (int64_t)ng;
    for (int Q = warp; Q < ktiles; Q += 4) {
        const int64_t tix = (int64_t)R * ktiles + Q;
        uint32_t w[8][2];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            w[p][0] = w[p][1] = 0u;
            if (p < B) {
                const uint2 v = __ldg(reinterpret_cast<const uint2 *>(m.planes + p * m.plane_stride_words +
                                                                      tix * 64 + 2 * lane));
                w[p][0] = v.x;
                w[p][1] = v.y;
            }
        }
        const float fac = lf * ldexpf(1.0f, -(tab.f + xe[Q]));
        int dh[4] = {0, 0, 0, 0}, dl[4] = {0, 0, 0, 0};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            uint32_t ah[4], al[4];
            dev::decode_kstep<B>(w, s, tab, big, ah, al);
            uint32_t b0 = 0u, b1 = 0u;
            if (!fz) {
                const uint2 v =
                    *reinterpret_cast<const uint2 *>(xf + (Q * 4 + s) * dev::kFragWords + dev::frag_offset(g, t));
                b0 = v.x;
                b1 = v.y;
            }
            dev::mma_s8(dh, ah, b0, b1);
            dev::mma_s8(dl, al, b0, b1);
            if ((s + 1) % GS == 0) {
                const int grp = (128 * Q + 32 * s) / (32 * GS);
                acc0 = __fmaf_rn(dev::combine24(dh[0], dh[1], dl[0], dl[1]), __ldg(srow0 + grp) * fac, acc0);
                acc1 = __fmaf_rn(dev::combine24(dh[2], dh[3], dl[2], dl[3]), __ldg(srow1 + grp) * fac, acc1);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dh[i] = dl[i] = 0;
            }
        }
    }
    acc0 += __shfl_down_sync(0xffffffffu, acc0, 1);
    acc1 += __shfl_down_sync(0xffffffffu, acc1, 1);
    if (t == 0) {
        red[warp * 16 + g] = acc0;
        red[warp * 16 + g + 8] = acc1;
    }
    __syncthreads();
    if (threadIdx.x < 16) {
        const int r = threadIdx.x;
        y[16 * R + r] = (red[r] + red[16 + r]) + (red[32 + r] + red[48 + r]);
    }
}

template <int B, int GS>
static pmoe_status launch_gemv_b(const pmoe_matrix &m, const void *x, bool bf, float *y, cudaStream_t st)
{
    const size_t smem = (size_t)(m.K / 32) * dev::kFragWords * 4 + (size_t)(m.K / 128) * 4 + 256 * 4 + 64 * 4;
    if (smem > 200 * 1024)
        return PMOE_ERR_UNSUPPORTED;
    auto kern = bf ? gemv_kernel<B, GS, true> : gemv_kernel<B, GS, false>;
    if (smem > 48 * 1024)
        PMOE_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    kern<<<m.N / 16, 128, smem, st>>>(m, x, y);
    return launch_status();
}

template <int GS>
static pmoe_status launch_gemv_g(const pmoe_matrix &m, int b, const void *x, bool bf, float *y,
                                 cudaStream_t st)
{
    switch (b) {
    case 1: return launch_gemv_b<1, GS>(m, x, bf, y, st);
    case 2: return launch_gemv_b<2, GS>(m, x, bf, y, st);
    case 3: return launch_gemv_b<3, GS>(m, x, bf, y, st);
    case 4: return launch_gemv_b<4, GS>(m, x, bf, y, st);
    case 5: return launch_gemv_b<5, GS>(m, x, bf, y, st);
    case 6: return launch_gemv_b<6, GS>(m, x, bf, y, st);
    case 7: return launch_gemv_b<7, GS>(m, x, bf, y, st);
    default: return launch_gemv_b<8, GS>(m, x, bf, y, st);
    }
}

} // namespace pmoe

using namespace pmoe;

extern "C" pmoe_status pmoe_expert_gemv(const pmoe_matrix *m, int b, const void *x, int x_is_bf16,
                                        float *y, pmoe_stream stream)
{
    if (!m || !x || !y || !m->planes || !m->scales || !m->codebook)
        return PMOE_ERR_INVALID_ARG;
    if (m->N <= 0 || m->K <= 0 || m->N % 16 || m->K % 128 || b < 1 || b > 8 ||
        !(m->G == 32 || m->G == 64 || m->G == 128) ||
        m->plane_stride_words < (int64_t)m->N * m->K / 32 || m->plane_stride_words % 2 ||
        !aligned(m->planes, 8) || !aligned(x, x_is_bf16 ? 8 : 16))
        return PMOE_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    switch (m->G) {
    case 32: return launch_gemv_g<1>(*m, b, x, x_is_bf16 != 0, y, st);
    case 64: return launch_gemv_g<2>(*m, b, x, x_is_bf16 != 0, y, st);
    default: return launch_gemv_g<4>(*m, b, x, x_is_bf16 != 0, y, st);
    }
}
