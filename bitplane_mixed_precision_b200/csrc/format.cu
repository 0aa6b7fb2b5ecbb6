// Format layer: tree codebook, quantiser, bitplane packing and prefix
// extraction (PagedMoE transcript cues 19-27; arxivlens Abstract).
#include <cmath>
#include <cstring>
#include <vector>

#include "common.h"
#include "dev.cuh"

namespace pmoe {

namespace {
thread_local int g_last_cuda_error = 0;
}

void set_cuda_error(cudaError_t e) { g_last_cuda_error = (int)e; }

// ---------------------------------------------------------------- Gaussian helpers

static double norm_cdf(double z) { return 0.5 * std::erfc(-z / std::sqrt(2.0)); }

static double norm_pdf(double z)
{
    if (std::isinf(z))
        return 0.0;
    return std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI);
}

// Inverse normal CDF: starting point from Abramowitz & Stegun 26.2.23 (rational
// approximation, |error| < 4.5e-4), then safeguarded Newton steps on
// Phi(z) - p (bracketed; a step leaving the bracket is replaced by bisection).
// The lower tail is solved directly and the upper tail by symmetry.
double norm_ppf(double p)
{
    if (!(p > 0.0 && p < 1.0))
        return p <= 0.0 ? -INFINITY : INFINITY;
    if (p == 0.5)
        return 0.0;
    if (p > 0.5)
        return -norm_ppf(1.0 - p);
    const double t = std::sqrt(-2.0 * std::log(p));
    double z = -(t - (2.515517 + 0.802853 * t + 0.010328 * t * t) /
                         (1.0 + 1.432788 * t + 0.189269 * t * t + 0.001308 * t * t * t));
    double lo = -40.0, hi = 0.0;
    for (int it = 0; it < 100; ++it) {
        const double F = norm_cdf(z) - p;
        if (F < 0.0)
            lo = z;
        else
            hi = z;
        const double d = norm_pdf(z);
        double zn = (d > 0.0) ? z - F / d : 0.5 * (lo + hi);
        if (!(zn > lo && zn < hi))
            zn = 0.5 * (lo + hi);
        if (zn == z)
            break;
        if (std::fabs(zn - z) <= 1e-17 * std::fabs(z)) {
            z = zn;
            break;
        }
        z = zn;
    }
    return z;
}

void tree_codebook(float *cb)
{
    for (int d = 1; d <= 8; ++d) {
        const int n = 1 << d;
        for (int i = 0; i < n; ++i) {
            const double a = (i == 0) ? -INFINITY : norm_ppf((double)i / n);
            const double b = (i == n - 1) ? INFINITY : norm_ppf((double)(i + 1) / n);
            cb[n - 2 + i] = (float)((double)n * (norm_pdf(a) - norm_pdf(b)));
        }
    }
}

void quantile_thresholds(double *t)
{
    t[0] = -INFINITY;
    for (int i = 1; i < 256; ++i)
        t[i] = norm_ppf((double)i / 256.0);
}

// ---------------------------------------------------------------- quantiser

__constant__ double c_thresholds[256];

// One thread per (row, group): sequential double sums, as the definition reads.
__global__ void quantize_kernel(const float *__restrict__ w, int N, int K, int G,
                                float *__restrict__ scales, uint8_t *__restrict__ codes)
{
    const int ng = K / G;
    const int64_t total = (int64_t)N * ng;
    for (int64_t gi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; gi < total;
         gi += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = gi / ng, g = gi % ng;
        const float *src = w + n * K + g * G;
        double mean = 0.0;
        for (int k = 0; k < G; ++k)
            mean = __dadd_rn(mean, (double)src[k]);
        mean = __ddiv_rn(mean, (double)G);
        double var = 0.0;
        for (int k = 0; k < G; ++k) {
            const double d = __dadd_rn((double)src[k], -mean);
            var = __dadd_rn(var, __dmul_rn(d, d));
        }
        var = __ddiv_rn(var, (double)G);
        float s = __double2float_rn(__dsqrt_rn(var));
        if (s == 0.0f)
            s = 1.0f;
        scales[gi] = s;
        const double sd = (double)s;
        uint8_t *dst = codes + n * K + g * G;
        for (int k = 0; k < G; ++k) {
            const double z = __ddiv_rn((double)src[k], sd);
            int lo = 0, hi = 256; // largest i with t_i <= z, t_0 = -inf
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (c_thresholds[mid] <= z)
                    lo = mid;
                else
                    hi = mid;
            }
            dst[k] = (uint8_t)lo;
        }
    }
}

// ---------------------------------------------------------------- packing

// One CTA per 16x128 tile; one warp ballot per output word.
__global__ void pack_kernel(const uint8_t *__restrict__ codes, int N, int K, int depth,
                            uint32_t *__restrict__ planes, int64_t stride)
{
    __shared__ uint8_t tile[16][128];
    const int ktiles = K / 128;
    const int64_t ntiles = (int64_t)(N / 16) * ktiles;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    for (int64_t tix = blockIdx.x; tix < ntiles; tix += gridDim.x) {
        const int R = (int)(tix / ktiles), Q = (int)(tix % ktiles);
        __syncthreads();
        for (int i = threadIdx.x; i < 16 * 32; i += blockDim.x) {
            const int row = i >> 5, c4 = i & 31;
            const uint32_t v =
                *reinterpret_cast<const uint32_t *>(codes + (int64_t)(16 * R + row) * K + 128 * Q + 4 * c4);
            *reinterpret_cast<uint32_t *>(&tile[row][4 * c4]) = v;
        }
        __syncthreads();
        for (int item = warp; item < depth * 64; item += nwarps) {
            const int p = item / 64, wd = item % 64;
            const int L = wd >> 1, h = wd & 1;
            const int pos = (lane - p) & 31; // = 4j + r
            const int j = pos >> 2, r = pos & 3;
            int row, col;
            dev::tile_coord(L, 4 * h + r, j, row, col);
            const int bit = (tile[row][col] >> (7 - p)) & 1;
            const uint32_t word = __ballot_sync(dev::FULL, bit);
            if (lane == 0)
                planes[p * stride + tix * 64 + wd] = word;
        }
    }
}

static void pack_host(const uint8_t *codes, int N, int K, int depth, uint32_t *planes, int64_t stride)
{
    const int ktiles = K / 128;
    const int64_t words = (int64_t)N * K / 32;
    for (int p = 0; p < depth; ++p)
        std::memset(planes + p * stride, 0, sizeof(uint32_t) * (size_t)words);
    for (int R = 0; R < N / 16; ++R)
        for (int Q = 0; Q < ktiles; ++Q) {
            const int64_t tix = (int64_t)R * ktiles + Q;
            for (int L = 0; L < 32; ++L)
                for (int q = 0; q < 8; ++q)
                    for (int j = 0; j < 8; ++j) {
                        int row, col;
                        dev::tile_coord(L, q, j, row, col);
                        const int c = codes[(int64_t)(16 * R + row) * K + 128 * Q + col];
                        const int h = q >> 2, r = q & 3;
                        for (int p = 0; p < depth; ++p) {
                            const int bit = (4 * j + p + r) & 31;
                            if ((c >> (7 - p)) & 1)
                                planes[p * stride + tix * 64 + 2 * L + h] |= 1u << bit;
                        }
                    }
        }
}

// ---------------------------------------------------------------- prefix extraction

template <int B>
__global__ void extract_kernel(const uint32_t *__restrict__ planes, int64_t stride, int N, int K,
                               uint8_t *__restrict__ idx)
{
    const int ktiles = K / 128;
    const int64_t ntiles = (int64_t)(N / 16) * ktiles;
    const int lane = threadIdx.x & 31;
    const int64_t gw = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t tix = gw; tix < ntiles; tix += nw) {
        uint32_t w[8][2];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            w[p][0] = w[p][1] = 0;
            if (p < B) {
                const uint2 v = *reinterpret_cast<const uint2 *>(planes + p * stride + tix * 64 + 2 * lane);
                w[p][0] = v.x;
                w[p][1] = v.y;
            }
        }
        uint8_t out[8][8];
        dev::prefix_indices<B>(w, out);
        const int R = (int)(tix / ktiles), Q = (int)(tix % ktiles);
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                int row, col;
                dev::tile_coord(lane, q, j, row, col);
                idx[(int64_t)(16 * R + row) * K + 128 * Q + col] = out[q][j];
            }
    }
}

} // namespace pmoe

using namespace pmoe;

extern "C" {

const char *pmoe_status_string(pmoe_status s)
{
    switch (s) {
    case PMOE_OK: return "ok";
    case PMOE_ERR_INVALID_ARG: return "invalid argument";
    case PMOE_ERR_CUDA: return "CUDA error";
    case PMOE_ERR_OUT_OF_SLOTS: return "prefix cache out of slots";
    case PMOE_ERR_BUDGET: return "infeasible bit budget";
    case PMOE_ERR_WORKSPACE: return "workspace too small";
    case PMOE_ERR_TIMEOUT: return "bounded device wait ran out";
    case PMOE_ERR_UNSUPPORTED: return "unsupported shape or option";
    }
    return "unknown status";
}

int pmoe_last_cuda_error(void) { return g_last_cuda_error; }

int pmoe_version(void) { return 1; }

pmoe_status pmoe_tree_codebook(float *codebook)
{
    if (codebook == nullptr)
        return PMOE_ERR_INVALID_ARG;
    tree_codebook(codebook);
    return PMOE_OK;
}

pmoe_status pmoe_tree_codebook_from_leaves(const float *leaves, const float *freq, float *codebook)
{
    if (!leaves || !freq || !codebook)
        return PMOE_ERR_INVALID_ARG;
    for (int i = 0; i < 256; ++i) {
        if (!(freq[i] >= 0.0f) || !std::isfinite(freq[i]) || !std::isfinite(leaves[i]))
            return PMOE_ERR_INVALID_ARG;
        if (i > 0 && leaves[i] < leaves[i - 1])
            return PMOE_ERR_INVALID_ARG;
    }
    // node values and masses of the level below, in double; depth 8 = the leaves
    double val[256], mass[256];
    for (int i = 0; i < 256; ++i) {
        val[i] = (double)leaves[i];
        mass[i] = (double)freq[i];
        codebook[254 + i] = leaves[i];
    }
    for (int d = 7; d >= 1; --d) {
        const int n = 1 << d;
        for (int i = 0; i < n; ++i) {
            const double m0 = mass[2 * i], m1 = mass[2 * i + 1];
            const double v = (m0 + m1 > 0.0) ? (m0 * val[2 * i] + m1 * val[2 * i + 1]) / (m0 + m1)
                                             : 0.5 * (val[2 * i] + val[2 * i + 1]);
            val[i] = v;
            mass[i] = m0 + m1;
            codebook[n - 2 + i] = (float)v;
        }
    }
    return PMOE_OK;
}

pmoe_status pmoe_quantize(const float *w, int N, int K, int G, float *scales, uint8_t *codes,
                          pmoe_stream stream)
{
    if (!w || !scales || !codes || N <= 0 || K <= 0 || G <= 0 || K % G)
        return PMOE_ERR_INVALID_ARG;
    // thresholds are a constant of the format; uploaded once per device
    static bool ready[128] = {};
    int devno = 0;
    PMOE_CUDA(cudaGetDevice(&devno));
    if (devno < 0 || devno >= 128)
        return PMOE_ERR_UNSUPPORTED;
    if (!ready[devno]) {
        double t[256];
        quantile_thresholds(t);
        PMOE_CUDA(cudaMemcpyToSymbol(c_thresholds, t, sizeof(t)));
        ready[devno] = true;
    }
    const int64_t groups = (int64_t)N * (K / G);
    int64_t blocks = (groups + 127) / 128;
    if (blocks > kNumSMs * 32)
        blocks = kNumSMs * 32;
    quantize_kernel<<<(unsigned)blocks, 128, 0, (cudaStream_t)stream>>>(w, N, K, G, scales, codes);
    return launch_status();
}

pmoe_status pmoe_pack_bitplanes(const uint8_t *codes, int N, int K, int depth, uint32_t *planes,
                                int64_t plane_stride_words, int on_device, pmoe_stream stream)
{
    if (!codes || !planes || N <= 0 || K <= 0 || N % 16 || K % 128 || depth < 1 || depth > 8 ||
        plane_stride_words < (int64_t)N * K / 32)
        return PMOE_ERR_INVALID_ARG;
    if (!on_device) {
        pack_host(codes, N, K, depth, planes, plane_stride_words);
        return PMOE_OK;
    }
    if (!aligned(codes, 4))
        return PMOE_ERR_INVALID_ARG;
    const int64_t tiles = (int64_t)(N / 16) * (K / 128);
    const int64_t blocks = tiles < kNumSMs * 16 ? tiles : kNumSMs * 16;
    pack_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(codes, N, K, depth, planes,
                                                                     plane_stride_words);
    return launch_status();
}

pmoe_status pmoe_extract_prefix(const uint32_t *planes, int64_t plane_stride_words, int N, int K,
                                int b, uint8_t *idx, pmoe_stream stream)
{
    if (!planes || !idx || N <= 0 || K <= 0 || N % 16 || K % 128 || b < 1 || b > 8 ||
        plane_stride_words < (int64_t)N * K / 32 || !aligned(planes, 8) || plane_stride_words % 2)
        return PMOE_ERR_INVALID_ARG;
    const int64_t tiles = (int64_t)(N / 16) * (K / 128);
    int64_t blocks = (tiles + 3) / 4;
    if (blocks > kNumSMs * 8)
        blocks = kNumSMs * 8;
    cudaStream_t st = (cudaStream_t)stream;
    switch (b) {
    case 1: extract_kernel<1><<<(unsigned)blocks, 128, 0, st>>>(planes, plane_stride_words, N, K, idx); break;
    case 2: extract_kernel<2><<<(unsigned)blocks, 128, 0, st>>>(planes, plane_stride_words, N, K, idx); break;
    case 3: extract_kernel<3><<<(unsigned)blocks, 128, 0, st>>>(planes, plane_stride_words, N, K, idx); break;
    case 4: extract_kernel<4><<<(unsigned)blocks, 128, 0, st>>>(planes, plane_stride_words, N, K, idx); break;
    case 5: extract_kernel<5><<<(unsigned)blocks, 128, 0, st>>>(planes, plane_stride_words, N, K, idx); break;
    case 6: extract_kernel<6><<<(unsigned)blocks, 128, 0, st>>>(planes, plane_stride_words, N, K, idx); break;
    case 7: extract_kernel<7><<<(unsigned)blocks, 128, 0, st>>>(planes, plane_stride_words, N, K, idx); break;
    default: extract_kernel<8><<<(unsigned)blocks, 128, 0, st>>>(planes, plane_stride_words, N, K, idx); break;
    }
    return launch_status();
}

} // extern "C"
