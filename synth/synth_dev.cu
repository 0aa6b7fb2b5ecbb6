// Seeded, counter-based generator of synthetic inputs (device side).
//
// Second implementation of the generator in synth.c, for filling large
// weight pools directly in HBM. It draws numbers only; it holds no
// arithmetic of the method. Every floating-point step uses an explicitly
// rounded intrinsic (__dmul_rn, __dadd_rn, __ddiv_rn, __dsqrt_rn) in the
// same order as the host code, so no multiply-add is fused and the two
// sides agree bit for bit.
//
// Published definitions: SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) and
// the Marsaglia polar method (Marsaglia & Bray 1964); the natural log is
// the atanh series after frexp reduction, as on the host.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t fin(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t host_fin(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t ctr)
{
    return fin(key + (ctr + 1ULL) * 0x9E3779B97F4A7C15ULL);
}

__device__ __forceinline__ double sym_unit(uint64_t u)
{
    int64_t v = (int64_t)(u >> 11) - (int64_t)4503599627370496LL;
    return __dmul_rn(__dadd_rn((double)v, 0.5), 1.0 / 4503599627370496.0);
}

__device__ double dev_log(double s)
{
    int e;
    double m = frexp(s, &e);
    if (m < 0.70710678118654752440) {
        m = __dmul_rn(m, 2.0);
        e -= 1;
    }
    double f = __ddiv_rn(__dadd_rn(m, -1.0), __dadd_rn(m, 1.0));
    double f2 = __dmul_rn(f, f);
    double p = __ddiv_rn(1.0, 25.0);
    for (int i = 11; i >= 0; --i)
        p = __dadd_rn(__dmul_rn(p, f2), __ddiv_rn(1.0, (double)(2 * i + 1)));
    return __dadd_rn(__dmul_rn((double)e, 0.69314718055994530942), __dmul_rn(__dmul_rn(2.0, f), p));
}

// Fills out[i] = (float)(scale * z(start + i)) for i < n; one thread per pair.
__global__ void normal_f32_kernel(uint64_t key, uint64_t start, int64_t n, double scale, float *out)
{
    const uint64_t first_pair = start >> 1;
    const uint64_t last_pair = (start + (uint64_t)n - 1ULL) >> 1;
    const uint64_t npairs = last_pair - first_pair + 1ULL;
    for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < npairs;
         j += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t pair = first_pair + j;
        double zu = 0.0, zv = 0.0;
        for (int a = 0; a < 32; ++a) {
            double u = sym_unit(draw(key, pair * 64ULL + 2ULL * (uint64_t)a));
            double v = sym_unit(draw(key, pair * 64ULL + 2ULL * (uint64_t)a + 1ULL));
            double s = __dadd_rn(__dmul_rn(u, u), __dmul_rn(v, v));
            if (s >= 1.0 || s == 0.0)
                continue;
            double t = __ddiv_rn(__dmul_rn(-2.0, dev_log(s)), s);
            double r = __dsqrt_rn(t);
            zu = __dmul_rn(u, r);
            zv = __dmul_rn(v, r);
            break;
        }
        const uint64_t i0 = pair * 2ULL, i1 = i0 + 1ULL;
        if (i0 >= start && i0 < start + (uint64_t)n)
            out[i0 - start] = __double2float_rn(__dmul_rn(scale, zu));
        if (i1 >= start && i1 < start + (uint64_t)n)
            out[i1 - start] = __double2float_rn(__dmul_rn(scale, zv));
    }
}

} // namespace

extern "C" int syn_dev_normal_f32(uint64_t seed, uint64_t stream, uint64_t start, int64_t n,
                                  double scale, float *out, void *cuda_stream)
{
    if (n <= 0)
        return n == 0 ? 0 : 1;
    if (out == nullptr)
        return 1;
    const uint64_t key = host_fin(seed ^ host_fin(stream ^ 0xD1B54A32D192ED03ULL));
    const int64_t npairs = ((int64_t)((start + (uint64_t)n - 1ULL) >> 1)) - (int64_t)(start >> 1) + 1;
    int64_t blocks = (npairs + 255) / 256;
    if (blocks > 148 * 64)
        blocks = 148 * 64;
    normal_f32_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)cuda_stream>>>(key, start, n, scale, out);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
