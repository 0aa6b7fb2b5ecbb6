// Activation operand of the prefix MMAs: 16-bit fixed point per 128-column
// tile (power-of-two scale from the tile's max |x|), split into a high and a
// low signed byte and laid out as m16n8k32 B fragments.
//
// Fragment storage per vector: [K/32 k-steps][8][2] uint32. Entry (ks, 4*part
// + t, reg) holds 4 bytes of part (0 = high, 1 = low) for columns
// 32*ks + 16*reg + 4*t .. +3. In an MMA whose B column n = 2*c + part belongs
// to member c of a column block, lane (g = n, t) loads entry (ks, 4*(g&1)+t).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dev.cuh"

namespace pmoe {
namespace dev {

__device__ __forceinline__ void load4(const void *x, int64_t off, bool bf16, float (&v)[4])
{
    if (bf16) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(x) + off));
        v[0] = __uint_as_float(raw.x << 16);
        v[1] = __uint_as_float(raw.x & 0xffff0000u);
        v[2] = __uint_as_float(raw.y << 16);
        v[3] = __uint_as_float(raw.y & 0xffff0000u);
    } else {
        const float4 f = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(x) + off));
        v[0] = f.x;
        v[1] = f.y;
        v[2] = f.z;
        v[3] = f.w;
    }
}

// One warp converts 128-column tile Q of x (float or bf16) into fragments
// xf[(Q*4 + s)*16 ...] and the tile's exponent xe[Q].
template <bool XBF16>
__device__ __forceinline__ void make_xfrag_tile(const void *x, int Q, uint32_t *xf, int *xe)
{
    const int lane = threadIdx.x & 31;
    float v[4];
    load4(x, (int64_t)128 * Q + 4 * lane, XBF16, v);
    float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    m = warp_max(m);
    const int sx = fix_exponent(m);
    uint32_t ph = 0u, pl = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int hi, lo;
        split16(__float2int_rn(ldexpf(v[i], sx)), hi, lo);
        ph |= (uint32_t)(hi & 0xff) << (8 * i);
        pl |= (uint32_t)(lo & 0xff) << (8 * i);
    }
    const int s = lane >> 3, o = lane & 7, t = o & 3, reg = o >> 2;
    xf[((Q * 4 + s) * 8 + t) * 2 + reg] = ph;
    xf[((Q * 4 + s) * 8 + 4 + t) * 2 + reg] = pl;
    if (lane == 0)
        xe[Q] = sx;
}

} // namespace dev
} // namespace pmoe
