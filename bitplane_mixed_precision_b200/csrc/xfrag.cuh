// Activation operand of the prefix MMAs: 24-bit fixed point per 128-column tile
// (power-of-two scale from the tile's max |x|), split into a high, a middle and
// a low signed byte, laid out as m16n8k32 B fragments. Twenty-four bits keep a
// tile's small values exact to about 2^-22 of its largest one, so an outlier
// channel 1000 times the rest still leaves its neighbours 12 significant bits.
//
// Fragment storage per vector: [K/32 k-steps][3 parts][4][2] uint32 (24 words
// per k-step). Entry (ks, part, t, reg) holds 4 bytes of part (0 high, 1 middle,
// 2 low) for columns 32*ks + 16*reg + 4*t .. +3. In an MMA whose B column
// n = 4*c + part belongs to token c of a column block (part 3: zero), lane
// (g = n, t) loads the two words of entry (ks, part, t).
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


// The lane's 4 values (columns 4*lane .. +3 of a 128-column tile) at fixed-point exponent
// sx, as the three byte-part words of its fragment entry (parts 0, 1, 2).
__device__ __forceinline__ void frag_words(const float (&v)[4], int sx, uint32_t (&out)[3])
{
    uint32_t ph = 0u, pm = 0u, pl = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int hi, mid, lo;
        split24(__float2int_rn(ldexpf(v[i], sx)), hi, mid, lo);
        ph |= (uint32_t)(hi & 0xff) << (8 * i);
        pm |= (uint32_t)(mid & 0xff) << (8 * i);
        pl |= (uint32_t)(lo & 0xff) << (8 * i);
    }
    out[0] = ph;
    out[1] = pm;
    out[2] = pl;
}

// Word of the lane's part-0 entry within a tile's fragments (parts 1, 2 follow at +8, +16).
__device__ __forceinline__ int frag_lane_word(int lane)
{
    const int s = lane >> 3, o = lane & 7, t = o & 3, reg = o >> 2;
    return s * 24 + t * 2 + reg;
}

// Stores the lane's fragment words of a tile to xt (4 k-steps of 24 words).
__device__ __forceinline__ void frags_from_values(const float (&v)[4], int sx, uint32_t *xt)
{
    uint32_t w[3];
    frag_words(v, sx, w);
    uint32_t *d = xt + frag_lane_word(threadIdx.x & 31);
    d[0] = w[0];
    d[8] = w[1];
    d[16] = w[2];
}

constexpr int kFragWords = 24; // words of one k-step of a vector's fragments

// Word offset of lane (part, t)'s fragment within a k-step.
__host__ __device__ __forceinline__ int frag_offset(int part, int t) { return (part * 4 + t) * 2; }

// One warp converts 128-column tile Q of x (float or bf16) into fragments
// xf[(Q*4 + s)*24 ...] and the tile's exponent xe[Q].
template <bool XBF16>
__device__ __forceinline__ void make_xfrag_tile(const void *x, int Q, uint32_t *xf, int *xe)
{
    const int lane = threadIdx.x & 31;
    float v[4];
    load4(x, (int64_t)128 * Q + 4 * lane, XBF16, v);
    float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    m = warp_max(m);
    const int sx = fix_exponent24(m);
    frags_from_values(v, sx, xf + Q * 4 * kFragWords);
    if (lane == 0)
        xe[Q] = sx;
}

} // namespace dev
} // namespace pmoe
