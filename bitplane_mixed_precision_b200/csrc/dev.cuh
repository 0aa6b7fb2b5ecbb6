// Device core of the bitplane-prefix decode, shared by the GEMV, layer and
// extraction kernels.
//
// Decode path (per warp, per 16x128 tile of one matrix):
//  * Each lane reads two uint32 words of every plane it needs (planes 0..b-1,
//    PagedMoE transcript cue 25: a depth-b request reads exactly those planes).
//  * For each of its eight "t-words" (8 weights each) the lane ANDs every plane
//    word with a constant mask, ORs them and rotates once: nibble j of the
//    t-word then holds the weight's prefix with plane p at bit p (the b-bit
//    index, bit-reversed). The stored format places bits so that this works.
//  * A byte permute (prmt) with an 8-entry register table maps four nibbles to
//    four bytes at once. Tables hold the tree codebook's depth-b values
//    (transcript cue 21: a truncated index names its ancestor node) as 16-bit
//    fixed point split into a high and a low signed byte.
//  * The bytes are exactly the A operand fragments of mma.sync m16n8k32 (s8):
//    one MMA per k-step and byte plane multiplies 16 rows x 32 columns by the
//    activation, whose 24-bit fixed-point value is split into three bytes in
//    B columns (high, middle, low) per token (xfrag.cuh). Products are summed
//    exactly in int32 per scale group, then combined and scaled in float.
// No dequantised matrix is ever written (transcript cue 37).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace pmoe {
namespace dev {

constexpr unsigned FULL = 0xffffffffu;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t rotr(uint32_t x, int r) { return __funnelshift_r(x, x, r); }

__host__ __device__ constexpr uint32_t rotl_c(uint32_t x, int r)
{
    return r == 0 ? x : ((x << r) | (x >> (32 - r)));
}

// D += A * B, m16n8k32, signed 8-bit operands, int32 accumulators.
__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(FULL, v, o);
    return v;
}

// Exponent s such that |v| * 2^s < 2^14 for every |v| <= m (m >= 0); 0 for m == 0.
__device__ __forceinline__ int fix_exponent(float m)
{
    if (!(m > 0.0f))
        return 0;
    int e;
    frexpf(m, &e); // m = f * 2^e, f in [0.5, 1)
    return 14 - e;
}

// 16-bit fixed point split: v = 256*hi + lo, hi in [-64, 64], lo in [-128, 127].
__device__ __forceinline__ void split16(int v, int &hi, int &lo)
{
    hi = (v + 128) >> 8;
    lo = v - 256 * hi;
}

// Exponent s such that |v| * 2^s < 2^22 for every |v| <= m (m >= 0); 0 for m == 0.
__device__ __forceinline__ int fix_exponent24(float m)
{
    if (!(m > 0.0f))
        return 0;
    int e;
    frexpf(m, &e);
    return 22 - e;
}

// 24-bit fixed point split: v = 65536*hi + 256*mid + lo, hi in [-64, 64], mid and lo in
// [-128, 127] (|v| < 2^22).
__device__ __forceinline__ void split24(int v, int &hi, int &mid, int &lo)
{
    const int v1 = (v + 128) >> 8;
    lo = v - 256 * v1;
    split16(v1, hi, mid);
}

// Products of 16-bit fixed-point weights (high byte wh, low byte wl: A operands of two MMAs)
// and 24-bit fixed-point activations (high, middle, low byte in B columns 0, 1, 2; column 3
// zero). Lane t = 0 holds columns (0, 1) of both MMAs, lane t = 1 columns (2, 3): with
// dh0, dh1, dl0, dl1 the lane's int32 sums (wh by its first and second column, wl likewise),
//   F = 256 * (256*dh0 + dh1 + dl0) + dl1,
// and sum(w * x) = 2^8 * F(t = 0) + 2^-8 * F(t = 1), in units of the two fixed points. The
// integer part is exact (|256*dh0 + dh1 + dl0| < 2^28 for 128 products per group).
__device__ __forceinline__ float combine24(int dh0, int dh1, int dl0, int dl1)
{
    return __fmaf_rn((float)(dh0 * 256 + dh1 + dl0), 256.0f, (float)dl1);
}

// The lane factor of combine24's F: 2^8 for the lane holding columns 0, 1 of a token's three
// byte columns, 2^-8 for the lane holding its columns 2, 3; t = lane % 4, tokens at t/2.
__device__ __forceinline__ float combine24_lane_factor(int t) { return (t & 1) ? 0.00390625f : 256.0f; }

// Register tables of one (matrix, depth). For depth <= 3, h[0..1] / l[0..1]
// are the high / low bytes of entries 0..7 (entry v = value of the index whose
// bit-reversed b-bit form is v). For depth 4, h[0..1] hold entries 0..7 and
// h[2..3] entries 8..15. For depth >= 5 the table lives in shared memory as
// one 32-bit word per entry: byte 0 = hi, byte 1 = lo.
struct RegTab {
    uint32_t h[4];
    uint32_t l[4];
    int f; // fixed-point exponent: entry = round(C * 2^f)
};

// Builds the tables of depth b from the 510-entry codebook; one full warp.
// big (shared or global, 2^b entries of 32 or 16 bits: byte 0 = high, byte 1 =
// low) is written for b >= 5 when non-null.
template <typename BT = uint32_t>
__device__ __forceinline__ void build_tab(const float *__restrict__ cb, int b, RegTab &tab, BT *big)
{
    const int lane = threadIdx.x & 31;
    const int n = 1 << b;
    const float *C = cb + (n - 2);
    float m = 0.0f;
    for (int v = lane; v < n; v += 32)
        m = fmaxf(m, fabsf(__ldg(C + v)));
    m = warp_max(m);
    const int f = fix_exponent(m);
    uint32_t my = 0; // entry of v = lane (lanes 0..15)
    for (int v = lane; v < n; v += 32) {
        const int i = (int)(__brev((unsigned)v) >> (32 - b));
        const int vi = __float2int_rn(ldexpf(__ldg(C + i), f));
        int hi, lo;
        split16(vi, hi, lo);
        const uint32_t e = (uint32_t)(hi & 0xff) | ((uint32_t)(lo & 0xff) << 8);
        if (big != nullptr)
            big[v] = (BT)e;
        if (v == lane)
            my = e;
    }
    if (lane >= n)
        my = 0;
    // gather: word r of the hi (lo) table holds bytes of entries 4r..4r+3
    uint32_t hb = (my & 0xffu) << (8 * (lane & 3));
    uint32_t lb = ((my >> 8) & 0xffu) << (8 * (lane & 3));
    hb |= __shfl_xor_sync(FULL, hb, 1);
    lb |= __shfl_xor_sync(FULL, lb, 1);
    hb |= __shfl_xor_sync(FULL, hb, 2);
    lb |= __shfl_xor_sync(FULL, lb, 2);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        tab.h[r] = __shfl_sync(FULL, hb, 4 * r);
        tab.l[r] = __shfl_sync(FULL, lb, 4 * r);
    }
    tab.f = f;
}

// t-word q (0..7) of a lane: nibble j = prefix of weight j, plane p at bit p
// (planes 0..min(B,4)-1). w[p][h] are the lane's two words of plane p.
template <int B>
__device__ __forceinline__ uint32_t tword_lo(const uint32_t (&w)[8][2], int q)
{
    const int h = q >> 2, r = q & 3;
    uint32_t acc = 0;
#pragma unroll
    for (int p = 0; p < (B < 4 ? B : 4); ++p)
        acc |= w[p][h] & rotl_c(0x11111111u << p, r);
    return r ? rotr(acc, r) : acc;
}

// Same for planes 4..B-1 (B >= 5): plane p at nibble bit p-4.
template <int B>
__device__ __forceinline__ uint32_t tword_hi(const uint32_t (&w)[8][2], int q)
{
    const int h = q >> 2, r = q & 3;
    uint32_t acc = 0;
#pragma unroll
    for (int p = 4; p < B; ++p)
        acc |= w[p][h] & rotl_c(0x11111111u << (p - 4), r + 4);
    return rotr(acc, r + 4);
}

// A fragments (hi and lo byte planes) of k-step s (0..3) of the lane's tile.
// ah/al[0]: row g, k 4t..4t+3; [1]: row g+8, same k; [2]: row g, k 16+4t..;
// [3]: row g+8, k 16+4t.. (PTX m16n8k32 .s8 A layout).
template <int B, typename BT = uint32_t>
__device__ __forceinline__ void decode_kstep(const uint32_t (&w)[8][2], int s, const RegTab &tab,
                                             const BT *big, uint32_t (&ah)[4],
                                             uint32_t (&al)[4])
{
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int q = 2 * s + u;
        const uint32_t t = tword_lo<B>(w, q);
        if constexpr (B <= 3) {
            const uint32_t t2 = t >> 16;
            ah[u] = prmt(tab.h[0], tab.h[1], t);
            al[u] = prmt(tab.l[0], tab.l[1], t);
            ah[2 + u] = prmt(tab.h[0], tab.h[1], t2);
            al[2 + u] = prmt(tab.l[0], tab.l[1], t2);
        } else if constexpr (B == 4) {
            const uint32_t t7 = t & 0x77777777u;
            const uint32_t ms = ((t >> 1) & 0x44444444u) | 0x32103210u;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint32_t sel = hf ? (t7 >> 16) : t7;
                const uint32_t m = hf ? (ms >> 16) : ms;
                ah[2 * hf + u] = prmt(prmt(tab.h[0], tab.h[1], sel), prmt(tab.h[2], tab.h[3], sel), m);
                al[2 * hf + u] = prmt(prmt(tab.l[0], tab.l[1], sel), prmt(tab.l[2], tab.l[3], sel), m);
            }
        } else {
            const uint32_t th = tword_hi<B>(w, q);
            const uint32_t even = (t & 0x0f0f0f0fu) | ((th << 4) & 0xf0f0f0f0u);
            const uint32_t odd = ((t >> 4) & 0x0f0f0f0fu) | (th & 0xf0f0f0f0u);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint32_t e0 = (uint32_t)big[(even >> (16 * hf)) & 0xffu];
                const uint32_t e1 = (uint32_t)big[(odd >> (16 * hf)) & 0xffu];
                const uint32_t e2 = (uint32_t)big[(even >> (16 * hf + 8)) & 0xffu];
                const uint32_t e3 = (uint32_t)big[(odd >> (16 * hf + 8)) & 0xffu];
                const uint32_t x01 = prmt(e0, e1, 0x5140u);
                const uint32_t x23 = prmt(e2, e3, 0x5140u);
                ah[2 * hf + u] = prmt(x01, x23, 0x5410u);
                al[2 * hf + u] = prmt(x01, x23, 0x7632u);
            }
        }
    }
}

// Depth 1 with an antisymmetric table (C[1][0] = -C[1][1], as for the Gaussian
// tree): the value is C[1][1] * (2*bit - 1), so the A bytes are the signs +-1
// themselves and one MMA per k-step suffices (no high/low split). The plane
// word is masked to the t-word's bit of each nibble (bit r); r = 3 is moved to
// bit 2, because a selector nibble with bit 3 set asks prmt for a sign fill.
// Byte table: selector 0 -> -1, selector 1, 2 or 4 -> +1.
__device__ __forceinline__ void decode_kstep_sign(const uint32_t (&w)[8][2], int s, uint32_t (&a)[4])
{
    constexpr uint32_t kLo = 0x000101FFu, kHi = 0x00000001u;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int q = 2 * s + u, h = q >> 2, r = q & 3;
        uint32_t t = w[0][h] & (0x11111111u << r);
        if (r == 3)
            t >>= 1;
        a[u] = prmt(kLo, kHi, t);
        a[2 + u] = prmt(kLo, kHi, t >> 16);
    }
}

// Prefix index (b bits, MSB first) of every weight of the lane's tile, in the
// A-fragment order: out[q][j] for t-word q, nibble j.
template <int B>
__device__ __forceinline__ void prefix_indices(const uint32_t (&w)[8][2], uint8_t (&out)[8][8])
{
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t t = tword_lo<B>(w, q);
        uint32_t th = 0;
        if constexpr (B >= 5)
            th = tword_hi<B>(w, q);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t v = ((t >> (4 * j)) & 0xfu) | (((th >> (4 * j)) & 0xfu) << 4);
            out[q][j] = (uint8_t)(__brev(v) >> (32 - B));
        }
    }
}

// Element (row, col) inside the 16x128 tile of weight j of t-word q for lane.
__host__ __device__ __forceinline__ void tile_coord(int lane, int q, int j, int &row, int &col)
{
    const int g = lane >> 2, t = lane & 3;
    const int s = q >> 1, u = q & 1;
    row = g + 8 * u;
    col = 32 * s + 16 * (j >> 2) + 4 * t + (j & 3);
}

} // namespace dev
} // namespace pmoe
