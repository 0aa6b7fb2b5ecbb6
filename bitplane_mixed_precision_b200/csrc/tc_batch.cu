// Batched tensor-core path of the MoE layer (PagedMoE transcript cues 13, 29,
// 35; arxivlens Methodology): experts that many tokens of a batch route to are
// multiplied on the fifth-generation tensor cores (tcgen05) instead of being
// decoded again for every pair of tokens.
//
// For such an expert ("TC unit": one expert, up to 64 of its (token, slot)
// pairs, all at depth <= 4) the tree value at depth b is written as a sum of
// level deltas (children = parent + delta):
//     C_b[i] = sum_{d=1..b} Delta_d[i >> (b-d)],  Delta_1 = C_1,
//     Delta_d[j] = C_d[j] - C_{d-1}[j >> 1],
// and every level d has its own accumulator. A 128-row tile of a matrix is
// decoded once per level into f16 operands in shared memory, and one MMA per
// level multiplies it with all the unit's tokens at once. The entries of level
// 1, the largest deltas, are split into a high and a low f16 part (two MMAs):
// one f16 per entry repeats the entry's rounding error on every weight that
// uses it, and those errors add up coherently in a dot product; for levels
// 2..4 (smaller deltas) the single f16 stays inside the layer's tolerance. Accumulators hold one scale group
// (G columns of K) at a time; the epilogue applies the rows' group scales in
// fp32 and sums, per token, the first b level accumulators of its depth b.
// Tokens at different depths of one expert thus share the planes they have in
// common and all the MMA work of their common levels.
//
// Launches (after the prep kernel has formed the units):
//  * tc_xb_kernel: each unit's activations as f16 MMA operands (B), one
//    power-of-two scale per token, in the k-step layout of umma.cuh.
//  * tc_gemm_kernel<0>: gate and up rows, (unit, matrix, 128-row tile) items.
//  * tc_h_kernel: h = silu(g) * u per pair, as f16 operands like x.
//  * tc_gemm_kernel<1>: down rows, (unit, 128-row tile of H) items; each pair's
//    output rows go to the layer's per-pair rows, and the last of a token's k
//    pairs for a 128-row strip sums them into y in slot order (the same
//    protocol the persistent kernel follows for the other pairs).
//
// tc_gemm_kernel is persistent (one CTA per SM) with warp roles:
//  * warps 0-7, decoders: warp w decodes rows 16w..16w+15 of the tile, one
//    k-step (32 k) at a time, every level, into a shared-memory stage;
//  * warp 12, producer: 1-D bulk copies of each chunk of up to 512 k (the
//    tile's planes, 1 KB per plane and 16-row block, and the unit's B
//    operand) into a two-slot ring;
//  * warp 13: allocates tensor memory and issues the MMAs (one thread);
//  * warps 8-11, epilogue: after each scale group, read its accumulators
//    (tcgen05.ld), add them times the group scale into per-token fp32 sums in
//    registers; at the end of an item, unscale and store.
// The group accumulators are double-buffered in tensor memory (columns 0-255 /
// 256-511), so a group's MMAs overlap the epilogue of the one before. Every
// wait is bounded; a wait that runs out records error 3 and the CTA stops.
#include <cuda_fp16.h>

#include "common.h"
#include "dev.cuh"
#include "layer.cuh"
#include "pipe.cuh"
#include "umma.cuh"

namespace pmoe {
namespace tc {

constexpr int NDEC = 8, W_EPI = 8, NEPI = 4, W_PROD = 12, W_MMA = 13;
constexpr int NTHREADS = 14 * 32;
constexpr int TPC_MAX = 4;                                   // plane tiles (128 k each) per ring chunk
constexpr int NSLOT = 2, NST = 2;                            // ring slots, decoded stages
constexpr int PLANES_CH = NDEC * kTcMaxLevels * TPC_MAX * 256; // plane tiles of a chunk (32 KB)
constexpr int BOPS_CH = 32 * 1024;                           // B operand of a chunk (tiles x 4 k-steps x
                                                             // npad x 64 B: items of 64 columns take 2 tiles)
constexpr int SLOT_BYTES = PLANES_CH + BOPS_CH;
constexpr int LEV_BYTES = 128 * 32 * 2;                      // one level part of a decoded k-step
constexpr int LO1 = kTcMaxLevels;                            // part index of level 1's low part
constexpr int STAGE_BYTES = (kTcMaxLevels + 1) * LEV_BYTES;  // levels' high parts, level 1's low part
constexpr uint64_t kDrainNs = 200ull * 1000 * 1000;

struct Smem {
    alignas(1024) unsigned char ring[NSLOT][SLOT_BYTES];
    alignas(1024) unsigned char A[NST][STAGE_BYTES];
    alignas(16) uint32_t tab[2][kTcMaxLevels][16]; // by item parity: level d: high part (hi bytes [4],
                                                   // lo bytes [4]), then the low part likewise
    uint64_t full[NSLOT], cempty[NSLOT], afull[NST], aempty[NST];
    uint64_t gfull[2], gempty[2];     // group accumulator buffers: MMAs done / epilogue done
    uint64_t tabready[2], epidone[2]; // level tables of an item built; its down rows written (by parity)
    uint32_t tmem;
};
static_assert(sizeof(Smem) <= 227 * 1024, "shared memory of the tensor-core kernel exceeds one SM's");

struct Args {
    pmoe_layer L;
    int k;
    const float *wts; // routing weights [T*k] (the combine)
    float *y;
    LayerWs W;
    uint64_t limit_ns;
};

constexpr int kErrNoPlane = 2, kErrTimeout = 3;

__device__ __forceinline__ void set_error(const LayerWs &W, int code, int where)
{
    if (atomicCAS(&W.flags[kFlagError], 0, code) == 0)
        W.flags[kFlagWhere] = where;
}

__device__ __forceinline__ int atom_add_acq_rel(int *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// floor(log2(m)) for a finite m > 0 (normal or not), -127 for m == 0
__device__ __forceinline__ int ilog2f(float m)
{
    if (!(m > 0.0f))
        return -127;
    int e;
    frexpf(m, &e);
    return e - 1;
}

// power-of-two exponent f with max * 2^f in [2^top, 2^(top+1)) (0 for an all-zero max)
__device__ __forceinline__ int pow2_exponent(float max_abs, int top)
{
    return max_abs > 0.0f ? top - ilog2f(max_abs) : 0;
}

// exponent of a matrix's level tables: the deltas of levels 1..4 stay below 2^8 after scaling by 2^fa
// (|delta| <= 2 * max |C| over depths 1..4); every lane of a warp gets the same value
__device__ __forceinline__ int table_exponent(const float *cb)
{
    const int lane = threadIdx.x & 31;
    float m = (lane < 30) ? fabsf(__ldg(cb + lane)) : 0.0f; // depths 1..4: entries 0..29
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return pow2_exponent(m, 6);
}

// Byte tables (hi bytes [4], lo bytes [4]) of 16-bit entries e (lanes 0..15) into dst[0..7].
__device__ __forceinline__ void gather_bytes(uint32_t e, uint32_t *dst)
{
    const int lane = threadIdx.x & 31;
    uint32_t hb = ((e >> 8) & 0xffu) << (8 * (lane & 3));
    uint32_t lb = (e & 0xffu) << (8 * (lane & 3));
    hb |= __shfl_xor_sync(0xffffffffu, hb, 1);
    lb |= __shfl_xor_sync(0xffffffffu, lb, 1);
    hb |= __shfl_xor_sync(0xffffffffu, hb, 2);
    lb |= __shfl_xor_sync(0xffffffffu, lb, 2);
    uint32_t h[4], l[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        h[r] = __shfl_sync(0xffffffffu, hb, 4 * r);
        l[r] = __shfl_sync(0xffffffffu, lb, 4 * r);
    }
    if (lane < 4) {
        dst[lane] = lane == 0 ? h[0] : lane == 1 ? h[1] : lane == 2 ? h[2] : h[3];
        dst[4 + lane] = lane == 0 ? l[0] : lane == 1 ? l[1] : lane == 2 ? l[2] : l[3];
    }
}

// Level table of depth d (one warp): entry v (v < 2^d; the prefix index is v bit-reversed, as the
// t-words of the plane format hold it) of Delta_d * 2^fa as an f16 high part (dst[0..7]) and the f16
// of the remainder (dst[8..15]), each as byte tables of entries 4r..4r+3.
__device__ void build_level(const float *cb, int d, int fa, uint32_t *dst)
{
    const int lane = threadIdx.x & 31;
    const int n = 1 << d;
    uint32_t eh = 0, el = 0;
    if (lane < n) {
        const int i = (int)(__brev((unsigned)lane) >> (32 - d));
        const float c = __ldg(cb + (n - 2) + i);
        const float par = d > 1 ? __ldg(cb + (n / 2 - 2) + (i >> 1)) : 0.0f;
        const float v = ldexpf(c - par, fa);
        const __half h = __float2half_rn(v);
        eh = (uint32_t)__half_as_ushort(h);
        el = (uint32_t)__half_as_ushort(__float2half_rn(v - __half2float(h)));
    }
    gather_bytes(eh, dst);
    gather_bytes(el, dst + 8);
}

// ---------------------------------------------------------------- items

struct Item {
    int u, m, tile, e, n, npad, nlev, rowoff, K;
    int tpc; // plane tiles per ring chunk: the largest of 4, 2, 1 dividing K / 128 whose B operand fits
};

__device__ __forceinline__ bool get_item(const LayerWs &W, int mode, int idx, int H, int I, Item &o)
{
    const int nu = W.flags[kFlagTcUnits];
    const int per = mode == 0 ? 2 * (I / 128) : H / 128;
    if (idx >= nu * per)
        return false;
    o.u = idx / per;
    const int r = idx - o.u * per;
    if (mode == 0) {
        o.m = r / (I / 128);
        o.tile = r - o.m * (I / 128);
        o.K = H;
    } else {
        o.m = 2;
        o.tile = r;
        o.K = I;
    }
    const int4 ur = W.tc_unit[o.u];
    o.e = ur.x;
    o.n = ur.y;
    o.npad = ur.z & 0xffff;
    o.nlev = ur.z >> 16;
    o.rowoff = ur.w;
    const int nt = o.K / 128, cap = BOPS_CH / (4 * 64 * o.npad); // the chunk's B operand fits its region
    o.tpc = (nt % 4 == 0 && cap >= 4) ? 4 : ((nt % 2 == 0 && cap >= 2) ? 2 : 1);
    return true;
}

// ---------------------------------------------------------------- decode of one k-step

// Four weights' f16 values (two words) from byte tables t[0..7] of up to 16 entries, selector = the
// four weights' t-word nibbles.
template <bool WIDE>
__device__ __forceinline__ void lookup4(const uint32_t *t, uint32_t sel, uint32_t &v01, uint32_t &v23)
{
    uint32_t hb, lb;
    if (!WIDE) {
        hb = prmt(t[0], t[1], sel);
        lb = prmt(t[4], t[5], sel);
    } else {
        const uint32_t s7 = sel & 0x7777u;
        const uint32_t ms = ((sel >> 1) & 0x4444u) | 0x3210u;
        hb = prmt(prmt(t[0], t[1], s7), prmt(t[2], t[3], s7), ms);
        lb = prmt(prmt(t[4], t[5], s7), prmt(t[6], t[7], s7), ms);
    }
    v01 = prmt(lb, hb, 0x5140u);
    v23 = prmt(lb, hb, 0x7362u);
}

// The lane's 16 weights of k-step s (of the 16 x 128 tile whose plane words are w) at every level
// d < NL: the high and low f16 parts of Delta_d * 2^fa, stored into the stage's level blocks.
template <int NL>
__device__ __forceinline__ void decode_kstep(const uint32_t (&w)[kTcMaxLevels][2], int s,
                                             const uint32_t (&tb)[kTcMaxLevels][8], const uint32_t (&tlo)[8],
                                             unsigned char *stage, int rb, int lane)
{
    const int t = lane & 3, gq = lane >> 2;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int q = 2 * s + u, h = q >> 2, r = q & 3;
        const int row = 16 * rb + gq + 8 * u;
        uint32_t acc = 0;
#pragma unroll
        for (int d = 0; d < NL; ++d) {
            // (select, not an index: s is a run-time loop variable, and an indexed w would live in local
            // memory)
            acc |= (h ? w[d][1] : w[d][0]) & dev::rotl_c(0x11111111u << d, r);
            const uint32_t tw = r ? __funnelshift_r(acc, acc, r) : acc;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint32_t sel = hf ? (tw >> 16) : tw;
                uint32_t h01, h23;
                if (d >= 3)
                    lookup4<true>(tb[d], sel, h01, h23);
                else
                    lookup4<false>(tb[d], sel, h01, h23);
                const uint32_t off = umma::a_offset_sw32(row, 16 * hf + 4 * t);
                *reinterpret_cast<uint2 *>(stage + d * LEV_BYTES + off) = make_uint2(h01, h23);
                if (d == 0) { // the low part: level 1 only (see the header)
                    uint32_t l01, l23;
                    lookup4<false>(tlo, sel, l01, l23);
                    *reinterpret_cast<uint2 *>(stage + LO1 * LEV_BYTES + off) = make_uint2(l01, l23);
                }
            }
        }
    }
}

} // namespace tc
} // namespace pmoe

namespace pmoe {
namespace tc {

// ---------------------------------------------------------------- the MMA kernel

__device__ __forceinline__ void decode_any(int nl, const uint32_t (&w)[kTcMaxLevels][2], int s,
                                           const uint32_t (&tb)[kTcMaxLevels][8], const uint32_t (&tlo)[8],
                                           unsigned char *stage, int rb, int lane)
{
    switch (nl) {
    case 1: decode_kstep<1>(w, s, tb, tlo, stage, rb, lane); break;
    case 2: decode_kstep<2>(w, s, tb, tlo, stage, rb, lane); break;
    case 3: decode_kstep<3>(w, s, tb, tlo, stage, rb, lane); break;
    default: decode_kstep<4>(w, s, tb, tlo, stage, rb, lane); break;
    }
}

template <int MODE> // 0: gate/up, 1: down
__global__ void __launch_bounds__(NTHREADS, 1) tc_gemm_kernel(Args a)
{
    extern __shared__ __align__(1024) unsigned char smraw[];
    Smem &S = *reinterpret_cast<Smem *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const pmoe_layer &L = a.L;
    const LayerWs &W = a.W;
    const int H = L.H, I = L.I, G = L.G;
    const int KPG = G / 32; // k-steps per scale group
    const uint64_t deadline = pipe::globaltimer() + a.limit_ns;
    const int64_t mat_words = (int64_t)H * I / 32;
    const int64_t escale_len = 2 * (int64_t)I * (H / G) + (int64_t)H * (I / G);

    if (tid == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            pipe::mbar_init(&S.full[s], 1);
            pipe::mbar_init(&S.cempty[s], 1);
        }
        for (int s = 0; s < NST; ++s) {
            pipe::mbar_init(&S.afull[s], NDEC);
            pipe::mbar_init(&S.aempty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            pipe::mbar_init(&S.gfull[s], 1);
            pipe::mbar_init(&S.gempty[s], NEPI);
            pipe::mbar_init(&S.tabready[s], kTcMaxLevels);
            pipe::mbar_init(&S.epidone[s], NEPI);
        }
        pipe::fence_barrier_init();
    }
    if (warp == W_MMA) {
        umma::tmem_alloc(&S.tmem, 512);
        umma::tmem_relinquish();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = S.tmem;
    Item it;

    if (warp == W_PROD) {
        // ------------------------------------------------------------ producer
        const char *bsrc = reinterpret_cast<const char *>(MODE == 0 ? W.tc_xb : W.tc_hb);
        int gch = 0;
        bool ok = true;
        for (int idx = blockIdx.x; ok && get_item(W, MODE, idx, H, I, it); idx += gridDim.x) {
            const int K = it.K, tpc = it.tpc, nch = K / (128 * tpc);
            const uint32_t bbytes = (uint32_t)(4 * tpc * it.npad * 64), pbytes = (uint32_t)(tpc * 256);
            const char *bunit = bsrc + (int64_t)it.rowoff * K * 2;
            // lane = plane p (lane / 8) and 16-row block rb (lane % 8) of the tile
            const int p = lane >> 3, rb = lane & 7;
            const int ps = (lane < 8 * it.nlev) ? __ldg(L.slot_of + it.e * 8 + p) : -1;
            const unsigned have = __ballot_sync(0xffffffffu, ps >= 0);
            if (lane < 8 * it.nlev && ps < 0)
                set_error(W, kErrNoPlane, it.e * 8 + p);
            for (int c = 0; ok && c < nch; ++c, ++gch) {
                const int slot = gch % NSLOT;
                if (lane == 0) {
                    if (gch >= NSLOT && !pipe::mbar_wait_tight(&S.cempty[slot], ((gch - NSLOT) / NSLOT) & 1, deadline))
                        ok = false;
                    if (ok)
                        pipe::mbar_arrive_expect_tx(&S.full[slot], (uint32_t)__popc(have) * pbytes + bbytes);
                }
                ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
                if (!ok)
                    break;
                if (ps >= 0) {
                    const uint32_t *src = L.pool + (int64_t)ps * L.slot_words + it.m * mat_words +
                                          ((int64_t)(it.tile * 8 + rb) * (K / 128) + c * tpc) * 64;
                    pipe::bulk_g2s(S.ring[slot] + (p * 8 + rb) * (TPC_MAX * 256), src, pbytes, &S.full[slot]);
                }
                if (lane == 31)
                    pipe::bulk_g2s(S.ring[slot] + PLANES_CH, bunit + (int64_t)c * bbytes, bbytes, &S.full[slot]);
                __syncwarp();
            }
        }
        if (!ok && lane == 0)
            set_error(W, kErrTimeout, 20 + MODE);
        // no copy may still be landing in shared memory when the CTA exits
        if (lane == 0) {
            const uint64_t drain = pipe::globaltimer() + kDrainNs;
            for (int q = gch - NSLOT > 0 ? gch - NSLOT : 0; q < gch; ++q)
                pipe::mbar_wait(&S.full[q % NSLOT], (q / NSLOT) & 1, drain);
        }
    } else if (warp < NDEC) {
        // ------------------------------------------------------------ decoders
        const int rb = warp;
        int gch = 0, gks = 0, n_it = 0;
        bool ok = true;
        for (int idx = blockIdx.x; ok && get_item(W, MODE, idx, H, I, it); idx += gridDim.x, ++n_it) {
            const int par = n_it & 1, K = it.K, nl = it.nlev;
            const float *cb = L.codebooks + ((int64_t)it.e * 3 + it.m) * 510;
            const int fa = table_exponent(cb);
            // warps 0..3 build the item's level tables (those past its depth only arrive); every decoder
            // waits (bounded) for all four. Decoder warps are never more than two k-steps apart (the
            // decoded stages hold them together), so no warp still reads the tables of the item two back.
            if (warp < kTcMaxLevels) {
                if (warp < nl)
                    build_level(cb, warp + 1, fa, S.tab[par][warp]);
                __syncwarp();
                if (lane == 0)
                    pipe::mbar_arrive(&S.tabready[par]);
            }
            if (!pipe::mbar_wait_tight(&S.tabready[par], (n_it >> 1) & 1, deadline)) {
                ok = false;
                break;
            }
            uint32_t tb[kTcMaxLevels][8], tlo[8]; // high parts of every level; low part of level 1
#pragma unroll
            for (int d = 0; d < kTcMaxLevels; ++d)
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    tb[d][r] = S.tab[par][d][r];
#pragma unroll
            for (int r = 0; r < 8; ++r)
                tlo[r] = S.tab[par][0][8 + r];
            const int tpc = it.tpc, nch = K / (128 * tpc);
            for (int c = 0; ok && c < nch; ++c, ++gch) {
                const int slot = gch % NSLOT;
                if (!pipe::mbar_wait_tight(&S.full[slot], (gch / NSLOT) & 1, deadline)) {
                    ok = false;
                    break;
                }
#pragma unroll 1
                for (int j = 0; ok && j < tpc; ++j) {
                uint32_t w[kTcMaxLevels][2];
#pragma unroll
                for (int d = 0; d < kTcMaxLevels; ++d) {
                    w[d][0] = w[d][1] = 0u;
                    if (d < nl) {
                        const uint2 v = *reinterpret_cast<const uint2 *>(S.ring[slot] + (d * 8 + rb) * (TPC_MAX * 256) +
                                                                           j * 256 + lane * 8);
                        w[d][0] = v.x;
                        w[d][1] = v.y;
                    }
                }
#pragma unroll 1
                for (int s = 0; s < 4; ++s, ++gks) {
                    const int st = gks % NST;
                    if (gks >= NST && !pipe::mbar_wait_tight(&S.aempty[st], ((gks - NST) / NST) & 1, deadline)) {
                        ok = false;
                        break;
                    }
                    decode_any(nl, w, s, tb, tlo, S.A[st], rb, lane);
                    umma::fence_smem_async();
                    __syncwarp();
                    if (lane == 0)
                        pipe::mbar_arrive(&S.afull[st]);
                }
                }
            }
        }
        if (!ok && lane == 0)
            set_error(W, kErrTimeout, 22 + MODE);
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issue (one thread)
        int gch = 0, gks = 0, gg = 0; // chunks, k-steps, scale groups so far
        bool ok = true;
        for (int idx = blockIdx.x; ok && get_item(W, MODE, idx, H, I, it); idx += gridDim.x) {
            const int ksch = 4 * it.tpc, nch = it.K / (32 * ksch), nl = it.nlev, npad = it.npad;
            const uint32_t idesc = umma::idesc_f16(128, npad);
            int ks_item = 0;
            for (int c = 0; ok && c < nch; ++c, ++gch) {
                const int slot = gch % NSLOT;
                if (lane == 0 && !pipe::mbar_wait_tight(&S.full[slot], (gch / NSLOT) & 1, deadline))
                    ok = false;
                for (int kk = 0; ok && kk < ksch; ++kk, ++gks, ++ks_item) {
                    const int st = gks % NST;
                    const bool g_first = ks_item % KPG == 0, g_last = ks_item % KPG == KPG - 1;
                    const int buf = gg & 1;
                    // a group's buffer is free once the epilogue has read the group two back
                    if (lane == 0 && g_first && gg >= 2 && !pipe::mbar_wait_tight(&S.gempty[buf], ((gg - 2) >> 1) & 1, deadline))
                        ok = false;
                    if (lane == 0 && ok && !pipe::mbar_wait_tight(&S.afull[st], (gks / NST) & 1, deadline))
                        ok = false;
                    if (lane == 0 && ok) {
                        umma::fence_after_sync();
                        const uint32_t acc0 = tmem + (uint32_t)(buf * 256);
                        const unsigned char *bk = S.ring[slot] + PLANES_CH + kk * npad * 64;
                        for (int d = 0; d < nl; ++d)
#pragma unroll
                            for (int kh = 0; kh < 2; ++kh) {
                                const uint64_t bd = umma::smem_desc(bk + kh * 256);
                                const uint32_t dcol = acc0 + (uint32_t)(d * npad);
                                umma::mma_f16(dcol, umma::smem_desc_sw32(S.A[st] + d * LEV_BYTES + kh * 4096), bd, idesc,
                                              !(g_first && kh == 0));
                                if (d == 0)
                                    umma::mma_f16(dcol, umma::smem_desc_sw32(S.A[st] + LO1 * LEV_BYTES + kh * 4096), bd,
                                                  idesc, true);
                            }
                        umma::commit(&S.aempty[st]);
                        if (kk == ksch - 1)
                            umma::commit(&S.cempty[slot]);
                        if (g_last)
                            umma::commit(&S.gfull[buf]);
                    }
                    ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
                    if (g_last)
                        ++gg;
                }
            }
            __syncwarp();
        }
        if (!ok && lane == 0)
            set_error(W, kErrTimeout, 24 + MODE);
        // the tensor cores are done with shared memory before the CTA exits
        if (lane == 0 && gks > 0) {
            const uint64_t drain = pipe::globaltimer() + kDrainNs;
            const int q = gks - 1;
            pipe::mbar_wait(&S.aempty[q % NST], (q / NST) & 1, drain);
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 8-11: TMEM lanes 32q..)
        const int q = warp - W_EPI, row = 32 * q + lane;
        int gg = 0, n_it = 0;
        bool ok = true;
        for (int idx = blockIdx.x; ok && get_item(W, MODE, idx, H, I, it); idx += gridDim.x, ++n_it) {
            const int par = n_it & 1, K = it.K, ngr = K / G, npad = it.npad, n = it.n;
            const float *cb = L.codebooks + ((int64_t)it.e * 3 + it.m) * 510;
            const int fa = table_exponent(cb);
            const int grow = it.tile * 128 + row; // row of the matrix's output
            const float *srow = L.scales + (int64_t)it.e * escale_len +
                                (MODE == 0 ? (int64_t)it.m * I * (H / G) : 2 * (int64_t)I * (H / G)) + (int64_t)grow * ngr;
            // columns are ordered by depth, deepest first: column c takes level d + 1 iff c < nd_d (the
            // number of the unit's pairs deeper than d); held as scalars, not an array, so that they stay
            // in registers
            int nd1 = 0, nd2 = 0, nd3 = 0;
            for (int c = lane; c < n; c += 32) {
                const int dp = __ldg(W.tc_rdep + it.rowoff + c);
                nd1 += dp > 1 ? 1 : 0;
                nd2 += dp > 2 ? 1 : 0;
                nd3 += dp > 3 ? 1 : 0;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                nd1 += __shfl_xor_sync(0xffffffffu, nd1, o);
                nd2 += __shfl_xor_sync(0xffffffffu, nd2, o);
                nd3 += __shfl_xor_sync(0xffffffffu, nd3, o);
            }
            float R[kTcMaxCols];
#pragma unroll
            for (int c = 0; c < kTcMaxCols; ++c)
                R[c] = 0.0f;
            float sg_next = __ldg(srow); // the next group's scale is loaded while a group is waited for
            for (int g = 0; g < ngr; ++g, ++gg) {
                const int buf = gg & 1;
                const float sg = sg_next;
                if (g + 1 < ngr)
                    sg_next = __ldg(srow + g + 1);
                if (!pipe::mbar_wait_tight(&S.gfull[buf], (gg >> 1) & 1, deadline)) {
                    ok = false;
                    break;
                }
                umma::fence_after_sync();
                const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * 256);
#pragma unroll
                for (int cb0 = 0; cb0 < kTcMaxCols; cb0 += 16) {
                    if (cb0 < n) {
                        // the levels' 16 columns, two levels per load (levels past the unit's depth, or
                        // past a column's depth, are not added: nd_d = 0 past the unit's depth)
                        float v[2][16], sum[16];
                        umma::ld16x2(tl + (uint32_t)cb0, (uint32_t)npad, v);
#pragma unroll
                        for (int cc = 0; cc < 16; ++cc)
                            sum[cc] = v[0][cc] + (cb0 + cc < nd1 ? v[1][cc] : 0.0f);
                        if (cb0 < nd2) {
                            umma::ld16x2(tl + (uint32_t)(2 * npad + cb0), (uint32_t)npad, v);
#pragma unroll
                            for (int cc = 0; cc < 16; ++cc)
                                sum[cc] += (cb0 + cc < nd2 ? v[0][cc] : 0.0f) + (cb0 + cc < nd3 ? v[1][cc] : 0.0f);
                        }
#pragma unroll
                        for (int cc = 0; cc < 16; ++cc)
                            R[cb0 + cc] = __fmaf_rn(sum[cc], sg, R[cb0 + cc]);
                    }
                }
                umma::fence_before_sync();
                __syncwarp();
                if (lane == 0)
                    pipe::mbar_arrive(&S.gempty[buf]);
            }
            if (!ok)
                break;
            // unscale (2^fa of the tables, 2^xe of the token's operand row) and store
#pragma unroll
            for (int c = 0; c < kTcMaxCols; ++c) {
                if (c < n) {
                    const int r = it.rowoff + c;
                    const int pair = __ldg(W.tc_rpair + r);
                    const int xe = __ldg((MODE == 0 ? W.tc_rxe : W.tc_rhe) + r);
                    const float out = ldexpf(R[c], -(fa + xe));
                    if (MODE == 0)
                        __stcg(W.tc_gu + (int64_t)pair * 2 * I + it.m * I + grow, out);
                    else
                        __stcg(W.part + (int64_t)pair * H + grow, out);
                }
            }
            if (MODE == 1) {
                // the last of a token's k pairs for this 128-row strip sums them into y in slot order,
                // once all four epilogue warps have written their rows
                __syncwarp();
                if (lane == 0)
                    pipe::mbar_arrive(&S.epidone[par]);
                if (!pipe::mbar_wait_tight(&S.epidone[par], (n_it >> 1) & 1, deadline)) {
                    ok = false;
                    break;
                }
                const int k = a.k, s128 = it.tile;
                for (int col = q; col < n; col += NEPI) {
                    const int pair = __ldg(W.tc_rpair + it.rowoff + col), tok = pair / k;
                    int last = 0;
                    if (lane == 0) {
                        __threadfence();
                        last = atom_add_acq_rel(&W.ycnt[tok * (H / 128) + s128], 1) == k - 1;
                    }
                    last = __shfl_sync(0xffffffffu, last, 0);
                    if (!last)
                        continue;
                    const float *part = W.part + (int64_t)tok * k * H + 128 * s128 + lane;
                    float accy[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    for (int i0 = 0; i0 < k; ++i0) {
                        const float wt = __ldg(a.wts + tok * k + i0);
#pragma unroll
                        for (int rr = 0; rr < 4; ++rr)
                            accy[rr] = __fmaf_rn(wt, __ldcg(part + (int64_t)i0 * H + 32 * rr), accy[rr]);
                    }
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr)
                        a.y[(int64_t)tok * H + 128 * s128 + 32 * rr + lane] = accy[rr];
                }
            }
        }
        if (!ok && lane == 0)
            set_error(W, kErrTimeout, 26 + MODE);
    }
    umma::fence_before_sync();
    __syncthreads();
    if (warp == W_MMA) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- operand preparation

// One warp per operand row (a unit's token, or a padding row): the row's values times 2^f (f: the row's
// power-of-two scale, max |value| * 2^f in [2^13, 2^14)) as f16, in the k-step layout, for all K/32
// k-steps; padding rows are zero. MODE 0: x (bf16) of the pair's token; MODE 1: h = silu(g) * u.
// A lane handles 8 consecutive values at a time (two 8-byte loads of x, or four 16-byte loads of g, u).
template <int MODE>
__device__ __forceinline__ void row_values8(const uint16_t *__restrict__ x, const LayerWs &W, int pair, int k, int K,
                                            int j, float (&v)[8])
{
    if (MODE == 0) {
        const uint2 *p = reinterpret_cast<const uint2 *>(x + (int64_t)(pair / k) * K + j);
        const uint2 a = __ldg(p), b = __ldg(p + 1);
        const uint32_t w[4] = {a.x, a.y, b.x, b.y};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[2 * e] = __uint_as_float(w[e] << 16);
            v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
    } else {
        const float4 *g = reinterpret_cast<const float4 *>(W.tc_gu + (int64_t)pair * 2 * K + j);
        const float4 *u = reinterpret_cast<const float4 *>(W.tc_gu + (int64_t)pair * 2 * K + K + j);
        const float4 g0 = __ldcg(g), g1 = __ldcg(g + 1), u0 = __ldcg(u), u1 = __ldcg(u + 1);
        const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
            v[e] = gv[e] / (1.0f + expf(-gv[e])) * uv[e];
    }
}

template <int MODE>
__global__ void tc_operand_kernel(const uint16_t *__restrict__ x, int k, int K, LayerWs W)
{
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int nrows = W.flags[kFlagTcRows];
    if (gw >= nrows)
        return;
    const int pair = W.tc_rpair[gw];
    const int4 ur = W.tc_unit[W.tc_runit[gw]];
    const int npad = ur.z & 0xffff, rowoff = ur.w, r = gw - rowoff;
    unsigned char *dst = reinterpret_cast<unsigned char *>(MODE == 0 ? W.tc_xb : W.tc_hb) + (int64_t)rowoff * K * 2;
    int f = 0;
    if (pair >= 0) {
        float m = 0.0f;
        for (int j = 8 * lane; j < K; j += 256) {
            float v[8];
            row_values8<MODE>(x, W, pair, k, K, j, v);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                m = fmaxf(m, fabsf(v[e]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        f = pow2_exponent(m, 13);
    }
    // lane: 8-value group g8 of k-step ks (consecutive lanes take consecutive groups)
    for (int j = 8 * lane; j < K; j += 256) {
        const int ks = j / 32, g8 = (j % 32) / 8;
        float v[8];
        if (pair >= 0)
            row_values8<MODE>(x, W, pair, k, K, j, v);
        uint32_t wv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __half2 h2 = pair >= 0 ? __floats2half2_rn(ldexpf(v[2 * e], f), ldexpf(v[2 * e + 1], f))
                                         : __floats2half2_rn(0.0f, 0.0f);
            wv[e] = *reinterpret_cast<const uint32_t *>(&h2);
        }
        *reinterpret_cast<uint4 *>(dst + (int64_t)ks * npad * 64 + umma::kstep_offset(r, g8 * 8)) =
            make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
    if (lane == 0)
        (MODE == 0 ? W.tc_rxe : W.tc_rhe)[gw] = f;
}

// ---------------------------------------------------------------- tensor-core operand self-check

// D[128 x N] = A[128 x K] * B[N x K]^T with the operand layouts (A swizzled, B not), descriptors, MMA,
// commit and tensor-memory loads of the kernel above (one CTA, 128 threads; K <= 128 in k-steps of 32, N a multiple of 16 <= 64).
constexpr int kCheckSmem = 4 * 8192 + 4 * 64 * 64;
__global__ void __launch_bounds__(128) tc_selfcheck_kernel(const uint16_t *__restrict__ A,
                                                          const uint16_t *__restrict__ B, float *__restrict__ D,
                                                          int N, int K)
{
    extern __shared__ __align__(1024) unsigned char sck[];
    unsigned char *sa = sck, *sb = sck + 4 * 8192;
    __shared__ uint64_t done;
    __shared__ uint32_t taddr;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nks = K / 32;
    for (int i = tid; i < nks * 128 * 4; i += 128) { // (k-step, row, 8-group)
        const int ks = i / 512, r = (i / 4) % 128, g8 = i % 4;
        const uint4 v = *reinterpret_cast<const uint4 *>(A + (int64_t)r * K + ks * 32 + g8 * 8);
        *reinterpret_cast<uint4 *>(sa + ks * 8192 + umma::a_offset_sw32(r, g8 * 8)) = v;
    }
    for (int i = tid; i < nks * N * 4; i += 128) {
        const int ks = i / (N * 4), r = (i / 4) % N, g8 = i % 4;
        const uint4 v = *reinterpret_cast<const uint4 *>(B + (int64_t)r * K + ks * 32 + g8 * 8);
        *reinterpret_cast<uint4 *>(sb + ks * N * 64 + umma::kstep_offset(r, g8 * 8)) = v;
    }
    if (tid == 0) {
        pipe::mbar_init(&done, 1);
        pipe::fence_barrier_init();
    }
    if (warp == 0) {
        umma::tmem_alloc(&taddr, 64);
        umma::tmem_relinquish();
    }
    umma::fence_smem_async();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tm = taddr;
    if (tid == 0) {
        for (int ks = 0; ks < nks; ++ks)
            for (int kh = 0; kh < 2; ++kh)
                umma::mma_f16(tm, umma::smem_desc_sw32(sa + ks * 8192 + kh * 4096),
                              umma::smem_desc(sb + ks * N * 64 + kh * 256), umma::idesc_f16(128, N), ks > 0 || kh > 0);
        umma::commit(&done);
    }
    __syncwarp();
    const bool fin = pipe::mbar_wait(&done, 0, pipe::globaltimer() + 100ull * 1000 * 1000);
    umma::fence_after_sync();
    if (fin) {
        for (int c0 = 0; c0 < N; c0 += 16) {
            float v[16];
            umma::ld16(tm + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, v);
#pragma unroll
            for (int c = 0; c < 16; ++c)
                D[(int64_t)(32 * warp + lane) * N + c0 + c] = v[c];
        }
    }
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tm, 64);
    }
}

} // namespace tc

static int g_num_sms_tc[128] = {};

pmoe_status launch_tc(const pmoe_layer *L, const uint16_t *x, const float *wts, int T, int k, float *y,
                      const LayerWs &W, cudaStream_t st)
{
    const int P = T * k;
    const int max_rows = tc_max_rows(P);
    int dev = 0;
    PMOE_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 128)
        return PMOE_ERR_UNSUPPORTED;
    if (g_num_sms_tc[dev] == 0)
        PMOE_CUDA(cudaDeviceGetAttribute(&g_num_sms_tc[dev], cudaDevAttrMultiProcessorCount, dev));
    const int opw = (max_rows * 32 + 255) / 256;
    tc::tc_operand_kernel<0><<<opw, 256, 0, st>>>(x, k, L->H, W);
    PMOE_TRY(launch_status());
    const size_t smem = sizeof(tc::Smem);
    tc::Args a{*L, k, wts, y, W, wait_limit_ns()};
    PMOE_CUDA(cudaFuncSetAttribute(tc::tc_gemm_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    PMOE_CUDA(cudaFuncSetAttribute(tc::tc_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    tc::tc_gemm_kernel<0><<<g_num_sms_tc[dev], tc::NTHREADS, smem, st>>>(a);
    PMOE_TRY(launch_status());
    tc::tc_operand_kernel<1><<<opw, 256, 0, st>>>(nullptr, k, L->I, W);
    PMOE_TRY(launch_status());
    tc::tc_gemm_kernel<1><<<g_num_sms_tc[dev], tc::NTHREADS, smem, st>>>(a);
    PMOE_TRY(launch_status());
    return PMOE_OK;
}

} // namespace pmoe

extern "C" pmoe_status pmoe_tc_selfcheck(const uint16_t *A, const uint16_t *B, float *D, int N, int K,
                                         pmoe_stream stream)
{
    if (!A || !B || !D || N < 16 || N > 64 || N % 16 || K < 32 || K > 128 || K % 32 ||
        ((uintptr_t)A | (uintptr_t)B) % 16)
        return PMOE_ERR_INVALID_ARG;
    PMOE_CUDA(cudaFuncSetAttribute(pmoe::tc::tc_selfcheck_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   pmoe::tc::kCheckSmem));
    pmoe::tc::tc_selfcheck_kernel<<<1, 128, pmoe::tc::kCheckSmem, (cudaStream_t)stream>>>(A, B, D, N, K);
    return pmoe::launch_status();
}
