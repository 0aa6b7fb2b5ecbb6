// MoE layer on bitplane prefixes: (token, expert) pairs grouped by expert,
// gate/up prefix GEMV + SwiGLU, down prefix GEMV, routing-weighted combine
// (PagedMoE transcript cues 4 and 37; arxivlens Abstract and Methodology).
//
// Pairs of one expert are sorted by depth (deepest first) and cut into
// column blocks of up to 4 pairs with equal depth; a CTA works on one expert
// ("unit": up to 8 blocks) and one 16-row strip. Every plane word of the strip
// is read once per unit and decoded for each block at the block's depth, so
// tokens at different depths share the planes they have in common.
#include <cuda_bf16.h>

#include "common.h"
#include "dev.cuh"
#include "layer.cuh"
#include "route.cuh"
#include "xfrag.cuh"

namespace pmoe {

using dev::RegTab;

static inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

LayerWs carve_layer_ws(void *ws, int T, int k, int H, int I, size_t *bytes)
{
    const size_t P = (size_t)T * k;
    size_t off = 0;
    auto take = [&](size_t n) {
        size_t o = off;
        off = al256(off + n);
        return o;
    };
    const size_t o_flags = take(64 * 4);
    const size_t o_bd = take(P * 4), o_bn = take(P * 4), o_bp = take(P * 16), o_be = take(P * 4);
    const size_t o_ue = take(P * 4), o_u0 = take(P * 4), o_un = take(P * 4), o_ub = take(P * 4);
    const size_t o_tab = take(P * 3 * kTabWords * 4);
    const size_t o_xf = take((size_t)T * (H / 32) * 16 * 4), o_xe = take((size_t)T * (H / 128) * 4);
    const size_t o_h = take(P * I * 4);
    const size_t o_hf = take(P * (I / 32) * 16 * 4), o_he = take(P * (I / 128) * 4);
    const size_t o_part = take(P * H * 4);
    const size_t o_ids = take(P * 4), o_w = take(P * 4), o_dep = take(P);
    if (bytes)
        *bytes = off;
    LayerWs L{};
    if (!ws)
        return L;
    char *b = static_cast<char *>(ws);
    L.flags = reinterpret_cast<int *>(b + o_flags);
    L.blk_depth = reinterpret_cast<int *>(b + o_bd);
    L.blk_nmem = reinterpret_cast<int *>(b + o_bn);
    L.blk_pair = reinterpret_cast<int *>(b + o_bp);
    L.blk_expert = reinterpret_cast<int *>(b + o_be);
    L.unit_expert = reinterpret_cast<int *>(b + o_ue);
    L.unit_blk0 = reinterpret_cast<int *>(b + o_u0);
    L.unit_nblk = reinterpret_cast<int *>(b + o_un);
    L.unit_bmax = reinterpret_cast<int *>(b + o_ub);
    L.tabs = reinterpret_cast<uint32_t *>(b + o_tab);
    L.xfrag = reinterpret_cast<uint32_t *>(b + o_xf);
    L.xexp = reinterpret_cast<int *>(b + o_xe);
    L.h = reinterpret_cast<float *>(b + o_h);
    L.hfrag = reinterpret_cast<uint32_t *>(b + o_hf);
    L.hexp = reinterpret_cast<int *>(b + o_he);
    L.part = reinterpret_cast<float *>(b + o_part);
    L.ids = reinterpret_cast<int32_t *>(b + o_ids);
    L.w = reinterpret_cast<float *>(b + o_w);
    L.depth = reinterpret_cast<uint8_t *>(b + o_dep);
    return L;
}

// ---------------------------------------------------------------- grouping (1 CTA)

__global__ void group_kernel(const int32_t *__restrict__ ids, const uint8_t *__restrict__ depth, int P,
                             int E, LayerWs W)
{
    extern __shared__ int sorted[];
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        const int e = ids[p], d = depth[p];
        int rank = 0;
        for (int q = 0; q < P; ++q) {
            const int eq = ids[q], dq = depth[q];
            rank += (eq < e || (eq == e && (dq > d || (dq == d && q < p)))) ? 1 : 0;
        }
        sorted[rank] = p;
    }
    __syncthreads();
    if (threadIdx.x != 0)
        return;
    int nb = 0, nu = 0, prev_e = -1, prev_d = -1, cur_nmem = 0, cur_unit_blocks = 0, bad = 0;
    for (int r = 0; r < P; ++r) {
        const int p = sorted[r];
        const int e = ids[p], d = depth[p];
        if (e < 0 || e >= E || d < 1 || d > 8) {
            bad = 1;
            continue;
        }
        const bool new_group = (e != prev_e);
        if (new_group || d != prev_d || cur_nmem == 4) {
            if (new_group || cur_unit_blocks == 8) {
                W.unit_expert[nu] = e;
                W.unit_blk0[nu] = nb;
                W.unit_bmax[nu] = d;
                W.unit_nblk[nu] = 0;
                ++nu;
                cur_unit_blocks = 0;
            }
            W.blk_depth[nb] = d;
            W.blk_expert[nb] = e;
            W.blk_nmem[nb] = 0;
            W.unit_nblk[nu - 1] = ++cur_unit_blocks;
            ++nb;
            cur_nmem = 0;
        }
        W.blk_pair[(nb - 1) * 4 + cur_nmem] = p;
        W.blk_nmem[nb - 1] = ++cur_nmem;
        prev_e = e;
        prev_d = d;
    }
    W.flags[kFlagBlocks] = nb;
    W.flags[kFlagUnits] = nu;
    if (bad)
        W.flags[kFlagError] = 1;
}

// ---------------------------------------------------------------- fragments and tables

__global__ void prep_kernel(const uint16_t *__restrict__ x, int T, int H, pmoe_layer L, LayerWs W)
{
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int xt = T * (H / 128);
    if (gw < xt) {
        const int t = gw / (H / 128), Q = gw % (H / 128);
        dev::make_xfrag_tile<true>(x + (int64_t)t * H, Q, W.xfrag + (int64_t)t * (H / 32) * 16,
                                   W.xexp + (int64_t)t * (H / 128));
        return;
    }
    const int j = gw - xt;
    const int blk = j / 3, m = j % 3;
    if (blk >= W.flags[kFlagBlocks])
        return;
    const int e = W.blk_expert[blk], d = W.blk_depth[blk];
    uint32_t *dst = W.tabs + ((int64_t)blk * 3 + m) * kTabWords;
    RegTab tab;
    dev::build_tab(L.codebooks + ((int64_t)e * 3 + m) * 510, d, tab, d >= 5 ? dst + 16 : nullptr);
    const int lane = threadIdx.x & 31;
    if (lane < 4) {
        dst[lane] = tab.h[lane];
        dst[4 + lane] = tab.l[lane];
    }
    if (lane == 0)
        dst[8] = (uint32_t)tab.f;
}

// h (float, per pair) -> fragments for the down projection; one warp per tile.
__global__ void hprep_kernel(int P, int I, LayerWs W)
{
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (gw >= P * (I / 128))
        return;
    const int p = gw / (I / 128), Q = gw % (I / 128);
    dev::make_xfrag_tile<false>(W.h + (int64_t)p * I, Q, W.hfrag + (int64_t)p * (I / 32) * 16,
                                W.hexp + (int64_t)p * (I / 128));
}

// ---------------------------------------------------------------- prefix MMA on one tile

__device__ __forceinline__ void load_tab(const uint32_t *src, RegTab &t)
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        t.h[i] = src[i];
        t.l[i] = src[4 + i];
    }
    t.f = (int)src[8];
}

// One 16x128 tile of one matrix for one column block: decode at depth B, MMA
// with the block's fragments, epilogue per scale group into acc (shared).
//  frow[c]: fragment base of member c (nullptr if absent); fexp[c]: exponents.
template <int B, int GS>
__device__ __forceinline__ void tile_block(const uint32_t (&w)[8][2], const uint32_t *tabsrc, int Q,
                                           const uint32_t *frow_lane, const int *fexp_t,
                                           const float *srow0, const float *srow1, float *acc0,
                                           float *acc1)
{
    RegTab tab;
    load_tab(tabsrc, tab);
    const uint32_t *big = tabsrc + 16;
    int dh[4] = {0, 0, 0, 0}, dl[4] = {0, 0, 0, 0};
    float fac = 0.0f;
    if (fexp_t != nullptr)
        fac = ldexpf(1.0f, -(tab.f + fexp_t[Q]));
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t ah[4], al[4];
        dev::decode_kstep<B>(w, s, tab, big, ah, al);
        uint32_t b0 = 0u, b1 = 0u;
        if (frow_lane != nullptr) {
            const uint2 v = *reinterpret_cast<const uint2 *>(frow_lane + (Q * 4 + s) * 16);
            b0 = v.x;
            b1 = v.y;
        }
        dev::mma_s8(dh, ah, b0, b1);
        dev::mma_s8(dl, al, b0, b1);
        if ((s + 1) % GS == 0) {
            if (fexp_t != nullptr) {
                const int grp = (128 * Q + 32 * s) / (32 * GS);
                *acc0 += dev::combine(dh[0], dh[1], dl[0], dl[1]) * (__ldg(srow0 + grp) * fac);
                *acc1 += dev::combine(dh[2], dh[3], dl[2], dl[3]) * (__ldg(srow1 + grp) * fac);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dh[i] = dl[i] = 0;
        }
    }
}

template <int GS>
__device__ __forceinline__ void tile_block_any(int d, const uint32_t (&w)[8][2], const uint32_t *tabsrc,
                                               int Q, const uint32_t *frow_lane, const int *fexp_t,
                                               const float *srow0, const float *srow1, float *acc0,
                                               float *acc1)
{
    switch (d) {
    case 1: tile_block<1, GS>(w, tabsrc, Q, frow_lane, fexp_t, srow0, srow1, acc0, acc1); break;
    case 2: tile_block<2, GS>(w, tabsrc, Q, frow_lane, fexp_t, srow0, srow1, acc0, acc1); break;
    case 3: tile_block<3, GS>(w, tabsrc, Q, frow_lane, fexp_t, srow0, srow1, acc0, acc1); break;
    case 4: tile_block<4, GS>(w, tabsrc, Q, frow_lane, fexp_t, srow0, srow1, acc0, acc1); break;
    case 5: tile_block<5, GS>(w, tabsrc, Q, frow_lane, fexp_t, srow0, srow1, acc0, acc1); break;
    case 6: tile_block<6, GS>(w, tabsrc, Q, frow_lane, fexp_t, srow0, srow1, acc0, acc1); break;
    case 7: tile_block<7, GS>(w, tabsrc, Q, frow_lane, fexp_t, srow0, srow1, acc0, acc1); break;
    default: tile_block<8, GS>(w, tabsrc, Q, frow_lane, fexp_t, srow0, srow1, acc0, acc1); break;
    }
}

__device__ __forceinline__ void load_words(const uint32_t *const *base, int bmax, int64_t tix, int lane,
                                           uint32_t (&w)[8][2])
{
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        w[p][0] = w[p][1] = 0u;
        if (p < bmax) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(base[p] + tix * 64 + 2 * lane));
            w[p][0] = v.x;
            w[p][1] = v.y;
        }
    }
}

// Phase A: gate and up for one unit and one 16-row strip of I; writes h.
// Phase B (DOWN): down for one unit and one 16-row strip of H; writes part.
template <bool DOWN, int GS>
__global__ void __launch_bounds__(128) expert_phase_kernel(pmoe_layer L, int k, LayerWs W)
{
    __shared__ float acc[4][8][2][16][4];
    __shared__ const uint32_t *base[2][8];
    const int unit = blockIdx.x;
    if (unit >= W.flags[kFlagUnits])
        return;
    const int R = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
    const int H = L.H, I = L.I, G = L.G;
    const int e = W.unit_expert[unit], blk0 = W.unit_blk0[unit], nblk = W.unit_nblk[unit];
    const int bmax = W.unit_bmax[unit];
    const int nmat = DOWN ? 1 : 2;
    const int Kdim = DOWN ? I : H;
    const int ktiles = Kdim / 128;
    const int64_t mat_words = (int64_t)H * I / 32;
    if (threadIdx.x < 16) {
        const int m = threadIdx.x >> 3, p = threadIdx.x & 7;
        const uint32_t *ptr = nullptr;
        if (p < bmax && m < nmat) {
            const int slot = L.slot_of[e * 8 + p];
            if (slot < 0)
                W.flags[kFlagError] = 2;
            else
                ptr = L.pool + (int64_t)slot * L.slot_words + (DOWN ? 2 : m) * mat_words;
        }
        base[m][p] = ptr;
    }
    for (int i = threadIdx.x; i < 4 * 8 * 2 * 16 * 4; i += blockDim.x)
        (&acc[0][0][0][0][0])[i] = 0.0f;
    __syncthreads();
    for (int p = 0; p < bmax; ++p)
        if (base[0][p] == nullptr || (!DOWN && base[1][p] == nullptr))
            return;

    const int64_t escale = (int64_t)e * (2 * (int64_t)I * (H / G) + (int64_t)H * (I / G));
    const int srow_len = Kdim / G;
    const float *sbase[2];
    if (DOWN) {
        sbase[0] = L.scales + escale + 2 * (int64_t)I * (H / G);
        sbase[1] = sbase[0];
    } else {
        sbase[0] = L.scales + escale;
        sbase[1] = L.scales + escale + (int64_t)I * (H / G);
    }
    const int frag_words = (Kdim / 32) * 16; // per fragment row
    for (int Q = warp; Q < ktiles; Q += 4) {
        const int64_t tix = (int64_t)R * ktiles + Q;
        uint32_t wv[2][8][2];
        load_words(base[0], bmax, tix, lane, wv[0]);
        if (!DOWN)
            load_words(base[1], bmax, tix, lane, wv[1]);
        for (int bi = 0; bi < nblk; ++bi) {
            const int blk = blk0 + bi;
            const int d = W.blk_depth[blk], nmem = W.blk_nmem[blk];
            // B operand source of this lane: member c = g/2, part g&1
            const int c = g >> 1;
            const uint32_t *frow_lane = nullptr;
            if (c < nmem) {
                const int pair = W.blk_pair[blk * 4 + c];
                const int row = DOWN ? pair : pair / k;
                frow_lane = (DOWN ? W.hfrag : W.xfrag) + (int64_t)row * frag_words + (4 * (g & 1) + t) * 2;
            }
            // epilogue member of this lane: t
            const int *fexp_t = nullptr;
            if (t < nmem) {
                const int pair = W.blk_pair[blk * 4 + t];
                fexp_t = DOWN ? W.hexp + (int64_t)pair * (I / 128) : W.xexp + (int64_t)(pair / k) * (H / 128);
            }
            for (int m = 0; m < nmat; ++m) {
                const uint32_t *tabsrc = W.tabs + ((int64_t)blk * 3 + (DOWN ? 2 : m)) * kTabWords;
                const float *srow0 = sbase[m] + (int64_t)(16 * R + g) * srow_len;
                const float *srow1 = srow0 + 8 * (int64_t)srow_len;
                tile_block_any<GS>(d, wv[m], tabsrc, Q, frow_lane, fexp_t, srow0, srow1,
                                   &acc[warp][bi][m][g][t], &acc[warp][bi][m][g + 8][t]);
            }
        }
    }
    __syncthreads();
    // reduce over warps; one thread per (block, row, member)
    for (int i = threadIdx.x; i < nblk * 16 * 4; i += blockDim.x) {
        const int bi = i / 64, row = (i / 4) % 16, c = i % 4;
        const int blk = blk0 + bi;
        if (c >= W.blk_nmem[blk])
            continue;
        const int pair = W.blk_pair[blk * 4 + c];
        float v0 = 0.0f, v1 = 0.0f;
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) {
            v0 += acc[ww][bi][0][row][c];
            if (!DOWN)
                v1 += acc[ww][bi][1][row][c];
        }
        if (DOWN) {
            W.part[(int64_t)pair * H + 16 * R + row] = v0;
        } else {
            const float hval = v0 / (1.0f + expf(-v0)) * v1;
            W.h[(int64_t)pair * I + 16 * R + row] = hval;
        }
    }
}

// y[t][n] = sum over slots i of w[t,i] * part[t*k+i][n], in slot order.
__global__ void combine_kernel(const float *__restrict__ w, int T, int k, int H, LayerWs W,
                               float *__restrict__ y)
{
    const int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (n >= (int64_t)T * H)
        return;
    const int t = (int)(n / H), c = (int)(n % H);
    float s = 0.0f;
    for (int i = 0; i < k; ++i)
        s = __fmaf_rn(w[t * k + i], W.part[(int64_t)(t * k + i) * H + c], s);
    y[n] = s;
}

// Route + select for the decode step: one warp per token.
__global__ void route_select_kernel(const float *__restrict__ logits, const float *__restrict__ sens,
                                    int T, int E, int k, int B, int32_t *__restrict__ ids,
                                    float *__restrict__ w, uint8_t *__restrict__ depth)
{
    const int tok = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (tok >= T)
        return;
    const int lane = threadIdx.x & 31;
    int id;
    float wt;
    dev::route_token(logits + (int64_t)tok * E, E, k, id, wt);
    const float v = (lane < k) ? __fmul_rn(wt, __ldg(sens + id)) : 0.0f;
    const int b = dev::select_token(v, k, B, nullptr);
    if (lane < k) {
        ids[tok * k + lane] = id;
        w[tok * k + lane] = wt;
        depth[tok * k + lane] = (uint8_t)b;
    }
}

namespace {
thread_local cudaEvent_t g_prof_start = nullptr, g_prof_stop = nullptr;
}

pmoe_status check_layer(const pmoe_layer *L, int T, int k)
{
    if (!L || !L->pool || !L->slot_of || !L->scales || !L->codebooks)
        return PMOE_ERR_INVALID_ARG;
    if (L->E <= 0 || L->H <= 0 || L->I <= 0 || L->H % 128 || L->I % 128 ||
        !(L->G == 32 || L->G == 64 || L->G == 128) || L->slot_words < 3 * (int64_t)L->H * L->I / 32 ||
        L->slot_words % 2 || !aligned(L->pool, 8))
        return PMOE_ERR_INVALID_ARG;
    if (T < 0 || k < 1 || k > 32 || k > L->E || (int64_t)T * k > kMaxPairs)
        return PMOE_ERR_INVALID_ARG;
    return PMOE_OK;
}

pmoe_status layer_fwd(const pmoe_layer *L, const uint16_t *x, const int32_t *ids, const float *w,
                      const uint8_t *depth, int T, int k, float *y, void *ws, size_t ws_bytes,
                      cudaStream_t st)
{
    size_t need = 0;
    carve_layer_ws(nullptr, T, k, L->H, L->I, &need);
    if (ws_bytes < need)
        return PMOE_ERR_WORKSPACE;
    LayerWs W = carve_layer_ws(ws, T, k, L->H, L->I, nullptr);
    const int P = T * k;
    PMOE_CUDA(cudaMemsetAsync(W.flags, 0, 64 * 4, st));
    group_kernel<<<1, 512, P * sizeof(int), st>>>(ids, depth, P, L->E, W);
    PMOE_TRY(launch_status());
    {
        const int warps = T * (L->H / 128) + P * 3;
        prep_kernel<<<(warps + 3) / 4, 128, 0, st>>>(x, T, L->H, *L, W);
        PMOE_TRY(launch_status());
    }
    const int GS = L->G / 32;
    dim3 ga(P, L->I / 16), gb(P, L->H / 16);
    if (g_prof_start)
        PMOE_CUDA(cudaEventRecord(g_prof_start, st));
    if (GS == 1)
        expert_phase_kernel<false, 1><<<ga, 128, 0, st>>>(*L, k, W);
    else if (GS == 2)
        expert_phase_kernel<false, 2><<<ga, 128, 0, st>>>(*L, k, W);
    else
        expert_phase_kernel<false, 4><<<ga, 128, 0, st>>>(*L, k, W);
    PMOE_TRY(launch_status());
    {
        const int warps = P * (L->I / 128);
        hprep_kernel<<<(warps + 3) / 4, 128, 0, st>>>(P, L->I, W);
        PMOE_TRY(launch_status());
    }
    if (GS == 1)
        expert_phase_kernel<true, 1><<<gb, 128, 0, st>>>(*L, k, W);
    else if (GS == 2)
        expert_phase_kernel<true, 2><<<gb, 128, 0, st>>>(*L, k, W);
    else
        expert_phase_kernel<true, 4><<<gb, 128, 0, st>>>(*L, k, W);
    PMOE_TRY(launch_status());
    if (g_prof_stop)
        PMOE_CUDA(cudaEventRecord(g_prof_stop, st));
    const int64_t n = (int64_t)T * L->H;
    combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(w, T, k, L->H, W, y);
    return launch_status();
}

} // namespace pmoe

using namespace pmoe;

extern "C" {

pmoe_status pmoe_profile_events(pmoe_event start, pmoe_event stop)
{
    if ((start == nullptr) != (stop == nullptr))
        return PMOE_ERR_INVALID_ARG;
    g_prof_start = (cudaEvent_t)start;
    g_prof_stop = (cudaEvent_t)stop;
    return PMOE_OK;
}

size_t pmoe_layer_workspace_bytes(int T, int k, int E, int H, int I)
{
    (void)E;
    if (T < 0 || k < 1 || H <= 0 || I <= 0)
        return 0;
    size_t b = 0;
    carve_layer_ws(nullptr, T, k, H, I, &b);
    return b;
}

pmoe_status pmoe_moe_layer_fwd(const pmoe_layer *L, const uint16_t *x, const int32_t *ids,
                               const float *w, const uint8_t *depth, int T, int k, float *y,
                               void *ws, size_t ws_bytes, pmoe_stream stream)
{
    PMOE_TRY(check_layer(L, T, k));
    if (T == 0)
        return PMOE_OK;
    if (!x || !ids || !w || !depth || !y || !ws || !aligned(x, 8) || !aligned(ws, 256))
        return PMOE_ERR_INVALID_ARG;
    return layer_fwd(L, x, ids, w, depth, T, k, y, ws, ws_bytes, (cudaStream_t)stream);
}

pmoe_status pmoe_moe_decode_step(const pmoe_layer *L, const float *logits, const float *sens,
                                 const uint16_t *x, int T, int k, float avg_bits, float *y,
                                 int32_t *ids_out, float *w_out, uint8_t *depth_out, void *ws,
                                 size_t ws_bytes, pmoe_stream stream)
{
    PMOE_TRY(check_layer(L, T, k));
    if (T == 0)
        return PMOE_OK;
    if (!logits || !sens || !x || !y || !ws || !aligned(x, 8) || !aligned(ws, 256) ||
        !(avg_bits == avg_bits))
        return PMOE_ERR_INVALID_ARG;
    size_t need = 0;
    carve_layer_ws(nullptr, T, k, L->H, L->I, &need);
    if (ws_bytes < need)
        return PMOE_ERR_WORKSPACE;
    LayerWs W = carve_layer_ws(ws, T, k, L->H, L->I, nullptr);
    int32_t *ids = ids_out ? ids_out : W.ids;
    float *w = w_out ? w_out : W.w;
    uint8_t *depth = depth_out ? depth_out : W.depth;
    cudaStream_t st = (cudaStream_t)stream;
    const int B = select_budget(k, avg_bits);
    route_select_kernel<<<(T + 3) / 4, 128, 0, st>>>(logits, sens, T, L->E, k, B, ids, w, depth);
    PMOE_TRY(launch_status());
    return layer_fwd(L, x, ids, w, depth, T, k, y, ws, ws_bytes, st);
}

} // extern "C"
