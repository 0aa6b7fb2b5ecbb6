// MoE layer on bitplane prefixes (PagedMoE transcript cues 4, 29, 35, 37;
// arxivlens Abstract and Methodology): route, prefix selection, grouping of
// (token, expert) pairs by expert, gate/up prefix GEMV + SwiGLU, down prefix
// GEMV and the routing-weighted combine.
//
// Launches per call:
//  * xfrag_kernel, only when the batch is too large for the prep kernel to do
//    it: the activations' MMA fragments.
//  * layer_prep_kernel (one CTA): routing and selection (decode step), pairs
//    grouped by expert into column blocks (<= 2 pairs of one depth) and units
//    (<= 4 blocks of one expert, deepest units first), one record per unit,
//    decode tables, activation fragments (small batches) and zeroed counters.
//  * moe_main_kernel (persistent, one CTA per SM, launched as a programmatic
//    dependent of the prep kernel): a producer warp claims work items from a
//    global counter and streams their plane chunks into a shared-memory ring
//    with 1-D bulk copies; 16 consumer warps decode and multiply; an epilogue
//    warp finishes items of one column block. Gate/up items (unit, 16 rows of
//    I) come first; each writes its rows of h = silu(g) * u, and the last one
//    of a 128-row tile of h turns the tile into MMA fragments and counts it
//    toward the unit's ready count. Down items (unit, 128 rows of H) wait for
//    that count, write each pair's output rows, and the last pair of a token
//    row strip sums the k contributions in slot order into y.
// A plane chunk is read once per unit and decoded for every column block at
// the block's own depth, so tokens at different depths of one expert share
// the planes they have in common (transcript cues 13, 35).
#include <cuda_bf16.h>

#include "common.h"
#include "dev.cuh"
#include "layer.cuh"
#include "pipe.cuh"
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
    const size_t o_ut = take(P * 12 * 4);
    const size_t o_ca = take(P * (I / 16) * 4), o_ch = take(P * (I / 128) * 4), o_rb = take(P * 4);
    const size_t o_cb = take(P * (H / 128) * 4), o_yc = take((size_t)T * (H / 128) * 4);
    const size_t o_pa = take(P * (size_t)(I / 16) * 8 * 32 * 4), o_pb = take(P * (size_t)(H / 16) * 2 * 16 * 4);
    const size_t o_tab = take(P * 3 * kTabWords * 4);
    const size_t o_xf = take((size_t)T * (H / 32) * dev::kFragWords * 4), o_xe = take((size_t)T * (H / 128) * 4);
    const size_t o_h = take(P * I * 4);
    const size_t o_hf = take(P * (I / 32) * dev::kFragWords * 4), o_he = take(P * (size_t)hexp_stride(I) * 4);
    const size_t o_part = take(P * H * 4);
    const size_t o_ids = take(P * 4), o_w = take(P * 4), o_dep = take(P);
    // tensor-core path
    const bool tc = T >= kTcMinTokens;
    const size_t R = tc ? (size_t)tc_max_rows((int)P) : 0, U = tc ? P / kTcMinTokens + 1 : 0;
    const size_t o_tu = take(U * 16), o_trp = take(R * 4), o_trd = take(R * 4), o_tru = take(R * 4);
    const size_t o_trx = take(R * 4), o_trh = take(R * 4);
    const size_t o_txb = take(R * H * 2), o_thb = take(R * I * 2), o_tgu = take(tc ? P * 2 * I * 4 : 0);
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
    L.utab = reinterpret_cast<int *>(b + o_ut);
    L.cntA = reinterpret_cast<int *>(b + o_ca);
    L.cntH = reinterpret_cast<int *>(b + o_ch);
    L.readyB = reinterpret_cast<int *>(b + o_rb);
    L.cntB = reinterpret_cast<int *>(b + o_cb);
    L.ycnt = reinterpret_cast<int *>(b + o_yc);
    L.pA = reinterpret_cast<float *>(b + o_pa);
    L.pB = reinterpret_cast<float *>(b + o_pb);
    L.tabs = reinterpret_cast<uint32_t *>(b + o_tab);
    L.xfrag = reinterpret_cast<uint32_t *>(b + o_xf);
    L.xexp = reinterpret_cast<int *>(b + o_xe);
    L.h = reinterpret_cast<float *>(b + o_h);
    L.hfrag = reinterpret_cast<uint32_t *>(b + o_hf);
    L.hexp = reinterpret_cast<int *>(b + o_he);
    L.part = reinterpret_cast<float *>(b + o_part);
    if (tc) {
        L.tc_unit = reinterpret_cast<int4 *>(b + o_tu);
        L.tc_rpair = reinterpret_cast<int *>(b + o_trp);
        L.tc_rdep = reinterpret_cast<int *>(b + o_trd);
        L.tc_runit = reinterpret_cast<int *>(b + o_tru);
        L.tc_rxe = reinterpret_cast<int *>(b + o_trx);
        L.tc_rhe = reinterpret_cast<int *>(b + o_trh);
        L.tc_xb = reinterpret_cast<uint16_t *>(b + o_txb);
        L.tc_hb = reinterpret_cast<uint16_t *>(b + o_thb);
        L.tc_gu = reinterpret_cast<float *>(b + o_tgu);
    }
    L.ids = reinterpret_cast<int32_t *>(b + o_ids);
    L.w = reinterpret_cast<float *>(b + o_w);
    L.depth = reinterpret_cast<uint8_t *>(b + o_dep);
    return L;
}

// error codes written to flags[kFlagError]
constexpr int kErrBadPair = 1;     // an expert id or depth out of range
constexpr int kErrNoPlane = 2;     // a needed plane has no slot
constexpr int kErrTimeout = 3;     // a bounded wait ran out

// ---------------------------------------------------------------- prep kernel

struct PrepArgs {
    pmoe_layer L;
    const float *logits; // decode step only (else nullptr)
    const float *sens;
    const uint16_t *x;
    int T, k, B;
    int32_t *ids;
    float *w;
    uint8_t *depth;
    int frags_here; // 1: this kernel converts x; 0: a separate grid kernel did
    int tc;         // > 0: experts with at least this many pairs at depth <= kTcMaxLevels go to the
                    // tensor-core units (0: none)
    int n_rw;       // routing warps (decode step), each with E floats of staging
    LayerWs W;
};

constexpr int kPrepThreads = 1024;

__global__ void __launch_bounds__(kPrepThreads) layer_prep_kernel(PrepArgs a)
{
    pipe::launch_dependents();
    extern __shared__ int sm[]; // [P] key | [P] sorted pairs | 4 x [P] unit scratch | n_rw x [E] logits
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int T = a.T, k = a.k, P = T * k, E = a.L.E, H = a.L.H, I = a.L.I;
    LayerWs W = a.W;
    int *key = sm;           // expert * 16 + (15 - depth), or -1 for a bad pair
    int *sorted = sm + P;
    if (tid == 0) {
        W.flags[kFlagError] = 0;
        W.flags[kFlagWhere] = 0;
        W.flags[kFlagSched] = 0;
    }
    // 1. routing and selection (decode step) on warps [0, n_rw), the pairs' keys
    //    to shared memory; meanwhile the other warps convert x and zero counters.
    const int n_rw = (a.logits != nullptr) ? a.n_rw : 0;
    if (a.logits == nullptr) {
        for (int p = tid; p < P; p += blockDim.x) {
            const int e = a.ids[p], d = a.depth[p];
            key[p] = (e < 0 || e >= E || d < 1 || d > 8) ? -1 : e * 16 + (15 - d);
        }
    }
    if (warp < n_rw) {
        float *stage = reinterpret_cast<float *>(sm + 6 * P) + (int64_t)warp * E; // (used beyond 512 experts)
        for (int tok = warp; tok < T; tok += n_rw) {
            int id;
            float wt;
            if (E <= 512)
                dev::route_token_reg<16>(a.logits + (int64_t)tok * E, E, k, id, wt);
            else
                dev::route_token(a.logits + (int64_t)tok * E, E, k, stage, id, wt);
            const float v = (lane < k) ? __fmul_rn(wt, __ldg(a.sens + id)) : 0.0f;
            const int b = dev::select_token(v, k, a.B, nullptr);
            if (lane < k) {
                a.ids[tok * k + lane] = id;
                a.w[tok * k + lane] = wt;
                a.depth[tok * k + lane] = (uint8_t)b;
                key[tok * k + lane] = id * 16 + (15 - b);
            }
        }
    } else {
        const int wi = warp - n_rw, nw = nwarps - n_rw;
        if (a.frags_here) {
            for (int j = wi; j < T * (H / 128); j += nw) {
                const int t = j / (H / 128), Q = j % (H / 128);
                dev::make_xfrag_tile<true>(a.x + (int64_t)t * H, Q, W.xfrag + (int64_t)t * (H / 32) * dev::kFragWords,
                                           W.xexp + (int64_t)t * (H / 128));
            }
        }
        const int ti = tid - 32 * n_rw, nt = 32 * nw;
        for (int i = ti; i < P * (I / 16); i += nt)
            W.cntA[i] = 0;
        for (int i = ti; i < P * (I / 128); i += nt)
            W.cntH[i] = 0;
        for (int i = ti; i < P * (H / 128); i += nt)
            W.cntB[i] = 0;
        for (int i = ti; i < P; i += nt)
            W.readyB[i] = 0;
        for (int i = ti; i < T * (H / 128); i += nt)
            W.ycnt[i] = 0;
    }
    __syncthreads();
    // 2. group: rank of every pair under (expert asc, depth desc, pair asc)
    for (int p = tid; p < P; p += blockDim.x) {
        const int kp = key[p];
        int rank = 0;
        for (int q = 0; q < P; ++q) {
            const int kq = key[q];
            rank += (kq < kp || (kq == kp && q < p)) ? 1 : 0;
        }
        sorted[rank] = p;
    }
    __syncthreads();
    int *u_e = sm + 2 * P, *u_b0 = sm + 3 * P, *u_nb = sm + 4 * P, *u_bm = sm + 5 * P;
    __shared__ int s_nb, s_nu;
    if (tid == 0) {
        // 2a. tensor-core units: an expert whose pairs at depth <= kTcMaxLevels number at least
        //     kTcMinTokens gives them to units of at most kTcMaxCols pairs (the pairs of a run of one
        //     expert are ordered by depth, deepest first, so they are the run's tail); its deeper pairs
        //     stay with the persistent kernel. Operand rows: a unit's pairs, then zero rows up to a
        //     multiple of 16.
        int ntc = 0, nrow = 0;
        if (a.tc) {
            for (int r0 = 0; r0 < P;) {
                const int k0 = key[sorted[r0]];
                int r1 = r0 + 1;
                while (r1 < P && k0 >= 0 && (key[sorted[r1]] >> 4) == (k0 >> 4))
                    ++r1;
                if (k0 >= 0) {
                    int rs = r0;
                    while (rs < r1 && 15 - (key[sorted[rs]] & 15) > kTcMaxLevels)
                        ++rs;
                    const int cnt = r1 - rs;
                    if (cnt >= a.tc) {
                        const int nun = (cnt + kTcMaxCols - 1) / kTcMaxCols;
                        for (int j = 0, r = rs; j < nun; ++j) {
                            const int n = cnt / nun + (j < cnt % nun ? 1 : 0), npad = (n + 15) & ~15;
                            const int bmax = 15 - (key[sorted[r]] & 15);
                            W.tc_unit[ntc] = make_int4(k0 >> 4, n, npad | (bmax << 16), nrow);
                            for (int c = 0; c < npad; ++c, ++nrow) {
                                const int pr = c < n ? sorted[r + c] : -1;
                                W.tc_rpair[nrow] = pr;
                                W.tc_rdep[nrow] = pr >= 0 ? 15 - (key[pr] & 15) : 0;
                                W.tc_runit[nrow] = ntc;
                            }
                            for (int c = 0; c < n; ++c)
                                sorted[r + c] = -1; // leaves the persistent kernel's blocks
                            r += n;
                            ++ntc;
                        }
                    }
                }
                r0 = r1;
            }
        }
        W.flags[kFlagTcUnits] = ntc;
        W.flags[kFlagTcRows] = nrow;
        int nb = 0, nu = 0, prev_e = -1, prev_d = -1, nmem = 0, ublk = 0, bad = 0;
        for (int r = 0; r < P; ++r) {
            const int p = sorted[r];
            if (p < 0)
                continue;
            const int kk = key[p];
            if (kk < 0) {
                bad = 1;
                continue;
            }
            const int e = kk >> 4, d = 15 - (kk & 15);
            const bool new_e = (e != prev_e);
            if (new_e || d != prev_d || nmem == kMaxMembers) {
                if (new_e || ublk == kMaxBlocksPerUnit) {
                    u_e[nu] = e;
                    u_b0[nu] = nb;
                    u_bm[nu] = d;
                    u_nb[nu] = 0;
                    ++nu;
                    ublk = 0;
                }
                W.blk_depth[nb] = d;
                W.blk_expert[nb] = e;
                W.blk_nmem[nb] = 0;
                u_nb[nu - 1] = ++ublk;
                ++nb;
                nmem = 0;
            }
            W.blk_pair[(nb - 1) * 4 + nmem] = p;
            W.blk_nmem[nb - 1] = ++nmem;
            prev_e = e;
            prev_d = d;
        }
        s_nb = nb;
        s_nu = nu;
        W.flags[kFlagBlocks] = nb;
        W.flags[kFlagUnits] = nu;
        if (bad)
            W.flags[kFlagError] = kErrBadPair;
    }
    __syncthreads();
    const int nb = s_nb, nu = s_nu;
    // 3. units ordered by depth, deepest first (stable)
    for (int i = tid; i < nu; i += blockDim.x) {
        int rank = 0;
        for (int j = 0; j < nu; ++j)
            rank += (u_bm[j] > u_bm[i] || (u_bm[j] == u_bm[i] && j < i)) ? 1 : 0;
        W.unit_expert[rank] = u_e[i];
        W.unit_blk0[rank] = u_b0[i];
        W.unit_nblk[rank] = u_nb[i];
        W.unit_bmax[rank] = u_bm[i];
        // the same unit as one record with its page-table entries, for the persistent kernel
        int *ut = W.utab + rank * 12;
        ut[0] = u_e[i];
        ut[1] = u_bm[i];
        ut[2] = u_b0[i];
        ut[3] = u_nb[i];
        for (int p = 0; p < 8; ++p)
            ut[4 + p] = __ldg(a.L.slot_of + u_e[i] * 8 + p);
    }
    // 4. decode tables: one warp per (block, matrix)
    for (int j = warp; j < nb * 3; j += nwarps) {
        const int blk = j / 3, m = j % 3;
        const int e = W.blk_expert[blk], d = W.blk_depth[blk];
        uint32_t *dst = W.tabs + ((int64_t)blk * 3 + m) * kTabWords;
        RegTab tab;
        dev::build_tab(a.L.codebooks + ((int64_t)e * 3 + m) * 510, d, tab, d >= 5 ? dst + 16 : nullptr);
        if (lane < 4) {
            const int r = lane;
            dst[r] = r == 0 ? tab.h[0] : r == 1 ? tab.h[1] : r == 2 ? tab.h[2] : tab.h[3];
            dst[4 + r] = r == 0 ? tab.l[0] : r == 1 ? tab.l[1] : r == 2 ? tab.l[2] : tab.l[3];
        }
        if (lane == 0) {
            dst[8] = (uint32_t)tab.f;
            if (d == 1) {
                // depth 1 of an antisymmetric table decodes to signs (see dev::decode_kstep_sign)
                const float *cb = a.L.codebooks + ((int64_t)e * 3 + m) * 510;
                const float c0 = __ldg(cb), c1 = __ldg(cb + 1);
                dst[9] = __float_as_uint(c1);
                dst[10] = (c0 == -c1) ? 1u : 0u;
            }
        }
    }
}

__global__ void xfrag_kernel(const uint16_t *__restrict__ x, int T, int H, LayerWs W)
{
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (gw >= T * (H / 128))
        return;
    const int t = gw / (H / 128), Q = gw % (H / 128);
    dev::make_xfrag_tile<true>(x + (int64_t)t * H, Q, W.xfrag + (int64_t)t * (H / 32) * dev::kFragWords,
                               W.xexp + (int64_t)t * (H / 128));
}

// ---------------------------------------------------------------- persistent kernel

#include "moe_main.cuh"

namespace {
thread_local cudaEvent_t g_prof_start = nullptr, g_prof_stop = nullptr;
}

pmoe_status check_layer(const pmoe_layer *L, int T, int k)
{
    if (!L || !L->pool || !L->slot_of || !L->scales || !L->codebooks)
        return PMOE_ERR_INVALID_ARG;
    if (L->E <= 0 || L->H <= 0 || L->I <= 0 || L->H % 128 || L->I % 128 ||
        !(L->G == 32 || L->G == 64 || L->G == 128) || L->slot_words < 3 * (int64_t)L->H * L->I / 32 ||
        L->slot_words % 4 || !aligned(L->pool, 16))
        return PMOE_ERR_INVALID_ARG;
    if (T < 0 || k < 1 || k > 32 || k > L->E || (int64_t)T * k > kMaxPairs)
        return PMOE_ERR_INVALID_ARG;
    // shapes the persistent kernel tiles: 8 warps share each matrix of a 16-row gate/up item
    // (H/128 tiles), 2 warps a 16-row strip of down (I/128 tiles); a ring slot holds the 16
    // gate and 16 up rows of one plane, or 128 down rows of one plane.
    if (L->H % 1024 || L->H > 4096 || L->I % 256 || L->I > 1024)
        return PMOE_ERR_UNSUPPORTED;
    // an item's scale rows and table heads travel in one ring slot
    if (mk::meta_bytes_gateup(L->H, L->G, kMaxBlocksPerUnit) > mk::CHUNK ||
        mk::meta_bytes_down(L->I, L->G, kMaxBlocksPerUnit) > mk::CHUNK ||
        mk::meta_bytes_down(L->I, L->G, 1) + mk::meta_bytes_down_frags(L->I, kMaxMembers) > mk::CHUNK ||
        !aligned(L->scales, 16))
        return PMOE_ERR_UNSUPPORTED;
    return PMOE_OK;
}

static int g_num_sms[128] = {};
static unsigned g_smem_set[128] = {}; // per device: persistent-kernel variants whose shared-memory limit is set
static uint64_t g_wait_limit_ns = 200ull * 1000 * 1000;
static int g_tc_min = kTcMinTokens;

void set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns; }
uint64_t wait_limit_ns() { return g_wait_limit_ns; }

pmoe_status launch_layer(const pmoe_layer *L, const float *logits, const float *sens, const uint16_t *x,
                         int32_t *ids, float *w, uint8_t *depth, int T, int k, int B, float *y, void *ws,
                         size_t ws_bytes, cudaStream_t st)
{
    size_t need = 0;
    carve_layer_ws(nullptr, T, k, L->H, L->I, &need);
    if (ws_bytes < need)
        return PMOE_ERR_WORKSPACE;
    LayerWs W = carve_layer_ws(ws, T, k, L->H, L->I, nullptr);
    const int P = T * k;
    const bool frags_here = (int64_t)T * (L->H / 128) <= 128;
    if (!frags_here) {
        const int warps = T * (L->H / 128);
        xfrag_kernel<<<(warps + 7) / 8, 256, 0, st>>>(x, T, L->H, W);
        PMOE_TRY(launch_status());
    }
    // routing warps: at most one per token, one warp left for the x fragments; up to 512 experts a
    // warp keeps the logits in registers, beyond that it stages them (E floats of shared memory each)
    const bool staged_routing = L->E > 512;
    int n_rw = 0;
    if (logits != nullptr) {
        n_rw = (kPrepThreads / 32) - 1;
        n_rw = n_rw < T ? n_rw : T;
        if (staged_routing) {
            const int cap = (int)((32 * 1024) / ((size_t)L->E * sizeof(float)));
            n_rw = n_rw < cap ? n_rw : cap;
        }
        n_rw = n_rw > 1 ? n_rw : 1;
    }
    // (the tensor-core epilogue reads one scale per group: at most 32 groups along K keep the
    // group accumulators' turnover below the decode rate)
    const bool tc = W.tc_unit != nullptr && g_tc_min > 0 && L->H / L->G <= 32 && L->I / L->G <= 32;
    PrepArgs pa{*L, logits, sens, x, T, k, B, ids, w, depth, frags_here ? 1 : 0, tc ? g_tc_min : 0, n_rw, W};
    const size_t prep_smem = 6 * (size_t)P * sizeof(int) + (staged_routing ? (size_t)n_rw * L->E * sizeof(float) : 0);
    if (prep_smem > 40 * 1024)
        PMOE_CUDA(cudaFuncSetAttribute(layer_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem));
    layer_prep_kernel<<<1, kPrepThreads, prep_smem, st>>>(pa);
    PMOE_TRY(launch_status());

    if (g_prof_start)
        PMOE_CUDA(cudaEventRecord(g_prof_start, st));
    if (tc)
        PMOE_TRY(launch_tc(L, x, w, T, k, y, W, st));
    int dev = 0;
    PMOE_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 128)
        return PMOE_ERR_UNSUPPORTED;
    if (g_num_sms[dev] == 0)
        PMOE_CUDA(cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev));
    mk::Args ma{*L, T, k, w, y, W, wait_limit_ns()};
    const size_t smem = sizeof(mk::Smem);
    void (*kern)(mk::Args);
    switch (L->G) {
    case 32: kern = mk::moe_main_kernel<1>; break;
    case 64: kern = mk::moe_main_kernel<2>; break;
    default: kern = mk::moe_main_kernel<4>; break;
    }
    const unsigned vbit = 1u << (L->G == 32 ? 0 : (L->G == 64 ? 1 : 2));
    if (!(g_smem_set[dev] & vbit)) {
        PMOE_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        g_smem_set[dev] |= vbit;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g_num_sms[dev]);
    cfg.blockDim = dim3(mk::NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    PMOE_CUDA(cudaLaunchKernelEx(&cfg, kern, ma));
    if (g_prof_stop)
        PMOE_CUDA(cudaEventRecord(g_prof_stop, st));
    return PMOE_OK;
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

} // extern "C"

// Device address of page-locked host memory that is mapped into the current device's address
// space (the CUDA runtime's attributes of the pointer), else nullptr: pageable memory, device
// memory, or pinned memory registered without a mapping.
static void *mapped_host(const void *p)
{
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        (void)cudaGetLastError(); // (older runtimes report pageable memory as an error)
        return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || at.devicePointer == nullptr)
        return nullptr;
    return at.devicePointer;
}

extern "C" {

size_t pmoe_decode_host_workspace_bytes(int T, int k, int E, int H, int I)
{
    const size_t b = pmoe_layer_workspace_bytes(T, k, E, H, I);
    if (b == 0 || E <= 0)
        return 0;
    return b + al256((size_t)T * E * 4) + al256((size_t)T * H * 2) + al256((size_t)T * H * 4);
}

pmoe_status pmoe_set_wait_limit_ns(uint64_t ns)
{
    set_wait_limit_ns(ns == 0 ? 200ull * 1000 * 1000 : ns);
    return PMOE_OK;
}

pmoe_status pmoe_layer_error(const void *ws, int *code, int *detail, pmoe_stream stream)
{
    if (!ws || !code)
        return PMOE_ERR_INVALID_ARG;
    int f[8];
    PMOE_CUDA(cudaMemcpyAsync(f, ws, sizeof(f), cudaMemcpyDeviceToHost, (cudaStream_t)stream));
    PMOE_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
    *code = f[kFlagError];
    if (detail)
        *detail = f[kFlagWhere];
    return PMOE_OK;
}

pmoe_status pmoe_set_tc_min_tokens(int n)
{
    if (n != 0 && n < kTcMinTokens)
        return PMOE_ERR_INVALID_ARG;
    g_tc_min = n;
    return PMOE_OK;
}

pmoe_status pmoe_layer_counts(const void *ws, int *counts, pmoe_stream stream)
{
    if (!ws || !counts)
        return PMOE_ERR_INVALID_ARG;
    int f[16];
    PMOE_CUDA(cudaMemcpyAsync(f, ws, sizeof(f), cudaMemcpyDeviceToHost, (cudaStream_t)stream));
    PMOE_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
    counts[0] = f[kFlagBlocks];
    counts[1] = f[kFlagUnits];
    counts[2] = f[kFlagTcUnits];
    counts[3] = f[kFlagTcRows];
    return PMOE_OK;
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
    return launch_layer(L, nullptr, nullptr, x, const_cast<int32_t *>(ids), const_cast<float *>(w),
                        const_cast<uint8_t *>(depth), T, k, 0, y, ws, ws_bytes, (cudaStream_t)stream);
}

pmoe_status pmoe_moe_decode_step(const pmoe_layer *L, const float *logits, const float *sens,
                                 const uint16_t *x, int T, int k, float avg_bits, float *y,
                                 int32_t *ids_out, float *w_out, uint8_t *depth_out, void *ws,
                                 size_t ws_bytes, pmoe_stream stream)
{
    PMOE_TRY(check_layer(L, T, k));
    if (T == 0)
        return PMOE_OK;
    if (!logits || !sens || !x || !y || !ws || !aligned(x, 8) || !aligned(ws, 256) || !(avg_bits == avg_bits) ||
        L->E > 4096)
        return PMOE_ERR_INVALID_ARG;
    size_t need = 0;
    carve_layer_ws(nullptr, T, k, L->H, L->I, &need);
    if (ws_bytes < need)
        return PMOE_ERR_WORKSPACE;
    LayerWs W = carve_layer_ws(ws, T, k, L->H, L->I, nullptr);
    int32_t *ids = ids_out ? ids_out : W.ids;
    float *w = w_out ? w_out : W.w;
    uint8_t *depth = depth_out ? depth_out : W.depth;
    return launch_layer(L, logits, sens, x, ids, w, depth, T, k, select_budget(k, avg_bits), y, ws, ws_bytes,
                        (cudaStream_t)stream);
}

pmoe_status pmoe_moe_decode_step_host(const pmoe_layer *L, const float *logits, const float *sens,
                                      const uint16_t *x, int T, int k, float avg_bits, float *y, void *ws,
                                      size_t ws_bytes, pmoe_stream stream)
{
    PMOE_TRY(check_layer(L, T, k));
    if (T == 0)
        return PMOE_OK;
    if (!logits || !sens || !x || !y || !ws || !aligned(ws, 256))
        return PMOE_ERR_INVALID_ARG;
    if (ws_bytes < pmoe_decode_host_workspace_bytes(T, k, L->E, L->H, L->I))
        return PMOE_ERR_WORKSPACE;
    // Page-locked host buffers mapped into the device's address space are read and written by the
    // kernels in place (the prep kernel reads logits and x, the combine writes y); others go
    // through [layer workspace | logits | x | y] with copies queued on the stream.
    const size_t lb = pmoe_layer_workspace_bytes(T, k, L->E, L->H, L->I);
    const size_t nl = (size_t)T * L->E * 4, nx = (size_t)T * L->H * 2, ny = (size_t)T * L->H * 4;
    char *b = static_cast<char *>(ws);
    const cudaStream_t st = (cudaStream_t)stream;
    const float *logits_d = static_cast<const float *>(mapped_host(logits));
    const uint16_t *x_d = static_cast<const uint16_t *>(mapped_host(x));
    float *y_d = static_cast<float *>(mapped_host(y));
    if (!logits_d) {
        float *p = reinterpret_cast<float *>(b + lb);
        PMOE_CUDA(cudaMemcpyAsync(p, logits, nl, cudaMemcpyHostToDevice, st));
        logits_d = p;
    }
    if (!x_d || !aligned(x_d, 8)) {
        uint16_t *p = reinterpret_cast<uint16_t *>(b + lb + al256(nl));
        PMOE_CUDA(cudaMemcpyAsync(p, x, nx, cudaMemcpyHostToDevice, st));
        x_d = p;
    }
    const bool y_copy = y_d == nullptr;
    if (y_copy)
        y_d = reinterpret_cast<float *>(b + lb + al256(nl) + al256(nx));
    PMOE_TRY(pmoe_moe_decode_step(L, logits_d, sens, x_d, T, k, avg_bits, y_d, nullptr, nullptr, nullptr, ws, lb,
                                  stream));
    if (y_copy)
        PMOE_CUDA(cudaMemcpyAsync(y, y_d, ny, cudaMemcpyDeviceToHost, st));
    return PMOE_OK;
}

} // extern "C"
