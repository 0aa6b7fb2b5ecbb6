// Persistent expert kernel of the MoE layer (included by layer.cu).
//
// One CTA per SM: warp NCW is the producer, warps 0..NCW-1 consume, warp NCW+1
// is the epilogue warp.
//
// Producer: takes work items from a global counter (gate/up items first, then
// down items; units deepest first), one at a time once the two-entry item
// queue has room, publishes each item in that queue and streams the item's
// bytes into a ring of 16 KB shared-memory slots with 1-D bulk copies that
// all complete on the item's mbarrier (one per queue entry, armed once with
// the item's bytes): one chunk per plane ([16 gate rows | 16 up rows] of
// a gate/up item, 128 rows of a down item) and then a "meta" chunk (the scale
// rows of the item's matrices and the decode tables of its column blocks; for
// down items of one column block also the members' h fragments). An item has
// at most 9 chunks, fewer than the ring's slots, so no copy of an item ever
// waits for a slot the same item still holds. An item's slots are free again
// once the item is complete (its queue entry released), so consumers do not
// release slots one by one.
//
// Consumers: every consumer warp takes every item and multiplies its share of
// the item's tiles (gate/up: warps 0-7 the gate rows, 8-15 the up rows, each
// an eighth of the columns). For items of one column block the partial sums go
// to a shared-memory slot of the item (one per queue entry); the consumer warp
// that finishes last (a shared-memory atomic) hands the item to the epilogue
// warp, which reduces the partials in a fixed order, so results are
// deterministic, releases the queue entry, then writes h = silu(g) * u
// (gate/up) or the pair's output rows (down) and moves the global counters:
// the last gate/up item of a 128-row tile of h converts it to MMA fragments and
// bumps the unit's ready count; the last pair of a token's 128 output rows sums
// the k pair outputs into y in slot order. Down items wait (bounded) until their
// unit's h fragments are all ready. Items with several column blocks (batched
// tokens) keep their partials in global memory, and the consumer warp that
// finishes last (a global atomic) reduces them.
namespace mk {

constexpr int NCW = 16;                    // consumer warps
constexpr int NTHREADS = (NCW + 2) * 32; // + producer warp + epilogue warp
constexpr int NSLOT = 12;                  // ring slots
constexpr int CHUNK = 16384;               // bytes per ring slot
constexpr int QDEPTH = 2;                  // item queue (= partial-sum slots): claim at most one item ahead
// The producer's slot reuse waits only for the item before the current one: every older item is
// complete once the current one is claimed, which holds for a two-entry queue.
static_assert(QDEPTH == 2, "ring slot reuse assumes a two-entry item queue");
constexpr int RED_WORDS = 16 * 4;          // per warp: [row][member]
constexpr int KFW = dev::kFragWords;        // words per k-step of a vector's activation fragments
constexpr int XS_WORDS = (4096 / 32) * dev::kFragWords; // shared copy of the x fragments (T == 1, H <= 4096)
constexpr int TAB_BYTES = 64;              // decode-table head copied per (block, matrix)
constexpr uint64_t kDeadlineNs = 200ull * 1000 * 1000;

struct Desc {
    int kind; // 0 gate/up, 1 down, 2 stop
    int u;    // unit
    int strip;
    int c0;   // first chunk of the item
};

constexpr int UT_MAX = 32; // units (and column blocks) whose layout is staged in shared memory

struct UnitTab {
    int e, bmax, blk0, nblk;
    int slot[8]; // slot of each plane of the unit's expert
};

struct BlkTab {
    int depth, nmem, pair[4];
};

struct Smem {
    alignas(128) unsigned char ring[NSLOT][CHUNK];
    float red[QDEPTH][NCW][RED_WORDS];
    uint32_t xs[XS_WORDS];
    uint32_t zeros[4];
    int xse[32];
    uint64_t ifull[QDEPTH], qfull[QDEPTH], qempty[QDEPTH], epi[QDEPTH]; // ifull: all of an item's bytes landed
    Desc q[QDEPTH];
    int cnt[QDEPTH];
    UnitTab ut[UT_MAX];
    BlkTab bt[UT_MAX];
};
static_assert(sizeof(Smem) <= 227 * 1024, "shared memory of the persistent kernel exceeds one SM's");

struct Args {
    pmoe_layer L;
    int T, k;
    const float *wts; // routing weights [T*k]
    float *y;         // [T*H]
    LayerWs W;
    uint64_t limit_ns; // bound of every wait (one deadline per launch)
};

// The units' and column blocks' layout: from the shared-memory copy when the
// call has few of them (decode), else from the workspace.
struct UnitView {
    const Smem &S;
    const LayerWs &W;
    const int32_t *slot_of;
    bool staged;
    __device__ int expert(int u) const { return staged ? S.ut[u].e : __ldg(W.unit_expert + u); }
    __device__ int bmax(int u) const { return staged ? S.ut[u].bmax : __ldg(W.unit_bmax + u); }
    __device__ int blk0(int u) const { return staged ? S.ut[u].blk0 : __ldg(W.unit_blk0 + u); }
    __device__ int nblk(int u) const { return staged ? S.ut[u].nblk : __ldg(W.unit_nblk + u); }
    __device__ int slot(int u, int e, int p) const { return staged ? S.ut[u].slot[p] : __ldg(slot_of + e * 8 + p); }
    __device__ int bdepth(int b) const { return staged ? S.bt[b].depth : __ldg(W.blk_depth + b); }
    __device__ int bnmem(int b) const { return staged ? S.bt[b].nmem : __ldg(W.blk_nmem + b); }
    __device__ int bpair(int b, int c) const { return staged ? S.bt[b].pair[c] : __ldg(W.blk_pair + b * 4 + c); }
};

// bytes of an item's meta chunk: scales of its rows, then table heads
__host__ __device__ inline int meta_bytes_gateup(int H, int G, int nblk) { return 2 * 16 * (H / G) * 4 + nblk * 2 * TAB_BYTES; }
__host__ __device__ inline int meta_bytes_down(int I, int G, int nblk) { return 128 * (I / G) * 4 + nblk * TAB_BYTES; }
// down items with one column block also carry the members' h fragments and exponents
__host__ __device__ inline int meta_bytes_down_frags(int I, int nmem) { return nmem * (3 * I + hexp_stride(I) * 4); }

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

__device__ __forceinline__ void red_add_release(int *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void load_tab_smem(const unsigned char *src, RegTab &t)
{
    const uint4 a = *reinterpret_cast<const uint4 *>(src);
    const uint4 b = *reinterpret_cast<const uint4 *>(src + 16);
    t.h[0] = a.x; t.h[1] = a.y; t.h[2] = a.z; t.h[3] = a.w;
    t.l[0] = b.x; t.l[1] = b.y; t.l[2] = b.z; t.l[3] = b.w;
    t.f = *reinterpret_cast<const int *>(src + 32);
}

// 2^-e as a float (e in [-126, 127]).
__device__ __forceinline__ float pow2neg(int e) { return __int_as_float((127 - e) << 23); }

// The four int32 partial sums of one row (dh0 = sum vh*xh, dh1 = sum vh*xl,
// dl0 = sum vl*xh, dl1 = sum vl*xl) as one integer in units of 256 (the
// vl*xl term rounded to that unit, far below the float resolution of the sum).
__device__ __forceinline__ float combine256(int dh0, int dh1, int dl0, int dl1)
{
    return (float)(dh0 * 256 + dh1 + dl0 + ((dl1 + 128) >> 8));
}

// B fragment sources: 0 = x fragments in shared memory, 1 = x fragments in
// global memory (written by the prep kernel), 2 = h fragments in global memory
// (written by other CTAs of this kernel: read through L2).
template <int FRAG>
__device__ __forceinline__ uint2 frag_at(const uint32_t *p)
{
    if constexpr (FRAG == 2)
        return __ldcg(reinterpret_cast<const uint2 *>(p));
    else if constexpr (FRAG == 1)
        return __ldg(reinterpret_cast<const uint2 *>(p));
    else
        return *reinterpret_cast<const uint2 *>(p);
}

template <int FRAG>
__device__ __forceinline__ int exp_at(const int *p)
{
    if constexpr (FRAG == 2)
        return __ldcg(p);
    else if constexpr (FRAG == 1)
        return __ldg(p);
    else
        return *p;
}

// One column block over this warp's tiles of one matrix.
//  pp[p]: plane p's chunk + this warp's first tile + lane offset (shared).
//  tabs: table head in shared memory; big: full table (global) for depth >= 5.
//  fptr/fstep: this lane's B-fragment words at the first tile and the step per
//  k-step in words (FRAG 0: always valid, a zero block for absent members).
//  exps: exponents of this lane's epilogue member (nullptr: no epilogue).
//  sc0/sc1: scale rows (shared) of rows g, g+8 at the warp's first group.
template <int B, int GS, int FRAG>
__device__ __forceinline__ void warp_block(const unsigned char *const (&pp)[8], int ntiles, int Q0,
                                           const unsigned char *tabs, const uint32_t *big, const uint32_t *fptr,
                                           int fstep, const int *exps, const float *sc0, const float *sc1,
                                           float &acc0, float &acc1)
{
    constexpr int NG = 4 / GS; // scale groups per 128-column tile
    RegTab tab;
    load_tab_smem(tabs, tab);
    const bool epi = exps != nullptr;
    const float lf = dev::combine24_lane_factor(threadIdx.x & 3);
    for (int j = 0; j < ntiles; ++j) {
        uint32_t w[8][2];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            w[p][0] = w[p][1] = 0u;
            if (p < B) {
                const uint2 v = *reinterpret_cast<const uint2 *>(pp[p] + j * 256);
                w[p][0] = v.x;
                w[p][1] = v.y;
            }
        }
        const float fac = epi ? lf * pow2neg(tab.f + exp_at<FRAG>(exps + Q0 + j)) : 0.0f;
        int dh[4] = {0, 0, 0, 0}, dl[4] = {0, 0, 0, 0};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            uint32_t ah[4], al[4];
            dev::decode_kstep<B>(w, s, tab, big, ah, al);
            uint2 bv = make_uint2(0u, 0u);
            if (FRAG == 0 || fptr != nullptr)
                bv = frag_at<FRAG>(fptr + (j * 4 + s) * fstep);
            dev::mma_s8(dh, ah, bv.x, bv.y);
            dev::mma_s8(dl, al, bv.x, bv.y);
            if ((s + 1) % GS == 0) {
                const int gi = j * NG + s / GS;
                acc0 = __fmaf_rn(dev::combine24(dh[0], dh[1], dl[0], dl[1]), sc0[gi] * fac, acc0);
                acc1 = __fmaf_rn(dev::combine24(dh[2], dh[3], dl[2], dl[3]), sc1[gi] * fac, acc1);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dh[i] = dl[i] = 0;
            }
        }
    }
}

// Depth 1 of an antisymmetric table: +-1 bytes, one MMA per k-step, and the
// group sums scaled by C[1][1] (table head word 9).
template <int GS, int FRAG>
__device__ __forceinline__ void warp_block_sign(const unsigned char *const (&pp)[8], int ntiles, int Q0,
                                                const unsigned char *tabs, const uint32_t *fptr, int fstep,
                                                const int *exps, const float *sc0, const float *sc1, float &acc0,
                                                float &acc1)
{
    constexpr int NG = 4 / GS;
    const float c1 = __uint_as_float(reinterpret_cast<const uint32_t *>(tabs)[9]);
    const bool epi = exps != nullptr;
    const float lf = dev::combine24_lane_factor(threadIdx.x & 3);
    for (int j = 0; j < ntiles; ++j) {
        uint32_t w[8][2];
        const uint2 v = *reinterpret_cast<const uint2 *>(pp[0] + j * 256);
        w[0][0] = v.x;
        w[0][1] = v.y;
        const float fac = epi ? c1 * lf * 0.00390625f * pow2neg(exp_at<FRAG>(exps + Q0 + j)) : 0.0f;
        int dh[4] = {0, 0, 0, 0};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            uint32_t a[4];
            dev::decode_kstep_sign(w, s, a);
            uint2 bv = make_uint2(0u, 0u);
            if (FRAG == 0 || fptr != nullptr)
                bv = frag_at<FRAG>(fptr + (j * 4 + s) * fstep);
            dev::mma_s8(dh, a, bv.x, bv.y);
            if ((s + 1) % GS == 0) {
                const int gi = j * NG + s / GS;
                acc0 = __fmaf_rn(dev::combine24(dh[0], dh[1], 0, 0), sc0[gi] * fac, acc0);
                acc1 = __fmaf_rn(dev::combine24(dh[2], dh[3], 0, 0), sc1[gi] * fac, acc1);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dh[i] = 0;
            }
        }
    }
}

template <int GS, int FRAG>
__device__ __forceinline__ void warp_block_any(int d, const unsigned char *const (&pp)[8], int ntiles, int Q0,
                                               const unsigned char *tabs, const uint32_t *big, const uint32_t *fptr,
                                               int fstep, const int *exps, const float *sc0, const float *sc1,
                                               float &acc0, float &acc1)
{
    switch (d) {
    case 1:
        if (reinterpret_cast<const uint32_t *>(tabs)[10] != 0u)
            warp_block_sign<GS, FRAG>(pp, ntiles, Q0, tabs, fptr, fstep, exps, sc0, sc1, acc0, acc1);
        else
            warp_block<1, GS, FRAG>(pp, ntiles, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1);
        break;
    case 2: warp_block<2, GS, FRAG>(pp, ntiles, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1); break;
    case 3: warp_block<3, GS, FRAG>(pp, ntiles, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1); break;
    case 4: warp_block<4, GS, FRAG>(pp, ntiles, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1); break;
    case 5: warp_block<5, GS, FRAG>(pp, ntiles, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1); break;
    case 6: warp_block<6, GS, FRAG>(pp, ntiles, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1); break;
    case 7: warp_block<7, GS, FRAG>(pp, ntiles, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1); break;
    default: warp_block<8, GS, FRAG>(pp, ntiles, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1); break;
    }
    // lanes t = 0, 2 hold tokens 0, 1 of the block once their partners t = 1, 3 are added
    acc0 += __shfl_down_sync(0xffffffffu, acc0, 1);
    acc1 += __shfl_down_sync(0xffffffffu, acc1, 1);
}

// h of one pair, one 128-column tile -> B fragments (one warp); h read through L2.
__device__ void h_to_frags(const LayerWs &W, int I, int pair, int Q)
{
    const int lane = threadIdx.x & 31;
    const float4 f = __ldcg(reinterpret_cast<const float4 *>(W.h + (int64_t)pair * I + 128 * Q + 4 * lane));
    float v[4] = {f.x, f.y, f.z, f.w};
    float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    m = dev::warp_max(m);
    const int sx = dev::fix_exponent24(m);
    uint32_t fw[3];
    dev::frag_words(v, sx, fw);
    uint32_t *xf = W.hfrag + ((int64_t)pair * (I / 32) + Q * 4) * dev::kFragWords + dev::frag_lane_word(lane);
    __stcg(xf, fw[0]);
    __stcg(xf + 8, fw[1]);
    __stcg(xf + 16, fw[2]);
    if (lane == 0)
        __stcg(W.hexp + (int64_t)pair * hexp_stride(I) + Q, sx);
}

// After the h rows of a gate/up item are written: count the item on its
// 128-row tile of h; the last one converts the tile and bumps the unit's ready count.
__device__ void gateup_tile_done(const LayerWs &W, const UnitView &V, int I, int u, int s16, int blk0, int nblk)
{
    const int lane = threadIdx.x & 31;
    __syncwarp();
    int last = 0;
    if (lane == 0)
        last = (atom_add_acq_rel(&W.cntH[u * (I / 128) + s16 / 8], 1) == 7);
    last = __shfl_sync(0xffffffffu, last, 0);
    __syncwarp();
    if (!last)
        return;
    for (int bi = 0; bi < nblk; ++bi) {
        const int blk = blk0 + bi, nmem = V.bnmem(blk);
        for (int c = 0; c < nmem; ++c)
            h_to_frags(W, I, V.bpair(blk, c), s16 / 8);
    }
    __syncwarp();
    if (lane == 0)
        red_add_release(&W.readyB[u], 1);
}

// After a pair's 128 output rows are written: the last of the token's k pairs
// sums them into y in slot order. Lane owns rows lane + 32*i (i < 4); the
// partial rows of 4 slots at a time are loaded before they are summed, so the
// L2 round trips overlap instead of following one another.
__device__ void down_rows_done(const Args &a, int pair, int s128)
{
    const LayerWs &W = a.W;
    const int lane = threadIdx.x & 31, H = a.L.H, k = a.k;
    const int tok = pair / k;
    __syncwarp();
    int last = 0;
    if (lane == 0)
        last = (atom_add_acq_rel(&W.ycnt[tok * (H / 128) + s128], 1) == k - 1);
    last = __shfl_sync(0xffffffffu, last, 0);
    __syncwarp();
    if (!last)
        return;
    const float *part = W.part + (int64_t)tok * k * H + 128 * s128 + lane;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int i0 = 0; i0 < k; i0 += 4) {
        float v[4][4], wt[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool ok = i0 + j < k;
            wt[j] = ok ? __ldg(a.wts + tok * k + i0 + j) : 0.0f;
#pragma unroll
            for (int r = 0; r < 4; ++r)
                v[j][r] = ok ? __ldcg(part + (int64_t)(i0 + j) * H + 32 * r) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (i0 + j < k) {
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    acc[r] = __fmaf_rn(wt[j], v[j][r], acc[r]);
            }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
        a.y[(int64_t)tok * H + 128 * s128 + 32 * r + lane] = acc[r];
}

template <int GS>
__global__ void __launch_bounds__(NTHREADS, 1) moe_main_kernel(Args a)
{
    extern __shared__ __align__(128) unsigned char smraw[];
    Smem &S = *reinterpret_cast<Smem *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const pmoe_layer &L = a.L;
    const LayerWs &W = a.W;
    const int H = L.H, I = L.I, G = L.G, T = a.T, k = a.k;
    const uint64_t deadline = pipe::globaltimer() + a.limit_ns;

    if (tid == 0) {
        for (int s = 0; s < QDEPTH; ++s) {
            pipe::mbar_init(&S.ifull[s], 1);
            pipe::mbar_init(&S.qfull[s], 1);
            pipe::mbar_init(&S.qempty[s], NCW + 1); // consumers + epilogue warp
            pipe::mbar_init(&S.epi[s], 1);
            S.cnt[s] = 0;
        }
        pipe::fence_barrier_init();
    }
    if (tid < 4)
        S.zeros[tid] = 0u;
    __syncthreads();
    pipe::wait_prerequisites(); // the prep kernel's results are visible from here on

    const int nunits = W.flags[kFlagUnits];
    const int SA = I / 16;  // gate/up items per unit (16 rows of I each)
    const int SB = H / 128; // down items per unit (128 rows of H each)
    const int totalA = nunits * SA, total = totalA + nunits * SB;
    const int64_t mat_words = (int64_t)H * I / 32;
    const int64_t escale_len = 2 * (int64_t)I * (H / G) + (int64_t)H * (I / G);
    const bool stage_x = (T == 1 && H <= 4096);
    // ---- producer state and item issue (warp NCW, lane 0 only)
    int c = 0, pq = 0; // chunks and items the producer has issued
    bool ok = true;
    // Ring slots are released per item, by the item's completion (its queue entry's qempty phase):
    // a slot was last used by chunk c - NSLOT; every item before the previous one is complete once
    // the current item has been claimed (the claim waits for the item QDEPTH back), so only a
    // chunk of the previous item (first chunk prev_c0) has to wait, for that item to complete.
    int prev_c0 = 0;
    bool prev_done = true;
    auto next_slot = [&](int &s) {
        s = c % NSLOT;
        if (c >= NSLOT && !prev_done && c - NSLOT >= prev_c0) {
            const int n1 = pq - 2; // the previous item (pq already counts the current one)
            if (!pipe::mbar_wait_tight(&S.qempty[n1 % QDEPTH], (n1 / QDEPTH) & 1, deadline)) {
                set_error(W, kErrTimeout, 2);
                ok = false;
            }
            prev_done = true;
        }
    };
    auto make_desc = [&](int u) {
        Desc d;
        if (u >= total) {
            d.kind = 2;
            d.u = d.strip = 0;
        } else if (u < totalA) {
            d.kind = 0;
            d.u = u / SA;
            d.strip = u % SA;
        } else {
            d.kind = 1;
            d.u = (u - totalA) / SB;
            d.strip = (u - totalA) % SB;
        }
        d.c0 = c;
        return d;
    };
    int last_item = -1; // index of the last item whose copies were issued
    auto issue_item = [&](const UnitView &UV, const Desc &d, int n) {
        const int e = UV.expert(d.u), bmax = UV.bmax(d.u);
        const int blk0 = UV.blk0(d.u), nblk = UV.nblk(d.u);
        const float *esc = L.scales + (int64_t)e * escale_len;
        // all of the item's copies complete on its queue entry's barrier: one expect_tx with the
        // item's bytes (planes present + meta), so that consumers wait once per item
        uint64_t *bar = &S.ifull[n % QDEPTH];
        {
            const uint32_t pbytes = d.kind == 0 ? (uint32_t)(2 * (H / 128) * 256) : (uint32_t)(8 * (I / 128) * 256);
            uint32_t total = d.kind == 0 ? (uint32_t)meta_bytes_gateup(H, G, nblk) : (uint32_t)meta_bytes_down(I, G, nblk);
            if (d.kind == 1 && nblk == 1)
                total += meta_bytes_down_frags(I, UV.bnmem(blk0));
            for (int p = 0; p < bmax; ++p)
                if (UV.slot(d.u, e, p) >= 0)
                    total += pbytes;
            pipe::mbar_arrive_expect_tx(bar, total);
        }
        last_item = n;
        // chunk order [planes | meta]: an item has at most 9 chunks, fewer than NSLOT, so none of
        // its copies waits for a slot the item itself holds. A gate/up plane chunk holds the
        // plane's 16 gate rows then its 16 up rows; a down plane chunk 128 rows of the down matrix.
        auto issue_planes = [&]() {
            for (int p = 0; p < bmax && ok; ++p) {
                int s;
                next_slot(s);
                if (!ok)
                    break;
                const int slot = UV.slot(d.u, e, p);
                const uint32_t bytes = d.kind == 0 ? (uint32_t)(2 * (H / 128) * 256) : (uint32_t)(8 * (I / 128) * 256);
                if (slot >= 0) {
                    const uint32_t *base = L.pool + (int64_t)slot * L.slot_words;
                    if (d.kind == 0) {
                        const int64_t off = (int64_t)d.strip * (H / 128) * 64;
                        pipe::bulk_g2s(S.ring[s], base + off, bytes / 2, bar);
                        pipe::bulk_g2s(S.ring[s] + bytes / 2, base + mat_words + off, bytes / 2, bar);
                    } else {
                        pipe::bulk_g2s(S.ring[s], base + 2 * mat_words + (int64_t)d.strip * 8 * (I / 128) * 64,
                                       bytes, bar);
                    }
                } else {
                    // a missing plane: report it (its bytes were not expected; the slot stays empty)
                    set_error(W, kErrNoPlane, e * 8 + p);
                }
                ++c;
            }
        };
        auto issue_meta = [&]() {
            int s;
            next_slot(s);
            if (!ok)
                return;
            if (d.kind == 0) {
                const uint32_t sb = 16 * (H / G) * 4;
                for (int m = 0; m < 2; ++m)
                    pipe::bulk_g2s(S.ring[s] + m * sb,
                                   esc + (int64_t)m * I * (H / G) + (int64_t)d.strip * 16 * (H / G), sb, bar);
                for (int bi = 0; bi < nblk; ++bi)
                    for (int m = 0; m < 2; ++m)
                        pipe::bulk_g2s(S.ring[s] + 2 * sb + (bi * 2 + m) * TAB_BYTES,
                                       W.tabs + ((int64_t)(blk0 + bi) * 3 + m) * kTabWords, TAB_BYTES, bar);
            } else {
                const uint32_t sb = 128 * (I / G) * 4;
                int nmem = 0;
                if (nblk == 1) {
                    // the h fragments come along: wait (bounded) until the unit's h is converted
                    nmem = UV.bnmem(blk0);
                    while (pipe::ld_acquire(&W.readyB[d.u]) < I / 128) {
                        if (pipe::globaltimer() > deadline) {
                            set_error(W, kErrTimeout, 5);
                            break;
                        }
                        __nanosleep(256);
                    }
                    pipe::fence_proxy_async();
                }
                pipe::bulk_g2s(S.ring[s], esc + 2 * (int64_t)I * (H / G) + (int64_t)d.strip * 128 * (I / G), sb,
                               bar);
                for (int bi = 0; bi < nblk; ++bi)
                    pipe::bulk_g2s(S.ring[s] + sb + bi * TAB_BYTES,
                                   W.tabs + ((int64_t)(blk0 + bi) * 3 + 2) * kTabWords, TAB_BYTES, bar);
                unsigned char *fb = S.ring[s] + sb + nblk * TAB_BYTES;
                for (int c2 = 0; c2 < nmem; ++c2) {
                    const int pair = UV.bpair(blk0, c2);
                    pipe::bulk_g2s(fb + c2 * 3 * I, W.hfrag + (int64_t)pair * (I / 32) * dev::kFragWords, 3 * I,
                                   bar);
                    pipe::bulk_g2s(fb + nmem * 3 * I + c2 * hexp_stride(I) * 4,
                                   W.hexp + (int64_t)pair * hexp_stride(I), hexp_stride(I) * 4, bar);
                }
            }
            ++c;
        };
        issue_planes();
        if (ok)
            issue_meta();
        prev_c0 = d.c0;
        prev_done = false;
    };
    // A gate/up first item is issued before the staging below, from the unit records in
    // global memory, so that its copies are in flight while the CTA stages its tables.
    if (warp == NCW && lane == 0 && (int)blockIdx.x < totalA) {
        const UnitView VG{S, W, L.slot_of, false};
        const Desc d = make_desc((int)blockIdx.x);
        S.q[0] = d;
        pipe::mbar_arrive(&S.qfull[0]);
        pq = 1;
        issue_item(VG, d, 0);
    }
    if (stage_x) {
        for (int i = tid; i < (H / 32) * dev::kFragWords; i += NTHREADS)
            S.xs[i] = W.xfrag[i];
        for (int i = tid; i < H / 128; i += NTHREADS)
            S.xse[i] = W.xexp[i];
    }
    // few units (decode): their layout and page-table entries go to shared memory once
    const int nblocks = W.flags[kFlagBlocks];
    const UnitView V{S, W, L.slot_of, nunits <= UT_MAX && nblocks <= UT_MAX};
    if (V.staged) {
        static_assert(sizeof(UnitTab) == 12 * sizeof(int), "unit record layout");
        for (int i = tid; i < nunits * 12; i += NTHREADS)
            reinterpret_cast<int *>(S.ut)[i] = __ldg(W.utab + i);
        for (int i = tid; i < nblocks; i += NTHREADS) {
            S.bt[i].depth = __ldg(W.blk_depth + i);
            S.bt[i].nmem = __ldg(W.blk_nmem + i);
            for (int c2 = 0; c2 < 4; ++c2)
                S.bt[i].pair[c2] = __ldg(W.blk_pair + i * 4 + c2);
        }
    }
    __syncthreads();

    if (warp == NCW) {
        // ------------------------------------------------------------ producer
        if (lane != 0)
            return;
        while (ok) {
            // claim only once the queue has room: an item is taken when this SM can start on it soon
            const int qs = pq % QDEPTH;
            if (pq >= QDEPTH && !pipe::mbar_wait_tight(&S.qempty[qs], ((pq / QDEPTH) + 1) & 1, deadline)) {
                set_error(W, kErrTimeout, 1);
                break;
            }
            // the first item of each SM is its own index; the counter hands out the rest
            const int u = (pq == 0) ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(&W.flags[kFlagSched], 1);
            const Desc d = make_desc(u);
            S.q[qs] = d;
            pipe::mbar_arrive(&S.qfull[qs]);
            ++pq;
            if (d.kind == 2)
                break;
            issue_item(V, d, pq - 1);
        }
        // no copy may still be landing in shared memory when the CTA exits: items before the last
        // two are complete (their consumers finished), so wait for those two
        for (int n = (last_item > 0 ? last_item - 1 : 0); n <= last_item; ++n)
            pipe::mbar_wait(&S.ifull[n % QDEPTH], (n / QDEPTH) & 1, deadline + kDeadlineNs);
        return;
    }

    if (warp == NCW + 1) {
        // ------------------------------------------------------------ epilogue warp
        // Items of one column block: once the last consumer warp has handed the item over,
        // reduce its shared-memory partials in a fixed order, release the queue slot, then do
        // the item's global work (h rows and the tile count, or the pair's output rows and the
        // slot-order combine) while the consumers already work on the next items.
        uint32_t epi_phase = 0; // bit qs: parity of the next phase of epi[qs] (only handed-over items use it)
        for (int qi = 0;; ++qi) {
            const int qs = qi % QDEPTH;
            if (!pipe::mbar_wait_tight(&S.qfull[qs], (qi / QDEPTH) & 1, deadline)) {
                set_error(W, kErrTimeout, 7);
                break;
            }
            const Desc d = S.q[qs];
            if (d.kind == 2)
                break;
            const int blk0 = V.blk0(d.u);
            if (V.nblk(d.u) != 1) {
                // several column blocks: the consumers' last warp does it through global memory
                __syncwarp();
                if (lane == 0)
                    pipe::mbar_arrive(&S.qempty[qs]);
                continue;
            }
            if (!pipe::mbar_wait_tight(&S.epi[qs], (epi_phase >> qs) & 1u, deadline)) {
                set_error(W, kErrTimeout, 8);
                break;
            }
            epi_phase ^= 1u << qs;
            const int nmem = V.bnmem(blk0);
            if (d.kind == 0) {
                // h rows: lanes 0-15 = row, one value per member
                const int rr = lane & 15;
                float hv[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float gv = 0.0f, uv = 0.0f;
                    if (c < nmem) {
#pragma unroll
                        for (int kq = 0; kq < 8; ++kq) {
                            gv += S.red[qs][kq][rr * 4 + c];
                            uv += S.red[qs][8 + kq][rr * 4 + c];
                        }
                    }
                    hv[c] = gv / (1.0f + expf(-gv)) * uv;
                }
                __syncwarp();
                if (lane == 0)
                    pipe::mbar_arrive(&S.qempty[qs]);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (c < nmem && lane < 16)
                        __stcg(W.h + (int64_t)V.bpair(blk0, c) * I + 16 * d.strip + rr, hv[c]);
                gateup_tile_done(W, V, I, d.u, d.strip, blk0, 1);
            } else {
                // output rows: lane owns rows lane + 32*i
                float ov[4][4];
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = lane + 32 * i, s8 = r >> 4, rr = r & 15;
                        ov[c][i] = c < nmem ? S.red[qs][2 * s8][rr * 4 + c] + S.red[qs][2 * s8 + 1][rr * 4 + c] : 0.0f;
                    }
                __syncwarp();
                if (lane == 0)
                    pipe::mbar_arrive(&S.qempty[qs]);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (c < nmem) {
                        const int pair = V.bpair(blk0, c);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            __stcg(W.part + (int64_t)pair * H + 128 * d.strip + lane + 32 * i, ov[c][i]);
                    }
                for (int c = 0; c < nmem; ++c)
                    down_rows_done(a, V.bpair(blk0, c), d.strip);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int g = lane >> 2, t = lane & 3;
    for (int qi = 0;; ++qi) {
        const int qs = qi % QDEPTH;
        if (!pipe::mbar_wait_tight(&S.qfull[qs], (qi / QDEPTH) & 1, deadline)) {
            set_error(W, kErrTimeout, 3);
            break;
        }
        const Desc d = S.q[qs];
        if (d.kind == 2)
            break;
        const int blk0 = V.blk0(d.u);
        const int nblk = V.nblk(d.u), bmax = V.bmax(d.u);
        const bool fast = (nblk == 1);
        float *red = S.red[qs][warp];
        bool fine = true;
        const int cm = d.c0 + bmax; // meta chunk (after the item's planes)
        const unsigned char *meta = S.ring[cm % NSLOT];
        if (!pipe::mbar_wait_tight(&S.ifull[qs], (qi / QDEPTH) & 1, deadline)) // the item's bytes
            fine = false;

        // The warp's share of the item: tpw tiles from K tile Q0 of 16 rows (tiles tix0.. of every
        // plane chunk). Gate/up: warp -> matrix m (warps 0-7 gate, 8-15 up) and K part kp (of 8) of
        // the item's 16 rows (a plane chunk holds [gate rows | up rows] of one plane); down: warp ->
        // strip sb (of 8 x 16 rows) and K part kp (of 2). Both kinds share one decode call per
        // fragment source, so that the decode code of a depth exists once.
        const bool up = d.kind == 0;
        const int m = up ? warp >> 3 : 2, sb = up ? 0 : warp >> 1, kp = up ? (warp & 7) : (warp & 1);
        const int tpw = up ? (H / 128) / 8 : (I / 128) / 2, Q0 = kp * tpw;
        const int tix0 = (up ? m * (H / 128) : sb * (I / 128)) + Q0;
        const int ngr = (up ? H : I) / G;
        if (!up && !fast && lane == 0) {
            while (pipe::ld_acquire(&W.readyB[d.u]) < I / 128) {
                if (pipe::globaltimer() > deadline) {
                    fine = false;
                    break;
                }
                __nanosleep(256);
            }
        }
        fine = __shfl_sync(0xffffffffu, (int)fine, 0) != 0;
        __syncwarp();
        const unsigned char *pp[8];
#pragma unroll
        for (int p = 0; p < 8; ++p)
            pp[p] = S.ring[(d.c0 + p) % NSLOT] + tix0 * 256 + lane * 8;
        // meta chunk: scale rows (gate/up [16 gate | 16 up] rows, down 128 rows) x ngr groups, then the
        // table heads (gate/up: gate and up per block; down: one per block), then (down items of one
        // block) the members' h fragments and exponents
        const float *sc0 = reinterpret_cast<const float *>(meta) + (up ? m * 16 + g : 16 * sb + g) * ngr + Q0 * (128 / G);
        const float *sc1 = sc0 + 8 * ngr;
        const unsigned char *tab0 = meta + (up ? 2 * 16 : 128) * ngr * 4;
        for (int bi = 0; bi < nblk; ++bi) {
            const int blk = blk0 + bi;
            const int dd = V.bdepth(blk), nmem = V.bnmem(blk);
            // B column g = 4*c + part: byte part of token c (part 3 and absent tokens: zero);
            // lane t accumulates token t/2 (xfrag.cuh, dev::combine24)
            const int c = g >> 2, part = g & 3, me = t >> 1;
            const bool has = c < nmem && part < 3;
            float acc0 = 0.0f, acc1 = 0.0f;
            const unsigned char *tabs = tab0 + (up ? bi * 2 + m : bi) * TAB_BYTES;
            const uint32_t *big = W.tabs + ((int64_t)blk * 3 + m) * kTabWords + 16;
            const uint32_t *fptr = nullptr;
            const int *exps = nullptr;
            int fstep = KFW, fm;
            if (up && stage_x) {
                fm = 0;
                fptr = has ? S.xs + Q0 * 4 * KFW + dev::frag_offset(part, t) : S.zeros;
                fstep = has ? KFW : 0;
                if (me < nmem)
                    exps = S.xse;
            } else if (up) {
                fm = 1;
                if (has)
                    fptr = W.xfrag + ((int64_t)(V.bpair(blk, c) / k) * (H / 32) + Q0 * 4) * KFW + dev::frag_offset(part, t);
                if (me < nmem)
                    exps = W.xexp + (int64_t)(V.bpair(blk, me) / k) * (H / 128);
            } else if (fast) {
                // h fragments and exponents of the members arrived with the meta chunk
                fm = 0;
                const uint32_t *hf = reinterpret_cast<const uint32_t *>(tab0 + TAB_BYTES);
                const int *he = reinterpret_cast<const int *>(hf + nmem * (I / 32) * KFW);
                fptr = has ? hf + ((int64_t)c * (I / 32) + Q0 * 4) * KFW + dev::frag_offset(part, t) : S.zeros;
                fstep = has ? KFW : 0;
                if (me < nmem)
                    exps = he + me * hexp_stride(I);
            } else {
                fm = 2;
                if (has)
                    fptr = W.hfrag + ((int64_t)V.bpair(blk, c) * (I / 32) + Q0 * 4) * KFW + dev::frag_offset(part, t);
                if (me < nmem)
                    exps = W.hexp + (int64_t)V.bpair(blk, me) * hexp_stride(I);
            }
            if (fm == 0)
                warp_block_any<GS, 0>(dd, pp, tpw, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1);
            else if (fm == 1)
                warp_block_any<GS, 1>(dd, pp, tpw, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1);
            else
                warp_block_any<GS, 2>(dd, pp, tpw, Q0, tabs, big, fptr, fstep, exps, sc0, sc1, acc0, acc1);
            if ((t & 1) == 0 && me < nmem) {
                if (fast) {
                    red[g * 4 + me] = acc0;
                    red[(g + 8) * 4 + me] = acc1;
                } else {
                    const int pair = V.bpair(blk, me);
                    float *dst = up ? W.pA + (((int64_t)pair * (I / 16) + d.strip) * 8 + kp) * 32 + m * 16
                                    : W.pB + (((int64_t)pair * (H / 16) + 8 * d.strip + sb) * 2 + kp) * 16;
                    __stcg(dst + g, acc0);
                    __stcg(dst + g + 8, acc1);
                }
            }
        }
        __syncwarp();
        int last = 0;
        if (fast) {
            // the epilogue warp reduces the partials; the last warp only hands the item over
            if (lane == 0) {
                __threadfence_block();
                if (atomicAdd(&S.cnt[qs], 1) == NCW - 1) {
                    S.cnt[qs] = 0;
                    pipe::mbar_arrive(&S.epi[qs]);
                }
            }
        } else if (lane == 0) {
            last = (atom_add_acq_rel(up ? &W.cntA[d.u * SA + d.strip] : &W.cntB[d.u * SB + d.strip], 1) == NCW - 1);
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        __syncwarp();
        if (last && up) {
            // h rows of the item: lanes 0-15 = row, every member of every block
            for (int bi = 0; bi < nblk; ++bi) {
                const int blk = blk0 + bi, nmem = V.bnmem(blk);
                for (int c = 0; c < nmem; ++c) {
                    const int pair = V.bpair(blk, c);
                    const int rr = lane & 15;
                    float gv = 0.0f, uv = 0.0f;
                    const float *src = W.pA + (((int64_t)pair * (I / 16) + d.strip) * 8) * 32;
#pragma unroll
                    for (int kq = 0; kq < 8; ++kq) {
                        gv += __ldcg(src + kq * 32 + rr);
                        uv += __ldcg(src + kq * 32 + 16 + rr);
                    }
                    if (lane < 16)
                        __stcg(W.h + (int64_t)pair * I + 16 * d.strip + rr, gv / (1.0f + expf(-gv)) * uv);
                }
            }
            gateup_tile_done(W, V, I, d.u, d.strip, blk0, nblk);
        } else if (last) {
            for (int bi = 0; bi < nblk; ++bi) {
                const int blk = blk0 + bi, nmem = V.bnmem(blk);
                for (int c = 0; c < nmem; ++c) {
                    const int pair = V.bpair(blk, c);
                    for (int r = lane; r < 128; r += 32) {
                        const int s8 = r >> 4, rr = r & 15;
                        const float *src = W.pB + (((int64_t)pair * (H / 16) + 8 * d.strip + s8) * 2) * 16;
                        __stcg(W.part + (int64_t)pair * H + 128 * d.strip + r, __ldcg(src + rr) + __ldcg(src + 16 + rr));
                    }
                }
            }
            for (int bi = 0; bi < nblk; ++bi) {
                const int blk = blk0 + bi, nmem = V.bnmem(blk);
                for (int c = 0; c < nmem; ++c)
                    down_rows_done(a, V.bpair(blk, c), d.strip);
            }
        }
        __syncwarp();
        if (lane == 0)
            pipe::mbar_arrive(&S.qempty[qs]);
        if (!fine) {
            set_error(W, kErrTimeout, 4);
            break;
        }
    }
}

} // namespace mk
