// Batch-1 MoE layer on bitplane prefixes in one launch (PagedMoE transcript
// cues 4, 29, 35, 37; arxivlens Abstract and Methodology): routing and prefix
// selection, gate/up prefix GEMV + SwiGLU, down prefix GEMV and the
// routing-weighted combine for one token.
//
// One CTA per SM. Every CTA routes the token itself (the same deterministic
// result everywhere), so no kernel runs before this one. The k routed experts
// ("units") are ordered deepest first and split into two halves P and Q of
// about equal gate/up cost. The work is cut into items of 16 rows x 256 (gate
// and up) or 16 rows x 512 (down) weights, 8K weights each, in four sets
// processed in this order by every CTA:
//     A(P)  gate/up of P,   A(Q)  gate/up of Q,   B(P)  down of P,   B(Q)  down of Q.
// Each set is cut into one contiguous, cost-balanced range per CTA, so all
// CTAs move through the sets together: the down items of P start after every
// CTA has gone through the gate/up items of Q, long after h of P is complete,
// and likewise for Q. A CTA's items are grouped into regions (consecutive
// items of one row block of gate/up, or of one unit's down matrix, up to about
// 48 KB), and the schedule, the regions and their places in the shared-memory
// ring are a deterministic function of the routing result, computed by every
// warp that needs them.
//
// Warps: 16 consumers, a producer, an epilogue warp and an h stager.
//  * Producer: streams each region's plane tiles (one 1-D bulk copy per plane
//    and matrix) and scale rows into the ring; all land on the region slot's
//    "full" mbarrier. It reuses ring bytes once the epilogue has released them.
//  * Consumers: item i of the CTA's stream goes to warp i % 16. A warp decodes
//    the item's tiles of every plane it needs (planes 0..b-1 only, cue 25)
//    into int8 high/low bytes of the 16-bit fixed-point tree values with byte
//    permutes, multiplies them with mma.sync m16n8k32 (s8) against the
//    activation's high/low bytes, sums exactly in int32 per scale group and
//    scales in float; it leaves 16 row sums per item in shared memory and
//    marks the region consumed once it is past it.
//  * Epilogue: reduces each region's item sums in item order. A complete row
//    block of gate/up becomes 16 rows of h = silu(g) * u; the last row block
//    of a 128-row tile of h turns the tile into MMA fragments (one power-of-two
//    exponent per tile) and publishes it. A complete row block of down is one
//    expert's contribution to 16 output rows; the last expert to finish those
//    rows sums the k contributions into y in slot order (deterministic).
//    Row blocks whose K range is split between CTAs (at range boundaries) meet
//    through partial sums in the workspace, summed in K order by whichever
//    piece completes them.
//  * Stager: waits (bounded) until every h tile of a unit the CTA's down items
//    use is published, then copies the unit's h fragments into shared memory.
// Every wait is bounded by one deadline per launch; a wait that runs out
// records an error and the CTA stops work, waits (with a separate, long
// limit) for its own copies in flight, and exits.
// Counters: CTA 0 zeroes the call's counters and flags, builds the decode
// tables of depth >= 5 in the workspace, then publishes a "go" word tagged
// with the call's epoch; nothing else touches counters before it sees it.
// The last CTA to finish advances the epoch.
#include <cuda_bf16.h>

#include "common.h"
#include "dev.cuh"
#include "layer.cuh"
#include "pipe.cuh"
#include "route.cuh"
#include "xfrag.cuh"

namespace pmoe {
namespace d1 {

using dev::RegTab;

constexpr int NCW = 16;                     // consumer warps
constexpr int W_PROD = NCW, W_EPI = NCW + 1, W_STG = NCW + 2;
constexpr int NTHREADS = (NCW + 3) * 32;
constexpr int NREG = 8;                     // region slots
constexpr int RING = 164 * 1024;            // ring bytes
constexpr int REG_CAP = 48 * 1024;          // target bytes per region
constexpr int MAXI = 16;                    // items per region
constexpr int MAXU = 32;                    // units (k)
constexpr int HSLOTS = 4;                   // units whose h a CTA's down items read
constexpr int KGA = 2;                      // k-tiles per gate/up item
constexpr int HMAX = 4096, IMAX = 1024;
constexpr uint64_t kDrainNs = 1000ull * 1000 * 1000; // limit for waiting on one's own copies at exit

struct TabS {                               // register table of one (unit, matrix) in shared memory
    uint32_t h[4], l[4];
    int f;
    uint32_t c1;                            // C[1][1] bits (depth-1 sign path)
    uint32_t anti;                          // depth-1 table is antisymmetric
    uint32_t pad;
};

struct Smem {
    alignas(128) unsigned char ring[RING];
    float red[NREG][MAXI][32];
    alignas(16) uint32_t xs[(HMAX / 32) * 16];
    alignas(16) uint32_t hs[HSLOTS][(IMAX / 32) * 16];
    alignas(16) int xse[HMAX / 128];
    alignas(16) int hse[HSLOTS][IMAX / 128];
    TabS tab[MAXU][3];
    // routing result per slot, and units (order: depth desc, slot asc)
    int s_e[MAXU], s_b[MAXU];
    float s_w[MAXU];
    int u_slot[MAXU];                       // unit -> routing slot
    int u_ps[MAXU][8];                      // plane slots of the unit's expert
    int hslot_of[MAXU];
    // sets: units, item offsets, this CTA's range
    int setN[4], setU[4][MAXU], setStart[4][MAXU + 1], lo[4], hi[4];
    int nitems;                             // items in this CTA's stream
    int bad;                                // nonzero: invalid routing input (no work is done)
    int missing;                            // >= 0: e*8 + p of a needed plane without a slot
    uint64_t full[NREG], consumed[NREG], freeb[NREG], hfull[HSLOTS];
};
static_assert(sizeof(Smem) <= 227 * 1024, "shared memory of the batch-1 kernel exceeds one SM's");

struct Args {
    pmoe_layer L;
    const float *logits; // decode step (else nullptr: ids/w/depth are inputs)
    const float *sens;
    const uint16_t *x;
    int32_t *ids;
    float *w;
    uint8_t *depth;
    int k, B;
    float *y;
    LayerWs W;
    uint64_t limit_ns;
};

// error codes (as layer.cu)
constexpr int kErrBadPair = 1, kErrNoPlane = 2, kErrTimeout = 3, kErrUnsupported = 4;

__device__ __forceinline__ uint32_t epoch_tag(uint32_t seq) { return seq * 0x9E3779B1u + 0x7F4A7C15u; }

// Waits (bounded) for CTA 0's "go" word of this call's epoch.
__device__ bool wait_go(const LayerWs &W, uint32_t tag, uint64_t deadline)
{
    while ((uint32_t)pipe::ld_acquire(&W.flags[kFlagGo]) != tag) {
        if (pipe::globaltimer() > deadline)
            return false;
        __nanosleep(128);
    }
    return true;
}

__device__ void set_error(const LayerWs &W, uint32_t tag, uint64_t deadline, int code, int where)
{
    wait_go(W, tag, deadline + 1000000ull); // errors are kept only once the call's record is reset
    if (atomicCAS(&W.flags[kFlagError], 0, code) == 0)
        W.flags[kFlagWhere] = where;
}

__device__ __forceinline__ int atom_add_acq_rel(int *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ float pow2neg(int e) { return __int_as_float((127 - e) << 23); }

__device__ __forceinline__ float combine256(int dh0, int dh1, int dl0, int dl1)
{
    return (float)(dh0 * 256 + dh1 + dl0 + ((dl1 + 128) >> 8));
}

// ---------------------------------------------------------------- schedule

struct Geo {
    int H, I, G, NKA, NKB, KGB, k, nblk;
    __device__ int items_A() const { return (I / 16) * NKA; }
    __device__ int items_B() const { return (H / 16) * NKB; }
};

// relative cost of one item of depth b (plane bytes + a constant for decode work)
__device__ __forceinline__ int64_t item_cost(int b) { return 1024 * b + 2560; }

// Region of the CTA's stream (see RegionIter).
struct Region {
    int set, u, local, n, i0, off, bytes;
};

// Walks this CTA's regions in stream order, with their ring offsets.
struct RegionIter {
    const Smem &S;
    const Geo &g;
    int set, idx, i0, head;
    __device__ RegionIter(const Smem &s, const Geo &gg) : S(s), g(gg), set(0), idx(s.lo[0]), i0(0), head(0) {}
    // items per gate/up region: a row block split into equal pieces that fit the target
    __device__ int capA(int b) const
    {
        int n = (REG_CAP - 2 * 16 * (g.H / g.G) * 4) / (2 * b * KGA * 256);
        n = n < 1 ? 1 : (n > MAXI ? MAXI : n);
        const int pieces = (g.NKA + n - 1) / n;
        return (g.NKA + pieces - 1) / pieces;
    }
    // items per down region: whole row blocks when they fit
    __device__ int capB(int b) const
    {
        int n = REG_CAP / (b * g.KGB * 256 + 16 * (g.I / g.G) * 4 / g.NKB);
        n = n < 1 ? 1 : (n > MAXI ? MAXI : n);
        return n >= g.NKB ? n - n % g.NKB : n;
    }
    __device__ bool next(Region &r)
    {
        while (set < 4 && idx >= S.hi[set]) {
            ++set;
            if (set < 4)
                idx = S.lo[set];
        }
        if (set >= 4)
            return false;
        int p = 0;
        while (S.setStart[set][p + 1] <= idx)
            ++p;
        const int u = S.setU[set][p];
        const int b = S.s_b[S.u_slot[u]];
        const int local = idx - S.setStart[set][p];
        int n, bytes;
        if (set < 2) {
            const int kg = local % g.NKA;
            n = g.NKA - kg;
            n = min(n, S.hi[set] - idx);
            n = min(n, capA(b));
            bytes = 2 * b * n * KGA * 256 + 2 * 16 * (g.H / g.G) * 4;
        } else {
            n = S.setStart[set][p + 1] - idx;
            n = min(n, S.hi[set] - idx);
            n = min(n, capB(b));
            const int rb0 = local / g.NKB, rb1 = (local + n - 1) / g.NKB;
            bytes = b * n * g.KGB * 256 + (rb1 - rb0 + 1) * 16 * (g.I / g.G) * 4;
        }
        if (head + bytes > RING)
            head = 0;
        r.set = set;
        r.u = u;
        r.local = local;
        r.n = n;
        r.i0 = i0;
        r.off = head;
        r.bytes = bytes;
        head += bytes;
        i0 += n;
        idx += n;
        return true;
    }
};

// Boundary of CTA c in a set: the first item whose cumulative cost reaches c/nc of the total.
__device__ int set_boundary(const Smem &S, int set, const int64_t *ucost, int64_t total, int c, int nc)
{
    if (c >= nc)
        return S.setStart[set][S.setN[set]];
    const int64_t target = (total * c) / nc;
    int64_t before = 0;
    for (int p = 0; p < S.setN[set]; ++p) {
        const int n = S.setStart[set][p + 1] - S.setStart[set][p];
        const int64_t cu = ucost[S.setU[set][p]];
        if (target <= before + cu * n) {
            const int64_t j = (target - before + cu - 1) / cu;
            return S.setStart[set][p] + (int)j;
        }
        before += cu * n;
    }
    return S.setStart[set][S.setN[set]];
}

// ---------------------------------------------------------------- consumer tiles

// One 16x128 tile of one matrix at depth B: rows g, g+8 of this lane accumulate
// sum over the tile's groups of int32 group sum * scale * fac.
//  pl: plane 0 of the tile + 8*lane bytes; pstep: bytes between planes.
//  xf: B fragments of the tile's first k-step for this lane (uint2 per k-step, 16 words apart).
//  sc0/sc1: scale rows g / g+8 at the tile's first group.
template <int B, int GS>
__device__ __forceinline__ void tile_dot(const unsigned char *pl, int pstep, const RegTab &tab, const uint32_t *big,
                                         const uint32_t *xf, const float *sc0, const float *sc1, float fac,
                                         float &acc0, float &acc1)
{
    uint32_t w[8][2];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        w[p][0] = w[p][1] = 0u;
        if (p < B) {
            const uint2 v = *reinterpret_cast<const uint2 *>(pl + p * pstep);
            w[p][0] = v.x;
            w[p][1] = v.y;
        }
    }
    int dh[4] = {0, 0, 0, 0}, dl[4] = {0, 0, 0, 0};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t ah[4], al[4];
        dev::decode_kstep<B>(w, s, tab, big, ah, al);
        const uint2 bv = *reinterpret_cast<const uint2 *>(xf + s * 16);
        dev::mma_s8(dh, ah, bv.x, bv.y);
        dev::mma_s8(dl, al, bv.x, bv.y);
        if ((s + 1) % GS == 0) {
            const int gi = s / GS;
            acc0 = __fmaf_rn(combine256(dh[0], dh[1], dl[0], dl[1]), sc0[gi] * fac, acc0);
            acc1 = __fmaf_rn(combine256(dh[2], dh[3], dl[2], dl[3]), sc1[gi] * fac, acc1);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dh[i] = dl[i] = 0;
        }
    }
}

// Depth 1 of an antisymmetric table: +-1 bytes, one MMA per k-step; fac includes C[1][1].
template <int GS>
__device__ __forceinline__ void tile_dot_sign(const unsigned char *pl, const uint32_t *xf, const float *sc0,
                                              const float *sc1, float fac, float &acc0, float &acc1)
{
    uint32_t w[8][2];
    const uint2 v = *reinterpret_cast<const uint2 *>(pl);
    w[0][0] = v.x;
    w[0][1] = v.y;
    int dh[4] = {0, 0, 0, 0};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t a[4];
        dev::decode_kstep_sign(w, s, a);
        const uint2 bv = *reinterpret_cast<const uint2 *>(xf + s * 16);
        dev::mma_s8(dh, a, bv.x, bv.y);
        if ((s + 1) % GS == 0) {
            const int gi = s / GS;
            acc0 = __fmaf_rn((float)(dh[0] * 256 + dh[1]), sc0[gi] * fac, acc0);
            acc1 = __fmaf_rn((float)(dh[2] * 256 + dh[3]), sc1[gi] * fac, acc1);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dh[i] = 0;
        }
    }
}

__device__ __forceinline__ void load_tab(const TabS &t, RegTab &r)
{
    const uint4 a = *reinterpret_cast<const uint4 *>(t.h);
    const uint4 b = *reinterpret_cast<const uint4 *>(t.l);
    r.h[0] = a.x; r.h[1] = a.y; r.h[2] = a.z; r.h[3] = a.w;
    r.l[0] = b.x; r.l[1] = b.y; r.l[2] = b.z; r.l[3] = b.w;
    r.f = t.f;
}

// ntiles consecutive tiles (k-tiles kt0..) of one matrix at depth B.
template <int B, int GS>
__device__ __forceinline__ void tiles_dot(int ntiles, const unsigned char *pl, int pstep, const TabS &ts,
                                          const uint32_t *big, const uint32_t *xf, const int *xe, int kt0,
                                          const float *sc0, const float *sc1, int gpt, float &acc0, float &acc1)
{
    if constexpr (B == 1) {
        if (ts.anti) {
            const float c1 = __uint_as_float(ts.c1);
            for (int j = 0; j < ntiles; ++j)
                tile_dot_sign<GS>(pl + j * 256, xf + (kt0 + j) * 64, sc0 + j * gpt, sc1 + j * gpt,
                                  c1 * pow2neg(xe[kt0 + j]), acc0, acc1);
            return;
        }
    }
    RegTab tab;
    load_tab(ts, tab);
    for (int j = 0; j < ntiles; ++j)
        tile_dot<B, GS>(pl + j * 256, pstep, tab, big, xf + (kt0 + j) * 64, sc0 + j * gpt, sc1 + j * gpt,
                        256.0f * pow2neg(tab.f + xe[kt0 + j]), acc0, acc1);
}

template <int GS>
__device__ __forceinline__ void tiles_any(int b, int ntiles, const unsigned char *pl, int pstep, const TabS &ts,
                                          const uint32_t *big, const uint32_t *xf, const int *xe, int kt0,
                                          const float *sc0, const float *sc1, int gpt, float &acc0, float &acc1)
{
    switch (b) {
    case 1: tiles_dot<1, GS>(ntiles, pl, pstep, ts, big, xf, xe, kt0, sc0, sc1, gpt, acc0, acc1); break;
    case 2: tiles_dot<2, GS>(ntiles, pl, pstep, ts, big, xf, xe, kt0, sc0, sc1, gpt, acc0, acc1); break;
    case 3: tiles_dot<3, GS>(ntiles, pl, pstep, ts, big, xf, xe, kt0, sc0, sc1, gpt, acc0, acc1); break;
    case 4: tiles_dot<4, GS>(ntiles, pl, pstep, ts, big, xf, xe, kt0, sc0, sc1, gpt, acc0, acc1); break;
    case 5: tiles_dot<5, GS>(ntiles, pl, pstep, ts, big, xf, xe, kt0, sc0, sc1, gpt, acc0, acc1); break;
    case 6: tiles_dot<6, GS>(ntiles, pl, pstep, ts, big, xf, xe, kt0, sc0, sc1, gpt, acc0, acc1); break;
    case 7: tiles_dot<7, GS>(ntiles, pl, pstep, ts, big, xf, xe, kt0, sc0, sc1, gpt, acc0, acc1); break;
    default: tiles_dot<8, GS>(ntiles, pl, pstep, ts, big, xf, xe, kt0, sc0, sc1, gpt, acc0, acc1); break;
    }
}

// ---------------------------------------------------------------- epilogue helpers

// Converts 128 rows of h (tile q of unit u) into B fragments and publishes the tile.
__device__ void h_tile_to_frags(const LayerWs &W, int I, int u, int q)
{
    const int lane = threadIdx.x & 31;
    const float4 f = __ldcg(reinterpret_cast<const float4 *>(W.h + (int64_t)u * I + 128 * q + 4 * lane));
    float v[4] = {f.x, f.y, f.z, f.w};
    float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    m = dev::warp_max(m);
    const int sx = dev::fix_exponent(m);
    uint32_t ph = 0u, pl = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int hi, lo;
        dev::split16(__float2int_rn(ldexpf(v[i], sx)), hi, lo);
        ph |= (uint32_t)(hi & 0xff) << (8 * i);
        pl |= (uint32_t)(lo & 0xff) << (8 * i);
    }
    const int s = lane >> 3, o = lane & 7, t = o & 3, reg = o >> 2;
    uint32_t *xf = W.hfrag + (int64_t)u * (I / 32) * 16;
    __stcg(xf + ((q * 4 + s) * 8 + t) * 2 + reg, ph);
    __stcg(xf + ((q * 4 + s) * 8 + 4 + t) * 2 + reg, pl);
    if (lane == 0)
        __stcg(W.hexp + (int64_t)u * hexp_stride(I) + q, sx);
    __syncwarp();
    __threadfence();
    __syncwarp();
    if (lane == 0)
        pipe::st_release(&W.readyH[(int64_t)u * (I / 128) + q], 1);
}

// ---------------------------------------------------------------- kernel

template <int GS>
__global__ void __launch_bounds__(NTHREADS, 1) decode1_kernel(Args a)
{
    extern __shared__ __align__(128) unsigned char smraw[];
    Smem &S = *reinterpret_cast<Smem *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const pmoe_layer &L = a.L;
    const LayerWs &W = a.W;
    const int H = L.H, I = L.I, G = L.G, k = a.k, E = L.E;
    const uint64_t t_start = pipe::globaltimer();
    const uint64_t deadline = t_start + a.limit_ns;
    const uint32_t seq = (uint32_t)*reinterpret_cast<volatile int *>(&W.flags[kFlagSeq]);
    const uint32_t tag = epoch_tag(seq);

    Geo g;
    g.H = H;
    g.I = I;
    g.G = G;
    g.NKA = H / (128 * KGA);
    g.KGB = ((I / 128) % 4 == 0) ? 4 : (((I / 128) % 2 == 0) ? 2 : 1);
    g.NKB = (I / 128) / g.KGB;
    g.k = k;

    // ---- setup 1: routing (warp 0); x fragments and barriers (other warps)
    if (warp == 0) {
        int id = 0, b = 1;
        float wt = 0.0f;
        if (a.logits != nullptr) {
            if (E <= 512)
                dev::route_token_reg<16>(a.logits, E, k, id, wt);
            else
                dev::route_token(a.logits, E, k, reinterpret_cast<float *>(S.ring), id, wt);
            const float v = (lane < k) ? __fmul_rn(wt, __ldg(a.sens + id)) : 0.0f;
            b = dev::select_token(v, k, a.B, nullptr);
        } else if (lane < k) {
            id = __ldg(a.ids + lane);
            wt = __ldg(a.w + lane);
            b = __ldg(a.depth + lane);
        }
        const bool badl = lane < k && (id < 0 || id >= E || b < 1 || b > 8);
        const unsigned badm = __ballot_sync(0xffffffffu, badl);
        if (lane < k) {
            S.s_e[lane] = badl ? 0 : id;
            S.s_b[lane] = badl ? 1 : b;
            S.s_w[lane] = wt;
        }
        if (lane == 0) {
            S.bad = badm != 0u;
            S.missing = -1;
        }
        if (blockIdx.x == 0 && a.logits != nullptr && lane < k) {
            a.ids[lane] = id;
            a.w[lane] = wt;
            a.depth[lane] = (uint8_t)b;
        }
    } else {
        for (int Q = warp - 1; Q < H / 128; Q += (NTHREADS / 32) - 1)
            dev::make_xfrag_tile<true>(a.x, Q, S.xs, S.xse);
        if (tid == 32) {
            for (int s = 0; s < NREG; ++s) {
                pipe::mbar_init(&S.full[s], 1);
                pipe::mbar_init(&S.consumed[s], NCW);
                pipe::mbar_init(&S.freeb[s], 1);
            }
            for (int s = 0; s < HSLOTS; ++s)
                pipe::mbar_init(&S.hfull[s], 1);
            pipe::fence_barrier_init();
        }
    }
    __syncthreads();

    // ---- setup 2: schedule (warp 0); tables, plane slots, CTA 0's resets (other warps)
    if (warp == 0) {
        // unit order: depth descending, slot ascending (rank by comparison)
        if (lane < k) {
            const int b = S.s_b[lane];
            int rank = 0;
            for (int j = 0; j < k; ++j) {
                const int bj = S.s_b[j];
                rank += (bj > b || (bj == b && j < lane)) ? 1 : 0;
            }
            S.u_slot[rank] = lane;
        }
        __syncwarp();
        if (lane == 0) {
            int64_t costA[MAXU], costB[MAXU];
            int64_t totA = 0;
            for (int u = 0; u < k; ++u) {
                const int b = S.s_b[S.u_slot[u]];
                costA[u] = item_cost(b);
                costB[u] = item_cost(b);
                totA += costA[u] * g.items_A();
            }
            // P: the shortest prefix of units with at least half the gate/up cost (Q keeps one unit)
            int np = 0;
            int64_t acc = 0;
            while (np < k && 2 * acc < totA) {
                acc += costA[np] * g.items_A();
                ++np;
            }
            if (np == k && k > 1)
                np = k - 1;
            for (int s = 0; s < 4; ++s) {
                const int u0 = (s == 0 || s == 2) ? 0 : np, u1 = (s == 0 || s == 2) ? np : k;
                S.setN[s] = u1 - u0;
                S.setStart[s][0] = 0;
                for (int p = 0; p < u1 - u0; ++p) {
                    S.setU[s][p] = u0 + p;
                    S.setStart[s][p + 1] = S.setStart[s][p] + (s < 2 ? g.items_A() : g.items_B());
                }
                const int64_t *uc = s < 2 ? costA : costB;
                int64_t tot = 0;
                for (int p = 0; p < u1 - u0; ++p)
                    tot += uc[u0 + p] * (S.setStart[s][p + 1] - S.setStart[s][p]);
                S.lo[s] = set_boundary(S, s, uc, tot, (int)blockIdx.x, (int)gridDim.x);
                S.hi[s] = set_boundary(S, s, uc, tot, (int)blockIdx.x + 1, (int)gridDim.x);
            }
            int n = 0;
            for (int s = 0; s < 4; ++s)
                n += S.hi[s] - S.lo[s];
            S.nitems = n;
            // h slots: units of the CTA's down items, in stream order
            for (int u = 0; u < MAXU; ++u)
                S.hslot_of[u] = -1;
            int nh = 0;
            for (int s = 2; s < 4; ++s)
                for (int p = 0; p < S.setN[s]; ++p)
                    if (S.lo[s] < S.setStart[s][p + 1] && S.hi[s] > S.setStart[s][p]) {
                        const int u = S.setU[s][p];
                        if (S.hslot_of[u] < 0)
                            S.hslot_of[u] = nh < HSLOTS ? nh++ : HSLOTS;
                    }
        }
    } else {
        const int wi = warp - 1, nw = (NTHREADS / 32) - 1;
        // decode tables, one warp per (slot, matrix); CTA 0 also writes the depth >= 5 tables
        for (int j = wi; j < k * 3; j += nw) {
            const int sl = j / 3, m = j % 3, e = S.s_e[sl], b = S.s_b[sl];
            const float *cb = L.codebooks + ((int64_t)e * 3 + m) * 510;
            uint32_t *big = (blockIdx.x == 0 && b >= 5) ? W.tabs + ((int64_t)sl * 3 + m) * kTabWords + 16 : nullptr;
            RegTab t;
            dev::build_tab(cb, b, t, big);
            if (lane == 0) {
                TabS &d = S.tab[sl][m];
                for (int r = 0; r < 4; ++r) {
                    d.h[r] = t.h[r];
                    d.l[r] = t.l[r];
                }
                d.f = t.f;
                const float c0 = __ldg(cb), c1 = __ldg(cb + 1);
                d.c1 = __float_as_uint(c1);
                d.anti = (c0 == -c1) ? 1u : 0u;
            }
        }
        // plane slots of every routed expert; a needed plane without one is an error of the call
        for (int j = tid - 32; j < k * 8; j += NTHREADS - 32) {
            const int sl = j / 8, p = j % 8;
            const int ps = __ldg(L.slot_of + S.s_e[sl] * 8 + p);
            S.u_ps[sl][p] = ps;
            if (ps < 0 && p < S.s_b[sl])
                atomicMax(&S.missing, S.s_e[sl] * 8 + p);
        }
        if (blockIdx.x == 0) {
            const int t0 = tid - 32, nt = NTHREADS - 32;
            for (int i = t0; i < k * (I / 16); i += nt)
                W.cntA[i] = 0;
            for (int i = t0; i < k * (I / 128); i += nt) {
                W.cntH[i] = 0;
                W.readyH[i] = 0;
            }
            for (int i = t0; i < k * (H / 16); i += nt)
                W.cntB1[i] = 0;
            for (int i = t0; i < H / 16; i += nt)
                W.ycnt1[i] = 0;
            if (t0 == 0) {
                W.flags[kFlagError] = 0;
                W.flags[kFlagWhere] = 0;
                W.flags[kFlagDone] = 0;
            }
        }
    }
    __syncthreads();
    if (blockIdx.x == 0 && tid == 0) {
        __threadfence();
        pipe::st_release(&W.flags[kFlagGo], (int)tag);
    }
    if (S.bad || S.missing >= 0) {
        // no work: record the error once; the epoch still advances below
        if (blockIdx.x == 0 && tid == 0)
            set_error(W, tag, deadline, S.bad ? kErrBadPair : kErrNoPlane, S.bad ? 0 : S.missing);
    } else if (warp == W_PROD) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const float *scales = L.scales;
            const int64_t mat_words = (int64_t)H * I / 32;
            const int64_t escale_len = 2 * (int64_t)I * (H / G) + (int64_t)H * (I / G);
            RegionIter it(S, g);
            Region r;
            int nr = 0, ft = 0;
            int roff[NREG], rbytes[NREG];
            bool ok = true;
            while (ok && it.next(r)) {
                // slot reuse and ring bytes: wait for the epilogue to release older regions
                if (nr >= NREG && ft <= nr - NREG) {
                    const int q = nr - NREG;
                    if (!pipe::mbar_wait(&S.freeb[q % NREG], (q / NREG) & 1, deadline)) {
                        ok = false;
                        break;
                    }
                    ft = q + 1;
                }
                for (int q = ft; q < nr && ok; ++q) {
                    const int qo = roff[q % NREG], qb = rbytes[q % NREG];
                    if (qo < r.off + r.bytes && r.off < qo + qb) {
                        if (!pipe::mbar_wait(&S.freeb[q % NREG], (q / NREG) & 1, deadline))
                            ok = false;
                        ft = q + 1;
                    }
                }
                if (!ok)
                    break;
                roff[nr % NREG] = r.off;
                rbytes[nr % NREG] = r.bytes;
                const int sl = S.u_slot[r.u];
                const int e = S.s_e[sl], b = S.s_b[sl];
                uint64_t *bar = &S.full[nr % NREG];
                unsigned char *dst = S.ring + r.off;
                const float *esc = scales + (int64_t)e * escale_len;
                pipe::mbar_arrive_expect_tx(bar, (uint32_t)r.bytes);
                if (r.set < 2) {
                    const int rb = r.local / g.NKA, kg = r.local % g.NKA;
                    const int nt = r.n * KGA;
                    const int64_t t0 = (int64_t)rb * (H / 128) + kg * KGA; // first tile
                    for (int p = 0; p < b; ++p) {
                        const uint32_t *base = L.pool + (int64_t)S.u_ps[sl][p] * L.slot_words;
                        pipe::bulk_g2s(dst + (2 * p) * nt * 256, base + t0 * 64, nt * 256, bar);
                        pipe::bulk_g2s(dst + (2 * p + 1) * nt * 256, base + mat_words + t0 * 64, nt * 256, bar);
                    }
                    const uint32_t sb = 16 * (H / G) * 4;
                    unsigned char *sd = dst + 2 * b * nt * 256;
                    pipe::bulk_g2s(sd, esc + (int64_t)rb * 16 * (H / G), sb, bar);
                    pipe::bulk_g2s(sd + sb, esc + (int64_t)I * (H / G) + (int64_t)rb * 16 * (H / G), sb, bar);
                } else {
                    const int nt = r.n * g.KGB;
                    const int64_t t0 = (int64_t)r.local * g.KGB; // tile index in the down matrix
                    for (int p = 0; p < b; ++p) {
                        const uint32_t *base = L.pool + (int64_t)S.u_ps[sl][p] * L.slot_words + 2 * mat_words;
                        pipe::bulk_g2s(dst + p * nt * 256, base + t0 * 64, nt * 256, bar);
                    }
                    const int rb0 = r.local / g.NKB, rb1 = (r.local + r.n - 1) / g.NKB;
                    pipe::bulk_g2s(dst + b * nt * 256, esc + 2 * (int64_t)I * (H / G) + (int64_t)rb0 * 16 * (I / G),
                                   (rb1 - rb0 + 1) * 16 * (I / G) * 4, bar);
                }
                ++nr;
            }
            if (!ok)
                set_error(W, tag, deadline, kErrTimeout, 1);
            // no copy may still be landing in shared memory when the CTA exits
            const uint64_t drain = pipe::globaltimer() + kDrainNs;
            for (int q = nr - NREG > 0 ? nr - NREG : 0; q < nr; ++q)
                pipe::mbar_wait(&S.full[q % NREG], (q / NREG) & 1, drain);
        }
    } else if (warp == W_EPI) {
        // ------------------------------------------------------------ epilogue
        if (!wait_go(W, tag, deadline)) {
            set_error(W, tag, deadline, kErrTimeout, 7);
        } else {
            RegionIter it(S, g);
            Region r;
            int nr = 0;
            const int NKA = g.NKA, NKB = g.NKB;
            while (it.next(r)) {
                const int slot = nr % NREG;
                if (!pipe::mbar_wait(&S.consumed[slot], (nr / NREG) & 1, deadline)) {
                    set_error(W, tag, deadline, kErrTimeout, 8);
                    break;
                }
                const int u = r.u, sl = S.u_slot[u];
                if (r.set < 2) {
                    // gate (lanes 0-15) and up (16-31) row sums over the region's items, in order
                    float v = 0.0f;
                    for (int i = 0; i < r.n; ++i)
                        v += S.red[slot][i][lane];
                    __syncwarp();
                    if (lane == 0)
                        pipe::mbar_arrive(&S.freeb[slot]);
                    const int rb = r.local / NKA, kg0 = r.local % NKA;
                    bool complete = (kg0 == 0 && r.n == NKA);
                    if (!complete) {
                        // a piece of the row block: partial sums meet in the workspace
                        float *pa = W.pA1 + (((int64_t)sl * (I / 16) + rb) * NKA + kg0) * 32;
                        __stcg(pa + lane, v);
                        if (lane == 0)
                            __stcg(W.pendA + ((int64_t)sl * (I / 16) + rb) * NKA + kg0, kg0 + r.n);
                        __syncwarp();
                        int last = 0;
                        if (lane == 0)
                            last = atom_add_acq_rel(&W.cntA[sl * (I / 16) + rb], r.n) + r.n == NKA;
                        last = __shfl_sync(0xffffffffu, last, 0);
                        __syncwarp();
                        if (last) {
                            v = 0.0f;
                            for (int kg = 0; kg < NKA;) {
                                v += __ldcg(W.pA1 + (((int64_t)sl * (I / 16) + rb) * NKA + kg) * 32 + lane);
                                kg = __ldcg(W.pendA + ((int64_t)sl * (I / 16) + rb) * NKA + kg);
                            }
                            complete = true;
                        }
                    }
                    if (complete) {
                        const float uv = __shfl_down_sync(0xffffffffu, v, 16);
                        if (lane < 16)
                            __stcg(W.h + (int64_t)sl * I + 16 * rb + lane, v / (1.0f + expf(-v)) * uv);
                        __syncwarp();
                        int last = 0;
                        if (lane == 0)
                            last = atom_add_acq_rel(&W.cntH[sl * (I / 128) + rb / 8], 1) == 7;
                        last = __shfl_sync(0xffffffffu, last, 0);
                        __syncwarp();
                        if (last)
                            h_tile_to_frags(W, I, sl, rb / 8);
                    }
                } else {
                    // down: lanes 0-15 = rows of the region's first row block, 16-31 of the next
                    const int rbf = r.local / NKB, rbl = (r.local + r.n - 1) / NKB;
                    float vr[MAXI / 2 + 1];
                    int nrb = rbl - rbf + 1;
                    for (int j = 0; j * 2 < nrb; ++j) {
                        const int rb = rbf + 2 * j + (lane >> 4);
                        float v = 0.0f;
                        if (rb <= rbl) {
                            const int i0 = max(rb * NKB, r.local) - r.local;
                            const int i1 = min((rb + 1) * NKB, r.local + r.n) - r.local;
                            for (int i = i0; i < i1; ++i)
                                v += S.red[slot][i][lane & 15];
                        }
                        vr[j] = v;
                    }
                    __syncwarp();
                    if (lane == 0)
                        pipe::mbar_arrive(&S.freeb[slot]);
                    for (int j = 0; j * 2 < nrb; ++j) {
                        const int rb = rbf + 2 * j + (lane >> 4);
                        const bool has = rb <= rbl;
                        float v = vr[j];
                        const int kg0 = has ? max(rb * NKB, r.local) - rb * NKB : 0;
                        const int kg1 = has ? min((rb + 1) * NKB, r.local + r.n) - rb * NKB : 0;
                        bool complete = has && kg0 == 0 && kg1 == NKB;
                        if (has && !complete) {
                            float *pb = W.pB1 + (((int64_t)sl * (H / 16) + rb) * NKB + kg0) * 16;
                            __stcg(pb + (lane & 15), v);
                            if ((lane & 15) == 0)
                                __stcg(W.pendB + ((int64_t)sl * (H / 16) + rb) * NKB + kg0, kg1);
                        }
                        __syncwarp();
                        int last = 0;
                        if (has && !complete && (lane & 15) == 0)
                            last = atom_add_acq_rel(&W.cntB1[sl * (H / 16) + rb], kg1 - kg0) + (kg1 - kg0) == NKB;
                        last = __shfl_sync(0xffffffffu, last, lane & 16);
                        __syncwarp();
                        if (last) {
                            v = 0.0f;
                            for (int kg = 0; kg < NKB;) {
                                v += __ldcg(W.pB1 + (((int64_t)sl * (H / 16) + rb) * NKB + kg) * 16 + (lane & 15));
                                kg = __ldcg(W.pendB + ((int64_t)sl * (H / 16) + rb) * NKB + kg);
                            }
                            complete = true;
                        }
                        // this expert's contribution to 16 output rows; the last expert sums y
                        if (complete)
                            __stcg(W.part + (int64_t)sl * H + 16 * rb + (lane & 15), v);
                        __syncwarp();
                        int ylast = 0;
                        if (complete && (lane & 15) == 0)
                            ylast = atom_add_acq_rel(&W.ycnt1[rb], 1) == k - 1;
                        ylast = __shfl_sync(0xffffffffu, ylast, lane & 16);
                        __syncwarp();
                        if (ylast) {
                            float acc = 0.0f;
                            for (int s = 0; s < k; ++s)
                                acc = __fmaf_rn(S.s_w[s], __ldcg(W.part + (int64_t)s * H + 16 * rb + (lane & 15)), acc);
                            a.y[16 * rb + (lane & 15)] = acc;
                        }
                    }
                }
                ++nr;
            }
        }
    } else if (warp == W_STG) {
        // ------------------------------------------------------------ h stager
        if (lane == 0) {
            int nh = 0;
            bool ok = wait_go(W, tag, deadline);
            for (int s = 2; s < 4 && ok; ++s)
                for (int p = 0; p < S.setN[s] && ok; ++p) {
                    const int u = S.setU[s][p];
                    if (!(S.lo[s] < S.setStart[s][p + 1] && S.hi[s] > S.setStart[s][p]))
                        continue;
                    const int hsl = S.hslot_of[u];
                    if (hsl >= HSLOTS || hsl < nh) {
                        if (hsl >= HSLOTS) {
                            set_error(W, tag, deadline, kErrUnsupported, 9);
                            ok = false;
                        }
                        continue;
                    }
                    const int sl = S.u_slot[u];
                    for (int q = 0; q < I / 128 && ok; ++q)
                        while (pipe::ld_acquire(&W.readyH[sl * (I / 128) + q]) == 0) {
                            if (pipe::globaltimer() > deadline) {
                                set_error(W, tag, deadline, kErrTimeout, 5);
                                ok = false;
                                break;
                            }
                            __nanosleep(200);
                        }
                    if (!ok)
                        break;
                    pipe::fence_proxy_async();
                    const uint32_t fb = (I / 32) * 16 * 4, eb = (I / 128) * 4;
                    pipe::mbar_arrive_expect_tx(&S.hfull[hsl], fb + ((eb + 15) & ~15u));
                    pipe::bulk_g2s(S.hs[hsl], W.hfrag + (int64_t)sl * (I / 32) * 16, fb, &S.hfull[hsl]);
                    pipe::bulk_g2s(S.hse[hsl], W.hexp + (int64_t)sl * hexp_stride(I), (eb + 15) & ~15u,
                                   &S.hfull[hsl]);
                    nh = hsl + 1;
                }
            const uint64_t drain = pipe::globaltimer() + kDrainNs;
            for (int h = 0; h < nh; ++h)
                pipe::mbar_wait(&S.hfull[h], 0, drain);
        }
    } else {
        // ------------------------------------------------------------ consumers
        RegionIter it(S, g);
        Region r;
        r.n = 0;
        r.i0 = 0;
        int nr = -1;
        bool ok = true;
        int hwait = -1; // h slot this warp has already waited for
        bool go_seen = false;
        const int t = lane & 3, gq = lane >> 2;
        const int fo = (4 * (gq & 1) + t) * 2; // this lane's B-fragment word within a k-step
        for (int i = warp; i < S.nitems && ok; i += NCW) {
            while (i >= r.i0 + r.n) {
                __syncwarp();
                if (nr >= 0 && lane == 0)
                    pipe::mbar_arrive(&S.consumed[nr % NREG]);
                if (!it.next(r)) {
                    ok = false;
                    break;
                }
                ++nr;
                if (!pipe::mbar_wait(&S.full[nr % NREG], (nr / NREG) & 1, deadline)) {
                    set_error(W, tag, deadline, kErrTimeout, 3);
                    ok = false;
                    break;
                }
            }
            if (!ok)
                break;
            const int ii = i - r.i0;
            const int u = r.u, sl = S.u_slot[u], b = S.s_b[sl];
            const unsigned char *reg = S.ring + r.off;
            float *red = S.red[nr % NREG][ii];
            const uint32_t *big = nullptr;
            if (b >= 5) {
                if (!go_seen) {
                    go_seen = wait_go(W, tag, deadline);
                    if (!go_seen) {
                        set_error(W, tag, deadline, kErrTimeout, 6);
                        ok = false;
                        break;
                    }
                }
            }
            if (r.set < 2) {
                const int kg0 = r.local % g.NKA, nt = r.n * KGA;
                const int kt0 = (kg0 + ii) * KGA;       // first k-tile of the item
                const int jt = ii * KGA;                // its tile offset in the region
                const float *scb = reinterpret_cast<const float *>(reg + 2 * b * nt * 256);
                const int ngr = H / G, gpt = 128 / G;
                float acc[2][2];
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    acc[m][0] = acc[m][1] = 0.0f;
                    if (b >= 5)
                        big = W.tabs + ((int64_t)sl * 3 + m) * kTabWords + 16;
                    const float *sc0 = scb + m * 16 * ngr + gq * ngr + kt0 * gpt;
                    tiles_any<GS>(b, KGA, reg + (2 * 0 + m) * nt * 256 + jt * 256 + lane * 8, 2 * nt * 256,
                                  S.tab[sl][m], big, S.xs + fo, S.xse, kt0, sc0, sc0 + 8 * ngr, gpt, acc[m][0],
                                  acc[m][1]);
                }
                if (t == 0) {
                    red[gq] = acc[0][0];
                    red[gq + 8] = acc[0][1];
                    red[16 + gq] = acc[1][0];
                    red[24 + gq] = acc[1][1];
                }
            } else {
                const int hsl = S.hslot_of[u];
                if (hsl < 0 || hsl >= HSLOTS) { // more down units than staging slots: reported by the stager
                    ok = false;
                    break;
                }
                if (hwait != hsl) {
                    if (!pipe::mbar_wait(&S.hfull[hsl], 0, deadline)) {
                        set_error(W, tag, deadline, kErrTimeout, 4);
                        ok = false;
                        break;
                    }
                    hwait = hsl;
                }
                const int nt = r.n * g.KGB;
                const int lin = r.local + ii;
                const int rb = lin / g.NKB, kt0 = (lin % g.NKB) * g.KGB;
                const int rbf = r.local / g.NKB;
                const float *scb = reinterpret_cast<const float *>(reg + b * nt * 256);
                const int ngr = I / G, gpt = 128 / G;
                const float *sc0 = scb + ((rb - rbf) * 16 + gq) * ngr + kt0 * gpt;
                if (b >= 5)
                    big = W.tabs + ((int64_t)sl * 3 + 2) * kTabWords + 16;
                float a0 = 0.0f, a1 = 0.0f;
                tiles_any<GS>(b, g.KGB, reg + ii * g.KGB * 256 + lane * 8, nt * 256, S.tab[sl][2], big,
                              S.hs[hsl] + fo, S.hse[hsl], kt0, sc0, sc0 + 8 * ngr, gpt, a0, a1);
                if (t == 0) {
                    red[gq] = a0;
                    red[gq + 8] = a1;
                }
            }
        }
        // past the last item: every remaining region is consumed as far as this warp is concerned
        // (its slot's barrier is in that region's phase only once the region has been issued)
        if (ok) {
            __syncwarp();
            if (nr >= 0 && lane == 0)
                pipe::mbar_arrive(&S.consumed[nr % NREG]);
            while (it.next(r)) {
                ++nr;
                if (!pipe::mbar_wait(&S.full[nr % NREG], (nr / NREG) & 1, deadline)) {
                    set_error(W, tag, deadline, kErrTimeout, 3);
                    break;
                }
                __syncwarp();
                if (lane == 0)
                    pipe::mbar_arrive(&S.consumed[nr % NREG]);
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        // the last CTA to finish advances the epoch of the workspace
        if (wait_go(W, tag, deadline + kDrainNs)) {
            if (atom_add_acq_rel(&W.flags[kFlagDone], 1) == (int)gridDim.x - 1)
                pipe::st_release(&W.flags[kFlagSeq], (int)(seq + 1u));
        }
    }
}

} // namespace d1

static int g_num_sms1[128] = {};
static uint64_t g_wait_limit_ns = 200ull * 1000 * 1000;

void set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns; }
uint64_t wait_limit_ns() { return g_wait_limit_ns; }

pmoe_status launch_decode1(const pmoe_layer *L, const float *logits, const float *sens, const uint16_t *x,
                           int32_t *ids, float *w, uint8_t *depth, int k, int B, float *y, const LayerWs &W,
                           cudaStream_t st, cudaEvent_t ev0, cudaEvent_t ev1)
{
    if (k > d1::MAXU || L->H > d1::HMAX || L->I > d1::IMAX || (L->H / 128) % d1::KGA)
        return PMOE_ERR_UNSUPPORTED;
    int dev = 0;
    PMOE_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 128)
        return PMOE_ERR_UNSUPPORTED;
    if (g_num_sms1[dev] == 0)
        PMOE_CUDA(cudaDeviceGetAttribute(&g_num_sms1[dev], cudaDevAttrMultiProcessorCount, dev));
    d1::Args a{*L, logits, sens, x, ids, w, depth, k, B, y, W, g_wait_limit_ns};
    void (*kern)(d1::Args);
    switch (L->G) {
    case 32: kern = d1::decode1_kernel<1>; break;
    case 64: kern = d1::decode1_kernel<2>; break;
    default: kern = d1::decode1_kernel<4>; break;
    }
    const size_t smem = sizeof(d1::Smem);
    PMOE_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    // the CTAs wait on one another (h tiles, row blocks split between CTAs), so all of them must be
    // resident at once: a cooperative launch of one CTA per SM guarantees that
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g_num_sms1[dev]);
    cfg.blockDim = dim3(d1::NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (ev0)
        PMOE_CUDA(cudaEventRecord(ev0, st));
    PMOE_CUDA(cudaLaunchKernelEx(&cfg, kern, a));
    if (ev1)
        PMOE_CUDA(cudaEventRecord(ev1, st));
    return PMOE_OK;
}

} // namespace pmoe
