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
//  * Epilogue: reduces each region's item sums in item order and releases the
//    region's slot. A complete row block of gate/up becomes 16 rows of
//    h = silu(g) * u, published with a flag tagged with the call's epoch. A
//    complete row block of down is one expert's contribution to 16 output
//    rows; the last expert to finish those rows (one atomic per row block, the
//    region's row blocks side by side on the warp's lanes) sums the k
//    contributions into y in slot order (deterministic). Row blocks whose K
//    range is split between regions or CTAs meet through partial sums in the
//    workspace, summed in K order by whichever piece completes them.
//  * Stager: waits (bounded) until every row block of h of a unit the CTA's
//    down items use is flagged, then turns the unit's h into MMA fragments in
//    shared memory itself (24-bit fixed point, one exponent per 128 rows).
// The producer reuses ring bytes as soon as the consumers are past a region,
// and a region slot once the epilogue has read its sums. Decode tables are
// built per CTA for the experts its items touch; tables of depth >= 5 (256
// entries) live in shared memory as 16-bit entries.
// Every wait is bounded by one deadline per launch; a wait that runs out
// records an error and the CTA stops work, waits (with a separate, long
// limit) for its own copies in flight, and exits.
// Counters: CTA 0 zeroes the call's counters and error record, then publishes
// a "go" word tagged with the call's epoch; nothing else touches counters
// before it sees it. The last CTA to finish advances the epoch.
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
constexpr int NEPI = 2;                     // epilogue warps (regions alternate between them)
constexpr int W_PROD = NCW, W_EPI = NCW + 1, W_STG = NCW + 1 + NEPI;
constexpr int NTHREADS = (NCW + 2 + NEPI) * 32;
constexpr int NREG = 8;                     // region slots
constexpr int RING = 168 * 1024;            // ring bytes
constexpr int REG_CAP = 48 * 1024;          // target bytes per region
constexpr int MAXI = 16;                    // items per region
constexpr int MAXU = 32;                    // units (k)
constexpr int HSLOTS = 4;                   // units whose h a CTA's down items read
constexpr int BIGS = 4;                     // depth >= 5 units per matrix kind whose full tables a CTA holds
constexpr int KGA = 2;                      // k-tiles per gate/up item
constexpr int HMAX = 4096, IMAX = 1024;
constexpr uint64_t kDrainNs = 1000ull * 1000 * 1000; // limit for waiting on one's own copies at exit

struct TabS {                               // register table of one (unit, matrix) in shared memory
    uint32_t h[4], l[4];
    int f;
    uint32_t c1;                            // C[1][1] bits (depth-1 sign path)
    uint32_t anti;                          // depth-1 table is antisymmetric
    int big;                                // slot of its 256-entry table (depth >= 5), else -1
};

struct Smem {
    alignas(128) unsigned char ring[RING];
    float red[NREG][MAXI][32];
    alignas(16) uint32_t xs[(HMAX / 32) * dev::kFragWords];
    alignas(16) uint32_t hs[HSLOTS][(IMAX / 32) * dev::kFragWords];
    alignas(16) uint32_t zeros[4];
    alignas(16) int xse[HMAX / 128];
    alignas(16) int hse[HSLOTS][IMAX / 128];
    alignas(16) uint16_t big[3 * BIGS][256]; // [0, 2*BIGS): gate/up tables, [2*BIGS, 3*BIGS): down
    TabS tab[MAXU][3];
    // routing result per slot, and units (order: depth desc, slot asc)
    int s_e[MAXU], s_b[MAXU];
    float s_w[MAXU];
    int u_slot[MAXU];                       // unit -> routing slot
    int u_ps[MAXU][8];                      // plane slots of the slot's expert
    int hslot_of[MAXU];                     // h staging slot of a slot whose down rows this CTA computes
    int bigA_of[MAXU], bigB_of[MAXU];       // 256-entry table slots of depth >= 5 slots (gate/up pair, down)
    // sets: units, item offsets, this CTA's range
    int setN[4], setU[4][MAXU], setStart[4][MAXU + 1], lo[4], hi[4];
    int nitems;                             // items in this CTA's stream
    int ntab, tabwork[3 * MAXU];            // tables to build: slot * 3 + matrix
    int bad;                                // nonzero: invalid routing input (no work is done)
    int unsup;                              // nonzero: more experts than the per-CTA slots (no work is done)
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

// ---------------------------------------------------------------- schedule

struct Geo {
    int H, I, G, NKA, NKB, KGB, k;
    __device__ int items_A() const { return (I / 16) * NKA; }
    __device__ int items_B() const { return (H / 16) * NKB; }
};

// relative cost of one item of depth b: its decode time, measured on B200 (consumer time per item
// of depths 1..4 about 1.8, 2.3, 2.6, 5.5 us with 16 warps sharing an SM; depth >= 5 decodes from
// a 256-entry table in shared memory). Small integers, so that a set's total times the grid size
// fits in 32 bits.
__device__ __forceinline__ int item_cost(int b)
{
    constexpr int c[9] = {0, 18, 23, 26, 55, 60, 65, 70, 75};
    return c[b < 1 ? 1 : (b > 8 ? 8 : b)];
}

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

// Whether this CTA's range of set s covers any item of the set's unit at position p.
__device__ __forceinline__ bool touches(const Smem &S, int s, int p)
{
    return S.lo[s] < S.setStart[s][p + 1] && S.hi[s] > S.setStart[s][p];
}

// ---------------------------------------------------------------- consumer tiles

// One 16x128 tile of one matrix at depth B: rows g, g+8 of this lane accumulate
// sum over the tile's groups of F (combine24) * scale * fac, fac including the
// lane's factor (lanes t = 0 and t = 1 hold complementary parts of the sum).
//  pl: plane 0 of the tile + 8*lane bytes; pstep: bytes between planes.
//  xf: this lane's B fragment of the tile's first k-step; xstep: words per k-step (0: zeros).
//  sc0/sc1: scale rows g / g+8 at the tile's first group.
template <int B, int GS>
__device__ __forceinline__ void tile_dot(const unsigned char *pl, int pstep, const RegTab &tab, const uint16_t *big,
                                         const uint32_t *xf, int xstep, const float *sc0, const float *sc1, float fac,
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
        dev::decode_kstep<B, uint16_t>(w, s, tab, big, ah, al);
        const uint2 bv = *reinterpret_cast<const uint2 *>(xf + s * xstep);
        dev::mma_s8(dh, ah, bv.x, bv.y);
        dev::mma_s8(dl, al, bv.x, bv.y);
        if ((s + 1) % GS == 0) {
            const int gi = s / GS;
            acc0 = __fmaf_rn(dev::combine24(dh[0], dh[1], dl[0], dl[1]), sc0[gi] * fac, acc0);
            acc1 = __fmaf_rn(dev::combine24(dh[2], dh[3], dl[2], dl[3]), sc1[gi] * fac, acc1);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dh[i] = dl[i] = 0;
        }
    }
}

// Depth 1 of an antisymmetric table: +-1 bytes, one MMA per k-step; fac includes C[1][1]
// and the lane factor of an A operand without a low byte.
template <int GS>
__device__ __forceinline__ void tile_dot_sign(const unsigned char *pl, const uint32_t *xf, int xstep,
                                              const float *sc0, const float *sc1, float fac, float &acc0,
                                              float &acc1)
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
        const uint2 bv = *reinterpret_cast<const uint2 *>(xf + s * xstep);
        dev::mma_s8(dh, a, bv.x, bv.y);
        if ((s + 1) % GS == 0) {
            const int gi = s / GS;
            acc0 = __fmaf_rn(dev::combine24(dh[0], dh[1], 0, 0), sc0[gi] * fac, acc0);
            acc1 = __fmaf_rn(dev::combine24(dh[2], dh[3], 0, 0), sc1[gi] * fac, acc1);
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

// ntiles consecutive tiles (k-tiles kt0..) of one matrix at depth B. xf: the lane's fragment of
// k-step 0 of the vector (xstep words per k-step); xe: the vector's tile exponents; lf: the
// lane factor (combine24_lane_factor).
template <int B, int GS>
__device__ __forceinline__ void tiles_dot(int ntiles, const unsigned char *pl, int pstep, const TabS &ts,
                                          const uint16_t *big, const uint32_t *xf, int xstep, const int *xe, int kt0,
                                          float lf, const float *sc0, const float *sc1, int gpt, float &acc0,
                                          float &acc1)
{
    if constexpr (B == 1) {
        if (ts.anti) {
            const float c1 = __uint_as_float(ts.c1) * lf * 0.00390625f;
            for (int j = 0; j < ntiles; ++j)
                tile_dot_sign<GS>(pl + j * 256, xf + (kt0 + j) * 4 * xstep, xstep, sc0 + j * gpt, sc1 + j * gpt,
                                  c1 * pow2neg(xe[kt0 + j]), acc0, acc1);
            return;
        }
    }
    RegTab tab;
    load_tab(ts, tab);
    for (int j = 0; j < ntiles; ++j)
        tile_dot<B, GS>(pl + j * 256, pstep, tab, big, xf + (kt0 + j) * 4 * xstep, xstep, sc0 + j * gpt,
                        sc1 + j * gpt, lf * pow2neg(tab.f + xe[kt0 + j]), acc0, acc1);
}

template <int GS>
__device__ __forceinline__ void tiles_any(int b, int ntiles, const unsigned char *pl, int pstep, const TabS &ts,
                                          const uint16_t *big, const uint32_t *xf, int xstep, const int *xe,
                                          int kt0, float lf, const float *sc0, const float *sc1, int gpt,
                                          float &acc0, float &acc1)
{
#define PMOE_TILES(BB) tiles_dot<BB, GS>(ntiles, pl, pstep, ts, big, xf, xstep, xe, kt0, lf, sc0, sc1, gpt, acc0, acc1)
    switch (b) {
    case 1: PMOE_TILES(1); break;
    case 2: PMOE_TILES(2); break;
    case 3: PMOE_TILES(3); break;
    case 4: PMOE_TILES(4); break;
    case 5: PMOE_TILES(5); break;
    case 6: PMOE_TILES(6); break;
    case 7: PMOE_TILES(7); break;
    default: PMOE_TILES(8); break;
    }
#undef PMOE_TILES
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

    // ---- setup. The producer waits only for routing and the schedule (warp 0), which wait only for
    // the staged sensitivities and plane-slot table (warps 1, 2); the activation fragments, CTA 0's
    // resets and the decode tables are done by the other warps while the first copies are in flight.
    //   bar 2 (warps 0-2):        sensitivities and slot table staged, top-k done
    //   bar 3 (warp 0, producer): schedule known
    //   bar 4 (all but producer): fragments, resets and schedule done
    //   bar 1 (all but producer): decode tables built
    float *sens_s = reinterpret_cast<float *>(S.ring);                      // [E]
    int32_t *slot_s = reinterpret_cast<int32_t *>(S.ring + 4 * E);          // [E*8] when staged
    const bool stage_sens = a.logits != nullptr && 4 * E <= RING;
    const bool stage_slots = 36 * E <= RING;
    if (warp == 0) {
        int my_id = 0;
        float my_w = 0.0f;
        if (a.logits != nullptr) {
            if (E <= 512)
                dev::route_token_reg<16>(a.logits, E, k, my_id, my_w);
            else
                dev::route_token(a.logits, E, k, reinterpret_cast<float *>(S.red), my_id, my_w);
        } else if (lane < k) {
            my_id = __ldg(a.ids + lane);
            my_w = __ldg(a.w + lane);
        }
        pipe::named_bar(2, 96);
        // prefix selection from the staged sensitivities
        const bool idok = lane >= k || (my_id >= 0 && my_id < E);
        int b = 1;
        if (a.logits != nullptr) {
            const float v = (lane < k && idok) ? __fmul_rn(my_w, stage_sens ? sens_s[my_id] : __ldg(a.sens + my_id)) : 0.0f;
            b = dev::select_token(v, k, a.B, nullptr);
        } else if (lane < k) {
            b = __ldg(a.depth + lane);
        }
        const bool badl = lane < k && (!idok || b < 1 || b > 8);
        const unsigned badm = __ballot_sync(0xffffffffu, badl);
        if (badl) {
            my_id = 0;
            b = 1;
        }
        if (lane < k) {
            S.s_e[lane] = my_id;
            S.s_b[lane] = b;
            S.s_w[lane] = my_w;
        }
        if (lane == 0) {
            S.bad = badm != 0u;
            S.missing = -1;
        }
        if (blockIdx.x == 0 && a.logits != nullptr && lane < k) {
            a.ids[lane] = my_id;
            a.w[lane] = my_w;
            a.depth[lane] = (uint8_t)b;
        }
        __syncwarp();
        // schedule (lane u holds unit u). Unit order: depth descending, slot ascending.
        const int my_b = lane < k ? b : 0;
        int rank = 0;
        for (int j = 0; j < k; ++j) {
            const int bj = __shfl_sync(0xffffffffu, my_b, j);
            rank += (bj > my_b || (bj == my_b && j < lane)) ? 1 : 0;
        }
        if (lane < k)
            S.u_slot[rank] = lane;
        // plane slots of every routed expert; a needed plane without one is an error of the call
        for (int j = lane; j < k * 8; j += 32) {
            const int sl = j / 8, p = j % 8;
            const int ps = stage_slots ? slot_s[S.s_e[sl] * 8 + p] : __ldg(L.slot_of + S.s_e[sl] * 8 + p);
            S.u_ps[sl][p] = ps;
            if (ps < 0 && p < S.s_b[sl])
                atomicMax(&S.missing, S.s_e[sl] * 8 + p);
        }
        __syncwarp();
        const bool isu = lane < k;
        const int usl = isu ? S.u_slot[lane] : 0;
        const int ub = isu ? S.s_b[usl] : 0;
        const int cost = isu ? item_cost(ub) : 0;
        int incl = cost; // inclusive prefix of cost over units
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += v;
        }
        const int excl = incl - cost, tot = __shfl_sync(0xffffffffu, incl, 31);
        // P = the shortest prefix of units holding at least half the gate/up cost (Q keeps one unit)
        int np = __popc(__ballot_sync(0xffffffffu, isu && 2 * excl < tot));
        if (np == k && k > 1)
            np = k - 1;
        const int nA = g.items_A(), nB = g.items_B();
        // lanes 0-7: boundary of set s = lane/2 (0 A(P), 1 A(Q), 2 B(P), 3 B(Q)) for CTA c = this CTA
        // (even lanes) or the next (odd lanes): the first item whose cumulative cost reaches c/nc of the
        // set's total. Unit p of a set holds items [p*n, (p+1)*n).
        const int ms = (lane >> 1) & 3, mc = (int)blockIdx.x + (lane & 1);
        const int mu0 = (ms == 0 || ms == 2) ? 0 : np, mu1 = (ms == 0 || ms == 2) ? np : k;
        const int mn = ms < 2 ? nA : nB;
        const int cbase = __shfl_sync(0xffffffffu, excl, mu0 & 31);       // cost of the units before the set
        const int cend = __shfl_sync(0xffffffffu, incl, (mu1 - 1) & 31);  // ... up to its last unit
        const int stot = (mu1 > mu0 ? cend - cbase : 0) * mn;
        // (costs <= 75, units <= 32, items <= 1024, CTAs <= 148: products < 2^31)
        const int target = mc >= (int)gridDim.x ? -1 : (stot * mc) / (int)gridDim.x;
        int bnd = (mu1 - mu0) * mn;
        bool found = mc >= (int)gridDim.x;
        for (int p = 0; p < k; ++p) {
            const int ep = __shfl_sync(0xffffffffu, excl, p), cp = __shfl_sync(0xffffffffu, cost, p);
            if (!found && p >= mu0 && p < mu1) {
                const int before = (ep - cbase) * mn;
                if (target <= before + cp * mn) {
                    bnd = (p - mu0) * mn + (target - before + cp - 1) / cp;
                    found = true;
                }
            }
        }
        if (lane < 8) {
            if (lane & 1)
                S.hi[ms] = bnd;
            else
                S.lo[ms] = bnd;
        }
        for (int s2 = 0; s2 < 4; ++s2) {
            const int u0 = (s2 == 0 || s2 == 2) ? 0 : np, u1 = (s2 == 0 || s2 == 2) ? np : k;
            const int n = s2 < 2 ? nA : nB;
            if (lane == 0)
                S.setN[s2] = u1 - u0;
            for (int p = lane; p <= u1 - u0; p += 32) {
                S.setStart[s2][p] = p * n;
                if (p < u1 - u0)
                    S.setU[s2][p] = u0 + p;
            }
        }
        __syncwarp();
        // units each range touches (lane u): tables to build, h slots, 256-entry table slots
        bool tA = false, tB = false;
        if (isu) {
            const int sA = lane < np ? 0 : 1, pA = lane < np ? lane : lane - np;
            tA = S.lo[sA] < (pA + 1) * nA && S.hi[sA] > pA * nA;
            tB = S.lo[sA + 2] < (pA + 1) * nB && S.hi[sA + 2] > pA * nB;
        }
        const unsigned mA = __ballot_sync(0xffffffffu, tA), mB = __ballot_sync(0xffffffffu, tB);
        const unsigned below = (1u << lane) - 1u;
        const unsigned dA = __ballot_sync(0xffffffffu, tA && ub >= 5), dB = __ballot_sync(0xffffffffu, tB && ub >= 5);
        const int nAt = __popc(mA);
        S.hslot_of[lane] = -1;
        S.bigA_of[lane] = -1;
        S.bigB_of[lane] = -1;
        __syncwarp();
        if (tA) {
            const int pos = 2 * __popc(mA & below);
            S.tabwork[pos] = usl * 3;
            S.tabwork[pos + 1] = usl * 3 + 1;
            if (ub >= 5)
                S.bigA_of[usl] = __popc(dA & below);
        }
        if (tB) {
            const int pos = __popc(mB & below);
            S.tabwork[2 * nAt + pos] = usl * 3 + 2;
            S.hslot_of[usl] = pos;
            if (ub >= 5)
                S.bigB_of[usl] = __popc(dB & below);
        }
        if (lane == 0) {
            int n = 0;
            for (int s2 = 0; s2 < 4; ++s2)
                n += S.hi[s2] - S.lo[s2];
            S.nitems = n;
            S.ntab = 2 * nAt + __popc(mB);
            S.unsup = (__popc(dA) > BIGS || __popc(dB) > BIGS || __popc(mB) > HSLOTS) ? 1 : 0;
        }
        __syncwarp();
        pipe::named_bar(3, 64);
    } else if (warp == 1 || warp == 2) {
        const int t0 = tid - 32;
        if (stage_sens)
            for (int i = t0; i < E; i += 64)
                sens_s[i] = __ldg(a.sens + i);
        if (stage_slots)
            for (int i = t0; i < E * 8; i += 64)
                slot_s[i] = __ldg(L.slot_of + i);
        if (tid >= 32 && tid < 36)
            S.zeros[tid - 32] = 0u;
        if (tid == 32) {
            for (int s2 = 0; s2 < NREG; ++s2) {
                pipe::mbar_init(&S.full[s2], 1);
                pipe::mbar_init(&S.consumed[s2], NCW);
                pipe::mbar_init(&S.freeb[s2], 1);
            }
            for (int s2 = 0; s2 < HSLOTS; ++s2)
                pipe::mbar_init(&S.hfull[s2], 1);
            pipe::fence_barrier_init();
        }
        pipe::named_bar(2, 96);
    } else if (warp == W_PROD) {
        pipe::named_bar(3, 64);
    } else {
        // activation fragments and CTA 0's resets (warps 3..: all but 0-2 and the producer)
        const int wi = warp - 3 - (warp > W_PROD ? 1 : 0), nw = (NTHREADS / 32) - 4;
        for (int Q = wi; Q < H / 128; Q += nw)
            dev::make_xfrag_tile<true>(a.x, Q, S.xs, S.xse);
        if (blockIdx.x == 0) {
            const int t0 = wi * 32 + lane, nt = nw * 32;
            for (int i = t0; i < k * (I / 16); i += nt)
                W.cntA[i] = 0;
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
    if (warp != W_PROD) {
        pipe::named_bar(4, NTHREADS - 32);
        if (blockIdx.x == 0 && tid == 0) {
            __threadfence();
            pipe::st_release(&W.flags[kFlagGo], (int)tag);
        }
    }
    const bool fail = S.bad || S.missing >= 0 || S.unsup;

    if (!fail && warp == W_PROD) {
        // ------------------------------------------------------------ producer
        // Lane 0 takes the waits and arms the region's barrier; the region's copies (one per plane and
        // matrix, one per scale block) are issued by the warp's lanes side by side, since one thread
        // issuing copies of a few KB one after another cannot keep an SM's share of HBM busy.
        const float *scales = L.scales;
        const int64_t mat_words = (int64_t)H * I / 32;
        const int64_t escale_len = 2 * (int64_t)I * (H / G) + (int64_t)H * (I / G);
        RegionIter it(S, g);
        Region r;
        int nr = 0, fs = 0, fc = 0; // regions issued; first region whose slot / bytes may be in use
        int roff[NREG], rbytes[NREG];
        bool ok = true;
        while (ok && it.next(r)) {
            if (lane == 0) {
                // a region slot is reused once the epilogue has read the sums of its last region
                if (nr >= NREG && fs <= nr - NREG) {
                    const int q = nr - NREG;
                    if (!pipe::mbar_wait(&S.freeb[q % NREG], (q / NREG) & 1, deadline))
                        ok = false;
                    fs = q + 1;
                    fc = max(fc, fs);
                }
                // ring bytes are reused once every consumer is past the regions that held them
                for (int q = fc; q < nr && ok; ++q) {
                    const int qo = roff[q % NREG], qb = rbytes[q % NREG];
                    if (qo < r.off + r.bytes && r.off < qo + qb) {
                        if (!pipe::mbar_wait(&S.consumed[q % NREG], (q / NREG) & 1, deadline))
                            ok = false;
                        fc = q + 1;
                    }
                }
                roff[nr % NREG] = r.off;
                rbytes[nr % NREG] = r.bytes;
                if (ok)
                    pipe::mbar_arrive_expect_tx(&S.full[nr % NREG], (uint32_t)r.bytes);
            }
            ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
            if (!ok)
                break;
            const int sl = S.u_slot[r.u];
            const int e = S.s_e[sl], b = S.s_b[sl];
            uint64_t *bar = &S.full[nr % NREG];
            unsigned char *dst = S.ring + r.off;
            const float *esc = scales + (int64_t)e * escale_len;
            if (r.set < 2) {
                // copies 0 .. 2b-1: plane c/2 of gate (c even) or up (c odd); 2b, 2b+1: their scale rows
                const int rb = r.local / g.NKA, kg = r.local % g.NKA;
                const int nt = r.n * KGA;
                const int64_t t0 = (int64_t)rb * (H / 128) + kg * KGA; // first tile
                const uint32_t sb = 16 * (H / G) * 4;
                if (lane < 2 * b) {
                    const int p = lane >> 1, m = lane & 1;
                    const uint32_t *base = L.pool + (int64_t)S.u_ps[sl][p] * L.slot_words + m * mat_words;
                    pipe::bulk_g2s(dst + lane * nt * 256, base + t0 * 64, nt * 256, bar);
                } else if (lane < 2 * b + 2) {
                    const int m = lane - 2 * b;
                    pipe::bulk_g2s(dst + 2 * b * nt * 256 + m * sb,
                                   esc + (int64_t)m * I * (H / G) + (int64_t)rb * 16 * (H / G), sb, bar);
                }
            } else {
                // copies 0 .. b-1: plane c of down; b: its scale rows
                const int nt = r.n * g.KGB;
                const int64_t t0 = (int64_t)r.local * g.KGB; // tile index in the down matrix
                if (lane < b) {
                    const uint32_t *base = L.pool + (int64_t)S.u_ps[sl][lane] * L.slot_words + 2 * mat_words;
                    pipe::bulk_g2s(dst + lane * nt * 256, base + t0 * 64, nt * 256, bar);
                } else if (lane == b) {
                    const int rb0 = r.local / g.NKB, rb1 = (r.local + r.n - 1) / g.NKB;
                    pipe::bulk_g2s(dst + b * nt * 256, esc + 2 * (int64_t)I * (H / G) + (int64_t)rb0 * 16 * (I / G),
                                   (rb1 - rb0 + 1) * 16 * (I / G) * 4, bar);
                }
            }
            __syncwarp();
            ++nr;
        }
        if (lane == 0) {
            if (!ok)
                set_error(W, tag, deadline, kErrTimeout, 1);
            // no copy may still be landing in shared memory when the CTA exits
            const uint64_t drain = pipe::globaltimer() + kDrainNs;
            for (int q = nr - NREG > 0 ? nr - NREG : 0; q < nr; ++q)
                pipe::mbar_wait(&S.full[q % NREG], (q / NREG) & 1, drain);
        }
    } else if (!fail) {
        // ---- setup 3 (all warps but the producer): decode tables of the experts this CTA touches
        for (int j = warp - (warp > W_PROD ? 1 : 0); j < S.ntab; j += (NTHREADS / 32) - 1) {
            const int sl = S.tabwork[j] / 3, m = S.tabwork[j] % 3, b = S.s_b[sl];
            const int bs = (m < 2) ? (S.bigA_of[sl] >= 0 ? 2 * S.bigA_of[sl] + m : -1)
                                   : (S.bigB_of[sl] >= 0 ? 2 * BIGS + S.bigB_of[sl] : -1);
            const float *cb = L.codebooks + ((int64_t)S.s_e[sl] * 3 + m) * 510;
            RegTab t;
            dev::build_tab<uint16_t>(cb, b, t, bs >= 0 ? S.big[bs] : nullptr);
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
                d.big = bs;
            }
        }
        pipe::named_bar(1, NTHREADS - 32);

        if (warp >= W_EPI && warp < W_EPI + NEPI) {
            // ------------------------------------------------------------ epilogue
            const int ew = warp - W_EPI; // this warp takes regions ew, ew + NEPI, ...
            if (!wait_go(W, tag, deadline)) {
                set_error(W, tag, deadline, kErrTimeout, 7);
            } else {
                RegionIter it(S, g);
                Region r;
                int nr = 0;
                const int NKA = g.NKA, NKB = g.NKB;
                while (it.next(r)) {
                    const int slot = nr % NREG;
                    if (nr % NEPI != ew) {
                        ++nr;
                        continue;
                    }
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
                            // 16 rows of h stored by lane 0, then the row block's flag (a release by
                            // the same thread) for every CTA's stager
                            const float uv = __shfl_down_sync(0xffffffffu, v, 16);
                            const float hv = v / (1.0f + expf(-v)) * uv;
                            float hr[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                hr[j] = __shfl_sync(0xffffffffu, hv, j);
                            if (lane == 0) {
                                float4 *hp = reinterpret_cast<float4 *>(W.h + (int64_t)sl * I + 16 * rb);
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    __stcg(hp + j, make_float4(hr[4 * j], hr[4 * j + 1], hr[4 * j + 2], hr[4 * j + 3]));
                                pipe::st_release(&W.hflag[sl * (I / 16) + rb], (int)tag);
                            }
                        }
                    } else {
                        // down: the region's row blocks, two at a time (lanes 0-15 and 16-31)
                        const int rbf = r.local / NKB, rbl = (r.local + r.n - 1) / NKB;
                        const int nrb = rbl - rbf + 1;
                        float vr[MAXI / 2 + 1];
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
                        unsigned done = 0u; // bit rb - rbf: this expert's 16 rows of that row block are written
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
                            if (complete)
                                __stcg(W.part + (int64_t)sl * H + 16 * rb + (lane & 15), v);
                            const unsigned cm = __ballot_sync(0xffffffffu, complete && (lane & 15) == 0);
                            if (cm & 1u)
                                done |= 1u << (2 * j);
                            if (cm & 0x10000u)
                                done |= 1u << (2 * j + 1);
                        }
                        // one atomic per finished row block, all on the lanes side by side (each a release
                        // after the warp barrier that follows the rows' stores); the last expert of a row
                        // block sums the k contributions in slot order
                        __syncwarp();
                        int ylast = 0;
                        if (lane < nrb && ((done >> lane) & 1u))
                            ylast = atom_add_acq_rel(&W.ycnt1[rbf + lane], 1) == k - 1;
                        unsigned lm = __ballot_sync(0xffffffffu, ylast);
                        __syncwarp();
                        while (lm) {
                            const int j0 = __ffs(lm) - 1;
                            lm &= lm - 1;
                            int j1 = -1;
                            if (lm) {
                                j1 = __ffs(lm) - 1;
                                lm &= lm - 1;
                            }
                            const int jj = (lane < 16) ? j0 : j1;
                            if (jj >= 0) {
                                const int rb = rbf + jj, row = 16 * rb + (lane & 15);
                                float acc = 0.0f;
                                // the k contributions, eight loads in flight at a time, summed in slot order
                                for (int s0 = 0; s0 < k; s0 += 8) {
                                    float pv[8];
#pragma unroll
                                    for (int j = 0; j < 8; ++j)
                                        pv[j] = (s0 + j < k) ? __ldcg(W.part + (int64_t)(s0 + j) * H + row) : 0.0f;
#pragma unroll
                                    for (int j = 0; j < 8; ++j)
                                        if (s0 + j < k)
                                            acc = __fmaf_rn(S.s_w[s0 + j], pv[j], acc);
                                }
                                a.y[row] = acc;
                            }
                        }
                    }
                    ++nr;
                }
            }
        } else if (warp == W_STG) {
            // ------------------------------------------------------------ h stager
            int nh = 0;
            bool ok = true;
            for (int s = 2; s < 4 && ok; ++s)
                for (int p = 0; p < S.setN[s] && ok; ++p) {
                    if (!touches(S, s, p))
                        continue;
                    const int sl = S.u_slot[S.setU[s][p]];
                    const int hsl = S.hslot_of[sl];
                    if (hsl != nh)
                        continue;
                    // every row block of the unit's h flagged in this call (lanes: row blocks lane, lane + 32)
                    for (;;) {
                        bool mine = true;
                        for (int rb = lane; rb < I / 16; rb += 32)
                            mine = mine && (uint32_t)pipe::ld_acquire(&W.hflag[sl * (I / 16) + rb]) == tag;
                        if (__all_sync(0xffffffffu, mine))
                            break;
                        if (pipe::globaltimer() > deadline) {
                            if (lane == 0)
                                set_error(W, tag, deadline, kErrTimeout, 5);
                            ok = false;
                            break;
                        }
                        __nanosleep(100);
                    }
                    if (!ok)
                        break;
                    __threadfence();
                    // h -> fragments of the down items' B operand, 128 rows per tile (all tiles' loads
                    // in flight together)
                    float4 hv4[IMAX / 128];
#pragma unroll
                    for (int q = 0; q < IMAX / 128; ++q)
                        if (q < I / 128)
                            hv4[q] = __ldcg(reinterpret_cast<const float4 *>(W.h + (int64_t)sl * I + 128 * q + 4 * lane));
#pragma unroll
                    for (int q = 0; q < IMAX / 128; ++q) {
                        if (q >= I / 128)
                            break;
                        float v[4] = {hv4[q].x, hv4[q].y, hv4[q].z, hv4[q].w};
                        float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
                        m = dev::warp_max(m);
                        const int sx = dev::fix_exponent24(m);
                        dev::frags_from_values(v, sx, S.hs[hsl] + q * 4 * dev::kFragWords);
                        if (lane == 0)
                            S.hse[hsl][q] = sx;
                    }
                    __syncwarp();
                    if (lane == 0)
                        pipe::mbar_arrive(&S.hfull[hsl]);
                    ++nh;
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
            const int t = lane & 3, gq = lane >> 2;
            // B column gq: part gq of the token's three byte columns for gq < 3, zero otherwise
            const bool fz = gq >= 3;
            const int fo = fz ? 0 : dev::frag_offset(gq, t);
            const int xstep = fz ? 0 : dev::kFragWords;
            const float lf = dev::combine24_lane_factor(t);
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
                const int sl = S.u_slot[r.u], b = S.s_b[sl];
                const unsigned char *reg = S.ring + r.off;
                float *red = S.red[nr % NREG][ii];
                // one tile loop for both kinds of item: gate/up items take two passes (gate, up)
                // of KGA k-tiles, down items one pass of KGB k-tiles
                int npass, ntl, kt0, m0, pstep, ngr, hsl = -1;
                const unsigned char *pl0;
                const float *scb;
                if (r.set < 2) {
                    const int kg0 = r.local % g.NKA, nt = r.n * KGA;
                    kt0 = (kg0 + ii) * KGA;
                    npass = 2;
                    ntl = KGA;
                    m0 = 0;
                    pstep = 2 * nt * 256;
                    pl0 = reg + ii * KGA * 256 + lane * 8;
                    ngr = H / G;
                    scb = reinterpret_cast<const float *>(reg + 2 * b * nt * 256) + gq * ngr + kt0 * (128 / G);
                } else {
                    hsl = S.hslot_of[sl];
                    if (hwait != hsl) {
                        if (!pipe::mbar_wait(&S.hfull[hsl], 0, deadline)) {
                            set_error(W, tag, deadline, kErrTimeout, 4);
                            ok = false;
                            break;
                        }
                        hwait = hsl;
                    }
                    const int nt = r.n * g.KGB, lin = r.local + ii;
                    const int rb = lin / g.NKB, rbf = r.local / g.NKB;
                    kt0 = (lin % g.NKB) * g.KGB;
                    npass = 1;
                    ntl = g.KGB;
                    m0 = 2;
                    pstep = nt * 256;
                    pl0 = reg + ii * g.KGB * 256 + lane * 8;
                    ngr = I / G;
                    scb = reinterpret_cast<const float *>(reg + b * nt * 256) + ((rb - rbf) * 16 + gq) * ngr +
                          kt0 * (128 / G);
                }
                const uint32_t *xf = fz ? S.zeros : (hsl < 0 ? S.xs : S.hs[hsl]) + fo;
                const int *xe = hsl < 0 ? S.xse : S.hse[hsl];
#pragma unroll 1
                for (int pass = 0; pass < npass; ++pass) {
                    const TabS &ts = S.tab[sl][m0 + pass];
                    const uint16_t *big = ts.big >= 0 ? S.big[ts.big] : nullptr;
                    // gate/up: plane p of matrix m at (2p + m) tile blocks; scales of up after gate's 16 rows
                    const unsigned char *pl = pl0 + pass * (pstep / 2);
                    const float *sc0 = scb + pass * 16 * ngr;
                    float a0 = 0.0f, a1 = 0.0f;
                    tiles_any<GS>(b, ntl, pl, pstep, ts, big, xf, xstep, xe, kt0, lf, sc0, sc0 + 8 * ngr,
                                  128 / G, a0, a1);
                    a0 += __shfl_down_sync(0xffffffffu, a0, 1);
                    a1 += __shfl_down_sync(0xffffffffu, a1, 1);
                    if (t == 0) {
                        red[16 * pass + gq] = a0;
                        red[16 * pass + gq + 8] = a1;
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
    }
    if (fail && blockIdx.x == 0 && tid == 0) // no work: record the error; the epoch still advances below
        set_error(W, tag, deadline, S.bad ? kErrBadPair : S.missing >= 0 ? kErrNoPlane : kErrUnsupported,
                  S.bad ? 0 : S.missing >= 0 ? S.missing : 11);
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
