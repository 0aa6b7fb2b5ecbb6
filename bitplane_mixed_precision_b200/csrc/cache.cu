// HBM prefix cache of routed experts (PagedMoE transcript cues 11, 13, 35;
// arxivlens Abstract and Methodology).
//
// One shared state per (layer, expert): the resident depth r (planes 0..r-1,
// each in a slot of the caller's device pool) and a last-use time per plane.
// An access at depth b refreshes planes 0..min(r,b)-1; a miss (r < b) copies
// only planes r..b-1 from pinned host memory (cudaMemcpyAsync on the side
// stream, one copy per plane) and the page-table entries follow on the same
// stream. A full pool evicts the resident plane with the oldest time: since a
// use refreshes a prefix, that is always the deepest plane of some entry, so
// deep planes age out first and an entry keeps a usable, shorter prefix.
// Candidates are kept in an ordered set keyed by (time of the deepest plane,
// entry); entries used in the current batch are skipped.
//
// Also here: the independent-precision baseline of transcript cue 11 (every
// (layer, expert, bits) a separate object, whole-object LRU), used to report
// the hit rate that per-precision caching would have had on the same trace;
// and host-side routing for callers that plan cache top-ups before the
// device runs (top-k + softmax, as pmoe_route).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <set>
#include <utility>
#include <vector>

#include "common.h"

namespace pmoe {

namespace {

constexpr int kStageBufs = 8;         // page-table update buffers in flight
constexpr int kStageEntries = 16384;  // updates per buffer

// Order of routing keys: larger float first, -0 equal to +0 (as the device routing's keys).
inline uint32_t ord_key_host(float f)
{
    uint32_t u;
    std::memcpy(&u, &f, 4);
    u = (u == 0x80000000u) ? 0u : u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Writes page-table entries: upd[i] = (index, value), read from mapped pinned memory.
__global__ void page_table_update_kernel(int32_t *pt, const int2 *upd, int n)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int2 u = upd[i];
        pt[u.x] = u.y;
    }
}

} // namespace

} // namespace pmoe

struct pmoe_cache {
    int L = 0, E = 0;
    int64_t slots = 0, slot_words = 0;
    uint32_t *pool = nullptr;
    int32_t *page_table = nullptr; // device, or nullptr (host-only cache)
    bool keep_log = false;

    std::vector<int32_t> pt;        // host mirror [L*E*8]
    std::vector<unsigned char> dirty; // [L*E*8]: entry changed in the current call
    std::vector<uint8_t> depth;     // [L*E]
    std::vector<int64_t> ts;        // [L*E*8] last use of each plane
    std::vector<int64_t> last_batch; // [L*E]: batch of the last access (meaningful while resident)
    std::set<std::pair<int64_t, int64_t>> order; // (time of deepest plane, entry) for resident entries
    std::vector<int32_t> free_slots;
    int64_t used = 0;
    int64_t clock = 0;
    pmoe_cache_stats stats{};
    std::vector<int64_t> log;
    int64_t fail_copy_in = 0; // > 0: the fail_copy_in-th next host-to-device copy reports failure (testing)

    // page-table updates staged in mapped pinned memory
    int2 *stage = nullptr;
    cudaEvent_t stage_ev[pmoe::kStageBufs] = {};
    bool stage_used[pmoe::kStageBufs] = {};
    int stage_next = 0;

    int64_t deepest_ts(int64_t x) const { return ts[x * 8 + depth[x] - 1]; }
};

namespace pmoe {
namespace {

void release(pmoe_cache *c)
{
    if (!c)
        return;
    for (int i = 0; i < kStageBufs; ++i)
        if (c->stage_ev[i])
            cudaEventDestroy(c->stage_ev[i]);
    if (c->stage)
        cudaFreeHost(c->stage);
    delete c;
}

// Flushes staged page-table updates to the device on stream st.
pmoe_status flush_updates(pmoe_cache *c, const std::vector<int2> &upd, cudaStream_t st)
{
    for (size_t off = 0; off < upd.size(); off += kStageEntries) {
        const int n = (int)std::min<size_t>(kStageEntries, upd.size() - off);
        const int b = c->stage_next;
        c->stage_next = (b + 1) % kStageBufs;
        if (c->stage_used[b])
            PMOE_CUDA(cudaEventSynchronize(c->stage_ev[b])); // the buffer's last kernel has read it
        int2 *buf = c->stage + (size_t)b * kStageEntries;
        std::memcpy(buf, upd.data() + off, sizeof(int2) * (size_t)n);
        page_table_update_kernel<<<(n + 255) / 256, 256, 0, st>>>(c->page_table, buf, n);
        PMOE_TRY(launch_status());
        PMOE_CUDA(cudaEventRecord(c->stage_ev[b], st));
        c->stage_used[b] = true;
    }
    return PMOE_OK;
}

} // namespace
} // namespace pmoe

using namespace pmoe;

extern "C" {

pmoe_status pmoe_cache_create(int layers, int experts, int64_t slots, int64_t slot_words, uint32_t *pool,
                              int32_t *page_table, int keep_log, pmoe_cache **out)
{
    if (!out || layers <= 0 || experts <= 0 || slots <= 0 || slot_words <= 0 || slot_words % 4 ||
        (pool == nullptr) != (page_table == nullptr) || (int64_t)layers * experts * 8 > INT32_MAX ||
        slots > INT32_MAX || (pool && !aligned(pool, 16)))
        return PMOE_ERR_INVALID_ARG;
    *out = nullptr;
    pmoe_cache *c = new (std::nothrow) pmoe_cache();
    if (!c)
        return PMOE_ERR_INVALID_ARG;
    const int64_t NE = (int64_t)layers * experts;
    c->L = layers;
    c->E = experts;
    c->slots = slots;
    c->slot_words = slot_words;
    c->pool = pool;
    c->page_table = page_table;
    c->keep_log = keep_log != 0;
    try {
        c->pt.assign((size_t)NE * 8, -1);
        c->dirty.assign((size_t)NE * 8, 0);
        c->depth.assign((size_t)NE, 0);
        c->ts.assign((size_t)NE * 8, 0);
        c->last_batch.assign((size_t)NE, 0);
        c->free_slots.resize((size_t)slots);
    } catch (...) {
        release(c);
        return PMOE_ERR_INVALID_ARG;
    }
    for (int64_t s = 0; s < slots; ++s) // popped from the back: slot 0 first
        c->free_slots[(size_t)s] = (int32_t)(slots - 1 - s);
    if (page_table) {
        cudaError_t e = cudaHostAlloc(reinterpret_cast<void **>(&c->stage),
                                      sizeof(int2) * (size_t)kStageBufs * kStageEntries,
                                      cudaHostAllocMapped | cudaHostAllocPortable);
        for (int i = 0; e == cudaSuccess && i < kStageBufs; ++i)
            e = cudaEventCreateWithFlags(&c->stage_ev[i], cudaEventDisableTiming);
        if (e == cudaSuccess)
            e = cudaMemset(page_table, 0xff, sizeof(int32_t) * (size_t)NE * 8);
        if (e == cudaSuccess)
            e = cudaDeviceSynchronize();
        if (e != cudaSuccess) {
            set_cuda_error(e);
            release(c);
            return PMOE_ERR_CUDA;
        }
    }
    *out = c;
    return PMOE_OK;
}

pmoe_status pmoe_cache_destroy(pmoe_cache *c)
{
    if (!c)
        return PMOE_ERR_INVALID_ARG;
    for (int i = 0; i < kStageBufs; ++i)
        if (c->stage_used[i])
            cudaEventSynchronize(c->stage_ev[i]);
    release(c);
    return PMOE_OK;
}

pmoe_status pmoe_cache_extend(pmoe_cache *c, int layer, const int32_t *experts, const uint8_t *need, int n,
                              int64_t batch, const uint32_t *const *host_planes, pmoe_stream side,
                              pmoe_event after, pmoe_event done, uint8_t *resident_before,
                              pmoe_cache_stats *stats)
{
    if (!c || n < 0 || (n > 0 && (!experts || !need)) || layer < 0 || layer >= c->L)
        return PMOE_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (experts[i] < 0 || experts[i] >= c->E || need[i] < 1 || need[i] > 8)
            return PMOE_ERR_INVALID_ARG;
    const bool moves = c->page_table != nullptr;
    const uint32_t *src = nullptr;
    if (moves) {
        if (!host_planes || !host_planes[layer])
            return PMOE_ERR_INVALID_ARG;
        src = host_planes[layer];
    }
    cudaStream_t st = (cudaStream_t)side;
    std::vector<int> touched; // page-table entries changed by this call (each once)
    auto touch = [&](size_t k) {
        if (moves && !c->dirty[k]) {
            c->dirty[k] = 1;
            touched.push_back((int)k);
        }
    };
    bool waited_after = false; // `side` waits for `after` before the first copy into an evicted slot
    pmoe_status rc = PMOE_OK;
    // Enqueues one plane copy; the testing hook can make it report failure without enqueueing.
    auto copy_plane = [&](int32_t slot, int64_t from) -> pmoe_status {
        if (c->fail_copy_in > 0 && --c->fail_copy_in == 0) {
            set_cuda_error(cudaErrorInvalidValue);
            return PMOE_ERR_CUDA;
        }
        return cuda_status(cudaMemcpyAsync(c->pool + (int64_t)slot * c->slot_words, src + from,
                                           (size_t)c->slot_words * 4, cudaMemcpyHostToDevice, st));
    };

    for (int i = 0; i < n; ++i) {
        const int e = experts[i], b = need[i];
        const int64_t x = (int64_t)layer * c->E + e;
        const int r = c->depth[(size_t)x];
        // what this access changes on the entry, so that a failed copy can take it back
        int64_t old_ts[8];
        for (int p = 0; p < 8; ++p)
            old_ts[p] = c->ts[(size_t)x * 8 + p];
        const int64_t old_batch = c->last_batch[(size_t)x];
        const int64_t now = c->clock++;
        if (resident_before)
            resident_before[i] = (uint8_t)r;
        c->stats.requests += 1;
        c->last_batch[(size_t)x] = batch;
        if (r > 0)
            c->order.erase({c->deepest_ts(x), x});
        if (r >= b) {
            c->stats.hits += 1;
            for (int p = 0; p < b; ++p)
                c->ts[(size_t)x * 8 + p] = now;
            c->order.insert({c->deepest_ts(x), x});
            continue;
        }
        for (int p = 0; p < r; ++p)
            c->ts[(size_t)x * 8 + p] = now;
        const int want = b - r;
        bool evicted_here = false;
        // evict the oldest deepest planes of entries outside this batch until the suffix fits
        while (c->used + want > c->slots) {
            auto it = c->order.begin();
            while (it != c->order.end() && c->last_batch[(size_t)it->second] == batch)
                ++it;
            if (it == c->order.end()) {
                rc = PMOE_ERR_OUT_OF_SLOTS;
                break;
            }
            const int64_t y = it->second;
            c->order.erase(it);
            const int p = --c->depth[(size_t)y];
            const size_t k = (size_t)y * 8 + p;
            c->free_slots.push_back(c->pt[k]);
            c->pt[k] = -1;
            touch(k);
            c->used -= 1;
            c->stats.planes_evicted += 1;
            if (c->keep_log)
                c->log.push_back(y * 8 + p);
            if (c->depth[(size_t)y] > 0)
                c->order.insert({c->deepest_ts(y), y});
            evicted_here = true;
        }
        if (rc != PMOE_OK) {
            if (r > 0)
                c->order.insert({c->deepest_ts(x), x});
            break;
        }
        if (moves && evicted_here && after && !waited_after) {
            rc = cuda_status(cudaStreamWaitEvent(st, (cudaEvent_t)after, 0));
            waited_after = rc == PMOE_OK;
        }
        int p_ok = r; // planes r..p_ok-1 have their copies enqueued
        for (int p = r; p < b && rc == PMOE_OK; ++p) {
            const int32_t slot = c->free_slots.back();
            if (moves)
                rc = copy_plane(slot, ((int64_t)e * 8 + p) * c->slot_words);
            if (rc != PMOE_OK)
                break;
            c->free_slots.pop_back();
            const size_t k = (size_t)x * 8 + p;
            c->pt[k] = slot;
            c->ts[k] = now;
            touch(k);
            p_ok = p + 1;
        }
        if (rc != PMOE_OK) {
            // a copy could not be enqueued: this access is taken back. Its planes whose copies were
            // enqueued go back to the free list (their data lands in free slots); the entry keeps
            // its depth, times and batch as before the access; the evictions above stay (the
            // enqueued copies may have overwritten evicted slots).
            for (int p = p_ok - 1; p >= r; --p) {
                const size_t k = (size_t)x * 8 + p;
                c->free_slots.push_back(c->pt[k]);
                c->pt[k] = -1;
            }
            for (int p = 0; p < 8; ++p)
                c->ts[(size_t)x * 8 + p] = old_ts[p];
            c->last_batch[(size_t)x] = old_batch;
            c->stats.requests -= 1;
            if (r > 0)
                c->order.insert({c->deepest_ts(x), x});
            break;
        }
        c->depth[(size_t)x] = (uint8_t)b;
        c->used += want;
        c->stats.planes_fetched += want;
        c->stats.bytes_fetched += (int64_t)want * c->slot_words * 4;
        c->order.insert({c->deepest_ts(x), x});
    }

    // the device page table follows the host state, also after an error: entries changed by
    // this call are written once, with their final value
    std::vector<int2> upd;
    upd.reserve(touched.size());
    for (int k : touched) {
        upd.push_back(make_int2(k, c->pt[(size_t)k]));
        c->dirty[(size_t)k] = 0;
    }
    if (moves && !upd.empty()) {
        const pmoe_status f = flush_updates(c, upd, st);
        if (rc == PMOE_OK)
            rc = f;
    }
    if (moves && done) {
        const pmoe_status f = cuda_status(cudaEventRecord((cudaEvent_t)done, st));
        if (rc == PMOE_OK)
            rc = f;
    }
    if (stats)
        *stats = c->stats;
    return rc;
}

pmoe_status pmoe_cache_inject_copy_failure(pmoe_cache *c, int64_t nth)
{
    if (!c || nth < 0)
        return PMOE_ERR_INVALID_ARG;
    c->fail_copy_in = nth;
    return PMOE_OK;
}

pmoe_status pmoe_cache_get_stats(const pmoe_cache *c, pmoe_cache_stats *stats)
{
    if (!c || !stats)
        return PMOE_ERR_INVALID_ARG;
    *stats = c->stats;
    return PMOE_OK;
}

pmoe_status pmoe_cache_resident_depth(const pmoe_cache *c, int layer, uint8_t *depth)
{
    if (!c || !depth || layer < 0 || layer >= c->L)
        return PMOE_ERR_INVALID_ARG;
    std::memcpy(depth, c->depth.data() + (size_t)layer * c->E, (size_t)c->E);
    return PMOE_OK;
}

pmoe_status pmoe_cache_eviction_log(const pmoe_cache *c, int64_t *log, int64_t cap, int64_t *n)
{
    if (!c || !n || cap < 0 || (cap > 0 && !log))
        return PMOE_ERR_INVALID_ARG;
    if (!c->keep_log)
        return PMOE_ERR_UNSUPPORTED;
    const int64_t m = (int64_t)c->log.size();
    std::memcpy(log, c->log.data(), sizeof(int64_t) * (size_t)std::min(m, cap));
    *n = m;
    return PMOE_OK;
}

pmoe_status pmoe_cache_sim_independent(int layers, int experts, int64_t cap_planes, int64_t n,
                                       const int32_t *layer, const int32_t *expert, const uint8_t *need,
                                       const int64_t *batch, uint8_t *hit, int64_t *planes_fetched)
{
    if (layers <= 0 || experts <= 0 || cap_planes <= 0 || n < 0 || !planes_fetched ||
        (n > 0 && (!layer || !expert || !need || !batch || !hit)))
        return PMOE_ERR_INVALID_ARG;
    for (int64_t a = 0; a < n; ++a)
        if (layer[a] < 0 || layer[a] >= layers || expert[a] < 0 || expert[a] >= experts || need[a] < 1 ||
            need[a] > 8)
            return PMOE_ERR_INVALID_ARG;
    // object id = ((layer * E) + expert) * 8 + (bits - 1); LRU set keyed by (last use, object)
    const int64_t NO = (int64_t)layers * experts * 8;
    std::vector<int64_t> last(NO, -1), obj_batch(NO, 0);
    std::set<std::pair<int64_t, int64_t>> lru;
    int64_t used = 0, fetched = 0;
    pmoe_status rc = PMOE_OK;
    for (int64_t a = 0; a < n && rc == PMOE_OK; ++a) {
        const int b = need[a];
        const int64_t o = ((int64_t)layer[a] * experts + expert[a]) * 8 + (b - 1);
        obj_batch[o] = batch[a];
        if (last[o] >= 0) {
            hit[a] = 1;
            lru.erase({last[o], o});
            last[o] = a;
            lru.insert({a, o});
            continue;
        }
        hit[a] = 0;
        while (used + b > cap_planes) {
            auto it = lru.begin();
            while (it != lru.end() && obj_batch[it->second] == batch[a])
                ++it;
            if (it == lru.end()) {
                rc = PMOE_ERR_OUT_OF_SLOTS;
                break;
            }
            const int64_t y = it->second;
            used -= (y % 8) + 1;
            last[y] = -1;
            lru.erase(it);
        }
        if (rc != PMOE_OK)
            break;
        last[o] = a;
        lru.insert({a, o});
        used += b;
        fetched += b;
    }
    *planes_fetched = fetched;
    return rc;
}

pmoe_status pmoe_cache_sim_independent_down(int layers, int experts, int64_t cap_planes, int64_t n,
                                            const int32_t *layer, const int32_t *expert, const uint8_t *need,
                                            const int64_t *batch, uint8_t *hit, int64_t *planes_fetched)
{
    if (layers <= 0 || experts <= 0 || cap_planes <= 0 || n < 0 || !planes_fetched ||
        (n > 0 && (!layer || !expert || !need || !batch || !hit)))
        return PMOE_ERR_INVALID_ARG;
    for (int64_t a = 0; a < n; ++a)
        if (layer[a] < 0 || layer[a] >= layers || expert[a] < 0 || expert[a] >= experts || need[a] < 1 ||
            need[a] > 8)
            return PMOE_ERR_INVALID_ARG;
    // one copy per (layer, expert): its depth, last use and batch; LRU set of resident copies
    const int64_t NE = (int64_t)layers * experts;
    std::vector<uint8_t> depth(NE, 0);
    std::vector<int64_t> last(NE, 0), obj_batch(NE, 0);
    std::set<std::pair<int64_t, int64_t>> lru;
    int64_t used = 0, fetched = 0;
    pmoe_status rc = PMOE_OK;
    for (int64_t a = 0; a < n && rc == PMOE_OK; ++a) {
        const int b = need[a];
        const int64_t x = (int64_t)layer[a] * experts + expert[a];
        obj_batch[x] = batch[a];
        if (depth[x] > 0)
            lru.erase({last[x], x});
        last[x] = a;
        if (depth[x] >= b) {
            hit[a] = 1;
            lru.insert({a, x});
            continue;
        }
        hit[a] = 0;
        used -= depth[x]; // promotion replaces the old copy
        depth[x] = 0;
        while (used + b > cap_planes) {
            auto it = lru.begin();
            while (it != lru.end() && obj_batch[it->second] == batch[a])
                ++it;
            if (it == lru.end()) {
                rc = PMOE_ERR_OUT_OF_SLOTS;
                break;
            }
            used -= depth[it->second];
            depth[it->second] = 0;
            lru.erase(it);
        }
        if (rc != PMOE_OK)
            break;
        depth[x] = (uint8_t)b;
        lru.insert({a, x});
        used += b;
        fetched += b;
    }
    *planes_fetched = fetched;
    return rc;
}

pmoe_status pmoe_route_host(const float *logits, int T, int E, int k, int32_t *ids, float *w)
{
    if (!logits || !ids || !w || T < 0 || k < 1 || k > 32 || E < k || E > 4096)
        return PMOE_ERR_INVALID_ARG;
    std::vector<unsigned char> taken((size_t)E);
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (int64_t)t * E;
        std::fill(taken.begin(), taken.end(), 0);
        double ex[32];
        for (int s = 0; s < k; ++s) {
            int best = -1;
            for (int j = 0; j < E; ++j) {
                if (taken[(size_t)j])
                    continue;
                // ties to the lower id
                if (best < 0 || ord_key_host(l[j]) > ord_key_host(l[best]))
                    best = j;
            }
            taken[(size_t)best] = 1;
            ids[t * k + s] = best;
        }
        const double l0 = (double)l[ids[t * k]];
        double sum = 0.0;
        for (int s = 0; s < k; ++s) {
            ex[s] = std::exp((double)l[ids[t * k + s]] - l0);
            sum += ex[s];
        }
        for (int s = 0; s < k; ++s)
            w[t * k + s] = (float)(ex[s] / sum);
    }
    return PMOE_OK;
}

} // extern "C"
