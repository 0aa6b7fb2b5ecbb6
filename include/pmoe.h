/*
 * pmoe.h — C ABI of libpmoe: direct execution of bitplane prefixes of routed
 * MoE experts on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages on PagedMoE, cited by page and section):
 *   [T#n] "PagedMoE: Cross-Precision Expert Caching for SSD-Resident MoE
 *         Inference", podcast transcript, subtitle cue n.
 *   [A]   "PagedMoE: Cross-Precision Expert Caching for Token-Level Dynamic
 *         Precision in SSD-Resident MoE Inference", arxivlens page, Abstract
 *         and Methodology.
 *
 * Conventions for every entry point:
 *   - Pointers are plain host or device pointers, as stated per argument.
 *     All memory is owned by the caller; no entry point frees or keeps a
 *     pointer after it returns, except the cache object (pmoe_cache_*),
 *     which keeps the device pool and page-table pointers given at creation.
 *   - Calls that take a stream are asynchronous on it. Argument errors that
 *     the host can see are returned before anything is enqueued, and then
 *     nothing has been written.
 *   - No entry point allocates device memory. Scratch is passed in by the
 *     caller (workspace arguments) with the size given by the matching
 *     *_workspace_bytes query.
 *   - Return value: PMOE_OK or an error code below; pmoe_status_string()
 *     names it. PMOE_ERR_CUDA means a CUDA call (launch or copy) failed;
 *     pmoe_last_cuda_error() returns its cudaError_t value.
 *
 * Stored format of one expert matrix W (N rows x K columns) [T#19-#27, A]:
 *   - codebook: 510 float32, the binary tree of a 256-entry sorted codebook;
 *     depth d (1..8) node i at offset (1<<d)-2+i; truncating an 8-bit index
 *     to its top b bits names its depth-b ancestor [T#21].
 *   - scales: float32 [N][K/G], one per row and group of G columns.
 *   - planes: 8 bitplanes of the 8-bit indices, MSB first: plane p holds bit
 *     (7-p) of every index, so a depth-b read touches planes 0..b-1 only
 *     [T#25]. Each plane is N*K/32 uint32 words; weight (n,k) of plane p is
 *       tile = (n/16)*(K/128) + k/128, rr = n%16, kk = k%128,
 *       g = rr%8, u = rr/8, s = kk/32, half = (kk%32)/16, t = (kk%16)/4,
 *       i = kk%4, j = 4*half + i, L = 4*g + t, q = 2*s + u, h = q/4, r = q%4,
 *       word = tile*64 + 2*L + h, bit = (4*j + p + r) mod 32.
 *     (16x128 tiles; inside a tile lane L of a warp owns words 2L, 2L+1, and
 *     the bit order lets a lane assemble 4-bit prefix indices with one AND
 *     per plane and one rotate.) N % 16 == 0 and K % 128 == 0.
 *   - The depth-b value of weight (n,k) is scales[n][k/G] * C[b][code>>(8-b)].
 */
#ifndef PMOE_H
#define PMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PMOE_API __attribute__((visibility("default")))
#else
#define PMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pmoe_stream; /* a cudaStream_t; NULL = legacy default stream */
typedef struct CUevent_st *pmoe_event;   /* a cudaEvent_t */

typedef enum {
    PMOE_OK = 0,
    PMOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, shape or alignment */
    PMOE_ERR_CUDA = 2,         /* a CUDA runtime call failed */
    PMOE_ERR_OUT_OF_SLOTS = 3, /* the prefix cache cannot hold the request */
    PMOE_ERR_BUDGET = 4,       /* infeasible bit budget */
    PMOE_ERR_WORKSPACE = 5,    /* workspace too small */
    PMOE_ERR_TIMEOUT = 6,      /* a bounded device wait ran out (see pmoe_moe_layer_fwd) */
    PMOE_ERR_UNSUPPORTED = 7   /* shape or option this build does not handle */
} pmoe_status;

PMOE_API const char *pmoe_status_string(pmoe_status s);
PMOE_API int pmoe_last_cuda_error(void);
PMOE_API int pmoe_version(void);

/* ------------------------------------------------------------------ */
/* Format                                                              */
/* ------------------------------------------------------------------ */

/*
 * pmoe_tree_codebook [T#19, T#21]: the tree codebook of N(0,1) values cut into
 * 256 equiprobable bins: depth-d node i = conditional mean of N(0,1) on the
 * quantile interval [i/2^d, (i+1)/2^d) (children have equal mass, so each
 * parent is the mean of its children). Host only, synchronous.
 *   codebook: host float[510], written. Returns PMOE_ERR_INVALID_ARG if NULL.
 */
PMOE_API pmoe_status pmoe_tree_codebook(float *codebook);

/*
 * pmoe_tree_codebook_from_leaves [T#19, T#21]: the tree codebook of a sorted
 * 256-entry leaf table (for example a per-block K-means codebook): the leaves
 * are depth 8, and every parent is the frequency-weighted mean of its two
 * children, carrying the sum of their frequencies (a pair with both
 * frequencies zero gets the plain mean). Computed in double level by level,
 * stored as float. Host only, synchronous.
 *   leaves: host float[256], ascending. freq: host float[256], >= 0 (e.g. how
 *   many weights each leaf quantises). codebook: host float[510], written.
 *   Returns PMOE_ERR_INVALID_ARG for NULL, unsorted leaves, a negative or
 *   non-finite value.
 */
PMOE_API pmoe_status pmoe_tree_codebook_from_leaves(const float *leaves, const float *freq, float *codebook);

/*
 * pmoe_quantize: per-group scale and 8-bit index of every weight for the
 * Gaussian tree codebook. scale = population std (double, sequential sum,
 * rounded to float; 0 -> 1) of the G weights of a row group; index = number
 * of thresholds Phi^-1(i/256), i = 1..255, at or below w/scale (double).
 *   w: device float [N*K] row-major. scales: device float [N*(K/G)].
 *   codes: device uint8 [N*K]. G divides K; N, K > 0.
 */
PMOE_API pmoe_status pmoe_quantize(const float *w, int N, int K, int G, float *scales, uint8_t *codes,
                          pmoe_stream stream);

/*
 * pmoe_pack_bitplanes [T#25, A]: writes planes 0..depth-1 of the codes in the
 * layout above. Plane p starts at planes + p*plane_stride_words
 * (plane_stride_words >= N*K/32; it lets a caller pack straight into a slot
 * pool). on_device = 1: codes and planes are device pointers, a warp-ballot
 * kernel runs on the stream; 0: host pointers, synchronous host loop.
 *   N % 16 == 0, K % 128 == 0, 1 <= depth <= 8.
 */
PMOE_API pmoe_status pmoe_pack_bitplanes(const uint8_t *codes, int N, int K, int depth, uint32_t *planes,
                                int64_t plane_stride_words, int on_device, pmoe_stream stream);

/*
 * pmoe_extract_prefix [T#21, T#25]: reads planes 0..b-1 the way the GEMV
 * kernels do and writes the b-bit prefix index code>>(8-b) of every weight.
 * Device pointers. idx: device uint8 [N*K] row-major. 1 <= b <= 8.
 */
PMOE_API pmoe_status pmoe_extract_prefix(const uint32_t *planes, int64_t plane_stride_words, int N, int K,
                                int b, uint8_t *idx, pmoe_stream stream);

/* ------------------------------------------------------------------ */
/* Routing and prefix selection                                        */
/* ------------------------------------------------------------------ */

/*
 * pmoe_route [T#4]: per token, the k largest logits (ties to the lower expert
 * id) in descending order, and their softmax weights: exp(l - l_max)/sum in
 * double, rounded to float. Device pointers: logits float [T*E],
 * ids int32 [T*k], w float [T*k]. 1 <= k <= 32, k <= E <= 4096.
 */
PMOE_API pmoe_status pmoe_route(const float *logits, int T, int E, int k, int32_t *ids, float *w,
                       pmoe_stream stream);

/*
 * pmoe_select_prefix [T#29, T#31, A]: per token, depth b_i in 1..8 for each
 * of its k experts minimising sum w_i^2 * s_e^2 * 4^-b_i under
 * sum b_i = B = floor(avg_bits*k + 1e-4) clamped to [k, 8k]: all start at 1
 * bit; B-k times the expert with the largest w_i*s_e*2^-b_i (float product,
 * exact ldexp compares, ties to the lower slot, 8-bit experts skipped) gets
 * one more bit. The same as b = clamp(ceil(c + log2(w*s/geomean)), 1, 8)
 * with the offset c that spends the budget.
 *   w float [T*k], ids int32 [T*k], sens float [E] (indexed by ids),
 *   depth uint8 [T*k] out. on_device = 1: device pointers, async on stream;
 *   0: host pointers, synchronous. 1 <= k <= 32.
 */
PMOE_API pmoe_status pmoe_select_prefix(const float *w, const int32_t *ids, const float *sens, int T, int k,
                               float avg_bits, uint8_t *depth, int on_device, pmoe_stream stream);

/*
 * pmoe_select_prefix_cache_aware [T#61]: the allocator budgeted in planes to
 * fetch instead of bits requested. Per token, with resident[t*k+i] the depth
 * already cached for slot i's expert: each slot starts at max(1, resident)
 * (cached planes cost nothing; a slot with nothing cached needs its first
 * plane, one fetch), then while fewer than fetch_budget planes are fetched,
 * the slot with the largest w*s_e*2^-b below 8 bits (ties to the lower slot)
 * gets one more plane. Host pointers, synchronous: w float [T*k], ids int32
 * [T*k], sens float [E], resident uint8 [T*k], depth uint8 [T*k] out.
 */
PMOE_API pmoe_status pmoe_select_prefix_cache_aware(const float *w, const int32_t *ids, const float *sens,
                                                    const uint8_t *resident, int T, int k, int fetch_budget,
                                                    uint8_t *depth);

/*
 * pmoe_select_prefix_cache_aware_matched [T#29, T#61]: the cache-aware
 * allocator with its budget matched to the cache-oblivious one, per token:
 * the depths pmoe_select_prefix(avg_bits) would pick determine the planes
 * they would fetch given resident[], and that count is the fetch budget of
 * pmoe_select_prefix_cache_aware, whose depths are returned. Both choices
 * therefore move the same bytes; resident planes come free.
 *   Host pointers, synchronous; arguments as pmoe_select_prefix_cache_aware.
 *   surrogate: NULL, or host double[2] to which the call adds the error
 *   surrogate sum of (w*s_e)^2 * 4^-b over its slots, [0] for the
 *   cache-oblivious depths and [1] for the returned ones (w*s_e in double).
 */
PMOE_API pmoe_status pmoe_select_prefix_cache_aware_matched(const float *w, const int32_t *ids, const float *sens,
                                                            const uint8_t *resident, int T, int k, float avg_bits,
                                                            uint8_t *depth, double *surrogate);

/*
 * Profile-driven allocation [T#29, T#31]./*
 * Profile-driven allocation [T#29, T#31]. An expert's error profile E_e(b),
 * b = 1..8, is its relative output error at depth b, measured offline on
 * random Gaussian inputs; the allocator then grants bits by the profile's
 * gains instead of the closed form s_e^2 4^-b.
 *
 * pmoe_relative_error: err[0] = mean over the T rows of
 *   ||y_t - ref_t||^2 / ||ref_t||^2 (double sums, fixed order). Device
 *   pointers: y, ref float [T*H], err float [1]. Async on the stream.
 * pmoe_profile_repair (host, synchronous): raw float [n][8] (entry b-1 =
 *   E(b)) -> table float [n][8]: the gains E(b)-E(b+1) are replaced by their
 *   least-squares non-increasing fit (pool adjacent violators), clamped at 0,
 *   and the profile is rebuilt from E(8) upward, so that greedy allocation
 *   grants bit b+1 of an expert only after bit b.
 * pmoe_select_prefix_table: as pmoe_select_prefix, with the gain of giving a
 *   slot its (b+1)-th bit = (w*w) * (E_e(b) - E_e(b+1)) in float (ties to the
 *   lower slot). table float [E][8] (host or device with on_device).
 */
PMOE_API pmoe_status pmoe_relative_error(const float *y, const float *ref, int T, int H, float *err,
                                         pmoe_stream stream);
PMOE_API pmoe_status pmoe_profile_repair(const float *raw, int n, float *table);
PMOE_API pmoe_status pmoe_select_prefix_table(const float *w, const int32_t *ids, const float *table, int T, int k,
                                              float avg_bits, uint8_t *depth, int on_device, pmoe_stream stream);

/* ------------------------------------------------------------------ */
/* Execution                                                           */
/* ------------------------------------------------------------------ */

/* One stored expert matrix (device pointers). */
typedef struct {
    const uint32_t *planes;     /* plane p at planes + p*plane_stride_words */
    int64_t plane_stride_words; /* >= N*K/32 */
    const float *scales;        /* [N][K/G] */
    const float *codebook;      /* [510] */
    int N, K, G;                /* N%16 == 0, K%128 == 0, G in {32, 64, 128} */
} pmoe_matrix;

/*
 * pmoe_expert_gemv [T#37, A: Methodology]: y[n] = sum_k scales[n][k/G] *
 * C[b][code>>(8-b)] * x[k], reading only planes 0..b-1 and decoding in
 * registers (no dequantised matrix is written).
 *   x: device, K values, bf16 if x_is_bf16 else float32. y: device float [N].
 *   1 <= b <= 8. Numerics: weights and x are carried as 16-bit fixed point
 *   (power-of-two scales per table and per 128 columns), products summed
 *   exactly in int32 per group, groups in float32.
 */
PMOE_API pmoe_status pmoe_expert_gemv(const pmoe_matrix *m, int b, const void *x, int x_is_bf16, float *y,
                             pmoe_stream stream);

/*
 * One MoE layer's experts in a plane-slot pool (device pointers).
 * A slot holds plane p of one expert for all three matrices:
 *   [gate plane (I x H) | up plane (I x H) | down plane (H x I)], each H*I/32
 * words, at pool + slot*slot_words. slot_of[e*8 + p] is the slot of plane p
 * of expert e, or -1 if absent (a depth-b read needs planes 0..b-1 present).
 * scales: per expert 3 matrices back to back: gate [I][H/G], up [I][H/G],
 * down [H][I/G]. codebooks: per expert 3 x 510 floats (gate, up, down).
 */
typedef struct {
    int E, H, I, G;           /* H%128 == 0, I%128 == 0, G in {32, 64, 128} */
    const uint32_t *pool;
    int64_t slot_words;       /* >= 3*H*I/32 */
    const int32_t *slot_of;   /* [E*8] */
    const float *scales;      /* [E][2*I*(H/G) + H*(I/G)] */
    const float *codebooks;   /* [E][3][510] */
} pmoe_layer;

/* Workspace needed by pmoe_moe_layer_fwd / pmoe_moe_decode_step for T tokens, top-k. */
PMOE_API size_t pmoe_layer_workspace_bytes(int T, int k, int E, int H, int I);

/*
 * pmoe_moe_layer_fwd [T#4, T#37, A]: for each token t and slot i with expert
 * e = ids[t*k+i] at depth b = depth[t*k+i]:
 *   g = Wg_b x_t, u = Wu_b x_t, h = silu(g)*u, y_t += w[t*k+i] * (Wd_b h),
 * with (token, expert) pairs grouped by expert so that tokens at different
 * depths of one expert share one read of the planes they have in common.
 *   x: device bf16 [T*H]. ids, w, depth: device [T*k]. y: device float [T*H]
 *   (overwritten). ws: device scratch of >= pmoe_layer_workspace_bytes().
 *   Expert ids must be distinct within a token. Output is deterministic (the
 *   k contributions are summed in slot order). T*k <= 2048.
 *   Shapes: H % 1024 == 0, H <= 4096, I % 256 == 0, I <= 1024 (else
 *   PMOE_ERR_UNSUPPORTED). Errors found on the device (an expert id or depth
 *   out of range, a plane without a slot, a bounded wait that ran out) do not
 *   stop the call; they are recorded in the workspace: see pmoe_layer_error.
 */
PMOE_API pmoe_status pmoe_moe_layer_fwd(const pmoe_layer *L, const uint16_t *x, const int32_t *ids,
                               const float *w, const uint8_t *depth, int T, int k, float *y,
                               void *ws, size_t ws_bytes, pmoe_stream stream);

/*
 * pmoe_moe_layer_fwd_noalloc: the same layer call as pmoe_moe_layer_fwd for
 * callers that cannot hand the library a device allocation for scratch, for
 * example an engine that owns all device memory in a fixed pool and forbids
 * libraries from allocating, or code whose memory budget is fixed before the
 * library is called. The PagedMoE pages have no counterpart of this entry
 * point; it only changes where the scratch lives.
 *   Scratch: a fixed array of pmoe_noalloc_scratch_bytes() bytes inside the
 *   library's device image. Every GPU that loads the library holds it until
 *   the process exits. The call itself allocates nothing (no cudaMalloc, no
 *   cudaFree, no allocating library routine).
 *   Limit: T, k, H, I must need at most that many workspace bytes
 *   (pmoe_layer_workspace_bytes); larger requests return PMOE_ERR_WORKSPACE.
 *   First call on a device: looks up the array's device address once
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   Sharing: all calls on a device use the same array and it keeps the last
 *   call's contents; each call resets what must start at zero. Calls that
 *   overlap on the GPU (other streams, or without ordering between them)
 *   race on the array and give wrong results. Errors the kernels record
 *   there are read with pmoe_noalloc_layer_error.
 *   The array's device address is looked up once per device and kept: do
 *   not use the library across a reset of the device (cudaDeviceReset).
 * Arguments as pmoe_moe_layer_fwd, without ws and ws_bytes.
 */
PMOE_API size_t pmoe_noalloc_scratch_bytes(void);
/* pmoe_layer_error for the allocation-free call's array (synchronises the stream). */
PMOE_API pmoe_status pmoe_noalloc_layer_error(int *code, int *detail, pmoe_stream stream);
PMOE_API pmoe_status pmoe_moe_layer_fwd_noalloc(const pmoe_layer *L, const uint16_t *x, const int32_t *ids,
                                                const float *w, const uint8_t *depth, int T, int k, float *y,
                                                pmoe_stream stream);

/*
 * pmoe_set_tc_min_tokens: pairs at depth <= 4 that an expert needs in one
 * layer call (of T >= 8 tokens) before its tensor-core units take them
 * (process-wide; default 8). n >= 8 sets it, 0 sends every pair to the
 * persistent kernel; INVALID_ARG for 1..7 (the workspace is sized for units
 * of at least 8 pairs).
 */
PMOE_API pmoe_status pmoe_set_tc_min_tokens(int n);

/*
 * pmoe_layer_counts: how the last layer call that used workspace ws grouped
 * its pairs (synchronises the stream): counts[0] column blocks and counts[1]
 * expert units of the persistent kernel, counts[2] tensor-core units (experts
 * hit by at least 8 pairs at depth <= 4, see pmoe_set_tc_min_tokens; batches
 * of T >= 8 tokens), counts[3]
 * their operand rows (pairs padded to multiples of 16 per unit).
 */
PMOE_API pmoe_status pmoe_layer_counts(const void *ws, int *counts, pmoe_stream stream);

/*
 * pmoe_tc_selfcheck: checks the tensor-core operand path that the batched
 * layer uses for experts hit by many tokens (tcgen05 MMA, f16 operands in
 * shared memory, fp32 accumulator in tensor memory). Computes
 * D[128 x N] = A[128 x K] * B[N x K]^T on the device with the same operand
 * layout, descriptors, MMA, completion and tensor-memory loads as the layer's
 * kernel. A, B: device, row-major f16 (bit patterns as uint16), 16-byte
 * aligned; D: device fp32, row-major. 16 <= N <= 64, N % 16 == 0;
 * 32 <= K <= 128, K % 32 == 0. Asynchronous on stream; INVALID_ARG for other
 * shapes or null pointers.
 */
PMOE_API pmoe_status pmoe_tc_selfcheck(const uint16_t *A, const uint16_t *B, float *D, int N, int K,
                                       pmoe_stream stream);

/*
 * pmoe_layer_error: reads the device-side error record of the last layer call
 * that used workspace ws (synchronises the stream). code: 0 none, 1 expert id
 * or depth out of range, 2 a needed plane has no slot (detail = e*8 + plane),
 * 3 a bounded wait inside the kernel ran out (detail = where).
 */
PMOE_API pmoe_status pmoe_layer_error(const void *ws, int *code, int *detail, pmoe_stream stream);

/*
 * pmoe_set_wait_limit_ns: bound of every wait inside the layer kernels of
 * later pmoe_moe_layer_fwd / pmoe_moe_decode_step calls (process-wide): each
 * launch gives up on any wait once this many nanoseconds have passed since it
 * started, records error 3 (see pmoe_layer_error) and finishes. Waits for the
 * kernel's own copies to land before it exits have a separate bound, 200 ms
 * past that one.
 * 0 restores the default of 200 ms. Host only; the kernels stay correct with
 * any limit that is not reached.
 */
PMOE_API pmoe_status pmoe_set_wait_limit_ns(uint64_t ns);

/*
 * pmoe_moe_decode_step: the whole hot path for T tokens on the device:
 * pmoe_route, then pmoe_select_prefix (sens indexed by expert id), then
 * pmoe_moe_layer_fwd. ids_out, w_out, depth_out: device [T*k], written (may
 * be NULL to keep them in the workspace only).
 */
PMOE_API pmoe_status pmoe_moe_decode_step(const pmoe_layer *L, const float *logits, const float *sens,
                                 const uint16_t *x, int T, int k, float avg_bits, float *y,
                                 int32_t *ids_out, float *w_out, uint8_t *depth_out, void *ws,
                                 size_t ws_bytes, pmoe_stream stream);

/*
 * pmoe_moe_decode_step_host: pmoe_moe_decode_step for tokens whose inputs and
 * output live in host memory, as a serving loop holds them: copies logits
 * (host float [T*E]) and x (host bf16 [T*H]) into the workspace, runs the
 * step there and copies y (host float [T*H]) back, all queued on `stream` in
 * this one call (the routing and depths stay in the workspace). The call
 * returns once the work is queued: y is written when the stream reaches it.
 * Page-locked host buffers mapped into the device's address space (as
 * cudaHostAlloc/cudaMallocHost memory is under unified addressing) are read
 * and written by the kernels in place, with no copies; other page-locked
 * buffers are copied asynchronously; pageable ones are accepted and make the
 * copies synchronise with the host. The result is the same either way.
 *   sens: device float [E]. ws: device scratch of >=
 *   pmoe_decode_host_workspace_bytes() bytes, 256-byte aligned (smaller:
 *   PMOE_ERR_WORKSPACE). Shapes and errors as pmoe_moe_decode_step.
 */
PMOE_API pmoe_status pmoe_moe_decode_step_host(const pmoe_layer *L, const float *logits, const float *sens,
                                      const uint16_t *x, int T, int k, float avg_bits, float *y, void *ws,
                                      size_t ws_bytes, pmoe_stream stream);

/* Workspace of pmoe_moe_decode_step_host: the layer workspace plus room for T tokens' logits, x and y. */
PMOE_API size_t pmoe_decode_host_workspace_bytes(int T, int k, int E, int H, int I);

/*
 * pmoe_profile_events: when both events are non-NULL, every later
 * pmoe_moe_layer_fwd / pmoe_moe_decode_step call on this host thread records
 * `start` on its stream just before the expert kernels (gate/up + SwiGLU and
 * down) and `stop` just after them, so cudaEventElapsedTime gives their
 * device time without routing, grouping and combine. NULL, NULL turns it
 * off. The events are the caller's (cudaEventCreate); nothing is kept beyond
 * the two handles.
 */
PMOE_API pmoe_status pmoe_profile_events(pmoe_event start, pmoe_event stop);

/*
 * Materialise-then-multiply ablation [T#37, A: Results]: decodes the depth-b
 * prefixes of every selected expert to bf16 matrices in the workspace (the
 * dequantised weights scale*C rounded to bf16), then runs plain GEMVs
 * (bf16 x bf16, float accumulation) for gate/up, SwiGLU, down and the
 * weighted combine. Same arguments and output as pmoe_moe_layer_fwd.
 */
PMOE_API size_t pmoe_materialise_workspace_bytes(int T, int k, int E, int H, int I);
PMOE_API pmoe_status pmoe_materialise_layer_fwd(const pmoe_layer *L, const uint16_t *x, const int32_t *ids,
                                       const float *w, const uint8_t *depth, int T, int k,
                                       float *y, void *ws, size_t ws_bytes, pmoe_stream stream);

/* ------------------------------------------------------------------ */
/* Prefix cache [T#11, T#13, T#35, A: Abstract]                        */
/* ------------------------------------------------------------------ */

/*
 * An HBM cache of expert prefixes for `layers` MoE layers of `experts`
 * experts each, in a pool of plane slots (one slot = plane p of one expert,
 * all three matrices, the pmoe_layer slot layout). Every (layer, expert) has
 * one shared state whatever precision is asked of it [T#13]: its resident
 * depth r (planes 0..r-1 in slots) and a last-use time per plane. An access
 * (layer, expert, need b), time = its index since creation:
 *   r >= b: hit, nothing copied; planes 0..b-1 take the current time;
 *   r <  b: planes 0..r-1 take the current time; only the missing planes
 *           r..b-1 are copied from host memory into free slots [T#35] and
 *           take the current time; the depth becomes b.
 * When no slot is free, the resident plane with the oldest time is evicted,
 * which is always the deepest plane of its entry since a use refreshes a
 * prefix (ties to the lowest layer*experts + expert); that entry's depth
 * drops by one. Entries accessed in the current batch are never evicted.
 *
 * Memory (caller-owned, kept by the cache until destroyed):
 *   pool: device uint32 [slots * slot_words]; slot s at pool + s*slot_words.
 *   page_table: device int32 [layers][experts][8]: slot of plane p of expert
 *     e of layer l, or -1. pmoe_layer.slot_of of layer l is
 *     page_table + l*experts*8 (and pmoe_layer.pool = pool).
 *   host planes of layer l (pmoe_cache_extend): pinned host uint32
 *     [experts][8][slot_words]: plane p of expert e at (e*8 + p)*slot_words.
 */
typedef struct pmoe_cache pmoe_cache;

typedef struct {
    int64_t requests;       /* accesses */
    int64_t hits;           /* accesses whose resident depth covered the need */
    int64_t planes_fetched; /* expert-planes copied host -> device */
    int64_t bytes_fetched;  /* their bytes */
    int64_t planes_evicted;
} pmoe_cache_stats;

/*
 * pmoe_cache_create: empty cache of `slots` slots of slot_words words
 * (slot_words % 4 == 0). pool and page_table both NULL make a host-only
 * cache: the same decisions and statistics, no data moved (planning and
 * simulation). Otherwise the page table is set to -1 (synchronously).
 * keep_log != 0 records every eviction (pmoe_cache_eviction_log).
 * Allocates host memory only: the state, and a small mapped pinned area for
 * page-table updates. layers*experts*8 and slots must fit in int32.
 */
PMOE_API pmoe_status pmoe_cache_create(int layers, int experts, int64_t slots, int64_t slot_words,
                                       uint32_t *pool, int32_t *page_table, int keep_log, pmoe_cache **out);

/*
 * pmoe_cache_extend: applies the accesses (layer, experts[i], need[i]),
 * i < n, in order, all in batch `batch` (the caller's id of the step whose
 * kernels use them; an entry accessed in the current batch is pinned).
 * Missing planes are copied with one cudaMemcpyAsync each on stream `side`
 * from host_planes[layer] (host pointer array, indexed by layer; pinned
 * memory), then the page-table entries of fetched and evicted planes are
 * written by a small kernel on `side`, then `done` (may be NULL) is recorded
 * on `side`. Kernels that read the pool must wait for `done`.
 * Evicted slots are overwritten: if the call evicts and `after` is not NULL,
 * `side` first waits for `after`, which the caller records on its compute
 * stream after the last kernel of the previous batch.
 *   experts: host int32 [n], need: host uint8 [n] in 1..8,
 *   resident_before: host uint8 [n], the depth each access found (may be
 *   NULL); stats: the cache's accumulated counters after the call (may be
 *   NULL). Host-only caches ignore host_planes, side, after and done.
 * Errors: PMOE_ERR_INVALID_ARG (nothing changed); PMOE_ERR_OUT_OF_SLOTS
 * when the pinned entries of the batch leave no room (the accesses before
 * the failing one are applied and their copies enqueued); PMOE_ERR_CUDA when
 * a copy, the page-table kernel or an event call cannot be enqueued. For a
 * copy that cannot be enqueued, the accesses before it are applied; its own
 * access is taken back (depth, plane times, batch and counters as before
 * it; slots it took are free again) and later accesses are not made; planes
 * evicted on its behalf stay evicted, since copies already enqueued may
 * overwrite their slots. In every case the device page table is brought in
 * line with the host state before the call returns.
 */
PMOE_API pmoe_status pmoe_cache_extend(pmoe_cache *c, int layer, const int32_t *experts, const uint8_t *need,
                                       int n, int64_t batch, const uint32_t *const *host_planes,
                                       pmoe_stream side, pmoe_event after, pmoe_event done,
                                       uint8_t *resident_before, pmoe_cache_stats *stats);

/*
 * pmoe_cache_inject_copy_failure (testing hook): the nth next host-to-device
 * plane copy of this cache (nth >= 1) reports failure instead of being
 * enqueued, as a failing cudaMemcpyAsync would (PMOE_ERR_CUDA, last CUDA error
 * cudaErrorInvalidValue); nth = 0 disarms. Host state only; touches no GPU.
 */
PMOE_API pmoe_status pmoe_cache_inject_copy_failure(pmoe_cache *c, int64_t nth);

/* Accumulated counters. */
PMOE_API pmoe_status pmoe_cache_get_stats(const pmoe_cache *c, pmoe_cache_stats *stats);
/* Resident depth of every expert of a layer: host uint8 [experts]. */
PMOE_API pmoe_status pmoe_cache_resident_depth(const pmoe_cache *c, int layer, uint8_t *depth);
/*
 * Evictions so far, oldest first, as (layer*experts + expert)*8 + plane:
 * up to cap written to log (host int64), the total count to *n.
 * PMOE_ERR_UNSUPPORTED if the cache was created without keep_log.
 */
PMOE_API pmoe_status pmoe_cache_eviction_log(const pmoe_cache *c, int64_t *log, int64_t cap, int64_t *n);
/* Frees the host state (waits for its pending page-table updates); the pool and page table stay the caller's. */
PMOE_API pmoe_status pmoe_cache_destroy(pmoe_cache *c);

/*
 * pmoe_cache_sim_independent [T#11]: hit rate of the independent-precision
 * design on an access trace, host only: every (layer, expert, bits) is its
 * own object of `bits` planes; an access hits only if that exact object is
 * resident; a miss loads all its planes and evicts whole least-recently-used
 * objects (not those of the current batch) until it fits in cap_planes.
 *   layer, expert: host int32 [n]; need: host uint8 [n]; batch: host int64
 *   [n]; hit: host uint8 [n] out (1 hit, 0 miss); *planes_fetched out.
 * PMOE_ERR_OUT_OF_SLOTS if an access cannot fit (outputs up to it written).
 */
PMOE_API pmoe_status pmoe_cache_sim_independent(int layers, int experts, int64_t cap_planes, int64_t n,
                                                const int32_t *layer, const int32_t *expert,
                                                const uint8_t *need, const int64_t *batch, uint8_t *hit,
                                                int64_t *planes_fetched);

/*
 * pmoe_cache_sim_independent_down [T#51]: the independent design with
 * downward reuse, host only: one copy per (layer, expert) at some depth r; an
 * access at depth b hits when r >= b (the deeper copy serves it); otherwise a
 * whole copy of b planes is loaded and replaces the old one (copies share no
 * bits). Whole copies are evicted least-recently-used first (not those of the
 * current batch) within cap_planes. Arguments and errors as
 * pmoe_cache_sim_independent.
 */
PMOE_API pmoe_status pmoe_cache_sim_independent_down(int layers, int experts, int64_t cap_planes, int64_t n,
                                                     const int32_t *layer, const int32_t *expert,
                                                     const uint8_t *need, const int64_t *batch, uint8_t *hit,
                                                     int64_t *planes_fetched);

/*
 * pmoe_route_host: pmoe_route on host pointers (synchronous), for callers
 * that plan cache top-ups before launching the layer: ids (ties to the lower
 * id, larger logits first) and softmax weights in double rounded to float.
 */
PMOE_API pmoe_status pmoe_route_host(const float *logits, int T, int E, int k, int32_t *ids, float *w);

/*
 * pmoe_residual_norm: the residual stream between stacked layers, per token
 * t: r_t += y_t (skipped when y is NULL), then x_t = bf16(r_t * (1/rms(r_t)))
 * with rms = sqrt(mean of r_t^2) (x_t = 0 when rms is 0). Deterministic
 * (fixed-order float sums). r: device float [T*H] (updated), y: device float
 * [T*H] or NULL, x: device bf16 [T*H] out. H % 4 == 0.
 */
PMOE_API pmoe_status pmoe_residual_norm(float *r, const float *y, int T, int H, uint16_t *x, pmoe_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* PMOE_H */
