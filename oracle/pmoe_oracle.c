/*
 * ORACLE — test infrastructure only.
 *
 * A plain, slow, single-threaded CPU implementation of what the
 * bitplane-prefix MoE expert path computes, in double precision. Only the
 * tests, the smoke check and the benchmark's CPU-baseline leg may load or
 * call it. It shares no code, header, table or helper with the CUDA
 * library; inputs come from the seeded generators in synth/.
 *
 * Sources (web pages on PagedMoE):
 *   [T#n]  PagedMoE podcast transcript, subtitle cue n
 *          ("PagedMoE: Cross-Precision Expert Caching for SSD-Resident MoE
 *          Inference", AI Post Transformers episode .srt)
 *   [A]    "PagedMoE: Cross-Precision Expert Caching for Token-Level Dynamic
 *          Precision in SSD-Resident MoE Inference", arxivlens page:
 *          Abstract / Methodology
 *
 * Pins: every function here is checked in tests/test_oracle_*.py against
 * something other than itself (closed forms, numerical integration,
 * brute force, hand traces, invariants). See the header of each function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Normal distribution helpers                                         */
/* ------------------------------------------------------------------ */

static double or_cdf(double z) { return 0.5 * erfc(-z / sqrt(2.0)); }

static double or_pdf(double z)
{
    if (isinf(z))
        return 0.0;
    return exp(-0.5 * z * z) / sqrt(2.0 * M_PI);
}

/* Inverse normal CDF. For p < 1/2: bisection on erfc over z < 0, where
 * Phi(z) = erfc(-z/sqrt 2)/2 has full relative accuracy; the result is the
 * smallest double z (to the resolution of bisection) with Phi(z) >= p.
 * p = 1/2 gives 0; p > 1/2 uses the symmetry Phi^-1(p) = -Phi^-1(1 - p)
 * (1 - p is exact for the dyadic p used here). p in (0, 1). */
double or_norm_ppf(double p)
{
    if (p == 0.5)
        return 0.0;
    if (p > 0.5)
        return -or_norm_ppf(1.0 - p);
    double lo = -40.0, hi = 0.0;
    for (int it = 0; it < 4000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi)
            break;
        if (or_cdf(mid) < p)
            lo = mid;
        else
            hi = mid;
    }
    return hi;
}

/* ------------------------------------------------------------------ */
/* Tree codebook [T#19, T#21, A: Abstract]                             */
/* ------------------------------------------------------------------ */
/*
 * 256 sorted 8-bit codewords sit at the leaves of a binary tree; each parent
 * is the frequency-weighted mean of its two children, so truncating an index
 * to b bits lands on the depth-b ancestor [T#19, T#21]. For N(0,1) values cut
 * into 256 equiprobable bins, the depth-d node i is the conditional mean of
 * N(0,1) over the quantile interval [i/2^d, (i+1)/2^d):
 *     C[d][i] = 2^d * (phi(a) - phi(b)),  a = Phi^-1(i/2^d), b = Phi^-1((i+1)/2^d)
 * (equal child probabilities make the parent the plain mean of its children).
 * Storage: depth d at offset 2^d - 2, d = 1..8, 510 entries.
 * Pins: C[1][1] = sqrt(2/pi); every entry against numerical integration of
 * z*phi(z) over its bin; parent = mean of children; antisymmetry.
 */
void or_tree_codebook(double *cb /* [510] */)
{
    for (int d = 1; d <= 8; ++d) {
        int n = 1 << d;
        for (int i = 0; i < n; ++i) {
            double a = (i == 0) ? -INFINITY : or_norm_ppf((double)i / n);
            double b = (i == n - 1) ? INFINITY : or_norm_ppf((double)(i + 1) / n);
            cb[(n - 2) + i] = (double)n * (or_pdf(a) - or_pdf(b));
        }
    }
}

void or_tree_codebook_f32(float *cb /* [510] */)
{
    double tmp[510];
    or_tree_codebook(tmp);
    for (int i = 0; i < 510; ++i)
        cb[i] = (float)tmp[i];
}

/*
 * Tree codebook from a sorted 256-entry leaf set with leaf frequencies
 * [T#19, T#21]: the leaves sit at depth 8 in sorted order; every parent is
 * the frequency-weighted mean of its two children and carries the sum of
 * their frequencies, level by level up to depth 1. A pair whose frequencies
 * are both zero gets the plain mean of its children (and frequency 0).
 * Storage as or_tree_codebook. All in double.
 * Pins: equal frequencies on the Gaussian leaves give the closed-form tree
 * (equal-mass children); every node equals the weighted average of the leaves
 * below it (numpy, computed directly from the leaves, not level by level).
 */
void or_tree_from_leaves(const double *leaves /* [256] */, const double *freq /* [256] */,
                         double *cb /* [510] */)
{
    double f[256], v[256];
    for (int i = 0; i < 256; ++i) {
        v[i] = leaves[i];
        f[i] = freq[i];
        cb[254 + i] = leaves[i];
    }
    for (int d = 7; d >= 1; --d) {
        int n = 1 << d;
        for (int i = 0; i < n; ++i) {
            double fl = f[2 * i], fr = f[2 * i + 1];
            double m = (fl + fr > 0.0) ? (fl * v[2 * i] + fr * v[2 * i + 1]) / (fl + fr)
                                       : 0.5 * (v[2 * i] + v[2 * i + 1]);
            v[i] = m;
            f[i] = fl + fr;
            cb[(n - 2) + i] = m;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Quantiser: per-group std scale, 256 equiprobable N(0,1) bins         */
/* ------------------------------------------------------------------ */
/*
 * Group g of row n covers columns [g*G, (g+1)*G). scale = population standard
 * deviation of the group's weights about their mean, in double, rounded to
 * float; a zero scale becomes 1. code = #{ i in 1..255 : w/scale >= t_i },
 * t_i = Phi^-1(i/256): the index of the equiprobable bin, half-open on the
 * right, so a value exactly on a threshold goes to the upper bin. (The count
 * is taken by bisection over the sorted thresholds.)
 * The reconstruction at depth b is scale * C[b][code >> (8-b)].
 * Pins: hand examples on thresholds; chi-square uniformity of codes on
 * N(0,1) data; scales against numpy's population std.
 */
void or_thresholds(double *t /* [256]; t[0] unused */)
{
    t[0] = -INFINITY;
    for (int i = 1; i < 256; ++i)
        t[i] = or_norm_ppf((double)i / 256.0);
}

void or_quantize(const float *w, int N, int K, int G, float *scales /* [N*(K/G)] */,
                 uint8_t *codes /* [N*K] */)
{
    double t[256];
    or_thresholds(t);
    int ng = K / G;
    for (int n = 0; n < N; ++n) {
        for (int g = 0; g < ng; ++g) {
            const float *src = w + (size_t)n * K + (size_t)g * G;
            double mean = 0.0;
            for (int k = 0; k < G; ++k)
                mean += (double)src[k];
            mean /= (double)G;
            double var = 0.0;
            for (int k = 0; k < G; ++k) {
                double d = (double)src[k] - mean;
                var += d * d;
            }
            var /= (double)G;
            float s = (float)sqrt(var);
            if (s == 0.0f)
                s = 1.0f;
            scales[(size_t)n * ng + g] = s;
            for (int k = 0; k < G; ++k) {
                double z = (double)src[k] / (double)s;
                /* #{i in 1..255 : t_i <= z}; the thresholds are sorted, so the
                 * count is found by bisection over them */
                int lo = 0, hi = 256; /* t[lo] <= z < t[hi] (t[256] = +inf) */
                while (hi - lo > 1) {
                    int mid = (lo + hi) / 2;
                    if (t[mid] <= z)
                        lo = mid;
                    else
                        hi = mid;
                }
                codes[(size_t)n * K + (size_t)g * G + k] = (uint8_t)lo;
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* Bitplane layout [T#25, A: Abstract]                                  */
/* ------------------------------------------------------------------ */
/*
 * Plane p (0-based) holds bit (7-p) of every weight's 8-bit index, MSB
 * first, so a depth-b request reads exactly planes 0..b-1 [T#25]. Where each
 * weight's bit sits inside a plane is this format's choice (the pages fix
 * only that plane j holds the j-th index bit of every weight):
 *
 *   tiles of 16 rows x 128 columns, row-strip major: tile = (n/16)*(K/128) + k/128;
 *   inside a tile: rr = n%16, kk = k%128, g = rr%8, u = rr/8,
 *     s = kk/32, half = (kk%32)/16, t = (kk%16)/4, i = kk%4,
 *     j = 4*half + i, L = 4*g + t, q = 2*s + u, h = q/4, r = q%4;
 *   word = tile*64 + 2*L + h   (64 words per tile per plane),
 *   bit  = (4*j + p + r) mod 32.
 *
 * Words of plane p start at planes + p*(N*K/32).
 * Pins: unpack(pack(x)) = x; pack at depth b equals the first b planes of
 * pack at depth b' (prefix property); the per-lane reading of the layout
 * reproduces the documented m16n8k32 operand fragments (host test).
 */
static void or_bit_position(int n, int k, int K, int p, int64_t *word, int *bit)
{
    int rr = n % 16, kk = k % 128;
    int g = rr % 8, u = rr / 8;
    int s = kk / 32, half = (kk % 32) / 16, t = (kk % 16) / 4, i = kk % 4;
    int j = 4 * half + i;
    int L = 4 * g + t;
    int q = 2 * s + u, h = q / 4, r = q % 4;
    int64_t tile = (int64_t)(n / 16) * (K / 128) + (k / 128);
    *word = tile * 64 + 2 * L + h;
    *bit = (4 * j + p + r) % 32;
}

int or_pack(const uint8_t *codes, int N, int K, int depth, uint32_t *planes)
{
    if (N <= 0 || K <= 0 || N % 16 || K % 128 || depth < 1 || depth > 8)
        return 1;
    int64_t pw = (int64_t)N * K / 32;
    memset(planes, 0, sizeof(uint32_t) * (size_t)(pw * depth));
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            int c = codes[(size_t)n * K + k];
            for (int p = 0; p < depth; ++p) {
                int64_t w;
                int bit;
                or_bit_position(n, k, K, p, &w, &bit);
                if ((c >> (7 - p)) & 1)
                    planes[p * pw + w] |= (1u << bit);
            }
        }
    return 0;
}

/* b-bit prefix index of every weight, read from planes 0..b-1 */
int or_unpack(const uint32_t *planes, int N, int K, int b, uint8_t *idx)
{
    if (N <= 0 || K <= 0 || N % 16 || K % 128 || b < 1 || b > 8)
        return 1;
    int64_t pw = (int64_t)N * K / 32;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            int v = 0;
            for (int p = 0; p < b; ++p) {
                int64_t w;
                int bit;
                or_bit_position(n, k, K, p, &w, &bit);
                v = (v << 1) | (int)((planes[p * pw + w] >> bit) & 1u);
            }
            idx[(size_t)n * K + k] = (uint8_t)v;
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Prefix GEMV: dequantise at depth b, then matvec [T#21, T#37]          */
/* ------------------------------------------------------------------ */
/*
 *   y[n] = sum_k scale[n][k/G] * C[b][code[n][k] >> (8-b)] * x[k]
 * with the fp32 codebook entries and scales widened to double. When
 * bf16_weights is set, each dequantised weight scale*C (computed in float)
 * is rounded to bf16 first: the materialise-to-bf16 ablation [T#37].
 * Pins: numpy dequantise-then-matmul on small inputs; unit vectors x = e_k.
 */
static float or_round_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    u &= 0xFFFF0000u;
    float r;
    memcpy(&r, &u, 4);
    return r;
}

void or_gemv(const uint8_t *codes, const float *scales, const float *cb, int N, int K, int G, int b,
             const double *x, double *y, int bf16_weights)
{
    int ng = K / G;
    int off = (1 << b) - 2;
    for (int n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int k = 0; k < K; ++k) {
            int idx = codes[(size_t)n * K + k] >> (8 - b);
            float s = scales[(size_t)n * ng + k / G];
            double wv;
            if (bf16_weights)
                wv = (double)or_round_bf16(s * cb[off + idx]);
            else
                wv = (double)s * (double)cb[off + idx];
            acc += wv * x[k];
        }
        y[n] = acc;
    }
}

/* ------------------------------------------------------------------ */
/* Routing [T#4]: top-k of the router logits, softmax over the k          */
/* ------------------------------------------------------------------ */
/*
 * The router picks k experts per token with weights that sum to one [T#4].
 * Reading: the k largest logits (ties to the lower expert id), in descending
 * order; weights = softmax over those k logits, evaluated in double
 * (exp(l_i - l_max) / sum) and rounded to float.
 * Pins: hand examples with ties; sum to one; equal logits give equal weights.
 */
void or_route(const float *logits, int T, int E, int k, int32_t *ids, float *w)
{
    char *taken = (char *)malloc((size_t)E);
    double *ex = (double *)malloc(sizeof(double) * (size_t)k);
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int s = 0; s < k; ++s) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e])
                    continue;
                if (best < 0 || l[e] > l[best])
                    best = e;
            }
            taken[best] = 1;
            ids[(size_t)t * k + s] = best;
        }
        double lmax = (double)l[ids[(size_t)t * k]];
        double sum = 0.0;
        for (int s = 0; s < k; ++s) {
            ex[s] = exp((double)l[ids[(size_t)t * k + s]] - lmax);
            sum += ex[s];
        }
        for (int s = 0; s < k; ++s)
            w[(size_t)t * k + s] = (float)(ex[s] / sum);
    }
    free(taken);
    free(ex);
}

/* ------------------------------------------------------------------ */
/* Prefix selection [T#29, T#31, A: Abstract]                           */
/* ------------------------------------------------------------------ */
/*
 * Per token, minimise the surrogate sum_i w_i^2 * E_e(b_i) with the error
 * profile E_e(b) = s_e^2 * 4^-b under the budget sum_i b_i = B: start every
 * expert at 1 bit and repeatedly grant one more bit to the expert with the
 * largest gain, until the budget is spent [T#29]. The gain of b -> b+1 is
 * (3/4) w^2 s^2 4^-b, ordered as v_i * 2^-b_i with v_i = w_i * s_{e_i} (one
 * float multiply); comparisons are exact in float (ldexpf). Ties go to the
 * lower slot; an expert at 8 bits takes no more. Budget:
 *     B = floor(avg_bits * k + 1e-4) (in double), clamped to [k, 8k].
 * Returns 0, or 1 on bad arguments.
 * Pins: brute force over all depth vectors for k <= 4; the equivalent
 * closed rule b_i = clamp(ceil(c + log2(w_i s_i / geomean)), 1, 8) with c
 * chosen so that sum b_i = B.
 */
int or_budget(int k, float avg_bits)
{
    int B = (int)floor((double)avg_bits * (double)k + 1e-4);
    if (B < k)
        B = k;
    if (B > 8 * k)
        B = 8 * k;
    return B;
}

int or_select(const float *w, const int32_t *ids, const float *sens, int T, int k, float avg_bits,
              uint8_t *depth)
{
    if (T < 0 || k <= 0 || k > 64)
        return 1;
    int B = or_budget(k, avg_bits);
    float v[64];
    int b[64];
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < k; ++i) {
            v[i] = w[(size_t)t * k + i] * sens[ids[(size_t)t * k + i]];
            b[i] = 1;
        }
        for (int step = 0; step < B - k; ++step) {
            int best = -1;
            float bestp = 0.0f;
            for (int i = 0; i < k; ++i) {
                if (b[i] >= 8)
                    continue;
                float pr = ldexpf(v[i], -b[i]);
                if (best < 0 || pr > bestp) {
                    best = i;
                    bestp = pr;
                }
            }
            if (best < 0)
                break;
            b[best] += 1;
        }
        for (int i = 0; i < k; ++i)
            depth[(size_t)t * k + i] = (uint8_t)b[i];
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* MoE layer [T#4, T#37, A: Methodology]                                */
/* ------------------------------------------------------------------ */
/*
 * For token t and slot i with expert e = ids[t][i], depth b = depth[t][i]:
 *   g = Wg_b x,  u = Wu_b x   (I rows, K = H),  h = silu(g) * u,
 *   y_t += w[t][i] * (Wd_b h) (H rows, K = I),  silu(z) = z / (1 + exp(-z)),
 * where W*_b is the depth-b dequantisation of the expert's matrix. All in
 * double. codes_*[e], scales_*[e], cb_*[e] may be NULL for experts that no
 * token selects. x is [T*H] in double (the caller widens bf16), y [T*H].
 * Pins: numpy brute force (dequantise, matmul, silu) on small layers.
 */
int or_moe_layer(int T, int k, int H, int I, int G,
                 const uint8_t *const *codes_g, const uint8_t *const *codes_u,
                 const uint8_t *const *codes_d,
                 const float *const *scales_g, const float *const *scales_u,
                 const float *const *scales_d,
                 const float *const *cb_g, const float *const *cb_u, const float *const *cb_d,
                 const int32_t *ids, const float *w, const uint8_t *depth,
                 const double *x, double *y, int bf16_weights)
{
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    double *o = (double *)malloc(sizeof(double) * (size_t)H);
    if (!g || !u || !h || !o)
        return 2;
    for (int t = 0; t < T; ++t) {
        double *yt = y + (size_t)t * H;
        for (int n = 0; n < H; ++n)
            yt[n] = 0.0;
        for (int i = 0; i < k; ++i) {
            int e = ids[(size_t)t * k + i];
            int b = depth[(size_t)t * k + i];
            if (!codes_g[e] || !codes_u[e] || !codes_d[e])
                return 1;
            or_gemv(codes_g[e], scales_g[e], cb_g[e], I, H, G, b, x + (size_t)t * H, g, bf16_weights);
            or_gemv(codes_u[e], scales_u[e], cb_u[e], I, H, G, b, x + (size_t)t * H, u, bf16_weights);
            for (int j = 0; j < I; ++j)
                h[j] = g[j] / (1.0 + exp(-g[j])) * u[j];
            or_gemv(codes_d[e], scales_d[e], cb_d[e], H, I, G, b, h, o, bf16_weights);
            double wt = (double)w[(size_t)t * k + i];
            for (int n = 0; n < H; ++n)
                yt[n] += wt * o[n];
        }
    }
    free(g);
    free(u);
    free(h);
    free(o);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Prefix cache simulator [T#11, T#13, T#35, A: Abstract]                */
/* ------------------------------------------------------------------ */
/*
 * One shared state per (layer, expert): its resident depth r (planes 0..r-1,
 * a plane being usable only when every earlier plane is resident) and a
 * timestamp per plane. An access at depth b at time tau [T#13, T#35]:
 *   r >= b : no I/O; planes 0..b-1 refreshed to tau (deeper ones keep theirs,
 *            so the deepest planes age out first);
 *   r <  b : planes 0..r-1 refreshed; planes r..b-1 fetched (b-r planes) and
 *            stamped tau, after evicting, while the capacity (in planes) would
 *            be exceeded, the globally oldest resident plane, which is always
 *            the deepest plane of some entry (ties to the lowest
 *            layer*E+expert). Entries accessed in the current batch (one
 *            token-layer step) are not evicted.
 * tau is the access index. Outputs, per access: the resident depth before it;
 * and the log of evicted planes as (layer*E+expert)*8 + plane.
 * Returns 0; 1 on bad arguments; 3 if an access cannot fit.
 * Pins: hand traces (3 resident / 5 requested reads planes 4-5; 5 resident /
 * 3 requested reads nothing; deepest-first eviction order).
 */
int or_cache_sim_prefix(int L, int E, int64_t cap_planes, int64_t n_acc,
                        const int32_t *acc_layer, const int32_t *acc_expert,
                        const uint8_t *acc_depth, const int32_t *acc_batch,
                        uint8_t *resident_before, int64_t *evict_log, int64_t evict_cap,
                        int64_t *n_evicted, int64_t *planes_fetched)
{
    int64_t NE = (int64_t)L * E;
    uint8_t *dep = (uint8_t *)calloc((size_t)NE, 1);
    int64_t *ts = (int64_t *)calloc((size_t)NE * 8, sizeof(int64_t));
    int32_t *last_batch = (int32_t *)malloc(sizeof(int32_t) * (size_t)NE);
    if (!dep || !ts || !last_batch)
        return 2;
    for (int64_t x = 0; x < NE; ++x)
        last_batch[x] = -1;
    int64_t used = 0, nev = 0, fetched = 0;
    int rc = 0;
    for (int64_t a = 0; a < n_acc; ++a) {
        int l = acc_layer[a], e = acc_expert[a], b = acc_depth[a];
        if (l < 0 || l >= L || e < 0 || e >= E || b < 1 || b > 8) {
            rc = 1;
            break;
        }
        int64_t x = (int64_t)l * E + e;
        int r = dep[x];
        resident_before[a] = (uint8_t)r;
        last_batch[x] = acc_batch[a];
        if (r >= b) {
            for (int p = 0; p < b; ++p)
                ts[x * 8 + p] = a;
            continue;
        }
        for (int p = 0; p < r; ++p)
            ts[x * 8 + p] = a;
        int need = b - r;
        while (used + need > cap_planes) {
            int64_t victim = -1, vts = 0;
            for (int64_t y = 0; y < NE; ++y) {
                if (dep[y] == 0 || last_batch[y] == acc_batch[a])
                    continue;
                int64_t t0 = ts[y * 8 + dep[y] - 1];
                if (victim < 0 || t0 < vts) {
                    victim = y;
                    vts = t0;
                }
            }
            if (victim < 0) {
                rc = 3;
                break;
            }
            dep[victim] -= 1;
            used -= 1;
            if (nev < evict_cap)
                evict_log[nev] = victim * 8 + dep[victim];
            nev += 1;
        }
        if (rc)
            break;
        for (int p = r; p < b; ++p)
            ts[x * 8 + p] = a;
        dep[x] = (uint8_t)b;
        used += need;
        fetched += need;
    }
    *n_evicted = nev;
    *planes_fetched = fetched;
    free(dep);
    free(ts);
    free(last_batch);
    return rc;
}

/*
 * Independent-precision baseline [T#11, A: Abstract]: every (layer, expert,
 * bits) is its own cache object of b planes; an access hits only when that
 * exact object is resident; a miss fetches all b planes and evicts whole
 * least-recently-used objects (not those accessed in the current batch)
 * until it fits in the same plane capacity.
 * Outputs per access: 1 on hit, 0 on miss.
 */
int or_cache_sim_independent(int L, int E, int64_t cap_planes, int64_t n_acc,
                             const int32_t *acc_layer, const int32_t *acc_expert,
                             const uint8_t *acc_depth, const int32_t *acc_batch,
                             uint8_t *hit, int64_t *planes_fetched)
{
    int64_t NO = (int64_t)L * E * 8;
    int64_t *ts = (int64_t *)malloc(sizeof(int64_t) * (size_t)NO);
    int32_t *last_batch = (int32_t *)malloc(sizeof(int32_t) * (size_t)NO);
    char *present = (char *)calloc((size_t)NO, 1);
    int64_t *list = (int64_t *)malloc(sizeof(int64_t) * (size_t)NO); /* present objects */
    if (!ts || !last_batch || !present || !list)
        return 2;
    int64_t nlist = 0, used = 0, fetched = 0;
    int rc = 0;
    for (int64_t a = 0; a < n_acc; ++a) {
        int l = acc_layer[a], e = acc_expert[a], b = acc_depth[a];
        if (l < 0 || l >= L || e < 0 || e >= E || b < 1 || b > 8) {
            rc = 1;
            break;
        }
        int64_t o = ((int64_t)l * E + e) * 8 + (b - 1);
        last_batch[o] = acc_batch[a];
        if (present[o]) {
            hit[a] = 1;
            ts[o] = a;
            continue;
        }
        hit[a] = 0;
        while (used + b > cap_planes) {
            int64_t vi = -1;
            for (int64_t q = 0; q < nlist; ++q) {
                int64_t y = list[q];
                if (last_batch[y] == acc_batch[a])
                    continue;
                if (vi < 0 || ts[y] < ts[list[vi]] || (ts[y] == ts[list[vi]] && y < list[vi]))
                    vi = q;
            }
            if (vi < 0) {
                rc = 3;
                break;
            }
            int64_t y = list[vi];
            present[y] = 0;
            used -= (y % 8) + 1;
            list[vi] = list[nlist - 1];
            nlist -= 1;
        }
        if (rc)
            break;
        present[o] = 1;
        ts[o] = a;
        list[nlist++] = o;
        used += b;
        fetched += b;
    }
    *planes_fetched = fetched;
    free(ts);
    free(last_batch);
    free(present);
    free(list);
    return rc;
}

/*
 * Independent objects with downward reuse [T#51]: one resident copy per
 * (layer, expert) at some depth r (r planes, loaded as one object). An access
 * at depth b hits when r >= b (the deeper copy serves the shallower request);
 * otherwise the copy is promoted: a whole new object of b planes is fetched
 * (objects share no bits) and replaces the old one. Whole objects are evicted
 * least-recently-used first (not those accessed in the current batch) until
 * the new one fits in the same plane capacity.
 * Outputs per access: 1 on hit, 0 on miss; *planes_fetched.
 */
int or_cache_sim_independent_down(int L, int E, int64_t cap_planes, int64_t n_acc,
                                  const int32_t *acc_layer, const int32_t *acc_expert,
                                  const uint8_t *acc_depth, const int32_t *acc_batch,
                                  uint8_t *hit, int64_t *planes_fetched)
{
    int64_t NE = (int64_t)L * E;
    uint8_t *dep = (uint8_t *)calloc((size_t)NE, 1);
    int64_t *ts = (int64_t *)malloc(sizeof(int64_t) * (size_t)NE);
    int32_t *last_batch = (int32_t *)malloc(sizeof(int32_t) * (size_t)NE);
    if (!dep || !ts || !last_batch)
        return 2;
    int64_t used = 0, fetched = 0;
    int rc = 0;
    for (int64_t a = 0; a < n_acc; ++a) {
        int l = acc_layer[a], e = acc_expert[a], b = acc_depth[a];
        if (l < 0 || l >= L || e < 0 || e >= E || b < 1 || b > 8) {
            rc = 1;
            break;
        }
        int64_t x = (int64_t)l * E + e;
        last_batch[x] = acc_batch[a];
        ts[x] = a;
        if (dep[x] >= b) {
            hit[a] = 1;
            continue;
        }
        hit[a] = 0;
        used -= dep[x]; /* the old copy is replaced */
        dep[x] = 0;
        while (used + b > cap_planes) {
            int64_t victim = -1;
            for (int64_t y = 0; y < NE; ++y) {
                if (dep[y] == 0 || last_batch[y] == acc_batch[a])
                    continue;
                if (victim < 0 || ts[y] < ts[victim])
                    victim = y;
            }
            if (victim < 0) {
                rc = 3;
                break;
            }
            used -= dep[victim];
            dep[victim] = 0;
        }
        if (rc)
            break;
        dep[x] = (uint8_t)b;
        used += b;
        fetched += b;
    }
    *planes_fetched = fetched;
    free(dep);
    free(ts);
    free(last_batch);
    return rc;
}

/*
 * Cache-aware prefix selection [T#61]: the cache-oblivious allocator budgets
 * requested bits; this one budgets planes that must be fetched. Per token,
 * with r_i the resident depth of slot i's expert (0..8):
 *   b_i starts at max(1, r_i): resident planes cost no I/O, and every expert
 *   needs at least its first plane (a fetch when r_i = 0);
 *   then, while fewer than `fetch` planes have been fetched, the slot with the
 *   largest w_i*s_e*2^-b_i among b_i < 8 (ties to the lower slot, exact
 *   ldexpf) gets one more plane, each costing one fetch.
 * This minimises sum w_i^2 s_e^2 4^-b_i under the fetch budget, because each
 * further plane of a slot helps less than the one before.
 */
int or_select_cache_aware(const float *w, const int32_t *ids, const float *sens, const uint8_t *resident,
                          int T, int k, int fetch, uint8_t *depth)
{
    if (T < 0 || k <= 0 || k > 64 || fetch < 0)
        return 1;
    float v[64];
    int b[64];
    for (int t = 0; t < T; ++t) {
        int used = 0;
        for (int i = 0; i < k; ++i) {
            int r = resident[(size_t)t * k + i];
            if (r > 8)
                r = 8;
            v[i] = w[(size_t)t * k + i] * sens[ids[(size_t)t * k + i]];
            b[i] = r > 0 ? r : 1;
            if (r == 0)
                used += 1;
        }
        while (used < fetch) {
            int best = -1;
            float bestp = 0.0f;
            for (int i = 0; i < k; ++i) {
                if (b[i] >= 8)
                    continue;
                float pr = ldexpf(v[i], -b[i]);
                if (best < 0 || pr > bestp) {
                    best = i;
                    bestp = pr;
                }
            }
            if (best < 0)
                break;
            b[best] += 1;
            used += 1;
        }
        for (int i = 0; i < k; ++i)
            depth[(size_t)t * k + i] = (uint8_t)b[i];
    }
    return 0;
}

/*
 * Error profiles [T#29, T#31]: E_e(b) for b = 1..8, the relative output error
 * of an expert at depth b. Greedy allocation is valid when each further bit
 * helps less than the one before; profiles that break this are repaired by
 * isotonic regression. Reading: the gains g_b = E(b) - E(b+1), b = 1..7, are
 * replaced by their least-squares non-increasing fit (pool adjacent
 * violators, equal weights), clamped at 0, and E is rebuilt from E(8) upward
 * (E(8) kept): E(b) = E(b+1) + g_b.
 */
void or_isotonic_nonincreasing(double *g, int n)
{
    double val[16];
    int cnt[16];
    int m = 0;
    for (int i = 0; i < n; ++i) {
        val[m] = g[i];
        cnt[m] = 1;
        ++m;
        while (m > 1 && val[m - 2] < val[m - 1]) { /* violation of non-increasing order: pool */
            double v = (val[m - 2] * cnt[m - 2] + val[m - 1] * cnt[m - 1]) / (cnt[m - 2] + cnt[m - 1]);
            cnt[m - 2] += cnt[m - 1];
            val[m - 2] = v;
            --m;
        }
    }
    int i = 0;
    for (int j = 0; j < m; ++j)
        for (int c = 0; c < cnt[j]; ++c)
            g[i++] = val[j];
}

void or_profile_repair(const double *raw, int n, double *table)
{
    for (int e = 0; e < n; ++e) {
        const double *E = raw + (size_t)e * 8;
        double g[7];
        for (int b = 0; b < 7; ++b)
            g[b] = E[b] - E[b + 1];
        or_isotonic_nonincreasing(g, 7);
        double *out = table + (size_t)e * 8;
        out[7] = E[7];
        for (int b = 6; b >= 0; --b)
            out[b] = out[b + 1] + (g[b] > 0.0 ? g[b] : 0.0);
    }
}

/*
 * Prefix selection from a profile table [T#29]: as or_select, with the gain of
 * giving slot i its (b+1)-th bit = w_i^2 * (E_e(b) - E_e(b+1)) computed in
 * float ((w*w) * (E[b-1] - E[b]), table of floats [E][8], entry b-1 = E(b)).
 * Largest gain first, ties to the lower slot, 8-bit slots skipped.
 */
int or_select_table(const float *w, const int32_t *ids, const float *table, int T, int k, float avg_bits,
                    uint8_t *depth)
{
    if (T < 0 || k <= 0 || k > 64)
        return 1;
    int B = or_budget(k, avg_bits);
    int b[64];
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < k; ++i)
            b[i] = 1;
        for (int step = 0; step < B - k; ++step) {
            int best = -1;
            float bestp = 0.0f;
            for (int i = 0; i < k; ++i) {
                if (b[i] >= 8)
                    continue;
                float wi = w[(size_t)t * k + i];
                const float *E = table + (size_t)ids[(size_t)t * k + i] * 8;
                float gain = E[b[i] - 1] - E[b[i]];
                float pr = (wi * wi) * gain;
                if (best < 0 || pr > bestp) {
                    best = i;
                    bestp = pr;
                }
            }
            if (best < 0)
                break;
            b[best] += 1;
        }
        for (int i = 0; i < k; ++i)
            depth[(size_t)t * k + i] = (uint8_t)b[i];
    }
    return 0;
}
