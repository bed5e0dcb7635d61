/*
 * CPU oracle for the forward pass of one Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant generator with the GPU path and is deliberately
 * plain: fp64 accumulation, straight loops in the order the definitions are
 * written, OpenMP only over independent tokens or rows.
 *
 * Sources (web pages on MoE routing; each function names the passage it
 * follows):
 *   [P3] "Advanced GPU Optimization: How to tech an LLM with CUDA and ROCm? -
 *        Part 5 (Final Part)", section 1.1 "The Router Kernel (Top-k Gating)"
 *        and "The Math".
 *   [P4] "MoE: what it costs to train and serve", sections "Expert parallelism
 *        and two all-to-alls", "Worked example: how many bytes does one token
 *        send?", "Numerical precision".
 *   [P5] "moe communication costs", paragraphs "Router design",
 *        "Load balancing - the critical auxiliary loss", "Capacity factor and
 *        token dropping".
 *   OCP 8-bit Floating Point Specification (OFP8) rev 1.0, E4M3 format.
 *
 * Readings taken where the pages are silent are marked READING.
 *
 * Parity status: every function below is pinned by tests under tests/ that do
 * not call back into this file's formulas (brute-force sorts, closed forms,
 * library routines, invariants, page-printed values).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

enum { ORC_F32 = 0, ORC_BF16 = 1 };
enum { ORC_GATE_R = 0, ORC_GATE_F = 1 };
enum { ORC_RELU = 0, ORC_SWIGLU = 1 };

/* Exact decode of one stored element to double. */
static inline double ld(const void *p, int dt, int64_t i)
{
    if (dt == ORC_F32)
        return (double)((const float *)p)[i];
    uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* ------------------------------------------------------------------ */
/* Router logits.  [P5 Router design]: the router maps x in R^d to     */
/* W_g x (+ noise, which a forward pass leaves out); W_g is N x d.     */
/* The Switch-shaped workload adds a fixed per-expert bias b to skew   */
/* the routing.  logits[t - t0][e] = sum_j x[t][j] W_g[e][j] + b[e].   */
/* ------------------------------------------------------------------ */
void orc_router_logits(int64_t t0, int64_t t1, int d, int N,
                       const void *x, int xdt, const void *Wg, int wdt,
                       const float *bias, double *logits)
{
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = t0; t < t1; ++t) {
        for (int e = 0; e < N; ++e) {
            double s = 0.0;
            for (int j = 0; j < d; ++j)
                s += ld(x, xdt, t * (int64_t)d + j) * ld(Wg, wdt, (int64_t)e * d + j);
            if (bias)
                s += (double)bias[e];
            logits[(t - t0) * (int64_t)N + e] = s;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Top-k selection and gate weights.                                   */
/*                                                                     */
/* Order: experts sorted by logit, largest first; equal logits keep    */
/* the lower expert index first (the [P3] router updates its running   */
/* maxima only on a strictly larger score, so the earliest index wins; */
/* slot 0 holds the largest).  Implemented as a stable insertion sort  */
/* of the indices 0..N-1 by descending logit.                          */
/*                                                                     */
/* Mode R ([P3] section 1.1, sparse softmax): softmax over the k        */
/*   selected logits only, shifted by the largest for stability.       */
/* Mode F ([P5] Router design): G(x) = softmax over all N logits; the  */
/*   k largest entries are the mixture coefficients; with renormalize  */
/*   they are divided by their sum.                                    */
/* probs (optional, [nt][N]) always receives the full softmax over N   */
/* (the router probability used by the aux loss, [P5] Load balancing).*/
/*                                                                     */
/* Node-limited routing ([P4] "Limit how many machines a token         */
/* touches": each token may go to at most a few nodes, chosen by the   */
/* sum of the highest expert scores on each node).  READING: the N     */
/* experts sit on n_groups nodes of N / n_groups consecutive experts;  */
/* an expert's score is its router probability softmax(l)_e; a node's  */
/* score is the sum of its m = ceil(k / topk_groups) highest; nodes are */
/* ranked by score, largest first, the lower node index first on equal */
/* scores; the top-k is then taken, in the order above, among the      */
/* experts of the first topk_groups nodes only.  n_groups <= 1 or       */
/* topk_groups >= n_groups: no limit.                                  */
/* ------------------------------------------------------------------ */
void orc_topk_gate(int64_t nt, int N, int k, int gate_mode, int renormalize,
                   const double *logits, int32_t *idx, double *gate, double *probs,
                   int n_groups, int topk_groups)
{
    const int limited = n_groups > 1 && topk_groups < n_groups;
    const int gsize = limited ? N / n_groups : N;
    const int m = limited ? (k + topk_groups - 1) / topk_groups : 0;
    #pragma omp parallel
    {
        int *ord = (int *)malloc(sizeof(int) * (size_t)N);
        int *sel = (int *)malloc(sizeof(int) * (size_t)N);
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *gscore = (double *)malloc(sizeof(double) * (size_t)(n_groups > 0 ? n_groups : 1));
        int *gcnt = (int *)malloc(sizeof(int) * (size_t)(n_groups > 0 ? n_groups : 1));
        int *gord = (int *)malloc(sizeof(int) * (size_t)(n_groups > 0 ? n_groups : 1));
        char *allowed = (char *)malloc((size_t)(n_groups > 0 ? n_groups : 1));
        #pragma omp for schedule(static)
        for (int64_t t = 0; t < nt; ++t) {
            const double *l = logits + t * (int64_t)N;
            /* stable insertion sort, descending by logit */
            for (int e = 0; e < N; ++e) {
                int pos = e;
                while (pos > 0 && l[ord[pos - 1]] < l[e]) {
                    ord[pos] = ord[pos - 1];
                    --pos;
                }
                ord[pos] = e;
            }
            /* full softmax over N */
            double mx = l[ord[0]], den = 0.0;
            for (int e = 0; e < N; ++e) {
                p[e] = exp(l[e] - mx);
                den += p[e];
            }
            for (int e = 0; e < N; ++e)
                p[e] /= den;
            if (probs)
                memcpy(probs + t * (int64_t)N, p, sizeof(double) * (size_t)N);

            /* the experts the token may use, in the order above */
            int nsel = 0;
            if (!limited) {
                for (int e = 0; e < N; ++e)
                    sel[nsel++] = ord[e];
            } else {
                for (int g = 0; g < n_groups; ++g) {
                    gscore[g] = 0.0;
                    gcnt[g] = 0;
                }
                for (int r = 0; r < N; ++r) {       /* each node's m highest, largest first */
                    const int e = ord[r], g = e / gsize;
                    if (gcnt[g] < m) {
                        gscore[g] += p[e];
                        ++gcnt[g];
                    }
                }
                for (int g = 0; g < n_groups; ++g) { /* stable insertion sort of the nodes */
                    int pos = g;
                    while (pos > 0 && gscore[gord[pos - 1]] < gscore[g]) {
                        gord[pos] = gord[pos - 1];
                        --pos;
                    }
                    gord[pos] = g;
                }
                for (int g = 0; g < n_groups; ++g)
                    allowed[g] = 0;
                for (int j = 0; j < topk_groups; ++j)
                    allowed[gord[j]] = 1;
                for (int r = 0; r < N; ++r)
                    if (allowed[ord[r] / gsize])
                        sel[nsel++] = ord[r];
            }

            for (int j = 0; j < k; ++j)
                idx[t * k + j] = sel[j];
            if (gate_mode == ORC_GATE_R) {
                double top = l[sel[0]], s = 0.0;
                for (int j = 0; j < k; ++j)
                    s += exp(l[sel[j]] - top);
                for (int j = 0; j < k; ++j)
                    gate[t * k + j] = exp(l[sel[j]] - top) / s;
            } else {
                double s = 0.0;
                for (int j = 0; j < k; ++j)
                    s += p[sel[j]];
                for (int j = 0; j < k; ++j)
                    gate[t * k + j] = renormalize ? p[sel[j]] / s : p[sel[j]];
            }
        }
        free(ord);
        free(sel);
        free(p);
        free(gscore);
        free(gcnt);
        free(gord);
        free(allowed);
    }
}

/* ------------------------------------------------------------------ */
/* Dispatch as a local permutation.                                    */
/*                                                                     */
/* [P4 Expert parallelism]: step 1 sends every token to the owners of  */
/* the experts it chose; on one GPU that becomes grouping the (token,  */
/* slot) pairs by expert.  [P5 Capacity factor]: an expert takes at    */
/* most C = capacity_factor * T / N tokens, the overflow is dropped.   */
/* READING: C = floor(cf*T/N); cf <= 0 means no limit; an expert's     */
/* entries are taken in increasing token order and the first C kept.   */
/*                                                                     */
/* Outputs: counts[e] = pairs routed to e before dropping; kept[e] =   */
/* min(counts[e], C); offsets = exclusive prefix sum of kept (N+1);    */
/* perm[offsets[e] + r] = t*k + j of the r-th kept pair of e;          */
/* inv_row[t*k + j] = its row or -1; drop[t*k + j] = 1 if dropped.     */
/* Returns R = offsets[N].                                             */
/* ------------------------------------------------------------------ */
/*                                                                     */
/* The same paragraph: overflowing tokens are "either dropped ... or    */
/* re-routed to a shared fallback expert".  READING (fallback != 0):    */
/* the fallback is one more expert, index N, stored after the N routed */
/* experts and without a capacity limit; every pair an expert cannot   */
/* keep goes to it, in the order the pairs are taken, and keeps its    */
/* gate weight.  offsets then has N + 2 entries (the fallback's rows   */
/* are [offsets[N], offsets[N+1])).                                     */
/* Order in which pairs are taken: token by token (t, then slot j),    */
/* or, with slot_priority, slot by slot (every token's first choice    */
/* before any token's second; READING of priority dropping for k > 1).  */
/* expert_of[i]: the group pair i went to (its expert, N, or -1).       */
/* ------------------------------------------------------------------ */
int64_t orc_dispatch(int64_t T, int N, int k, double capacity_factor,
                     const int32_t *idx, int32_t *counts, int32_t *kept,
                     int32_t *offsets, int32_t *perm, int32_t *inv_row, uint8_t *drop,
                     int fallback, int slot_priority, int32_t *expert_of)
{
    int64_t C = -1;
    if (capacity_factor > 0)
        C = (int64_t)floor(capacity_factor * (double)T / (double)N);
    for (int e = 0; e < N; ++e)
        counts[e] = 0;
    for (int64_t i = 0; i < T * k; ++i)
        counts[idx[i]] += 1;
    offsets[0] = 0;
    int64_t over = 0;
    for (int e = 0; e < N; ++e) {
        kept[e] = (C < 0 || counts[e] <= C) ? counts[e] : (int32_t)C;
        offsets[e + 1] = offsets[e] + kept[e];
        over += counts[e] - kept[e];
    }
    if (fallback)
        offsets[N + 1] = offsets[N] + (int32_t)over;
    int32_t *seen = (int32_t *)calloc((size_t)N, sizeof(int32_t));
    int32_t fb = 0;
    for (int64_t p = 0; p < T * k; ++p) {
        const int64_t i = slot_priority ? (p % T) * k + p / T : p;
        const int e = idx[i];
        const int32_t r = seen[e]++;
        if (C < 0 || r < C) {
            drop[i] = 0;
            inv_row[i] = offsets[e] + r;
            perm[offsets[e] + r] = (int32_t)i;
            expert_of[i] = e;
        } else if (fallback) {
            const int32_t row = offsets[N] + fb++;
            drop[i] = 0;
            inv_row[i] = row;
            perm[row] = (int32_t)i;
            expert_of[i] = N;
        } else {
            drop[i] = 1;
            inv_row[i] = -1;
            expert_of[i] = -1;
        }
    }
    free(seen);
    return fallback ? offsets[N + 1] : offsets[N];
}

/* ------------------------------------------------------------------ */
/* Aux load-balancing statistics.  [P5 Load balancing]:                */
/*   L_aux = alpha * N * sum_i f_i * p_i                                */
/* f_i: share of routed assignments that went to expert i; p_i: mean   */
/* router probability of expert i over the batch.                      */
/* READING: f_i counts the router's assignments before capacity        */
/* dropping and is normalised by T*k (so the f_i sum to 1); p_i is the */
/* full softmax over N averaged over the T tokens.                     */
/* ------------------------------------------------------------------ */
void orc_aux(int64_t T, int N, int k, double alpha, const int32_t *counts,
             const double *probs, double *f, double *pmean, double *laux)
{
    double s = 0.0;
    for (int e = 0; e < N; ++e) {
        f[e] = (double)counts[e] / (double)(T * k);
        double acc = 0.0;
        for (int64_t t = 0; t < T; ++t)
            acc += probs[t * (int64_t)N + e];
        pmean[e] = acc / (double)T;
        s += f[e] * pmean[e];
    }
    *laux = alpha * (double)N * s;
}

/* ------------------------------------------------------------------ */
/* FP8 E4M3 (OCP OFP8 rev 1.0): 1 sign bit, 4 exponent bits (bias 7),  */
/* 3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; field  */
/* 15 with mantissa 7 is NaN, so the largest finite value is           */
/* 1.75 * 2^8 = 448; there are no infinities.                          */
/* ------------------------------------------------------------------ */
double orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, E = (c >> 3) & 15, M = c & 7;
    double v;
    if (E == 15 && M == 7)
        return NAN;
    if (E == 0)
        v = ldexp((double)M, -9);
    else
        v = ldexp(1.0 + M / 8.0, E - 7);
    return s ? -v : v;
}

/* Round-to-nearest-even to E4M3 with saturation to +-448 (finite input). */
uint8_t orc_e4m3_encode(double v)
{
    uint8_t s = (v < 0 || (v == 0 && signbit(v))) ? 0x80 : 0;
    double a = fabs(v);
    if (a >= 448.0)
        return s | 0x7E;
    /* spacing of representable values around a */
    double q;
    if (a < ldexp(1.0, -6)) {
        q = ldexp(1.0, -9);
    } else {
        int ex;
        frexp(a, &ex);              /* a = f * 2^ex, f in [0.5, 1) */
        q = ldexp(1.0, (ex - 1) - 3);
    }
    double r = nearbyint(a / q) * q;   /* default rounding: to nearest, ties even */
    if (r >= 448.0)
        return s | 0x7E;
    if (r == 0.0)
        return s;
    if (r < ldexp(1.0, -6))
        return s | (uint8_t)(r / ldexp(1.0, -9));
    int ex;
    double f = frexp(r, &ex);          /* r = f * 2^ex, f in [0.5,1) -> 1.m * 2^(ex-1) */
    int E = (ex - 1) + 7;
    int M = (int)((f * 2.0 - 1.0) * 8.0);
    return s | (uint8_t)(E << 3) | (uint8_t)M;
}

/* ------------------------------------------------------------------ */
/* Per-token FP8 quantisation of the dispatch payload.  [P4 Worked      */
/* example: bytes per token]: the payload is quantised to FP8 before   */
/* dispatch (one byte per number).  READING: one fp32 scale per token,  */
/* scale = amax / 448 (1 if the row is all zero), code =                */
/* E4M3_RNE_satfinite(x / scale).  amax/448 and x/scale are evaluated   */
/* as IEEE fp32 operations so that the code each element gets is       */
/* decided in the same precision as on the device.                     */
/* ------------------------------------------------------------------ */
void orc_quantize_rows(int64_t nrows, int d, const void *x, int xdt,
                       uint8_t *q, float *scale)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nrows; ++t) {
        float amax = 0.0f;
        for (int j = 0; j < d; ++j) {
            float a = (float)fabs(ld(x, xdt, t * (int64_t)d + j));
            if (a > amax)
                amax = a;
        }
        volatile float s = (amax > 0.0f) ? amax / 448.0f : 1.0f;
        scale[t] = s;
        for (int j = 0; j < d; ++j) {
            volatile float v = (float)ld(x, xdt, t * (int64_t)d + j) / s;
            q[t * (int64_t)d + j] = orc_e4m3_encode((double)v);
        }
    }
}

/* ------------------------------------------------------------------ */
/* One expert FFN applied to one row (fp64).  The pages call the       */
/* experts feed-forward networks ([P5] core idea); the two forms used  */
/* here come from the workload definitions:                            */
/*   ReLU:   y = max(x W1, 0) W2                                       */
/*   SwiGLU: y = (silu(x W1) * (x W3)) W2,  silu(a) = a / (1 + e^-a)   */
/* W1, W3 stored [H][d] (row h = column h of the d x H matrix), W2     */
/* stored [d][H]; the pointers address this expert's block.            */
/* ------------------------------------------------------------------ */
void orc_ffn_row(int d, int H, int act, const double *xrow,
                 const void *W1, const void *W3, const void *W2, int wdt,
                 double *y)
{
    double *h = (double *)malloc(sizeof(double) * (size_t)H);
    for (int c = 0; c < H; ++c) {
        double a = 0.0;
        for (int j = 0; j < d; ++j)
            a += xrow[j] * ld(W1, wdt, (int64_t)c * d + j);
        if (act == ORC_RELU) {
            h[c] = a > 0.0 ? a : 0.0;
        } else {
            double b = 0.0;
            for (int j = 0; j < d; ++j)
                b += xrow[j] * ld(W3, wdt, (int64_t)c * d + j);
            h[c] = a / (1.0 + exp(-a)) * b;
        }
    }
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int c = 0; c < H; ++c)
            s += h[c] * ld(W2, wdt, (int64_t)i * H + c);
        y[i] = s;
    }
    free(h);
}

/* ------------------------------------------------------------------ */
/* Layer output for a list of tokens.  [P5 Router design] and [P3 The  */
/* Math]: y = sum over the selected experts i of G(x)_i E_i(x).         */
/* A dropped (token, slot) contributes nothing ([P5 Capacity factor]);  */
/* the always-on shared expert ([P5] DeepSeek-V2 note) is added with   */
/* coefficient 1 to every token on the unquantised input.              */
/*                                                                     */
/* xin: expert input rows, one per token of the list, fp64 [ntok][d]   */
/*      (the dequantised FP8 payload when dispatch is FP8);             */
/* xsh: shared-expert input rows [ntok][d] or NULL;                     */
/* idx, gate, drop: routing of the listed tokens, [ntok][k].           */
/* ------------------------------------------------------------------ */
void orc_layer_rows(int64_t ntok, int d, int H, int k, int act, int wdt,
                    const double *xin, const double *xsh,
                    const int32_t *idx, const double *gate, const uint8_t *drop,
                    const void *W1, const void *W3, const void *W2,
                    int Hs, const void *Ws1, const void *Ws3, const void *Ws2,
                    double *y)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < ntok; ++t) {
        double *yt = y + t * (int64_t)d;
        double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
        for (int i = 0; i < d; ++i)
            yt[i] = 0.0;
        for (int j = 0; j < k; ++j) {
            if (drop[t * k + j])
                continue;
            int64_t e = idx[t * k + j];
            size_t wsz = (wdt == ORC_F32) ? 4 : 2;
            const char *w1 = (const char *)W1 + (size_t)e * H * d * wsz;
            const char *w3 = W3 ? (const char *)W3 + (size_t)e * H * d * wsz : NULL;
            const char *w2 = (const char *)W2 + (size_t)e * d * H * wsz;
            orc_ffn_row(d, H, act, xin + t * (int64_t)d, w1, w3, w2, wdt, tmp);
            for (int i = 0; i < d; ++i)
                yt[i] += gate[t * k + j] * tmp[i];
        }
        if (Hs > 0 && xsh) {
            orc_ffn_row(d, Hs, act, xsh + t * (int64_t)d, Ws1, Ws3, Ws2, wdt, tmp);
            for (int i = 0; i < d; ++i)
                yt[i] += tmp[i];
        }
        free(tmp);
    }
}
