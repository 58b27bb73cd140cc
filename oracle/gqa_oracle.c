/*
 * gqa_oracle.c -- plain, slow, fp64 CPU restatement of grouped-query
 * attention (GQA).  TEST INFRASTRUCTURE ONLY: the test suite, the package
 * smoke check and the CPU-baseline leg of bench.py are the only code allowed
 * to load this library.  The CUDA library never links or calls it, and it
 * shares no source with the CUDA kernels.
 *
 * What it follows (page title, section):
 *   - "Grouped-Query Attention" (llm-arch-kb), section 2 "Derivation":
 *       the group index of query head i is g(i) = ceil(i*G/H) over 1-indexed
 *       heads, with G | H and contiguous groups ("The grouping"); each new
 *       GQA key/value head is initialised as the mean of the original heads
 *       assigned to its group ("Uptraining recipe (averaging-init)");
 *       the KV cache holds 2*G*d_h scalars per token per layer
 *       ("KV-cache footprint").
 *   - same page, section 3 "Reference implementation": scores are
 *       q.k / sqrt(d_h), a causal mask is applied, softmax runs over the key
 *       axis, and the probabilities weight the values; each KV head is shared
 *       by H/G query heads (repeat_interleave along the head axis).
 *   - same page, section 1 "Premise": at decode every cached key/value of
 *       the sequence is read to produce the next token.
 *
 * Readings taken where the pages are silent:
 *   - decode attends over exactly seqlens[b] cached positions; an empty
 *     cache (seqlens[b] == 0) yields a zero output row;
 *   - the causal mask keeps key t for query s when t <= s (diagonal kept);
 *   - a sliding window of W keys (section 4 names sliding-window attention
 *     alongside GQA for Mistral 7B) keeps, for prefill query s, the keys
 *     s - W < t <= s, and for decode the last W cached positions;
 *   - softmax is evaluated in two plain passes (maximum, then exp/sum);
 *     there is no running rescale and no split of the key axis.
 *
 * Every arithmetic step is IEEE binary64 in the order written; build with
 * -ffp-contract=off and without -ffast-math.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { OR_F64 = 0, OR_F32 = 1, OR_BF16 = 2 };

/* Exact upcast of one stored element to binary64. */
static double ld(const void *p, int dt, size_t i) {
    if (dt == OR_F64) return ((const double *)p)[i];
    if (dt == OR_F32) return (double)((const float *)p)[i];
    /* bfloat16 is the top half of a binary32 word */
    uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------ */
/* group map                                                           */
/* ------------------------------------------------------------------ */

/* g(i) = ceil(i*G/H) for 1-indexed head i ("Grouped-Query Attention",
 * section 2, "The grouping").  Takes and returns 0-indexed numbers. */
int oracle_group_of_head(int i0, int H, int G) {
    long i = (long)i0 + 1;
    long g = (i * (long)G + (long)H - 1) / (long)H; /* ceil for positive ints */
    return (int)(g - 1);
}

/* ------------------------------------------------------------------ */
/* KV-cache size                                                       */
/* ------------------------------------------------------------------ */

/* Bytes the cache adds per token: one key and one value vector of d_h
 * scalars for each of the G KV heads in each of L layers ("Grouped-Query
 * Attention", section 2, "KV-cache footprint"; G = H gives the MHA figure of
 * section 1). */
uint64_t oracle_kv_cache_bytes(int G, int d_h, int L, int elem_bytes) {
    return (uint64_t)2 * (uint64_t)G * (uint64_t)d_h * (uint64_t)L *
           (uint64_t)elem_bytes;
}

/* ------------------------------------------------------------------ */
/* one attention row                                                   */
/* ------------------------------------------------------------------ */

typedef struct {
    const void *p;
    int dt;
} arr_t;

/* out[0..d_h) = sum_t softmax_t(scale * <q, k_t>) v_t over t in [0, n).
 * q at q_off (contiguous d_h), key t at k_off + t*kv_stride, value t at
 * v_off + t*kv_stride.  s is caller scratch of n doubles. */
static void attend_row(arr_t q, size_t q_off, arr_t K, size_t k_off, arr_t V,
                       size_t v_off, size_t kv_stride, long n, int d_h,
                       double scale, double *out, double *s) {
    for (int c = 0; c < d_h; ++c) out[c] = 0.0;
    if (n <= 0) return;
    /* pass 1: scores and their maximum */
    double mx = -INFINITY;
    for (long t = 0; t < n; ++t) {
        double acc = 0.0;
        for (int c = 0; c < d_h; ++c)
            acc += ld(q.p, q.dt, q_off + (size_t)c) *
                   ld(K.p, K.dt, k_off + (size_t)t * kv_stride + (size_t)c);
        s[t] = scale * acc;
        if (s[t] > mx) mx = s[t];
    }
    /* pass 2: exponentials, their sum, and the weighted sum of values */
    double den = 0.0;
    for (long t = 0; t < n; ++t) {
        double e = exp(s[t] - mx);
        den += e;
        for (int c = 0; c < d_h; ++c)
            out[c] += e * ld(V.p, V.dt, v_off + (size_t)t * kv_stride + (size_t)c);
    }
    for (int c = 0; c < d_h; ++c) out[c] /= den;
}

/* ------------------------------------------------------------------ */
/* a tiny work-sharing pool over independent output rows               */
/* ------------------------------------------------------------------ */

typedef void (*unit_fn)(void *ctx, long unit, double *scratch);

typedef struct {
    unit_fn fn;
    void *ctx;
    long n_units;
    long next;
    size_t scratch_len;
    int failed;
} pool_t;

static void *pool_worker(void *arg) {
    pool_t *pl = (pool_t *)arg;
    double *scratch = (double *)malloc(pl->scratch_len * sizeof(double) + 64);
    if (!scratch) {
        __atomic_store_n(&pl->failed, 1, __ATOMIC_SEQ_CST);
        return NULL;
    }
    for (;;) {
        long u = __atomic_fetch_add(&pl->next, 1, __ATOMIC_RELAXED);
        if (u >= pl->n_units) break;
        pl->fn(pl->ctx, u, scratch);
    }
    free(scratch);
    return NULL;
}

int oracle_default_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

static int run_pool(unit_fn fn, void *ctx, long n_units, size_t scratch_len,
                    int nthreads) {
    pool_t pl = {fn, ctx, n_units, 0, scratch_len, 0};
    if (nthreads <= 0) nthreads = oracle_default_threads();
    if (nthreads > n_units) nthreads = n_units > 0 ? (int)n_units : 1;
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!th) return -1;
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, pool_worker, &pl) == 0) ++started;
    if (started == 0) pool_worker(&pl);
    for (int i = 0; i < nthreads; ++i)
        if (th[i]) pthread_join(th[i], NULL);
    free(th);
    return pl.failed ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* decode: one new query token per sequence                            */
/* ------------------------------------------------------------------ */

typedef struct {
    arr_t q, K, V;
    const int32_t *seqlens;
    double scale;
    double *out;
    int B, H, G, d_h, T_cap;
    int kv_heads;          /* G for GQA, H for per-head MHA */
    int per_head_kv;       /* 1: head i reads KV head i (MHA)  */
    const int64_t *rows;   /* optional list of (b*H + i) rows */
    int window;            /* > 0: only the last `window` cached positions */
} dec_ctx;

static void decode_unit(void *vc, long u, double *s) {
    dec_ctx *c = (dec_ctx *)vc;
    long row = c->rows ? (long)c->rows[u] : u;
    int b = (int)(row / c->H), i = (int)(row % c->H);
    int kvh = c->per_head_kv ? i : oracle_group_of_head(i, c->H, c->G);
    long n = c->seqlens[b];
    if (n > c->T_cap) n = c->T_cap;
    if (n < 0) n = 0;
    long first = 0; /* first cached position attended */
    if (c->window > 0 && n > c->window) first = n - c->window;
    size_t q_off = ((size_t)b * c->H + i) * c->d_h;
    size_t kv_off = ((((size_t)b * c->kv_heads + kvh) * c->T_cap) + (size_t)first) * c->d_h;
    attend_row(c->q, q_off, c->K, kv_off, c->V, kv_off, (size_t)c->d_h, n - first,
               c->d_h, c->scale, c->out + (size_t)u * c->d_h, s);
}

/* GQA decode.  q [B,H,d_h]; K,V [B,G,T_cap,d_h]; seqlens [B];
 * out [B,H,d_h] (or [n_rows,d_h] when rows != NULL, rows[j] = b*H + i). */
int oracle_gqa_decode(const void *q, int q_dt, const void *K, const void *V,
                      int kv_dt, const int32_t *seqlens, double scale,
                      double *out, int B, int H, int G, int d_h, int T_cap,
                      const int64_t *rows, long n_rows, int nthreads, int window) {
    if (G <= 0 || H % G != 0) return -1;
    dec_ctx c = {{q, q_dt}, {K, kv_dt}, {V, kv_dt}, seqlens, scale, out,
                 B, H, G, d_h, T_cap, G, 0, rows, window};
    long n = rows ? n_rows : (long)B * H;
    return run_pool(decode_unit, &c, n, (size_t)T_cap, nthreads);
}

/* Per-head MHA decode (each head owns its K/V head).  K,V [B,H,T_cap,d_h]. */
int oracle_mha_decode(const void *q, int q_dt, const void *K, const void *V,
                      int kv_dt, const int32_t *seqlens, double scale,
                      double *out, int B, int H, int d_h, int T_cap,
                      int nthreads) {
    dec_ctx c = {{q, q_dt}, {K, kv_dt}, {V, kv_dt}, seqlens, scale, out,
                 B, H, H, d_h, T_cap, H, 1, NULL, 0};
    return run_pool(decode_unit, &c, (long)B * H, (size_t)T_cap, nthreads);
}

/* ------------------------------------------------------------------ */
/* causal prefill                                                      */
/* ------------------------------------------------------------------ */

typedef struct {
    arr_t q, k, v;
    double scale;
    double *out;
    int B, S, H, G, d_h;
    const int64_t *rows; /* optional list of ((b*S + s)*H + i) */
    int window;          /* > 0: keys s - window < t <= s */
} pre_ctx;

static void prefill_unit(void *vc, long u, double *sc) {
    pre_ctx *c = (pre_ctx *)vc;
    long row = c->rows ? (long)c->rows[u] : u;
    int i = (int)(row % c->H);
    long bs = row / c->H;
    int s = (int)(bs % c->S), b = (int)(bs / c->S);
    int g = oracle_group_of_head(i, c->H, c->G);
    size_t q_off = (((size_t)b * c->S + s) * c->H + i) * c->d_h;
    long first = 0; /* causal mask: query s sees keys first..s */
    if (c->window > 0 && (long)s + 1 > c->window) first = (long)s + 1 - c->window;
    size_t kv_off = (((size_t)b * c->S + (size_t)first) * c->G + g) * c->d_h;
    size_t stride = (size_t)c->G * c->d_h; /* token-major k/v */
    attend_row(c->q, q_off, c->k, kv_off, c->v, kv_off, stride, (long)s + 1 - first,
               c->d_h, c->scale, c->out + (size_t)u * c->d_h, sc);
}

/* Causal GQA prefill.  q [B,S,H,d_h]; k,v [B,S,G,d_h];
 * out [B,S,H,d_h] or [n_rows,d_h] for rows[j] = (b*S + s)*H + i. */
int oracle_gqa_prefill_causal(const void *q, const void *k, const void *v,
                              int dt, double scale, double *out, int B, int S,
                              int H, int G, int d_h, const int64_t *rows,
                              long n_rows, int nthreads, int window) {
    if (G <= 0 || H % G != 0) return -1;
    pre_ctx c = {{q, dt}, {k, dt}, {v, dt}, scale, out, B, S, H, G, d_h, rows, window};
    long n = rows ? n_rows : (long)B * S * H;
    return run_pool(prefill_unit, &c, n, (size_t)S, nthreads);
}

/* ------------------------------------------------------------------ */
/* mean-pool initialisation of the G key/value heads                   */
/* ------------------------------------------------------------------ */

/* W [H, n] (n = d_h*d, one head's projection flattened) -> mean [G, n].
 * Each group's head is the plain mean of the heads i with g(i) == g,
 * summed in ascending head order in binary64 and divided by their count
 * ("Grouped-Query Attention", section 2, "Uptraining recipe"). */
int oracle_meanpool(const void *W, int dt, int H, int G, size_t n,
                    double *mean) {
    if (G <= 0 || H % G != 0) return -1;
    long *count = (long *)calloc((size_t)G, sizeof(long));
    if (!count) return -1;
    memset(mean, 0, sizeof(double) * (size_t)G * n);
    for (int i = 0; i < H; ++i) {
        int g = oracle_group_of_head(i, H, G);
        count[g] += 1;
        double *acc = mean + (size_t)g * n;
        for (size_t e = 0; e < n; ++e) acc[e] += ld(W, dt, (size_t)i * n + e);
    }
    for (int g = 0; g < G; ++g)
        for (size_t e = 0; e < n; ++e)
            mean[(size_t)g * n + e] /= (double)count[g];
    free(count);
    return 0;
}

/* ------------------------------------------------------------------ */
/* rounding of binary64 results to the storage types                   */
/* ------------------------------------------------------------------ */

/* Round-to-nearest-even of x to bfloat16 (8 significant bits, binary32
 * exponent range, subnormals spaced 2^-133), returned as its bit pattern. */
static uint16_t bf16_rne_bits(double x) {
    if (isnan(x)) return (uint16_t)0x7FC0;
    uint16_t sign = signbit(x) ? (uint16_t)0x8000 : (uint16_t)0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e;
    (void)frexp(a, &e);          /* a in [2^(e-1), 2^e) */
    int lead = e - 1;
    if (lead < -126) lead = -126; /* below the normal range the spacing is fixed */
    double ulp = ldexp(1.0, lead - 7);
    double r = nearbyint(a / ulp) * ulp; /* a/ulp is exact: power-of-two scale */
    if (r > 0x1.FEp127) return (uint16_t)(sign | 0x7F80);
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

void oracle_round_bf16(const double *x, uint16_t *bits, size_t n) {
    for (size_t i = 0; i < n; ++i) bits[i] = bf16_rne_bits(x[i]);
}

/* Round-to-nearest-even to binary32 (C conversion under the default mode). */
void oracle_round_f32(const double *x, float *y, size_t n) {
    for (size_t i = 0; i < n; ++i) y[i] = (float)x[i];
}

/* ------------------------------------------------------------------ */
/* projections of one token (decode step) and the KV-cache append      */
/* ------------------------------------------------------------------ */

/* out[b, n] = sum_k h[b, k] * W[k, n] in binary64 (ascending k).
 * h [B, d]; W [d, N] row-major as in the sketch's h @ W ("Grouped-Query
 * Attention", section 3: q = h @ W_Q, k = h @ W_K, v = h @ W_V). */
int oracle_project(const void *h, int h_dt, const void *W, int w_dt, double *out, int B, int d,
                   int N) {
    for (int b = 0; b < B; ++b)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < d; ++k)
                acc += ld(h, h_dt, (size_t)b * d + k) * ld(W, w_dt, (size_t)k * N + n);
            out[(size_t)b * N + n] = acc;
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* other initialisations of the G heads from the H MHA heads           */
/* ------------------------------------------------------------------ */

/* mode 1: out[g] = W[g*r + sel] -- picking one head per group, the first
 *         alternative the GQA paper compares with averaging ("Grouped-Query
 *         Attention", section 2, "Uptraining recipe");
 * mode 2: out[g] = sum_{i: g(i)=g} w[i] * W[i], ascending i, binary64 products
 *         and sums -- a weighted average over the heads of a group with
 *         caller-given weights (section 4, weighted grouped-query attention).
 * W [H, n]; out [G, n] in binary64 (rounded by the caller). */
int oracle_init_heads(const void *W, int dt, int H, int G, size_t n, int mode, const double *w,
                      int sel, double *out) {
    if (G <= 0 || H % G != 0) return -1;
    const int r = H / G;
    if (mode == 1) {
        if (sel < 0 || sel >= r) return -1;
        for (int i = 0; i < H; ++i) {
            int g = oracle_group_of_head(i, H, G);
            if (i - g * r != sel) continue; /* the head's position inside its group */
            for (size_t e = 0; e < n; ++e) out[(size_t)g * n + e] = ld(W, dt, (size_t)i * n + e);
        }
        return 0;
    }
    if (mode == 2) {
        memset(out, 0, sizeof(double) * (size_t)G * n);
        for (int i = 0; i < H; ++i) {
            int g = oracle_group_of_head(i, H, G);
            for (size_t e = 0; e < n; ++e)
                out[(size_t)g * n + e] += w[i] * ld(W, dt, (size_t)i * n + e);
        }
        return 0;
    }
    return -1;
}
