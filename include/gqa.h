/*
 * gqa.h -- C ABI of libgqa.so: grouped-query attention (GQA) on NVIDIA B200
 * (sm_100a).
 *
 * Notation.  B batch, H query heads, G key/value heads with G | H, r = H/G
 * query heads per group, d_h head dimension, T_cap cache capacity, S prompt
 * length, d model dimension.  Query head i (0-indexed) reads KV head i / r,
 * the 0-indexed form of g(i) = ceil(i*G/H) over 1-indexed heads
 * ("Grouped-Query Attention", llm-arch-kb, section 2 "Derivation", "The
 * grouping": G contiguous groups of H/G query heads).
 *
 * Conventions shared by every call.
 *   - Pointers named as device pointers must point to device memory (or
 *     memory the device can address) that stays valid until the work queued
 *     on `stream` has finished.  Host pointers are read before the call
 *     returns.  The library keeps no pointer after a call returns, allocates
 *     no device memory, and owns nothing but a device status word.
 *   - Tensors are dense and row-major in the order of their shape; no strides.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and returns a status code.  Arguments are
 *     validated on the host before any launch; an invalid call launches
 *     nothing and returns a negative code, with the reason available from
 *     gqa_last_error_string() on the calling thread.
 *   - Conditions only the device can see (a seqlens entry outside [0, T_cap],
 *     a bounded wait that ran out) set bits of a device status word that
 *     gqa_get_status() reads and clears.  No kernel traps.
 *   - libgqa_debug.so is the same library built with device-side index
 *     checks: before a kernel uses an index it derived (a cache row, a
 *     partial-record slot, a head, a weight row) it checks that the index
 *     stays inside its buffer; a failed check skips the access and sets a
 *     status bit (GQA_ERR_INDEX from gqa_get_status).  Same ABI and results.
 *   - Results are deterministic: the same inputs and launch give the same bits.
 *   - Kernels are launched as programmatic dependents: a call's set-up may
 *     overlap the end of the work before it on `stream`, but no kernel uses an
 *     input's value before that work has completed, so ordinary stream
 *     ordering holds.  (The decode kernels read seqlens early to guess their
 *     first cache tiles and ask L2 to fetch them: a hint, which a value still
 *     being written can make wasted but cannot make wrong.)  Calls can be
 *     captured in CUDA graphs.
 */
#ifndef GQA_H
#define GQA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GQA_API __attribute__((visibility("default")))
#else
#define GQA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *gqa_stream_t; /* same type as cudaStream_t */

typedef enum { GQA_F32 = 0, GQA_BF16 = 1 } gqa_dtype;

enum {
    GQA_OK = 0,
    GQA_ERR_INVALID = -1,     /* bad shape, null pointer, G does not divide H */
    GQA_ERR_UNSUPPORTED = -2, /* valid but not built: d_h, dtype, group size  */
    GQA_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned             */
    GQA_ERR_CUDA = -4,        /* a CUDA runtime or driver call failed         */
    GQA_ERR_WORKSPACE = -5,   /* workspace missing or too small               */
    GQA_ERR_TIMEOUT = -6,     /* device: a bounded wait ran out               */
    GQA_ERR_SEQLEN = -7,      /* device: a seqlens entry was outside [0,T_cap] */
    GQA_ERR_INDEX = -8        /* device, debug build only: an index check failed */
};

/*
 * gqa_kv_cache_bytes -- bytes the KV cache grows by per token: one key and one
 * value vector of d_h scalars for each of G KV heads in each of L layers,
 * 2 * G * d_h * L * elem_bytes ("Grouped-Query Attention", llm-arch-kb,
 * section 2 "KV-cache footprint"; G = H gives the MHA figure of section 1
 * "Premise", G = 1 the MQA one).  Pure host arithmetic; returns 0 if any
 * argument is not positive.
 */
GQA_API uint64_t gqa_kv_cache_bytes(int G, int d_h, int L, int elem_bytes);

/*
 * gqa_decode_workspace_bytes -- device workspace gqa_decode needs for this
 * shape on the current device (it depends on the device's SM count).  Returns
 * 0 for an invalid shape.  The caller allocates it (any device allocation,
 * 256-byte aligned) and may reuse it across calls on one stream; calls that
 * run concurrently need separate workspaces.
 */
GQA_API size_t gqa_decode_workspace_bytes(int B, int H, int G, int d_h, int T_cap,
                                  gqa_dtype dt);

/*
 * gqa_decode -- one decode step of GQA attention over a KV cache: for each
 * sequence b and query head i,
 *     out[b,i,:] = sum_{t < T_b} softmax_t(scale * <q[b,i,:], K[b,g,t,:]>) V[b,g,t,:]
 * with g = i / (H/G) and T_b = seqlens[b].  Every cached key and value of the
 * sequence is read once for the new token ("Grouped-Query Attention",
 * llm-arch-kb, section 1 "Premise"; scores, softmax over keys and the value
 * sum as in section 3 "Reference implementation").  Pass scale = 1/sqrt(d_h)
 * for the page's scaling.
 *
 *   q        device, [B, H, d_h]        dtype dt, 16-byte aligned
 *   k_cache  device, [B, G, T_cap, d_h] dtype dt, 16-byte aligned
 *   v_cache  device, [B, G, T_cap, d_h] dtype dt, 16-byte aligned
 *   seqlens  device, [B] int32; entries 0 <= T_b <= T_cap.  Positions >= T_b
 *            are never used (their contents may be anything, NaN included).
 *            Entries outside the range are clamped and flag GQA_ERR_SEQLEN.
 *            T_b = 0 gives a zero output row.
 *   out      device, [B, H, d_h] dtype dt, 16-byte aligned
 *   workspace device, >= gqa_decode_workspace_bytes(...) bytes, 256-byte
 *            aligned; scratch for per-split partial results and their
 *            completion flags.  Its contents need no initialisation.  Its
 *            first 256 bytes carry, from one call to the next, the generation
 *            number the completion flags are compared against; the device
 *            advances it on every call, so a call captured in a CUDA graph
 *            and replayed many times (with inputs changed in place between
 *            replays) never accepts flags an earlier replay left behind.  Do
 *            not write the workspace between calls that share it; after a
 *            call on it reports GQA_ERR_TIMEOUT, re-capture graphs that use it.
 *   dt       GQA_BF16 (tensor-core scores and P.V, fp32 softmax/accumulate)
 *            or GQA_F32 (fp32 CUDA-core arithmetic throughout).
 *   Supported: d_h in {64, 128}; bf16 needs H/G <= 64.
 * Internally: a split-KV kernel over equal shares of the cache tiles (TMA
 * staged, fp32 online softmax per split; warp-level MMAs for H/G <= 15,
 * tcgen05 with S, P and O in tensor memory for 16 <= H/G <= 64) and a combine
 * kernel that merges the per-split (max, sum, partial output) triples
 * exactly, starting on a segment as soon as its splits have published their
 * results.
 */
GQA_API int gqa_decode(const void *q, const void *k_cache, const void *v_cache,
               const int32_t *seqlens, float scale, void *out, int B, int H,
               int G, int d_h, int T_cap, gqa_dtype dt, void *workspace,
               size_t workspace_bytes, gqa_stream_t stream);

/*
 * gqa_decode_window -- gqa_decode with a sliding window: each sequence
 * attends over its last min(T_b, window) cached positions only,
 * [T_b - window, T_b), instead of all T_b ("Grouped-Query Attention",
 * llm-arch-kb, section 4: Mistral 7B pairs GQA with sliding-window
 * attention).  window = 0 is gqa_decode.  Same arguments, workspace and
 * limits as gqa_decode; window < 0 is GQA_ERR_INVALID.
 */
GQA_API int gqa_decode_window(const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *seqlens, float scale, void *out, int B, int H,
                              int G, int d_h, int T_cap, int window, gqa_dtype dt,
                              void *workspace, size_t workspace_bytes, gqa_stream_t stream);

/*
 * gqa_decode_noalloc -- gqa_decode for callers that cannot allocate device
 * memory.  (The pages have no counterpart: this is a deployment convenience.)
 *
 * gqa_decode needs scratch for its per-split partial results, which its caller
 * allocates.  Some callers cannot: a plug-in inside a host runtime that has
 * already reserved the device's memory for its own allocator, or a serving loop
 * that must not allocate after start-up because an allocation could stall or
 * fail it.  This entry point takes the same arguments as gqa_decode minus the
 * workspace and uses a scratch array compiled into the library instead:
 *   - the array holds GQA_DECODE_NOALLOC_SCRATCH_BYTES (8 MiB) and stays
 *     resident on every GPU that loads the library until the process exits;
 *   - shapes whose scratch (gqa_decode_workspace_bytes) exceeds it are rejected
 *     with GQA_ERR_WORKSPACE before anything is launched;
 *   - the first call on a device looks up the array's device address on that
 *     device (a one-time set-up); make that first call before any stream
 *     capture;
 *   - all calls on a device share the one array: two calls whose kernels can
 *     overlap on the GPU (different streams with no ordering) race on it;
 *   - the array keeps the last call's contents; nothing in it needs to start
 *     at zero, since each call writes every record it reads.
 * It never calls cudaMalloc, cudaFree or any allocating routine.  Results are
 * those of gqa_decode on the same inputs.
 */
#define GQA_DECODE_NOALLOC_SCRATCH_BYTES (8u << 20)
GQA_API int gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *seqlens, float scale, void *out, int B, int H,
                               int G, int d_h, int T_cap, gqa_dtype dt, gqa_stream_t stream);

/*
 * gqa_prefill_causal -- causal GQA attention over a whole prompt: for each b,
 * position s and query head i,
 *     out[b,s,i,:] = sum_{t <= s} softmax_t(scale * <q[b,s,i,:], k[b,t,g,:]>) v[b,t,g,:]
 * with g = i / (H/G) ("Grouped-Query Attention", llm-arch-kb, section 3
 * "Reference implementation": scores over sqrt(d_h), causal mask, softmax on
 * the key axis, K/V broadcast to the H/G heads of each group).  The mask keeps
 * the diagonal (t = s).  Pass scale = 1/sqrt(d_h) for the page's scaling.
 *
 *   q    device, [B, S, H, d_h] bf16, 16-byte aligned
 *   k, v device, [B, S, G, d_h] bf16, 16-byte aligned
 *   out  device, [B, S, H, d_h] bf16, 16-byte aligned
 *   Supported: dt = GQA_BF16, d_h in {64, 128}, any G | H (G = H is MHA,
 *   G = 1 is MQA), scale > 0, any S >= 1.
 * Internally: tcgen05 tensor-core MMAs with fp32 accumulators in tensor
 * memory, TMA-fed shared-memory tiles, fp32 online softmax, P in bf16.  One
 * CTA takes 128 positions of two heads of a group (both read the same K/V
 * tiles); with an odd H/G the last head of each group runs alone.
 */
GQA_API int gqa_prefill_causal(const void *q, const void *k, const void *v, void *out,
                       int B, int S, int H, int G, int d_h, float scale,
                       gqa_dtype dt, gqa_stream_t stream);

/*
 * gqa_prefill_causal_window -- causal prefill with a sliding window of
 * `window` keys: query s sees keys s - window < t <= s (itself and the
 * window - 1 before it); KV tiles wholly outside every row's window are not
 * read.  window = 0 is gqa_prefill_causal.  Same arguments and limits.
 */
GQA_API int gqa_prefill_causal_window(const void *q, const void *k, const void *v, void *out,
                                      int B, int S, int H, int G, int d_h, float scale,
                                      int window, gqa_dtype dt, gqa_stream_t stream);

/*
 * gqa_meanpool_kv -- averaging initialisation of GQA key/value projections
 * from an MHA checkpoint: each of the G new heads is the plain mean of the H/G
 * original heads of its group,
 *     WK_out[g,:,:] = (sum_{j < r} WK[g*r + j,:,:]) / r,  same for WV,
 * summed in ascending head order in binary64, divided by r, then rounded once
 * to nearest-even in dt ("Grouped-Query Attention", llm-arch-kb, section 2
 * "Uptraining recipe (averaging-init)").  Bit-exact with that definition.
 *
 *   WK, WV          device, [H, d_h, d] dtype dt
 *   WK_out, WV_out  device, [G, d_h, d] dtype dt (must not overlap inputs)
 *   dt              GQA_BF16 or GQA_F32; any d_h, d >= 1.
 */
GQA_API int gqa_meanpool_kv(const void *WK, const void *WV, void *WK_out, void *WV_out,
                    int H, int G, int d_h, int d, gqa_dtype dt,
                    gqa_stream_t stream);

/*
 * gqa_qkv_append -- the step before decode, fused: one new token's query,
 * key and value projections, with the key and value written straight into
 * the KV cache ("Grouped-Query Attention", llm-arch-kb, section 3
 * "Reference implementation": q = h W_Q, k = h W_K, v = h W_V with only G
 * key/value heads; section 1 "Premise": the cache grows by one key and one
 * value vector per token, head and layer):
 *     q_out[b]               = h[b] W_Q                      (H heads of d_h)
 *     k_cache[b, g, T_b, :]  = (h[b] W_K)[g d_h : (g+1) d_h]  for each of G heads
 *     v_cache[b, g, T_b, :]  = (h[b] W_V)[g d_h : (g+1) d_h]
 *     seqlens_out[b]         = T_b + 1,     T_b = seqlens[b].
 * bf16 inputs, fp32 accumulation, each output rounded once to bf16.  Cache
 * positions other than T_b are not touched.  A sequence whose cache is full
 * (T_b >= T_cap) or whose T_b is negative gets no append, keeps
 * seqlens_out[b] = T_b and flags GQA_ERR_SEQLEN.
 *
 *   h                 device, [B, d] bf16, 16-byte aligned
 *   W_Q               device, [d, H*d_h] bf16 row-major, 16-byte aligned
 *   W_K, W_V          device, [d, G*d_h] bf16 row-major, 16-byte aligned
 *   q_out             device, [B, H, d_h] bf16
 *   k_cache, v_cache  device, [B, G, T_cap, d_h] bf16 (updated in place)
 *   seqlens           device, [B] int32 (read only)
 *   seqlens_out       device, [B] int32, or NULL; must not overlap seqlens
 *   workspace         device, >= gqa_project_workspace_bytes((H + 2G) d_h, d)
 *                     bytes, 256-byte aligned, or NULL (see below)
 *   Supported: dt = GQA_BF16, d a multiple of 128, d_h in {64, 128}.
 * Internally: a skinny GEMM bound by reading the weights once, one CTA per
 * 64 output columns.  With a workspace and at most a quarter as many column
 * blocks as SMs, each block's rows are also split into floor(SMs / blocks)
 * ranges on separate CTAs, all in one wave, and the ranges' fp32 partial sums
 * are added in a fixed order from the workspace (same results on every call;
 * they may differ from the unsplit kernel's in the last bit, since the sums
 * are grouped differently).  With more blocks the workspace is not used (on
 * B200 the split measured slower there).  It needs no initialisation; calls
 * that run concurrently need separate workspaces.
 */
GQA_API int gqa_qkv_append(const void *h, const void *W_Q, const void *W_K, const void *W_V,
                           void *q_out, void *k_cache, void *v_cache, const int32_t *seqlens,
                           int32_t *seqlens_out, int B, int d, int H, int G, int d_h, int T_cap,
                           gqa_dtype dt, void *workspace, size_t workspace_bytes, gqa_stream_t stream);

/*
 * gqa_project_workspace_bytes -- workspace the split-K projection kernel of
 * gqa_qkv_append and gqa_out_project needs on the current device (it depends
 * on the SM count) for ncols output columns (all three weights' for
 * gqa_qkv_append, (H + 2G) d_h; N for gqa_out_project) and a reduction over d
 * rows (K for gqa_out_project).  0 for a shape the kernels do not take.
 */
GQA_API size_t gqa_project_workspace_bytes(int ncols, int d);

/*
 * gqa_init_kv_heads -- the mean-pool initialisation and the two alternatives
 * the pages set against it, selected by `mode`:
 *   GQA_INIT_MEAN      the group mean, identical to gqa_meanpool_kv;
 *   GQA_INIT_SELECT    WK_out[g] = WK[g*r + select], picking one head of each
 *                      group ("Grouped-Query Attention", llm-arch-kb, section 2
 *                      "Uptraining recipe", the alternative reported worse than
 *                      averaging); an exact copy;
 *   GQA_INIT_WEIGHTED  WK_out[g] = sum_j wK[g*r + j] * WK[g*r + j] (same for V
 *                      with wV), a weighted average over the group's heads with
 *                      caller-given weights (section 4, weighted grouped-query
 *                      attention); binary64 products and sums in ascending head
 *                      order, one nearest-even rounding, bit-exact with that
 *                      definition.
 *   head_weights  device, [2, H] float: wK then wV (mode GQA_INIT_WEIGHTED only)
 *   select        0 <= select < H/G (mode GQA_INIT_SELECT only)
 * Other arguments and limits as gqa_meanpool_kv.
 */
enum { GQA_INIT_MEAN = 0, GQA_INIT_SELECT = 1, GQA_INIT_WEIGHTED = 2 };
GQA_API int gqa_init_kv_heads(const void *WK, const void *WV, void *WK_out, void *WV_out,
                              int H, int G, int d_h, int d, int mode,
                              const float *head_weights, int select, gqa_dtype dt,
                              gqa_stream_t stream);

/*
 * gqa_out_project -- the output projection of the attention block, the
 * concatenated heads times W_O ("Grouped-Query Attention", llm-arch-kb,
 * section 2: the outputs concatenate across heads and are projected by W_O;
 * section 3: o.reshape(B, T, H*d_h) @ W_O), for one token per sequence:
 *     out[b, :] = x[b, :] W                 x [B, K], W [K, N], out [B, N]
 * bf16 in, fp32 accumulation, one rounding to bf16.  Same skinny-GEMM kernels
 * as gqa_qkv_append, with the same optional workspace
 * (>= gqa_project_workspace_bytes(N, K) bytes, or NULL).  Supported: bf16, K
 * a multiple of 128, N of 64; x and W 16-byte aligned.
 */
GQA_API int gqa_out_project(const void *x, const void *W, void *out, int B, int K, int N,
                            gqa_dtype dt, void *workspace, size_t workspace_bytes,
                            gqa_stream_t stream);

/*
 * gqa_layer_decode_step -- one decode step of a whole GQA attention layer
 * (section 3's gqa() for one new token per sequence): gqa_qkv_append (q, and
 * k/v appended at seqlens[b]), then gqa_decode_window over seqlens_out
 * (which includes the new token), then gqa_out_project of the attention
 * output with W_O into out [B, d].  q and the attention output are kept in
 * bf16 in the workspace between the steps, and so are the projections'
 * partial sums when a projection takes the split-K kernel.
 *   W_O          device, [H*d_h, d] bf16
 *   seqlens_out  required: the lengths after the append
 *   workspace    >= gqa_layer_decode_workspace_bytes(...), 256-byte aligned
 * Other arguments as gqa_qkv_append and gqa_decode_window (window 0 = full).
 */
GQA_API size_t gqa_layer_decode_workspace_bytes(int B, int d, int H, int G, int d_h, int T_cap,
                                                gqa_dtype dt);
GQA_API int gqa_layer_decode_step(const void *h, const void *W_Q, const void *W_K,
                                  const void *W_V, const void *W_O, void *k_cache,
                                  void *v_cache, const int32_t *seqlens, int32_t *seqlens_out,
                                  float scale, int window, void *out, int B, int d, int H, int G,
                                  int d_h, int T_cap, gqa_dtype dt, void *workspace,
                                  size_t workspace_bytes, gqa_stream_t stream);

/*
 * gqa_get_status -- synchronises `stream`, then reads and clears the device
 * status word: GQA_OK, GQA_ERR_SEQLEN, GQA_ERR_TIMEOUT or (debug build)
 * GQA_ERR_INDEX (device-side conditions of earlier calls on this device; the
 * most severe is returned), or GQA_ERR_CUDA if the synchronisation itself
 * failed.
 */
GQA_API int gqa_get_status(gqa_stream_t stream);

/*
 * gqa_selftest_wait_timeout -- checks the failure-detection path without
 * hanging or faulting the GPU: one CTA waits, with the bounded wait every
 * kernel here uses, on a barrier that nothing arrives at; after `limit_ns`
 * nanoseconds (0 < limit_ns <= 1e10) it gives up, sets the GQA_ERR_TIMEOUT
 * status bit and returns.  `waited` (device int, may be NULL) receives 1 if
 * the wait ran out.  A following gqa_get_status returns GQA_ERR_TIMEOUT and
 * the context stays usable.  (A host-side test hook; the pages have no
 * counterpart.)
 */
GQA_API int gqa_selftest_wait_timeout(uint64_t limit_ns, int *waited, gqa_stream_t stream);

/* Reason for the last non-OK return on the calling thread ("" if none). */
GQA_API const char *gqa_last_error_string(void);

/* ABI version of this header: major * 100 + minor (1.01: optional projection workspaces). */
GQA_API int gqa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GQA_H */
