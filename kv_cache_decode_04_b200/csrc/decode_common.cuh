// decode_common.cuh -- the split-KV partition shared by the decode kernels.
//
// The cache tiles of all (b, g) segments ("Grouped-Query Attention",
// llm-arch-kb, section 1: G key/value heads per sequence) are laid end to end
// and cut into gridDim.x equal shares.  CTA c takes share c; a share may cover
// the tail of one segment and the head of the next.  For each piece (the part
// of one segment inside one share) the CTA emits one partial record (running
// max m in log2 units, sum l, unnormalised o[d_h]) per query head at record
// index c + segment: distinct for all pieces, since two pieces with equal
// c + segment would need an earlier CTA to hold a later segment.  Each record
// and the tile prefix carry a completion flag, so the combine can start on a
// segment as soon as its records exist.
#pragma once

#include "common.cuh"

namespace gqa {
namespace dec {

constexpr int kTile = 64;                // tokens per K/V tile, bf16 kernels
constexpr int kHalfBytes = kTile * 128;  // one [64 tokens x 64 dims] bf16 box
constexpr int kSplitPMaxLen = 256;       // sequences this short carry P as two bf16 terms

struct DecodeParams {
    const void *q;
    const int32_t *seqlens;
    void *out;
    int *ws_cu;     // [B+1] tile prefix, written by CTA 0 of the split kernel
    float2 *ws_ml;  // [n_rec * r]: (max in log2 units, sum)
    float *ws_o;    // [n_rec * r * d_h]: unnormalised outputs
    long long n_rec;  // records the workspace holds (the debug build's index checks)
    // Cache bases, typed for the fp32 path; the bf16 kernels use them only for
    // L2 prefetch hints (their loads go through tensor maps).
    const float *k32, *v32;
    unsigned *status;
    float scale_log2;
    int B, H, G, r, T_cap;
    unsigned long long timeout_ns;
    int window;  // > 0: attend over the last `window` cached positions only
    int warm;    // nonzero: warm L2 with the first tiles before griddepcontrol.wait
    // Completion flags, [1 + records]: flag 0 = the tile prefix ws_cu, flag 1 + i
    // = record i.  A flag holds the generation of the call that completed it.
    unsigned long long *ws_flag;
    // Workspace header (first 256 bytes): the generation of the last call that
    // completed on this workspace and a check word, and the combine's count of
    // finished CTAs.  See call_generation().
    unsigned long long *ws_hdr;
    // Generation to start from when the header is not valid (fresh memory):
    // random per host call.
    unsigned long long seed;
};

// Header words.
enum { HDR_EPOCH = 0, HDR_CHECK = 1, HDR_DONE = 2 };
constexpr unsigned long long kHdrMagic = 0x6a09e667f3bcc909ull;

// This call's generation, the value its completion flags carry.  Derived on
// the device, so a call replayed from a CUDA graph (whose kernel arguments are
// frozen) still gets a new one every time:
//   - the combine's last CTA of every call stores that call's generation in
//     the header with a check word; the next call on the workspace uses it + 1,
//     so every flag an earlier call left behind holds a smaller value;
//   - a header that fails the check (memory never used by a decode call, or
//     invalidated after a timed-out wait) gives the host's random seed.
// The split kernel reads the header after griddepcontrol.wait, when the last
// call's combine has completed; the combine reads it before any of its CTAs
// can advance it (the advance waits for all of them).  Every thread of a
// kernel computes the same value.
__device__ __forceinline__ unsigned long long call_generation(const DecodeParams &p) {
    const volatile unsigned long long *h = p.ws_hdr;
    const unsigned long long e = h[HDR_EPOCH], c = h[HDR_CHECK];
    return c == (e ^ kHdrMagic) ? e + 1 : p.seed;
}

// Publishes a completion flag with release semantics at GPU scope.  Every
// thread that wrote part of the flagged data has executed __threadfence()
// and a barrier shared with the publishing thread before this call.
__device__ __forceinline__ void publish_flag(unsigned long long *flag, unsigned long long gen) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(flag), "l"(gen) : "memory");
}

// Waits, for at most limit_ns, until *flag == gen (acquire at GPU scope, so
// this thread's later loads see the flagged data).  False on time-out.
__device__ __forceinline__ bool wait_flag(const unsigned long long *flag, unsigned long long gen,
                                          unsigned long long limit_ns) {
    auto load = [&]() {
        unsigned long long v;
        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(flag) : "memory");
        return v;
    };
    if (load() == gen) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        for (int i = 0; i < 32; ++i) {
            __nanosleep(64);
            if (load() == gen) return true;
        }
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}

// CTA 0 of a split kernel: writes the tile prefix for the combine, zeroes the
// combine's finished-CTA count, and publishes both with the prefix flag (every
// combine CTA waits for that flag before it counts itself).  Every thread of
// the block calls it.
__device__ __forceinline__ void publish_prefix(const DecodeParams &p, const int *cu, unsigned long long gen) {
    if (blockIdx.x != 0) return;
    for (int i = threadIdx.x; i <= p.B; i += blockDim.x) p.ws_cu[i] = cu[i];
    if (threadIdx.x == 0) p.ws_hdr[HDR_DONE] = 0ull;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) publish_flag(&p.ws_flag[0], gen);
}

__device__ __forceinline__ int clamp_len(int T, int T_cap) {
    return T < 0 ? 0 : (T > T_cap ? T_cap : T);
}

// Cached positions a sequence attends over: all T_b of them, or with a sliding
// window of W > 0 only the last min(T_b, W), i.e. [T_b - len, T_b).
__device__ __forceinline__ int attended_len(int T, const DecodeParams &p) {
    const int t = clamp_len(T, p.T_cap);
    return (p.window > 0 && t > p.window) ? p.window : t;
}

// cu[b] = G * sum_{b' < b} ceil(len_b' / TILE), len as attended_len;
// cu[B] = total tiles.  Every thread of the block must call it; blockDim.x
// is a multiple of 32 and scratch holds 32 ints.  When tb is given it
// receives T_b clamped to [0, T_cap] for every b.
template <int TILE>
__device__ int build_tile_prefix(const DecodeParams &p, int *cu, int *scratch, bool report, int *tb = nullptr) {
    const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int chunk = (p.B + nt - 1) / nt;
    const int b0 = min(p.B, tid * chunk), b1 = min(p.B, b0 + chunk);
    int local = 0;
    bool bad = false;
    for (int b = b0; b < b1; ++b) {
        const int T = p.seqlens[b];
        bad |= (T < 0 || T > p.T_cap);
        local += (attended_len(T, p) + TILE - 1) / TILE;
        if (tb) tb[b] = clamp_len(T, p.T_cap);
    }
    if (bad && report) set_status(p.status, STATUS_SEQLEN);
    // exclusive block scan of `local`: warp scans, then a scan of the warp totals
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) scratch[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        const int nw = nt >> 5;
        int w = lane < nw ? scratch[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += v;
        }
        if (lane < nw) scratch[lane] = w;  // inclusive prefix of warp totals
        if (lane == nw - 1) cu[p.B] = w * p.G;
    }
    __syncthreads();
    int run = incl - local + (wid > 0 ? scratch[wid - 1] : 0);
    for (int b = b0; b < b1; ++b) {
        cu[b] = run * p.G;
        run += (attended_len(p.seqlens[b], p) + TILE - 1) / TILE;
    }
    __syncthreads();
    return cu[p.B];
}

// L2 warm-up for a split kernel's first tiles, issued by one warp before
// griddepcontrol.wait, so that the cache reads start while the kernel before
// this one ends.  seqlens may be an output of that kernel and is read here
// only to guess this CTA's share (B <= 32: one warp scans it); a stale guess
// costs bandwidth, never correctness, since the loads proper come after the
// wait.  Prefetches up to `ntiles` tiles of TILE positions (row_bytes each)
// from the start of the share, within the sequence the share starts in.
template <int TILE>
__device__ __forceinline__ void warm_first_tiles(const DecodeParams &p, int lane, int ntiles, int row_bytes) {
    if (!p.warm || p.B > 32) return;
    int T = 0, n = 0;
    if (lane < p.B) {
        // cached at L2 only (ld.global.cg): no L1 line of a value that may be
        // about to change outlives the wait
        T = clamp_len(__ldcg(p.seqlens + lane), p.T_cap);
        n = p.G * ((attended_len(T, p) + TILE - 1) / TILE);
    }
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    const int u0 = (int)((long long)blockIdx.x * total / gridDim.x);
    const int u1 = (int)((long long)(blockIdx.x + 1) * total / gridDim.x);
    const int excl = incl - n;
    if (lane >= p.B || u0 >= u1 || u0 < excl || u0 >= incl) return;  // not the lane holding u0
    const int len = attended_len(T, p), start = T - len, nt = (len + TILE - 1) / TILE;
    const uint8_t *kb = reinterpret_cast<const uint8_t *>(p.k32);
    const uint8_t *vb = reinterpret_cast<const uint8_t *>(p.v32);
    int idx = u0 - excl;  // tile of this sequence's G segments, g-major
    for (int k = 0; k < ntiles && u0 + k < u1 && idx < p.G * nt; ++k, ++idx) {
        const int g = idx / nt, j = idx - g * nt;
        const int ntok = min(TILE, len - j * TILE);
        const size_t row = ((size_t)lane * p.G + g) * p.T_cap + start + (size_t)j * TILE;
        prefetch_l2(kb + row * row_bytes, (uint32_t)(ntok * row_bytes));
        prefetch_l2(vb + row * row_bytes, (uint32_t)(ntok * row_bytes));
    }
}

// Position in the tile line: sequence b, KV head g, tile j of the segment,
// tiles per segment of b.
struct Cursor {
    int b, g, j, ntb;
};

__device__ __forceinline__ void cursor_seek(const int *cu, int B, int G, int u, Cursor &c) {
    int lo = 0, hi = B - 1;  // largest b with cu[b] <= u (then cu[b] <= u < cu[b+1])
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= u) lo = mid; else hi = mid - 1;
    }
    c.b = lo;
    c.ntb = (cu[lo + 1] - cu[lo]) / G;
    const int off = u - cu[lo];
    c.g = off / c.ntb;
    c.j = off - c.g * c.ntb;
}

__device__ __forceinline__ void cursor_next(const int *cu, int B, int G, Cursor &c) {
    if (++c.j < c.ntb) return;
    c.j = 0;
    if (++c.g < G) return;
    c.g = 0;
    do {
        ++c.b;
    } while (c.b < B && cu[c.b + 1] == cu[c.b]);
    if (c.b < B) c.ntb = (cu[c.b + 1] - cu[c.b]) / G;
}

// Launches a split kernel as a programmatic dependent of the work before it in
// the stream: its prologue (barrier set-up, TMEM allocation, tensor-map
// prefetch) may overlap the tail of that work; the kernel calls
// griddepcontrol.wait before it reads any input.
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ------------------------------------------------- tensor-core split kernel

// Groups of at least this many query heads use the tcgen05 split kernel.
constexpr int kTcMinHeads = 16;

bool tc_eligible(int r, int d_h, int B);
size_t tc_smem_bytes(int d_h, int B);
// Launches the tcgen05 split kernel on `ctas` CTAs (one per SM).
cudaError_t run_split_tc(const DecodeParams &p, const CUtensorMap *tmk, const CUtensorMap *tmv, int d_h, int ctas,
                         cudaStream_t st);

}  // namespace dec
}  // namespace gqa
