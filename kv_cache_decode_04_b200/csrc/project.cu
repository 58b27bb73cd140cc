// project.cu -- one decode token's Q/K/V projections and the KV-cache append.
//
// What is computed ("Grouped-Query Attention", llm-arch-kb, section 3
// "Reference implementation": q = h W_Q, k = h W_K, v = h W_V with W_Q
// [d, H d_h] and W_K, W_V [d, G d_h]; section 1 "Premise": the cache grows by
// one key and one value vector per token, head and layer):
//     q[b]                     = h[b] W_Q                 -> q_out [B, H, d_h]
//     k_cache[b, g, T_b, :]    = (h[b] W_K)[g*d_h : (g+1)*d_h]
//     v_cache[b, g, T_b, :]    = (h[b] W_V)[g*d_h : (g+1)*d_h]
//     seqlens_out[b]           = T_b + 1,   with T_b = seqlens[b].
// The K/V projection is G/H the size of the Q one: the "GEMM shrink" of
// section 2 ("at decode the GEMM and the cache read both shrink by H/G").
//
// This is a skinny GEMM (B rows) bound by reading the weights once.  One CTA
// owns 64 output columns of one of the three weights and streams them in
// [128 rows x 64 columns] TMA tiles (128-byte swizzle) through a 9-stage
// ring (144 KB of weights in flight per SM: at this grid size the rate is
// in-flight bytes over DRAM latency), with the matching [32 sequences x 128]
// slice of h; four
// warps split each tile's sixteen-row K-steps and run warp-level bf16 MMAs (B
// padded to 16-row blocks), then the four partial sums are added in a fixed
// order in shared memory, rounded once to bf16 and written.
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "gqa.h"
#include "internal.h"

namespace gqa {

namespace {

constexpr int kNT = 64;                    // output columns per CTA
constexpr int kKT = 128;                   // weight rows per stage
constexpr int kStagesP = 9;
constexpr int kCW = 4;                     // MMA warps
constexpr int kThreadsP = (kCW + 1) * 32;  // + 1 TMA warp
constexpr int kTileB = kKT * kNT * 2;      // 16 KB of weights per stage
constexpr int kHRows = 32;                 // sequences per launch (h box height)
constexpr int kHHalf = kHRows * 128;       // one [32 x 64] bf16 box of h, 4 KB
constexpr int kStageB = kTileB + 2 * kHHalf;

struct ProjParams {
    const __nv_bfloat16 *h;   // [B, d]
    __nv_bfloat16 *q_out;     // [B, H*d_h]
    __nv_bfloat16 *k_cache;   // [B, G, T_cap, d_h]
    __nv_bfloat16 *v_cache;
    const int32_t *seqlens;
    int32_t *seqlens_out;     // may be null
    unsigned *status;
    int B, d, H, G, d_h, T_cap;
    int b0;                   // first sequence of this launch
    int nq, nk;               // 64-column blocks of W_Q and of W_K (= of W_V); nk = 0: one weight
    int out_ld;               // row stride of q_out (H*d_h, or N for a single weight)
    unsigned long long timeout_ns;
    int warm;                 // nonzero: ask L2 for the first weight tiles before the wait
};

// [128 rows x 64 bf16] tile, 128-byte swizzle: 16-byte chunk ^= row mod 8.
__device__ __forceinline__ uint32_t swz64(int row, int col) {
    return (uint32_t)(row * 128 + ((((col >> 3) ^ (row & 7))) << 4) + ((col & 7) << 1));
}

template <int RB>  // 16-row blocks of sequences in this launch (1 or 2)
__global__ void __launch_bounds__(kThreadsP, 1)
    qkv_append_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmh,
                      const ProjParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    // After the main loop the ring is idle and holds the warps' partial sums,
    // [kCW][RB*16][kNT] floats.
    float *red = reinterpret_cast<float *>(sm);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + kStagesP * kStageB);
    uint64_t *empty = full + kStagesP;
    int *abort_flag = reinterpret_cast<int *>(empty + kStagesP);
    volatile int *vabort = abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cb = blockIdx.x;
    const int region = cb < p.nq ? 0 : (cb < p.nq + p.nk ? 1 : 2);  // Q, K, V
    const int col0 = (cb - (region == 0 ? 0 : (region == 1 ? p.nq : p.nq + p.nk))) * kNT;
    const CUtensorMap *tm = region == 0 ? &tmq : (region == 1 ? &tmk : &tmv);
    const int n_kt = p.d / kKT;

    if (tid == 0) {
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCW);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (p.warm && warp == kCW && lane == 0) {  // L2 hint: the first ring of weight tiles
        tma_prefetch_desc(tm);
        for (int kt = 0; kt < min(kStagesP, n_kt); ++kt)
            asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                             reinterpret_cast<uint64_t>(tm)), "r"(col0), "r"(kt * kKT)
                         : "memory");
    }
    pdl_wait_primary();  // h and seqlens written by the kernels before this one are visible

    if (warp == kCW) {  // ---------------- TMA producer
        if (lane == 0) {
            tma_prefetch_desc(tm);
            tma_prefetch_desc(&tmh);
            const uint64_t pol = l2_policy_evict_first();
            const uint64_t pol_h = l2_policy_evict_last();  // h is read by every CTA
            int issued = 0;
            for (int kt = 0; kt < n_kt; ++kt) {
                const int s = kt % kStagesP;
                const uint32_t ph = (kt / kStagesP) & 1;
                if (*vabort || !mbar_wait(&empty[s], ph ^ 1, p.timeout_ns)) {
                    set_status(p.status, STATUS_TIMEOUT);
                    *vabort = 1;
                    break;
                }
                uint8_t *st = sm + s * kStageB;
                mbar_arrive_expect_tx(&full[s], kStageB);
                tma_load_2d(st, tm, &full[s], col0, kt * kKT, pol);
                tma_load_2d(st + kTileB, &tmh, &full[s], kt * kKT, p.b0, pol_h);
                tma_load_2d(st + kTileB + kHHalf, &tmh, &full[s], kt * kKT + 64, p.b0, pol_h);
                issued = kt + 1;
            }
            if (*vabort)  // let copies still in flight land before the ring is reused or freed
                for (int kt = max(0, issued - kStagesP); kt < issued; ++kt)
                    mbar_wait(&full[kt % kStagesP], (kt / kStagesP) & 1, p.timeout_ns);
        }
        return;
    }

    // ---------------- MMA warps: warp w takes K-steps 2w and 2w+1 of each tile
    const int g8 = lane >> 2, q4 = lane & 3;
    float acc[RB][8][4];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) acc[rb][nt][0] = acc[rb][nt][1] = acc[rb][nt][2] = acc[rb][nt][3] = 0.f;
    bool dead = false;
    for (int kt = 0; kt < n_kt; ++kt) {
        const int s = kt % kStagesP;
        const uint32_t ph = (kt / kStagesP) & 1;
        if (!dead && (*vabort || !mbar_wait(&full[s], ph, p.timeout_ns))) {
            dead = true;
            *vabort = 1;
            set_status(p.status, STATUS_TIMEOUT);
        }
        if (!dead) {
            const uint32_t base = smem_u32(sm + s * kStageB);
            const uint32_t hbase = base + kTileB;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int ks = 2 * warp + k2;
                // A fragments of h (rows = sequences, k contiguous) from the staged slice;
                // sequences past B were zero-filled by the copy
                uint32_t a[RB][4];
                const int kc = ks * 16 + ((lane >> 4) << 3);  // k column in the 128-wide slice
#pragma unroll
                for (int rb = 0; rb < RB; ++rb) {
                    const int hr = rb * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    ldsm_x4(hbase + (kc >> 6) * kHHalf + swz64(hr, kc & 63), a[rb][0], a[rb][1], a[rb][2],
                            a[rb][3]);
                }
                const int row = ks * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(base + swz64(row, n2 * 16 + ((lane >> 4) << 3)), b0, b1, b2, b3);
#pragma unroll
                    for (int rb = 0; rb < RB; ++rb) {
                        mma_16816(acc[rb][2 * n2], a[rb], b0, b1);
                        mma_16816(acc[rb][2 * n2 + 1], a[rb], b2, b3);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---------------- fixed-order sum of the four K-slices, one rounding, write
    // (the ring is reused: wait until every MMA warp is done with its last tile)
    asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory");
    float *my = red + warp * RB * 16 * kNT;
#pragma unroll
    for (int rb = 0; rb < RB; ++rb)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int c = nt * 8 + 2 * q4;
            my[(rb * 16 + g8) * kNT + c] = acc[rb][nt][0];
            my[(rb * 16 + g8) * kNT + c + 1] = acc[rb][nt][1];
            my[(rb * 16 + g8 + 8) * kNT + c] = acc[rb][nt][2];
            my[(rb * 16 + g8 + 8) * kNT + c + 1] = acc[rb][nt][3];
        }
    asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory");
    if (dead) return;
    const int per = RB * 16 * kNT;
    for (int idx = tid; idx < per; idx += kCW * 32) {
        const int row = idx / kNT, c = idx - row * kNT;
        const int b = p.b0 + row;
        if (b >= p.B) continue;
        float v = red[idx];
#pragma unroll
        for (int w = 1; w < kCW; ++w) v += red[w * per + idx];
        const __nv_bfloat16 o = __float2bfloat16_rn(v);
        const int n = col0 + c;
        if (region == 0) {
            if (!index_ok(n < p.out_ld, p.status)) continue;
            p.q_out[(size_t)b * p.out_ld + n] = o;
        } else {
            const int T = p.seqlens[b];
            if (T < 0 || T >= p.T_cap) {
                if (c == 0 && col0 == 0) set_status(p.status, STATUS_SEQLEN);  // full cache: no append
                continue;
            }
            const int g = n / p.d_h, dim = n - g * p.d_h;
            if (!index_ok(g < p.G, p.status)) continue;
            __nv_bfloat16 *cache = region == 1 ? p.k_cache : p.v_cache;
            cache[(((size_t)b * p.G + g) * p.T_cap + T) * p.d_h + dim] = o;
        }
    }
    if (cb == 0 && p.nk > 0 && p.seqlens_out)
        for (int b = p.b0 + tid; b < min(p.B, p.b0 + RB * 16); b += kCW * 32) {
            const int T = p.seqlens[b];
            p.seqlens_out[b] = (T >= 0 && T < p.T_cap) ? T + 1 : T;
        }
}

// ------------------------------------------------------------------------
// Split-K variant for projections with few column blocks.  The column-block
// kernel above gives each 64-column block of the weights one CTA, which
// leaves most SMs idle when there are only a few blocks.  Here each block's
// 128-row K tiles are also cut into ks equal row ranges: items (block cb,
// range s), item = s * nblocks + cb, taken by CTA item mod gridDim.x in
// increasing order.  The host takes ks = floor(SMs / blocks), so every item
// has a CTA of its own in one wave, and uses this kernel only when ks >= 4
// (split_plan and proj_kernel below).  Items of the same
// range start together on different CTAs, so the CTAs running at one time
// read the same weight rows (different column blocks): the DRAM pages a row
// spans are read by many CTAs at once, as in the column-block kernel.  (Equal
// shares of a block-major line were tried first: concurrent CTAs then sat on
// different rows, and the kernel ran at half the column-block kernel's rate.)
// With ks = 1 an item is a whole block, rounded and stored directly;
// otherwise each item writes its fp32 partial sums to slot `item` of the
// workspace and counts itself on the block's counter, and the item that
// completes the count adds the block's ks partials in range order (the same
// order whichever finishes last: deterministic), rounds once and stores.
// Each MMA warp owns 16 of the block's 64 columns over all K steps, so a
// warp's partial needs no reduction across warps.
//
// Block counters carry the call's tag in their high 32 bits: a counter whose
// tag is not this call's is taken as 0 (fresh memory, an interrupted call),
// and the item that completes a block puts its counter back to 0, so the
// next call, or the next replay of a captured graph, starts from zero.
struct SplitWs {
    unsigned long long *ctr;  // [nblocks]
    float *part;              // [ks * nblocks][32 rows][64 columns]
    unsigned long long tag;   // nonzero, < 2^32
    int ks;                   // row ranges per block
};

__device__ __forceinline__ void store_out(const ProjParams &p, int region, int col0, int b, int c, float v) {
    const __nv_bfloat16 o = __float2bfloat16_rn(v);
    const int n = col0 + c;
    if (region == 0) {
        if (!index_ok(n < p.out_ld, p.status)) return;
        p.q_out[(size_t)b * p.out_ld + n] = o;
    } else {
        const int T = p.seqlens[b];
        if (T < 0 || T >= p.T_cap) {
            if (c == 0 && col0 == 0) set_status(p.status, STATUS_SEQLEN);  // full cache: no append
            return;
        }
        const int g = n / p.d_h, dim = n - g * p.d_h;
        if (!index_ok(g < p.G, p.status)) return;
        __nv_bfloat16 *cache = region == 1 ? p.k_cache : p.v_cache;
        cache[(((size_t)b * p.G + g) * p.T_cap + T) * p.d_h + dim] = o;
    }
}

constexpr int kStagesS = 9;

template <int RB>
__global__ void __launch_bounds__(kThreadsP, 1)
    proj_split_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmh,
                      const ProjParams p, const SplitWs ws) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + kStagesS * kStageB);
    uint64_t *empty = full + kStagesS;
    int *abort_flag = reinterpret_cast<int *>(empty + kStagesS);
    int *last_flag = abort_flag + 1;
    volatile int *vabort = abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int KT = p.d / kKT;
    const int NB = p.nq + 2 * p.nk;
    const int n_items = NB * ws.ks;
    auto region_of = [&](int cb) { return cb < p.nq ? 0 : (cb < p.nq + p.nk ? 1 : 2); };
    auto col0_of = [&](int cb) {
        const int r = region_of(cb);
        return (cb - (r == 0 ? 0 : (r == 1 ? p.nq : p.nq + p.nk))) * kNT;
    };
    // K tiles [kt_lo(r), kt_lo(r + 1)) of row range r
    auto kt_lo = [&](int r) { return (int)((long long)r * KT / ws.ks); };

    if (tid == 0) {
        for (int s = 0; s < kStagesS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCW);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait_primary();  // h, seqlens and the workspace of the call before are settled

    if (warp == kCW) {  // ---------------- TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmq);
            tma_prefetch_desc(&tmh);
            if (p.nk > 0) {
                tma_prefetch_desc(&tmk);
                tma_prefetch_desc(&tmv);
            }
            const uint64_t pol = l2_policy_evict_first();
            const uint64_t pol_h = l2_policy_evict_last();  // h is read by every CTA
            int issued = 0, it = 0;
            for (int item = blockIdx.x; item < n_items && !*vabort; item += gridDim.x) {
                const int cb = item % NB, rg = item / NB;
                const int region = region_of(cb), col0 = col0_of(cb);
                const CUtensorMap *tm = region == 0 ? &tmq : (region == 1 ? &tmk : &tmv);
                for (int kt = kt_lo(rg); kt < kt_lo(rg + 1); ++kt, ++it) {
                    const int s = it % kStagesS;
                    const uint32_t ph = (it / kStagesS) & 1;
                    if (*vabort || !mbar_wait(&empty[s], ph ^ 1, p.timeout_ns)) {
                        set_status(p.status, STATUS_TIMEOUT);
                        *vabort = 1;
                        break;
                    }
                    uint8_t *st = sm + s * kStageB;
                    mbar_arrive_expect_tx(&full[s], kStageB);
                    tma_load_2d(st, tm, &full[s], col0, kt * kKT, pol);
                    tma_load_2d(st + kTileB, &tmh, &full[s], kt * kKT, p.b0, pol_h);
                    tma_load_2d(st + kTileB + kHHalf, &tmh, &full[s], kt * kKT + 64, p.b0, pol_h);
                    issued = it + 1;
                }
            }
            if (*vabort)  // let copies still in flight land before the CTA exits
                for (int it = max(0, issued - kStagesS); it < issued; ++it)
                    mbar_wait(&full[it % kStagesS], (it / kStagesS) & 1, p.timeout_ns);
        }
        return;
    }

    // ---------------- MMA warps: warp w owns columns [16w, 16w + 16) of every block
    const int g8 = lane >> 2, q4 = lane & 3;
    float acc[RB][2][4];
    auto zero_acc = [&]() {
#pragma unroll
        for (int rb = 0; rb < RB; ++rb)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) acc[rb][nt][0] = acc[rb][nt][1] = acc[rb][nt][2] = acc[rb][nt][3] = 0.f;
    };
    zero_acc();
    bool dead = false;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const int cb = item % NB, rg = item / NB;
      for (int kt = kt_lo(rg); kt < kt_lo(rg + 1); ++kt, ++it) {
        const int s = it % kStagesS;
        const uint32_t ph = (it / kStagesS) & 1;
        if (!dead && (*vabort || !mbar_wait(&full[s], ph, p.timeout_ns))) {
            dead = true;
            *vabort = 1;
            set_status(p.status, STATUS_TIMEOUT);
        }
        if (!dead) {
            const uint32_t base = smem_u32(sm + s * kStageB);
            const uint32_t hbase = base + kTileB;
#pragma unroll
            for (int ks = 0; ks < kKT / 16; ++ks) {
                uint32_t a[RB][4];
                const int kc = ks * 16 + ((lane >> 4) << 3);
#pragma unroll
                for (int rb = 0; rb < RB; ++rb) {
                    const int hr = rb * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    ldsm_x4(hbase + (kc >> 6) * kHHalf + swz64(hr, kc & 63), a[rb][0], a[rb][1], a[rb][2],
                            a[rb][3]);
                }
                const int row = ks * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(base + swz64(row, warp * 16 + ((lane >> 4) << 3)), b0, b1, b2, b3);
#pragma unroll
                for (int rb = 0; rb < RB; ++rb) {
                    mma_16816(acc[rb][0], a[rb], b0, b1);
                    mma_16816(acc[rb][1], a[rb], b2, b3);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
        // ---------------- item done: rows [kt_lo(rg), kt_lo(rg + 1)) of block cb
        const int region = region_of(cb), col0 = col0_of(cb);
        if (ws.ks == 1) {  // the whole block: round and store
            if (!dead)
#pragma unroll
                for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int r = rb * 16 + g8 + (e >> 1) * 8, b = p.b0 + r;
                            if (b < p.B) store_out(p, region, col0, b, warp * 16 + nt * 8 + 2 * q4 + (e & 1), acc[rb][nt][e]);
                        }
        } else {
            // partial sums to this item's slot, then count the item on the block
            float *mine = ws.part + (long long)item * (32 * kNT);
            if (!dead)
#pragma unroll
                for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int c = warp * 16 + nt * 8 + 2 * q4;
                        *reinterpret_cast<float2 *>(mine + (rb * 16 + g8) * kNT + c) =
                            make_float2(acc[rb][nt][0], acc[rb][nt][1]);
                        *reinterpret_cast<float2 *>(mine + (rb * 16 + g8 + 8) * kNT + c) =
                            make_float2(acc[rb][nt][2], acc[rb][nt][3]);
                    }
            __threadfence();
            asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory");
            if (tid == 0) {
                int last = 0;
                if (!*vabort) {
                    unsigned long long *ctr = ws.ctr + cb;
                    unsigned long long v = *reinterpret_cast<volatile unsigned long long *>(ctr);
                    for (int tries = 0; tries < 256; ++tries) {  // ks items per block contend
                        const unsigned long long nv = (v >> 32) == ws.tag ? v + 1 : ((ws.tag << 32) | 1ull);
                        const unsigned long long old = atomicCAS(ctr, v, nv);
                        if (old == v) {
                            last = (nv & 0xffffffffull) == (unsigned long long)ws.ks;
                            break;
                        }
                        v = old;
                    }
                    if (last) {
                        __threadfence();
                        *ctr = 0ull;  // ready for the next call
                    }
                }
                *last_flag = last;
            }
            asm volatile("bar.sync 1, %0;" ::"r"(kCW * 32) : "memory");
            if (*last_flag && !dead) {
                // the block's ks partials, in range order, one rounding
                __threadfence();
#pragma unroll
                for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int r = rb * 16 + g8 + hf * 8, c = warp * 16 + nt * 8 + 2 * q4;
                            float2 sum = make_float2(0.f, 0.f);
                            for (int r2 = 0; r2 < ws.ks; ++r2) {
                                const float2 t = __ldcg(reinterpret_cast<const float2 *>(
                                    ws.part + ((long long)r2 * NB + cb) * (32 * kNT) + r * kNT + c));
                                sum.x += t.x;
                                sum.y += t.y;
                            }
                            const int b = p.b0 + r;
                            if (b < p.B) {
                                store_out(p, region, col0, b, c, sum.x);
                                store_out(p, region, col0, b, c + 1, sum.y);
                            }
                        }
            }
        }
        zero_acc();
    }

    if (blockIdx.x == 0 && p.nk > 0 && p.seqlens_out)
        for (int b = p.b0 + tid; b < min(p.B, p.b0 + RB * 16); b += kCW * 32) {
            const int T = p.seqlens[b];
            p.seqlens_out[b] = (T >= 0 && T < p.T_cap) ? T + 1 : T;
        }
}

template <int RB>
struct ProjTag {};

template <int RB>
cudaError_t run_proj(const ProjParams &p, const CUtensorMap *tq, const CUtensorMap *tk, const CUtensorMap *tv,
                     const CUtensorMap *th, cudaStream_t st) {
    const size_t smem = 1024 + (size_t)kStagesP * kStageB + 2 * kStagesP * 8 + 16;
    static_assert((size_t)kCW * 2 * 16 * kNT * 4 <= (size_t)kStagesP * kStageB, "partials fit in the ring");
    cudaError_t e = once_per_device<ProjTag<RB>>([&] {
        return cudaFuncSetAttribute(qkv_append_kernel<RB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.nq + 2 * p.nk));
    cfg.blockDim = dim3(kThreadsP);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];  // programmatic dependent: the prologue may overlap the previous kernel
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, qkv_append_kernel<RB>, *tq, *tk, *tv, *th, p);
}

template <int RB>
struct SplitTag {};

// Row ranges per block (ks) and CTAs of the split-K grid.  Weight tiles are
// 128-byte column segments of 128 rows; they stream at full rate only while
// the CTAs on neighbouring column blocks move down the rows together, as the
// column-block kernel's do.  So every item must run in the one wave:
// ks = floor(SMs / blocks).  The split pays only when it spreads the weights
// over several times the SMs the column-block kernel would use: graph-timed
// with the weights cycled past L2, a 64-block W_O took 12.7 us split in two
// (128 CTAs) against 10.1 us in column blocks, and the 96-block Q/K/V
// projection 12.1 us against 11.7 us.  Hence kMinSplit.
constexpr int kMinSplit = 4;
struct SplitPlan {
    int ks, ctas;
};
SplitPlan split_plan(int nblocks, int d, int num_sms) {
    const int KT = d / kKT;
    int ks = nblocks > 0 ? num_sms / nblocks : 1;
    // GQA_PROJ_KS=k forces k row ranges (tests of the split paths, measurements)
    const char *force = getenv("GQA_PROJ_KS");
    if (force && atoi(force) > 0) ks = atoi(force);
    if (ks > KT) ks = KT;
    if (ks < 1) ks = 1;
    return {ks, nblocks * ks};
}

template <int RB>
cudaError_t run_split(const ProjParams &p, const SplitWs &ws, int ctas, const CUtensorMap *tq, const CUtensorMap *tk,
                      const CUtensorMap *tv, const CUtensorMap *th, cudaStream_t st) {
    const size_t smem = 1024 + (size_t)kStagesS * kStageB + 2 * kStagesS * 8 + 16;
    cudaError_t e = once_per_device<SplitTag<RB>>([&] {
        return cudaFuncSetAttribute(proj_split_kernel<RB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(kThreadsP);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];  // programmatic dependent: the prologue may overlap the previous kernel
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, proj_split_kernel<RB>, *tq, *tk, *tv, *th, p, ws);
}

// Which kernel a projection takes: the column-block kernel, or with a
// workspace and at most a quarter as many column blocks as SMs the split-K
// kernel (split_plan).  GQA_PROJ_KERNEL=column|split forces one (tests of
// both paths, A/Bs).
enum class ProjKernel { Column, Split };
ProjKernel proj_kernel(int nblocks, int d, int num_sms, bool have_ws) {
    const char *force = getenv("GQA_PROJ_KERNEL");
    if (force && !strcmp(force, "column")) return ProjKernel::Column;
    if (force && !strcmp(force, "split")) return have_ws ? ProjKernel::Split : ProjKernel::Column;
    return have_ws && split_plan(nblocks, d, num_sms).ks >= kMinSplit ? ProjKernel::Split : ProjKernel::Column;
}

// Launches one grid per 32 sequences.
cudaError_t launch_proj(ProjParams p, void *workspace, int num_sms, unsigned long long tag, const CUtensorMap *tq,
                        const CUtensorMap *tk, const CUtensorMap *tv, const CUtensorMap *th, cudaStream_t st) {
    const int nblocks = p.nq + 2 * p.nk;
    const ProjKernel kind = proj_kernel(nblocks, p.d, num_sms, workspace != nullptr);
    if (kind == ProjKernel::Column) workspace = nullptr;
    SplitWs ws = {};
    int ctas = 0;
    if (workspace) {
        const SplitPlan plan = split_plan(nblocks, p.d, num_sms);
        ctas = plan.ctas;
        uint8_t *w = static_cast<uint8_t *>(workspace);
        ws.ctr = reinterpret_cast<unsigned long long *>(w);
        ws.part = reinterpret_cast<float *>(w + (((size_t)nblocks * 8 + 255) & ~size_t(255)));
        ws.tag = tag;
        ws.ks = plan.ks;
    }
    for (int b0 = 0; b0 < p.B; b0 += 32) {  // 32 sequences per launch
        p.b0 = b0;
        const bool two = p.B - b0 > 16;
        cudaError_t e;
        if (workspace)
            e = two ? run_split<2>(p, ws, ctas, tq, tk, tv, th, st) : run_split<1>(p, ws, ctas, tq, tk, tv, th, st);
        else
            e = two ? run_proj<2>(p, tq, tk, tv, th, st) : run_proj<1>(p, tq, tk, tv, th, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

size_t proj_workspace_bytes(int ncols, int d, int num_sms) {
    if (ncols <= 0 || d <= 0 || ncols % kNT != 0 || d % kKT != 0) return 0;
    const int nblocks = ncols / kNT;
    const SplitPlan plan = split_plan(nblocks, d, num_sms);
    return (((size_t)nblocks * 8 + 255) & ~size_t(255)) + (size_t)plan.ks * nblocks * 32 * kNT * sizeof(float);
}

cudaError_t launch_qkv_append(const QkvArgs &a, const CUtensorMap *tq, const CUtensorMap *tk,
                              const CUtensorMap *tv, const CUtensorMap *th, cudaStream_t st) {
    ProjParams p = {};
    p.h = static_cast<const __nv_bfloat16 *>(a.h);
    p.q_out = static_cast<__nv_bfloat16 *>(a.q_out);
    p.k_cache = static_cast<__nv_bfloat16 *>(a.k_cache);
    p.v_cache = static_cast<__nv_bfloat16 *>(a.v_cache);
    p.seqlens = a.seqlens;
    p.seqlens_out = a.seqlens_out;
    p.status = a.status;
    p.B = a.B;
    p.d = a.d;
    p.H = a.H;
    p.G = a.G;
    p.d_h = a.d_h;
    p.T_cap = a.T_cap;
    p.nq = a.H * a.d_h / kNT;
    p.nk = a.G * a.d_h / kNT;
    p.out_ld = a.H * a.d_h;
    p.timeout_ns = a.timeout_ns;
    p.warm = a.warm;
    return launch_proj(p, a.workspace, a.num_sms, a.tag, tq, tk, tv, th, st);
}

// out[B, N] = x[B, K] W[K, N]: the same kernels with one weight and no cache.
cudaError_t launch_out_project(const void *x, void *out, int B, int K, int N, unsigned *status,
                               uint64_t timeout_ns, void *workspace, int num_sms, unsigned long long tag,
                               const CUtensorMap *tw, const CUtensorMap *tx, cudaStream_t st) {
    ProjParams p = {};
    p.h = static_cast<const __nv_bfloat16 *>(x);
    p.q_out = static_cast<__nv_bfloat16 *>(out);
    p.status = status;
    p.B = B;
    p.d = K;
    p.nq = N / kNT;
    p.nk = 0;
    p.out_ld = N;
    p.timeout_ns = timeout_ns;
    return launch_proj(p, workspace, num_sms, tag, tw, tw, tw, tx, st);
}

}  // namespace gqa
