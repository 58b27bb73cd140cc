// decode_tc.cu -- GQA decode split kernel on the 5th-generation tensor cores
// (sm_100a), for groups of many query heads (16 <= H/G <= 64).
//
// What is computed ("Grouped-Query Attention", llm-arch-kb, sections 1-3): for
// sequence b and query head i of group g = i / (H/G),
//     out[b,i] = sum_{t < T_b} softmax_t(scale * q[b,i] . K[b,g,t]) V[b,g,t].
// With H/G heads sharing one K/V head, every cached K/V element takes part in
// 2 * H/G multiply-adds (scores and P.V).  For H/G = 32 at ~6.5 TB/s that is
// ~210 TFLOP/s of dense contraction, more than warp-level MMAs sustain next to
// the softmax, so here both products run on tcgen05.
//
// Tensor-core cost: a tcgen05.mma with M = 128 and K = 16 takes 56 SM cycles
// at N = 64 and 64 at N = 128 when one thread streams them (measured on B200),
// so below N = 128 the instruction count matters as much as the flops.
// Tiles are 128 positions: S = Q K^T is 8 instructions of N = 128 and P.V 8
// of N = d_h per tile, about a third of the HBM time of the tile's 64 KB.
//
// Rows of the M = 128 tile: the group's H/G query rows, replicated NREP times
// (4 copies of 32 rows for H/G <= 32, 2 copies of 64 rows above).  Copy k is
// read by the softmax warps that own its TMEM lanes, and those warps handle
// only token slice k of every tile (32 or 64 positions): their P rows are zero
// outside the slice, so the P.V of copy k accumulates the slice's share of the
// output.  The copies cost no tensor time (the instruction is M = 128 either
// way) and spread the softmax over all four SM sub-partitions.  Each slice
// keeps its own online softmax; at the end of a piece the slices' partial
// results are merged in shared memory into the piece's one record, which
// decode_combine merges with the other pieces' records.
//
// Partition and records follow decode_common.cuh, with 128-position tiles.
//
// One CTA per SM, 224 threads:
//   warps 0-3  softmax + records: warp w owns TMEM lanes 32w..32w+31, i.e.
//              rows of copy k = w / NSW, heads 32 (w % NSW) + lane.  They also
//              write the q rows of each piece into TMEM, one piece ahead.
//   warp 4     TMA producer: [128 positions x d_h] K and V tiles through a
//              3-stage ring (6 for d_h = 64; 128-byte swizzle).
//   warp 5     allocates 512 TMEM columns; one lane issues S = Q K^T
//              (M = 128, N = 128, Q from TMEM, fp32 S in TMEM, two buffers).
//   warp 6     one lane issues O += P V (P bf16 read back from TMEM, fp32 O).
// With separate issuing threads a tile's scores go out as soon as its K has
// landed, whatever the P.V of the tile before is waiting for, so the softmax
// of one tile overlaps the tensor core's work on its neighbours.
// TMEM columns: [128i, 128i+128) S/P buffer i (i < 2), [256, 256+d_h) O,
// [384 + (d_h/2) j, ...) Q buffer j (j < 2).  P_hi (bf16 pairs) overwrites
// the first 64 columns of its S buffer; sequences of at most 256 positions
// also carry P_lo in the next 64 (P = P_hi + P_lo).
// Online softmax in the base-2 domain; a slice's running max moves (and its O
// rows are rescaled in TMEM) only when it grows by more than 8, so p <= 2^8,
// with the same stale maximum in numerator and denominator.
#include "common.cuh"
#include "decode_common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace gqa {
namespace dec {

namespace {

constexpr int kTcThreads = 224;
constexpr int kTT = 128;                     // tokens per tile of this kernel's partition
constexpr int kBox = kTT * 128;              // [128 tokens x 64 dims] bf16: two stacked 64-row TMA boxes
constexpr int kNS = 2;                       // S/P buffers in TMEM (kTT columns each)
constexpr uint32_t kOCol = kNS * kTT;        // first TMEM column of O (d_h columns)
constexpr uint32_t kQCol = kOCol + 128;      // two Q buffers of d_h / 2 columns (bf16 pairs)
constexpr uint32_t kTcTmemCols = 512;
constexpr int kMaxRows = 64;         // query heads per group this kernel takes

// Shared memory: the K/V ring, barriers, the record transpose and the tile prefix.
template <int D>
struct TcLayout {
    static constexpr int HALVES = D / 64;
    static constexpr int STAGES = D == 128 ? 3 : 6;
    static constexpr int KV_BYTES = kTT * D * 2;
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int OFF_RING = 0;
    static constexpr int OFF_BAR = OFF_RING + STAGES * STAGE_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int OFF_XP = OFF_BAR + BAR_BYTES;    // record merge, [4 warps][32][33] floats
    static constexpr int XP_BYTES = 4 * 32 * 33 * 4;
    static constexpr int OFF_ML = OFF_XP + XP_BYTES;      // slices' (m, l), [4 warps][32] float2
    static constexpr int OFF_CU = OFF_ML + 4 * 32 * 8;    // cu[B+1], scratch[32], tb[B]
};

template <int D>
size_t smem_tc(int B) {
    return 1024 + (size_t)TcLayout<D>::OFF_CU + (size_t)(B + 1) * 4 + 32 * 4 + (size_t)B * 4;
}

__device__ __forceinline__ uint64_t f32x2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Warp-uniform bounded wait: every lane polls; the warp agrees on the result.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, uint64_t limit) {
    const bool ok = mbar_wait(bar, parity, limit);
    return __all_sync(0xffffffffu, ok);
}

// N (32 or 64) consecutive 32-bit TMEM columns of this warp's lanes.
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 32 || N == 64, "x32 or 2 x32");
    tc::ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    if constexpr (N == 64) tc::ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}
__device__ __forceinline__ void st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&r)[N]) {
    static_assert(N == 16 || N == 32, "x16 or x32");
    if constexpr (N == 16) tc::st16(taddr, r); else tc::st32(taddr, r);
}

// Piece bookkeeping every role repeats over its share: the tile's segment and
// whether the tile opens or closes a piece.
struct TileInfo {
    int b, g, bg, j, seq_len, n_valid;
    int seg_end;  // tile index just past this tile's segment
    bool first, last;
};

template <int D, int NSW>
__global__ void __launch_bounds__(kTcThreads, 1)
    decode_split_tc(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const DecodeParams p) {
    using Lay = TcLayout<D>;
    constexpr int HALVES = Lay::HALVES, STAGES = Lay::STAGES;
    constexpr int NREP = 4 / NSW;      // copies of the group's rows in M = 128
    constexpr int CW = kTT / NREP;     // tokens per slice (32 or 64)
    constexpr int PCW = CW / 2;        // TMEM columns of a slice's bf16 P pairs
    constexpr int PLO = kTT / 2;       // TMEM column offset of P_lo in an S buffer
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Lay::OFF_BAR);
    uint64_t *full = bars;                   // [STAGES] K+V tile landed
    uint64_t *empty = full + STAGES;         // [STAGES] tile consumed by its P.V
    uint64_t *q_full = empty + STAGES;       // [2] q rows of a piece written to TMEM Q buffer i
    uint64_t *s_full = q_full + 2;           // [kNS] scores of the tile in S buffer i
    uint64_t *p_ready = s_full + kNS;        // [kNS] P of the tile in S buffer i
    uint64_t *pv_done = p_ready + kNS;       // [kNS] P.V of the tile in S buffer i
    uint64_t *drain = pv_done + kNS;         // [2] one per MMA-issuing thread
    uint64_t *ep_bar = drain + 2;            // the softmax warps' record merge (128 arrivals a phase)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ep_bar + 1);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    int *cu = reinterpret_cast<int *>(sm + Lay::OFF_CU);
    int *scratch = cu + p.B + 1;
    int *tb = scratch + 32;  // T_b clamped to [0, T_cap]
    volatile int *vabort = abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&q_full[s], 128);
            mbar_init(&drain[s], 1);
        }
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_ready[s], 128);
            mbar_init(&pv_done[s], 1);
        }
        mbar_init(ep_bar, 128);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 4) {
        if (lane == 0) {
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
        }
        // one ring's worth: deeper warm-ups measured no better here
        warm_first_tiles<kTT>(p, lane, STAGES, D * 2);
    }
    if (warp == 5) {
        tc::tmem_alloc(tmem_slot, kTcTmemCols);
        tc::fence_before();
    }
    pdl_wait_primary();  // inputs written by the kernels before this one are visible
    const unsigned long long gen = call_generation(p);
    const int W = build_tile_prefix<kTT>(p, cu, scratch, blockIdx.x == 0, tb);  // syncs the block
    publish_prefix(p, cu, gen);
    pdl_launch_dependents();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;

    const long long C = gridDim.x;
    const int u_begin = (int)((long long)blockIdx.x * W / C);
    const int u_end = (int)((long long)(blockIdx.x + 1) * W / C);

    // Walks the share: body(it, tile, first cache row) for every tile, in order.
    auto walk = [&](auto &&body) {
        if (u_begin >= u_end) return;
        Cursor c;
        cursor_seek(cu, p.B, p.G, u_begin, c);
        int prev_bg = -1, cached_b = -1, len_b = 0, start_b = 0;
        for (int u = u_begin, it = 0; u < u_end; ++u, ++it) {
            if (c.b != cached_b) {  // positions [start_b, start_b + len_b) of sequence b
                cached_b = c.b;
                const int Tb = tb[c.b];
                len_b = attended_len(Tb, p);
                start_b = Tb - len_b;
            }
            TileInfo t;
            t.b = c.b;
            t.g = c.g;
            t.bg = c.b * p.G + c.g;
            t.j = c.j;
            t.seq_len = len_b;
            t.n_valid = min(kTT, len_b - c.j * kTT);
            t.first = t.bg != prev_bg;
            t.seg_end = u - c.j + c.ntb;
            const int row = t.bg * p.T_cap + start_b + c.j * kTT;
            cursor_next(cu, p.B, p.G, c);
            t.last = (u + 1 == u_end) || (c.b * p.G + c.g != t.bg);
            prev_bg = t.bg;
            if (!body(it, t, row)) break;
        }
    };

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            int issued = 0;
            walk([&](int it, const TileInfo &t, int row) {
                const int s = it % STAGES;
                if (*vabort || !mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, p.timeout_ns)) {
                    set_status(p.status, STATUS_TIMEOUT);
                    *vabort = 1;
                    return false;
                }
                uint8_t *kdst = sm + Lay::OFF_RING + s * Lay::STAGE_BYTES;
                uint8_t *vdst = kdst + Lay::KV_BYTES;
                mbar_arrive_expect_tx(&full[s], Lay::STAGE_BYTES);
                // the tile starts inside its (b, g) segment of the cache (a skipped
                // tile leaves the barrier short: the bounded waits then end the CTA)
                const bool row_ok = index_ok(t.b < p.B && t.g < p.G && row - t.bg * p.T_cap >= 0 &&
                                                 row - t.bg * p.T_cap < p.T_cap,
                                             p.status);
#pragma unroll
                for (int h = 0; h < HALVES; ++h)
#pragma unroll
                    for (int r2 = 0; r2 < kTT / 64; ++r2) {
                        if (!row_ok) continue;
                        tma_load_2d(kdst + h * kBox + r2 * kHalfBytes, &tmk, &full[s], h * 64, row + r2 * 64, pol);
                        tma_load_2d(vdst + h * kBox + r2 * kHalfBytes, &tmv, &full[s], h * 64, row + r2 * 64, pol);
                    }
                issued = it + 1;
                return true;
            });
            if (*vabort) {  // let copies still in flight land before the CTA exits
                for (int it = max(0, issued - STAGES); it < issued; ++it)
                    mbar_wait(&full[it % STAGES], (it / STAGES) & 1, p.timeout_ns);
            }
        }
        __syncwarp();
    } else if (warp == 5 || warp == 6) {
        // ------------------------------------------------ MMA issuers
        // warp 5: S(it) = Q K^T once K(it) (and, opening a piece, its q rows) has
        //         landed and the P.V that last read S buffer it % kNS is complete;
        // warp 6: O (+)= P(it) V(it) once the softmax has written P(it).
        // Two issuing threads, so neither product waits behind the other's inputs.
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::idesc_bf16(128, kTT, false, false);
            constexpr uint32_t idesc_o = tc::idesc_bf16(128, D, false, true);
            const uint32_t ring = smem_u32(sm + Lay::OFF_RING);
            const bool is_s = warp == 5;
            bool ok = true, issued = false;
            auto wait = [&](uint64_t *bar, uint32_t par) {
                if (!ok || *vabort || !mbar_wait(bar, par, p.timeout_ns)) {
                    if (ok) set_status(p.status, STATUS_TIMEOUT);
                    ok = false;
                    *vabort = 1;
                }
                return ok;
            };
            int piece = -1;
            walk([&](int it, const TileInfo &t, int) {
                const int s = it % STAGES, sb = it % kNS;
                if (is_s) {
                    if (t.first) ++piece;
                    if (!wait(&full[s], (it / STAGES) & 1)) return false;
                    if (t.first && !wait(&q_full[piece & 1], (piece >> 1) & 1)) return false;
                    if (it >= kNS && !wait(&pv_done[sb], ((it / kNS) - 1) & 1)) return false;
                    tc::fence_after();
                    // S = Q K^T over d_h in K-steps of 16: Q (bf16 pairs) from TMEM Q
                    // buffer piece % 2, K from the ring's 64-wide swizzled boxes
                    const uint64_t dk = tc::sdesc_sw128(ring + s * Lay::STAGE_BYTES, 16, 1024);
                    const uint32_t tq = tmem + kQCol + (piece & 1) * (D / 2);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t ok_ = ((kk >> 2) * kBox + (kk & 3) * 32) >> 4;
                        tc::mma_ts(tmem + sb * kTT, tq + kk * 8, dk + ok_, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    tc::commit(&s_full[sb]);
                } else {
                    if (!wait(&p_ready[sb], (it / kNS) & 1)) return false;
                    tc::fence_after();
                    // O (+)= P V over the tile's 64 tokens in K-steps of 16; V is MN-major
                    // (d_h contiguous, 64-wide column blocks kBox apart).  A second pass adds P_lo.
                    const uint64_t dv =
                        tc::sdesc_sw128(ring + s * Lay::STAGE_BYTES + Lay::KV_BYTES, kBox, 1024);
                    const int passes = t.seq_len <= kSplitPMaxLen ? 2 : 1;
#pragma unroll 1
                    for (int ps = 0; ps < passes; ++ps)
#pragma unroll
                        for (int kk = 0; kk < kTT / 16; ++kk)
                            tc::mma_ts(tmem + kOCol, tmem + sb * kTT + ps * PLO + kk * 8, dv + ((kk * 2048) >> 4),
                                       idesc_o, (!t.first || ps > 0 || kk > 0) ? 1u : 0u);
                    tc::commit(&pv_done[sb]);
                    tc::commit(&empty[s]);
                }
                issued = true;
                return true;
            });
            if (issued && !ok) {  // let MMAs already issued finish before TMEM is freed
                tc::commit(&drain[is_s ? 0 : 1]);
                mbar_wait(&drain[is_s ? 0 : 1], 0, p.timeout_ns);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax + records
        const int k = warp / NSW;                   // copy = token slice [k*CW, (k+1)*CW)
        const int head = (warp % NSW) * 32 + lane;  // query head within the group
        const bool valid = head < p.r;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t tO = tmem + lane_off + kOCol;
        uint8_t *ring = sm + Lay::OFF_RING;
        const uint64_t sc2 = f32x2_pack(p.scale_log2, p.scale_log2);
        const uint32_t zero8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        // Q rows of the piece of segment (b, g) into TMEM Q buffer `buf`: this
        // thread's row is head `head` of the group (zeros past H/G), as bf16
        // pairs in d_h / 2 columns.  Then the QK issuer may use the buffer.
        auto write_q = [&](int buf, int b, int g) {
            const uint32_t tq = tmem + lane_off + kQCol + buf * (D / 2);
            const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.q) +
                                                               ((size_t)b * p.H + (size_t)g * p.r + head) * D);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t w[32];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint4 v4 = valid ? src[c * 8 + e] : make_uint4(0u, 0u, 0u, 0u);
                    w[4 * e] = v4.x;
                    w[4 * e + 1] = v4.y;
                    w[4 * e + 2] = v4.z;
                    w[4 * e + 3] = v4.w;
                }
                tc::st32(tq + c * 32, w);
            }
            tc::wait_st();
            tc::fence_before();
            mbar_arrive(&q_full[buf]);
        };
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        int piece = -1;
        uint32_t ep_phase = 0;
        // all 128 softmax threads meet (bounded: false when a wait ran out)
        auto ep_sync = [&]() {
            mbar_arrive(ep_bar);
            const bool done = warp_wait(ep_bar, ep_phase & 1, p.timeout_ns);
            ++ep_phase;
            return done;
        };
        if (u_begin < u_end) {  // the first piece's rows
            Cursor c0;
            cursor_seek(cu, p.B, p.G, u_begin, c0);
            write_q(0, c0.b, c0.g);
        }
        walk([&](int it, const TileInfo &t, int) {
            const int sb = it % kNS;
            const uint32_t tS = tmem + lane_off + sb * kTT;
            const bool aborted = __any_sync(0xffffffffu, *vabort != 0);
            if (aborted || !warp_wait(&s_full[sb], (it / kNS) & 1, p.timeout_ns)) {
                ok = false;
                return false;
            }
            tc::fence_after();
            uint32_t sr[CW];
            tmem_ld<CW>(tS + k * CW, sr);
            tc::wait_ld();
            // this slice's scores into the log2 domain; positions past the end -inf
            float x[CW];
#pragma unroll
            for (int e = 0; e < CW / 2; ++e)
                f32x2_unpack(f32x2_mul(f32x2_pack(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), sc2),
                             x[2 * e], x[2 * e + 1]);
            const int nv = t.n_valid - k * CW;  // valid positions of this slice (may be <= 0)
            const bool partial = nv < CW;
            if (partial) {
#pragma unroll
                for (int e = 0; e < CW; ++e)
                    if (e >= nv) x[e] = -INFINITY;
                if (warp % NSW == 0) {  // zero the slice's V rows past the end: 0 * (stale data) stays 0
                    uint8_t *vt = ring + (it % STAGES) * Lay::STAGE_BYTES + Lay::KV_BYTES;
                    const int r0 = k * CW + max(nv, 0);
                    const int nz = (k * CW + CW - r0) * HALVES * 8;  // 16-byte chunks
                    for (int i = lane; i < nz; i += 32) {
                        const int rr = r0 + i / (HALVES * 8), rem = i % (HALVES * 8);
                        asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(
                                         smem_u32(vt + (rem >> 3) * kBox + rr * 128 + (rem & 7) * 16)),
                                     "r"(0u)
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                }
            }
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int e = 0; e < CW; ++e) mx4[e & 3] = fmaxf(mx4[e & 3], x[e]);
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            if (t.first) {
                m = mx;  // -inf when this slice of the tile holds no position
                l = 0.f;
            } else {
                const float mn = fmaxf(m, mx);
                const bool need = valid && mn > m + 8.f;  // also when m was -inf and mn is not
                if (__any_sync(0xffffffffu, need)) {
                    // O holds the P.V of tile it-1: wait for it, then scale the rows that move
                    const int pit = it - 1;
                    if (!warp_wait(&pv_done[pit % kNS], (pit / kNS) & 1, p.timeout_ns)) {
                        ok = false;
                        return false;
                    }
                    tc::fence_after();
                    const float alpha = need ? fast_exp2(m - mn) : 1.f;
                    if (need) {
                        m = mn;
                        l *= alpha;
                    }
#pragma unroll 1
                    for (int c = 0; c < D / 16; ++c) {
                        uint32_t orow[16];
                        tc::ld16(tO + c * 16, orow);
                        tc::wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
                        tc::st16(tO + c * 16, orow);
                    }
                }
            }
            // P = 2^(x - m) as bf16 pairs in this slice's columns of the S buffer,
            // zeros in the other slices' columns (every exponential on the
            // special-function unit).  Short sequences also store P_lo = P - bf16(P).
            const bool split = t.seq_len <= kSplitPMaxLen;
            const float mu = m == -INFINITY ? 0.f : m;  // no position seen yet: p = 0
            const uint64_t nm2 = f32x2_pack(-mu, -mu);
            uint64_t rs2[2] = {0ull, 0ull};
            uint32_t ph[PCW], pl[PCW];
#pragma unroll
            for (int e = 0; e < PCW; ++e) {
                float x0, x1;
                f32x2_unpack(f32x2_add(f32x2_pack(x[2 * e], x[2 * e + 1]), nm2), x0, x1);
                const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                rs2[e & 1] = f32x2_add(rs2[e & 1], f32x2_pack(p0, p1));
                ph[e] = pack_bf16x2(p0, p1);
                const float2 hv = unpack_bf16x2(ph[e]);
                pl[e] = pack_bf16x2(p0 - hv.x, p1 - hv.y);
            }
#pragma unroll
            for (int j = 0; j < NREP; ++j) {
                if (j == k) {
                    tmem_st<PCW>(tS + j * PCW, ph);
                    if (split) tmem_st<PCW>(tS + PLO + j * PCW, pl);
                } else {
#pragma unroll
                    for (int z = 0; z < PCW / 8; ++z) {
                        st8(tS + j * PCW + z * 8, zero8);
                        if (split) st8(tS + PLO + j * PCW + z * 8, zero8);
                    }
                }
            }
            float a0, a1, b0, b1;
            f32x2_unpack(rs2[0], a0, a1);
            f32x2_unpack(rs2[1], b0, b1);
            l += (a0 + a1) + (b0 + b1);
            tc::wait_st();
            tc::fence_before();
            mbar_arrive(&p_ready[sb]);
            if (t.first) {
                // The next piece's rows go to the other Q buffer: its last reader, the
                // final S of the piece before this one, completed before this piece's
                // first S did.
                ++piece;
                if (t.seg_end < u_end) {
                    Cursor cn;
                    cursor_seek(cu, p.B, p.G, t.seg_end, cn);
                    write_q((piece + 1) & 1, cn.b, cn.g);
                }
            }
            if (t.last) {
                // Piece done: wait for its last P.V, then merge the NREP slices' partial
                // results of every head into the piece's record:
                //   M = max_k m_k, L = sum_k 2^(m_k - M) l_k, o = sum_k 2^(m_k - M) O_k.
                // The warps of one head block (same warp % NSW) exchange (m, l) and their
                // scaled O rows through shared memory, 32 columns at a time; each warp
                // then adds up every NREP-th row in slice order and writes it with
                // coalesced 128-byte stores.
                if (!warp_wait(&pv_done[sb], (it / kNS) & 1, p.timeout_ns)) {
                    ok = false;
                    return false;
                }
                tc::fence_after();
                float2 *mlx = reinterpret_cast<float2 *>(sm + Lay::OFF_ML);
                float *xp = reinterpret_cast<float *>(sm + Lay::OFF_XP);
                const int hb = warp % NSW;
                mlx[warp * 32 + lane] = make_float2(m, l);
                if (!ep_sync()) {
                    ok = false;
                    return false;
                }
                float M = -INFINITY;
#pragma unroll
                for (int kk = 0; kk < NREP; ++kk) M = fmaxf(M, mlx[(kk * NSW + hb) * 32 + lane].x);
                float L = 0.f;
#pragma unroll
                for (int kk = 0; kk < NREP; ++kk) {
                    const float2 v = mlx[(kk * NSW + hb) * 32 + lane];
                    L += v.x == -INFINITY ? 0.f : fast_exp2(v.x - M) * v.y;
                }
                const float wgt = m == -INFINITY ? 0.f : fast_exp2(m - M);
                const long long rec = (long long)blockIdx.x + t.bg;
                float *dst0 = p.ws_o + (rec * p.r + hb * 32) * D;
                // the debug build's check: a record past the workspace is not written
                const int nrows = index_ok(rec < p.n_rec, p.status) ? min(32, p.r - hb * 32) : 0;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t orow[32];
                    tc::ld32(tO + c * 32, orow);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) xp[(warp * 32 + lane) * 33 + e] = __uint_as_float(orow[e]) * wgt;
                    if (!ep_sync()) {
                        ok = false;
                        return false;
                    }
                    for (int i = k; i < nrows; i += NREP) {
                        float acc = 0.f;
#pragma unroll
                        for (int kk = 0; kk < NREP; ++kk) acc += xp[((kk * NSW + hb) * 32 + i) * 33 + lane];
                        dst0[(size_t)i * D + c * 32 + lane] = acc;
                    }
                    if (c == D / 32 - 1) {  // last chunk: the (M, L) pairs too, then make all visible
                        if (k == 0 && valid && nrows > 0) p.ws_ml[rec * p.r + head] = make_float2(M, L);
                        __threadfence();
                    }
                    if (!ep_sync()) {
                        ok = false;
                        return false;
                    }
                }
                if (warp == 0 && lane == 0 && rec < p.n_rec) publish_flag(&p.ws_flag[1 + rec], gen);
            }
            return true;
        });
        if (!ok && lane == 0) {
            set_status(p.status, STATUS_TIMEOUT);
            *vabort = 1;
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 5) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, kTcTmemCols);
    }
}

template <int D, int NSW>
struct TcTag {};

template <int D, int NSW>
cudaError_t run(const DecodeParams &p, const CUtensorMap *tmk, const CUtensorMap *tmv, int ctas, cudaStream_t st) {
    const size_t smem = smem_tc<D>(p.B);
    auto kern = decode_split_tc<D, NSW>;
    // the attribute persists per device; set it (to the maximum) on first use
    cudaError_t e = once_per_device<TcTag<D, NSW>>(
        [&] { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024); });
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(ctas), dim3(kTcThreads), smem, st, *tmk, *tmv, p);
}

}  // namespace

bool tc_eligible(int r, int d_h, int B) {
    return r >= kTcMinHeads && r <= kMaxRows && (d_h == 64 || d_h == 128) && tc_smem_bytes(d_h, B) <= 227u * 1024u;
}

size_t tc_smem_bytes(int d_h, int B) { return d_h == 128 ? smem_tc<128>(B) : smem_tc<64>(B); }

cudaError_t run_split_tc(const DecodeParams &p, const CUtensorMap *tmk, const CUtensorMap *tmv, int d_h, int ctas,
                         cudaStream_t st) {
    const bool two = p.r > 32;
    if (d_h == 128) return two ? run<128, 2>(p, tmk, tmv, ctas, st) : run<128, 1>(p, tmk, tmv, ctas, st);
    return two ? run<64, 2>(p, tmk, tmv, ctas, st) : run<64, 1>(p, tmk, tmv, ctas, st);
}

}  // namespace dec
}  // namespace gqa
