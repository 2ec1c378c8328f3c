// Exact attention of a prefill chunk over sinks U selected units U local window on the
// 5th-generation tensor cores (tcgen05, bf16 operands, fp32 accumulators in TMEM).
//
// Method: "InfLLM Guide: Training-Free Long-Context Memory Units", "Core Innovation 2",
// item 3 "Exact Attention Evaluation": one softmax over Sinks U (U_{m in top-k} M_m) U Local
// Window; for a chunk this is a dense contraction per (query tile, KV tile).
//
// One CTA per (128 packed query rows, KV head): the rows are G q heads x 128/G consecutive
// queries of one KV group, so every K/V tile is read once per group.  Warp roles:
//   warp 0      TMA producer: the two query tiles once, then K and V tiles (2-stage rings)
//   warp 1      MMA issuer:   S_i = Q K_i^T into S buffer i & 1 (Q and K from shared memory);
//                             O_{i & 1} += P_i V_i with P read from TMEM
//   warps 2..9  softmax:      two groups of four warps (one warp per TMEM lane quarter, one thread
//                             per row): group g takes the KV tiles i with i & 1 == g, all 128
//                             columns of each.  Each group runs its own online softmax over its
//                             tiles -- its own running max, sum and accumulator O_g -- so the two
//                             never wait for each other inside the loop and work on different
//                             tiles at once; O_g is rescaled lazily (only when the group's max
//                             grows by > 2^8).  P_i goes as bf16 over the first 64 columns of S_i.
//                             After the last tile the groups exchange (max, sum) once through
//                             shared memory and each thread stores HD / 2 outputs of the merged row.
// Splitting a row's keys into two sets and merging the partial softmaxes at the end is exact (up
// to rounding): it is the log-sum-exp combination of two disjoint key sets.  S_i and P_i share a
// buffer, double buffered: the exponentials of tile i overlap QK of tile i + 1 and the PV product
// of tile i - 1, and QK of tile i + 2 (same buffer) is issued after PV(i) -- the tensor pipe
// executes one thread's MMAs in issue order.  The MMA-issuing thread keeps pace with the tensor
// pipe (its queue is short), so its loop holds no lookups: the K and V ring slots are released by
// the same two barriers that announce S_i and PV(i), and the query tile is chosen by tile index.
// Likewise each softmax group does what does not need S_i (the tile's column limit, consuming its
// previous PV) while QK(i) runs, so that only the max, the exponentials and the store follow S_i.
// Sinks and memory tiles use R(W) q with raw keys; window tiles use R(t) q with R(n) k.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_maps.cuh"
#include "tc_ptx.cuh"

namespace infllm {

namespace {

constexpr int BM = 128;  // packed query rows per CTA
constexpr int BN = 128;  // keys per tile
constexpr int NTHREADS = 320;  // producer warp, MMA warp, 8 softmax warps
constexpr int NSOFT = 256;     // softmax threads
constexpr uint32_t SWB = BN * 128;  // one 64-column swizzle block of a tile (128 rows x 128 B)
constexpr int NSTAGE = 2;           // K and V ring depth (= the S buffers: the ring reuses their barriers)
static_assert(NSTAGE == 2, "the K / V slots are released by the S / PV barriers of the two tile parities");
constexpr int MAX_SEL = 4096;       // selected unit ids of this KV head kept in shared memory

// Shared-memory layout for head dim HD (64 or 128): a tile is HD / 64 swizzle blocks.
template <int HD>
struct Lay {
    static constexpr uint32_t TILE = BN * HD * 2;  // bytes of one bf16 128 x HD tile
    static constexpr int OFF_QM = 0;               // R(W) q tile (sinks and memory units)
    static constexpr int OFF_QW = OFF_QM + (int)TILE;  // R(t) q tile (window)
    static constexpr int OFF_K = OFF_QW + (int)TILE;
    static constexpr int OFF_V = OFF_K + NSTAGE * (int)TILE;
    static constexpr int OFF_BAR = OFF_V + NSTAGE * (int)TILE;
    static constexpr int OFF_LSUM = OFF_BAR + 256;           // [2 groups][128] row sums
    static constexpr int OFF_MREF = OFF_LSUM + 2 * 128 * 4;  // [2 groups][128] reference maxima (log2 units)
    static constexpr int OFF_SEL = OFF_MREF + 2 * 128 * 4;   // selected unit ids of this KV head
    static constexpr int SMEM_BYTES = OFF_SEL + MAX_SEL * 4 + 1024;  // + alignment slack
};
static_assert(Lay<128>::SMEM_BYTES <= 227 * 1024, "shared-memory layout exceeds the per-CTA limit");

// TMEM columns: S0 / P0 [0,128), S1 / P1 [128,256), O_0 [256, 256 + HD), O_1 [256 + HD, 256 + 2 HD)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_O = 256;  // O_g: the products with the KV tiles of parity g
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_LOG2 = 8.0f;
constexpr int ERR_TIMEOUT = 16;

struct Bars {
    // sfull, pfull and pvdone alternate by tile parity: S(i) lands on sfull[i & 1], P(i) is released on
    // pfull[i & 1] and PV(i) completes on pvdone[i & 1], so that no consumer can fall two phases behind
    // one barrier (parity aliasing)
    // K / V slot i % NSTAGE is free again once QK(i) / PV(i) is complete: sfull / pvdone, as NSTAGE == 2
    uint64_t q, kfull[NSTAGE], vfull[NSTAGE], sfull[2], pfull[2], pvdone[2];
    uint32_t tmem;
    int abort;
};

static_assert(sizeof(Bars) <= 256, "barrier block overflows its shared-memory slot");

struct TileInfo {
    int kind;  // 0 sink, 1 memory unit, 2 window
    int64_t y0;
    int nv;
};

struct Plan {
    int a, hk, kk, nst, tpu, nut, nwt, NT, S_eff, par;
    int64_t t_hi, B, win_len;
    const int* sel;  // shared-memory copy; -1 marks an id that failed its range check

    __device__ TileInfo tile(const Dev& D, int i) const {
        if (i < nst) return {0, (int64_t)i * BN, min(BN, S_eff - i * BN)};
        i -= nst;
        if (i < nut) {
            const int u = tpu == 1 ? i : i / tpu, part = tpu == 1 ? 0 : i % tpu;
            const int j = sel[u];
            if (j < 0) return {1, 0, 0};
            return {1, (int64_t)D.S + (int64_t)j * D.U + (int64_t)part * BN, min(BN, D.U - part * BN)};
        }
        i -= nut;
        const int64_t rem = win_len - (int64_t)i * BN;
        return {2, B + (int64_t)i * BN, (int)(rem < BN ? rem : BN)};
    }
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars* bars, const Dev& D) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (*(volatile int*)&bars->abort) return false;
        if (clock64() - t0 > (1ll << 32)) {  // ~2 s: something is broken; give up cleanly
            *(volatile int*)&bars->abort = 1;
            set_err(D, ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// One tile row of HD bf16 is HD / 64 swizzle blocks, each its own 64-column TMA box.
template <int HD>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* m, uint64_t* bar, int y, int hk) {
#pragma unroll
    for (int b = 0; b < HD / 64; ++b) ptx::tma_load_3d(dst + b * SWB, m, bar, 64 * b, y, hk);
}

template <int HD>
__device__ void producer(const TcMaps& maps, const Plan& P, const Dev& D, uint8_t* sm, Bars* bars) {
    using Y = Lay<HD>;
    ptx::prefetch_tmap(&maps.qm);
    ptx::prefetch_tmap(&maps.qw);
    ptx::prefetch_tmap(&maps.kraw);
    ptx::prefetch_tmap(&maps.krot);
    ptx::prefetch_tmap(&maps.v);
    {   // both rotated query tiles of this CTA's 128 packed rows (slot par of the query buffers)
        const int y = P.par * (int)D.qrows_max + P.a * BM;
        ptx::mbar_expect_tx(&bars->q, 2 * Y::TILE);
        load_tile<HD>(sm + Y::OFF_QM, &maps.qm, &bars->q, y, P.hk);
        load_tile<HD>(sm + Y::OFF_QW, &maps.qw, &bars->q, y, P.hk);
    }
    int issued = 0;
    for (int i = 0; i < P.NT; ++i) {
        const int s = i % NSTAGE;
        const uint32_t use = (uint32_t)(i / NSTAGE);
        // K slot s held tile i - 2: free once QK(i - 2) is complete, which sfull[s] announces
        if (i >= NSTAGE && !wait_bar(&bars->sfull[s], (use - 1) & 1, bars, D)) break;
        const TileInfo T = P.tile(D, i);
        const CUtensorMap* km = T.kind == 2 ? &maps.krot : &maps.kraw;
        ptx::mbar_expect_tx(&bars->kfull[s], Y::TILE);
        load_tile<HD>(sm + Y::OFF_K + s * Y::TILE, km, &bars->kfull[s], (int)T.y0, P.hk);
        // V slot s: free once PV(i - 2) is complete (pvdone[s])
        if (i >= NSTAGE && !wait_bar(&bars->pvdone[s], (use - 1) & 1, bars, D)) {
            issued = i + 1;
            break;
        }
        ptx::mbar_expect_tx(&bars->vfull[s], Y::TILE);
        load_tile<HD>(sm + Y::OFF_V + s * Y::TILE, &maps.v, &bars->vfull[s], (int)T.y0, P.hk);
        issued = i + 1;
    }
    if (*(volatile int*)&bars->abort) {
        // let the copies already in flight land before the CTA exits (bounded)
        for (int i = issued - NSTAGE < 0 ? 0 : issued - NSTAGE; i < issued; ++i) {
            ptx::mbar_wait(&bars->kfull[i % NSTAGE], (uint32_t)(i / NSTAGE) & 1, 1ll << 28);
            ptx::mbar_wait(&bars->vfull[i % NSTAGE], (uint32_t)(i / NSTAGE) & 1, 1ll << 28);
        }
        ptx::mbar_wait(&bars->q, 0, 1ll << 28);
    }
}

template <int HD>
__device__ void mma_issuer(const Plan& P, const Dev& D, uint8_t* sm, Bars* bars, uint32_t tmem) {
    using Y = Lay<HD>;
    constexpr uint32_t IDESC_QK = ptx::idesc_bf16_f32(BM, BN, false, false);
    constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(BM, HD, false, true);
    if (!wait_bar(&bars->q, 0, bars, D)) return;  // the query tiles have landed
    ptx::tc_fence_after();
    const uint32_t qm = ptx::smem_u32(sm + Y::OFF_QM), qw = ptx::smem_u32(sm + Y::OFF_QW);
    const uint32_t kb = ptx::smem_u32(sm + Y::OFF_K), vb = ptx::smem_u32(sm + Y::OFF_V);
    for (int i = 0; i <= P.NT; ++i) {
        if (i < P.NT) {
            // S_i into buffer i & 1, which held P_{i-2}: PV(i - 2) was issued in the previous
            // iteration, before this MMA, and same-thread MMAs execute in order
            const int s = i % NSTAGE, b = i & 1;
            if (!wait_bar(&bars->kfull[s], (uint32_t)(i / NSTAGE) & 1, bars, D)) return;
            ptx::tc_fence_after();
            const uint32_t qa = i >= P.nst + P.nut ? qw : qm;
            const uint32_t ka = kb + s * Y::TILE;
#pragma unroll
            for (int ks = 0; ks < HD / 16; ++ks) {  // 16 of the head dim: swizzle block ks / 4, 32 B each
                const uint32_t off = (uint32_t)(ks >> 2) * SWB + (uint32_t)(ks & 3) * 32;
                ptx::mma_bf16(tmem + b * BN, ptx::sdesc_sw128(qa + off, 16, 1024), ptx::sdesc_sw128(ka + off, 16, 1024),
                              IDESC_QK, ks > 0 ? 1u : 0u);
            }
            ptx::mma_commit(&bars->sfull[b]);
        }
        if (i >= 1) {
            const int j = i - 1, sj = j % NSTAGE, bj = j & 1;
            if (!wait_bar(&bars->pfull[j & 1], (uint32_t)(j >> 1) & 1, bars, D)) return;
            if (!wait_bar(&bars->vfull[sj], (uint32_t)(j / NSTAGE) & 1, bars, D)) return;
            ptx::tc_fence_after();
            const uint32_t va = vb + sj * Y::TILE;
#pragma unroll
            for (int ks = 0; ks < BN / 16; ++ks)  // keys 16 ks .. 16 ks + 15 of P_j, into O_{j & 1}
                ptx::mma_bf16_ts(tmem + TM_O + (uint32_t)bj * HD, tmem + bj * BN + (uint32_t)ks * 8,
                                 ptx::sdesc_sw128(va + (uint32_t)ks * 2048, SWB, 1024), IDESC_PV,
                                 (j > 1 || ks > 0) ? 1u : 0u);
            ptx::mma_commit(&bars->pvdone[j & 1]);
        }
    }
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Bars* bars, const Dev& D) {
    const bool ok = wait_bar(bar, parity, bars, D);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// PV completions of one softmax group: the x-th PV product of group g (tile g + 2x) completes phase x
// of pvdone[g].  Consumed strictly in order and never two phases late: the group consumes its
// previous PV before it releases its next P, and that PV is issued only after the release.
struct PvTrack {
    int seen = 0;  // this group's PV products known complete: its first `seen` tiles
    __device__ __forceinline__ bool upto(int x, uint64_t* bar, Bars* bars, const Dev& D) {
        while (seen <= x) {
            if (!warp_wait(bar, (uint32_t)seen & 1, bars, D)) return false;
            ++seen;
        }
        return true;
    }
};

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int HD>
__device__ void softmax_role(const Plan& P, const Dev& D, Bars* bars, float* lsum, float* mref, uint32_t tmem,
                             int64_t c0, int n, __nv_bfloat16* __restrict__ out, int warp, int lane) {
    const int quarter = warp & 3;       // TMEM lanes this warp may access
    const int grp = (warp - 2) >> 2;    // KV tiles i with i & 1 == grp are this thread's
    const int row = quarter * 32 + lane;
    const uint32_t tl_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t sbase = tl_addr + (uint32_t)grp * BN;       // S_i / P_i of this group's tiles
    const uint32_t o_addr = tl_addr + TM_O + (uint32_t)grp * HD;  // this thread's row of O_grp
    const int hg = row / D.qt, tl = P.a * D.qt + row % D.qt;
    const bool valid = tl < n;
    const int64_t t = c0 + tl;
    const float sc = D.inv_sqrt_d * LOG2E;  // logits in log2 units: s * sc
    float m_used = -INFINITY, l = 0.f;
    PvTrack pv;
    uint64_t* pvbar = &bars->pvdone[grp];
    bool ok = true;
    for (int i = grp; i < P.NT; i += 2) {
        const int x = i >> 1;  // this group's tile count before tile i
        // columns [0, lim) of this tile are attended by this row (causal limit on sinks and window);
        // known before S(i) lands
        const TileInfo T = P.tile(D, i);
        int lim = T.nv;
        if (T.kind != 1) {
            const int64_t c = t - T.y0 + 1;
            lim = c < (int64_t)lim ? (int)(c < 0 ? 0 : c) : lim;
        }
        const bool full = __all_sync(0xffffffffu, lim >= BN);
        // O_grp holds this group's earlier products (and P_i may be released) once PV of its previous
        // tile is complete; PV(i - 2) was issued before QK(i), so it is complete before S(i) lands
        if (x >= 1 && !pv.upto(x - 1, pvbar, bars, D)) {
            ok = false;
            break;
        }
        if (!warp_wait(&bars->sfull[grp], (uint32_t)x & 1, bars, D)) {
            ok = false;
            break;
        }
        ptx::tc_fence_after();
        float s[128];
        ptx::tmem_ld32(sbase, s);
        ptx::tmem_ld32(sbase + 32, s + 32);
        ptx::tmem_ld32(sbase + 64, s + 64);
        ptx::tmem_ld32(sbase + 96, s + 96);
        ptx::tmem_wait_ld();
        float mq[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mq[e] = -INFINITY;
        if (!full) {
#pragma unroll
            for (int c = 0; c < 128; ++c) s[c] = c < lim ? s[c] : -INFINITY;
        }
#pragma unroll
        for (int c = 0; c < 128; c += 2) mq[(c >> 1) & 7] = max3(mq[(c >> 1) & 7], s[c], s[c + 1]);
        const float mx = fmaxf(fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])), fmaxf(fmaxf(mq[4], mq[5]), fmaxf(mq[6], mq[7])));
        const float mt = mx * sc;
        const bool need = mt > m_used + RESCALE_LOG2;
        const float m_new = need ? mt : m_used;
        const float f = need ? ex2(m_used - m_new) : 1.f;  // rescale of this group's O and sum
        m_used = m_new;
        const float nref = m_used == -INFINITY ? 0.f : -m_used;
        float rs[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) rs[e] = 0.f;
        uint32_t w[64];  // the tile's 128 keys as 64 columns of packed bf16 pairs
#pragma unroll
        for (int e = 0; e < 64; ++e) {
            const float p0 = ex2(fmaf(s[2 * e], sc, nref)), p1 = ex2(fmaf(s[2 * e + 1], sc, nref));
            rs[(2 * e) & 7] += p0;
            rs[(2 * e + 1) & 7] += p1;
            // bf16 pair on the integer pipe: round half up (+0x8000), keep the two high halves
            w[e] = __byte_perm(__float_as_uint(p0) + 0x8000u, __float_as_uint(p1) + 0x8000u, 0x7632);
        }
        ptx::tmem_st32(sbase, reinterpret_cast<const float*>(w));  // over columns [0, 64) of S_i, read above
        ptx::tmem_st32(sbase + 32, reinterpret_cast<const float*>(w + 32));
        l = fmaf(l, f, ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7])));
        // a growing maximum rescales O_grp here, before PV(i) adds to it
        if (x >= 1 && __any_sync(0xffffffffu, need)) {
            ptx::tc_fence_after();
#pragma unroll
            for (int c4 = 0; c4 < HD / 32; ++c4) {
                float o[32];
                ptx::tmem_ld32(o_addr + c4 * 32, o);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] *= f;
                ptx::tmem_st32(o_addr + c4 * 32, o);
            }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bars->pfull[grp]);
    }
    const int mine = P.NT > grp ? (P.NT - grp + 1) >> 1 : 0;  // tiles of this group
    ok = ok && (mine == 0 || pv.upto(mine - 1, pvbar, bars, D));
    // the two groups of a row meet: O = (2^(m_0 - M) O_0 + 2^(m_1 - M) O_1) / (same weights on
    // l_0, l_1), M = max(m_0, m_1); a group without tiles has m = -inf, weight 0 and an O that was
    // never written (selected away, not multiplied).  Each of the pair stores HD / 2 outputs.
    lsum[grp * 128 + row] = l;
    mref[grp * 128 + row] = m_used;
    asm volatile("bar.sync 1, %0;" ::"n"(NSOFT) : "memory");
    if (!__all_sync(0xffffffffu, ok)) return;
    ptx::tc_fence_after();
    const float m0 = mref[row], m1 = mref[128 + row];
    const float M = fmaxf(m0, m1);
    const float f0 = m0 == -INFINITY ? 0.f : ex2(m0 - M), f1 = m1 == -INFINITY ? 0.f : ex2(m1 - M);
    const float inv = 1.f / (lsum[row] * f0 + lsum[128 + row] * f1);
    const float g0 = f0 * inv, g1 = f1 * inv;
    const bool use0 = f0 != 0.f, use1 = f1 != 0.f;
    constexpr int OWN = HD / 2;
    __nv_bfloat16* orow = out + ((int64_t)tl * D.Hq + P.hk * D.G + hg) * HD + grp * OWN;
#pragma unroll 1
    for (int c4 = 0; c4 < OWN / 32; ++c4) {
        float o0[32], o1[32];
        ptx::tmem_ld32(tl_addr + TM_O + grp * OWN + c4 * 32, o0);
        ptx::tmem_ld32(tl_addr + TM_O + HD + grp * OWN + c4 * 32, o1);
        ptx::tmem_wait_ld();
        if (valid) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint32_t w4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int k = e * 8 + 2 * q;
                    const float a0 = use0 ? o0[k] * g0 : 0.f, a1 = use0 ? o0[k + 1] * g0 : 0.f;
                    const float b0 = use1 ? o1[k] * g1 : 0.f, b1 = use1 ? o1[k + 1] * g1 : 0.f;
                    __nv_bfloat162 h = __floats2bfloat162_rn(a0 + b0, a1 + b1);
                    w4[q] = *reinterpret_cast<uint32_t*>(&h);
                }
                *reinterpret_cast<uint4*>(orow + c4 * 32 + e * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        }
    }
}

template <int HD>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_tc(const __grid_constant__ TcMaps maps, Dev D, int64_t c0, int n, int kk, int64_t B, int par,
              __nv_bfloat16* __restrict__ out) {
    using Y = Lay<HD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    Bars* bars = reinterpret_cast<Bars*>(sm + Y::OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    Plan P;
    P.a = gridDim.x - 1 - blockIdx.x;  // query tiles with more keys start first
    P.hk = blockIdx.y;
    P.par = par;
    P.kk = kk;
    P.B = B;
    {
        const int last = min(n, (P.a + 1) * D.qt);
        P.t_hi = c0 + last - 1;
    }
    P.S_eff = (int)(D.S < P.t_hi + 1 ? D.S : P.t_hi + 1);
    P.nst = (P.S_eff + BN - 1) / BN;
    P.tpu = (D.U + BN - 1) / BN;
    P.nut = kk * P.tpu;
    P.win_len = P.t_hi + 1 - B;
    P.nwt = P.win_len > 0 ? (int)((P.win_len + BN - 1) / BN) : 0;
    P.NT = P.nst + P.nut + P.nwt;

    int* sel_s = reinterpret_cast<int*>(sm + Y::OFF_SEL);
    P.sel = sel_s;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bars->q, 1);
        for (int s = 0; s < NSTAGE; ++s) {
            ptx::mbar_init(&bars->kfull[s], 1);
            ptx::mbar_init(&bars->vfull[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&bars->sfull[b], 1);
            ptx::mbar_init(&bars->pfull[b], NSOFT / 2);  // the threads of group b
            ptx::mbar_init(&bars->pvdone[b], 1);
        }
        bars->abort = 0;
        ptx::mbar_fence_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(&bars->tmem, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    // Late kernel: the selection, the packed queries and this chunk's keys are complete past the
    // wait; the next chunk's store-side kernels may start once every CTA is here.
    pdl_wait();
    pdl_trigger();
    for (int u = threadIdx.x; u < kk; u += blockDim.x) {
        int j = D.sel[P.hk * D.topk + u];
        if (j < 0 || (int64_t)D.S + (int64_t)(j + 1) * D.U > B) {
            set_err(D, ERR_SEL_RANGE);
            j = -1;
        }
        sel_s[u] = j;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem;

    if (P.NT > 0) {
        if (warp == 0) {
            if (lane == 0) producer<HD>(maps, P, D, sm, bars);
        } else if (warp == 1) {
            if (lane == 0) mma_issuer<HD>(P, D, sm, bars, tmem);
        } else {
            softmax_role<HD>(P, D, bars, reinterpret_cast<float*>(sm + Y::OFF_LSUM),
                             reinterpret_cast<float*>(sm + Y::OFF_MREF), tmem, c0, n, out, warp, lane);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, TMEM_COLS);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// 3-D bf16 map over [dim2][dim1][hd] with box [1][128][64], 128-byte swizzle.
bool encode_3d(CUtensorMap* m, void* base, uint64_t hd, uint64_t dim1, uint64_t dim2) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t gdim[3] = {(cuuint64_t)hd, (cuuint64_t)dim1, (cuuint64_t)dim2};
    cuuint64_t gstride[2] = {(cuuint64_t)hd * 2, (cuuint64_t)hd * 2 * dim1};
    cuuint32_t box[3] = {64, (cuuint32_t)BN, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attend_tc_supported(const Dev& D) {
    if ((D.d != 64 && D.d != 128) || D.G > BM || BM % D.G != 0 || D.qt * D.G != BM || D.topk > MAX_SEL) return false;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    return major == 10 && get_encode() != nullptr;
}

size_t tc_maps_size() { return sizeof(TcMaps); }

bool make_tc_maps(const Dev& D, void* out) {
    TcMaps* m = reinterpret_cast<TcMaps*>(out);
    const uint64_t hd = (uint64_t)D.d;
    return encode_3d(&m->kraw, D.Kraw, hd, (uint64_t)D.T_max, (uint64_t)D.Hkv) &&
           encode_3d(&m->krot, D.Krot, hd, (uint64_t)D.T_max, (uint64_t)D.Hkv) &&
           encode_3d(&m->v, D.V, hd, (uint64_t)D.T_max, (uint64_t)D.Hkv) &&
           encode_3d(&m->qm, D.Qm, hd, 3 * (uint64_t)D.qrows_max, (uint64_t)D.Hkv) &&
           encode_3d(&m->qw, D.Qw, hd, 3 * (uint64_t)D.qrows_max, (uint64_t)D.Hkv);
}

cudaError_t launch_attend_tc(const Dev& D, int64_t c0, int n, int kk, int64_t B, int par, void* out, cudaStream_t st,
                             const void* tmaps, bool pdl) {
    if (n <= 0) return cudaSuccess;
    const int tiles = (n + D.qt - 1) / D.qt;
    const TcMaps& maps = *reinterpret_cast<const TcMaps*>(tmaps);
    if (D.d == 64) {
        static std::atomic<unsigned long long> attr_done{0};
        cudaError_t e = smem_limit_once(k_attn_tc<64>, Lay<64>::SMEM_BYTES, attr_done);
        if (e != cudaSuccess) return e;
        return launch_k(k_attn_tc<64>, dim3(tiles, D.Hkv), dim3(NTHREADS), Lay<64>::SMEM_BYTES, st, pdl, maps, D, c0, n,
                        kk, B, par, (__nv_bfloat16*)out);
    }
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = smem_limit_once(k_attn_tc<128>, Lay<128>::SMEM_BYTES, attr_done);
    if (e != cudaSuccess) return e;
    return launch_k(k_attn_tc<128>, dim3(tiles, D.Hkv), dim3(NTHREADS), Lay<128>::SMEM_BYTES, st, pdl, maps, D, c0, n,
                    kk, B, par, (__nv_bfloat16*)out);
}

}  // namespace infllm
