// Decode step on the TMA path (bf16, head dim 128): the new token's store, then split-KV
// attention over its working context (sinks, selected units, window) with a log-sum-exp merge.
//
// Method: "InfLLM Guide: Training-Free Long-Context Memory Units", "Core Innovation 2",
// items 2-3: per generated token, score the units, keep the top-k, exact attention over
// Sinks U selected units U window.  The split-KV form is exact: each CTA returns the max m,
// the sum l of exp(s - m) and the unnormalised output over its 128 keys; the last CTA of each
// KV head rescales every partial by exp(m_s - M) and divides by the total sum.
//
// Launch sequence of one step (programmatic dependent launches after the first):
//   k_decode_attn, part 0     the token's store (by the CTA whose tile holds it) and the sink and
//                             window tiles, which need no selection; the last CTA of each KV head
//                             merges their partials into one (early kernel)
//   unit scoring + top-k      reads only the representative pool and the query, so it runs
//                             alongside part 0 (it holds its completion until part 0 is done)
//   k_decode_attn, part 1     the selected units' tiles (waits for the selection); the last CTA
//                             of each KV head merges them with part 0's partial into the output
#include <cuda.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc_maps.cuh"
#include "tc_ptx.cuh"
#include "topk.cuh"

namespace infllm {
namespace {

constexpr int DK = 128;                     // keys per tile / CTA
constexpr int DHD = 128;                    // head dim
constexpr uint32_t DTILE = DK * DHD * 2;    // bytes of a bf16 tile
constexpr uint32_t DHALF = DTILE / 2;       // one 64-column swizzle block
constexpr int DTHREADS = 128;
constexpr int MAXG = 8;  // q heads per KV head on this path (rows of the padded MMA tile)
constexpr int ERR_TIMEOUT = 16;
// dynamic shared memory: K tile | V tile | this tile's rotated query [16 rows][d] bf16 (rows >= G
// zero, padded row stride) | reductions | barrier and flags | (cos, sin)(t theta_i).  The P V
// partials of the four warps reuse the K tile, and the final merges reuse both tiles.
constexpr int QSTRIDE = DHD * 2 + 16;  // bytes per padded query row (conflict-free ldmatrix)
constexpr int OFF_K = 0;
constexpr int OFF_V = OFF_K + (int)DTILE;
constexpr int OFF_Q = OFF_V + (int)DTILE;
constexpr int OFF_RED = OFF_Q + 16 * QSTRIDE;
constexpr int OFF_MISC = OFF_RED + 2 * 4 * 8 * 4;
constexpr int OFF_CS = OFF_MISC + 64;
constexpr int DSMEM = OFF_CS + (DHD / 2) * 8 + 1024;  // + alignment slack
static_assert(MAXG * 64 * 4 + MAXG * 2 * 4 <= 16 * QSTRIDE, "merge weights do not fit the query rows' space");
// A tile's partial softmax per q head: m (natural-log units), l, two pad floats, o[d] unnormalised.
constexpr int PST = DHD + 4;

struct DTile {
    int kind;  // 0 sink, 1 unit, 2 window
    int64_t y0;
    int nv;
};

// Tile i of the token's working context: sinks, then the selected units, then the window.
__device__ __forceinline__ DTile decode_tile(const Dev& D, int hk, int i, int64_t t, int kk, int64_t B) {
    const int S_eff = (int)(D.S < t + 1 ? D.S : t + 1);
    const int nst = (S_eff + DK - 1) / DK;
    if (i < nst) return {0, (int64_t)i * DK, min(DK, S_eff - i * DK)};
    i -= nst;
    const int tpu = (D.U + DK - 1) / DK;
    if (i < kk * tpu) {
        const int u = i / tpu, part = i % tpu;
        const int j = D.sel[hk * D.topk + u];
        if (j < 0 || (int64_t)D.S + (int64_t)(j + 1) * D.U > B) {
            set_err(D, ERR_SEL_RANGE);
            return {1, 0, 0};
        }
        return {1, (int64_t)D.S + (int64_t)j * D.U + (int64_t)part * DK, min(DK, D.U - part * DK)};
    }
    i -= kk * tpu;
    const int64_t rem = (t - B + 1) - (int64_t)i * DK;
    return {2, B + (int64_t)i * DK, (int)(rem < DK ? rem : DK)};
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
// Shared address of the 16-byte chunk c (8 elements) of row j in a TMA tile (two 64-column
// blocks of 128 rows x 128 bytes, 16-byte chunks XOR-swizzled by row % 8).
__device__ __forceinline__ uint32_t tile_chunk(uint32_t base, int j, int c) {
    return base + (uint32_t)(c >> 3) * DHALF + (uint32_t)j * 128 + ((uint32_t)((c & 7) ^ (j & 7)) << 4);
}


// Combine the partial softmaxes of `ns` tiles of KV head hk (slot_of(i) gives the i-th tile's slot,
// in a fixed order) into one: per q head, M = max m, L = sum exp(m - M) l, O = sum exp(m - M) o.
// A batch of slots is copied into shared memory at once (16-byte asynchronous copies, every copy of
// the batch in flight together); then one warp per q head computes M, the weights and L, and each
// thread (one output dim) sums the weighted o.  Batches (when the slots exceed `cap` floats) are
// combined by the same rule.  Writes the normalised output O / L (out != null) or the merged partial
// into slot `dst_slot`.  Exact up to rounding: the log-sum-exp combination of disjoint key sets.
template <typename SlotOf>
__device__ void merge_partials(const Dev& D, int hk, int ns, SlotOf slot_of, float* sbuf, int cap,
                               float (*wts)[64], float (*stat)[2], __nv_bfloat16* __restrict__ out, int dst_slot) {
    // wts[MAXG][64]: weights of a batch's slots (at most 64 per batch); stat[MAXG][2]: a batch's (M, L)
    const int G = D.G, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sf = G * PST;  // floats per slot
    const int per = min(64, cap / sf);
    float* pbase = D.dec_part + (int64_t)hk * D.dec_splits_max * sf;
    float M[MAXG], L[MAXG], O[MAXG];  // running totals (thread: output dim tid)
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        M[h] = -INFINITY;
        L[h] = 0.f;
        O[h] = 0.f;
    }
    for (int r0 = 0; r0 < ns; r0 += per) {
        const int nr = min(per, ns - r0);
        const int w4 = sf / 4;
        for (int x = tid; x < nr * w4; x += DTHREADS) {
            const int sl = x / w4, w = x % w4;
            cp_async16(sbuf + (size_t)x * 4, pbase + (int64_t)slot_of(r0 + sl) * sf + 4 * w);
        }
        cp_async_wait_all();
        __syncthreads();
        for (int h = warp; h < G; h += DTHREADS / 32) {
            float mx = -INFINITY;
            for (int sl = lane; sl < nr; sl += 32) mx = fmaxf(mx, sbuf[sl * sf + h * PST]);
            mx = warp_max(mx);
            float l = 0.f;
            for (int sl = lane; sl < nr; sl += 32) {
                const float m = sbuf[sl * sf + h * PST];
                const float wgt = m == -INFINITY ? 0.f : expf(m - mx);  // a tile with no attended key weighs 0
                wts[h][sl] = wgt;
                l = fmaf(wgt, sbuf[sl * sf + h * PST + 1], l);
            }
            l = warp_sum(l);
            if (lane == 0) {
                stat[h][0] = mx;
                stat[h][1] = l;
            }
        }
        __syncthreads();
        // the batch's weighted sum for every q head at once: one independent chain per head, so the
        // slots' loads and multiply-adds of different heads overlap
        float acc[MAXG];
#pragma unroll
        for (int h = 0; h < MAXG; ++h) acc[h] = 0.f;
#pragma unroll 2
        for (int sl = 0; sl < nr; ++sl) {
            const float* srow = sbuf + sl * sf + 4 + tid;
#pragma unroll
            for (int h = 0; h < MAXG; ++h)
                if (h < G) acc[h] = fmaf(wts[h][sl], srow[h * PST], acc[h]);
        }
#pragma unroll
        for (int h = 0; h < MAXG; ++h) {
            if (h >= G) continue;
            const float o = acc[h];
            const float mb = stat[h][0], lb = stat[h][1];
            if (mb == -INFINITY) continue;
            if (mb > M[h]) {  // rescale the running totals to the larger max
                const float f = M[h] == -INFINITY ? 0.f : expf(M[h] - mb);
                L[h] = fmaf(L[h], f, lb);
                O[h] = fmaf(O[h], f, o);
                M[h] = mb;
            } else {
                const float f = expf(mb - M[h]);
                L[h] = fmaf(f, lb, L[h]);
                O[h] = fmaf(f, o, O[h]);
            }
        }
        __syncthreads();  // the batch's buffers are reused
    }
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        if (h >= G) continue;
        if (out) {
            out[(int64_t)(hk * G + h) * DHD + tid] = __float2bfloat16_rn(O[h] / L[h]);
        } else {
            float* p = pbase + (int64_t)dst_slot * sf + h * PST;
            p[4 + tid] = O[h];
            if (tid == 0) {
                p[0] = M[h];
                p[1] = L[h];
            }
        }
    }
}

// One 128-key tile of the token's working context against the group's G query heads: the partial
// softmax (m, l, o) of every q head into slot ti of KV head hk.  Block of 128 threads = 4 warps, warp
// w owns keys [32w, 32w + 32) of the tile.  The group's G query heads (rows, padded to 16 with
// zeros) times the tile on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate): S = Q K^T,
// then O = P V with P kept in registers; softmax statistics are combined across the four warps
// through shared memory.  With store_here (the tile that holds token t) the token is stored first
// (K, R(t) K and V of KV head hk, and its query block sum), so the step needs no store kernel.
// `phase` is the parity of the CTA's tile barrier, flipped per tile.  Returns false on a timeout.
__device__ bool tile_partial(const TcMaps& maps, const Dev& D, const __nv_bfloat16* __restrict__ q,
                             const __nv_bfloat16* __restrict__ knew, const __nv_bfloat16* __restrict__ vnew, int64_t t,
                             int hk, int ti, const DTile& T, bool store_here, uint8_t* sm, uint32_t& phase) {
    float* red = reinterpret_cast<float*>(sm + OFF_RED);  // [2][4 warps][8 rows]
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_MISC);
    const float2* cs_t = reinterpret_cast<const float2*>(sm + OFF_CS);  // (cos, sin)(t theta_i)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tg = lane & 3;
    const int G = D.G;
    if (store_here) {
        // this tile holds the new token: store it before the tile is loaded
        __nv_bfloat16* Kraw = (__nv_bfloat16*)D.Kraw;
        __nv_bfloat16* Krot = (__nv_bfloat16*)D.Krot;
        __nv_bfloat16* Vs = (__nv_bfloat16*)D.V;
        const int64_t dst = ((int64_t)hk * D.T_max + t) * DHD;
        for (int i = tid; i < DHD / 2; i += DTHREADS) {
            const __nv_bfloat16 a = knew[hk * DHD + i], b = knew[hk * DHD + i + DHD / 2];
            Kraw[dst + i] = a;
            Kraw[dst + i + DHD / 2] = b;
            const float x1 = __bfloat162float(a), x2 = __bfloat162float(b);
            const float2 c = cs_t[i];
            Krot[dst + i] = __float2bfloat16_rn(x1 * c.x - x2 * c.y);
            Krot[dst + i + DHD / 2] = __float2bfloat16_rn(x2 * c.x + x1 * c.y);
            Vs[dst + i] = vnew[hk * DHD + i];
            Vs[dst + i + DHD / 2] = vnew[hk * DHD + i + DHD / 2];
            if (t >= D.S) {  // the token's query block sum (same arithmetic as the chunk kernel)
                const int64_t blk = (t - D.S) / D.gblk, p = (t - D.S) % D.gblk;
                float qx[MAXG], qy[MAXG];
#pragma unroll
                for (int h = 0; h < MAXG; ++h) {
                    qx[h] = qy[h] = 0.f;
                    if (h < G) {
                        qx[h] = __bfloat162float(q[(hk * G + h) * DHD + i]);
                        qy[h] = __bfloat162float(q[(hk * G + h) * DHD + i + DHD / 2]);
                    }
                }
                float s1 = 0.f, s2 = 0.f;
#pragma unroll
                for (int h = 0; h < MAXG; ++h) {
                    s1 += qx[h];
                    s2 += qy[h];
                }
                const float2 cr = D.cs_rel[p * D.half + i];
                float* y = D.Y + (blk * D.Hkv + hk) * DHD;
                y[i] += s1 * cr.x - s2 * cr.y;
                y[i + DHD / 2] += s2 * cr.x + s1 * cr.y;
            }
        }
        // the rows just written are read next by this CTA's bulk tensor copy (async proxy)
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncthreads();
    }
    // shared memory written by the generic proxy (the previous tile's partial sums, a merge's copies)
    // is about to be overwritten by a bulk tensor copy
    ptx::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        const CUtensorMap* km = T.kind == 2 ? &maps.krot : &maps.kraw;
        ptx::mbar_expect_tx(bar, 2 * DTILE);
        ptx::tma_load_3d(sm + OFF_K, km, bar, 0, (int)T.y0, hk);
        ptx::tma_load_3d(sm + OFF_K + DHALF, km, bar, 64, (int)T.y0, hk);
        ptx::tma_load_3d(sm + OFF_V, &maps.v, bar, 0, (int)T.y0, hk);
        ptx::tma_load_3d(sm + OFF_V + DHALF, &maps.v, bar, 64, (int)T.y0, hk);
    }
    // this tile's query frame (R(W) q for sinks and memory, R(t) q for the window) as bf16 rows
    {
        const float2* cs = T.kind == 2 ? cs_t : D.cs_W;
        for (int idx = tid; idx < 16 * (DHD / 2); idx += DTHREADS) {
            const int h = idx / (DHD / 2), i = idx % (DHD / 2);
            float r1 = 0.f, r2 = 0.f;
            if (h < G) {
                const float x1 = __bfloat162float(q[(hk * G + h) * DHD + i]);
                const float x2 = __bfloat162float(q[(hk * G + h) * DHD + i + DHD / 2]);
                const float2 c = cs[i];
                r1 = x1 * c.x - x2 * c.y;
                r2 = x2 * c.x + x1 * c.y;
            }
            __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(sm + OFF_Q + h * QSTRIDE);
            row[i] = __float2bfloat16_rn(r1);
            row[i + DHD / 2] = __float2bfloat16_rn(r2);
        }
    }
    __syncthreads();
    uint32_t qa[DHD / 16][4];
    {
        const uint32_t qbase = ptx::smem_u32(sm + OFF_Q) + (uint32_t)(lane & 15) * QSTRIDE + (uint32_t)(lane >> 4) * 16;
#pragma unroll
        for (int ks = 0; ks < DHD / 16; ++ks) ldsm_x4(qbase + ks * 32, qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
    }
    bool ok = ptx::mbar_wait(bar, phase);
    phase ^= 1u;
    if (!ok) set_err(D, ERR_TIMEOUT);
    ok = __syncthreads_and(ok);
    // S for the warp's 32 keys: n-tiles nt -> keys 32w + 8nt + (0..7)
    const uint32_t kbase = ptx::smem_u32(sm + OFF_K), vbase = ptx::smem_u32(sm + OFF_V);
    float sacc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
    if (ok) {
        const int key_a = 32 * warp + (lane & 7);  // lanes 0-15: n-tile 2p, lanes 16-31: n-tile 2p + 1
#pragma unroll
        for (int ks = 0; ks < DHD / 16; ++ks) {
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                const int key = key_a + 16 * pr + ((lane >> 4) << 3);
                const int c = 2 * ks + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(tile_chunk(kbase, key, c), b0, b1, b2, b3);
                mma16816(sacc[2 * pr], qa[ks], b0, b1);
                mma16816(sacc[2 * pr + 1], qa[ks], b2, b3);
            }
        }
    }
    // softmax over the tile for row g (heads g < G); keys >= nv are masked
    const float sc = D.inv_sqrt_d * 1.4426950408889634f;
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int key = 32 * warp + 8 * nt + 2 * tg + e;
            if (!ok || key >= T.nv) sacc[nt][e] = -INFINITY;
            mx = fmaxf(mx, sacc[nt][e]);
        }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if (tg == 0) red[warp * 8 + g] = mx;
    __syncthreads();
    float m = fmaxf(fmaxf(red[g], red[8 + g]), fmaxf(red[16 + g], red[24 + g]));
    const float mref = m == -INFINITY ? 0.f : m;
    float rs = 0.f;
    uint32_t pa[2][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        float p0, p1;
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p0) : "f"((sacc[nt][0] - mref) * sc));
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p1) : "f"((sacc[nt][1] - mref) * sc));
        rs += p0 + p1;
        // A fragment of P for k-step nt / 2: n-tile 2s -> a0a1 (rows g), 2s + 1 -> a4a5; rows 8..15 zero
        pa[nt >> 1][(nt & 1) ? 2 : 0] = pack_bf16(p0, p1);
        pa[nt >> 1][(nt & 1) ? 3 : 1] = 0u;
    }
    rs += __shfl_xor_sync(0xffffffffu, rs, 1);
    rs += __shfl_xor_sync(0xffffffffu, rs, 2);
    if (tg == 0) red[32 + warp * 8 + g] = rs;
    // O partial of this warp's 32 keys: 16 n-tiles of output dims
    float oacc[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[nt][e] = 0.f;
    if (ok) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const int key = 32 * warp + 16 * ks + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                const int c = 2 * np + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(tile_chunk(vbase, key, c), b0, b1, b2, b3);
                mma16816(oacc[2 * np], pa[ks], b0, b1);
                mma16816(oacc[2 * np + 1], pa[ks], b2, b3);
            }
        }
    }
    __syncthreads();  // every warp is done with the K tile: reuse it for the cross-warp sum of O
    float* obuf = reinterpret_cast<float*>(sm + OFF_K);  // [4 warps][8 rows][DHD]
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        obuf[(warp * 8 + g) * DHD + 8 * nt + 2 * tg] = oacc[nt][0];
        obuf[(warp * 8 + g) * DHD + 8 * nt + 2 * tg + 1] = oacc[nt][1];
    }
    __syncthreads();
    float* pout = D.dec_part + ((int64_t)hk * D.dec_splits_max + ti) * G * PST;
    for (int h = 0; h < G; ++h) {
        const float o = obuf[(0 * 8 + h) * DHD + tid] + obuf[(1 * 8 + h) * DHD + tid] + obuf[(2 * 8 + h) * DHD + tid] +
                        obuf[(3 * 8 + h) * DHD + tid];
        pout[h * PST + 4 + tid] = o;
        if (tid == 0) {
            const float mh = fmaxf(fmaxf(red[h], red[8 + h]), fmaxf(red[16 + h], red[24 + h]));
            pout[h * PST + 0] = mh == -INFINITY ? -INFINITY : mh * D.inv_sqrt_d;  // natural-log units
            pout[h * PST + 1] = red[32 + h] + red[40 + h] + red[48 + h] + red[56 + h];
        }
    }
    return ok;
}

// The partials of KV head hk's tiles of one part are all written: merge them (part 0: sinks and
// window into slot NT, or the output when no unit is selected; part 1: part 0's slot and the units
// into the output).
__device__ void merge_part(const Dev& D, int hk, int part, int nst, int nut, int nwt, int kk, uint8_t* sm,
                           __nv_bfloat16* __restrict__ out) {
    float* sbuf = reinterpret_cast<float*>(sm + OFF_K);  // K and V tiles: 64 KB
    const int cap = (int)(2 * DTILE / 4);
    auto wts = reinterpret_cast<float(*)[64]>(sm + OFF_Q);  // the query rows' space: 2 KB + 64 B
    auto stat = reinterpret_cast<float(*)[2]>(sm + OFF_Q + MAXG * 64 * 4);
    const int NT = nst + nut + nwt;
    if (part == 0)
        merge_partials(D, hk, nst + nwt, [=](int i) { return i < nst ? i : i + nut; }, sbuf, cap, wts, stat,
                       kk == 0 ? out : nullptr, NT);
    else
        merge_partials(D, hk, 1 + nut, [=](int i) { return i == 0 ? NT : nst + i - 1; }, sbuf, cap, wts, stat, out, 0);
}

// Grid (tiles, Hkv), 128 threads: one tile per CTA.
//   part 0: the sink and window tiles (an early kernel: it reads no result of its predecessor);
//   part 1: the selected units' tiles, after the selection.
// The head's last CTA of each part (arrival counter, no CTA waits for another) merges its partials.
__global__ void __launch_bounds__(DTHREADS, 1) k_decode_attn(const __grid_constant__ TcMaps maps, Dev D,
                                                          const __nv_bfloat16* __restrict__ q,
                                                          const __nv_bfloat16* __restrict__ knew,
                                                          const __nv_bfloat16* __restrict__ vnew, int64_t t, int kk,
                                                          int64_t B, int part, __nv_bfloat16* __restrict__ out) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_MISC);
    int* is_last = reinterpret_cast<int*>(sm + OFF_MISC + 8);
    float2* cs_t = reinterpret_cast<float2*>(sm + OFF_CS);
    const int hk = blockIdx.y, tid = threadIdx.x;
    const int nst = ((D.S < t + 1 ? D.S : (int)(t + 1)) + DK - 1) / DK;
    const int nut = kk * ((D.U + DK - 1) / DK);
    const int nwt = (int)((t - B + 1 + DK - 1) / DK);
    const int ti = part == 1 ? nst + (int)blockIdx.x : ((int)blockIdx.x < nst ? (int)blockIdx.x : (int)blockIdx.x + nut);
    if (part == 0) pdl_trigger();  // early: the lookup runs alongside
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::mbar_fence_init();
    }
    for (int i = tid; i < DHD / 2; i += DTHREADS) cs_t[i] = cs_abs(D.cs_abs3, D.half, t, i);
    __syncthreads();
    if (part == 1) {
        pdl_wait();  // the selection (and everything before it) is complete past this point
        pdl_trigger();
    }
    const DTile T = decode_tile(D, hk, ti, t, kk, B);
    uint32_t phase = 0;
    tile_partial(maps, D, q, knew, vnew, t, hk, ti, T, part == 0 && t >= T.y0 && t < T.y0 + T.nv, sm, phase);
    __threadfence();
    __syncthreads();
    unsigned* ctr = D.counters + (2 + part) * D.Hkv + hk;
    const int nblocks = part == 0 ? nst + nwt : nut;
    if (tid == 0) *is_last = atomicAdd(ctr, 1u) == (unsigned)(nblocks - 1);
    __syncthreads();
    if (*is_last) {
        __threadfence();
        merge_part(D, hk, part, nst, nut, nwt, kk, sm, out);
        if (tid == 0) *ctr = 0u;  // re-armed for the next step
    }
    if (part == 0) pdl_hold();
}

}  // namespace

bool decode_tc_supported(const Dev& D) { return D.d == DHD && D.G <= MAXG && D.topk <= 32; }

cudaError_t launch_decode_tc(const Dev& D, const void* q, const void* k, const void* v, int64_t t, int kk, int64_t B,
                             int part, void* out, cudaStream_t st, const void* tmaps, bool pdl) {
    const int S_eff = (int)(D.S < t + 1 ? D.S : t + 1);
    const int64_t win = t - B + 1;
    const int nst = (S_eff + DK - 1) / DK, nut = kk * ((D.U + DK - 1) / DK), nwt = (int)((win + DK - 1) / DK);
    if (nst + nut + nwt + 1 > D.dec_splits_max) return cudaErrorInvalidValue;  // + the merged slot
    const int tiles = part == 1 ? nut : nst + nwt;
    if (tiles == 0) return cudaSuccess;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = smem_limit_once(k_decode_attn, DSMEM, attr_done);
    if (e != cudaSuccess) return e;
    return launch_k(k_decode_attn, dim3(tiles, D.Hkv), dim3(DTHREADS), DSMEM, st, pdl,
                    *reinterpret_cast<const TcMaps*>(tmaps), D, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                    (const __nv_bfloat16*)v, t, kk, B, part, (__nv_bfloat16*)out);
}

}  // namespace infllm
