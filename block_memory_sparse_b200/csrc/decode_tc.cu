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
#pragma unroll
        for (int h = 0; h < MAXG; ++h) {
            if (h >= G) continue;
            float o = 0.f;
            for (int sl = 0; sl < nr; ++sl) o = fmaf(wts[h][sl], sbuf[sl * sf + h * PST + 4 + tid], o);
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

// ---- one decode step in one cooperative launch ------------------------------------------------

// Per-step arguments of k_decode_step.
struct StepArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    __nv_bfloat16* out;
    int64_t t, B;
    unsigned long long qbase;  // value of the context's work counter when this step's unit tiles start
    int kk, nm, nst, nwt, nut;  // selected units, eligible units, sink / window / unit tiles per head
    int mode, tag;              // scoring operand; this step's flag value (> every earlier step's)
    // Static partition of the scoring rows (units of all heads, head-major: N = Hkv nm) over the first
    // gs CTAs.  weighted: CTA c < nw_cta also loads a window tile worth wr rows, so the ranges balance
    // rows + window rows: range start = floor(c T / gs) - wr min(c, nw_cta), T = N + nw_cta wr;
    // otherwise start = floor(c N / gs).
    int64_t N, T;
    int gs, weighted, wr, nw_cta;
};

// Start of CTA c's scoring range (flat unit index; N for c >= gs).  Non-decreasing in c, and strictly
// increasing over [0, gs] (the host checks the weighted split's rows per CTA exceed a window tile's).
__host__ __device__ __forceinline__ int64_t score_f0(const StepArgs& A, int c) {
    if (c >= A.gs) return A.N;
    if (A.weighted) {
        const int64_t r = (int64_t)c * A.T / A.gs - (int64_t)A.wr * (c < A.nw_cta ? c : A.nw_cta);
        return r < 0 ? 0 : (r > A.N ? A.N : r);
    }
    return (int64_t)c * A.N / A.gs;
}
// The CTA whose scoring range holds flat unit f (0 <= f < N): the largest c < gs with score_f0(c) <= f.
__host__ __device__ __forceinline__ int score_owner(const StepArgs& A, int64_t f) {
    int lo = 0, hi = A.gs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (score_f0(A, mid) <= f) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Bounded wait (one thread) for a flag another CTA of this grid sets to `tag` with a release store.
__device__ __forceinline__ bool wait_flag(const Dev& D, const int* flag, int tag) {
    if (ld_acquire(flag) == tag) return true;
    const long long t0 = clock64();
    while (ld_acquire(flag) != tag) {
        if (clock64() - t0 > (1ll << 32)) {  // ~2 s: something is broken; give up cleanly
            set_err(D, ERR_TIMEOUT);
            return false;
        }
        __nanosleep(100);
    }
    return true;
}

// Scoring rows stream through a ring of SSTAGES bulk copies of SBYTES each, in the K and V tiles'
// shared memory; each stage has its own mbarrier after the tile barrier.  The rest of the tiles'
// space stages the candidate lists of a head's selection (LSTAGE lists at a time).
constexpr int SSTAGES = 3;
constexpr uint32_t SBYTES = 16384;
constexpr int OFF_LSTAGE = OFF_K + SSTAGES * (int)SBYTES;
constexpr int LSTAGE = (int)((2 * DTILE - SSTAGES * SBYTES) / 256);
static_assert(LSTAGE >= 32, "no room to stage the candidate lists");
constexpr int OFF_SBAR = OFF_MISC + 16;
static_assert(16 + SSTAGES * 8 <= 64, "stage barriers overflow their slot");
// after the (cos, sin) table: the scoring query R(W) (sum of the group's q heads) of every KV head
constexpr int OFF_QB = OFF_CS + (DHD / 2) * 8;
__host__ __device__ constexpr int step_smem(int hkv) { return OFF_QB + hkv * DHD * 4 + 1024; }

// Scoring rows of flat unit f (head f / nm, unit f % nm) in the pool of the step's score mode.
template <int ROWB>
__device__ __forceinline__ const uint8_t* score_row(const Dev& D, const StepArgs& A, int64_t f) {
    const uint8_t* pool = A.mode == OP_REPS ? (const uint8_t*)D.rep_keys
                          : A.mode == OP_REPSUM ? (const uint8_t*)D.repsum
                                                : (const uint8_t*)D.meankey;
    return pool + ((f / A.nm) * D.units_max + f % A.nm) * ROWB;
}
// Units in the chunk that starts at flat unit f of a range ending at f1: at most a stage, and never
// across a head boundary (the heads' rows are not contiguous in the pool).
template <int ROWB>
__device__ __forceinline__ int chunk_units(const StepArgs& A, int64_t f, int64_t f1) {
    constexpr int UPS = (int)SBYTES / ROWB;
    const int64_t seg_end = min(f1, (f / A.nm + 1) * A.nm);
    return (int)min((int64_t)UPS, seg_end - f);
}

// Unit scores of this CTA's scoring range [f0, f1) of flat units (rows of ROWB bytes of E elements),
// streamed through the ring: thread 0 keeps SSTAGES bulk copies in flight from the first chunk to
// the last, across head boundaries.  The CTA's four warps score each stage from shared memory: a
// warp takes 4 units per step for 512- and 1024-byte rows, 8 units for 256-byte rows (consecutive
// lanes read consecutive 16 bytes), reduces each unit's dot product with the head's scoring query by
// a transpose-reduce and keeps a top-32 list.  At the end of each head's part of the range the CTA's
// list is published (part index = this CTA minus the head's first scoring CTA); the head's last CTA
// to publish selects the head's units and publishes them slot by slot.  `sph` holds the stage
// barriers' parities.  Returns false (error word set, copies in flight waited for) if a stage never
// arrived.
template <typename E, int ROWB>
__device__ bool score_range(const Dev& D, const StepArgs& A, int64_t f0, int64_t f1, uint8_t* sm, uint32_t& sph) {
    auto lists = reinterpret_cast<uint64_t(*)[32]>(sm + OFF_Q);  // [4][32]
    uint64_t* sbar = reinterpret_cast<uint64_t*>(sm + OFF_SBAR);
    constexpr int V = 16 / sizeof(E);
    constexpr int HALFROW = ROWB == 256;
    constexpr int CPL = HALFROW ? 1 : ROWB / 512;
    constexpr int UB = HALFROW ? 8 : 4;  // units per warp step
    constexpr int GRP = 32 / (HALFROW ? 8 : 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int64_t fi = f0;  // thread 0: next flat unit to put in flight
    int ki = 0;       // thread 0: chunks put in flight
    auto issue_next = [&]() {
        if (fi >= f1) return;
        const int n = chunk_units<ROWB>(A, fi, f1);
        uint64_t* bar = &sbar[ki % SSTAGES];
        ptx::mbar_expect_tx(bar, (uint32_t)(n * ROWB));
        ptx::bulk_load(sm + OFF_K + (ki % SSTAGES) * SBYTES, score_row<ROWB>(D, A, fi), (uint32_t)(n * ROWB), bar);
        fi += n;
        ++ki;
    };
    // the ring overwrites shared memory that the generic proxy wrote (a tile's partial sums, a merge's
    // copies); their use is over past the barrier
    ptx::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0)
        for (int c = 0; c < SSTAGES; ++c) issue_next();
    const int half = lane >> 4, piece = lane & 15;
    float qr[V];
    int hk = -1;
    uint64_t list = 0, cand = 0;
    int it = 0;
    int k = 0;
    for (int64_t fc = f0; fc < f1; ++k) {
        if (fc / A.nm != hk) {  // a new head's part of the range: its scoring query
            hk = (int)(fc / A.nm);
            const int i0 = ((HALFROW ? piece : lane) * V) % DHD;
            const float* qb = reinterpret_cast<const float*>(sm + OFF_QB) + hk * DHD;
#pragma unroll
            for (int x = 0; x < V; ++x) qr[x] = qb[i0 + x];
        }
        const int st = k % SSTAGES;
        const bool ok = __syncthreads_and(ptx::mbar_wait(&sbar[st], (sph >> st) & 1u));
        if (!ok) {  // the stage never landed: wait (bounded) for the copies in flight, then give up
            if (tid == 0) {
                set_err(D, ERR_TIMEOUT);
                for (int k2 = k + 1; k2 < ki; ++k2)  // at most SSTAGES - 1, each in its own stage
                    ptx::mbar_wait(&sbar[k2 % SSTAGES], (sph >> (k2 % SSTAGES)) & 1u, 1ll << 28);
            }
            __syncthreads();
            return false;
        }
        sph ^= 1u << st;
        const uint4* base = reinterpret_cast<const uint4*>(sm + OFF_K + st * SBYTES);
        const int u0c = (int)(fc % A.nm), nu = chunk_units<ROWB>(A, fc, f1);
        for (int g = warp; g * UB < nu; g += 4, ++it) {  // warp-uniform
            uint4 raw[4][CPL];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) {
                    const int u = HALFROW ? g * UB + 2 * i + half : g * UB + i;
                    raw[i][cc] = u < nu ? (HALFROW ? base[u * 16 + piece] : base[u * 32 * CPL + cc * 32 + lane])
                                        : make_uint4(0, 0, 0, 0);
                }
            float acc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float a = 0.f;
#pragma unroll
                for (int cc = 0; cc < CPL; ++cc) {
                    if (sizeof(E) == 2) {
                        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[i][cc]);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(h2[e]);
                            a += f.x * qr[2 * e] + f.y * qr[2 * e + 1];
                        }
                    } else {
                        const float* f = reinterpret_cast<const float*>(&raw[i][cc]);
#pragma unroll
                        for (int e = 0; e < 4; ++e) a += f[e] * qr[e];
                    }
                }
                acc[i] = a;
            }
            // halving steps then a butterfly: full rows -- masks 16, 8 then 4, 2, 1 (lane l: unit l / 8);
            // half rows -- masks 8, 4 then 2, 1 inside each half (lane l: unit 2 ((l / 4) % 4) + l / 16)
#pragma unroll
            for (int m = HALFROW ? 8 : 16, nv = 4; nv > 1; m >>= 1, nv >>= 1) {
                const bool upper = (lane & m) != 0;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (i < nv / 2) {
                        const float send = upper ? acc[i] : acc[i + nv / 2];
                        const float keep = upper ? acc[i + nv / 2] : acc[i];
                        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                    }
                }
            }
#pragma unroll
            for (int m = HALFROW ? 2 : 4; m >= 1; m >>= 1) acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], m);
            const int jl = HALFROW ? g * UB + 2 * ((lane >> 2) & 3) + half : g * UB + lane / 8;
            const int sub = HALFROW ? (lane & 3) : (lane & 7);
            const float sc = acc[0] * D.inv_sqrt_d;
            if (jl < nu) {
                const int j = u0c + jl;
                if (sub == 0) D.uscore[(int64_t)hk * D.units_max + j] = sc;
                if (sub == it % GRP) cand = make_key(sc, (uint32_t)j);
            }
            if (it % GRP == GRP - 1) {
                list = warp_topk_insert(list, cand);
                cand = 0;
            }
        }
        __syncthreads();  // every warp is done with stage st
        if (tid == 0) issue_next();
        fc += nu;
        if (fc == f1 || fc % A.nm == 0) {  // the end of this head's part: publish the CTA's list
            if (__any_sync(0xffffffffu, cand != 0)) list = warp_topk_insert(list, cand);
            lists[warp][lane] = list;
            for (int stride = 1; stride < 4; stride *= 2) {
                __syncthreads();
                if ((warp % (2 * stride)) == 0 && warp + stride < 4)
                    lists[warp][lane] = warp_merge_desc(lists[warp][lane], lists[warp + stride][lane]);
            }
            __syncthreads();
            const int c_first = score_owner(A, (int64_t)hk * A.nm);
            const int c_last = score_owner(A, (int64_t)(hk + 1) * A.nm - 1);
            publish_and_select(D, hk, (int)blockIdx.x - c_first, A.nm, c_last - c_first + 1, lists, 4, D.uflags,
                               (unsigned)A.tag, reinterpret_cast<uint64_t*>(sm + OFF_LSTAGE), LSTAGE);
            list = cand = 0;
            it = 0;
        }
    }
    return true;
}

// Bounded wait (one thread) for selected slot `slot` of KV head hk: returns the unit id, or -1 (error
// word set) if the slot is not published within ~2 s.
__device__ __forceinline__ int wait_slot(const Dev& D, int hk, int slot, unsigned tag) {
    const unsigned long long* f = D.uflags + hk * D.topk + slot;
    unsigned long long v = ld_acquire64(f);
    if ((unsigned)(v >> 32) != tag) {
        const long long t0 = clock64();
        while ((unsigned)((v = ld_acquire64(f)) >> 32) != tag) {
            if (clock64() - t0 > (1ll << 32)) {
                set_err(D, ERR_TIMEOUT);
                return -1;
            }
            __nanosleep(64);
        }
    }
    return (int)(uint32_t)v;
}

// One tile of the step's working context into its partial slot; the head's last tile of its part
// (arrival counter, re-armed by it) returns true.
__device__ __forceinline__ bool tile_and_count(const TcMaps& maps, const Dev& D, const StepArgs& A, int hk, int ti,
                                               int part, const DTile& T, uint8_t* sm, uint32_t& phase, int* sflag) {
    tile_partial(maps, D, A.q, A.k, A.v, A.t, hk, ti, T, part == 0 && A.t >= T.y0 && A.t < T.y0 + T.nv, sm, phase);
    __threadfence();
    __syncthreads();
    unsigned* ctr = D.counters + (2 + part) * D.Hkv + hk;
    const int nblocks = part == 0 ? A.nst + A.nwt : A.nut;
    if (threadIdx.x == 0) {
        *sflag = atomicAdd(ctr, 1u) == (unsigned)(nblocks - 1);
        if (*sflag) *ctr = 0u;  // re-armed for the next step (every arrival of this step is in)
    }
    __syncthreads();
    const bool last = *sflag != 0;
    if (last) __threadfence();
    return last;
}

// The merged sinks and window of KV head hk (its last window tile's CTA): into the merged slot,
// published on the head's window flag, or straight into the output when no unit is selected.
__device__ __forceinline__ void window_merge(const Dev& D, const StepArgs& A, int hk, uint8_t* sm) {
    merge_part(D, hk, 0, A.nst, A.nut, A.nwt, A.kk, sm, A.out);
    if (A.kk > 0) {
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) st_release(D.dflags + D.Hkv + hk, A.tag);
    }
    __syncthreads();
}

// A whole decode step in one cooperative launch (every CTA resident at once).  CTA c, in order:
//   1. window items c, c + grid, ...: the sink and window tiles of every KV head (the tile holding
//      token t stores it first); the head's last one merges them -- after its scoring (step 3), when
//      the grid covers every window tile, so that the merge's round trips do not delay its range;
//   2. its static range of the scoring rows (score_range): the unit scores, its lists, and for each
//      head the selection by the head's last CTA, published slot by slot with the unit ids;
//   3. the deferred window merges, published on the head's window flag;
//   4. unit tiles claimed from the context's counter: each waits (bounded) for its slot's flag; the
//      head's last one waits (bounded) for the window flag and merges everything into the output.
// Steps 1-3 wait for nothing, and the unit tiles wait only for them, so every wait ends.  The scoring
// ranges are balanced by rows plus window-tile rows (StepArgs), so all CTAs stream until about the
// same time and every byte is requested early.
template <typename E, int ROWB>
__global__ void __launch_bounds__(DTHREADS, 3) k_decode_step(const __grid_constant__ TcMaps maps, Dev D, StepArgs A) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_MISC);
    float2* cs_t = reinterpret_cast<float2*>(sm + OFF_CS);
    float* qball = reinterpret_cast<float*>(sm + OFF_QB);
    __shared__ int next_s, flag_s;
    const int tid = threadIdx.x, c = blockIdx.x, grid = gridDim.x;
    const int per_w = A.nst + A.nwt;
    const int NW = per_w * D.Hkv, NU = A.nut * D.Hkv;
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        for (int s = 0; s < SSTAGES; ++s) ptx::mbar_init(reinterpret_cast<uint64_t*>(sm + OFF_SBAR) + s, 1);
        ptx::mbar_fence_init();
    }
    for (int i = tid; i < DHD / 2; i += DTHREADS) cs_t[i] = cs_abs(D.cs_abs3, D.half, A.t, i);
    for (int x = tid; x < D.Hkv * (DHD / 2); x += DTHREADS) {  // R(W) of the summed group query, per KV head
        const int hk = x / (DHD / 2), i = x % (DHD / 2);
        float a = 0.f, b = 0.f;
        for (int h = 0; h < D.G; ++h) {
            a += __bfloat162float(A.q[(hk * D.G + h) * DHD + i]);
            b += __bfloat162float(A.q[(hk * D.G + h) * DHD + i + DHD / 2]);
        }
        const float2 cw = D.cs_W[i];
        qball[hk * DHD + i] = a * cw.x - b * cw.y;
        qball[hk * DHD + i + DHD / 2] = b * cw.x + a * cw.y;
    }
    __syncthreads();
    uint32_t phase = 0, sph = 0;
    int deferred = -1;  // KV head whose window merge waits for step 3
    // 1. window tiles
    for (int w = c; w < NW; w += grid) {
        const int hk = w / per_w, wi = w % per_w;
        const int ti = wi < A.nst ? wi : wi + A.nut;
        const DTile T = decode_tile(D, hk, ti, A.t, A.kk, A.B);
        if (tile_and_count(maps, D, A, hk, ti, 0, T, sm, phase, &flag_s)) {
            if (grid >= NW && A.kk > 0) deferred = hk;
            else window_merge(D, A, hk, sm);
        }
    }
    // 2. scoring range
    if (A.kk > 0) {
        const int64_t f0 = score_f0(A, c), f1 = score_f0(A, c + 1);
        if (f0 < f1 && !score_range<E, ROWB>(D, A, f0, f1, sm, sph)) return;  // error word set
    }
    // 3. deferred window merge
    if (deferred >= 0) window_merge(D, A, deferred, sm);
    // 4. unit tiles
    if (tid == 32) next_s = (int)(atomicAdd(D.dq, 1ull) - A.qbase);
    __syncthreads();
    const int tpu = (D.U + DK - 1) / DK;
    for (;;) {
        const int item = next_s;
        __syncthreads();
        if (item >= NU) break;
        if (tid == 32) next_s = (int)(atomicAdd(D.dq, 1ull) - A.qbase);  // the next claim overlaps this item
        const int hk = item / A.nut, ui = item % A.nut;
        const int ti = A.nst + ui, pt = ui % tpu;
        if (tid == 0) flag_s = wait_slot(D, hk, ui / tpu, (unsigned)A.tag);  // the slot's unit
        __syncthreads();
        const int id = flag_s;
        DTile T{1, 0, 0};
        if (id >= 0 && (int64_t)D.S + (int64_t)(id + 1) * D.U <= A.B)
            T = DTile{1, (int64_t)D.S + (int64_t)id * D.U + (int64_t)pt * DK, min(DK, D.U - pt * DK)};
        else if (id >= 0 && tid == 0)
            set_err(D, ERR_SEL_RANGE);
        if (!tile_and_count(maps, D, A, hk, ti, 1, T, sm, phase, &flag_s)) continue;
        if (tid == 0) flag_s = wait_flag(D, D.dflags + D.Hkv + hk, A.tag);  // the merged sinks and window
        __syncthreads();
        merge_part(D, hk, 1, A.nst, A.nut, A.nwt, A.kk, sm, A.out);
        __syncthreads();
    }
}

}  // namespace

constexpr int STEP_HKV_MAX = 64;  // KV heads the one-launch step keeps scoring queries for

bool decode_tc_supported(const Dev& D) { return D.d == DHD && D.G <= MAXG && D.topk <= 32 && D.Hkv <= STEP_HKV_MAX; }

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

template <typename E, int ROWB>
static cudaError_t launch_step(const Dev& D, const StepArgs& A, int grid, cudaStream_t st, const void* tmaps) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(DTHREADS);
    cfg.dynamicSmemBytes = step_smem(D.Hkv);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_decode_step<E, ROWB>, *reinterpret_cast<const TcMaps*>(tmaps), D, A);
}

// Resident CTAs of k_decode_step<E, ROWB> on the current device (the cooperative grid size).
template <typename E, int ROWB>
static int step_grid(const Dev& D, cudaError_t* err) {
    static std::atomic<unsigned long long> attr_done{0};
    *err = smem_limit_once(k_decode_step<E, ROWB>, step_smem(STEP_HKV_MAX), attr_done);
    if (*err != cudaSuccess) return 0;
    int dev = 0, sms = 0, per_sm = 0;
    if ((*err = cudaGetDevice(&dev)) != cudaSuccess) return 0;
    if ((*err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return 0;
    if ((*err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode_step<E, ROWB>, DTHREADS,
                                                              step_smem(D.Hkv))) !=
        cudaSuccess)
        return 0;
    return per_sm * sms;
}

cudaError_t launch_decode_step(const Dev& D, const void* q, const void* k, const void* v, int64_t t, int kk, int64_t B,
                               int nm, int score_mode, int tag, unsigned long long qbase, void* out, cudaStream_t st,
                               const void* tmaps, unsigned long long* consumed) {
    StepArgs A;
    A.q = (const __nv_bfloat16*)q;
    A.k = (const __nv_bfloat16*)k;
    A.v = (const __nv_bfloat16*)v;
    A.out = (__nv_bfloat16*)out;
    A.t = t;
    A.B = B;
    A.qbase = qbase;
    A.kk = kk;
    A.nm = nm;
    A.nst = (int)((std::min<int64_t>(D.S, t + 1) + DK - 1) / DK);
    A.nwt = (int)((t - B + 1 + DK - 1) / DK);
    A.nut = kk * ((D.U + DK - 1) / DK);
    A.mode = score_mode;
    A.tag = tag;
    if (A.nst + A.nut + A.nwt + 1 > D.dec_splits_max) return cudaErrorInvalidValue;  // + the merged slot
    const int row_bytes = score_mode == OP_REPS ? D.r * D.d * 2 : score_mode == OP_REPSUM ? D.d * 4 : D.d * 2;
    cudaError_t err = cudaSuccess;
    int grid = 0;
    switch (row_bytes) {
        case 1024: grid = step_grid<__nv_bfloat16, 1024>(D, &err); break;
        case 512: grid = score_mode == OP_REPSUM ? step_grid<float, 512>(D, &err) : step_grid<__nv_bfloat16, 512>(D, &err); break;
        case 256: grid = step_grid<__nv_bfloat16, 256>(D, &err); break;
        default: return cudaErrorInvalidValue;
    }
    if (err != cudaSuccess) return err;
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    // static split of the scoring rows (flat units, head-major) over the grid
    const int NW = (A.nst + A.nwt) * D.Hkv;
    A.N = kk > 0 ? (int64_t)D.Hkv * nm : 0;
    A.wr = (int)(2 * DTILE / row_bytes);  // a window tile's bytes, in scoring rows
    A.nw_cta = std::min(NW, grid);
    A.T = A.N + (int64_t)A.nw_cta * A.wr;
    A.weighted = grid > NW && A.T / grid >= A.wr + 1;  // then every range is at least one row
    A.gs = A.weighted ? grid : (int)std::max<int64_t>(1, std::min<int64_t>(grid, A.N / 16));  // plain: >= 16 rows each
    if (A.N > 0) {
        // every head's parts must fit its candidate-list slots: fewer, longer ranges until they do
        for (;;) {
            int worst = 0;
            for (int h = 0; h < D.Hkv; ++h)
                worst = std::max(worst, score_owner(A, (int64_t)(h + 1) * nm - 1) - score_owner(A, (int64_t)h * nm) + 1);
            if (worst <= D.score_splits_max) break;
            A.weighted = 0;
            A.gs = std::max(1, A.gs / 2);
        }
    }
    *consumed = (unsigned long long)A.nut * D.Hkv + (unsigned long long)grid;  // every CTA's last claim overshoots once
    switch (row_bytes) {
        case 1024: return launch_step<__nv_bfloat16, 1024>(D, A, grid, st, tmaps);
        case 512: return score_mode == OP_REPSUM ? launch_step<float, 512>(D, A, grid, st, tmaps)
                                                 : launch_step<__nv_bfloat16, 512>(D, A, grid, st, tmaps);
        default: return launch_step<__nv_bfloat16, 256>(D, A, grid, st, tmaps);
    }
}

}  // namespace infllm
