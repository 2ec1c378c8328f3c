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
//   k_decode_append           store the token (early kernel)
//   k_decode_attn, part 0     sink and window tiles: need the store, not the selection
//   unit scoring + top-k      reads only the representative pool and the query, so it runs
//                             alongside part 0 (it holds its completion until part 0 is done)
//   k_decode_attn, part 1     the selected units' tiles (waits for the selection)
//   k_decode_merge            log-sum-exp merge of every tile's partial
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_maps.cuh"
#include "tc_ptx.cuh"

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
// zero, padded row stride) | reductions.  The P V partials of the four warps reuse the K tile.
constexpr int QSTRIDE = DHD * 2 + 16;  // bytes per padded query row (conflict-free ldmatrix)
constexpr int OFF_K = 0;
constexpr int OFF_V = OFF_K + (int)DTILE;
constexpr int OFF_Q = OFF_V + (int)DTILE;
constexpr int OFF_RED = OFF_Q + 16 * QSTRIDE;
constexpr int OFF_MISC = OFF_RED + 2 * 4 * 8 * 4;
constexpr int DSMEM = OFF_MISC + 64 + 1024;  // + alignment slack

// One CTA per KV head: K, R(t) K and V of token t into the stores, the query block sum of t,
// and (cos, sin)(t theta_i) in fp64 for the attention kernel.
__global__ void __launch_bounds__(DTHREADS) k_decode_append(Dev D, const __nv_bfloat16* __restrict__ q,
                                                            const __nv_bfloat16* __restrict__ k,
                                                            const __nv_bfloat16* __restrict__ v, int64_t t) {
    __shared__ float2 cs[DHD / 2];
    pdl_trigger();  // early kernel: the lookup may start now (it reads none of these stores)
    const int hk = blockIdx.x;
    for (int i = threadIdx.x; i < D.half; i += blockDim.x) {
        cs[i] = cs_abs(D.cs_abs3, D.half, t, i);
        if (hk == 0) D.cs_chunk[i] = cs[i];
    }
    __syncthreads();
    __nv_bfloat16* Kraw = (__nv_bfloat16*)D.Kraw;
    __nv_bfloat16* Krot = (__nv_bfloat16*)D.Krot;
    __nv_bfloat16* V = (__nv_bfloat16*)D.V;
    const int64_t dst = ((int64_t)hk * D.T_max + t) * D.d;
    for (int i = threadIdx.x; i < D.half; i += blockDim.x) {
        const __nv_bfloat16 a = k[hk * D.d + i], b = k[hk * D.d + i + D.half];
        Kraw[dst + i] = a;
        Kraw[dst + i + D.half] = b;
        const float x1 = __bfloat162float(a), x2 = __bfloat162float(b);
        Krot[dst + i] = __float2bfloat16_rn(x1 * cs[i].x - x2 * cs[i].y);
        Krot[dst + i + D.half] = __float2bfloat16_rn(x2 * cs[i].x + x1 * cs[i].y);
        V[dst + i] = v[hk * D.d + i];
        V[dst + i + D.half] = v[hk * D.d + i + D.half];
        if (t >= D.S) {  // query block sum (same arithmetic as the chunk kernel for one token)
            const int64_t b = (t - D.S) / D.gblk, p = (t - D.S) % D.gblk;
            float qx[MAXG], qy[MAXG];
#pragma unroll
            for (int h = 0; h < MAXG; ++h) {
                qx[h] = qy[h] = 0.f;
                if (h < D.G) {
                    qx[h] = __bfloat162float(q[(hk * D.G + h) * D.d + i]);
                    qy[h] = __bfloat162float(q[(hk * D.G + h) * D.d + i + D.half]);
                }
            }
            float s1 = 0.f, s2 = 0.f;
#pragma unroll
            for (int h = 0; h < MAXG; ++h) {
                s1 += qx[h];
                s2 += qy[h];
            }
            const float2 c = D.cs_rel[p * D.half + i];
            float* y = D.Y + (b * D.Hkv + hk) * D.d;
            y[i] += s1 * c.x - s2 * c.y;
            y[i + D.half] += s2 * c.x + s1 * c.y;
        }
    }
    pdl_hold();
}

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

// Grid (tiles, Hkv), 128 threads = 4 warps, warp w owns keys [32w, 32w + 32) of the tile.
// The group's G query heads (rows, padded to 16 with zeros) times the tile on the tensor cores
// (mma.sync m16n8k16, bf16 in, fp32 accumulate): S = Q K^T, then O = P V with P kept in
// registers; softmax statistics are combined across the four warps through shared memory.
__global__ void __launch_bounds__(DTHREADS) k_decode_attn(const __grid_constant__ TcMaps maps, Dev D,
                                                          const __nv_bfloat16* __restrict__ q, int64_t t, int kk,
                                                          int64_t B, int part) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* red = reinterpret_cast<float*>(sm + OFF_RED);  // [2][4 warps][8 rows]
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_MISC);
    const int hk = blockIdx.y;
    // tile index in the working context (sinks, units, window): part 0 takes sinks and window,
    // part 1 the selected units
    const int nst = ((D.S < t + 1 ? D.S : (int)(t + 1)) + DK - 1) / DK;
    const int nut = kk * ((D.U + DK - 1) / DK);
    const int ti = part == 1 ? nst + (int)blockIdx.x : ((int)blockIdx.x < nst ? (int)blockIdx.x : (int)blockIdx.x + nut);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tg = lane & 3;
    const int G = D.G;
    pdl_trigger();  // the next kernel reads nothing this one writes before the merge
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::mbar_fence_init();
    }
    __syncthreads();
    pdl_wait();  // the token's store, its (cos, sin) and (part 1) the selection are ready past this point
    const DTile T = decode_tile(D, hk, ti, t, kk, B);
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
        const float2* cs = T.kind == 2 ? D.cs_chunk : D.cs_W;
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
    bool ok = ptx::mbar_wait(bar, 0);
    if (!ok) set_err(D, ERR_TIMEOUT);
    ok = __syncthreads_and(ok);
    // S for the warp's 32 keys: n-tiles nt -> keys 32w + 8nt + (0..7)
    const uint32_t kbase = ptx::smem_u32(sm + OFF_K), vbase = ptx::smem_u32(sm + OFF_V);
    float sacc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
    {
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
    __syncthreads();  // every warp is done with the K tile: reuse it for the cross-warp sum of O
    float* obuf = reinterpret_cast<float*>(sm + OFF_K);  // [4 warps][8 rows][DHD]
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        obuf[(warp * 8 + g) * DHD + 8 * nt + 2 * tg] = oacc[nt][0];
        obuf[(warp * 8 + g) * DHD + 8 * nt + 2 * tg + 1] = oacc[nt][1];
    }
    __syncthreads();
    float* pout = D.dec_part + ((int64_t)hk * D.dec_splits_max + ti) * G * (DHD + 2);
    for (int h = 0; h < G; ++h) {
        const float o = obuf[(0 * 8 + h) * DHD + tid] + obuf[(1 * 8 + h) * DHD + tid] + obuf[(2 * 8 + h) * DHD + tid] +
                        obuf[(3 * 8 + h) * DHD + tid];
        pout[h * (DHD + 2) + 2 + tid] = o;
        if (tid == 0) {
            const float mh = fmaxf(fmaxf(red[h], red[8 + h]), fmaxf(red[16 + h], red[24 + h]));
            pout[h * (DHD + 2) + 0] = mh == -INFINITY ? -INFINITY : mh * D.inv_sqrt_d;  // natural-log units
            pout[h * (DHD + 2) + 1] = red[32 + h] + red[40 + h] + red[48 + h] + red[56 + h];
        }
    }
}

// Log-sum-exp merge of the NT tile partials of one (KV head, q head): grid (G, Hkv), 512 threads
// = 4 slices of tiles x 128 output dims; every load of a slice issued in one batch.
constexpr int MERGE_SLICES = 4;
constexpr int MERGE_BATCH = 32;

__global__ void __launch_bounds__(MERGE_SLICES * DHD) k_decode_merge(Dev D, __nv_bfloat16* __restrict__ out, int NT) {
    __shared__ float ml[2][MERGE_SLICES * MERGE_BATCH];
    __shared__ float red[2][MERGE_SLICES][DHD];
    pdl_wait();     // the tile partials are complete past this point
    pdl_trigger();  // every earlier kernel is complete: the next step's store kernels may start
    const int h = blockIdx.x, hk = blockIdx.y, G = D.G, d = DHD;
    const int dim = threadIdx.x % DHD, z = threadIdx.x / DHD;
    const float* base = D.dec_part + (int64_t)hk * D.dec_splits_max * G * (d + 2) + (int64_t)h * (d + 2);
    const int64_t stride = (int64_t)G * (d + 2);
    for (int s = threadIdx.x; s < NT && s < MERGE_SLICES * MERGE_BATCH; s += blockDim.x) {
        ml[0][s] = base[s * stride];
        ml[1][s] = base[s * stride + 1];
    }
    __syncthreads();
    float M = -INFINITY;
    for (int s = 0; s < NT; ++s) M = fmaxf(M, ml[0][s]);
    float L = 0.f, O = 0.f;
    float acc[MERGE_BATCH];
#pragma unroll
    for (int u = 0; u < MERGE_BATCH; ++u) {
        const int s = z + MERGE_SLICES * u;
        acc[u] = s < NT ? base[s * stride + 2 + dim] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < MERGE_BATCH; ++u) {
        const int s = z + MERGE_SLICES * u;
        if (s < NT) {
            const float m = ml[0][s];
            const float w = m == -INFINITY ? 0.f : expf(m - M);
            L += w * ml[1][s];
            O += w * acc[u];
        }
    }
    red[0][z][dim] = L;
    red[1][z][dim] = O;
    __syncthreads();
    if (z == 0) {
        float Lt = 0.f, Ot = 0.f;
        for (int q = 0; q < MERGE_SLICES; ++q) {
            Lt += red[0][q][dim];
            Ot += red[1][q][dim];
        }
        out[(int64_t)(hk * G + h) * d + dim] = __float2bfloat16_rn(Ot / Lt);
    }
}

}  // namespace

bool decode_tc_supported(const Dev& D) { return D.d == DHD && D.G <= MAXG && D.topk <= 32; }

cudaError_t launch_decode_append(const Dev& D, const void* q, const void* k, const void* v, int64_t t,
                                 cudaStream_t st, bool pdl) {
    return launch_k(k_decode_append, dim3(D.Hkv), dim3(DTHREADS), 0, st, pdl, D, (const __nv_bfloat16*)q,
                    (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, t);
}

cudaError_t launch_decode_tc(const Dev& D, const void* q, int64_t t, int kk, int64_t B, int part, cudaStream_t st,
                             const void* tmaps, bool pdl) {
    const int S_eff = (int)(D.S < t + 1 ? D.S : t + 1);
    const int64_t win = t - B + 1;
    const int nst = (S_eff + DK - 1) / DK, nut = kk * ((D.U + DK - 1) / DK), nwt = (int)((win + DK - 1) / DK);
    if (nst + nut + nwt > D.dec_splits_max || nst + nut + nwt > MERGE_SLICES * MERGE_BATCH) return cudaErrorInvalidValue;
    const int tiles = part == 1 ? nut : nst + nwt;
    if (tiles == 0) return cudaSuccess;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = smem_limit_once(k_decode_attn, DSMEM, attr_done);
    if (e != cudaSuccess) return e;
    return launch_k(k_decode_attn, dim3(tiles, D.Hkv), dim3(DTHREADS), DSMEM, st, pdl,
                    *reinterpret_cast<const TcMaps*>(tmaps), D, (const __nv_bfloat16*)q, t, kk, B, part);
}

cudaError_t launch_decode_merge(const Dev& D, int64_t t, int kk, int64_t B, void* out, cudaStream_t st, bool pdl) {
    const int S_eff = (int)(D.S < t + 1 ? D.S : t + 1);
    const int NT = (S_eff + DK - 1) / DK + kk * ((D.U + DK - 1) / DK) + (int)((t - B + 1 + DK - 1) / DK);
    return launch_k(k_decode_merge, dim3(D.G, D.Hkv), dim3(MERGE_SLICES * DHD), 0, st, pdl, D, (__nv_bfloat16*)out, NT);
}

}  // namespace infllm
