// Decode step on the TMA path (bf16, head dim 128): the new token's store, then split-KV
// attention over its working context (sinks, selected units, window) with a log-sum-exp merge.
//
// Method: "InfLLM Guide: Training-Free Long-Context Memory Units", "Core Innovation 2",
// items 2-3: per generated token, score the units, keep the top-k, exact attention over
// Sinks U selected units U window.  The split-KV form is exact: each CTA returns the max m,
// the sum l of exp(s - m) and the unnormalised output over its 128 keys; the last CTA of each
// KV head rescales every partial by exp(m_s - M) and divides by the total sum.
//
// Launch sequence of one step: k_decode_append (plain launch) -> unit scoring + top-k
// (programmatic dependent launch: it reads only the representative pool and the query, so it
// overlaps the store) -> k_decode_attn (programmatic dependent launch; waits for both).
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
constexpr int MAXG = 8;
constexpr int ERR_TIMEOUT = 16;
// dynamic shared memory: K tile | V tile | q frames [2][G][d] | p [G][DK] | reductions
constexpr int OFF_K = 0;
constexpr int OFF_V = OFF_K + (int)DTILE;
constexpr int OFF_Q = OFF_V + (int)DTILE;
constexpr int OFF_PS = OFF_Q + 2 * MAXG * DHD * 4;
constexpr int OFF_RED = OFF_PS + MAXG * DK * 4;
constexpr int OFF_MISC = OFF_RED + 2 * 4 * MAXG * 4;
constexpr int DSMEM = OFF_MISC + 64 + 1024;  // + alignment slack

// One CTA per KV head: K, R(t) K and V of token t into the stores, the query block sum of t,
// and (cos, sin)(t theta_i) in fp64 for the attention kernel.
__global__ void __launch_bounds__(DTHREADS) k_decode_append(Dev D, const __nv_bfloat16* __restrict__ q,
                                                            const __nv_bfloat16* __restrict__ k,
                                                            const __nv_bfloat16* __restrict__ v, int64_t t) {
    __shared__ float2 cs[DHD / 2];
    asm volatile("griddepcontrol.launch_dependents;");  // the lookup kernel may start now
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
            float s1 = 0.f, s2 = 0.f;
            for (int h = 0; h < D.G; ++h) {
                s1 += __bfloat162float(q[(hk * D.G + h) * D.d + i]);
                s2 += __bfloat162float(q[(hk * D.G + h) * D.d + i + D.half]);
            }
            const float2 c = D.cs_rel[p * D.half + i];
            float* y = D.Y + (b * D.Hkv + hk) * D.d;
            y[i] += s1 * c.x - s2 * c.y;
            y[i + D.half] += s2 * c.x + s1 * c.y;
        }
    }
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

// Grid (tiles, Hkv), 128 threads.  Thread j owns key j of the tile for the logits and output
// dimension j for P V.
__global__ void __launch_bounds__(DTHREADS) k_decode_attn(const __grid_constant__ TcMaps maps, Dev D,
                                                          const __nv_bfloat16* __restrict__ q,
                                                          __nv_bfloat16* __restrict__ out, int64_t t, int kk, int64_t B,
                                                          int NT) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* qs = reinterpret_cast<float*>(sm + OFF_Q);    // [2][G][d]: R(W) q, R(t) q
    float* ps = reinterpret_cast<float*>(sm + OFF_PS);   // [G][DK]
    float* red = reinterpret_cast<float*>(sm + OFF_RED); // [2][4][G]
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_MISC);
    const int hk = blockIdx.y, ti = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = D.G, d = DHD;
    asm volatile("griddepcontrol.launch_dependents;");  // the merge kernel may start its prologue
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::mbar_fence_init();
    }
    __syncthreads();
    pdl_wait();  // the token's store, its (cos, sin) and the selection are ready past this point
    const DTile T = decode_tile(D, hk, ti, t, kk, B);
    if (tid == 0) {
        const CUtensorMap* km = T.kind == 2 ? &maps.krot : &maps.kraw;
        ptx::mbar_expect_tx(bar, 2 * DTILE);
        ptx::tma_load_3d(sm + OFF_K, km, bar, 0, (int)T.y0, hk);
        ptx::tma_load_3d(sm + OFF_K + DHALF, km, bar, 64, (int)T.y0, hk);
        ptx::tma_load_3d(sm + OFF_V, &maps.v, bar, 0, (int)T.y0, hk);
        ptx::tma_load_3d(sm + OFF_V + DHALF, &maps.v, bar, 64, (int)T.y0, hk);
    }
    // rotated queries of the group's heads while the tiles land
    for (int idx = tid; idx < G * D.half; idx += blockDim.x) {
        const int h = idx / D.half, i = idx % D.half;
        const float x1 = __bfloat162float(q[(hk * G + h) * d + i]), x2 = __bfloat162float(q[(hk * G + h) * d + i + D.half]);
        const float2 cw = D.cs_W[i], ct = D.cs_chunk[i];
        qs[h * d + i] = x1 * cw.x - x2 * cw.y;
        qs[h * d + i + D.half] = x2 * cw.x + x1 * cw.y;
        qs[(G + h) * d + i] = x1 * ct.x - x2 * ct.y;
        qs[(G + h) * d + i + D.half] = x2 * ct.x + x1 * ct.y;
    }
    __syncthreads();
    bool ok = ptx::mbar_wait(bar, 0);
    if (!ok) set_err(D, ERR_TIMEOUT);
    ok = __syncthreads_and(ok);
    float sc[MAXG];
#pragma unroll
    for (int h = 0; h < MAXG; ++h) sc[h] = -INFINITY;
    if (ok && tid < T.nv) {
        const float* qf = qs + (T.kind == 2 ? G : 0) * d;
        float acc[MAXG];
#pragma unroll
        for (int h = 0; h < MAXG; ++h) acc[h] = 0.f;
        const uint8_t* krow = sm + OFF_K + tid * 128;
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {  // 16-byte chunk c of the row (swizzled inside its 128-byte line)
            const uint4 u = *reinterpret_cast<const uint4*>(krow + (c >> 3) * DHALF + (((c & 7) ^ (tid & 7)) << 4));
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
            float kv[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                kv[2 * e] = f.x;
                kv[2 * e + 1] = f.y;
            }
#pragma unroll
            for (int h = 0; h < MAXG; ++h) {
                if (h < G) {
                    const float4 qa = *reinterpret_cast<const float4*>(qf + h * d + c * 8);
                    const float4 qb = *reinterpret_cast<const float4*>(qf + h * d + c * 8 + 4);
                    acc[h] += qa.x * kv[0] + qa.y * kv[1] + qa.z * kv[2] + qa.w * kv[3] + qb.x * kv[4] +
                              qb.y * kv[5] + qb.z * kv[6] + qb.w * kv[7];
                }
            }
        }
#pragma unroll
        for (int h = 0; h < MAXG; ++h) sc[h] = acc[h] * D.inv_sqrt_d;
    }
    // per-head max and sum over the tile
    float mh[MAXG], lh[MAXG];
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        if (h < G) {
            const float m = warp_max(sc[h]);
            if (lane == 0) red[warp * G + h] = m;
        }
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        mh[h] = -INFINITY;
        if (h < G)
            for (int w = 0; w < 4; ++w) mh[h] = fmaxf(mh[h], red[w * G + h]);
    }
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        if (h < G) {
            const float p = (tid < T.nv && ok) ? expf(sc[h] - mh[h]) : 0.f;
            ps[h * DK + tid] = p;
            const float s = warp_sum(p);
            if (lane == 0) red[4 * G + warp * G + h] = s;
        }
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        lh[h] = 0.f;
        if (h < G)
            for (int w = 0; w < 4; ++w) lh[h] += red[4 * G + w * G + h];
    }
    // P V: thread owns output dimension tid (d == blockDim)
    float o[MAXG];
#pragma unroll
    for (int h = 0; h < MAXG; ++h) o[h] = 0.f;
    {
        const int dim = tid;
        const uint8_t* vcol = sm + OFF_V + (dim >> 6) * DHALF + (dim & 7) * 2;
        const int chunk = (dim & 63) >> 3;
        for (int j = 0; j < T.nv; ++j) {
            const float vv = __bfloat162float(
                *reinterpret_cast<const __nv_bfloat16*>(vcol + j * 128 + ((chunk ^ (j & 7)) << 4)));
#pragma unroll
            for (int h = 0; h < MAXG; ++h)
                if (h < G) o[h] += ps[h * DK + j] * vv;
        }
    }
    float* part = D.dec_part + ((int64_t)hk * D.dec_splits_max + ti) * G * (d + 2);
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        if (h < G) {
            part[h * (d + 2) + 2 + tid] = o[h];
            if (tid == 0) {
                part[h * (d + 2) + 0] = mh[h];
                part[h * (d + 2) + 1] = lh[h];
            }
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
    pdl_wait();  // the tile partials are complete past this point
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
                                 cudaStream_t st) {
    k_decode_append<<<D.Hkv, DTHREADS, 0, st>>>(D, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                               (const __nv_bfloat16*)v, t);
    return cudaGetLastError();
}

cudaError_t launch_decode_tc(const Dev& D, const void* q, int64_t t, int kk, int64_t B, void* out, cudaStream_t st,
                             const void* tmaps, int* n_tiles_out) {
    const int S_eff = (int)(D.S < t + 1 ? D.S : t + 1);
    const int64_t win = t - B + 1;
    const int NT = (S_eff + DK - 1) / DK + kk * ((D.U + DK - 1) / DK) + (int)((win + DK - 1) / DK);
    *n_tiles_out = NT;
    if (NT > D.dec_splits_max || NT > MERGE_SLICES * MERGE_BATCH) return cudaErrorInvalidValue;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_decode_attn, cudaFuncAttributeMaxDynamicSharedMemorySize, DSMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(NT, D.Hkv);
    cfg.blockDim = dim3(DTHREADS);
    cfg.dynamicSmemBytes = DSMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_decode_attn, *reinterpret_cast<const TcMaps*>(tmaps), D,
                                       (const __nv_bfloat16*)q, (__nv_bfloat16*)out, t, kk, B, NT);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t mcfg = {};
    mcfg.gridDim = dim3(D.G, D.Hkv);
    mcfg.blockDim = dim3(MERGE_SLICES * DHD);
    mcfg.dynamicSmemBytes = 0;
    mcfg.stream = st;
    mcfg.attrs = attr;
    mcfg.numAttrs = 1;
    return cudaLaunchKernelEx(&mcfg, k_decode_merge, D, (__nv_bfloat16*)out, NT);
}

}  // namespace infllm
