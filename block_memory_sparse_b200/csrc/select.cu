// Unit lookup: score every eligible memory unit against the chunk's queries and keep the
// top-k per kv head, ties to the lower unit index.
//
// Method: "InfLLM Guide: Training-Free Long-Context Memory Units", "Core Innovation 2",
// item 2 "Query-Aware Top-K Scoring and Loading" (Score(M_j) = q . r_j / sqrt(d), keep the
// top-k); lookup per chunk during pre-filling: OpenReview rebuttal (paperhub.cn), Q2.
// A chunk's score of unit j sums the scaled logits of every (query, q head of the group,
// representative) triple, with the query at relative distance W:
//   sigma_j = <R(W) sum_t sum_h q_{t,h}, sum_m k_{j,m}> / sqrt(d)
// which is linear, so the queries are summed first (prep kernel) and each unit costs one
// read of its representative keys (REPS mode) or of their fp32 sum (REPSUM mode).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc_maps.cuh"
#include "topk.cuh"

namespace infllm {

// Rotated, packed queries of the chunk.  Grid (tiles, Hkv), 256 threads.  Tile a holds
// queries [a*qt, a*qt + qt); row r of a tile is (head hg = r / qt, query a*qt + r % qt).
// Thread = (vector v: elements [vV, vV+V) of each half, row group): 16-byte loads and stores,
// four rows per load batch.  Also writes each tile's raw query sum over its rows
// (fixed-order reduction).  An early kernel: it may run while an earlier chunk's attention
// reads another query slot, and while this chunk's keys are stored, so it takes the
// (cos, sin)(t theta_i) of its queries from the fp64 digit tables itself.
template <typename T>
__global__ void __launch_bounds__(256) k_prep(Dev D, const T* __restrict__ q, int64_t c0, int n, int par) {
    extern __shared__ float red[];  // [row groups][d], then (cos, sin) [qt][half]
    pdl_trigger();
    constexpr int V = 16 / sizeof(T);
    constexpr int RB = 4;
    union Vec { uint4 u; T h[V]; };
    const int a = blockIdx.x, hk = blockIdx.y;
    const int rows = D.qt * D.G;
    const int nv = D.half / V;
    const int o = threadIdx.x % nv, rg = threadIdx.x / nv, nrg = blockDim.x / nv;
    const int i0 = o * V;
    float2* cs_sh = reinterpret_cast<float2*>(red + nrg * D.d);
    for (int x = threadIdx.x; x < D.qt * D.half; x += blockDim.x) {
        const int tl = a * D.qt + x / D.half;
        cs_sh[x] = tl < n ? cs_abs(D.cs_abs3, D.half, c0 + tl, x % D.half) : make_float2(1.f, 0.f);
    }
    __syncthreads();
    const int64_t qbase = ((int64_t)hk * 3 + par) * D.qrows_max + (int64_t)a * rows;
    T* Qm = (T*)D.Qm + qbase * D.d;
    T* Qw = (T*)D.Qw + qbase * D.d;
    float2 cw[V];
#pragma unroll
    for (int e = 0; e < V; ++e) cw[e] = D.cs_W[i0 + e];
    float s1[V], s2[V];
#pragma unroll
    for (int e = 0; e < V; ++e) s1[e] = s2[e] = 0.f;
    for (int r0 = rg; r0 < rows; r0 += nrg * RB) {
        Vec x1[RB], x2[RB];
        float2 ct[RB][V];
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int r = r0 + u * nrg;
            const int hg = r / D.qt, tl = a * D.qt + r % D.qt;
            x1[u].u = x2[u].u = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int e = 0; e < V; ++e) ct[u][e] = make_float2(1.f, 0.f);
            if (r < rows && tl < n) {
                const T* src = q + ((int64_t)tl * D.Hq + hk * D.G + hg) * D.d;
                x1[u].u = *reinterpret_cast<const uint4*>(src + i0);
                x2[u].u = *reinterpret_cast<const uint4*>(src + i0 + D.half);
#pragma unroll
                for (int e = 0; e < V; ++e) ct[u][e] = cs_sh[(tl - a * D.qt) * D.half + i0 + e];
            }
        }
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int r = r0 + u * nrg;
            if (r >= rows) continue;
            Vec m1, m2, w1, w2;
#pragma unroll
            for (int e = 0; e < V; ++e) {
                const float a1 = to_f(x1[u].h[e]), a2 = to_f(x2[u].h[e]);
                s1[e] += a1;
                s2[e] += a2;
                m1.h[e] = from_f<T>(a1 * cw[e].x - a2 * cw[e].y);
                m2.h[e] = from_f<T>(a2 * cw[e].x + a1 * cw[e].y);
                w1.h[e] = from_f<T>(a1 * ct[u][e].x - a2 * ct[u][e].y);
                w2.h[e] = from_f<T>(a2 * ct[u][e].x + a1 * ct[u][e].y);
            }
            T* dm = Qm + (int64_t)r * D.d;
            T* dw = Qw + (int64_t)r * D.d;
            *reinterpret_cast<uint4*>(dm + i0) = m1.u;
            *reinterpret_cast<uint4*>(dm + i0 + D.half) = m2.u;
            *reinterpret_cast<uint4*>(dw + i0) = w1.u;
            *reinterpret_cast<uint4*>(dw + i0 + D.half) = w2.u;
        }
    }
    float* rr = red + rg * D.d;
#pragma unroll
    for (int e = 0; e < V; ++e) {
        rr[i0 + e] = s1[e];
        rr[i0 + e + D.half] = s2[e];
    }
    __syncthreads();
    for (int j = threadIdx.x; j < D.d; j += blockDim.x) {
        float acc = 0.f;
        for (int g = 0; g < nrg; ++g) acc += red[g * D.d + j];
        D.qbar_part[((int64_t)hk * D.qtiles_max + a) * D.d + j] = acc;
    }
    pdl_hold();
}

// 16-byte vector of the score operand, converted to floats.
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* f) {
        uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float2 x = __bfloat1622float2(h[c]);
            f[2 * c] = x.x;
            f[2 * c + 1] = x.y;
        }
    }
};
template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void load(const float* p, float* f) {
        float4 u = __ldg(reinterpret_cast<const float4*>(p));
        f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
    }
};

// Grid (n_split, Hkv), 512 threads.  Each unit is scored by a group of LPU lanes that split
// its operand (16-byte loads issued in batches of 8), reduced inside the group; PER = 512 / LPU
// units per CTA.  Writes the unit scores and, with do_select, the top-k (last CTA per head).
constexpr int SC_THREADS = 512;
constexpr int SC_WARPS = SC_THREADS / 32;

template <typename T, int MODE, int LPU>
__global__ void __launch_bounds__(SC_THREADS, 2) k_score_topk(Dev D, int n_mem, int n_split, int n_qtiles,
                                                           const T* qraw, int do_select, int wait_first) {
    __shared__ float qb[128];
    if (wait_first) pdl_wait();  // the query sums (and the representatives) come from the kernels before
    pdl_trigger();               // the attention kernel may start its prologue
    const int split = blockIdx.x, hk = blockIdx.y;
    for (int i = threadIdx.x; i < D.half; i += blockDim.x) {
        float a = 0.f, b = 0.f;
        if (qraw) {
            for (int h0 = 0; h0 < D.G; h0 += 8) {
                float x[8], y[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    x[u] = y[u] = 0.f;
                    if (h0 + u < D.G) {
                        x[u] = to_f(qraw[(hk * D.G + h0 + u) * D.d + i]);
                        y[u] = to_f(qraw[(hk * D.G + h0 + u) * D.d + i + D.half]);
                    }
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    a += x[u];
                    b += y[u];
                }
            }
        } else {
            for (int t0 = 0; t0 < n_qtiles; t0 += 8) {
                float x[8], y[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    x[u] = y[u] = 0.f;
                    if (t0 + u < n_qtiles) {
                        const float* p = D.qbar_part + ((int64_t)hk * D.qtiles_max + t0 + u) * D.d;
                        x[u] = p[i];
                        y[u] = p[i + D.half];
                    }
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    a += x[u];
                    b += y[u];
                }
            }
        }
        const float2 cw = D.cs_W[i];
        qb[i] = a * cw.x - b * cw.y;
        qb[i + D.half] = b * cw.x + a * cw.y;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int PER = SC_THREADS / LPU;  // units per CTA
    constexpr int UPW = 32 / LPU;          // units per warp
    const int j = split * PER + warp * UPW + lane / LPU;
    const int sub = lane % LPU;
    float acc = 0.f;
    if (j < n_mem) {
        // 16-byte vectors kept raw in registers (8 per batch), converted at use
        const T* p = MODE == OP_REPS ? (const T*)D.rep_keys + ((int64_t)hk * D.units_max + j) * D.r * D.d
                   : MODE == OP_MEANKEY ? (const T*)D.meankey + ((int64_t)hk * D.units_max + j) * D.d
                                        : nullptr;
        const float* pf = MODE == OP_REPSUM ? D.repsum + ((int64_t)hk * D.units_max + j) * D.d : nullptr;
        constexpr int N = MODE != OP_REPSUM ? Vec16<T>::N : 4;  // elements per vector
        const int total = MODE == OP_REPS ? D.r * D.d : D.d;
        for (int e0 = sub * N; e0 < total; e0 += 8 * LPU * N) {
            uint4 raw[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * LPU * N;
                if (e < total)
                    raw[u] = MODE != OP_REPSUM ? __ldg(reinterpret_cast<const uint4*>(p + e))
                                               : __ldg(reinterpret_cast<const uint4*>(pf + e));
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * LPU * N;
                if (e < total) {
                    const int i0 = e % D.d;
                    if (MODE != OP_REPSUM && sizeof(T) == 2) {
                        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const float2 f = __bfloat1622float2(h2[c]);
                            acc += f.x * qb[i0 + 2 * c] + f.y * qb[i0 + 2 * c + 1];
                        }
                    } else {
                        const float* f = reinterpret_cast<const float*>(&raw[u]);
#pragma unroll
                        for (int c = 0; c < 4; ++c) acc += f[c] * qb[i0 + c];
                    }
                }
            }
        }
    }
#pragma unroll
    for (int m = LPU / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    uint64_t cand = 0;
    if (j < n_mem && sub == 0) {
        const float sc = acc * D.inv_sqrt_d;
        D.uscore[(int64_t)hk * D.units_max + j] = sc;
        cand = make_key(sc, (uint32_t)j);
    }
    if (do_select) {  // this CTA's top-32 (composite keys, descending), then the head's selection
        __shared__ uint64_t lists[SC_WARPS][32];
        lists[warp][lane] = warp_sort_desc(cand);
#pragma unroll
        for (int stride = 1; stride < SC_WARPS; stride *= 2) {
            __syncthreads();
            if ((warp % (2 * stride)) == 0)
                lists[warp][lane] = warp_merge_desc(lists[warp][lane], lists[warp + stride][lane]);
        }
        __syncthreads();
        publish_and_select(D, hk, split, n_mem, n_split, lists, SC_WARPS);
    }
    // Without wait_first this grid may run while the preceding kernel runs (the scores do not
    // depend on it), but it must not complete before it: the kernels after rely on both.
    if (!wait_first) pdl_hold();
}

// Rotated sum of the chunk's (or the decode token's) queries of KV head hk into qb[d]:
// R(W) sum_t sum_h q_{t,h}, from the per-tile partial sums (or the single token's q heads).
template <typename T>
__device__ __forceinline__ void rotated_query_sum(const Dev& D, int hk, int n_qtiles, const T* qraw, float* qb) {
    for (int i = threadIdx.x; i < D.half; i += blockDim.x) {
        float a = 0.f, b = 0.f;
        const int n = qraw ? D.G : n_qtiles;
        for (int t0 = 0; t0 < n; t0 += 8) {
            float x[8], y[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                x[u] = y[u] = 0.f;
                if (t0 + u < n) {
                    if (qraw) {
                        x[u] = to_f(qraw[(hk * D.G + t0 + u) * D.d + i]);
                        y[u] = to_f(qraw[(hk * D.G + t0 + u) * D.d + i + D.half]);
                    } else {
                        const float* p = D.qbar_part + ((int64_t)hk * D.qtiles_max + t0 + u) * D.d;
                        x[u] = p[i];
                        y[u] = p[i + D.half];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                a += x[u];
                b += y[u];
            }
        }
        const float2 cw = D.cs_W[i];
        qb[i] = a * cw.x - b * cw.y;
        qb[i + D.half] = b * cw.x + a * cw.y;
    }
}

// Dot products of one 16-byte piece of an operand row (E = bf16 or fp32 elements) with V query values.
template <typename E>
__device__ __forceinline__ float dot16(const uint4& raw, const float* qr) {
    float a = 0.f;
    if (sizeof(E) == 2) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            a += f.x * qr[2 * e] + f.y * qr[2 * e + 1];
        }
    } else {
        const float* f = reinterpret_cast<const float*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) a += f[e] * qr[e];
    }
    return a;
}

// The scoring operand of KV head hk: representative keys, their fp32 sum, or the mean key.
template <typename T>
__device__ __forceinline__ const uint4* score_operand(const Dev& D, int mode, int hk) {
    if (mode == OP_REPS) return reinterpret_cast<const uint4*>((const T*)D.rep_keys + (int64_t)hk * D.units_max * D.r * D.d);
    if (mode == OP_REPSUM) return reinterpret_cast<const uint4*>(D.repsum + (int64_t)hk * D.units_max * D.d);
    return reinterpret_cast<const uint4*>((const T*)D.meankey + (int64_t)hk * D.units_max * D.d);
}

// One stage of the scoring pipeline: UB units' operand rows (C 16-byte chunks per lane each).
template <int UB, int C>
__device__ __forceinline__ void load_units(uint4 (&r)[UB][C], const uint4* base, int ub, int valid, int lane) {
#pragma unroll
    for (int u = 0; u < UB; ++u)
#pragma unroll
        for (int k = 0; k < C; ++k)
            r[u][k] = (ub + u < valid) ? __ldg(base + (int64_t)(ub + u) * 32 * C + k * 32 + lane) : make_uint4(0, 0, 0, 0);
}
template <typename T, int MODE, int UB, int C, int V>
__device__ __forceinline__ void dot_units(const uint4 (&r)[UB][C], const float (&qr)[C][V], float* acc) {
#pragma unroll
    for (int u = 0; u < UB; ++u) {
        float a = 0.f;
#pragma unroll
        for (int k = 0; k < C; ++k) {
            if (MODE != OP_REPSUM && sizeof(T) == 2) {
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&r[u][k]);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float2 f = __bfloat1622float2(h2[c]);
                    a += f.x * qr[k][2 * c] + f.y * qr[k][2 * c + 1];
                }
            } else {
                const float* f = reinterpret_cast<const float*>(&r[u][k]);
#pragma unroll
                for (int c = 0; c < 4; ++c) a += f[c] * qr[k][c];
            }
        }
        acc[u] = a;
    }
}

// Warp-per-32-units scoring.  Grid (n_split, Hkv), 32 * WPC threads; warp w of CTA s scores units
// [(s * WPC + w) * 32, +32).  Lane l loads 16-byte chunks l, l + 32, ... (C per unit) of every
// unit's operand -- consecutive lanes read consecutive 16 bytes, so each load instruction reads
// 512 contiguous bytes -- and multiplies them with the matching slice of the rotated query sum,
// held in registers.  The 32 partial sums of the warp's 32 units are then transposed across the
// warp (recursive halving, 31 shuffles) so that lane u ends with unit u's score.  Writes the scores
// and, with do_select, the top-k (see publish_and_select).
template <typename T, int MODE, int C>
__global__ void __launch_bounds__(256, 2) k_score_wpu(Dev D, int n_mem, int n_split, int n_qtiles, const T* qraw,
                                                      int do_select, int wait_first) {
    __shared__ float qb[128];
    __shared__ uint64_t lists[8][32];
    if (wait_first) pdl_wait();  // as in k_score_topk
    pdl_trigger();
    const int split = blockIdx.x, hk = blockIdx.y;
    constexpr int V = MODE != OP_REPSUM ? (int)(16 / sizeof(T)) : 4;  // elements per 16-byte chunk
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int u0 = (split * nw + warp) * 32;
    const uint4* base = score_operand<T>(D, MODE, hk) + (int64_t)u0 * 32 * C;
    // two register stages of UB units: the loads of one stage are in flight while the other is
    // multiplied; the first stage is issued before the query sum, which it does not need
    constexpr int UB = C >= 4 ? 2 : 4;
    constexpr int NB = 32 / UB;
    const int valid = n_mem - u0;
    uint4 ra[UB][C], rb[UB][C];
    load_units<UB, C>(ra, base, 0, valid, lane);
    rotated_query_sum<T>(D, hk, n_qtiles, qraw, qb);
    __syncthreads();
    float qr[C][V];
#pragma unroll
    for (int k = 0; k < C; ++k) {
        const int i0 = ((k * 32 + lane) * V) % D.d;
#pragma unroll
        for (int v = 0; v < V; ++v) qr[k][v] = qb[i0 + v];
    }
    float acc[32];
#pragma unroll
    for (int bi = 0; bi < NB; bi += 2) {
        if (bi + 1 < NB) load_units<UB, C>(rb, base, (bi + 1) * UB, valid, lane);
        dot_units<T, MODE, UB, C, V>(ra, qr, acc + bi * UB);
        if (bi + 2 < NB) load_units<UB, C>(ra, base, (bi + 2) * UB, valid, lane);
        if (bi + 1 < NB) dot_units<T, MODE, UB, C, V>(rb, qr, acc + (bi + 1) * UB);
    }
    // transpose-reduce: afterwards acc[0] of lane l is the full dot product of unit u0 + l
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float send = upper ? acc[i] : acc[i + m];
            const float keep = upper ? acc[i + m] : acc[i];
            acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    const int j = u0 + lane;
    uint64_t cand = 0;
    if (j < n_mem) {
        const float sc = acc[0] * D.inv_sqrt_d;
        D.uscore[(int64_t)hk * D.units_max + j] = sc;
        cand = make_key(sc, (uint32_t)j);
    }
    if (do_select) {
        lists[warp][lane] = warp_sort_desc(cand);
        for (int stride = 1; stride < nw; stride *= 2) {
            __syncthreads();
            if ((warp % (2 * stride)) == 0 && warp + stride < nw)
                lists[warp][lane] = warp_merge_desc(lists[warp][lane], lists[warp + stride][lane]);
        }
        __syncthreads();
        publish_and_select(D, hk, split, n_mem, n_split, lists, nw);
    }
    if (!wait_first) pdl_hold();  // this grid must not complete before its predecessor (see k_score_topk)
}

// The CTA's top-32 candidate list from its warps' lists, then the head's selection (last CTA).
__device__ __forceinline__ void cta_lists_and_select(const Dev& D, int hk, int split, int n_mem, int n_split,
                                                     uint64_t (*lists)[32], uint64_t list) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    lists[warp][lane] = list;
    for (int stride = 1; stride < nw; stride *= 2) {
        __syncthreads();
        if ((warp % (2 * stride)) == 0 && warp + stride < nw)
            lists[warp][lane] = warp_merge_desc(lists[warp][lane], lists[warp + stride][lane]);
    }
    __syncthreads();
    publish_and_select(D, hk, split, n_mem, n_split, lists, nw);
}

// Streaming scoring for one query token (decode), the bandwidth-bound read of the whole scoring
// pool.  Grid (n_split, Hkv), 256 threads; CTA s scores units [s * upc, s * upc + upc) of KV head
// hk; every unit's operand row is 32 * CPL 16-byte pieces of E elements.  Each warp takes UB
// consecutive units per step: lane l loads the pieces l, l + 32, ... (CPL per unit) of every
// unit's row -- consecutive lanes on consecutive 16 bytes, so each load instruction reads 512
// contiguous bytes -- and multiplies them with its slice of the rotated query sum, held in
// registers (every piece of a lane covers the same dims, since 32 pieces span a whole number of
// d-element rows).  The UB partial sums are transposed across the warp (log2(UB) halving steps)
// and then summed over the 32/UB lanes that share a unit, which leaves the unit's score in each of
// those lanes.  The warp keeps a running top-32 list (one candidate per lane every 32/UB steps);
// the CTA's list and the head's selection follow as in k_score_wpu.
template <typename T, typename E, int CPL, int UB>
__global__ void __launch_bounds__(256) k_score_dec(Dev D, int mode, int n_mem, int upc, int n_split, const T* qraw,
                                                   int wait_first) {
    __shared__ float qb[128];
    __shared__ uint64_t lists[8][32];
    if (wait_first) pdl_wait();  // new representatives come from the kernels before
    pdl_trigger();
    constexpr int V = 16 / sizeof(E);  // elements per 16-byte piece
    constexpr int GRP = 32 / UB;       // lanes that end with one unit's score
    const int split = blockIdx.x, hk = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int u_begin = split * upc, u_end = min(n_mem, u_begin + upc);
    const uint4* base = score_operand<T>(D, mode, hk);
    // the first step's rows are requested before the query sum, which they do not need
    uint4 raw[UB][CPL];
    auto load = [&](int u0) {
#pragma unroll
        for (int u = 0; u < UB; ++u)
#pragma unroll
            for (int c = 0; c < CPL; ++c)
                raw[u][c] = u0 + u < u_end ? __ldg(base + (int64_t)(u0 + u) * 32 * CPL + c * 32 + lane)
                                           : make_uint4(0, 0, 0, 0);
    };
    load(u_begin + warp * UB);
    rotated_query_sum<T>(D, hk, 1, qraw, qb);
    __syncthreads();
    float qr[V];
    {
        const int i0 = (lane * V) % D.d;
#pragma unroll
        for (int v = 0; v < V; ++v) qr[v] = qb[i0 + v];
    }
    uint64_t list = 0, cand = 0;
    int it = 0;
    for (int u0 = u_begin + warp * UB; u0 < u_end; u0 += nw * UB, ++it) {  // warp-uniform
        if (it > 0) load(u0);
        float acc[UB];
#pragma unroll
        for (int u = 0; u < UB; ++u) {
            float a = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) a += dot16<E>(raw[u][c], qr);
            acc[u] = a;
        }
        // transpose: after the halving steps (masks 16 .. GRP) lane l holds unit l / GRP's partial,
        // then the butterfly over the GRP lanes of a unit completes it in each of them
#pragma unroll
        for (int m = 16, nv = UB; m >= 1; m >>= 1) {
            if (nv > 1) {
                const bool upper = (lane & m) != 0;
#pragma unroll
                for (int i = 0; i < UB / 2; ++i) {
                    if (i < nv / 2) {
                        const float send = upper ? acc[i] : acc[i + nv / 2];
                        const float keep = upper ? acc[i + nv / 2] : acc[i];
                        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                    }
                }
                nv >>= 1;
            } else {
                acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], m);
            }
        }
        const int j = u0 + lane / GRP;
        const float sc = acc[0] * D.inv_sqrt_d;
        if (j < u_end) {
            if ((lane % GRP) == 0) D.uscore[(int64_t)hk * D.units_max + j] = sc;
            if ((lane % GRP) == (it % GRP)) cand = make_key(sc, (uint32_t)j);
        }
        if ((it % GRP) == GRP - 1) {
            list = warp_topk_insert(list, cand);
            cand = 0;
        }
    }
    if (__any_sync(0xffffffffu, cand != 0)) list = warp_topk_insert(list, cand);
    cta_lists_and_select(D, hk, split, n_mem, n_split, lists, list);
    if (!wait_first) pdl_hold();  // this grid must not complete before its predecessor (see k_score_topk)
}

// The same for operand rows of 256 bytes (16 pieces: one bf16 mean key of d = 128, or an fp32 row of
// d = 64): each load instruction covers two units (lane l: unit l / 16, piece l % 16), four
// instructions per step, so a warp scores 8 units per step.  The four partials of a lane are
// transposed within its half-warp (masks 8 and 4) and summed over the 4 lanes left per unit
// (masks 2 and 1): lanes l with the same l / 4 then hold the score of unit u0 + 2 ((l / 4) % 4) + l / 16.
template <typename T, typename E>
__global__ void __launch_bounds__(256) k_score_dec_half(Dev D, int mode, int n_mem, int upc, int n_split,
                                                        const T* qraw, int wait_first) {
    __shared__ float qb[128];
    __shared__ uint64_t lists[8][32];
    if (wait_first) pdl_wait();
    pdl_trigger();
    constexpr int V = 16 / sizeof(E);
    const int split = blockIdx.x, hk = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int u_begin = split * upc, u_end = min(n_mem, u_begin + upc);
    const uint4* base = score_operand<T>(D, mode, hk);
    const int half = lane >> 4, piece = lane & 15;
    const int slot = (lane >> 2) & 3;
    const int stride = nw * 8;
    // two steps' rows in flight per warp (ping-pong buffers), the first two requested before the
    // query sum, which they do not need
    uint4 ra[4], rb[4];
    auto load = [&](uint4 (&raw)[4], int u0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int u = u0 + 2 * i + half;
            raw[i] = u < u_end ? __ldg(base + (int64_t)u * 16 + piece) : make_uint4(0, 0, 0, 0);
        }
    };
    int u0 = u_begin + warp * 8;
    load(ra, u0);
    load(rb, u0 + stride);
    rotated_query_sum<T>(D, hk, 1, qraw, qb);
    __syncthreads();
    float qr[V];
    {
        const int i0 = ((lane & 15) * V) % D.d;
#pragma unroll
        for (int v = 0; v < V; ++v) qr[v] = qb[i0 + v];
    }
    uint64_t list = 0, cand = 0;
    int it = 0;
    auto step = [&](const uint4 (&raw)[4], int s0) {  // one step: 8 units from s0 (warp-uniform)
        float acc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] = dot16<E>(raw[i], qr);
#pragma unroll
        for (int m = 8, nv = 4; m >= 4; m >>= 1, nv >>= 1) {
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
        acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 2);
        acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
        const int j = s0 + 2 * slot + half;
        const float sc = acc[0] * D.inv_sqrt_d;
        if (j < u_end) {
            if ((lane & 3) == 0) D.uscore[(int64_t)hk * D.units_max + j] = sc;
            if ((lane & 3) == (it & 3)) cand = make_key(sc, (uint32_t)j);
        }
        if ((it & 3) == 3) {
            list = warp_topk_insert(list, cand);
            cand = 0;
        }
        ++it;
    };
    for (; u0 < u_end; u0 += 2 * stride) {  // warp-uniform
        step(ra, u0);
        load(ra, u0 + 2 * stride);
        if (u0 + stride < u_end) {
            step(rb, u0 + stride);
            load(rb, u0 + 3 * stride);
        }
    }
    if (__any_sync(0xffffffffu, cand != 0)) list = warp_topk_insert(list, cand);
    cta_lists_and_select(D, hk, split, n_mem, n_split, lists, list);
    if (!wait_first) pdl_hold();
}

// Selection for top_k > 32: one CTA per kv head sorts every unit's composite key in shared
// memory (bitonic network, descending), keeps the first min(k, n_mem) and sorts their ids.
__global__ void __launch_bounds__(1024) k_topk_sort(Dev D, int n_mem, int p2) {
    extern __shared__ uint64_t keys[];
    const int hk = blockIdx.x;
    for (int i = threadIdx.x; i < p2; i += blockDim.x)
        keys[i] = i < n_mem ? make_key(D.uscore[(int64_t)hk * D.units_max + i], (uint32_t)i) : 0ull;
    __syncthreads();
    for (int k = 2; k <= p2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < p2; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const bool desc = (i & k) == 0;
                    const uint64_t a = keys[i], b = keys[ixj];
                    if ((a < b) == desc) {
                        keys[i] = b;
                        keys[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    const int kk = min(D.topk, n_mem);
    // ids of the kept units, re-keyed so that a descending sort gives ascending ids
    for (int i = threadIdx.x; i < p2; i += blockDim.x)
        keys[i] = i < kk ? (uint64_t)(0xffffffffu - key_index(keys[i])) : 0ull;
    __syncthreads();
    for (int k = 2; k <= p2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < p2; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const bool desc = (i & k) == 0;
                    const uint64_t a = keys[i], b = keys[ixj];
                    if ((a < b) == desc) {
                        keys[i] = b;
                        keys[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = threadIdx.x; i < D.topk; i += blockDim.x) {
        int o = -1;
        if (i < kk) {
            o = (int)(0xffffffffu - (uint32_t)keys[i]);
            if (o < 0 || o >= n_mem) {
                set_err(D, ERR_SEL_RANGE);
                o = 0;
            }
        }
        D.sel[hk * D.topk + i] = o;
    }
}

// ---- launchers ----------------------------------------------------------------------------

template <typename T>
cudaError_t launch_prep(const Dev& D, const void* q, int64_t c0, int n, int par, cudaStream_t st, bool pdl) {
    if (n <= 0) return cudaSuccess;
    const int tiles = (n + D.qt - 1) / D.qt;
    const int threads = 256;
    const int nv = D.half / (16 / (int)sizeof(T));
    const size_t smem = (threads / nv) * D.d * sizeof(float) + (size_t)D.qt * D.half * sizeof(float2);
    static std::atomic<unsigned long long> attr_done{0};  // up to 80 KB (one q head per KV head: 128 queries a tile)
    cudaError_t e = smem_limit_once(k_prep<T>, 96 * 1024, attr_done);
    if (e != cudaSuccess) return e;
    return launch_k(k_prep<T>, dim3(tiles, D.Hkv), dim3(threads), smem, st, pdl, D, (const T*)q, c0, n, par);
}

// Lanes per unit: the fewest that still give at least one CTA per SM (148).
int score_lanes_per_unit(int n_mem, int Hkv) {
    int lpu = 1;
    while (lpu < 32 && (int64_t)((n_mem + SC_THREADS / lpu - 1) / (SC_THREADS / lpu)) * Hkv < 148) lpu *= 2;
    return lpu;
}

template <typename T, int MODE, int LPU>
static cudaError_t launch_score1(const Dev& D, dim3 grid, int n_mem, int n_split, int n_qtiles, const T* qraw,
                                 int do_select, cudaStream_t st, bool pdl, int wait_first) {
    return launch_k(k_score_topk<T, MODE, LPU>, grid, dim3(SC_THREADS), 0, st, pdl, D, n_mem, n_split, n_qtiles, qraw,
                    do_select, wait_first);
}

template <typename T, int MODE>
static cudaError_t launch_score(const Dev& D, int lpu, dim3 grid, int n_mem, int n_split, int n_qtiles, const T* qraw,
                                int do_select, cudaStream_t st, bool pdl, int wf) {
    switch (lpu) {
        case 1: return launch_score1<T, MODE, 1>(D, grid, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
        case 2: return launch_score1<T, MODE, 2>(D, grid, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
        case 4: return launch_score1<T, MODE, 4>(D, grid, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
        case 8: return launch_score1<T, MODE, 8>(D, grid, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
        case 16: return launch_score1<T, MODE, 16>(D, grid, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
        default: return launch_score1<T, MODE, 32>(D, grid, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
    }
}

template <typename T, int MODE, int C>
static cudaError_t launch_wpu1(const Dev& D, dim3 grid, int threads, int n_mem, int n_split, int n_qtiles,
                               const T* qraw, int do_select, cudaStream_t st, bool pdl, int wait_first) {
    return launch_k(k_score_wpu<T, MODE, C>, grid, dim3(threads), 0, st, pdl, D, n_mem, n_split, n_qtiles, qraw,
                    do_select, wait_first);
}

template <typename T, int MODE>
static cudaError_t launch_wpu_c(const Dev& D, int C, dim3 grid, int threads, int n_mem, int n_split, int n_qtiles,
                                const T* qraw, int do_select, cudaStream_t st, bool pdl, int wf) {
    if (C == 1) return launch_wpu1<T, MODE, 1>(D, grid, threads, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
    if (C == 2) return launch_wpu1<T, MODE, 2>(D, grid, threads, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
    return launch_wpu1<T, MODE, 4>(D, grid, threads, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
}

template <typename T>
static cudaError_t launch_wpu(const Dev& D, int mode, int C, dim3 grid, int threads, int n_mem, int n_split,
                              int n_qtiles, const T* qraw, int do_select, cudaStream_t st, bool pdl,
                              int wf) {
    if (mode == OP_REPS) return launch_wpu_c<T, OP_REPS>(D, C, grid, threads, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
    if (mode == OP_REPSUM)
        return launch_wpu_c<T, OP_REPSUM>(D, C, grid, threads, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
    return launch_wpu_c<T, OP_MEANKEY>(D, C, grid, threads, n_mem, n_split, n_qtiles, qraw, do_select, st, pdl, wf);
}

// Decode scoring kernels by operand row size: 256 bytes (half-warp rows) or 512 / 1024 bytes.
template <typename T, typename E>
static cudaError_t launch_dec(const Dev& D, int mode, int row_bytes, dim3 grid, int n_mem, int upc, int n_split,
                              const T* qraw, cudaStream_t st, bool pdl, int wf) {
    if (row_bytes == 256)
        return launch_k(k_score_dec_half<T, E>, grid, dim3(256), 0, st, pdl, D, mode, n_mem, upc, n_split, qraw, wf);
    if (row_bytes == 512)
        return launch_k(k_score_dec<T, E, 1, 4>, grid, dim3(256), 0, st, pdl, D, mode, n_mem, upc, n_split, qraw, wf);
    return launch_k(k_score_dec<T, E, 2, 4>, grid, dim3(256), 0, st, pdl, D, mode, n_mem, upc, n_split, qraw, wf);
}

template <typename T>
cudaError_t launch_select(const Dev& D, int score_mode, int n_mem, int n_qtiles, const void* qraw, cudaStream_t st,
                          int* launches, bool pdl, bool wait_first) {
    *launches = 0;
    const int wf = wait_first ? 1 : 0;
    if (n_mem <= 0 || D.topk <= 0) return cudaSuccess;
    const int fast = D.topk <= 32;
    // warp-per-32-units scoring when a unit's operand is a whole number of 512-byte rows
    const int unit_bytes = score_mode == OP_REPS ? D.r * D.d * (int)sizeof(T)
                         : score_mode == OP_REPSUM ? D.d * 4 : D.d * (int)sizeof(T);
    const int C = unit_bytes % 512 == 0 ? unit_bytes / 512 : 0;
    int n_split;
    cudaError_t err;
    if (qraw != nullptr && fast && (unit_bytes == 256 || unit_bytes == 512 || unit_bytes == 1024)) {
        // one query token: stream the pool with at most two CTAs of 256 threads per SM, so that the whole
        // grid is resident beside the decode step's sink and window tiles (they share the SMs)
        const int64_t want = ((int64_t)n_mem * D.Hkv + 2 * 148 - 1) / (2 * 148);
        int upc = (int)std::max<int64_t>(32, (want + 31) / 32 * 32);
        n_split = (n_mem + upc - 1) / upc;
        if (n_split > D.score_splits_max) return cudaErrorInvalidValue;
        const dim3 grid(n_split, D.Hkv);
        err = score_mode == OP_REPSUM
                  ? launch_dec<T, float>(D, score_mode, unit_bytes, grid, n_mem, upc, n_split, (const T*)qraw, st, pdl, wf)
                  : launch_dec<T, T>(D, score_mode, unit_bytes, grid, n_mem, upc, n_split, (const T*)qraw, st, pdl, wf);
    } else if (C == 1 || C == 2 || C == 4) {
        // warps per CTA (4..8, each warp scores 32 units): the one whose CTA count fills the
        // waves of 2 CTAs per SM on 148 SMs best, the larger on ties (fewer lists to merge); not
        // fewer than 4 warps, as the last CTA of a head merges the lists of the others
        int wpc = 8;
        double best = -1.0;
        for (int w = 8; w >= 4; --w) {
            const int64_t ctas = (int64_t)((n_mem + 32 * w - 1) / (32 * w)) * D.Hkv;
            const int64_t waves = (ctas + 295) / 296;
            const double eff = (double)ctas / (double)(waves * 296);
            if (eff > best + 1e-9) {
                best = eff;
                wpc = w;
            }
        }
        n_split = (n_mem + 32 * wpc - 1) / (32 * wpc);
        if (n_split > D.score_splits_max) return cudaErrorInvalidValue;
        err = launch_wpu<T>(D, score_mode, C, dim3(n_split, D.Hkv), 32 * wpc, n_mem, n_split, n_qtiles,
                            (const T*)qraw, fast, st, pdl, wf);
    } else {
        const int lpu = score_lanes_per_unit(n_mem, D.Hkv);
        const int per = SC_THREADS / lpu;
        n_split = (n_mem + per - 1) / per;
        if (n_split > D.score_splits_max) return cudaErrorInvalidValue;
        dim3 grid(n_split, D.Hkv);
        err = score_mode == OP_REPS
                  ? launch_score<T, OP_REPS>(D, lpu, grid, n_mem, n_split, n_qtiles, (const T*)qraw, fast, st, pdl, wf)
              : score_mode == OP_REPSUM
                  ? launch_score<T, OP_REPSUM>(D, lpu, grid, n_mem, n_split, n_qtiles, (const T*)qraw, fast, st, pdl, wf)
                  : launch_score<T, OP_MEANKEY>(D, lpu, grid, n_mem, n_split, n_qtiles, (const T*)qraw, fast, st, pdl, wf);
    }
    ++*launches;
    if (err != cudaSuccess) return err;
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (fast) return cudaSuccess;  // the scoring kernel's last CTA per head selected already
    int p2 = 1;
    while (p2 < n_mem) p2 <<= 1;  // n_mem <= 16384 (checked at create when top_k > 32)
    const size_t smem = (size_t)p2 * sizeof(uint64_t);
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(k_topk_sort, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    k_topk_sort<<<D.Hkv, 1024, smem, st>>>(D, n_mem, p2);
    ++*launches;
    return cudaGetLastError();
}

template cudaError_t launch_prep<float>(const Dev&, const void*, int64_t, int, int, cudaStream_t, bool);
template cudaError_t launch_prep<__nv_bfloat16>(const Dev&, const void*, int64_t, int, int, cudaStream_t, bool);
template cudaError_t launch_select<float>(const Dev&, int, int, int, const void*, cudaStream_t, int*, bool, bool);
template cudaError_t launch_select<__nv_bfloat16>(const Dev&, int, int, int, const void*, cudaStream_t, int*, bool,
                                                  bool);

}  // namespace infllm
