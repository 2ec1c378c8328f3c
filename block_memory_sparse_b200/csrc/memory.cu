// Context-memory kernels: token store (append), query block sums, representative tokens.
//
// Method: "InfLLM Guide: Training-Free Long-Context Memory Units", "Core Innovation 1:
// Structured Context Partitioning" (sinks / units / window); representative tokens chosen
// by attention scores, "InfLLM: Training-Free Long-Context Extrapolation ..." (atlas.scime.ai
// summary), "Approach".
#include "common.cuh"
#include "kernels.h"

namespace infllm {

// One CTA per appended token: (cos, sin)(t * theta_i) from the fp64 digit tables once per
// token (absolute positions reach ~1e6 rad, beyond fp32 angle accuracy), then the three stores.
template <typename T>
__global__ void k_append(Dev D, const T* __restrict__ k, const T* __restrict__ v, int64_t c0) {
    extern __shared__ float2 cs_sh[];
    pdl_trigger();  // early kernel: reads only the inputs and constant tables
    const int tl = blockIdx.x;
    const int64_t t = c0 + tl;
    for (int i = threadIdx.x; i < D.half; i += blockDim.x) {
        const float2 cs = cs_abs(D.cs_abs3, D.half, t, i);
        cs_sh[i] = cs;
        D.cs_chunk[(int64_t)tl * D.half + i] = cs;
    }
    __syncthreads();
    T* Kraw = (T*)D.Kraw;
    T* Krot = (T*)D.Krot;
    T* V = (T*)D.V;
    for (int idx = threadIdx.x; idx < D.Hkv * D.half; idx += blockDim.x) {
        const int hk = idx / D.half, i = idx % D.half;
        const T* ks = k + ((int64_t)tl * D.Hkv + hk) * D.d;
        const T* vs = v + ((int64_t)tl * D.Hkv + hk) * D.d;
        const int64_t dst = ((int64_t)hk * D.T_max + t) * D.d;
        const T a = ks[i], b = ks[i + D.half];
        Kraw[dst + i] = a;
        Kraw[dst + i + D.half] = b;
        const float x1 = to_f(a), x2 = to_f(b);
        const float2 cs = cs_sh[i];
        Krot[dst + i] = from_f<T>(x1 * cs.x - x2 * cs.y);
        Krot[dst + i + D.half] = from_f<T>(x2 * cs.x + x1 * cs.y);
        V[dst + i] = vs[i];
        V[dst + i + D.half] = vs[i + D.half];
    }
    pdl_hold();
}

// Y[b][hk] += sum over the chunk's tokens t in block b of sum_{h in group} R(t - s_b) q_{t,h}.
// Grid (blocks touched, Hkv), 1024 threads: thread = (octet of pairs, token), so every load of
// the block is issued at once (heads in batches of four).  Fixed-order reduction (warp shuffles,
// then warps in order), so results do not depend on scheduling.
template <typename T>
__global__ void __launch_bounds__(1024) k_ysum(Dev D, const T* __restrict__ q, int64_t c0, int n, int64_t b0) {
    extern __shared__ float red[];  // [warps][d]
    pdl_trigger();  // early kernel: the blocks it updates hold no position a running kernel reads
    constexpr int V = 16 / sizeof(T);
    constexpr int HB = 4;
    const int64_t b = b0 + blockIdx.x;
    const int hk = blockIdx.y;
    const int64_t sb = (int64_t)D.S + b * D.gblk;
    const int64_t lo = sb > c0 ? sb : c0;
    const int64_t hi = (sb + D.gblk) < (c0 + n) ? (sb + D.gblk) : (c0 + n);
    const int nv = D.half / V;  // octets per token (power of two, <= 8)
    const int o = threadIdx.x % nv, tg = threadIdx.x / nv, ntg = blockDim.x / nv;
    const int i0 = o * V;
    float a1[V], a2[V];
#pragma unroll
    for (int e = 0; e < V; ++e) a1[e] = a2[e] = 0.f;
    for (int64_t t = lo + tg; t < hi; t += ntg) {
        float x1[V], x2[V];
#pragma unroll
        for (int e = 0; e < V; ++e) x1[e] = x2[e] = 0.f;
        const T* qr = q + ((t - c0) * D.Hq + (int64_t)hk * D.G) * D.d;
        for (int h0 = 0; h0 < D.G; h0 += HB) {
            union { uint4 u; T v[V]; } r1[HB], r2[HB];
#pragma unroll
            for (int hh = 0; hh < HB; ++hh) {
                r1[hh].u = r2[hh].u = make_uint4(0, 0, 0, 0);
                if (h0 + hh < D.G) {
                    r1[hh].u = *reinterpret_cast<const uint4*>(qr + (h0 + hh) * D.d + i0);
                    r2[hh].u = *reinterpret_cast<const uint4*>(qr + (h0 + hh) * D.d + i0 + D.half);
                }
            }
#pragma unroll
            for (int hh = 0; hh < HB; ++hh)
#pragma unroll
                for (int e = 0; e < V; ++e) {  // the rotation is linear: sum the group's heads first
                    x1[e] += to_f(r1[hh].v[e]);
                    x2[e] += to_f(r2[hh].v[e]);
                }
        }
        const float2* cs = D.cs_rel + (t - sb) * D.half + i0;
#pragma unroll
        for (int e = 0; e < V; ++e) {
            const float2 c = cs[e];
            a1[e] += x1[e] * c.x - x2[e] * c.y;
            a2[e] += x2[e] * c.x + x1[e] * c.y;
        }
    }
    // lanes holding the same octet of different tokens: xor over the token bits of the lane
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        if (m < nv) break;
#pragma unroll
        for (int e = 0; e < V; ++e) {
            a1[e] += __shfl_xor_sync(0xffffffffu, a1[e], m);
            a2[e] += __shfl_xor_sync(0xffffffffu, a2[e], m);
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane < nv) {
        float* r = red + warp * D.d;
#pragma unroll
        for (int e = 0; e < V; ++e) {
            r[i0 + e] = a1[e];
            r[i0 + e + D.half] = a2[e];
        }
    }
    __syncthreads();
    const int nw = blockDim.x >> 5;
    for (int j = threadIdx.x; j < D.d; j += blockDim.x) {
        float acc = 0.f;
        for (int w = 0; w < nw; ++w) acc += red[w * D.d + j];
        D.Y[(b * D.Hkv + hk) * D.d + j] += acc;
    }
    pdl_hold();
}

// Representatives of units [j0, j0 + gridDim.x) for kv head blockIdx.y, 256 threads.  Also the
// unit's mean key (the mean-of-keys representation of "InfLLM: Training-Free Long-Context
// Extrapolation ..." (research-map summary), "Measured effects", ablation row on mean key vectors).
//   Qt = sum_{i=e}^{e+W-1} sum_h R(i - e) q_{i,h}  (from the block sums, e = unit end)
//   rho_m = <R(e - m) Qt, k_m> / sqrt(d)  ==  sum_i sum_h <R(i) q_{i,h}, R(m) k_m> / sqrt(d)
// then the top r by (rho desc, m asc), stored ascending, plus the raw rep keys and their sum.
template <typename T>
__global__ void __launch_bounds__(256) k_reps(Dev D, int64_t j0) {
    extern __shared__ float sm[];
    float* Qt = sm;                 // [d]
    float* rho = sm + D.d;          // [U]
    float* part = rho + D.U;        // [4][d] partial window sums
    __shared__ int ids[32];
    pdl_trigger();  // early kernel: reads block sums and keys of positions before the chunk
    const int64_t j = j0 + blockIdx.x;
    const int hk = blockIdx.y;
    const int64_t e = (int64_t)D.S + (j + 1) * D.U;
    const int64_t m0 = e - D.U;
    const int64_t be = (e - D.S) / D.gblk;
    const int nb = D.W / D.gblk;
    {
        const int i = threadIdx.x % D.half, pg = threadIdx.x / D.half, npg = blockDim.x / D.half;
        float a1 = 0.f, a2 = 0.f;
        constexpr int PB = 8;  // window blocks per load batch
        for (int p0 = pg; p0 < nb; p0 += npg * PB) {
            float y1[PB], y2[PB];
            float2 cs[PB];
#pragma unroll
            for (int u = 0; u < PB; ++u) {
                const int p = p0 + u * npg;
                y1[u] = y2[u] = 0.f;
                cs[u] = make_float2(0.f, 0.f);
                if (p < nb) {
                    const float* y = D.Y + ((be + p) * D.Hkv + hk) * D.d;
                    y1[u] = y[i];
                    y2[u] = y[i + D.half];
                    cs[u] = D.cs_rel[(int64_t)p * D.gblk * D.half + i];
                }
            }
#pragma unroll
            for (int u = 0; u < PB; ++u) {
                a1 += y1[u] * cs[u].x - y2[u] * cs[u].y;
                a2 += y2[u] * cs[u].x + y1[u] * cs[u].y;
            }
        }
        part[pg * D.d + i] = a1;
        part[pg * D.d + i + D.half] = a2;
        __syncthreads();
        for (int x = threadIdx.x; x < D.d; x += blockDim.x) {
            float acc = 0.f;
            for (int g = 0; g < npg; ++g) acc += part[g * D.d + x];
            Qt[x] = acc;
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const T* K = (const T*)D.Kraw + ((int64_t)hk * D.T_max + m0) * D.d;
    constexpr int UNR = 4;
    for (int mb = warp * UNR; mb < D.U; mb += nw * UNR) {
        float acc[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) acc[u] = 0.f;
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {  // half <= 64: pairs lane and lane + 32
            const int i = lane + 32 * ii;
            if (i < D.half) {
                const float q1 = Qt[i], q2 = Qt[i + D.half];
                float k1[UNR], k2[UNR];
                float2 cs[UNR];
#pragma unroll
                for (int u = 0; u < UNR; ++u) {
                    const int m = mb + u < D.U ? mb + u : D.U - 1;
                    cs[u] = D.cs_rel[(int64_t)(D.U - m) * D.half + i];  // distance e - (m0 + m)
                    k1[u] = to_f(K[(int64_t)m * D.d + i]);
                    k2[u] = to_f(K[(int64_t)m * D.d + i + D.half]);
                }
#pragma unroll
                for (int u = 0; u < UNR; ++u) {
                    const float r1 = q1 * cs[u].x - q2 * cs[u].y, r2 = q2 * cs[u].x + q1 * cs[u].y;
                    acc[u] += r1 * k1[u] + r2 * k2[u];
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const float v = warp_sum(acc[u]);
            if (lane == 0 && mb + u < D.U) rho[mb + u] = v * D.inv_sqrt_d;
        }
    }
    __syncthreads();
    if (warp == 0) {
        uint64_t below = ~0ull;  // keys are unique: extract the r largest in descending order
        int mine = 0x7fffffff;
        for (int qq = 0; qq < D.r; ++qq) {
            uint64_t best = 0;
            for (int m = lane; m < D.U; m += 32) {
                const uint64_t key = make_key(rho[m], (uint32_t)m);
                if (key < below && key > best) best = key;
            }
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) {
                const uint64_t o = shfl_xor64(best, s);
                best = o > best ? o : best;
            }
            below = best;
            if (lane == qq) mine = (int)key_index(best);
        }
        // ascending ids: sort keys ~id descending
        uint64_t sk = (lane < D.r) ? (uint64_t)(0xffffffffu - (uint32_t)mine) : 0ull;
        sk = warp_sort_desc(sk);
        if (lane < D.r) {
            int id = (int)(0xffffffffu - (uint32_t)sk);
            if (id < 0 || id >= D.U) {
                set_err(D, ERR_REP_RANGE);
                id = 0;
            }
            ids[lane] = id;
        }
    }
    __syncthreads();
    int32_t* rid = D.rep_ids + ((int64_t)hk * D.units_max + j) * D.r;
    if (threadIdx.x < D.r) rid[threadIdx.x] = ids[threadIdx.x];
    T* rk = (T*)D.rep_keys + ((int64_t)hk * D.units_max + j) * D.r * D.d;
    float* rs = D.repsum + ((int64_t)hk * D.units_max + j) * D.d;
    for (int i = threadIdx.x; i < D.d; i += blockDim.x) {
        float s = 0.f;
        for (int q0 = 0; q0 < D.r; q0 += 8) {
            T x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (q0 + u < D.r) x[u] = K[(int64_t)ids[q0 + u] * D.d + i];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (q0 + u < D.r) {
                    rk[(int64_t)(q0 + u) * D.d + i] = x[u];
                    s += to_f(x[u]);
                }
        }
        rs[i] = s;
    }
    // the unit's mean key: the sum of its U keys in fp64 (exact for bf16 keys), divided by U, rounded
    // once to the context dtype
    T* mk = (T*)D.meankey + ((int64_t)hk * D.units_max + j) * D.d;
    for (int i = threadIdx.x; i < D.d; i += blockDim.x) {
        double s = 0.0;
        for (int m0b = 0; m0b < D.U; m0b += 8) {
            T x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = m0b + u < D.U ? K[(int64_t)(m0b + u) * D.d + i] : from_f<T>(0.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) s += (double)to_f(x[u]);
        }
        mk[i] = from_d<T>(s / (double)D.U);
    }
    pdl_hold();
}

// ---- launchers ----------------------------------------------------------------------------

template <typename T>
cudaError_t launch_append(const Dev& D, const void* k, const void* v, int64_t c0, int n, cudaStream_t st, bool pdl) {
    if (n <= 0) return cudaSuccess;
    return launch_k(k_append<T>, dim3(n), dim3(256), D.half * sizeof(float2), st, pdl, D, (const T*)k, (const T*)v, c0);
}

template <typename T>
cudaError_t launch_ysum(const Dev& D, const void* q, int64_t c0, int n, cudaStream_t st, int* launches, bool pdl) {
    const int64_t lo = c0 > D.S ? c0 : (int64_t)D.S;
    const int64_t hi = c0 + n;
    if (hi <= lo) return cudaSuccess;
    const int64_t b0 = (lo - D.S) / D.gblk, b1 = (hi - 1 - D.S) / D.gblk;
    const int threads = 1024;  // (half / V) octets x tokens
    dim3 grid((unsigned)(b1 - b0 + 1), D.Hkv);
    ++*launches;
    return launch_k(k_ysum<T>, grid, dim3(threads), (threads / 32) * D.d * sizeof(float), st, pdl, D, (const T*)q, c0,
                    n, b0);
}

template <typename T>
cudaError_t launch_reps(const Dev& D, int64_t j0, int64_t j1, cudaStream_t st, bool pdl) {
    if (j1 <= j0) return cudaSuccess;
    dim3 grid((unsigned)(j1 - j0), D.Hkv);
    return launch_k(k_reps<T>, grid, dim3(256), (D.d + D.U + (256 / D.half) * D.d) * sizeof(float), st, pdl, D, j0);
}

template cudaError_t launch_append<float>(const Dev&, const void*, const void*, int64_t, int, cudaStream_t, bool);
template cudaError_t launch_append<__nv_bfloat16>(const Dev&, const void*, const void*, int64_t, int, cudaStream_t,
                                                  bool);
template cudaError_t launch_ysum<float>(const Dev&, const void*, int64_t, int, cudaStream_t, int*, bool);
template cudaError_t launch_ysum<__nv_bfloat16>(const Dev&, const void*, int64_t, int, cudaStream_t, int*, bool);
template cudaError_t launch_reps<float>(const Dev&, int64_t, int64_t, cudaStream_t, bool);
template cudaError_t launch_reps<__nv_bfloat16>(const Dev&, int64_t, int64_t, cudaStream_t, bool);

}  // namespace infllm
