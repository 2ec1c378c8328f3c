// Context-memory kernels: token store (append), query block sums, representative tokens.
//
// Method: "InfLLM Guide: Training-Free Long-Context Memory Units", "Core Innovation 1:
// Structured Context Partitioning" (sinks / units / window); representative tokens chosen
// by attention scores, "InfLLM: Training-Free Long-Context Extrapolation ..." (atlas.scime.ai
// summary), "Approach".
#include "common.cuh"
#include "kernels.h"

namespace infllm {

// One CTA per appended token: (cos, sin)(t * theta_i) in fp64 once per token (absolute
// positions reach ~1e6 rad, beyond fp32 angle accuracy), then the three stores.
template <typename T>
__global__ void k_append(Dev D, const T* __restrict__ k, const T* __restrict__ v, int64_t c0) {
    extern __shared__ float2 cs_sh[];
    const int tl = blockIdx.x;
    const int64_t t = c0 + tl;
    for (int i = threadIdx.x; i < D.half; i += blockDim.x) {
        double s, c;
        sincos((double)t * D.inv_freq[i], &s, &c);
        float2 cs = make_float2((float)c, (float)s);
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
}

// Y[b][hk] += sum over the chunk's tokens t in block b of sum_{h in group} R(t - s_b) q_{t,h}.
// Grid (blocks touched, Hkv), 512 threads: thread = (pair couple pc: pairs 2pc, 2pc+1; token
// group tg).  Fixed-order reduction over token groups, so results do not depend on scheduling.
template <typename T>
__global__ void __launch_bounds__(512) k_ysum(Dev D, const T* __restrict__ q, int64_t c0, int n, int64_t b0) {
    extern __shared__ float red[];
    const int64_t b = b0 + blockIdx.x;
    const int hk = blockIdx.y;
    const int64_t sb = (int64_t)D.S + b * D.gblk;
    const int64_t lo = sb > c0 ? sb : c0;
    const int64_t hi = (sb + D.gblk) < (c0 + n) ? (sb + D.gblk) : (c0 + n);
    const int npc = D.half / 2;
    const int pc = threadIdx.x % npc, tg = threadIdx.x / npc, ntg = blockDim.x / npc;
    const int i = 2 * pc;
    float a1x = 0.f, a1y = 0.f, a2x = 0.f, a2y = 0.f;
#pragma unroll 2
    for (int64_t t = lo + tg; t < hi; t += ntg) {
        const float4 cs = *reinterpret_cast<const float4*>(D.cs_rel + (t - sb) * D.half + i);  // (c_i, s_i, c_i+1, s_i+1)
        const T* qr = q + ((t - c0) * D.Hq + (int64_t)hk * D.G) * D.d;
        float2 x1 = make_float2(0.f, 0.f), x2 = make_float2(0.f, 0.f);
        for (int h = 0; h < D.G; ++h) {  // the rotation is linear: sum the group's heads first
            const float2 u = ld2f(qr + h * D.d + i), w = ld2f(qr + h * D.d + i + D.half);
            x1.x += u.x; x1.y += u.y;
            x2.x += w.x; x2.y += w.y;
        }
        a1x += x1.x * cs.x - x2.x * cs.y;
        a2x += x2.x * cs.x + x1.x * cs.y;
        a1y += x1.y * cs.z - x2.y * cs.w;
        a2y += x2.y * cs.z + x1.y * cs.w;
    }
    float* r = red + tg * D.d;
    r[i] = a1x; r[i + 1] = a1y; r[i + D.half] = a2x; r[i + D.half + 1] = a2y;
    __syncthreads();
    for (int j = threadIdx.x; j < D.d; j += blockDim.x) {
        float acc = 0.f;
        for (int g = 0; g < ntg; ++g) acc += red[g * D.d + j];
        D.Y[(b * D.Hkv + hk) * D.d + j] += acc;
    }
}

// Representatives of units [j0, j0 + gridDim.x) for kv head blockIdx.y, 256 threads.
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
    const int64_t j = j0 + blockIdx.x;
    const int hk = blockIdx.y;
    const int64_t e = (int64_t)D.S + (j + 1) * D.U;
    const int64_t m0 = e - D.U;
    const int64_t be = (e - D.S) / D.gblk;
    const int nb = D.W / D.gblk;
    {
        const int i = threadIdx.x % D.half, pg = threadIdx.x / D.half, npg = blockDim.x / D.half;
        float a1 = 0.f, a2 = 0.f;
        for (int p = pg; p < nb; p += npg) {
            const float* y = D.Y + ((be + p) * D.Hkv + hk) * D.d;
            const float2 cs = D.cs_rel[(int64_t)p * D.gblk * D.half + i];
            const float y1 = y[i], y2 = y[i + D.half];
            a1 += y1 * cs.x - y2 * cs.y;
            a2 += y2 * cs.x + y1 * cs.y;
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
        for (int i = lane; i < D.half; i += 32) {
            const float q1 = Qt[i], q2 = Qt[i + D.half];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int m = mb + u;
                if (m < D.U) {
                    const float2 cs = D.cs_rel[(int64_t)(D.U - m) * D.half + i];  // distance e - (m0 + m)
                    const float r1 = q1 * cs.x - q2 * cs.y, r2 = q2 * cs.x + q1 * cs.y;
                    acc[u] += r1 * to_f(K[(int64_t)m * D.d + i]) + r2 * to_f(K[(int64_t)m * D.d + i + D.half]);
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
        for (int qq = 0; qq < D.r; ++qq) {
            const T x = K[(int64_t)ids[qq] * D.d + i];
            rk[(int64_t)qq * D.d + i] = x;
            s += to_f(x);
        }
        rs[i] = s;
    }
}

// ---- launchers ----------------------------------------------------------------------------

template <typename T>
cudaError_t launch_append(const Dev& D, const void* k, const void* v, int64_t c0, int n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    k_append<T><<<n, 256, D.half * sizeof(float2), st>>>(D, (const T*)k, (const T*)v, c0);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ysum(const Dev& D, const void* q, int64_t c0, int n, cudaStream_t st, int* launches) {
    const int64_t lo = c0 > D.S ? c0 : (int64_t)D.S;
    const int64_t hi = c0 + n;
    if (hi <= lo) return cudaSuccess;
    const int64_t b0 = (lo - D.S) / D.gblk, b1 = (hi - 1 - D.S) / D.gblk;
    const int threads = 512;  // (half / 2) pair couples x token groups
    dim3 grid((unsigned)(b1 - b0 + 1), D.Hkv);
    k_ysum<T><<<grid, threads, (threads / (D.half / 2)) * D.d * sizeof(float), st>>>(D, (const T*)q, c0, n, b0);
    ++*launches;
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_reps(const Dev& D, int64_t j0, int64_t j1, cudaStream_t st) {
    if (j1 <= j0) return cudaSuccess;
    dim3 grid((unsigned)(j1 - j0), D.Hkv);
    k_reps<T><<<grid, 256, (D.d + D.U + (256 / D.half) * D.d) * sizeof(float), st>>>(D, j0);
    return cudaGetLastError();
}

template cudaError_t launch_append<float>(const Dev&, const void*, const void*, int64_t, int, cudaStream_t);
template cudaError_t launch_append<__nv_bfloat16>(const Dev&, const void*, const void*, int64_t, int, cudaStream_t);
template cudaError_t launch_ysum<float>(const Dev&, const void*, int64_t, int, cudaStream_t, int*);
template cudaError_t launch_ysum<__nv_bfloat16>(const Dev&, const void*, int64_t, int, cudaStream_t, int*);
template cudaError_t launch_reps<float>(const Dev&, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_reps<__nv_bfloat16>(const Dev&, int64_t, int64_t, cudaStream_t);

}  // namespace infllm
