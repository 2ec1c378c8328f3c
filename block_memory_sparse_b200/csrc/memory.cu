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
// Grid (blocks touched, Hkv); blockDim a multiple of half.  Fixed-order reduction.
template <typename T>
__global__ void k_ysum(Dev D, const T* __restrict__ q, int64_t c0, int n, int64_t b0) {
    extern __shared__ float red[];
    const int64_t b = b0 + blockIdx.x;
    const int hk = blockIdx.y;
    const int64_t sb = (int64_t)D.S + b * D.gblk;
    const int64_t lo = sb > c0 ? sb : c0;
    const int64_t hi = (sb + D.gblk) < (c0 + n) ? (sb + D.gblk) : (c0 + n);
    const int i = threadIdx.x % D.half, tg = threadIdx.x / D.half, ntg = blockDim.x / D.half;
    float a1 = 0.f, a2 = 0.f;
    for (int64_t t = lo + tg; t < hi; t += ntg) {
        const float2 cs = D.cs_rel[(t - sb) * D.half + i];
        const T* qr = q + ((t - c0) * D.Hq + (int64_t)hk * D.G) * D.d;
        for (int h = 0; h < D.G; ++h) {
            const float x1 = to_f(qr[h * D.d + i]), x2 = to_f(qr[h * D.d + i + D.half]);
            a1 += x1 * cs.x - x2 * cs.y;
            a2 += x2 * cs.x + x1 * cs.y;
        }
    }
    red[tg * D.d + i] = a1;
    red[tg * D.d + i + D.half] = a2;
    __syncthreads();
    if (tg == 0) {
        float s1 = 0.f, s2 = 0.f;
        for (int g = 0; g < ntg; ++g) {
            s1 += red[g * D.d + i];
            s2 += red[g * D.d + i + D.half];
        }
        float* y = D.Y + (b * D.Hkv + hk) * D.d;
        y[i] += s1;
        y[i + D.half] += s2;
    }
}

// Representatives of units [j0, j0 + gridDim.x) for kv head blockIdx.y.
//   Qt = sum_{i=e}^{e+W-1} sum_h R(i - e) q_{i,h}  (from the block sums, e = unit end)
//   rho_m = <R(e - m) Qt, k_m> / sqrt(d)  ==  sum_i sum_h <R(i) q_{i,h}, R(m) k_m> / sqrt(d)
// then the top r by (rho desc, m asc), stored ascending, plus the raw rep keys and their sum.
template <typename T>
__global__ void k_reps(Dev D, int64_t j0) {
    extern __shared__ float sm[];
    float* Qt = sm;          // [d]
    float* rho = sm + D.d;   // [U]
    __shared__ int ids[32];
    const int64_t j = j0 + blockIdx.x;
    const int hk = blockIdx.y;
    const int64_t e = (int64_t)D.S + (j + 1) * D.U;
    const int64_t m0 = e - D.U;
    const int64_t be = (e - D.S) / D.gblk;
    const int nb = D.W / D.gblk;
    for (int i = threadIdx.x; i < D.half; i += blockDim.x) {
        float a1 = 0.f, a2 = 0.f;
        for (int p = 0; p < nb; ++p) {
            const float* y = D.Y + ((be + p) * D.Hkv + hk) * D.d;
            const float2 cs = D.cs_rel[(int64_t)p * D.gblk * D.half + i];
            const float y1 = y[i], y2 = y[i + D.half];
            a1 += y1 * cs.x - y2 * cs.y;
            a2 += y2 * cs.x + y1 * cs.y;
        }
        Qt[i] = a1;
        Qt[i + D.half] = a2;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const T* K = (const T*)D.Kraw + ((int64_t)hk * D.T_max + m0) * D.d;
    for (int m = warp; m < D.U; m += nw) {
        const int dist = D.U - m;  // e - (m0 + m)
        float part = 0.f;
        for (int i = lane; i < D.half; i += 32) {
            const float2 cs = D.cs_rel[(int64_t)dist * D.half + i];
            const float q1 = Qt[i], q2 = Qt[i + D.half];
            const float r1 = q1 * cs.x - q2 * cs.y, r2 = q2 * cs.x + q1 * cs.y;
            part += r1 * to_f(K[(int64_t)m * D.d + i]) + r2 * to_f(K[(int64_t)m * D.d + i + D.half]);
        }
        part = warp_sum(part);
        if (lane == 0) rho[m] = part * D.inv_sqrt_d;
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
    const int threads = D.half * (256 / D.half);
    dim3 grid((unsigned)(b1 - b0 + 1), D.Hkv);
    k_ysum<T><<<grid, threads, (threads / D.half) * D.d * sizeof(float), st>>>(D, (const T*)q, c0, n, b0);
    ++*launches;
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_reps(const Dev& D, int64_t j0, int64_t j1, cudaStream_t st) {
    if (j1 <= j0) return cudaSuccess;
    dim3 grid((unsigned)(j1 - j0), D.Hkv);
    k_reps<T><<<grid, 128, (D.d + D.U) * sizeof(float), st>>>(D, j0);
    return cudaGetLastError();
}

template cudaError_t launch_append<float>(const Dev&, const void*, const void*, int64_t, int, cudaStream_t);
template cudaError_t launch_append<__nv_bfloat16>(const Dev&, const void*, const void*, int64_t, int, cudaStream_t);
template cudaError_t launch_ysum<float>(const Dev&, const void*, int64_t, int, cudaStream_t, int*);
template cudaError_t launch_ysum<__nv_bfloat16>(const Dev&, const void*, int64_t, int, cudaStream_t, int*);
template cudaError_t launch_reps<float>(const Dev&, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_reps<__nv_bfloat16>(const Dev&, int64_t, int64_t, cudaStream_t);

}  // namespace infllm
