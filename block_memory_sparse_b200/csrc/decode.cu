// Decode attention for one new token: split-KV partials over the token's working context
// (sinks, selected units, window) merged with a log-sum-exp reduction.
//
// Method: "InfLLM Guide: Training-Free Long-Context Memory Units", "Core Innovation 2",
// items 2-3 (per generated token: score units, keep the top-k, exact attention over
// Sinks U selected units U window).  The split-KV form is exact: each CTA returns the
// running max m, the sum l of exp(s - m) and the unnormalised output over its keys; the
// merge rescales by exp(m_s - M) and divides by the total sum.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace infllm {

template <typename T> struct DecodeCfg;
template <> struct DecodeCfg<__nv_bfloat16> { static constexpr int SK = 128; };
template <> struct DecodeCfg<float> { static constexpr int SK = 64; };

int decode_split_keys(int elt_bytes) { return elt_bytes == 2 ? DecodeCfg<__nv_bfloat16>::SK : DecodeCfg<float>::SK; }

// Map a position in the token's virtual key list to (token, window frame?).
struct KeyMap {
    int64_t S_eff, n_units_tok, B;
    int U, S, kk;
    const int32_t* sel;
    __device__ __forceinline__ int64_t token(int64_t v, bool& win, bool& bad) const {
        win = false;
        bad = false;
        if (v < S_eff) return v;
        v -= S_eff;
        if (v < n_units_tok) {
            const int u = (int)(v / U), off = (int)(v % U);
            const int j = sel[u];
            if (j < 0 || (int64_t)S + (int64_t)(j + 1) * U > B) {
                bad = true;
                return 0;
            }
            return (int64_t)S + (int64_t)j * U + off;
        }
        win = true;
        return B + (v - n_units_tok);
    }
};

// Grid (n_split, Hkv), 128 threads.  Each CTA takes SK consecutive keys of the virtual list.
template <typename T>
__global__ void __launch_bounds__(128) k_decode(Dev D, const T* __restrict__ q, T* __restrict__ out, int64_t t, int kk,
                                                int64_t B, int64_t Ktot, int n_split) {
    constexpr int SK = DecodeCfg<T>::SK;
    extern __shared__ float sm[];
    const int d = D.d, G = D.G;
    const int hk = blockIdx.y, s = blockIdx.x;
    float* qf = sm;                         // [G][d]  R(W) q
    float* qw = qf + G * d;                 // [G][d]  R(t) q
    float* p_s = qw + G * d;                // [G][SK]
    float* red = p_s + G * SK;              // [4][G] cross-warp reductions
    float* accs = red + 4 * G;              // [128 / d][G][d] partial outputs
    T* k_s = (T*)(accs + (128 / d) * G * d);  // [SK][d + 2]
    T* v_s = k_s + SK * (d + 2);            // [SK][d]
    __shared__ int win_s[SK];
    __shared__ int is_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    KeyMap km{(int64_t)(D.S < t + 1 ? D.S : t + 1), (int64_t)kk * D.U, B, D.U, D.S, kk, D.sel + hk * D.topk};
    const int64_t v0 = (int64_t)s * SK;
    const int nk = (int)((Ktot - v0) < SK ? (Ktot - v0) : SK);

    // rotated queries of the group's heads
    for (int idx = tid; idx < G * D.half; idx += blockDim.x) {
        const int h = idx / D.half, i = idx % D.half;
        const T* src = q + (int64_t)(hk * G + h) * d;
        const float x1 = to_f(src[i]), x2 = to_f(src[i + D.half]);
        const float2 cw = D.cs_W[i], ct = D.cs_chunk[i];
        qf[h * d + i] = x1 * cw.x - x2 * cw.y;
        qf[h * d + i + D.half] = x2 * cw.x + x1 * cw.y;
        qw[h * d + i] = x1 * ct.x - x2 * ct.y;
        qw[h * d + i + D.half] = x2 * ct.x + x1 * ct.y;
    }
    // stage K (padded rows) and V
    const int vec = 16 / sizeof(T);
    for (int idx = tid; idx < SK * (d / vec); idx += blockDim.x) {
        const int kr = idx / (d / vec), c = idx % (d / vec);
        uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
        bool win = false;
        if (kr < nk) {
            bool bad;
            const int64_t tok = km.token(v0 + kr, win, bad);
            if (bad) set_err(D, ERR_SEL_RANGE);
            const int64_t off = ((int64_t)hk * D.T_max + tok) * d + c * vec;
            kv = __ldg(reinterpret_cast<const uint4*>((const T*)(win ? D.Krot : D.Kraw) + off));
            vv = __ldg(reinterpret_cast<const uint4*>((const T*)D.V + off));
        }
        if (c == 0) win_s[kr] = win;
        // padded K rows are only 4-byte aligned: store as 32-bit words
        const uint32_t* kw = reinterpret_cast<const uint32_t*>(&kv);
        uint32_t* kd = reinterpret_cast<uint32_t*>(k_s + kr * (d + 2) + c * vec);
        kd[0] = kw[0]; kd[1] = kw[1]; kd[2] = kw[2]; kd[3] = kw[3];
        *reinterpret_cast<uint4*>(v_s + kr * d + c * vec) = vv;
    }
    __syncthreads();
    // logits: thread per key, all G heads
    float sc[8];
    for (int h = 0; h < G && h < 8; ++h) sc[h] = -INFINITY;
    if (tid < nk) {
        const float* qq = win_s[tid] ? qw : qf;
        const T* kr = k_s + tid * (d + 2);
        for (int h = 0; h < G && h < 8; ++h) {
            float a = 0.f;
            for (int i = 0; i < d; ++i) a += qq[h * d + i] * to_f(kr[i]);
            sc[h] = a * D.inv_sqrt_d;
        }
    }
    // per-head max and sum over the CTA's keys
    for (int h = 0; h < G && h < 8; ++h) {
        const float mx = warp_max(sc[h]);
        if (lane == 0) red[warp * G + h] = mx;
    }
    __syncthreads();
    float mh[8];
    for (int h = 0; h < G && h < 8; ++h) {
        float mx = red[h];
        for (int w = 1; w < 4; ++w) mx = fmaxf(mx, red[w * G + h]);
        mh[h] = mx;
    }
    __syncthreads();
    for (int h = 0; h < G && h < 8; ++h) {
        const float p = tid < nk ? expf(sc[h] - mh[h]) : 0.f;
        if (tid < SK) p_s[h * SK + tid] = p;
        const float sum = warp_sum(p);
        if (lane == 0) red[warp * G + h] = sum;
    }
    __syncthreads();
    // P V: thread owns dim tid % d for key slice tid / d
    const int nslice = 128 / d, dim = tid % d, slc = tid / d;
    for (int h = 0; h < G; ++h) {
        float a = 0.f;
        for (int kr = slc; kr < nk; kr += nslice) a += p_s[h * SK + kr] * to_f(v_s[kr * d + dim]);
        accs[(slc * G + h) * d + dim] = a;
    }
    __syncthreads();
    float* part = D.dec_part + ((int64_t)hk * D.dec_splits_max + s) * G * (d + 2);
    for (int idx = tid; idx < G * d; idx += blockDim.x) {
        const int h = idx / d, i = idx % d;
        float a = 0.f;
        for (int sl = 0; sl < nslice; ++sl) a += accs[(sl * G + h) * d + i];
        part[h * (d + 2) + 2 + i] = a;
    }
    if (tid < G) {
        float l = 0.f;
        for (int w = 0; w < 4; ++w) l += red[w * G + tid];
        part[tid * (d + 2) + 0] = mh[tid];
        part[tid * (d + 2) + 1] = l;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(&D.counters[D.Hkv + hk], 1u) == (unsigned)(n_split - 1));
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    const float* base = D.dec_part + (int64_t)hk * D.dec_splits_max * G * (d + 2);
    for (int idx = tid; idx < G * d; idx += blockDim.x) {
        const int h = idx / d, i = idx % d;
        float M = -INFINITY;
        for (int ss = 0; ss < n_split; ++ss) M = fmaxf(M, __ldcg(base + ((int64_t)ss * G + h) * (d + 2)));
        float L = 0.f, O = 0.f;
        for (int ss = 0; ss < n_split; ++ss) {
            const float* pp = base + ((int64_t)ss * G + h) * (d + 2);
            const float w = expf(__ldcg(pp) - M);
            L += w * __ldcg(pp + 1);
            O += w * __ldcg(pp + 2 + i);
        }
        out[(int64_t)(hk * G + h) * d + i] = from_f<T>(O / L);
    }
    if (tid == 0) D.counters[D.Hkv + hk] = 0u;
}

template <typename T>
cudaError_t launch_decode(const Dev& D, const void* q, int64_t t, int kk, int64_t B, void* out, cudaStream_t st,
                          int* n_split_out) {
    constexpr int SK = DecodeCfg<T>::SK;
    const int64_t S_eff = D.S < t + 1 ? D.S : t + 1;
    const int64_t Ktot = S_eff + (int64_t)kk * D.U + (t - B + 1);
    int n_split = (int)((Ktot + SK - 1) / SK);
    *n_split_out = n_split;
    if (n_split > D.dec_splits_max) return cudaErrorInvalidValue;
    const size_t smem = (size_t)(2 * D.G * D.d + D.G * SK + 4 * D.G + (128 / D.d) * D.G * D.d) * sizeof(float) +
                        (size_t)SK * (D.d + 2) * sizeof(T) + (size_t)SK * D.d * sizeof(T) + 16;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_decode<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(n_split, D.Hkv);
    k_decode<T><<<grid, 128, smem, st>>>(D, (const T*)q, (T*)out, t, kk, B, Ktot, n_split);
    return cudaGetLastError();
}

template cudaError_t launch_decode<float>(const Dev&, const void*, int64_t, int, int64_t, void*, cudaStream_t, int*);
template cudaError_t launch_decode<__nv_bfloat16>(const Dev&, const void*, int64_t, int, int64_t, void*, cudaStream_t,
                                                  int*);

}  // namespace infllm
