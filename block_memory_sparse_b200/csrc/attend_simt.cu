// Exact attention of a chunk over sinks U selected units U local window, on the CUDA cores
// with fp32 arithmetic.  This is the path of fp32 layers: fp32 inputs need fp32 products, and
// TF32 tensor cores are not accurate enough.  bf16 layers always run on the tensor cores.
//
// Method: "InfLLM Guide: Training-Free Long-Context Memory Units", "Core Innovation 2",
// item 3 "Exact Attention Evaluation": one softmax over the working context
// Sinks U (U_{m in top-k} M_m) U Local Window.
// Positions: sinks and memory keys at distance W (query R(W) q, key raw); window keys at
// true relative distance (query R(t) q, key R(n) k).
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace infllm {

constexpr int SIMT_ROWS = 8;   // packed query rows per CTA (one per warp)
constexpr int SIMT_KT = 32;    // keys per smem tile (one per lane)

// Grid (row CTAs, Hkv, nsplit).  With nsplit > 1 (a small chunk that would leave most SMs idle),
// split sp takes every nsplit-th 32-key tile of the working context, writes its rows' partial
// softmax (m, l, unnormalised o) to D.simt_part, and the CTA that finishes a row group's last split
// (arrival counter, no CTA waits for another) merges the nsplit partials: the log-sum-exp
// combination of disjoint key sets, in split order.
template <typename T>
__global__ void __launch_bounds__(256) k_attn_simt(Dev D, int64_t c0, int n, int kk, int64_t B, int par,
                                                   T* __restrict__ out, int nsplit) {
    extern __shared__ float sm[];
    pdl_wait();  // late kernel: selection, packed queries and keys are complete past this point
    pdl_trigger();
    const int d = D.d;
    float* qm_s = sm;                                  // [ROWS][d]
    float* qw_s = qm_s + SIMT_ROWS * d;                // [ROWS][d]
    float* k_s = qw_s + SIMT_ROWS * d;                 // [KT][d + 1]
    float* v_s = k_s + SIMT_KT * (d + 1);              // [KT][d]
    const int hk = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rpt = D.qt * D.G;
    // rows of this CTA and the largest query position among them
    int64_t t_hi = -1;
    for (int w = 0; w < SIMT_ROWS; ++w) {
        const int64_t R = (int64_t)blockIdx.x * SIMT_ROWS + w;
        const int a = (int)(R / rpt), r = (int)(R % rpt);
        const int tl = a * D.qt + r % D.qt;
        if (tl < n && c0 + tl > t_hi) t_hi = c0 + tl;
    }
    const int64_t R = (int64_t)blockIdx.x * SIMT_ROWS + warp;
    const int a = (int)(R / rpt), r = (int)(R % rpt);
    const int hg = r / D.qt, tl = a * D.qt + r % D.qt;
    const bool valid = tl < n;
    const int64_t t = c0 + tl;
    if (valid) {  // rows past the packed tiles (rows % 8 != 0) are never read
        const T* Qm = (const T*)D.Qm + (((int64_t)hk * 3 + par) * D.qrows_max + R) * d;
        const T* Qw = (const T*)D.Qw + (((int64_t)hk * 3 + par) * D.qrows_max + R) * d;
        for (int i = lane; i < d; i += 32) {
            qm_s[warp * d + i] = to_f(Qm[i]);
            qw_s[warp * d + i] = to_f(Qw[i]);
        }
    }
    float m = -INFINITY, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int ndim = d / 32;
    if (t_hi < 0) return;  // whole CTA is padding (uniform; every split of it returns here)
    const int nseg = 2 + kk;
    const int sp = blockIdx.z;
    int g = 0;  // tiles of the working context seen so far (all splits walk the same sequence)
    for (int sg = 0; sg < nseg; ++sg) {
        int64_t base, len;
        bool win = false, causal = false;
        if (sg == 0) {
            base = 0;
            len = D.S < t_hi + 1 ? D.S : t_hi + 1;
            causal = true;
        } else if (sg <= kk) {
            int j = D.sel[hk * D.topk + sg - 1];
            if (j < 0 || (int64_t)D.S + (int64_t)(j + 1) * D.U > B) {
                set_err(D, ERR_SEL_RANGE);
                continue;
            }
            base = (int64_t)D.S + (int64_t)j * D.U;
            len = D.U;
        } else {
            base = B;
            len = t_hi + 1 - B;
            win = true;
            causal = true;
        }
        const T* Ks = (const T*)(win ? D.Krot : D.Kraw) + ((int64_t)hk * D.T_max + base) * d;
        const T* Vs = (const T*)D.V + ((int64_t)hk * D.T_max + base) * d;
        for (int64_t k0 = 0; k0 < len; k0 += SIMT_KT) {
            if (g++ % nsplit != sp) continue;  // another split's tile (CTA-uniform)
            const int nk = (int)((len - k0) < SIMT_KT ? (len - k0) : SIMT_KT);
            __syncthreads();
            for (int idx = threadIdx.x; idx < SIMT_KT * d; idx += blockDim.x) {
                const int kr = idx / d, i = idx % d;
                float kv = 0.f, vv = 0.f;
                if (kr < nk) {
                    kv = to_f(Ks[(k0 + kr) * d + i]);
                    vv = to_f(Vs[(k0 + kr) * d + i]);
                }
                k_s[kr * (d + 1) + i] = kv;
                v_s[kr * d + i] = vv;
            }
            __syncthreads();
            if (!valid) continue;
            const float* qv = (win ? qw_s : qm_s) + warp * d;
            float s = 0.f;
            for (int i = 0; i < d; ++i) s += qv[i] * k_s[lane * (d + 1) + i];
            s *= D.inv_sqrt_d;
            const int64_t ntok = base + k0 + lane;
            const bool ok = lane < nk && (!causal || ntok <= t);
            s = ok ? s : -INFINITY;
            const float m_new = fmaxf(m, warp_max(s));
            if (m_new == -INFINITY) continue;
            const float alpha = expf(m - m_new);
            const float p = ok ? expf(s - m_new) : 0.f;
            l = l * alpha + warp_sum(p);
            for (int c = 0; c < ndim; ++c) acc[c] *= alpha;
            for (int kr = 0; kr < nk; ++kr) {
                const float pk = __shfl_sync(0xffffffffu, p, kr);
                for (int c = 0; c < ndim; ++c) acc[c] += pk * v_s[kr * d + lane + 32 * c];
            }
            m = m_new;
        }
    }
    if (nsplit == 1) {
        if (valid) {
            T* o = out + ((int64_t)tl * D.Hq + hk * D.G + hg) * d;
            const float inv = 1.f / l;
            for (int c = 0; c < ndim; ++c) o[lane + 32 * c] = from_f<T>(acc[c] * inv);
        }
        return;
    }
    // this split's partial of the row (m, l, o) -> slot [row group][split][row]
    const int grp = hk * gridDim.x + blockIdx.x;
    float* part = D.simt_part + ((int64_t)grp * nsplit * SIMT_ROWS) * (d + 2);
    float* mine = part + ((int64_t)sp * SIMT_ROWS + warp) * (d + 2);
    if (lane == 0) {
        mine[0] = m;
        mine[1] = l;
    }
    for (int c = 0; c < ndim; ++c) mine[2 + lane + 32 * c] = acc[c];
    __threadfence();
    __syncthreads();
    __shared__ int last;
    if (threadIdx.x == 0) last = atomicAdd(D.simt_ctr + grp, 1u) == (unsigned)(nsplit - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    if (valid) {
        float M = -INFINITY;
        for (int x = 0; x < nsplit; ++x) M = fmaxf(M, __ldcg(part + ((int64_t)x * SIMT_ROWS + warp) * (d + 2)));
        float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
        for (int x = 0; x < nsplit; ++x) {
            const float* px = part + ((int64_t)x * SIMT_ROWS + warp) * (d + 2);
            const float mx = __ldcg(px);
            if (mx == -INFINITY) continue;  // no attended key in this split
            const float f = expf(mx - M);
            L = fmaf(f, __ldcg(px + 1), L);
            for (int c = 0; c < ndim; ++c) o[c] = fmaf(f, __ldcg(px + 2 + lane + 32 * c), o[c]);
        }
        T* orow = out + ((int64_t)tl * D.Hq + hk * D.G + hg) * d;
        const float inv = 1.f / L;
        for (int c = 0; c < ndim; ++c) orow[lane + 32 * c] = from_f<T>(o[c] * inv);
    }
    if (threadIdx.x == 0) D.simt_ctr[grp] = 0u;  // re-armed for the next launch
}

template <typename T>
cudaError_t launch_attend_simt(const Dev& D, int64_t c0, int n, int kk, int64_t B, int par, void* out, cudaStream_t st,
                               bool pdl) {
    if (n <= 0) return cudaSuccess;
    const int tiles = (n + D.qt - 1) / D.qt;
    const int rows = tiles * D.qt * D.G;
    const int ctas = (rows + SIMT_ROWS - 1) / SIMT_ROWS;
    // split the keys over up to SIMT_MAX_SPLIT CTAs per row group while the grid stays under
    // SIMT_PART_GROUPS CTAs (the partial slots and counters allocated at create)
    const int groups = ctas * D.Hkv;
    const int nsplit = groups >= SIMT_PART_GROUPS / 2 ? 1 : std::min(SIMT_MAX_SPLIT, SIMT_PART_GROUPS / groups);
    dim3 grid(ctas, D.Hkv, nsplit);
    const size_t smem = (size_t)(2 * SIMT_ROWS * D.d + SIMT_KT * (D.d + 1) + SIMT_KT * D.d) * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_attn_simt<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_k(k_attn_simt<T>, grid, dim3(256), smem, st, pdl, D, c0, n, kk, B, par, (T*)out, nsplit);
}

template cudaError_t launch_attend_simt<float>(const Dev&, int64_t, int, int, int64_t, int, void*, cudaStream_t, bool);

}  // namespace infllm
