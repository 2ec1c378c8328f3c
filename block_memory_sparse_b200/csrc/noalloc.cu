// Unit scoring + top-k selection for one query token that allocates nothing.
//
// Some callers cannot call cudaMalloc: code that runs while a framework captures its stream
// into a CUDA graph and forbids allocation there, engines whose memory planner owns every
// device byte, and real-time serving loops where an allocation may synchronise the device.
// This variant of the lookup kernel takes every input and output from the caller and keeps
// its scratch (per-CTA candidate lists and per-head arrival counters) in one file-scope
// static device array of fixed size, which every GPU that loads the library holds until the
// process exits.  The InfLLM pages have no counterpart to this entry point; it computes the
// same unit scores and selection as the lookup step of infllm_decode_step.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "../../include/infllm.h"
#include "common.cuh"

namespace infllm {
namespace {

constexpr int NA_MAX_HKV = 64;       // kv heads
constexpr int NA_UNITS_PER_CTA = 256;
constexpr int NA_MAX_SPLITS = 64;    // => at most 64 * 256 = 16384 units
constexpr int NA_MAX_UNITS = NA_MAX_SPLITS * NA_UNITS_PER_CTA;
constexpr int NA_MAX_DEVICES = 64;

struct NoallocScratch {
    uint64_t cand[NA_MAX_HKV][NA_MAX_SPLITS][32];  // 1 MiB of candidate lists
    unsigned counters[NA_MAX_HKV];
};

// The scratch area (about 1 MiB).  In host code this name is only a stand-in for the symbol:
// kernels get its device address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[sizeof(NoallocScratch)];

std::mutex g_mu;
void* g_addr[NA_MAX_DEVICES] = {nullptr};
unsigned long long g_ctx[NA_MAX_DEVICES] = {0};  // id of the context g_addr[dev] was resolved in

// Unique id (for the process lifetime) of the calling thread's current CUDA context, 0 if none.  A
// device reset replaces the primary context and reloads the module, which moves the scratch array;
// a new id tells the entry point to look its address up again.
unsigned long long current_context_id() {
    typedef CUresult (*GetCurrentFn)(CUcontext*);
    typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    if (!get_current || !get_id) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = (GetCurrentFn)p;
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = (GetIdFn)p;
        if (!get_current || !get_id) return 0;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

template <typename T>
__global__ void __launch_bounds__(256) k_select_noalloc(NoallocScratch* scr, const T* __restrict__ rep_keys,
                                                        const T* __restrict__ q, int G, int d, int n_units, int r,
                                                        int window, double rope_base, int topk, int n_split,
                                                        int32_t* __restrict__ sel, float* __restrict__ scores) {
    __shared__ float qb[128];
    __shared__ uint64_t lists[8][32];
    __shared__ int is_last;
    const int split = blockIdx.x, hk = blockIdx.y, half = d / 2;
    const float inv_sqrt_d = (float)(1.0 / sqrt((double)d));
    // query of the group summed over its heads, rotated by R(window) (angles in fp64)
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        float a = 0.f, b = 0.f;
        for (int h = 0; h < G; ++h) {
            a += to_f(q[(hk * G + h) * d + i]);
            b += to_f(q[(hk * G + h) * d + i + half]);
        }
        double s, c;
        sincos((double)window * pow(rope_base, -2.0 * i / (double)d), &s, &c);
        const float cw = (float)c, sw = (float)s;
        qb[i] = a * cw - b * sw;
        qb[i + half] = b * cw + a * sw;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = split * NA_UNITS_PER_CTA;
    const int u1 = min(n_units, u0 + NA_UNITS_PER_CTA);
    // A unit's row (r * d elements) is read by the whole warp in 16-byte pieces, consecutive lanes
    // on consecutive pieces; the warp takes four units at a time, all their loads issued first.
    constexpr int V = 16 / sizeof(T);
    const int cpr = r * d / V;  // 16-byte pieces per row (a multiple of 4)
    uint64_t list = 0;
    for (int jb = u0 + warp * 32; jb < u1; jb += 8 * 32) {
        uint64_t cand = 0;
        for (int jj = 0; jj < 32 && jb + jj < u1; jj += 4) {  // warp-uniform
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int c0 = 0; c0 < cpr; c0 += 32) {
                const int c = c0 + lane;
                uint4 raw[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = jb + jj + u;
                    raw[u] = (c < cpr && j < u1)
                                 ? __ldg(reinterpret_cast<const uint4*>(rep_keys + ((int64_t)hk * n_units + j) * r * d) + c)
                                 : make_uint4(0, 0, 0, 0);
                }
                const int i0 = (c * V) % d;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const T* e = reinterpret_cast<const T*>(&raw[u]);
#pragma unroll
                    for (int v = 0; v < V; ++v) acc[u] += c < cpr ? to_f(e[v]) * qb[i0 + v] : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float s = warp_sum(acc[u]) * inv_sqrt_d;
                const int j = jb + jj + u;
                if (j < u1 && lane == jj + u) {
                    if (scores) scores[(int64_t)hk * n_units + j] = s;
                    cand = make_key(s, (uint32_t)j);
                }
            }
        }
        list = warp_topk_insert(list, cand);
    }
    lists[warp][lane] = list;
    __syncthreads();
    if (warp == 0) {
        uint64_t acc = lists[0][lane];
        for (int w = 1; w < 8; ++w) acc = warp_merge_desc(acc, lists[w][lane]);
        scr->cand[hk][split][lane] = acc;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomicAdd(&scr->counters[hk], 1u) == (unsigned)(n_split - 1));
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (warp == 0) {
        uint64_t acc = 0;
        for (int s = 0; s < n_split; ++s) acc = warp_merge_desc(acc, __ldcg(&scr->cand[hk][s][lane]));
        const int kk = min(topk, n_units);
        uint64_t sk = (lane < kk) ? (uint64_t)(0xffffffffu - key_index(acc)) : 0ull;
        sk = warp_sort_desc(sk);
        if (lane < topk) sel[hk * topk + lane] = (lane < kk) ? (int)(0xffffffffu - (uint32_t)sk) : -1;
        if (lane == 0) scr->counters[hk] = 0u;
    }
}

}  // namespace
}  // namespace infllm

using namespace infllm;

extern "C" infllm_status infllm_select_units_noalloc(const void* rep_keys, const void* q, int32_t n_q_heads,
                                                     int32_t n_kv_heads, int32_t head_dim, int32_t n_units,
                                                     int32_t n_reps, int32_t window, double rope_base, int32_t dtype,
                                                     int32_t top_k, int32_t* sel, float* scores, void* cuda_stream) {
    if (!q || !sel || n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads) return INFLLM_EINVAL;
    if (head_dim != 64 && head_dim != 128) return INFLLM_EINVAL;
    if (n_units < 0 || n_reps < 1 || window < 1 || !(rope_base > 1.0)) return INFLLM_EINVAL;
    if (top_k < 1 || top_k > 32) return INFLLM_EINVAL;
    if (dtype != INFLLM_F32 && dtype != INFLLM_BF16) return INFLLM_EINVAL;
    if (n_units > 0 && !rep_keys) return INFLLM_EINVAL;
    if ((uintptr_t)rep_keys % 16 != 0) return INFLLM_EINVAL;  // read in 16-byte pieces
    // beyond the fixed scratch area
    if (n_kv_heads > NA_MAX_HKV || n_units > NA_MAX_UNITS) return INFLLM_ECAPACITY;
    cudaStream_t st = (cudaStream_t)cuda_stream;
    if (n_units == 0) {
        return cudaMemsetAsync(sel, 0xff, sizeof(int32_t) * (size_t)n_kv_heads * top_k, st) == cudaSuccess
                   ? INFLLM_OK : INFLLM_ECUDA;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NA_MAX_DEVICES) return INFLLM_ECUDA;
    void* base = nullptr;
    {
        // the current device's runtime context exists from here on (cudaGetSymbolAddress creates it)
        std::lock_guard<std::mutex> lk(g_mu);
        unsigned long long ctx = current_context_id();
        if (!g_addr[dev] || ctx == 0 || ctx != g_ctx[dev]) {  // once per device and context, that device current
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return INFLLM_ECUDA;
            g_addr[dev] = p;
            g_ctx[dev] = ctx != 0 ? ctx : current_context_id();
        }
        base = g_addr[dev];
    }
    NoallocScratch* scr = (NoallocScratch*)base;
    // the arrival counters must start at zero whatever an earlier call left behind
    if (cudaMemsetAsync(scr->counters, 0, sizeof(unsigned) * n_kv_heads, st) != cudaSuccess) return INFLLM_ECUDA;
    const int n_split = (n_units + NA_UNITS_PER_CTA - 1) / NA_UNITS_PER_CTA;
    const int G = n_q_heads / n_kv_heads;
    dim3 grid(n_split, n_kv_heads);
    if (dtype == INFLLM_BF16)
        k_select_noalloc<__nv_bfloat16><<<grid, 256, 0, st>>>(scr, (const __nv_bfloat16*)rep_keys,
                                                              (const __nv_bfloat16*)q, G, head_dim, n_units, n_reps,
                                                              window, rope_base, top_k, n_split, sel, scores);
    else
        k_select_noalloc<float><<<grid, 256, 0, st>>>(scr, (const float*)rep_keys, (const float*)q, G, head_dim,
                                                      n_units, n_reps, window, rope_base, top_k, n_split, sel, scores);
    return cudaGetLastError() == cudaSuccess ? INFLLM_OK : INFLLM_ECUDA;
}
