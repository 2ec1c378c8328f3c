// Shared device-side definitions for the InfLLM layer kernels (sm_100a).
#pragma once

#include <atomic>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace infllm {

// Everything a kernel needs to know about the layer and the context's device buffers.
// Passed by value to every kernel.
// Split of the CUDA-core chunk attention over keys: at most SIMT_MAX_SPLIT splits, and
// (row groups x splits) <= SIMT_PART_GROUPS, the CTAs whose partials the context keeps room for.
constexpr int SIMT_MAX_SPLIT = 16;
constexpr int SIMT_PART_GROUPS = 296;

struct Dev {
    // shape
    int Hq, Hkv, G, d, half;
    int S, W, U, r, topk;
    int gblk;             // query-sum block length (gcd(U, W)); blocks start at token S
    int64_t T_max;        // token capacity
    int64_t units_max;    // unit capacity
    float inv_sqrt_d;
    // stores, [Hkv][T_max][d] in the context dtype
    void* Kraw;           // keys as given (sinks and memory frame)
    void* Krot;           // R(n) k_n (window frame, absolute position n)
    void* V;
    // query block sums: Y[b][hk][d] = sum_{t in block b} sum_{h in group hk} R(t - s_b) q_{t,h}
    float* Y;
    // representatives
    int32_t* rep_ids;     // [Hkv][units_max][r] unit-local offsets, ascending
    void* rep_keys;       // [Hkv][units_max][r][d] raw keys (context dtype)
    float* repsum;        // [Hkv][units_max][d] fp32 sum of the r raw keys
    void* meankey;        // [Hkv][units_max][d] mean of the unit's U raw keys (context dtype)
    // lookup
    int32_t* sel;         // [Hkv][topk] ascending ids, -1 padded (the current lookup's of two buffers)
    float* uscore;        // [Hkv][units_max] last chunk's unit scores
    float* qbar_part;     // [Hkv][qtiles_max][d] per-tile raw query sums (the current lookup's of two)
    uint64_t* cand;       // [Hkv][score_splits_max][32] top-k candidate lists
    unsigned* counters;   // [4][Hkv] arrival counters (last CTA done): unit selection, CUDA-core decode merge,
                          // tile decode part 0 and part 1
    // rotated, packed queries of a chunk: [Hkv][3][qrows_max][d] (three slots, so later chunks'
    // queries can be packed while an earlier chunk's attention runs)
    void* Qm;             // R(W) q  (sink / memory frame)
    void* Qw;             // R(t) q  (window frame)
    int64_t qrows_max;    // rows per buffer and kv head
    int qt;               // queries per 128-row tile (128 / G, or 1 when G > 128)
    // position tables
    const double* inv_freq;  // [half] theta_i in fp64
    const float2* cs_rel;    // [P_rel][half] (cos, sin)(p theta_i), p < P_rel
    int P_rel;
    const float2* cs_W;      // [half] (cos, sin)(W theta_i)
    float2* cs_chunk;        // [max_chunk][half] (cos, sin)(t theta_i) for the current chunk
    // (cos, sin)(x 2^(11 L) theta_i) in fp64 for L < 3, x < 2048: exp(i t theta) for any
    // t < 2^33 is the product of three entries (t's 11-bit digits)
    const double2* cs_abs3;  // [3][2048][half]
    // CUDA-core chunk attention split over keys: partials [groups][splits][8 rows][d + 2] (m, l, o) and
    // one arrival counter per row group (SIMT_PART_GROUPS x 8 rows of slots in all)
    float* simt_part;
    unsigned* simt_ctr;
    // decode partials: [Hkv][dec_splits_max][G][d + 4] (the CUDA-core decode uses [G][d + 2] of a slot)
    float* dec_part;
    int dec_splits_max;
    int score_splits_max;
    int qtiles_max;
    // error word (host-mapped)
    int* err;
};

// Unit-scoring operand (the score modes of the C ABI): the n_reps representative keys, their fp32
// sum, or the mean of all of the unit's keys.
enum ScoreOperand : int { OP_REPS = 0, OP_REPSUM = 1, OP_MEANKEY = 2 };

// ---- programmatic dependent launch -------------------------------------------------------
// Kernels of one stream are chained with programmatic dependent launch.  Two kinds:
//   early: pdl_trigger() at entry, pdl_hold() at exit.  The body runs while the preceding
//          kernel may still run; it may read only data of kernels before the last "late" kernel.
//   late:  pdl_wait() at entry (after a prologue that reads no predecessor data), then
//          pdl_trigger().  Past the wait every earlier kernel of the stream is complete.
// A kernel launched without the attribute treats both instructions as no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// End of an early kernel: one thread of the first CTA waits, so the grid completes only after
// its predecessor has (completion stays transitive along the chain); the other CTAs leave freely.
__device__ __forceinline__ void pdl_hold() {
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) pdl_wait();
}

enum ErrBits : int {
    ERR_SEL_RANGE = 1,     // a selected unit id outside [0, n_mem)
    ERR_REP_RANGE = 2,     // a representative id outside [0, U)
    ERR_SPLIT_RANGE = 4,   // decode split bookkeeping out of range
    ERR_TILE_SCHED = 8,    // attention tile bookkeeping out of range
};

__device__ __forceinline__ void set_err(const Dev& D, int bit) { atomicOr(D.err, bit); }

// ---- element conversions --------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
// fp64 to the element type, one rounding (to nearest, ties to even)
template <typename T> __device__ __forceinline__ T from_d(double x);
template <> __device__ __forceinline__ float from_d<float>(double x) { return __double2float_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_d<__nv_bfloat16>(double x) { return __double2bfloat16(x); }

// ---- ordered composite keys for deterministic top-k ------------------------------------
// Larger key = better.  High word: order-preserving image of the float score (+0 == -0).
// Low word: ~index, so among equal scores the lower index wins.
__device__ __forceinline__ uint32_t ordered_bits(float s) {
    s = s + 0.0f;  // canonicalise -0 to +0
    uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint64_t make_key(float s, uint32_t idx) {
    return ((uint64_t)ordered_bits(s) << 32) | (uint64_t)(~idx);
}
__device__ __forceinline__ uint32_t key_index(uint64_t key) { return ~(uint32_t)(key & 0xffffffffu); }

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t x, int m) {
    return __shfl_xor_sync(0xffffffffu, x, m);
}
__device__ __forceinline__ uint64_t shfl64(uint64_t x, int src) { return __shfl_sync(0xffffffffu, x, src); }

// Sort one key per lane descending across the warp (bitonic network).
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            uint64_t o = shfl_xor64(x, j);
            bool desc = (lane & k) == 0;
            bool lower = (lane & j) == 0;
            uint64_t mx = x > o ? x : o, mn = x > o ? o : x;
            x = (lower == desc) ? mx : mn;
        }
    }
    return x;
}

// Merge two warp-wide descending lists (one element per lane) and keep the top 32, descending.
__device__ __forceinline__ uint64_t warp_merge_desc(uint64_t a, uint64_t b) {
    const int lane = threadIdx.x & 31;
    uint64_t br = shfl64(b, 31 - lane);
    uint64_t x = a > br ? a : br;  // bitonic sequence holding the top 32 of a U b
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        uint64_t o = shfl_xor64(x, j);
        bool lower = (lane & j) == 0;
        x = lower ? (x > o ? x : o) : (x > o ? o : x);
    }
    return x;
}

// Insert one candidate per lane (0 = none) into a running descending top-32 list.
__device__ __forceinline__ uint64_t warp_topk_insert(uint64_t list, uint64_t cand) {
    uint64_t thr = shfl64(list, 31);
    if (__ballot_sync(0xffffffffu, cand > thr) == 0u) return list;
    return warp_merge_desc(list, warp_sort_desc(cand));
}

// 16-byte asynchronous copy global -> shared, cached in L2 only (data other CTAs wrote this launch).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}
// Wait for every asynchronous copy this thread issued.
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, m));
    return x;
}

// Two consecutive elements as floats (a 4-byte bf16x2 or 8-byte float2 load; 2-element aligned).
__device__ __forceinline__ float2 ld2f(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ float2 ld2f(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ void st2f(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void st2f(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }

// (cos, sin)(t theta_i) in fp64 from the three digit tables, rounded to float.
__device__ __forceinline__ float2 cs_abs(const double2* tab, int half, int64_t t, int i) {
    const double2 a = tab[(size_t)(t & 2047) * half + i];
    const double2 b = tab[((size_t)2048 + ((t >> 11) & 2047)) * half + i];
    const double2 c = tab[((size_t)4096 + ((t >> 22) & 2047)) * half + i];
    const double re1 = a.x * b.x - a.y * b.y, im1 = a.x * b.y + a.y * b.x;
    const double re = re1 * c.x - im1 * c.y, im = re1 * c.y + im1 * c.x;
    return make_float2((float)re, (float)im);
}

__host__ __device__ __forceinline__ int64_t n_mem_at(int64_t c0, int S, int W, int U) {
    int64_t x = c0 - (int64_t)W - (int64_t)S;
    return x > 0 ? x / U : 0;
}

// Raise `kernel`'s dynamic shared-memory limit to `bytes` once per device (the attribute is per
// device; `done` holds one bit per device ordinal, ordinals >= 64 are set on every call).
template <typename... KArgs>
inline cudaError_t smem_limit_once(void (*kernel)(KArgs...), int bytes, std::atomic<unsigned long long>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// Launch `kernel` on `st`, with programmatic dependent launch when `pdl` is set.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                            Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace infllm
