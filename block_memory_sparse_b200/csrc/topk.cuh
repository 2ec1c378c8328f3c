// Unit selection from per-CTA candidate lists (shared by the chunk and decode scoring kernels).
#pragma once

#include "common.cuh"

namespace infllm {

// Top-k of one KV head from the scoring CTAs' top-32 lists (composite keys, descending), run by
// the last scoring CTA of that head: warp w merges lists w, w + nw, ... (loads of a batch issued
// together), then the warp lists are merged pairwise in shared memory; the k ids are written in
// ascending order.  Ties go to the lower unit index.  Valid for k <= 32.
static __device__ void merge_select(const Dev& D, int hk, int n_mem, int n_split, uint64_t (*lists)[32], int nw) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t* cb = D.cand + (int64_t)hk * D.score_splits_max * 32 + lane;
    uint64_t m = 0;
    for (int s0 = warp; s0 < n_split; s0 += nw * 4) {
        uint64_t b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int sp = s0 + nw * u;
            b[u] = sp < n_split ? __ldcg(cb + (int64_t)sp * 32) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (s0 + nw * u < n_split) m = warp_merge_desc(m, b[u]);
    }
    __syncthreads();  // the caller's use of lists[] is over
    lists[warp][lane] = m;
    for (int stride = 1; stride < nw; stride *= 2) {
        __syncthreads();
        if ((warp % (2 * stride)) == 0 && warp + stride < nw)
            lists[warp][lane] = warp_merge_desc(lists[warp][lane], lists[warp + stride][lane]);
    }
    __syncthreads();
    if (warp == 0) {
        const int kk = min(D.topk, n_mem);
        uint64_t sk = (lane < kk) ? (uint64_t)(0xffffffffu - key_index(lists[0][lane])) : 0ull;
        sk = warp_sort_desc(sk);  // ascending ids
        if (lane < D.topk) {
            int o = -1;
            if (lane < kk) {
                o = (int)(0xffffffffu - (uint32_t)sk);
                if (o < 0 || o >= n_mem) {
                    set_err(D, ERR_SEL_RANGE);
                    o = 0;
                }
            }
            D.sel[hk * D.topk + lane] = o;
        }
    }
}

// This CTA's top-32 list of KV head hk goes to D.cand; the last CTA of the head to finish (device
// counter, threadfence pattern: no CTA waits for another) merges all lists into the selection and
// re-arms the counter for the next launch.
static __device__ void publish_and_select(const Dev& D, int hk, int split, int n_mem, int n_split,
                                          uint64_t (*lists)[32], int nw) {
    __shared__ int is_last;
    if (threadIdx.x < 32) D.cand[((int64_t)hk * D.score_splits_max + split) * 32 + threadIdx.x] = lists[0][threadIdx.x];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(&D.counters[hk], 1u) == (unsigned)(n_split - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    merge_select(D, hk, n_mem, n_split, lists, nw);
    if (threadIdx.x == 0) D.counters[hk] = 0u;
}

}  // namespace infllm
