// Unit selection from per-CTA candidate lists (shared by the chunk and decode scoring kernels).
#pragma once

#include "common.cuh"

namespace infllm {

// Top-k of one KV head from the scoring CTAs' top-32 lists (composite keys, descending), run by
// the last scoring CTA of that head: warp w merges lists w, w + nw, ... (loads of a batch issued
// together), then the warp lists are merged pairwise in shared memory; the k ids are written in
// ascending order.  Ties go to the lower unit index.  Valid for k <= 32.
static __device__ void finish_select(const Dev& D, int hk, int n_mem, uint64_t (*lists)[32], int nw, uint64_t m,
                                     unsigned long long* slot_flags = nullptr, unsigned tag = 0);

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
    finish_select(D, hk, n_mem, lists, nw, m);
}

// As merge_select, for a CTA that can lend `stage` (room for `stage_lists` lists of 32 keys in shared
// memory): the lists are copied there in batches of 16-byte asynchronous copies, a batch in one round
// trip to L2, and each warp merges its lists of the batch (w, w + nw, ...) in four independent chains,
// so that consecutive merges do not wait for each other.
static __device__ void merge_select_staged(const Dev& D, int hk, int n_mem, int n_split, uint64_t (*lists)[32], int nw,
                                           uint64_t* stage, int stage_lists, unsigned long long* slot_flags,
                                           unsigned tag) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t* cb = D.cand + (int64_t)hk * D.score_splits_max * 32;
    uint64_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
    for (int b0 = 0; b0 < n_split; b0 += stage_lists) {
        const int nb = min(stage_lists, n_split - b0);
        if (b0 > 0) __syncthreads();  // the previous batch is merged
        for (int x = tid; x < nb * 16; x += nw * 32) cp_async16(stage + 2 * x, cb + (int64_t)b0 * 32 + 2 * x);
        cp_async_wait_all();
        __syncthreads();
        int sp = warp;
        for (; sp + 3 * nw < nb; sp += 4 * nw) {  // four independent merges per pass
            const uint64_t x0 = stage[sp * 32 + lane], x1 = stage[(sp + nw) * 32 + lane];
            const uint64_t x2 = stage[(sp + 2 * nw) * 32 + lane], x3 = stage[(sp + 3 * nw) * 32 + lane];
            m0 = warp_merge_desc(m0, x0);
            m1 = warp_merge_desc(m1, x1);
            m2 = warp_merge_desc(m2, x2);
            m3 = warp_merge_desc(m3, x3);
        }
        for (; sp < nb; sp += nw) m0 = warp_merge_desc(m0, stage[sp * 32 + lane]);
    }
    finish_select(D, hk, n_mem, lists, nw, warp_merge_desc(warp_merge_desc(m0, m1), warp_merge_desc(m2, m3)),
                  slot_flags, tag);
}

// The warps' merged lists -> the head's selection (k ids, ascending) in D.sel.  With `slot_flags`,
// selected slot i of the head is also published as (tag << 32) | id with a release store, so that a
// reader of the slot needs no other load.
static __device__ void finish_select(const Dev& D, int hk, int n_mem, uint64_t (*lists)[32], int nw, uint64_t m,
                                     unsigned long long* slot_flags, unsigned tag) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
            if (slot_flags && lane < kk)
                st_release64(slot_flags + hk * D.topk + lane, ((unsigned long long)tag << 32) | (uint32_t)o);
        }
    }
}

// This CTA's top-32 list of KV head hk goes to D.cand; the last CTA of the head to finish (device
// counter, threadfence pattern: no CTA waits for another) merges all lists into the selection and
// re-arms the counter for the next launch.  With `slot_flags`, the selection is published slot by
// slot there (see finish_select); with `stage` (room for `stage_lists` lists in shared memory), the
// merge stages the lists there first.
static __device__ void publish_and_select(const Dev& D, int hk, int split, int n_mem, int n_split,
                                          uint64_t (*lists)[32], int nw, unsigned long long* slot_flags = nullptr,
                                          unsigned tag = 0, uint64_t* stage = nullptr, int stage_lists = 0) {
    __shared__ int is_last;
    if (threadIdx.x < 32) D.cand[((int64_t)hk * D.score_splits_max + split) * 32 + threadIdx.x] = lists[0][threadIdx.x];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(&D.counters[hk], 1u) == (unsigned)(n_split - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (stage && stage_lists > 0)
        merge_select_staged(D, hk, n_mem, n_split, lists, nw, stage, stage_lists, slot_flags, tag);
    else
        merge_select(D, hk, n_mem, n_split, lists, nw);
    if (threadIdx.x == 0) D.counters[hk] = 0u;
}

}  // namespace infllm
