// C ABI of the InfLLM layer (include/infllm.h): argument and state checks, device buffers,
// kernel sequencing on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <numeric>
#include <vector>

#include "../../include/infllm.h"
#include "common.cuh"
#include "kernels.h"

using namespace infllm;

namespace {

enum Kind { K_APPEND = 0, K_REPS, K_PREP, K_SELECT, K_ATTEND, K_DECODE, K_NKIND };

struct EventPair {
    cudaEvent_t a, b;
    int kind;
};

}  // namespace

struct infllm_ctx {
    infllm_config cfg;
    cudaStream_t stream = nullptr;
    int device = 0;
    int elt = 0;
    Dev D{};
    std::vector<void*> allocs;
    void* tmaps = nullptr;      // tensor-core path descriptors (device copy)
    bool use_tc = false;
    int* err_host = nullptr;    // mapped pinned word
    // stream state
    int64_t tokens = 0;
    int64_t units_done = 0;
    bool pending = false;
    int32_t pending_n = 0;
    int64_t pending_c0 = 0;
    int32_t last_nmem = 0, last_kk = 0;
    int64_t last_B = 0, last_active = 0;
    bool attended = false;
    int64_t launches = 0;
    // launch chaining: within one API call every launch after the first may start early
    // (programmatic dependent launch); the first waits for whatever precedes it on the stream
    int chaining = 1;   // infllm_set_launch_chaining
    int prefill_lookup = 1;  // infllm_set_prefill_lookup: unit lookup for chunks (decode always looks up)
    bool chain = false; // a kernel of the current call has been launched
    // lookups so far: lookup L packs its queries into slot L % 3, sums them into buffer L % 2 and
    // writes its selection to buffer L % 2 (so a lookup can run while the previous attention reads)
    int64_t nlook = 0;
    int last_sel = 0;   // selection buffer of the last attended chunk or token
    int32_t* sel_base = nullptr;
    float* qbar_base = nullptr;
    // profiling
    int profiling = 0;  // bit mask of kernel classes (1 << Kind) bracketed with events
    std::vector<EventPair> events;
    std::vector<cudaEvent_t> pool;
    double ms[K_NKIND] = {0};
    int64_t cnt[K_NKIND] = {0};
    char err[512] = {0};
};

namespace {

infllm_status fail(infllm_ctx* c, infllm_status s, const char* fmt, ...) {
    if (c) {
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(c->err, sizeof(c->err), fmt, ap);
        va_end(ap);
    }
    return s;
}

#define CK(call)                                                                                      \
    do {                                                                                              \
        cudaError_t e_ = (call);                                                                      \
        if (e_ != cudaSuccess) return fail(c, INFLLM_ECUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

cudaEvent_t get_event(infllm_ctx* c) {
    if (!c->pool.empty()) {
        cudaEvent_t e = c->pool.back();
        c->pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Bracket a launch with events when profiling is on.
struct Prof {
    infllm_ctx* c;
    int kind;
    cudaEvent_t a = nullptr;
    Prof(infllm_ctx* c_, int k) : c(c_), kind(k) {
        if (c->profiling & (1 << kind)) {
            a = get_event(c);
            cudaEventRecord(a, c->stream);
        }
    }
    void done() {
        if (a) {
            cudaEvent_t b = get_event(c);
            cudaEventRecord(b, c->stream);
            c->events.push_back({a, b, kind});
            a = nullptr;
        }
    }
};

// Whether the next launch may be chained to the previous one (same API call).
bool pdl_ok(const infllm_ctx* c) { return c->chaining && c->chain; }

void collect_events(infllm_ctx* c) {
    if (c->events.empty()) return;
    cudaStreamSynchronize(c->stream);
    for (auto& ev : c->events) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, ev.a, ev.b) == cudaSuccess) {
            c->ms[ev.kind] += ms;
            c->cnt[ev.kind] += 1;
        }
        c->pool.push_back(ev.a);
        c->pool.push_back(ev.b);
    }
    c->events.clear();
}

template <typename P>
infllm_status dalloc(infllm_ctx* c, P** p, size_t bytes) {
    void* q = nullptr;
    cudaError_t e = cudaMalloc(&q, bytes < 16 ? 16 : bytes);
    if (e != cudaSuccess) return fail(c, INFLLM_ECUDA, "cudaMalloc(%zu): %s", bytes, cudaGetErrorString(e));
    c->allocs.push_back(q);
    *p = (P*)q;
    return INFLLM_OK;
}

infllm_status check_device_error(infllm_ctx* c) {
    if (c->err_host && *(volatile int*)c->err_host != 0)
        return fail(c, INFLLM_EDEVICE, "device-side check failed (error bits 0x%x)", *(volatile int*)c->err_host);
    return INFLLM_OK;
}

infllm_status validate(const infllm_config* g, char* msg, size_t n) {
    auto bad = [&](const char* m) {
        snprintf(msg, n, "invalid config: %s", m);
        return INFLLM_EINVAL;
    };
    if (g->n_q_heads <= 0 || g->n_kv_heads <= 0) return bad("head counts must be positive");
    if (g->n_q_heads % g->n_kv_heads) return bad("n_q_heads must be a multiple of n_kv_heads");
    if (g->n_q_heads / g->n_kv_heads > 128) return bad("at most 128 q heads per kv head");
    if (g->head_dim != 64 && g->head_dim != 128) return bad("head_dim must be 64 or 128");
    if (g->n_sink < 0) return bad("n_sink must be >= 0");
    if (g->window < 1) return bad("window must be >= 1");
    if (g->unit_size < 1 || g->unit_size > 1024) return bad("unit_size must be in [1, 1024]");
    if (g->n_reps < 1 || g->n_reps > 32 || g->n_reps > g->unit_size) return bad("n_reps must be in [1, min(32, unit_size)]");
    if (g->top_k < 0) return bad("top_k must be >= 0");
    if (g->max_chunk < 1) return bad("max_chunk must be >= 1");
    if (g->max_tokens < 1 || g->max_tokens > ((int64_t)1 << 31)) return bad("max_tokens must be in [1, 2^31]");
    if (!(g->rope_base > 1.0)) return bad("rope_base must be > 1");
    if (g->dtype != INFLLM_F32 && g->dtype != INFLLM_BF16) return bad("dtype must be INFLLM_F32 or INFLLM_BF16");
    if (g->score_mode != INFLLM_SCORE_REPS && g->score_mode != INFLLM_SCORE_REPSUM && g->score_mode != INFLLM_SCORE_MEANKEY)
        return bad("unknown score_mode");
    const int64_t units = g->max_tokens / g->unit_size + 1;
    if (units > 16384) return bad("at most 16384 memory units (max_tokens / unit_size)");
    return INFLLM_OK;
}

// The state of lookup L: its selection buffer and query-sum buffer in a copy of the device view.
Dev lookup_dev(const infllm_ctx* c, int64_t L) {
    Dev D = c->D;
    D.sel = c->sel_base + (size_t)(L & 1) * D.Hkv * std::max(1, D.topk);
    D.qbar_part = c->qbar_base + (size_t)(L & 1) * D.Hkv * D.qtiles_max * D.d;
    return D;
}

// a1 + a2 for tokens [tokens, tokens + n): representatives of every unit that becomes eligible
// at the chunk start (they use queries before it only), then the chunk's stores.
template <typename T>
infllm_status stage_store(infllm_ctx* c, const void* q, const void* k, const void* v, int32_t n) {
    const Dev& D = c->D;
    const int64_t c0 = c->tokens;
    const int64_t target = n_mem_at(c0, D.S, D.W, D.U);
    if (target > c->units_done) {
        Prof p(c, K_REPS);
        CK(launch_reps<T>(D, c->units_done, target, c->stream, pdl_ok(c)));
        c->chain = true;
        p.done();
        c->launches += 1;
        c->units_done = target;
    }
    Prof p(c, K_APPEND);
    CK(launch_append<T>(D, k, v, c0, n, c->stream, pdl_ok(c)));
    c->chain = true;
    int l = 0;
    CK(launch_ysum<T>(D, q, c0, n, c->stream, &l, pdl_ok(c)));
    p.done();
    c->launches += 1 + l;
    c->tokens = c0 + n;
    return INFLLM_OK;
}

// Packed, rotated queries of chunk [c0, c0 + n) for lookup L, and their per-tile sums.
template <typename T>
infllm_status stage_prep(infllm_ctx* c, const void* q, int64_t c0, int32_t n, int64_t L) {
    Prof p(c, K_PREP);
    CK(launch_prep<T>(lookup_dev(c, L), q, c0, n, (int)(L % 3), c->stream, pdl_ok(c)));
    c->chain = true;
    p.done();
    c->launches += 1;
    return INFLLM_OK;
}

// a3: unit scores and top-k of lookup L.  wait_first: the scoring needs its predecessor's results.
template <typename T>
infllm_status stage_select(infllm_ctx* c, int64_t L, int nm, int n_qtiles, const void* qraw, bool wait_first) {
    int l = 0;
    Prof p(c, K_SELECT);
    CK(launch_select<T>(lookup_dev(c, L), c->cfg.score_mode, nm, n_qtiles, qraw, c->stream, &l, pdl_ok(c),
                        wait_first));
    if (l > 0) c->chain = true;
    p.done();
    c->launches += l;
    return INFLLM_OK;
}

void record_attend(infllm_ctx* c, int64_t L, int64_t c0, int n, int nm, int kk, int64_t B) {
    c->last_nmem = nm;
    c->last_kk = kk;
    c->last_B = B;
    c->last_sel = (int)(L & 1);
    const int64_t t = c0 + n - 1;
    const int64_t s_eff = std::min<int64_t>(c->cfg.n_sink, t + 1);
    c->last_active = s_eff + (int64_t)kk * c->cfg.unit_size + std::max<int64_t>(0, t - B + 1);
    c->attended = true;
}

// a4: attention of chunk [c0, c0 + n) with lookup L's packed queries and selection.
template <typename T>
infllm_status stage_attend(infllm_ctx* c, int64_t L, int64_t c0, int32_t n, void* out, bool lookup) {
    const Dev D = lookup_dev(c, L);
    const int nm = (int)n_mem_at(c0, D.S, D.W, D.U);
    const int kk = lookup ? std::min(D.topk, nm) : 0;  // without lookup: sinks and window only
    const int64_t B = (int64_t)D.S + (int64_t)D.U * nm;
    Prof p(c, K_ATTEND);
    if constexpr (sizeof(T) == 2) {  // bf16: always the tensor cores (create refuses shapes they cannot take)
        CK(launch_attend_tc(D, c0, n, kk, B, (int)(L % 3), out, c->stream, c->tmaps, pdl_ok(c)));
    } else {  // fp32 operands: CUDA cores
        CK(launch_attend_simt<T>(D, c0, n, kk, B, (int)(L % 3), out, c->stream, pdl_ok(c)));
    }
    c->chain = true;
    p.done();
    c->launches += 1;
    record_attend(c, L, c0, n, nm, kk, B);
    return INFLLM_OK;
}

template <typename T>
infllm_status append_impl(infllm_ctx* c, const void* q, const void* k, const void* v, int32_t n) {
    const int64_t c0 = c->tokens;
    infllm_status s = stage_store<T>(c, q, k, v, n);
    if (s != INFLLM_OK) return s;
    c->pending = true;
    c->pending_n = n;
    c->pending_c0 = c0;
    return INFLLM_OK;
}

template <typename T>
infllm_status attend_impl(infllm_ctx* c, const void* q, int32_t n, void* out, bool decoding = false) {
    const Dev& D = c->D;
    const int64_t c0 = c->pending_c0;
    c->pending = false;
    if (n == 0) return INFLLM_OK;
    const int64_t L = c->nlook++;
    const int nm = (int)n_mem_at(c0, D.S, D.W, D.U);
    const bool lookup = decoding || c->prefill_lookup;
    infllm_status s = stage_prep<T>(c, q, c0, n, L);
    if (s == INFLLM_OK && lookup && std::min(D.topk, nm) > 0)
        s = stage_select<T>(c, L, nm, (n + D.qt - 1) / D.qt, nullptr, true);
    if (s == INFLLM_OK) s = stage_attend<T>(c, L, c0, n, out, lookup);
    return s;
}

// A whole prompt, one chunk ahead: after the first chunk the stream runs
//   attend(c-1) | store + pack (c+1) | lookup (c) | attend (c) | store + pack (c+2) | ...
// The lookup of chunk c reads only results of kernels before attend(c-1) (its representatives and
// query sums were made a chunk earlier), so it is chained to run alongside attend(c-1); the store
// side of chunk c+1 runs there as well.  Three query slots and two selection / query-sum buffers
// keep the overlapping chunks apart.  Every store side after the second follows an attention (a
// late kernel), so it starts only once the chunks before are complete; the second follows the
// first lookup, or is a plain launch.
template <typename T>
infllm_status prefill_impl(infllm_ctx* c, const char* q, const char* k, const char* v, int64_t n, int32_t chunk,
                           char* out) {
    const Dev& D = c->D;
    const size_t qrow = (size_t)D.Hq * D.d * c->elt, krow = (size_t)D.Hkv * D.d * c->elt;
    const int64_t N = (n + chunk - 1) / chunk, L0 = c->nlook, t0 = c->tokens;
    auto len = [&](int64_t i) { return (int32_t)std::min<int64_t>(chunk, n - i * chunk); };
    auto store_pack = [&](int64_t i) {
        const int64_t off = i * chunk;
        infllm_status s = stage_store<T>(c, q + off * qrow, k + off * krow, v + off * krow, len(i));
        return s == INFLLM_OK ? stage_prep<T>(c, q + off * qrow, t0 + off, len(i), L0 + i) : s;
    };
    const bool lk = c->prefill_lookup != 0;
    auto lookup = [&](int64_t i, bool wait_first) {
        const int64_t c0 = t0 + i * chunk;
        const int nm = (int)n_mem_at(c0, D.S, D.W, D.U);
        if (!lk || std::min(D.topk, nm) == 0) return INFLLM_OK;
        return stage_select<T>(c, L0 + i, nm, (len(i) + D.qt - 1) / D.qt, nullptr, wait_first);
    };
    infllm_status s = store_pack(0);
    const int64_t before = c->launches;
    if (s == INFLLM_OK) s = lookup(0, true);
    // chunk 1's store side (representatives from chunk 0's block sums) must see chunk 0 complete:
    // the first lookup waited for it; without one, chunk 1's first kernel is a plain launch
    if (c->launches == before) c->chain = false;
    for (int64_t i = 0; i < N && s == INFLLM_OK; ++i) {
        if (i + 1 < N) s = store_pack(i + 1);
        if (s == INFLLM_OK && i > 0) s = lookup(i, false);
        if (s == INFLLM_OK) s = stage_attend<T>(c, L0 + i, t0 + i * chunk, len(i), out + i * chunk * qrow, lk);
    }
    c->nlook = L0 + N;
    return s;
}

template <typename T>
infllm_status decode_impl(infllm_ctx* c, const void* q, const void* k, const void* v, void* out) {
    infllm_status s;
    if (sizeof(T) == 2 && c->use_tc && decode_tc_supported(c->D)) {
        // store + sink and window tiles (part 0) | lookup alongside | unit tiles + merge (part 1)
        const int64_t t = c->tokens;
        bool new_reps = false;  // the lookup then needs the representatives just computed
        {
            const Dev& D = c->D;
            const int64_t target = n_mem_at(t, D.S, D.W, D.U);
            if (target > c->units_done) {
                Prof p(c, K_REPS);
                CK(launch_reps<T>(D, c->units_done, target, c->stream, pdl_ok(c)));
                c->chain = true;
                p.done();
                c->launches += 1;
                c->units_done = target;
                new_reps = true;
            }
        }
        const int64_t L = c->nlook++;
        const Dev D = lookup_dev(c, L);
        const int nm = (int)n_mem_at(t, D.S, D.W, D.U);
        const int kk = std::min(D.topk, nm);
        const int64_t B = (int64_t)D.S + (int64_t)D.U * nm;
        {
            Prof p(c, K_DECODE);
            cudaError_t e = launch_decode_tc(D, q, k, v, t, kk, B, 0, out, c->stream, c->tmaps, pdl_ok(c));
            if (e != cudaSuccess) return fail(c, INFLLM_ECUDA, "decode launch (store, sinks, window): %s", cudaGetErrorString(e));
            c->chain = true;
            p.done();
            c->launches += 1;
        }
        c->tokens = t + 1;
        c->pending = false;
        if (kk > 0) {
            s = stage_select<T>(c, L, nm, 1, q, new_reps);
            if (s != INFLLM_OK) return s;
            Prof p(c, K_DECODE);
            cudaError_t e = launch_decode_tc(D, q, k, v, t, kk, B, 1, out, c->stream, c->tmaps, pdl_ok(c));
            if (e != cudaSuccess) return fail(c, INFLLM_ECUDA, "decode launch (units): %s", cudaGetErrorString(e));
            p.done();
            c->launches += 1;
        }
        record_attend(c, L, t, 1, nm, kk, B);
        return INFLLM_OK;
    }
    s = append_impl<T>(c, q, k, v, 1);
    if (s != INFLLM_OK) return s;
    const int64_t t = c->pending_c0;
    if (c->D.G > 8) {  // wide groups: the chunk kernels handle a single token as well
        return attend_impl<T>(c, q, 1, out, /*decoding=*/true);
    }
    c->pending = false;
    const int64_t L = c->nlook++;
    const Dev D = lookup_dev(c, L);
    const int nm = (int)n_mem_at(t, D.S, D.W, D.U);
    const int kk = std::min(D.topk, nm);
    const int64_t B = (int64_t)D.S + (int64_t)D.U * nm;
    if (kk > 0) {
        s = stage_select<T>(c, L, nm, 1, q, true);
        if (s != INFLLM_OK) return s;
    }
    Prof p(c, K_DECODE);
    int n_split = 0;
    cudaError_t e = launch_decode<T>(D, q, t, kk, B, out, c->stream, &n_split);
    if (e != cudaSuccess) return fail(c, INFLLM_ECUDA, "decode launch (%d splits): %s", n_split, cudaGetErrorString(e));
    p.done();
    c->launches += 1;
    record_attend(c, L, t, 1, nm, kk, B);
    return INFLLM_OK;
}

infllm_status zero_state(infllm_ctx* c) {
    CK(cudaMemsetAsync(c->D.Y, 0, sizeof(float) * (size_t)((c->D.T_max / c->D.gblk) + 2) * c->D.Hkv * c->D.d, c->stream));
    CK(cudaMemsetAsync(c->D.counters, 0, sizeof(unsigned) * 4 * c->D.Hkv, c->stream));
    CK(cudaMemsetAsync(c->D.simt_ctr, 0, sizeof(unsigned) * SIMT_PART_GROUPS, c->stream));
    CK(cudaMemsetAsync(c->sel_base, 0xff, sizeof(int32_t) * 2 * (size_t)c->D.Hkv * std::max(1, c->D.topk), c->stream));
    c->tokens = 0;
    c->units_done = 0;
    c->pending = false;
    c->pending_n = 0;
    c->attended = false;
    c->last_nmem = c->last_kk = 0;
    c->last_B = c->last_active = 0;
    c->nlook = 0;
    c->last_sel = 0;
    return INFLLM_OK;
}

void free_all(infllm_ctx* c) {
    for (void* p : c->allocs) cudaFree(p);
    c->allocs.clear();
    if (c->err_host) cudaFreeHost(c->err_host);
    free(c->tmaps);
    c->tmaps = nullptr;
    c->err_host = nullptr;
    for (auto& ev : c->events) {
        cudaEventDestroy(ev.a);
        cudaEventDestroy(ev.b);
    }
    c->events.clear();
    for (auto e : c->pool) cudaEventDestroy(e);
    c->pool.clear();
}

infllm_status create_impl(infllm_ctx* c) {
    const infllm_config& g = c->cfg;
    Dev& D = c->D;
    c->elt = g.dtype == INFLLM_BF16 ? 2 : 4;
    D.Hq = g.n_q_heads;
    D.Hkv = g.n_kv_heads;
    D.G = g.n_q_heads / g.n_kv_heads;
    D.d = g.head_dim;
    D.half = g.head_dim / 2;
    D.S = g.n_sink;
    D.W = g.window;
    D.U = g.unit_size;
    D.r = g.n_reps;
    D.topk = g.top_k;
    D.gblk = std::gcd(g.unit_size, g.window);
    D.T_max = g.max_tokens;
    D.units_max = g.max_tokens / g.unit_size + 1;
    D.inv_sqrt_d = (float)(1.0 / sqrt((double)g.head_dim));
    D.qt = std::max(1, 128 / D.G);
    const int rpt = D.qt * D.G;
    D.qtiles_max = (g.max_chunk + D.qt - 1) / D.qt;
    D.qrows_max = (int64_t)D.qtiles_max * rpt;
    D.score_splits_max = (int)((D.units_max + 3) / 4 + 1);  // up to 32 lanes per unit => 4 units per CTA
    const int SK = decode_split_keys(c->elt);
    D.dec_splits_max = (int)((std::min<int64_t>(g.n_sink, g.max_tokens) + (int64_t)g.top_k * g.unit_size +
                              (int64_t)g.window + g.unit_size + 1 + SK - 1) / SK) + 1;
    {   // tile-per-CTA decode: sink tiles + top_k * tiles per unit + window tiles
        const int64_t tiles = (std::min<int64_t>(g.n_sink, g.max_tokens) + 127) / 128 +
                              (int64_t)g.top_k * ((g.unit_size + 127) / 128) + ((int64_t)g.window + g.unit_size + 1 + 127) / 128 + 2;
        D.dec_splits_max = std::max<int>(D.dec_splits_max, (int)tiles);
    }
    D.P_rel = std::max(g.window, g.unit_size) + 1;

    CK(cudaGetDevice(&c->device));
    const size_t store = (size_t)D.Hkv * D.T_max * D.d * c->elt;
    infllm_status s;
#define AL(ptr, bytes)                         \
    if ((s = dalloc(c, &(ptr), (bytes))) != INFLLM_OK) return s;
    AL(D.Kraw, store);
    AL(D.Krot, store);
    AL(D.V, store);
    AL(D.Y, sizeof(float) * (size_t)((D.T_max / D.gblk) + 2) * D.Hkv * D.d);
    AL(D.rep_ids, sizeof(int32_t) * (size_t)D.Hkv * D.units_max * D.r);
    AL(D.rep_keys, (size_t)D.Hkv * D.units_max * D.r * D.d * c->elt);
    AL(D.repsum, sizeof(float) * (size_t)D.Hkv * D.units_max * D.d);
    AL(D.meankey, (size_t)D.Hkv * D.units_max * D.d * c->elt);
    AL(D.sel, sizeof(int32_t) * 2 * (size_t)D.Hkv * std::max(1, D.topk));  // two buffers
    AL(D.uscore, sizeof(float) * (size_t)D.Hkv * D.units_max);
    AL(D.qbar_part, sizeof(float) * 2 * (size_t)D.Hkv * D.qtiles_max * D.d);  // two buffers
    AL(D.cand, sizeof(uint64_t) * (size_t)D.Hkv * D.score_splits_max * 32);
    AL(D.counters, sizeof(unsigned) * 4 * D.Hkv);
    AL(D.simt_part, sizeof(float) * (size_t)SIMT_PART_GROUPS * 8 * (D.d + 2));
    AL(D.simt_ctr, sizeof(unsigned) * SIMT_PART_GROUPS);
    AL(D.Qm, (size_t)D.Hkv * 3 * D.qrows_max * D.d * c->elt);  // three slots
    AL(D.Qw, (size_t)D.Hkv * 3 * D.qrows_max * D.d * c->elt);
    AL(D.cs_chunk, sizeof(float2) * (size_t)g.max_chunk * D.half);
    AL(D.dec_part, sizeof(float) * (size_t)D.Hkv * D.dec_splits_max * D.G * (D.d + 4));


    double* invf = nullptr;
    float2* cs_rel = nullptr;
    float2* cs_w = nullptr;
    double2* cs3 = nullptr;
    AL(invf, sizeof(double) * D.half);
    AL(cs3, sizeof(double2) * 3 * 2048 * (size_t)D.half);
    AL(cs_rel, sizeof(float2) * (size_t)D.P_rel * D.half);
    AL(cs_w, sizeof(float2) * D.half);
#undef AL
    // position tables, fp64 on the host
    std::vector<double> th(D.half);
    for (int i = 0; i < D.half; ++i) th[i] = pow(g.rope_base, -2.0 * i / (double)D.d);
    std::vector<float2> rel((size_t)D.P_rel * D.half), w(D.half);
    for (int p = 0; p < D.P_rel; ++p)
        for (int i = 0; i < D.half; ++i) rel[(size_t)p * D.half + i] = make_float2((float)cos(p * th[i]), (float)sin(p * th[i]));
    for (int i = 0; i < D.half; ++i) w[i] = make_float2((float)cos(g.window * th[i]), (float)sin(g.window * th[i]));
    {
        std::vector<double2> t3((size_t)3 * 2048 * D.half);
        for (int L = 0; L < 3; ++L)
            for (int x = 0; x < 2048; ++x)
                for (int i = 0; i < D.half; ++i) {
                    const double ang = ldexp((double)x, 11 * L) * th[i];
                    t3[((size_t)L * 2048 + x) * D.half + i] = make_double2(cos(ang), sin(ang));
                }
        CK(cudaMemcpy(cs3, t3.data(), sizeof(double2) * t3.size(), cudaMemcpyHostToDevice));
        D.cs_abs3 = cs3;
    }
    CK(cudaMemcpy(invf, th.data(), sizeof(double) * D.half, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(cs_rel, rel.data(), sizeof(float2) * rel.size(), cudaMemcpyHostToDevice));
    CK(cudaMemcpy(cs_w, w.data(), sizeof(float2) * w.size(), cudaMemcpyHostToDevice));
    c->sel_base = D.sel;
    c->qbar_base = D.qbar_part;
    D.inv_freq = invf;
    D.cs_rel = cs_rel;
    D.cs_W = cs_w;
    CK(cudaHostAlloc((void**)&c->err_host, sizeof(int), cudaHostAllocMapped));
    *c->err_host = 0;
    CK(cudaHostGetDevicePointer((void**)&D.err, c->err_host, 0));
    c->use_tc = false;
    if (g.dtype == INFLLM_BF16) {
        if (!attend_tc_supported(D))
            return fail(c, INFLLM_EINVAL, "bf16 needs the tensor-core attention: head_dim 64 or 128, "
                        "q heads per KV head dividing 128, top_k <= 4096, an sm_100 device");
        c->tmaps = malloc(tc_maps_size());
        c->use_tc = c->tmaps && make_tc_maps(D, c->tmaps);
        if (!c->use_tc) return fail(c, INFLLM_ECUDA, "tensor map encoding failed");
    }
    infllm_status zs = zero_state(c);
    if (zs != INFLLM_OK) return zs;
    CK(cudaStreamSynchronize(c->stream));
    return INFLLM_OK;
}

}  // namespace

extern "C" {

const char* infllm_version(void) { return "infllm-b200 0.1"; }

const char* infllm_last_error(infllm_ctx* ctx) { return ctx ? ctx->err : "null context"; }

infllm_status infllm_create(const infllm_config* cfg, void* cuda_stream, infllm_ctx** out) {
    if (!out) return INFLLM_EINVAL;
    *out = nullptr;
    if (!cfg) return INFLLM_EINVAL;
    char msg[256];
    infllm_status s = validate(cfg, msg, sizeof(msg));
    if (s != INFLLM_OK) return s;
    infllm_ctx* c = new infllm_ctx();
    c->cfg = *cfg;
    c->stream = (cudaStream_t)cuda_stream;
    s = create_impl(c);
    if (s != INFLLM_OK) {
        fprintf(stderr, "infllm_create: %s\n", c->err);
        free_all(c);
        delete c;
        return s;
    }
    *out = c;
    return INFLLM_OK;
}

infllm_status infllm_destroy(infllm_ctx* c) {
    if (!c) return INFLLM_OK;
    cudaStreamSynchronize(c->stream);
    free_all(c);
    delete c;
    return INFLLM_OK;
}

infllm_status infllm_reset(infllm_ctx* c) {
    if (!c) return INFLLM_EINVAL;
    return zero_state(c);
}

infllm_status infllm_append_chunk(infllm_ctx* c, const void* q, const void* k, const void* v, int32_t n) {
    if (!c) return INFLLM_EINVAL;
    c->chain = false;
    infllm_status s = check_device_error(c);
    if (s != INFLLM_OK) return s;
    if (n < 0) return fail(c, INFLLM_EINVAL, "append: n = %d < 0", n);
    if (n > c->cfg.max_chunk) return fail(c, INFLLM_EINVAL, "append: n = %d > max_chunk = %d", n, c->cfg.max_chunk);
    if (c->tokens + n > c->cfg.max_tokens)
        return fail(c, INFLLM_ECAPACITY, "append: %lld + %d tokens exceed max_tokens = %lld", (long long)c->tokens, n,
                    (long long)c->cfg.max_tokens);
    if (n == 0) {
        c->pending = true;
        c->pending_n = 0;
        c->pending_c0 = c->tokens;
        return INFLLM_OK;
    }
    if (!q || !k || !v) return fail(c, INFLLM_EINVAL, "append: null pointer");
    return c->cfg.dtype == INFLLM_BF16 ? append_impl<__nv_bfloat16>(c, q, k, v, n) : append_impl<float>(c, q, k, v, n);
}

infllm_status infllm_attend_chunk(infllm_ctx* c, const void* q, int32_t n, void* out) {
    if (!c) return INFLLM_EINVAL;
    c->chain = false;
    infllm_status s = check_device_error(c);
    if (s != INFLLM_OK) return s;
    if (!c->pending) return fail(c, INFLLM_ESTATE, "attend: no appended chunk is waiting");
    if (n != c->pending_n)
        return fail(c, INFLLM_ESTATE, "attend: n = %d does not match the appended chunk (%d)", n, c->pending_n);
    if (n > 0 && (!q || !out)) return fail(c, INFLLM_EINVAL, "attend: null pointer");
    return c->cfg.dtype == INFLLM_BF16 ? attend_impl<__nv_bfloat16>(c, q, n, out) : attend_impl<float>(c, q, n, out);
}

infllm_status infllm_decode_step(infllm_ctx* c, const void* q, const void* k, const void* v, void* out) {
    if (!c) return INFLLM_EINVAL;
    c->chain = false;
    infllm_status s = check_device_error(c);
    if (s != INFLLM_OK) return s;
    if (!q || !k || !v || !out) return fail(c, INFLLM_EINVAL, "decode: null pointer");
    if (c->cfg.max_chunk < 1) return fail(c, INFLLM_EINVAL, "decode: max_chunk < 1");
    if (c->tokens + 1 > c->cfg.max_tokens)
        return fail(c, INFLLM_ECAPACITY, "decode: max_tokens = %lld reached", (long long)c->cfg.max_tokens);
    return c->cfg.dtype == INFLLM_BF16 ? decode_impl<__nv_bfloat16>(c, q, k, v, out) : decode_impl<float>(c, q, k, v, out);
}

infllm_status infllm_prefill(infllm_ctx* c, const void* q, const void* k, const void* v, int64_t n, int32_t chunk,
                             void* out) {
    if (!c) return INFLLM_EINVAL;
    c->chain = false;
    infllm_status s = check_device_error(c);
    if (s != INFLLM_OK) return s;
    if (n < 0) return fail(c, INFLLM_EINVAL, "prefill: n = %lld < 0", (long long)n);
    if (chunk < 1 || chunk > c->cfg.max_chunk)
        return fail(c, INFLLM_EINVAL, "prefill: chunk = %d not in [1, max_chunk = %d]", chunk, c->cfg.max_chunk);
    if (c->tokens + n > c->cfg.max_tokens)
        return fail(c, INFLLM_ECAPACITY, "prefill: %lld + %lld tokens exceed max_tokens = %lld", (long long)c->tokens,
                    (long long)n, (long long)c->cfg.max_tokens);
    if (n == 0) return INFLLM_OK;
    if (!q || !k || !v || !out) return fail(c, INFLLM_EINVAL, "prefill: null pointer");
    c->pending = false;  // a chunk appended and not attended stays in the context without its outputs
    return c->cfg.dtype == INFLLM_BF16
               ? prefill_impl<__nv_bfloat16>(c, (const char*)q, (const char*)k, (const char*)v, n, chunk, (char*)out)
               : prefill_impl<float>(c, (const char*)q, (const char*)k, (const char*)v, n, chunk, (char*)out);
}

infllm_status infllm_get_selection(infllm_ctx* c, int32_t* host_sel) {
    if (!c || !host_sel) return INFLLM_EINVAL;
    if (c->cfg.top_k == 0) return INFLLM_OK;
    CK(cudaStreamSynchronize(c->stream));
    CK(cudaMemcpy(host_sel, c->sel_base + (size_t)c->last_sel * c->D.Hkv * std::max(1, c->D.topk),
                  sizeof(int32_t) * (size_t)c->D.Hkv * c->D.topk, cudaMemcpyDeviceToHost));
    // entries beyond the last chunk's selection are not rewritten by the kernels
    for (int h = 0; h < c->D.Hkv; ++h)
        for (int i = c->last_kk; i < c->D.topk; ++i) host_sel[h * c->D.topk + i] = -1;
    return check_device_error(c);
}

infllm_status infllm_get_unit_scores(infllm_ctx* c, float* host_scores, int32_t capacity, int32_t* n_mem_out) {
    if (!c || !n_mem_out) return INFLLM_EINVAL;
    *n_mem_out = c->last_nmem;
    if (!host_scores) return INFLLM_OK;
    if (capacity < c->last_nmem) return fail(c, INFLLM_EINVAL, "unit scores: capacity %d < n_mem %d", capacity, c->last_nmem);
    if (c->last_nmem == 0 || c->cfg.top_k == 0) return INFLLM_OK;
    CK(cudaStreamSynchronize(c->stream));
    CK(cudaMemcpy2D(host_scores, sizeof(float) * c->last_nmem, c->D.uscore, sizeof(float) * c->D.units_max,
                    sizeof(float) * c->last_nmem, c->D.Hkv, cudaMemcpyDeviceToHost));
    return check_device_error(c);
}

infllm_status infllm_get_reps(infllm_ctx* c, int32_t unit_begin, int32_t n_units, int32_t* host_ids) {
    if (!c || !host_ids || unit_begin < 0 || n_units < 0) return INFLLM_EINVAL;
    if ((int64_t)unit_begin + n_units > c->units_done)
        return fail(c, INFLLM_ESTATE, "reps: units [%d, %d) requested, %lld have representatives", unit_begin,
                    unit_begin + n_units, (long long)c->units_done);
    if (n_units == 0) return INFLLM_OK;
    CK(cudaStreamSynchronize(c->stream));
    const size_t row = sizeof(int32_t) * (size_t)n_units * c->D.r;
    CK(cudaMemcpy2D(host_ids, row, c->D.rep_ids + (size_t)unit_begin * c->D.r, sizeof(int32_t) * (size_t)c->D.units_max * c->D.r,
                    row, c->D.Hkv, cudaMemcpyDeviceToHost));
    return check_device_error(c);
}

infllm_status infllm_get_stats(infllm_ctx* c, infllm_stats* o) {
    if (!c || !o) return INFLLM_EINVAL;
    collect_events(c);
    memset(o, 0, sizeof(*o));
    o->tokens = c->tokens;
    o->units_with_reps = c->units_done;
    o->n_mem = c->last_nmem;
    o->n_selected = c->last_kk;
    o->window_base = c->last_B;
    o->active_tokens = c->last_active;
    o->kernel_launches = c->launches;
    o->attend_path = c->use_tc ? 1 : 0;
    o->score_mode = c->cfg.score_mode;
    o->ms_append = c->ms[K_APPEND];
    o->ms_reps = c->ms[K_REPS];
    o->ms_prep = c->ms[K_PREP];
    o->ms_select = c->ms[K_SELECT];
    o->ms_attend = c->ms[K_ATTEND];
    o->ms_decode = c->ms[K_DECODE];
    o->n_append = c->cnt[K_APPEND];
    o->n_reps = c->cnt[K_REPS];
    o->n_prep = c->cnt[K_PREP];
    o->n_select = c->cnt[K_SELECT];
    o->n_attend = c->cnt[K_ATTEND];
    o->n_decode = c->cnt[K_DECODE];
    return INFLLM_OK;
}

infllm_status infllm_set_score_mode(infllm_ctx* c, int32_t mode) {
    if (!c) return INFLLM_EINVAL;
    if (mode != INFLLM_SCORE_REPS && mode != INFLLM_SCORE_REPSUM && mode != INFLLM_SCORE_MEANKEY)
        return fail(c, INFLLM_EINVAL, "unknown score_mode %d", mode);
    c->cfg.score_mode = mode;
    return INFLLM_OK;
}

infllm_status infllm_set_prefill_lookup(infllm_ctx* c, int32_t enable) {
    if (!c) return INFLLM_EINVAL;
    c->prefill_lookup = enable ? 1 : 0;
    return INFLLM_OK;
}

infllm_status infllm_set_launch_chaining(infllm_ctx* c, int32_t enable) {
    if (!c) return INFLLM_EINVAL;
    c->chaining = enable ? 1 : 0;
    return INFLLM_OK;
}

infllm_status infllm_set_profiling(infllm_ctx* c, int32_t enable) {
    if (!c) return INFLLM_EINVAL;
    collect_events(c);
    // 1 = every kernel class; otherwise bit (k + 1) selects class k (INFLLM_PROFILE_* in the header)
    c->profiling = enable == 1 ? ((1 << K_NKIND) - 1) : ((enable >> 1) & ((1 << K_NKIND) - 1));
    for (int k = 0; k < K_NKIND; ++k) {
        c->ms[k] = 0;
        c->cnt[k] = 0;
    }
    c->launches = 0;
    return INFLLM_OK;
}

}  // extern "C"
