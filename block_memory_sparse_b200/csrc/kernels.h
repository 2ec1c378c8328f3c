// Host-side launchers of the layer kernels (implemented in the .cu files of this directory).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace infllm {

template <typename T>
cudaError_t launch_append(const Dev& D, const void* k, const void* v, int64_t c0, int n, cudaStream_t st, bool pdl);
template <typename T>
cudaError_t launch_ysum(const Dev& D, const void* q, int64_t c0, int n, cudaStream_t st, int* launches, bool pdl);
template <typename T>
cudaError_t launch_reps(const Dev& D, int64_t j0, int64_t j1, cudaStream_t st, bool pdl);

// Rotated, packed queries of the chunk into query slot `par` (0..2) + per-tile raw query sums.
template <typename T>
cudaError_t launch_prep(const Dev& D, const void* q, int64_t c0, int n, int par, cudaStream_t st, bool pdl);

// Unit scores and top-k selection.  `qraw` != null: single-token query (decode) summed in place
// of the per-tile partials.  Returns the number of kernels launched in *launches.  With `pdl` the
// scoring kernel is chained to its predecessor: it waits for it at entry when `wait_first` (it
// needs that kernel's results), else it scores first and only holds its completion.
template <typename T>
cudaError_t launch_select(const Dev& D, int score_mode, int n_mem, int n_qtiles, const void* qraw,
                          cudaStream_t st, int* launches, bool pdl, bool wait_first);

// Exact attention over sinks U selected units U window for a chunk (SIMT fp32-accumulate path).
template <typename T>
cudaError_t launch_attend_simt(const Dev& D, int64_t c0, int n, int kk, int64_t B, int par, void* out, cudaStream_t st,
                               bool pdl);

// Exact attention for a chunk on the tcgen05 tensor cores (bf16 in, fp32 accumulate).
cudaError_t launch_attend_tc(const Dev& D, int64_t c0, int n, int kk, int64_t B, int par, void* out, cudaStream_t st,
                             const void* tmaps, bool pdl);
bool attend_tc_supported(const Dev& D);
size_t tc_maps_size();
bool make_tc_maps(const Dev& D, void* out);  // TMA descriptors of the stores and packed queries

// Split-KV decode attention for one token with a log-sum-exp merge.
template <typename T>
cudaError_t launch_decode(const Dev& D, const void* q, int64_t t, int kk, int64_t B, void* out, cudaStream_t st,
                          int* n_split_out);

int decode_split_keys(int elt_bytes);

// Decode on the TMA path (bf16, head dim 128, G <= 8): split-KV attention over 128-key tiles.
// part 0: the sink and window tiles; stores the token (k, v, its query block sum) and merges the
//         tiles' partials (into the output when kk == 0); runs alongside the lookup.
// part 1: the selected units' tiles, then the merge with part 0's partial into `out`.
bool decode_tc_supported(const Dev& D);
cudaError_t launch_decode_tc(const Dev& D, const void* q, const void* k, const void* v, int64_t t, int kk, int64_t B,
                             int part, void* out, cudaStream_t st, const void* tmaps, bool pdl);

}  // namespace infllm
