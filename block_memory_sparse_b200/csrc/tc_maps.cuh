// TMA descriptors of the context's K/V stores and packed query buffers (bf16, head dim 128,
// boxes of 64 columns x 128 rows, 128-byte swizzle), shared by the prefill and decode kernels.
#pragma once

#include <cuda.h>

namespace infllm {

struct TcMaps {
    CUtensorMap kraw, krot, v, qm, qw;
};


}  // namespace infllm
