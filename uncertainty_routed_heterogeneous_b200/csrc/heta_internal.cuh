// heta_internal.cuh -- declarations shared by the libheta translation units.
// Not part of the public ABI (that is include/heta.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "heta.h"

namespace heta {

// Raises *status to `code` (atomic max), if a status word was given.
__device__ __forceinline__ void raise_status(int32_t *status, int32_t code)
{
    if (status) atomicMax(reinterpret_cast<int *>(status), code);
}

// Largest N one routing CTA can hold in shared memory (4 bytes per token).
constexpr int kRouteMaxN = 53248;

cudaError_t launch_route(const float *u, int B, int N, int k, int32_t *dense_idx,
                         int32_t *local_idx, float *thresh, uint8_t *mask,
                         int32_t *status, cudaStream_t s);

cudaError_t launch_uncertainty(const uint16_t *X, const float *w, float bias,
                               int B, int N, int C, float *u, cudaStream_t s);

struct AttnArgs {
    const uint16_t *Q, *K, *V;
    uint16_t *out;
    const int32_t *dense_idx;
    int32_t *status;
    int B, H, d, N, k;
    int Tg, Hg, Wg, wt, wh, ww;
    float scale;
};

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t s);

}  // namespace heta
