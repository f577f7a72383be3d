// radix_select.cuh -- the block-wide step shared by the radix selections
// (top-k routing, the per-block random swap): given a histogram of the next
// digit of the keys still in the running, find the digit that holds the
// r-th largest of them.  Device code only; included by the .cu files.
#pragma once

#include <cstdint>

namespace heta {

// The digit of the r-th largest key among those counted in hist[0..nbins)
// (nbins = 1024 or 2048): *digit and *rank_in_digit (1-based) for the next
// pass.  Bins are scanned from the top; every thread of the CTA calls this.
template <int kThreads>
__device__ __forceinline__ void find_digit(const uint32_t *hist, int nbins, uint32_t r,
                                           uint32_t *warp_tot, uint32_t *s_digit,
                                           uint32_t *s_rank)
{
    static_assert(kThreads == 1024, "one warp total per lane of the final scan");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = nbins / kThreads;  // 1 or 2 bins per thread, descending
    uint32_t c[2] = {0u, 0u}, sum = 0u;
    for (int j = 0; j < per; ++j) {
        c[j] = hist[nbins - 1 - per * tid - j];
        sum += c[j];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    uint32_t wbefore = 0u;
    {
        const uint32_t wt = warp_tot[lane];
        uint32_t wi = wt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        wbefore = __shfl_sync(0xffffffffu, wi - wt, warp);
    }
    const uint32_t before = wbefore + incl - sum;
    if (before < r && r <= before + sum) {
        uint32_t acc = before;
        for (int j = 0; j < per; ++j) {
            if (acc < r && r <= acc + c[j]) {
                *s_digit = (uint32_t)(nbins - 1 - per * tid - j);
                *s_rank = r - acc;
            }
            acc += c[j];
        }
    }
    __syncthreads();
}

}  // namespace heta
