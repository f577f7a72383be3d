// route_threshold.cu -- routing by the paper's own rule T = mu + c*sigma.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion", §3.2.2 Eq. (11): T = mu_u + c * sigma_u over one sample's token
// uncertainties; Eq. (12): m_i = [u_i < T], so u_i >= T goes dense.  sigma
// is the population standard deviation.  The dense count varies per sample.
//
// One CTA per sample.  u is read once from HBM (16-byte loads) into shared
// memory; the mean and then the squared deviations are summed in fp64 in a
// fixed order (per thread, then a shuffle tree, then a tree over the warps),
// so a call's result does not depend on timing; every u is compared with T
// in fp64; warp ballots compact both index lists in increasing order.
#include "heta_internal.cuh"

namespace heta {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

// Sum of one double per thread over the CTA, the same on every thread.
__device__ __forceinline__ double block_sum(double v, double *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    double t = scratch[lane];  // kWarps == 32
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    __syncthreads();  // scratch is reused by the next call
    return t;
}

__global__ void __launch_bounds__(kThreads, 1)
route_threshold_kernel(const float *__restrict__ u, int N, double c,
                       int32_t *__restrict__ counts, int32_t *__restrict__ dense_idx,
                       int32_t *__restrict__ local_idx, double *__restrict__ thresh,
                       uint8_t *__restrict__ mask, int32_t *status)
{
    extern __shared__ float vals[];
    __shared__ double red[kWarps];
    __shared__ uint32_t w_dense[kWarps], w_dense_before[kWarps];
    __shared__ int s_nan;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x;
    const float *ub = u + (size_t)b * N;
    if (tid == 0) s_nan = 0;
    __syncthreads();

    // ---- 1. u into shared memory (16-byte loads from the first aligned element)
    bool nan_seen = false;
    int head = 0;  // scalar elements before the first 16-byte boundary
    {
        const uintptr_t a = reinterpret_cast<uintptr_t>(ub);
        head = (int)(((16u - (a & 15u)) & 15u) >> 2);
        if (head > N) head = N;
    }
    if (tid < head) {
        const float f = __ldg(ub + tid);
        nan_seen |= (f != f);
        vals[tid] = f;
    }
    const int n4 = (N - head) >> 2;
    const float4 *u4 = reinterpret_cast<const float4 *>(ub + head);
    for (int v = tid; v < n4; v += kThreads) {
        const float4 f = __ldg(u4 + v);
        nan_seen |= (f.x != f.x) | (f.y != f.y) | (f.z != f.z) | (f.w != f.w);
        const int i = head + 4 * v;
        vals[i] = f.x;
        vals[i + 1] = f.y;
        vals[i + 2] = f.z;
        vals[i + 3] = f.w;
    }
    for (int i = head + 4 * n4 + tid; i < N; i += kThreads) {
        const float f = __ldg(ub + i);
        nan_seen |= (f != f);
        vals[i] = f;
    }
    if (nan_seen) s_nan = 1;
    __syncthreads();
    if (tid == 0 && s_nan) raise_status(status, HETA_ERR_NONFINITE);

    // ---- 2. mu, sigma (population) and T in fp64
    double part = 0.0;
    for (int i = tid; i < N; i += kThreads) part += (double)vals[i];
    const double mu = block_sum(part, red) / (double)N;
    part = 0.0;
    for (int i = tid; i < N; i += kThreads) {
        const double dev = (double)vals[i] - mu;
        part = fma(dev, dev, part);
    }
    const double sigma = sqrt(block_sum(part, red) / (double)N);
    const double T = __dadd_rn(mu, __dmul_rn(c, sigma));  // two roundings, as written
    if (tid == 0 && thresh) thresh[b] = T;

    // ---- 3. compaction: each warp owns one contiguous segment
    const int per_lane = (N + kThreads - 1) / kThreads;
    const int seg = 32 * per_lane;
    const int seg_lo = warp * seg;
    const int seg_hi = min(N, seg_lo + seg);
    uint32_t nd = 0;
    for (int i = seg_lo + lane; i < seg_hi; i += 32) nd += (double)vals[i] >= T;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nd += __shfl_xor_sync(0xffffffffu, nd, o);
    if (lane == 0) w_dense[warp] = nd;
    __syncthreads();
    if (warp == 0) {
        const uint32_t here = w_dense[lane];
        uint32_t incl = here;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        w_dense_before[lane] = incl - here;
        if (lane == 31) counts[b] = (int32_t)incl;
    }
    __syncthreads();

    const unsigned lt = (1u << lane) - 1u;
    uint32_t rd = w_dense_before[warp];
    int32_t *dout = dense_idx + (size_t)b * N;
    int32_t *lout = local_idx + (size_t)b * N;
    uint8_t *mout = mask ? mask + (size_t)b * N : nullptr;
    for (int base = seg_lo; base < seg_hi; base += 32) {
        const int i = base + lane;
        const bool valid = i < seg_hi;
        const bool dense = valid && (double)vals[i] >= T;
        const unsigned d_mask = __ballot_sync(0xffffffffu, dense);
        const uint32_t pos = rd + __popc(d_mask & lt);  // dense tokens before i
        if (dense)
            dout[pos] = i;
        else if (valid)
            lout[i - pos] = i;
        if (mout && valid) mout[i] = dense ? 0 : 1;
        rd += __popc(d_mask);
    }
}

}  // namespace

cudaError_t launch_route_threshold(const float *u, int B, int N, double c, int32_t *counts,
                                   int32_t *dense_idx, int32_t *local_idx, double *thresh,
                                   uint8_t *mask, int32_t *status, cudaStream_t s)
{
    const size_t smem = sizeof(float) * (size_t)N;
    cudaError_t e = cudaFuncSetAttribute(route_threshold_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(sizeof(float) * kRouteMaxN));
    if (e != cudaSuccess) return e;
    route_threshold_kernel<<<B, kThreads, smem, s>>>(u, N, c, counts, dense_idx, local_idx,
                                                     thresh, mask, status);
    return cudaGetLastError();
}

}  // namespace heta
