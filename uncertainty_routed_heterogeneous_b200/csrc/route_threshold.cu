// route_threshold.cu -- routing by the paper's own rule T = mu + c*sigma.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion", §3.2.2 Eq. (11): T = mu_u + c * sigma_u over one sample's token
// uncertainties; Eq. (12): m_i = [u_i < T], so u_i >= T goes dense.  sigma
// is the population standard deviation.  The dense count varies per sample.
//
// The sums run in one fixed order, whatever the kernel: the sample is cut
// into eight slices of ceil(N/8) tokens; in each slice thread t (of 1024)
// adds its tokens t, t+1024, ... in fp64, a shuffle tree sums each warp and
// a second tree the 32 warps; the eight slice sums are added in slice order.
// Up to eight samples a call, and for samples too large for one CTA's
// shared memory, the slices are the eight CTAs of a cluster (their sums and
// dense counts exchanged through distributed shared memory); otherwise one
// CTA per sample computes the same eight slice sums.  Either
// way the same T comes out of the same u.  Every u is compared with T in
// fp64; warp ballots compact both index lists in increasing order.
#include "heta_internal.cuh"

namespace heta {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kSlices = 8;
constexpr unsigned kFull = 0xffffffffu;

// The sum over the CTA of one double per thread, in every thread: a
// shuffle tree in each warp, then the same tree over the warps' sums.
__device__ __forceinline__ double block_sum(double v, double *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    double t = scratch[lane];  // kWarps == 32
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(kFull, t, o);
    __syncthreads();  // scratch is reused by the next call
    return t;
}

// This thread's fp64 partial over tokens [lo, hi) (token i at vals[i - vbase]):
// tokens lo + t, lo + t + 1024, ...; kDev: the sum of (x - mu)^2 instead of x.
template <bool kDev>
__device__ __forceinline__ double slice_part(const float *vals, int vbase, int lo, int hi,
                                             double mu)
{
    double part = 0.0;
    for (int i = lo + (int)threadIdx.x; i < hi; i += kThreads) {
        const double x = (double)vals[i - vbase];
        if (kDev) {
            const double dev = x - mu;
            part = fma(dev, dev, part);
        } else {
            part += x;
        }
    }
    return part;
}

// Ballot compaction of one warp's tokens [lo, hi) of a sample: dense when
// u >= T; rd dense tokens of the sample lie before the warp's first token.
__device__ __forceinline__ void compact_threshold(const float *vals, int vbase, int lo, int hi,
                                                  double T, uint32_t rd, int32_t *dout,
                                                  int32_t *lout, uint8_t *mout, int lane)
{
    const unsigned lt = (1u << lane) - 1u;
    for (int base = lo; base < hi; base += 32) {  // warp-uniform
        const int i = base + lane;
        const bool valid = i < hi;
        const bool dense = valid && (double)vals[i - vbase] >= T;
        const unsigned d_mask = __ballot_sync(kFull, dense);
        const uint32_t pos = rd + __popc(d_mask & lt);  // dense tokens before i
        if (dense)
            dout[pos] = i;
        else if (valid)
            lout[i - pos] = i;
        if (mout && valid) mout[i] = dense ? 0 : 1;
        rd += __popc(d_mask);
    }
}

// ---------------------------------------------------------------- one CTA a sample

__global__ void __launch_bounds__(kThreads, 1)
route_threshold_kernel(const float *__restrict__ u, int N, double c,
                       int32_t *__restrict__ counts, int32_t *__restrict__ dense_idx,
                       int32_t *__restrict__ local_idx, double *__restrict__ thresh,
                       uint8_t *__restrict__ mask, int32_t *status)
{
    extern __shared__ float vals[];
    __shared__ double red[kSlices][kWarps];
    __shared__ double s_slice[kSlices];
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

    // ---- 2. mu, sigma and T: eight slice sums, each by the tree of a CTA
    const int L = (N + kSlices - 1) / kSlices;
    double mu = 0.0, sigma = 0.0;
    for (int pass = 0; pass < 2; ++pass) {
        double part[kSlices];
#pragma unroll
        for (int r = 0; r < kSlices; ++r) {
            const int lo = min(N, r * L), hi = min(N, lo + L);
            part[r] = pass == 0 ? slice_part<false>(vals, 0, lo, hi, 0.0)
                                : slice_part<true>(vals, 0, lo, hi, mu);
        }
        // Each slice's warp sum, by the same xor tree as block_sum (lane l
        // adds lane l^o's value at level o), with the eight slices spread
        // over the lanes as the tree goes: at levels 16, 8 and 4 a lane keeps
        // half of its slices and receives its partner's copies of them, so
        // every addition is the tree's own, in the same order.
        double q4[4], q2[2];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool hi16 = lane & 16;
            const double send = hi16 ? part[j] : part[j + 4];
            const double keep = hi16 ? part[j + 4] : part[j];
            q4[j] = keep + __shfl_xor_sync(kFull, send, 16);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const bool hi8 = lane & 8;
            const double send = hi8 ? q4[j] : q4[j + 2];
            const double keep = hi8 ? q4[j + 2] : q4[j];
            q2[j] = keep + __shfl_xor_sync(kFull, send, 8);
        }
        double q1;
        {
            const bool hi4 = lane & 4;
            const double send = hi4 ? q2[0] : q2[1];
            const double keep = hi4 ? q2[1] : q2[0];
            q1 = keep + __shfl_xor_sync(kFull, send, 4);
        }
        q1 += __shfl_xor_sync(kFull, q1, 2);
        q1 += __shfl_xor_sync(kFull, q1, 1);
        // lane l now holds the warp sum of slice 4*bit4 + 2*bit3 + bit2 of l
        if ((lane & 3) == 0) red[((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1)][warp] = q1;
        __syncthreads();
        if (warp < kSlices) {
            double t = red[warp][lane];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(kFull, t, o);
            if (lane == 0) s_slice[warp] = t;
        }
        __syncthreads();
        double total = 0.0;
#pragma unroll
        for (int r = 0; r < kSlices; ++r) total += s_slice[r];
        if (pass == 0) mu = total / (double)N;
        else sigma = sqrt(total / (double)N);
        __syncthreads();  // red and s_slice are reused by the next pass
    }
    const double T = __dadd_rn(mu, __dmul_rn(c, sigma));  // two roundings, as written
    if (tid == 0 && thresh) thresh[b] = T;

    // ---- 3. compaction: each warp owns one contiguous segment
    const int per_lane = (N + kThreads - 1) / kThreads;
    const int seg = 32 * per_lane;
    const int seg_lo = min(N, warp * seg);
    const int seg_hi = min(N, seg_lo + seg);
    uint32_t nd = 0;
    for (int i = seg_lo + lane; i < seg_hi; i += 32) nd += (double)vals[i] >= T;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nd += __shfl_xor_sync(kFull, nd, o);
    if (lane == 0) w_dense[warp] = nd;
    __syncthreads();
    if (warp == 0) {
        const uint32_t here = w_dense[lane];
        uint32_t incl = here;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += t;
        }
        w_dense_before[lane] = incl - here;
        if (lane == 31) counts[b] = (int32_t)incl;
    }
    __syncthreads();
    compact_threshold(vals, 0, seg_lo, seg_hi, T, w_dense_before[warp],
                      dense_idx + (size_t)b * N, local_idx + (size_t)b * N,
                      mask ? mask + (size_t)b * N : nullptr, lane);
}

// ------------------------------------------------------- a cluster of CTAs a sample

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// CTA `rank`'s copy of the shared variable at p (a generic address).
template <class T>
__device__ __forceinline__ const T *peer(const T *p, uint32_t rank)
{
    uint64_t r;
    asm("mapa.u64 %0, %1, %2;" : "=l"(r) : "l"(reinterpret_cast<uint64_t>(p)), "r"(rank));
    return reinterpret_cast<const T *>(r);
}

// CTA r of the cluster holds slice r of the sample.  Every cluster barrier
// is reached by every thread of every CTA, unconditionally.
__global__ void __launch_bounds__(kThreads, 1)
route_threshold_cluster_kernel(const float *__restrict__ u, int N, double c,
                               int32_t *__restrict__ counts, int32_t *__restrict__ dense_idx,
                               int32_t *__restrict__ local_idx, double *__restrict__ thresh,
                               uint8_t *__restrict__ mask, int32_t *status)
{
    extern __shared__ float vals[];  // this CTA's slice
    __shared__ double red[kWarps];
    __shared__ double s_sum[2];      // this CTA's slice sum of u, of (u - mu)^2
    __shared__ uint32_t s_nd;        // this CTA's dense tokens
    __shared__ uint32_t w_dense[kWarps], w_dense_before[kWarps];
    __shared__ int s_nan;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_rank();
    const int b = blockIdx.x / kSlices;
    const float *ub = u + (size_t)b * N;
    const int L = (N + kSlices - 1) / kSlices;
    const int lo = min(N, (int)rank * L), hi = min(N, lo + L);
    if (tid == 0) s_nan = 0;
    __syncthreads();

    // ---- 1. the slice into shared memory (vals[i - lo] = u[i])
    bool nan_seen = false;
    for (int i = lo + tid; i < hi; i += kThreads) {
        const float f = __ldg(ub + i);
        nan_seen |= (f != f);
        vals[i - lo] = f;
    }
    if (nan_seen) s_nan = 1;
    __syncthreads();
    if (tid == 0 && s_nan) raise_status(status, HETA_ERR_NONFINITE);

    // ---- 2. the slice sums (the same trees as one CTA's), summed in slice order
    double mu = 0.0, sigma = 0.0;
    for (int pass = 0; pass < 2; ++pass) {
        const double part = pass == 0 ? slice_part<false>(vals, lo, lo, hi, 0.0)
                                      : slice_part<true>(vals, lo, lo, hi, mu);
        const double t = block_sum(part, red);
        if (tid == 0) s_sum[pass] = t;
        cluster_sync();  // (1), (2): every CTA's slice sum
        double total = 0.0;
#pragma unroll
        for (int r = 0; r < kSlices; ++r) total += *peer(&s_sum[pass], (uint32_t)r);
        if (pass == 0) mu = total / (double)N;
        else sigma = sqrt(total / (double)N);
    }
    const double T = __dadd_rn(mu, __dmul_rn(c, sigma));
    if (tid == 0 && rank == 0 && thresh) thresh[b] = T;

    // ---- 3. dense tokens per warp (contiguous segments of the slice), per CTA
    const int n = hi - lo;
    const int per_lane = (n + kThreads - 1) / kThreads;
    const int seg = 32 * per_lane;
    const int seg_lo = lo + min(n, warp * seg);
    const int seg_hi = min(hi, seg_lo + seg);
    uint32_t nd = 0;
    for (int i = seg_lo + lane; i < seg_hi; i += 32) nd += (double)vals[i - lo] >= T;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nd += __shfl_xor_sync(kFull, nd, o);
    if (lane == 0) w_dense[warp] = nd;
    __syncthreads();
    if (warp == 0) {
        const uint32_t here = w_dense[lane];
        uint32_t incl = here;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += t;
        }
        w_dense_before[lane] = incl - here;
        if (lane == 31) s_nd = incl;
    }
    cluster_sync();  // (3) every CTA's dense count
    if (warp == 0) {
        // dense tokens in the CTAs before this one, and (rank 0) in all of them
        uint32_t before = 0u, all = 0u;
        if (lane < kSlices) {
            const uint32_t v = *peer(&s_nd, (uint32_t)lane);
            before = lane < (int)rank ? v : 0u;
            all = v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            before += __shfl_xor_sync(kFull, before, o);
            all += __shfl_xor_sync(kFull, all, o);
        }
        w_dense_before[lane] += before;
        if (lane == 0 && rank == 0) counts[b] = (int32_t)all;
    }
    __syncthreads();
    compact_threshold(vals, lo, seg_lo, seg_hi, T, w_dense_before[warp],
                      dense_idx + (size_t)b * N, local_idx + (size_t)b * N,
                      mask ? mask + (size_t)b * N : nullptr, lane);
    cluster_sync();  // (4) no CTA leaves while another may still read its shared memory
}

}  // namespace

cudaError_t launch_route_threshold(const float *u, int B, int N, double c, int32_t *counts,
                                   int32_t *dense_idx, int32_t *local_idx, double *thresh,
                                   uint8_t *mask, int32_t *status, cudaStream_t s)
{
    if (B <= kRouteClusterMaxB || N > kRouteMaxN) {
        const int L = (N + kSlices - 1) / kSlices;
        const int Lmax = (kRouteClusterMaxN + kSlices - 1) / kSlices;
        cudaError_t e = cudaFuncSetAttribute(route_threshold_cluster_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(sizeof(float) * Lmax));
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(B * kSlices), 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = sizeof(float) * (size_t)L;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kSlices;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, route_threshold_cluster_kernel, u, N, c, counts,
                                  dense_idx, local_idx, thresh, mask, status);
    }
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
