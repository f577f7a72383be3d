// route.cu -- per-sample top-k routing: radix select + ballot compaction.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion", §3.2.2 Eq. (11)-(12): tokens with high uncertainty go dense.
// Top-k reading: exactly k tokens per sample (k = ceil(rho*N), Eq. (14));
// equal u are taken in increasing token index; -0.0 == +0.0.
//
// One CTA per sample.  The sample's u is read from HBM once (coalesced
// 16-byte loads) into shared memory as order-preserving uint32 keys, and the
// histogram of their top 11 bits is counted on the way in; two more radix
// passes over the keys (the next 11 bits, the last 10) count only the keys
// still in the running, so after the first pass almost every key costs a
// compare.  That finds the k-th largest key K* and how many keys equal to K*
// are taken; a last pass compacts both index lists in increasing order with
// warp ballots and writes them as contiguous runs.
#include "heta_internal.cuh"
#include "radix_select.cuh"

namespace heta {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

// Monotone map float -> uint32: a > b (as reals) <=> key(a) > key(b).
// -0.0 is folded onto +0.0 first so the two compare equal.
__device__ __forceinline__ uint32_t order_key(float f)
{
    uint32_t b = __float_as_uint(f);
    if ((b & 0x7fffffffu) == 0u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key)
{
    uint32_t b = (key & 0x80000000u) ? (key & 0x7fffffffu) : ~key;
    return __uint_as_float(b);
}

__global__ void __launch_bounds__(kThreads, 1)
route_kernel(const float *__restrict__ u, int B, int N, int k,
             int32_t *__restrict__ dense_idx, int32_t *__restrict__ local_idx,
             float *__restrict__ thresh, uint8_t *__restrict__ mask,
             int32_t *status)
{
    extern __shared__ uint32_t keys[];
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t warp_tot[kWarps];
    __shared__ uint32_t s_digit, s_rank;
    __shared__ uint32_t w_gt[kWarps], w_eq[kWarps];
    __shared__ uint32_t w_dense_before[kWarps], w_eq_before[kWarps];
    __shared__ int s_nan;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // samples b = blockIdx.x, + gridDim.x, ...: while one is processed, the
    // next one's u is pulled into L2
    for (int b = blockIdx.x; b < B; b += gridDim.x) {
    const float *ub = u + (size_t)b * N;
    if (b + (int)gridDim.x < B) {
        const char *nx = reinterpret_cast<const char *>(ub + (size_t)gridDim.x * N);
        for (size_t off = (size_t)tid * 128; off < (size_t)N * 4; off += (size_t)kThreads * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(nx + off));
    }
    if (tid == 0) s_nan = 0;
    for (int i = tid; i < 2048; i += kThreads) hist[i] = 0u;
    __syncthreads();

    // ---- 1. one coalesced read of u into shared memory as keys, counting
    // the histogram of their top 11 bits on the way
    bool nan_seen = false;
    auto put = [&](int i, float f) {
        nan_seen |= (f != f);
        const uint32_t key = order_key(f);
        keys[i] = key;
        atomicAdd(&hist[key >> 21], 1u);
    };
    int head = 0;  // scalar elements before the first 16-byte boundary
    {
        uintptr_t a = reinterpret_cast<uintptr_t>(ub);
        head = (int)(((16u - (a & 15u)) & 15u) >> 2);
        if (head > N) head = N;
    }
    if (tid < head) put(tid, __ldg(ub + tid));
    const int n4 = (N - head) >> 2;
    const float4 *u4 = reinterpret_cast<const float4 *>(ub + head);
    // four loads in flight per thread before their keys are stored
    for (int v0 = tid; v0 < n4; v0 += 4 * kThreads) {
        float4 f[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int v = v0 + q * kThreads;
            f[q] = v < n4 ? __ldg(u4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int v = v0 + q * kThreads;
            if (v < n4) {
                const int i = head + 4 * v;
                put(i, f[q].x);
                put(i + 1, f[q].y);
                put(i + 2, f[q].z);
                put(i + 3, f[q].w);
            }
        }
    }
    for (int i = head + 4 * n4 + tid; i < N; i += kThreads) put(i, __ldg(ub + i));
    if (nan_seen) s_nan = 1;
    __syncthreads();
    if (tid == 0 && s_nan) raise_status(status, HETA_ERR_NONFINITE);

    // ---- 2. radix select of the k-th largest key: digits of 11, 11, 10 bits
    uint32_t kstar = 0xffffffffu, take = 0u;  // k == 0: nothing is dense
    if (k > 0) {
        find_digit<kThreads>(hist, 2048, (uint32_t)k, warp_tot, &s_digit, &s_rank);
        const uint32_t d1 = s_digit, r1 = s_rank;
        for (int i = tid; i < 2048; i += kThreads) hist[i] = 0u;
        __syncthreads();
        const uint4 *keys4 = reinterpret_cast<const uint4 *>(keys);
        // (the keys still in the running are few: one vote per four keys
        // skips the counting where a warp holds none)
        // (the loop runs warp-uniformly: the vote needs every lane)
        for (int vb = tid - lane; vb < (N >> 2); vb += kThreads) {
            const int v = vb + lane;
            const uint4 q = v < (N >> 2) ? keys4[v] : make_uint4(0u, 0u, 0u, 0u);
            const bool in = v < (N >> 2);
            const bool m0 = in && (q.x >> 21) == d1, m1 = in && (q.y >> 21) == d1;
            const bool m2 = in && (q.z >> 21) == d1, m3 = in && (q.w >> 21) == d1;
            if (__any_sync(0xffffffffu, m0 | m1 | m2 | m3)) {
                if (m0) atomicAdd(&hist[(q.x >> 10) & 2047u], 1u);
                if (m1) atomicAdd(&hist[(q.y >> 10) & 2047u], 1u);
                if (m2) atomicAdd(&hist[(q.z >> 10) & 2047u], 1u);
                if (m3) atomicAdd(&hist[(q.w >> 10) & 2047u], 1u);
            }
        }
        for (int i = 4 * (N >> 2) + tid; i < N; i += kThreads) {
            const uint32_t key = keys[i];
            if ((key >> 21) == d1) atomicAdd(&hist[(key >> 10) & 2047u], 1u);
        }
        __syncthreads();
        find_digit<kThreads>(hist, 2048, r1, warp_tot, &s_digit, &s_rank);
        const uint32_t p2 = (d1 << 11) | s_digit, r2 = s_rank;
        for (int i = tid; i < 1024; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int vb = tid - lane; vb < (N >> 2); vb += kThreads) {
            const int v = vb + lane;
            const uint4 q = v < (N >> 2) ? keys4[v] : make_uint4(0u, 0u, 0u, 0u);
            const bool in = v < (N >> 2);
            const bool m0 = in && (q.x >> 10) == p2, m1 = in && (q.y >> 10) == p2;
            const bool m2 = in && (q.z >> 10) == p2, m3 = in && (q.w >> 10) == p2;
            if (__any_sync(0xffffffffu, m0 | m1 | m2 | m3)) {
                if (m0) atomicAdd(&hist[q.x & 1023u], 1u);
                if (m1) atomicAdd(&hist[q.y & 1023u], 1u);
                if (m2) atomicAdd(&hist[q.z & 1023u], 1u);
                if (m3) atomicAdd(&hist[q.w & 1023u], 1u);
            }
        }
        for (int i = 4 * (N >> 2) + tid; i < N; i += kThreads) {
            const uint32_t key = keys[i];
            if ((key >> 10) == p2) atomicAdd(&hist[key & 1023u], 1u);
        }
        __syncthreads();
        find_digit<kThreads>(hist, 1024, r2, warp_tot, &s_digit, &s_rank);
        kstar = (p2 << 10) | s_digit;
        take = s_rank;
    }
    if (tid == 0 && thresh)
        thresh[b] = k > 0 ? key_value(kstar) : __uint_as_float(0x7f800000u);

    // ---- 3. compaction: each warp owns one contiguous segment -------------
    // (segments hold a multiple of 128 keys, so the counts read 16 bytes a lane)
    const int per_lane = ((N + kThreads - 1) / kThreads + 3) & ~3;
    const int seg = 32 * per_lane;
    const int seg_lo = min(N, warp * seg);
    const int seg_hi = min(N, seg_lo + seg);
    uint32_t n_gt = 0, n_eq = 0;
    {
        const int full4 = (seg_hi - seg_lo) >> 2;  // whole uint4 of the segment
        const uint4 *k4 = reinterpret_cast<const uint4 *>(keys + seg_lo);
        for (int v = lane; v < full4; v += 32) {
            const uint4 q = k4[v];
            n_gt += (q.x > kstar) + (q.y > kstar) + (q.z > kstar) + (q.w > kstar);
            n_eq += (q.x == kstar) + (q.y == kstar) + (q.z == kstar) + (q.w == kstar);
        }
        for (int i = seg_lo + 4 * full4 + lane; i < seg_hi; i += 32) {
            const uint32_t key = keys[i];
            n_gt += key > kstar;
            n_eq += key == kstar;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
        n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    }
    if (lane == 0) {
        w_gt[warp] = n_gt;
        w_eq[warp] = n_eq;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t eq = w_eq[lane], gt = w_gt[lane];
        uint32_t eq_incl = eq;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t t = __shfl_up_sync(0xffffffffu, eq_incl, o);
            if (lane >= o) eq_incl += t;
        }
        uint32_t eq_before = eq_incl - eq;
        uint32_t taken_eq = take > eq_before ? min(eq, take - eq_before) : 0u;
        uint32_t dense_here = gt + taken_eq;
        uint32_t d_incl = dense_here;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t t = __shfl_up_sync(0xffffffffu, d_incl, o);
            if (lane >= o) d_incl += t;
        }
        w_dense_before[lane] = d_incl - dense_here;
        w_eq_before[lane] = eq_before;
    }
    __syncthreads();

    const unsigned lt = (1u << lane) - 1u;
    uint32_t rd = w_dense_before[warp], re = w_eq_before[warp];
    int32_t *dout = dense_idx + (size_t)b * k;
    int32_t *lout = local_idx + (size_t)b * (N - k);
    uint8_t *mout = mask ? mask + (size_t)b * N : nullptr;
    // 128 tokens per warp step, four consecutive ones per lane: token
    // t0 + e (e < 4) is dense-ranked by the lanes before it (one ballot per e)
    // and by the lane's own earlier tokens
    for (int base = seg_lo; base < seg_hi; base += 128) {
        const int t0 = base + 4 * lane;
        uint32_t key[4];
        if (t0 + 3 < seg_hi) {
            const uint4 q = *reinterpret_cast<const uint4 *>(keys + t0);
            key[0] = q.x;
            key[1] = q.y;
            key[2] = q.z;
            key[3] = q.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) key[e] = t0 + e < seg_hi ? keys[t0 + e] : 0u;
        }
        bool valid[4], dense[4];
        bool any_eq = false;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            valid[e] = t0 + e < seg_hi;
            dense[e] = valid[e] && key[e] > kstar;
            any_eq |= valid[e] && key[e] == kstar;
        }
        if (__any_sync(0xffffffffu, any_eq)) {
            // keys equal to K*: the first `take` of them in token order
            uint32_t before = re, own = 0;
            unsigned em[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                em[e] = __ballot_sync(0xffffffffu, valid[e] && key[e] == kstar);
                before += __popc(em[e] & lt);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool eq = valid[e] && key[e] == kstar;
                dense[e] = dense[e] || (eq && before + own < take);
                own += eq;
                re += __popc(em[e]);
            }
        }
        unsigned dm[4];
        uint32_t pos = rd;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            dm[e] = __ballot_sync(0xffffffffu, dense[e]);
            pos += __popc(dm[e] & lt);
        }
        // one store per token into whichever list holds it; the select makes
        // |dense| == k exactly, the bounds only guard memory
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t t = (uint32_t)(t0 + e);
            const uint32_t slot = dense[e] ? pos : t - pos;
            const uint32_t cap = dense[e] ? (uint32_t)k : (uint32_t)(N - k);
            int32_t *const list = dense[e] ? dout : lout;
            if (valid[e] && slot < cap) list[slot] = (int32_t)t;
            if (mout && valid[e]) mout[t] = dense[e] ? 0 : 1;
            pos += dense[e];
            rd += __popc(dm[e]);
        }
    }
    __syncthreads();  // shared memory is reused by the next sample
    }
}

}  // namespace

cudaError_t launch_route(const float *u, int B, int N, int k, int32_t *dense_idx,
                         int32_t *local_idx, float *thresh, uint8_t *mask,
                         int32_t *status, cudaStream_t s)
{
    const size_t smem = sizeof(uint32_t) * (size_t)N;
    cudaError_t e = cudaFuncSetAttribute(route_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(sizeof(uint32_t) * kRouteMaxN));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    route_kernel<<<B < sms ? B : sms, kThreads, smem, s>>>(u, B, N, k, dense_idx, local_idx,
                                                         thresh, mask, status);
    return cudaGetLastError();
}

}  // namespace heta
