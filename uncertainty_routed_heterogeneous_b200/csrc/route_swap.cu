// route_swap.cu -- the per-block random swap of a top-k routing.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion", §3.2.2 (after Eq. (12)): at each transformer block a subset of
// the uncertain (dense) tokens trades places with randomly selected certain
// (local) tokens; App. B, Table 8: the swap ratio r = 7% of the tokens.
// Here: every token i of sample b draws rho_i = word 0 of Philox4x32-10
// (Salmon et al., SC 2011) with counter (i, b, block, 0) and key (seed low,
// seed high); of the dense set the s tokens with the smallest (rho_i, i) go
// local and of the local set the s tokens with the smallest (rho_i, i) go
// dense, so the count stays k.
//
// One CTA per (sample, block): the dense set becomes a bitmap in shared memory, the
// draws are computed once into shared memory, each set's s smallest draws
// are found by the same three-pass radix select as the top-k routing (on the
// complemented draws, so "largest" means smallest), and a ballot compaction
// writes both new lists in increasing order.
#include "heta_internal.cuh"
#include "radix_select.cuh"

namespace heta {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

// Philox4x32-10 word 0: ten rounds of the two multiply-xor lanes, the key
// advanced by the Weyl increments before every round after the first.
__device__ __forceinline__ uint32_t philox_word0(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
    }
    return c0;
}

__global__ void __launch_bounds__(kThreads, 1)
route_swap_kernel(const int32_t *dense_idx, int B, int N, int k, int s, uint32_t seed_lo,
                  uint32_t seed_hi, int block0, int32_t *dense_out, int32_t *local_out,
                  uint8_t *__restrict__ mask, int32_t *status)
{
    // blockIdx.x = beta * B + b: sample b at transformer block block0 + beta;
    // the outputs of block beta start at beta * B rows
    const int b = blockIdx.x % B;
    const int beta = blockIdx.x / B;
    const int block = block0 + beta;
    extern __shared__ uint32_t dyn[];
    uint32_t *key = dyn;       // [N] complemented draws: larger key = smaller draw
    uint32_t *bits = dyn + N;  // [ceil(N/32)] dense set of the input routing
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t warp_tot[kWarps];
    __shared__ uint32_t s_digit, s_rank;
    __shared__ uint32_t w_cnt[2][kWarps], w_before[2][kWarps];  // [group][warp]
    __shared__ uint32_t w_dense[kWarps], w_dense_before[kWarps];
    __shared__ int s_bad;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwords = (N + 31) >> 5;
    if (tid == 0) s_bad = 0;
    for (int w = tid; w < nwords; w += kThreads) bits[w] = 0u;
    __syncthreads();

    // ---- 1. the input dense set as a bitmap (read fully before any write,
    // so dense_out may be dense_idx itself)
    const int32_t *din = dense_idx + (size_t)b * k;
    for (int j = tid; j < k; j += kThreads) {
        const int32_t t = din[j];
        if ((unsigned)t < (unsigned)N)
            atomicOr(&bits[t >> 5], 1u << (t & 31));
        else
            s_bad = 1;
    }
    // ---- 2. the draws
    for (int i = tid; i < N; i += kThreads)
        key[i] = ~philox_word0((uint32_t)i, (uint32_t)b, (uint32_t)block, 0u, seed_lo, seed_hi);
    __syncthreads();
    if (s_bad) {
        if (tid == 0) raise_status(status, HETA_ERR_INVALID_ARG);
        return;
    }

    // ---- 3. per group (0: the input's local set, 1: its dense set) the s
    // largest keys: threshold key K[g] and how many keys equal to it are taken
    uint32_t kth[2] = {0xffffffffu, 0xffffffffu}, take[2] = {0u, 0u};
    auto in_group = [&](int i, int g) -> bool {
        return (int)((bits[i >> 5] >> (i & 31)) & 1u) == g;
    };
    for (int g = 0; g < 2 && s > 0; ++g) {
        for (int i = tid; i < 2048; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < N; i += kThreads)
            if (in_group(i, g)) atomicAdd(&hist[key[i] >> 21], 1u);
        __syncthreads();
        find_digit<kThreads>(hist, 2048, (uint32_t)s, warp_tot, &s_digit, &s_rank);
        const uint32_t d1 = s_digit, r1 = s_rank;
        for (int i = tid; i < 2048; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < N; i += kThreads) {
            const uint32_t kk = key[i];
            if ((kk >> 21) == d1 && in_group(i, g)) atomicAdd(&hist[(kk >> 10) & 2047u], 1u);
        }
        __syncthreads();
        find_digit<kThreads>(hist, 2048, r1, warp_tot, &s_digit, &s_rank);
        const uint32_t p2 = (d1 << 11) | s_digit, r2 = s_rank;
        for (int i = tid; i < 1024; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < N; i += kThreads) {
            const uint32_t kk = key[i];
            if ((kk >> 10) == p2 && in_group(i, g)) atomicAdd(&hist[kk & 1023u], 1u);
        }
        __syncthreads();
        find_digit<kThreads>(hist, 1024, r2, warp_tot, &s_digit, &s_rank);
        kth[g] = (p2 << 10) | s_digit;
        take[g] = s_rank;
    }

    // ---- 4. which keys equal to K[g] are taken: the first take[g] of them
    // in token order.  Each warp owns one contiguous segment of tokens.
    const int per_lane = (N + kThreads - 1) / kThreads;
    const int seg = 32 * per_lane;
    const int seg_lo = min(N, warp * seg);
    const int seg_hi = min(N, seg_lo + seg);
    uint32_t n_eq[2] = {0u, 0u};
    if (s > 0) {
        for (int i = seg_lo + lane; i < seg_hi; i += 32) {
            const int g = in_group(i, 1) ? 1 : 0;
            n_eq[g] += key[i] == kth[g];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n_eq[0] += __shfl_xor_sync(0xffffffffu, n_eq[0], o);
        n_eq[1] += __shfl_xor_sync(0xffffffffu, n_eq[1], o);
    }
    if (lane == 0) {
        w_cnt[0][warp] = n_eq[0];
        w_cnt[1][warp] = n_eq[1];
    }
    __syncthreads();
    if (warp < 2) {
        const uint32_t c = w_cnt[warp][lane];
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        w_before[warp][lane] = incl - c;
    }
    __syncthreads();

    // new dense flag of token i (eq_rank: its rank among its group's keys equal to K)
    auto selected = [&](int i, int g, uint32_t eq_rank) -> bool {
        const uint32_t kk = key[i];
        return s > 0 && (kk > kth[g] || (kk == kth[g] && eq_rank < take[g]));
    };

    // ---- 5. count the new dense tokens per warp, then compact both lists
    const unsigned lt = (1u << lane) - 1u;
    uint32_t nd = 0;
    {
        uint32_t re[2] = {w_before[0][warp], w_before[1][warp]};
        for (int base = seg_lo; base < seg_hi; base += 32) {
            const int i = base + lane;
            const bool valid = i < seg_hi;
            const int g = valid && in_group(i, 1) ? 1 : 0;
            const bool eq = valid && key[i] == kth[g];
            const unsigned eq0 = __ballot_sync(0xffffffffu, eq && g == 0);
            const unsigned eq1 = __ballot_sync(0xffffffffu, eq && g == 1);
            const uint32_t rank = g ? re[1] + __popc(eq1 & lt) : re[0] + __popc(eq0 & lt);
            const bool sel = valid && selected(i, g, rank);
            nd += valid && (g == 1) != sel;
            re[0] += __popc(eq0);
            re[1] += __popc(eq1);
        }
    }
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
    }
    __syncthreads();

    const size_t row = (size_t)beta * B + b;
    int32_t *dout = dense_out + row * k;
    int32_t *lout = local_out + row * (N - k);
    uint8_t *mout = mask ? mask + row * N : nullptr;
    uint32_t rd = w_dense_before[warp];
    uint32_t re[2] = {w_before[0][warp], w_before[1][warp]};
    for (int base = seg_lo; base < seg_hi; base += 32) {
        const int i = base + lane;
        const bool valid = i < seg_hi;
        const int g = valid && in_group(i, 1) ? 1 : 0;
        const bool eq = valid && key[i] == kth[g];
        const unsigned eq0 = __ballot_sync(0xffffffffu, eq && g == 0);
        const unsigned eq1 = __ballot_sync(0xffffffffu, eq && g == 1);
        const uint32_t rank = g ? re[1] + __popc(eq1 & lt) : re[0] + __popc(eq0 & lt);
        const bool dense = valid && (g == 1) != selected(i, g, rank);
        const unsigned d_mask = __ballot_sync(0xffffffffu, dense);
        const uint32_t pos = rd + __popc(d_mask & lt);
        // the swap keeps |dense| == k; the bounds only guard memory
        if (dense) {
            if (pos < (uint32_t)k) dout[pos] = i;
        } else if (valid && (uint32_t)i - pos < (uint32_t)(N - k)) {
            lout[i - pos] = i;
        }
        if (mout && valid) mout[i] = dense ? 0 : 1;
        rd += __popc(d_mask);
        re[0] += __popc(eq0);
        re[1] += __popc(eq1);
    }
}

}  // namespace

size_t route_swap_smem_bytes(int N)
{
    return sizeof(uint32_t) * ((size_t)N + (size_t)((N + 31) / 32));
}

cudaError_t launch_route_swap(const int32_t *dense_idx, int B, int N, int k, int s,
                              uint64_t seed, int block0, int nblocks, int32_t *dense_out,
                              int32_t *local_out, uint8_t *mask, int32_t *status,
                              cudaStream_t st)
{
    cudaError_t e = cudaFuncSetAttribute(route_swap_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)route_swap_smem_bytes(kRouteMaxN));
    if (e != cudaSuccess) return e;
    route_swap_kernel<<<(unsigned)((int64_t)B * nblocks), kThreads, route_swap_smem_bytes(N),
                        st>>>(dense_idx, B, N, k, s, (uint32_t)seed, (uint32_t)(seed >> 32),
                              block0, dense_out, local_out, mask, status);
    return cudaGetLastError();
}

}  // namespace heta
