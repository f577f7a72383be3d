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
// writes both new lists in increasing order.  A sample too large for its
// draws to fit in shared memory (N > kRouteMaxN, e.g. a 720p latent) keeps
// only the bitmap there and computes each token's draw again in every pass.
#include "heta_internal.cuh"
#include "radix_select.cuh"

namespace heta {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kSwapCand = 128;  // most keys of one bucket the exact rank takes

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

template <bool kStored>
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
    uint32_t *key = dyn;                    // [N] complemented draws (kStored)
    uint32_t *bits = kStored ? dyn + N : dyn;  // [ceil(N/32)] dense set of the input routing
    __shared__ uint32_t hist[2048];  // radix digits; or [group][1024] top-10-bit buckets
    __shared__ uint32_t cand_k[2][kSwapCand];
    __shared__ int cand_i[2][kSwapCand];
    __shared__ uint32_t s_ncand[2], s_kth[2];
    __shared__ int s_ith[2];
    __shared__ uint32_t warp_tot[kWarps];
    __shared__ uint32_t s_digit, s_rank;
    __shared__ uint32_t w_cnt[2][kWarps], w_before[2][kWarps];  // [group][warp]
    __shared__ uint32_t w_dense[kWarps], w_dense_before[kWarps];
    __shared__ int s_bad;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwords = (N + 31) >> 5;
    if (tid == 0) {
        s_bad = 0;
        s_ncand[0] = s_ncand[1] = 0u;
        s_kth[0] = s_kth[1] = 0xffffffffu;
        s_ith[0] = s_ith[1] = -1;
    }
    for (int w = tid; w < nwords; w += kThreads) bits[w] = 0u;
    for (int i = tid; i < 2048; i += kThreads) hist[i] = 0u;
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
    __syncthreads();  // (the bitmap is complete)
    if (s_bad) {
        if (tid == 0) raise_status(status, HETA_ERR_INVALID_ARG);
        return;
    }
    auto in_group = [&](int i, int g) -> bool {
        return (int)((bits[i >> 5] >> (i & 31)) & 1u) == g;
    };
    // token i's complemented draw: larger key = smaller draw
    auto draw = [&](int i) -> uint32_t {
        return ~philox_word0((uint32_t)i, (uint32_t)b, (uint32_t)block, 0u, seed_lo, seed_hi);
    };
    auto key_of = [&](int i) -> uint32_t { return kStored ? key[i] : draw(i); };

    // ---- 2. the draws, with each group's histogram of their top 10 bits
    // (group 0: the input's local set, 1: its dense set)
    for (int i = tid; i < N; i += kThreads) {
        const uint32_t kk = draw(i);
        if (kStored) key[i] = kk;
        atomicAdd(&hist[(in_group(i, 1) ? 1024 : 0) + (kk >> 22)], 1u);
    }
    __syncthreads();

    // each warp owns one contiguous segment of tokens (a whole number of
    // bitmap words)
    const int per_lane = (N + kThreads - 1) / kThreads;
    const int seg = 32 * per_lane;
    const int seg_lo = min(N, warp * seg);
    const int seg_hi = min(N, seg_lo + seg);
    const unsigned lt = (1u << lane) - 1u;
    int32_t *const dout = dense_out + ((size_t)beta * B + b) * k;
    int32_t *const lout = local_out + ((size_t)beta * B + b) * (N - k);
    uint8_t *const mout = mask ? mask + ((size_t)beta * B + b) * N : nullptr;

    // ---- 3. per group the s largest keys: threshold key K[g] and how many
    // keys equal to it are taken.  The draws are uniform, so the bucket of
    // the s-th largest key holds a few dozen keys at most: they are ranked
    // exactly as (key descending, token ascending) pairs.  A bucket of more
    // than kSwapCand keys (not seen with Philox draws) takes the radix select.
    uint32_t kth[2] = {0xffffffffu, 0xffffffffu}, take[2] = {0u, 0u};
    bool fast = s > 0;
    uint32_t bkt[2] = {0u, 0u}, rk[2] = {0u, 0u};
    for (int g = 0; g < 2 && fast; ++g) {
        find_digit<kThreads>(hist + 1024 * g, 1024, (uint32_t)s, warp_tot, &s_digit, &s_rank);
        bkt[g] = s_digit;
        rk[g] = s_rank;
        fast = fast && hist[1024 * g + bkt[g]] <= (uint32_t)kSwapCand;  // (the same in every thread)
    }
    if (fast) {
        // candidates (keys in the bucket of the s-th largest), and per warp
        // the tokens of each group in buckets above it: those all change sets
        uint32_t above[2] = {0u, 0u};
        for (int i = seg_lo + lane; i < seg_hi; i += 32) {
            const uint32_t kk = key_of(i);
            const int g = in_group(i, 1) ? 1 : 0;
            const uint32_t bk = kk >> 22;
            above[g] += bk > bkt[g];
            if (bk == bkt[g]) {
                const uint32_t at = atomicAdd(&s_ncand[g], 1u);
                if (at < (uint32_t)kSwapCand) {
                    cand_k[g][at] = kk;
                    cand_i[g][at] = i;
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            above[0] += __shfl_xor_sync(0xffffffffu, above[0], o);
            above[1] += __shfl_xor_sync(0xffffffffu, above[1], o);
        }
        if (lane == 0) {
            w_cnt[0][warp] = above[0];
            w_cnt[1][warp] = above[1];
        }
        __syncthreads();
        // the rk[g]-th largest candidate in (key descending, token ascending)
        // order: the pair (K*, i*) from which on a token changes sets
        if (tid < 2 * kSwapCand) {
            const int g = tid / kSwapCand, j = tid % kSwapCand;
            const int n = (int)min(s_ncand[g], (uint32_t)kSwapCand);
            if (j < n) {
                const uint32_t kj = cand_k[g][j];
                const int ij = cand_i[g][j];
                uint32_t before = 0u;
                for (int m = 0; m < n; ++m) {
                    const uint32_t km = cand_k[g][m];
                    before += km > kj || (km == kj && cand_i[g][m] < ij);
                }
                if (before + 1u == rk[g]) {
                    s_kth[g] = kj;
                    s_ith[g] = ij;
                }
            }
        }
        __syncthreads();
    }
    if (s > 0 && !fast) __syncthreads();  // (every thread has read the buckets)
    for (int g = 0; g < 2 && s > 0 && !fast; ++g) {
        for (int i = tid; i < 2048; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < N; i += kThreads)
            if (in_group(i, g)) atomicAdd(&hist[key_of(i) >> 21], 1u);
        __syncthreads();
        find_digit<kThreads>(hist, 2048, (uint32_t)s, warp_tot, &s_digit, &s_rank);
        const uint32_t d1 = s_digit, r1 = s_rank;
        for (int i = tid; i < 2048; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < N; i += kThreads) {
            const uint32_t kk = key_of(i);
            if ((kk >> 21) == d1 && in_group(i, g)) atomicAdd(&hist[(kk >> 10) & 2047u], 1u);
        }
        __syncthreads();
        find_digit<kThreads>(hist, 2048, r1, warp_tot, &s_digit, &s_rank);
        const uint32_t p2 = (d1 << 11) | s_digit, r2 = s_rank;
        for (int i = tid; i < 1024; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < N; i += kThreads) {
            const uint32_t kk = key_of(i);
            if ((kk >> 10) == p2 && in_group(i, g)) atomicAdd(&hist[kk & 1023u], 1u);
        }
        __syncthreads();
        find_digit<kThreads>(hist, 1024, r2, warp_tot, &s_digit, &s_rank);
        kth[g] = (p2 << 10) | s_digit;
        take[g] = s_rank;
    }

    if (fast) {
        // ---- 4'. per warp: the tokens that change sets, then the new dense
        // count (its old dense tokens are the popcount of its bitmap words)
        const uint32_t kst0 = s_kth[0], kst1 = s_kth[1];
        const int ist0 = s_ith[0], ist1 = s_ith[1];
        auto changes = [&](uint32_t kk, int i, int g) -> bool {
            const uint32_t ks = g ? kst1 : kst0;
            const int is = g ? ist1 : ist0;
            return kk > ks || (kk == ks && i <= is);
        };
        if (warp == 0) {
            for (int g = 0; g < 2; ++g) {
                const int n = (int)min(s_ncand[g], (uint32_t)kSwapCand);
                for (int j = lane; j < n; j += 32) {
                    const int i = cand_i[g][j];
                    if (changes(cand_k[g][j], i, g)) atomicAdd(&w_cnt[g][i / seg], 1u);
                }
            }
            __syncwarp();
            // lane w: warp w's old dense tokens, minus those leaving, plus those arriving
            const int wlo = min(N, lane * seg), whi = min(N, wlo + seg);
            uint32_t dense_old = 0u;
            if (wlo < whi)  // (a warp past the last token owns no word)
                for (int wd = wlo >> 5; wd < (whi + 31) >> 5; ++wd) dense_old += __popc(bits[wd]);
            const uint32_t here = dense_old - w_cnt[1][lane] + w_cnt[0][lane];
            uint32_t incl = here;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            w_dense_before[lane] = incl - here;
        }
        __syncthreads();
        // ---- 5'. compaction: a token is dense when it was dense and stays,
        // or was local and changes sets
        uint32_t rd = w_dense_before[warp];
        for (int base = seg_lo; base < seg_hi; base += 32) {  // warp-uniform
            const int i = base + lane;
            const bool valid = i < seg_hi;
            const int g = valid && in_group(i, 1) ? 1 : 0;
            const bool dense = valid && ((g == 1) != changes(valid ? key_of(i) : 0u, i, g));
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
        }
    } else {
        // ---- 4. which keys equal to K[g] are taken: the first take[g] of them
        // in token order.
        uint32_t n_eq[2] = {0u, 0u};
        if (s > 0) {
            for (int i = seg_lo + lane; i < seg_hi; i += 32) {
                const int g = in_group(i, 1) ? 1 : 0;
                n_eq[g] += key_of(i) == kth[g];
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
            const uint32_t kk = key_of(i);
            return s > 0 && (kk > kth[g] || (kk == kth[g] && eq_rank < take[g]));
        };

        // ---- 5. count the new dense tokens per warp, then compact both lists
        uint32_t nd = 0;
        {
            uint32_t re[2] = {w_before[0][warp], w_before[1][warp]};
            for (int base = seg_lo; base < seg_hi; base += 32) {
                const int i = base + lane;
                const bool valid = i < seg_hi;
                const int g = valid && in_group(i, 1) ? 1 : 0;
                const bool eq = valid && key_of(i) == kth[g];
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

        uint32_t rd = w_dense_before[warp];
        uint32_t re[2] = {w_before[0][warp], w_before[1][warp]};
        for (int base = seg_lo; base < seg_hi; base += 32) {
            const int i = base + lane;
            const bool valid = i < seg_hi;
            const int g = valid && in_group(i, 1) ? 1 : 0;
            const bool eq = valid && key_of(i) == kth[g];
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
}

}  // namespace

size_t route_swap_smem_bytes(int N)
{
    const size_t words = (size_t)((N + 31) / 32);  // the bitmap
    return sizeof(uint32_t) * (N <= kRouteMaxN ? (size_t)N + words : words);
}

cudaError_t launch_route_swap(const int32_t *dense_idx, int B, int N, int k, int s,
                              uint64_t seed, int block0, int nblocks, int32_t *dense_out,
                              int32_t *local_out, uint8_t *mask, int32_t *status,
                              cudaStream_t st)
{
    const bool stored = N <= kRouteMaxN;
    auto kern = stored ? route_swap_kernel<true> : route_swap_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
        (int)(stored ? route_swap_smem_bytes(kRouteMaxN) : route_swap_smem_bytes(kRouteClusterMaxN)));
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((int64_t)B * nblocks), kThreads, route_swap_smem_bytes(N), st>>>(
        dense_idx, B, N, k, s, (uint32_t)seed, (uint32_t)(seed >> 32), block0, dense_out,
        local_out, mask, status);
    return cudaGetLastError();
}

}  // namespace heta
