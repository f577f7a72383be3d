// route.cu -- per-sample top-k routing: bucket select + ballot compaction.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion", §3.2.2 Eq. (11)-(12): tokens with high uncertainty go dense.
// Top-k reading: exactly k tokens per sample (k = ceil(rho*N), Eq. (14));
// equal u are taken in increasing token index; -0.0 == +0.0.
//
// One CTA per sample (persistent over the samples).  The sample's u is read
// from HBM once (16-byte loads) into shared memory, with its minimum and
// maximum.  A histogram of 2048 equal-width buckets over [min, max] finds the
// bucket holding the k-th largest value; for any spread of values it holds a
// few dozen tokens, and an exact all-pairs rank among those "candidates"
// gives the k-th largest value T and how many tokens equal to T are taken.
// A last pass compacts both index lists in increasing token order with warp
// ballots, 32 consecutive tokens per step, so the stores of each list are
// contiguous runs.
//
// Inputs the bucket select does not suit -- a NaN or an infinity, all values
// equal or too close for fp32 bucket arithmetic, a bucket with more than 256
// tokens (heavy ties) -- take a radix select on order-preserving uint32 keys
// instead (digits of 11, 11 and 10 bits), with the same compaction.
#include "heta_internal.cuh"
#include "radix_select.cuh"
#include "route_common.cuh"

namespace heta {
namespace {

using namespace rt;

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
template <bool kMask>
__global__ void __launch_bounds__(kThreads, 1)
route_kernel(const float *__restrict__ u, int B, int N, int k,
             int32_t *__restrict__ dense_idx, int32_t *__restrict__ local_idx,
             float *__restrict__ thresh, uint8_t *__restrict__ mask,
             int32_t *status)
{
    // slot s holds token s - off of the sample, where off (0..3) is the
    // sample's offset from a 16-byte boundary: slots and u share their
    // alignment, so four slots ("a quad") move with one 16-byte access
    extern __shared__ uint4 slot4[];
    uint32_t *slot = reinterpret_cast<uint32_t *>(slot4);
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t cand_w[kCandCap];
    __shared__ int cand_t[kCandCap];
    __shared__ uint32_t cnt_gt[kCandCap], cnt_eq[kCandCap];
    __shared__ uint32_t warp_tot[kWarps];
    __shared__ float w_min[kWarps], w_max[kWarps];
    __shared__ uint32_t w_gt[kWarps], w_eq[kWarps];
    __shared__ uint32_t w_dense_before[kWarps], w_eq_before[kWarps];
    __shared__ uint32_t s_digit, s_rank, s_ncand, s_kstar, s_take;
    __shared__ int s_nan;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float kInf = __uint_as_float(0x7f800000u);

    for (int b = blockIdx.x; b < B; b += gridDim.x) {
        const float *ub = u + (size_t)b * N;
        // while this sample is processed, the next one's u is pulled into L2
        if (b + (int)gridDim.x < B) {
            const char *nx = reinterpret_cast<const char *>(ub + (size_t)gridDim.x * N);
            for (size_t o = (size_t)tid * 128; o < (size_t)N * 4; o += (size_t)kThreads * 128)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(nx + o));
        }
        const int off = (int)((reinterpret_cast<uintptr_t>(ub) >> 2) & 3u);
        const int nslots = off + N;
        const int nq = (nslots + 3) >> 2;
        const int pq = (nq + kThreads - 1) / kThreads;  // quads per lane
        const int wq = 32 * pq;                           // quads per warp
        // warp w owns quads [q_lo, q_hi), lane l the quads q_lo + l + 32 i
        const int q_lo = warp * wq;
        const int q_hi = max(q_lo, min(nq, q_lo + wq));
        const int qa = off ? 1 : 0;              // whole quads are [qa, qb)
        const int qb = (nslots & 3) ? nq - 1 : nq;
        // ... and the tokens of those quads
        const int t_lo = min(N, max(0, 4 * q_lo - off));
        const int t_hi = min(N, max(t_lo, 4 * q_hi - off));
        // the (at most two) quads holding slots that are no token
        const int qp0 = off ? 0 : -1;
        const int qp1 = ((nslots & 3) && nq - 1 != qp0) ? nq - 1 : -1;
        auto owns = [&](int q) {
            return q >= q_lo && q < q_hi && ((q - q_lo) & 31) == lane;
        };
        // 16-byte copies of this lane's whole quads [qa, qe) of the sample at
        // us into shared memory, as one commit group
        auto issue_quads = [&](const float *us, int o, int qlo, int qe, int qfirst, int ln) {
            const uint4 *g4 = reinterpret_cast<const uint4 *>(us - o);
            for (int q = qlo + ln; q < qe; q += 32) {
                if (q < qfirst) continue;
                const uint32_t dst = (uint32_t)__cvta_generic_to_shared(slot4 + q);
                const size_t src = __cvta_generic_to_global(g4 + q);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src)
                             : "memory");
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };

        if (tid == 0) {
            s_nan = 0;
            s_ncand = 0u;
        }
        for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
        if (tid < kCandCap) {
            cnt_gt[tid] = 0u;
            cnt_eq[tid] = 0u;
        }

        // ---- 1. u -> shared memory, with min and max (NaN if any u is NaN)
        float mn = kInf, mx = -kInf;
        {
            // every whole quad of the sample in flight at once: 16-byte
            // asynchronous copies straight into shared memory (when N is a
            // multiple of 4 each warp issued them at the end of the previous
            // sample, as soon as its own quads were free; see below)
            const int qe = min(q_hi, qb);
            if (!((N & 3) == 0 && b != (int)blockIdx.x)) issue_quads(ub, off, q_lo, qe, qa, lane);
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            for (int q = q_lo + lane; q < qe; q += 32) {
                if (q < qa) continue;
                const uint4 v = slot4[q];
                const float a = __uint_as_float(v.x), c = __uint_as_float(v.y);
                const float d = __uint_as_float(v.z), e = __uint_as_float(v.w);
                mn = min3n(mn, a, c);
                mn = min3n(mn, d, e);
                mx = max3n(mx, a, c);
                mx = max3n(mx, d, e);
            }
            // the partial quads at either end, element by element
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const int q = p ? qp1 : qp0;
                if (q >= 0 && owns(q)) {
                    for (int s = max(4 * q, off); s < min(4 * q + 4, nslots); ++s) {
                        const float x = __ldg(ub + (s - off));
                        slot[s] = __float_as_uint(x);
                        mn = min2n(mn, x);
                        mx = max2n(mx, x);
                    }
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = min2n(mn, __shfl_xor_sync(kFull, mn, o));
            mx = max2n(mx, __shfl_xor_sync(kFull, mx, o));
        }
        if (lane == 0) {
            w_min[warp] = mn;
            w_max[warp] = mx;
        }
        __syncthreads();
        mn = w_min[lane];
        mx = w_max[lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = min2n(mn, __shfl_xor_sync(kFull, mn, o));
            mx = max2n(mx, __shfl_xor_sync(kFull, mx, o));
        }
        // (CTA-uniform: every thread reduced the same partials)
        const bool finite = mn > -kInf && mx < kInf;  // false for a NaN too
        const float lo = mn;
        const float span = __fsub_rn(mx, mn);
        const float scale = __fdiv_rn(2044.f, span);
        const float lo_scale = __fmul_rn(lo, scale);
        const bool one_op = fabsf(lo_scale) <= 4194304.f;  // 2^22
        const float cb = one_op ? __fsub_rn(8388610.f, lo_scale) : 8388610.f;  // 2^23 + 2
        bool fast = k > 0 && finite && span > 0.f && scale > 0.f && scale < kInf;
        uint32_t rank_in_bucket = 0u, bstar = 0u;

        // ---- 2. bucket histogram; the bucket of the k-th largest value
        if (fast) {
            // slots that are no token take the smallest value: bucket 0, below
            // every value a rank k <= N reaches
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const int q = p ? qp1 : qp0;
                if (q >= 0 && owns(q)) {
                    for (int s = 4 * q; s < 4 * q + 4; ++s)
                        if (s < off || s >= nslots) slot[s] = __float_as_uint(lo);
                }
            }
            const uint32_t hist_at_magic =
                (uint32_t)__cvta_generic_to_shared(hist) - 4u * kMagicBits;
            if (one_op)
                bucket_histogram<true>(slot4, q_lo, q_hi, lane, lo, scale, cb, hist_at_magic);
            else
                bucket_histogram<false>(slot4, q_lo, q_hi, lane, lo, scale, cb, hist_at_magic);
            __syncthreads();
            find_digit<kThreads>(hist, kBins, (uint32_t)k, warp_tot, &s_digit, &s_rank);
            bstar = s_digit;
            rank_in_bucket = s_rank;
            fast = hist[bstar] <= (uint32_t)kCandCap;
        }

        if (fast) {
            // ---- 3. candidates (the tokens of that bucket) and, per warp,
            // the tokens of the buckets above it
            const uint32_t bbits = kMagicBits + bstar;
            const uint32_t above =
                one_op ? bucket_candidates<true>(slot4, q_lo, q_hi, lane, lo, scale, cb, bbits,
                                                 off, nslots, &s_ncand, cand_w, cand_t, kCandCap)
                       : bucket_candidates<false>(slot4, q_lo, q_hi, lane, lo, scale, cb, bbits,
                                                  off, nslots, &s_ncand, cand_w, cand_t,
                                                  kCandCap);
            if (lane == 0) {
                w_gt[warp] = above;
                w_eq[warp] = 0u;
            }
            __syncthreads();

            // ---- 4. exact rank among the candidates: each warp compares every
            // candidate with its slice of them
            const int c = (int)min(s_ncand, (uint32_t)kCandCap);
            {
                const int j0 = warp * c / kWarps, j1 = (warp + 1) * c / kWarps;
                if (j0 < j1) {
                    for (int i = lane; i < c; i += 32) {
                        const float vi = __uint_as_float(cand_w[i]);
                        uint32_t g = 0u, e = 0u;
                        for (int j = j0; j < j1; ++j) {
                            const float vj = __uint_as_float(cand_w[j]);
                            g += vj > vi;
                            e += vj == vi;
                        }
                        if (g) atomicAdd(&cnt_gt[i], g);
                        if (e) atomicAdd(&cnt_eq[i], e);
                    }
                }
            }
            __syncthreads();
            if (warp == 0) {
                // T = the candidate with (greater) < r <= (greater + equal)
                uint32_t tw = 0u, take = 0u;
                bool found = false;
                for (int i = lane; i < c; i += 32) {
                    const uint32_t g = cnt_gt[i], e = cnt_eq[i];
                    if (g < rank_in_bucket && rank_in_bucket <= g + e) {
                        tw = cand_w[i];
                        take = rank_in_bucket - g;
                        found = true;
                    }
                }
                const unsigned fm = __ballot_sync(kFull, found);
                const int src = fm ? __ffs(fm) - 1 : 0;
                tw = __shfl_sync(kFull, tw, src);
                take = __shfl_sync(kFull, take, src);
                const float fst = __uint_as_float(tw);
                // the candidates above T, and those equal to it, per owning warp
                for (int i = lane; i < c; i += 32) {
                    const float v = __uint_as_float(cand_w[i]);
                    const int owner = ((cand_t[i] + off) >> 2) / wq;
                    if (v > fst) atomicAdd(&w_gt[owner], 1u);
                    else if (v == fst) atomicAdd(&w_eq[owner], 1u);
                }
                if (lane == 0) {
                    s_kstar = tw;
                    s_take = take;
                    if (thresh) thresh[b] = fst;
                }
            }
        } else if (k > 0) {
            // ---- 2'-4'. radix select on order keys (kept in the slots)
            __syncthreads();  // (every thread has read the bucket histogram)
            for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
            __syncthreads();
            bool nan_seen = false;
            for (int i = 0; i < pq; ++i) {
                const int q = q_lo + lane + 32 * i;
                if (q < q_hi) {
                    const uint4 v = slot4[q];
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                    uint32_t key[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = 4 * q + e;
                        const float f = __uint_as_float(w[e]);
                        // slots that are no token take key 0, below every key
                        const bool tok = s >= off && s < nslots;
                        nan_seen |= tok && (f != f);
                        key[e] = tok ? order_key(f) : 0u;
                        atomicAdd(&hist[key[e] >> 21], 1u);
                    }
                    slot4[q] = make_uint4(key[0], key[1], key[2], key[3]);
                }
            }
            if (nan_seen) s_nan = 1;
            __syncthreads();
            find_digit<kThreads>(hist, kBins, (uint32_t)k, warp_tot, &s_digit, &s_rank);
            const uint32_t d1 = s_digit, r1 = s_rank;
            for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
            __syncthreads();
            // (the keys still in the running are few: one vote per quad skips
            // the counting where a warp holds none; the loop is warp-uniform)
            for (int i = 0; i < pq; ++i) {
                const int q = q_lo + lane + 32 * i;
                const bool in = q < q_hi;
                const uint4 v = in ? slot4[q] : make_uint4(0u, 0u, 0u, 0u);
                const bool m0 = in && (v.x >> 21) == d1, m1 = in && (v.y >> 21) == d1;
                const bool m2 = in && (v.z >> 21) == d1, m3 = in && (v.w >> 21) == d1;
                if (__any_sync(kFull, m0 | m1 | m2 | m3)) {
                    if (m0) atomicAdd(&hist[(v.x >> 10) & 2047u], 1u);
                    if (m1) atomicAdd(&hist[(v.y >> 10) & 2047u], 1u);
                    if (m2) atomicAdd(&hist[(v.z >> 10) & 2047u], 1u);
                    if (m3) atomicAdd(&hist[(v.w >> 10) & 2047u], 1u);
                }
            }
            __syncthreads();
            find_digit<kThreads>(hist, kBins, r1, warp_tot, &s_digit, &s_rank);
            const uint32_t p2 = (d1 << 11) | s_digit, r2 = s_rank;
            for (int i = tid; i < 1024; i += kThreads) hist[i] = 0u;
            __syncthreads();
            for (int i = 0; i < pq; ++i) {
                const int q = q_lo + lane + 32 * i;
                const bool in = q < q_hi;
                const uint4 v = in ? slot4[q] : make_uint4(0u, 0u, 0u, 0u);
                const bool m0 = in && (v.x >> 10) == p2, m1 = in && (v.y >> 10) == p2;
                const bool m2 = in && (v.z >> 10) == p2, m3 = in && (v.w >> 10) == p2;
                if (__any_sync(kFull, m0 | m1 | m2 | m3)) {
                    if (m0) atomicAdd(&hist[v.x & 1023u], 1u);
                    if (m1) atomicAdd(&hist[v.y & 1023u], 1u);
                    if (m2) atomicAdd(&hist[v.z & 1023u], 1u);
                    if (m3) atomicAdd(&hist[v.w & 1023u], 1u);
                }
            }
            __syncthreads();
            find_digit<kThreads>(hist, 1024, r2, warp_tot, &s_digit, &s_rank);
            const uint32_t kstar = (p2 << 10) | s_digit;
            // keys above K* and equal to it, per warp, over its tokens
            uint32_t n_gt = 0u, n_eq = 0u;
            for (int t = t_lo + lane; t < t_hi; t += 32) {
                const uint32_t key = slot[t + off];
                n_gt += key > kstar;
                n_eq += key == kstar;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                n_gt += __shfl_xor_sync(kFull, n_gt, o);
                n_eq += __shfl_xor_sync(kFull, n_eq, o);
            }
            if (lane == 0) {
                w_gt[warp] = n_gt;
                w_eq[warp] = n_eq;
            }
            if (tid == 0) {
                s_kstar = kstar;
                s_take = s_rank;
                if (thresh) thresh[b] = key_value(kstar);
            }
        } else {
            // k == 0: nothing is dense (a float threshold of +inf, no ties taken)
            if (!finite) {  // a NaN or an infinity: report a NaN
                bool nan_seen = false;
                for (int i = 0; i < pq; ++i) {
                    const int q = q_lo + lane + 32 * i;
                    if (q < q_hi) {
                        for (int s = max(4 * q, off); s < min(4 * q + 4, nslots); ++s) {
                            const float f = __uint_as_float(slot[s]);
                            nan_seen |= f != f;
                        }
                    }
                }
                if (nan_seen) s_nan = 1;
            }
            if (lane == 0) {
                w_gt[warp] = 0u;
                w_eq[warp] = 0u;
            }
            if (tid == 0) {
                s_kstar = 0x7f800000u;
                s_take = 0u;
                if (thresh) thresh[b] = kInf;
            }
        }
        const bool keys = !fast && k > 0;
        __syncthreads();
        if (tid == 0 && s_nan) raise_status(status, HETA_ERR_NONFINITE);

        // ---- 5. where each warp's dense and local tokens start
        if (warp == 0) {
            const uint32_t take = s_take;
            const uint32_t eq = w_eq[lane], gt = w_gt[lane];
            uint32_t eq_incl = eq;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(kFull, eq_incl, o);
                if (lane >= o) eq_incl += t;
            }
            const uint32_t eq_before = eq_incl - eq;
            const uint32_t taken_eq = take > eq_before ? min(eq, take - eq_before) : 0u;
            const uint32_t dense_here = gt + taken_eq;
            uint32_t d_incl = dense_here;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(kFull, d_incl, o);
                if (lane >= o) d_incl += t;
            }
            w_dense_before[lane] = d_incl - dense_here;
            w_eq_before[lane] = eq_before;
        }
        __syncthreads();

        // ---- 6. compaction, 32 consecutive tokens per warp step
        {
            const uint32_t kst = s_kstar, take = s_take;
            const uint32_t rd = w_dense_before[warp], re = w_eq_before[warp];
            const bool has_eq = w_eq[warp] != 0u;
            int32_t *dout = dense_idx + (size_t)b * k;
            int32_t *lout = local_idx + (size_t)b * (N - k);
            uint8_t *mout = mask ? mask + (size_t)b * N : nullptr;
            const uint32_t ku = (uint32_t)k, nl = (uint32_t)(N - k);
            if (keys) {
                if (has_eq)
                    compact<true, true, kMask>(slot, off, t_lo, t_hi, kst, take, rd, re, dout,
                                               lout, mout, ku, nl, lane);
                else
                    compact<true, false, kMask>(slot, off, t_lo, t_hi, kst, take, rd, re, dout,
                                                lout, mout, ku, nl, lane);
            } else {
                if (has_eq)
                    compact<false, true, kMask>(slot, off, t_lo, t_hi, kst, take, rd, re, dout,
                                                lout, mout, ku, nl, lane);
                else if (!kMask)
                    compact_float_plain(slot, off, t_lo, t_hi, kst, rd, dout, lout, lane);
                else
                    compact<false, false, true>(slot, off, t_lo, t_hi, kst, take, rd, re,
                                                dout, lout, mout, ku, nl, lane);
            }
        }
        // A warp's quads are free once it has compacted them (no other warp
        // reads them): when every sample has the same quads (N a multiple of
        // 4, so the same 16-byte phase), the next sample's copies go out now
        // and overlap the other warps' tails and the next sample's setup.
        if ((N & 3) == 0 && b + (int)gridDim.x < B) {
            const float *un = ub + (size_t)gridDim.x * N;
            issue_quads(un, off, q_lo, min(q_hi, qb), qa, lane);
        }
        __syncthreads();  // shared memory is reused by the next sample
    }
}

}  // namespace

cudaError_t launch_route(const float *u, int B, int N, int k, int32_t *dense_idx,
                         int32_t *local_idx, float *thresh, uint8_t *mask,
                         int32_t *status, cudaStream_t s)
{
    // N tokens plus up to 3 slots before and after them that are no token
    const size_t smem = sizeof(uint32_t) * (size_t)(N + 8);
    auto kern = mask ? route_kernel<true> : route_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(sizeof(uint32_t) * (kRouteMaxN + 8)));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    kern<<<B < sms ? B : sms, kThreads, smem, s>>>(u, B, N, k, dense_idx, local_idx, thresh,
                                                  mask, status);
    return cudaGetLastError();
}

}  // namespace heta
