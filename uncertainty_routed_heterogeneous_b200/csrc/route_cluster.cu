// route_cluster.cu -- per-sample top-k routing for a few samples, or for
// samples too large for one SM's shared memory: one sample over a cluster of
// eight CTAs.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion", §3.2.2 Eq. (11)-(12), in top-k form (k = ceil(rho*N) per
// sample, equal u taken in increasing token index, -0.0 == +0.0): the same
// selection as route.cu, whose one CTA a sample leaves a single-sample call
// latency-bound on one SM and holds at most kRouteMaxN tokens (a 720p Wan
// latent, 21x45x80 = 75600 tokens, needs two SMs' worth).  Here the sample's quads are cut into eight
// contiguous slices, one a CTA, and the CTAs combine what they found through
// distributed shared memory:
//   1. each CTA loads its slice and its min / max; the cluster's min / max;
//   2. each CTA's bucket histogram; every CTA sums the eight and finds the
//      bucket of the k-th largest value;
//   3. each CTA's candidates (that bucket's tokens) and per-warp counts of
//      the tokens above it; every CTA ranks the merged candidates (T and the
//      ties taken come out the same everywhere), then each CTA's count of
//      tokens above T and equal to it gives the CTAs after it their offsets;
//   4. each CTA compacts its own tokens.
// Samples the bucket select does not suit take the radix select on order
// keys, each of its three digit histograms summed over the cluster the same
// way.  Every cluster barrier sits in control flow that is the same in all
// eight CTAs: each branch depends only on values the whole cluster shares.
#include "heta_internal.cuh"
#include "radix_select.cuh"
#include "route_common.cuh"

namespace heta {
namespace {

using namespace rt;

constexpr int kCl = 8;  // CTAs a sample
constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster; shared-memory writes before it are
// visible to the whole cluster after it.
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// CTA `rank`'s copy of the shared variable at p, as a generic address: plain
// loads through it (ordered by the cluster barriers like any shared-memory
// access) let the compiler keep several of them in flight.
template <class T>
__device__ __forceinline__ const T *peer(const T *p, uint32_t rank)
{
    uint64_t r;
    asm("mapa.u64 %0, %1, %2;" : "=l"(r) : "l"(reinterpret_cast<uint64_t>(p)), "r"(rank));
    return reinterpret_cast<const T *>(r);
}

// A 32-bit word of CTA `rank`'s copy of the shared variable at p.
__device__ __forceinline__ uint32_t ld_peer(const void *p, uint32_t rank)
{
    return *peer(static_cast<const uint32_t *>(p), rank);
}

// hist_all[i] = the sum over the cluster's CTAs of hist[i], i < nbins
// (nbins = 1024 or 2048): four bins a 16-byte remote load, and every load a
// thread makes is issued before any of them is used.
__device__ __forceinline__ void merge_hist(const uint32_t *hist, uint32_t *hist_all, int nbins)
{
    const int i = 4 * (int)threadIdx.x;
    if (i < nbins) {  // (no barrier inside)
        uint4 a[kCl];
#pragma unroll
        for (int r = 0; r < kCl; ++r) a[r] = *peer(reinterpret_cast<const uint4 *>(hist + i), (uint32_t)r);
        uint4 sum = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int r = 0; r < kCl; ++r) {
            sum.x += a[r].x;
            sum.y += a[r].y;
            sum.z += a[r].z;
            sum.w += a[r].w;
        }
        *reinterpret_cast<uint4 *>(hist_all + i) = sum;
    }
}

template <bool kMask>
__global__ void __launch_bounds__(kThreads, 1)
route_cluster_kernel(const float *__restrict__ u, int N, int k,
                     int32_t *__restrict__ dense_idx, int32_t *__restrict__ local_idx,
                     float *__restrict__ thresh, uint8_t *__restrict__ mask, int32_t *status)
{
    // this CTA's slice of the sample: local quad q holds the sample's slot
    // quad c_lo + q (slots share u's 16-byte phase, as in route.cu)
    extern __shared__ uint4 slot4[];
    uint32_t *slot = reinterpret_cast<uint32_t *>(slot4);
    __shared__ __align__(16) uint32_t hist[kBins];      // this CTA's counts
    __shared__ __align__(16) uint32_t hist_all[kBins];  // the cluster's
    __shared__ uint32_t cand_w[kCandCap];
    __shared__ int cand_t[kCandCap];
    __shared__ uint32_t all_w[kCandCap];  // the cluster's candidates
    __shared__ uint32_t cnt_gt[kCandCap], cnt_eq[kCandCap];
    __shared__ uint32_t warp_tot[kWarps];
    __shared__ float w_min[kWarps], w_max[kWarps];
    __shared__ float s_mm[2];        // this CTA's min and max
    __shared__ uint32_t s_tot[2];    // this CTA's tokens above T, equal to T
    __shared__ uint32_t s_coff[kCl + 1];
    __shared__ uint32_t w_gt[kWarps], w_eq[kWarps];
    __shared__ uint32_t w_dense_before[kWarps], w_eq_before[kWarps];
    __shared__ uint32_t s_digit, s_rank, s_ncand, s_kstar, s_take;
    __shared__ int s_nan;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float kInf = __uint_as_float(0x7f800000u);
    const uint32_t rank = cluster_rank();
    const int b = blockIdx.x / kCl;
    const float *ub = u + (size_t)b * N;

    const int off = (int)((reinterpret_cast<uintptr_t>(ub) >> 2) & 3u);
    const int nslots = off + N;
    const int nq = (nslots + 3) >> 2;
    const int qc = (nq + kCl - 1) / kCl;
    const int c_lo = min(nq, (int)rank * qc);
    const int c_hi = min(nq, c_lo + qc);
    // local coordinates: quad q of this CTA is slot quad c_lo + q; slot s of it
    // holds token s - loff
    const int loff = off - 4 * c_lo;
    const int lslots = nslots - 4 * c_lo;
    const int nql = c_hi - c_lo;
    const int pq = (nql + kThreads - 1) / kThreads;
    const int wq = 32 * pq;
    const int q_lo = warp * wq;
    const int q_hi = max(q_lo, min(nql, q_lo + wq));
    const int t_lo = min(N, max(0, 4 * (c_lo + q_lo) - off));
    const int t_hi = min(N, max(t_lo, 4 * (c_lo + q_hi) - off));
    // the sample's partial quads (at its two ends), in local coordinates
    const int qa = (off && c_lo == 0) ? 1 : 0;
    const int qb = ((nslots & 3) && c_hi == nq) ? nql - 1 : nql;
    const int qp0 = (off && c_lo == 0 && nql > 0) ? 0 : -1;
    const int qp1 = ((nslots & 3) && c_hi == nq && nql > 0 && nql - 1 != qp0) ? nql - 1 : -1;
    auto owns = [&](int q) { return q >= q_lo && q < q_hi && ((q - q_lo) & 31) == lane; };

    if (tid == 0) {
        s_nan = 0;
        s_ncand = 0u;
    }
    for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
    if (tid < kCandCap) {
        cnt_gt[tid] = 0u;
        cnt_eq[tid] = 0u;
    }

    // ---- 1. the slice -> shared memory; the cluster's min and max
    float mn = kInf, mx = -kInf;
    {
        const uint4 *g4 = reinterpret_cast<const uint4 *>(ub - off) + c_lo;
        for (int q = q_lo + lane; q < min(q_hi, qb); q += 32) {
            if (q < qa) continue;
            const uint4 v = __ldg(g4 + q);
            slot4[q] = v;
            const float a = __uint_as_float(v.x), c = __uint_as_float(v.y);
            const float d = __uint_as_float(v.z), e = __uint_as_float(v.w);
            mn = min3n(mn, a, c);
            mn = min3n(mn, d, e);
            mx = max3n(mx, a, c);
            mx = max3n(mx, d, e);
        }
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int q = p ? qp1 : qp0;
            if (q >= 0 && owns(q)) {
                for (int s = max(4 * q, loff); s < min(4 * q + 4, lslots); ++s) {
                    const float x = __ldg(ub + (s - loff));
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
    if (warp == 0) {
        mn = w_min[lane];
        mx = w_max[lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = min2n(mn, __shfl_xor_sync(kFull, mn, o));
            mx = max2n(mx, __shfl_xor_sync(kFull, mx, o));
        }
        if (lane == 0) {
            s_mm[0] = mn;
            s_mm[1] = mx;
        }
    }
    cluster_sync();  // (1) every CTA's min / max
    mn = kInf;
    mx = -kInf;
    if (lane < kCl) {
        mn = __uint_as_float(ld_peer(&s_mm[0], (uint32_t)lane));
        mx = __uint_as_float(ld_peer(&s_mm[1], (uint32_t)lane));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = min2n(mn, __shfl_xor_sync(kFull, mn, o));
        mx = max2n(mx, __shfl_xor_sync(kFull, mx, o));
    }
    // (the same in every thread of the cluster: the same eight values, reduced
    // in the same order)
    const bool finite = mn > -kInf && mx < kInf;
    const float lo = mn;
    const float span = __fsub_rn(mx, mn);
    const float scale = __fdiv_rn(2044.f, span);
    const float lo_scale = __fmul_rn(lo, scale);
    const bool one_op = fabsf(lo_scale) <= 4194304.f;
    const float cb = one_op ? __fsub_rn(8388610.f, lo_scale) : 8388610.f;
    bool fast = k > 0 && finite && span > 0.f && scale > 0.f && scale < kInf;
    uint32_t rank_in_bucket = 0u, bstar = 0u;

    // ---- 2. bucket histograms, summed over the cluster
    if (fast) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int q = p ? qp1 : qp0;
            if (q >= 0 && owns(q)) {
                for (int s = 4 * q; s < 4 * q + 4; ++s)
                    if (s < loff || s >= lslots) slot[s] = __float_as_uint(lo);
            }
        }
        const uint32_t hist_at_magic = (uint32_t)__cvta_generic_to_shared(hist) - 4u * kMagicBits;
        if (one_op)
            bucket_histogram<true>(slot4, q_lo, q_hi, lane, lo, scale, cb, hist_at_magic);
        else
            bucket_histogram<false>(slot4, q_lo, q_hi, lane, lo, scale, cb, hist_at_magic);
        cluster_sync();  // (2) every CTA's histogram
        merge_hist(hist, hist_all, kBins);
        __syncthreads();
        find_digit<kThreads>(hist_all, kBins, (uint32_t)k, warp_tot, &s_digit, &s_rank);
        bstar = s_digit;
        rank_in_bucket = s_rank;
        fast = hist_all[bstar] <= (uint32_t)kCandCap;  // (the cluster's sum: the same everywhere)
    }

    if (fast) {
        // ---- 3. candidates and per-warp counts above them; the merged rank
        const uint32_t bbits = kMagicBits + bstar;
        const uint32_t above =
            one_op ? bucket_candidates<true>(slot4, q_lo, q_hi, lane, lo, scale, cb, bbits, loff,
                                             lslots, &s_ncand, cand_w, cand_t, kCandCap)
                   : bucket_candidates<false>(slot4, q_lo, q_hi, lane, lo, scale, cb, bbits,
                                              loff, lslots, &s_ncand, cand_w, cand_t, kCandCap);
        if (lane == 0) {
            w_gt[warp] = above;
            w_eq[warp] = 0u;
        }
        cluster_sync();  // (3) every CTA's candidates
        if (warp == 0) {
            const uint32_t n = lane < kCl ? ld_peer(&s_ncand, (uint32_t)lane) : 0u;
            uint32_t incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += t;
            }
            const uint32_t before = __shfl_up_sync(kFull, incl, 1);  // every lane takes part
            if (lane <= kCl) s_coff[lane] = lane == 0 ? 0u : before;
        }
        __syncthreads();
        const int c = (int)min(s_coff[kCl], (uint32_t)kCandCap);
        if (warp < kCl) {  // warp r copies CTA r's candidates
            const int o0 = (int)s_coff[warp], n = (int)s_coff[warp + 1] - o0;
            for (int j = lane; j < n; j += 32)
                if (o0 + j < kCandCap) all_w[o0 + j] = ld_peer(cand_w + j, (uint32_t)warp);
        }
        __syncthreads();
        {
            const int j0 = warp * c / kWarps, j1 = (warp + 1) * c / kWarps;
            if (j0 < j1) {
                for (int i = lane; i < c; i += 32) {
                    const float vi = __uint_as_float(all_w[i]);
                    uint32_t g = 0u, e = 0u;
                    for (int j = j0; j < j1; ++j) {
                        const float vj = __uint_as_float(all_w[j]);
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
            uint32_t tw = 0u, take = 0u;
            bool found = false;
            for (int i = lane; i < c; i += 32) {
                const uint32_t g = cnt_gt[i], e = cnt_eq[i];
                if (g < rank_in_bucket && rank_in_bucket <= g + e) {
                    tw = all_w[i];
                    take = rank_in_bucket - g;
                    found = true;
                }
            }
            const unsigned fm = __ballot_sync(kFull, found);
            const int src = fm ? __ffs(fm) - 1 : 0;
            tw = __shfl_sync(kFull, tw, src);
            take = __shfl_sync(kFull, take, src);
            const float fst = __uint_as_float(tw);
            // this CTA's own candidates above T and equal to it, per owning warp
            const int nc = (int)min(s_ncand, (uint32_t)kCandCap);
            for (int i = lane; i < nc; i += 32) {
                const float v = __uint_as_float(cand_w[i]);
                const int owner = (((cand_t[i] + off) >> 2) - c_lo) / wq;
                if (v > fst) atomicAdd(&w_gt[owner], 1u);
                else if (v == fst) atomicAdd(&w_eq[owner], 1u);
            }
            if (lane == 0) {
                s_kstar = tw;
                s_take = take;
                if (thresh && rank == 0) thresh[b] = fst;
            }
        }
    } else if (k > 0) {
        // ---- 2'-3'. radix select on order keys, each digit histogram summed
        // over the cluster
        cluster_sync();  // (every CTA has read the bucket histograms)
        for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
        __syncthreads();
        bool nan_seen = false;
        for (int q = q_lo + lane; q < q_hi; q += 32) {
            const uint4 v = slot4[q];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t key[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int s = 4 * q + e;
                const float f = __uint_as_float(w[e]);
                const bool tok = s >= loff && s < lslots;
                nan_seen |= tok && (f != f);
                key[e] = tok ? order_key(f) : 0u;
                atomicAdd(&hist[key[e] >> 21], 1u);
            }
            slot4[q] = make_uint4(key[0], key[1], key[2], key[3]);
        }
        if (nan_seen) s_nan = 1;
        cluster_sync();
        merge_hist(hist, hist_all, kBins);
        __syncthreads();
        find_digit<kThreads>(hist_all, kBins, (uint32_t)k, warp_tot, &s_digit, &s_rank);
        const uint32_t d1 = s_digit, r1 = s_rank;
        cluster_sync();  // (every CTA has read the histograms)
        for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int q = q_lo + lane; q < q_hi; q += 32) {
            const uint4 v = slot4[q];
            if ((v.x >> 21) == d1) atomicAdd(&hist[(v.x >> 10) & 2047u], 1u);
            if ((v.y >> 21) == d1) atomicAdd(&hist[(v.y >> 10) & 2047u], 1u);
            if ((v.z >> 21) == d1) atomicAdd(&hist[(v.z >> 10) & 2047u], 1u);
            if ((v.w >> 21) == d1) atomicAdd(&hist[(v.w >> 10) & 2047u], 1u);
        }
        cluster_sync();
        merge_hist(hist, hist_all, kBins);
        __syncthreads();
        find_digit<kThreads>(hist_all, kBins, r1, warp_tot, &s_digit, &s_rank);
        const uint32_t p2 = (d1 << 11) | s_digit, r2 = s_rank;
        cluster_sync();
        for (int i = tid; i < 1024; i += kThreads) hist[i] = 0u;
        __syncthreads();
        for (int q = q_lo + lane; q < q_hi; q += 32) {
            const uint4 v = slot4[q];
            if ((v.x >> 10) == p2) atomicAdd(&hist[v.x & 1023u], 1u);
            if ((v.y >> 10) == p2) atomicAdd(&hist[v.y & 1023u], 1u);
            if ((v.z >> 10) == p2) atomicAdd(&hist[v.z & 1023u], 1u);
            if ((v.w >> 10) == p2) atomicAdd(&hist[v.w & 1023u], 1u);
        }
        cluster_sync();
        merge_hist(hist, hist_all, 1024);
        __syncthreads();
        find_digit<kThreads>(hist_all, 1024, r2, warp_tot, &s_digit, &s_rank);
        const uint32_t kstar = (p2 << 10) | s_digit;
        uint32_t n_gt = 0u, n_eq = 0u;
        for (int t = t_lo + lane; t < t_hi; t += 32) {
            const uint32_t key = slot[t + loff];
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
            if (thresh && rank == 0) thresh[b] = key_value(kstar);
        }
    } else {
        // k == 0: nothing is dense
        if (!finite) {
            bool nan_seen = false;
            for (int q = q_lo + lane; q < q_hi; q += 32)
                for (int s = max(4 * q, loff); s < min(4 * q + 4, lslots); ++s) {
                    const float f = __uint_as_float(slot[s]);
                    nan_seen |= f != f;
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
            if (thresh && rank == 0) thresh[b] = kInf;
        }
    }
    const bool keys = !fast && k > 0;
    __syncthreads();
    if (tid == 0 && s_nan) raise_status(status, HETA_ERR_NONFINITE);

    // ---- the counts of the CTAs before this one
    if (warp == 0) {
        const uint32_t gt = w_gt[lane], eq = w_eq[lane];
        uint32_t a = gt, e = eq;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a += __shfl_xor_sync(kFull, a, o);
            e += __shfl_xor_sync(kFull, e, o);
        }
        if (lane == 0) {
            s_tot[0] = a;
            s_tot[1] = e;
        }
    }
    cluster_sync();  // (4) every CTA's totals
    if (warp == 0) {
        const uint32_t take = s_take;
        uint32_t g = 0u, e = 0u;
        if (lane < (int)rank) {
            g = ld_peer(&s_tot[0], (uint32_t)lane);
            e = ld_peer(&s_tot[1], (uint32_t)lane);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(kFull, g, o);
            e += __shfl_xor_sync(kFull, e, o);
        }
        // dense tokens before this CTA: those above T, and the ties taken so far
        const uint32_t dense0 = g + min(e, take), eq0 = e;
        const uint32_t eq = w_eq[lane], gt = w_gt[lane];
        uint32_t eq_incl = eq;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, eq_incl, o);
            if (lane >= o) eq_incl += t;
        }
        const uint32_t eq_before = eq0 + eq_incl - eq;
        const uint32_t taken_eq = take > eq_before ? min(eq, take - eq_before) : 0u;
        const uint32_t dense_here = gt + taken_eq;
        uint32_t d_incl = dense_here;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, d_incl, o);
            if (lane >= o) d_incl += t;
        }
        w_dense_before[lane] = dense0 + d_incl - dense_here;
        w_eq_before[lane] = eq_before;
    }
    __syncthreads();

    // ---- 4. compaction of this CTA's tokens
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
                compact<true, true, kMask>(slot, loff, t_lo, t_hi, kst, take, rd, re, dout, lout,
                                           mout, ku, nl, lane);
            else
                compact<true, false, kMask>(slot, loff, t_lo, t_hi, kst, take, rd, re, dout,
                                            lout, mout, ku, nl, lane);
        } else {
            if (has_eq)
                compact<false, true, kMask>(slot, loff, t_lo, t_hi, kst, take, rd, re, dout,
                                            lout, mout, ku, nl, lane);
            else if (!kMask)
                compact_float_plain(slot, loff, t_lo, t_hi, kst, rd, dout, lout, lane);
            else
                compact<false, false, true>(slot, loff, t_lo, t_hi, kst, take, rd, re, dout,
                                            lout, mout, ku, nl, lane);
        }
    }
    cluster_sync();  // (5) no CTA leaves while another may still read its shared memory
}

}  // namespace

bool route_cluster_fits(int B, int N)
{
    return B >= 1 && N <= kRouteClusterMaxN && (B <= kRouteClusterMaxB || N > kRouteMaxN);
}

cudaError_t launch_route_cluster(const float *u, int B, int N, int k, int32_t *dense_idx,
                                 int32_t *local_idx, float *thresh, uint8_t *mask,
                                 int32_t *status, cudaStream_t s)
{
    // a slice: up to ceil(quads / 8) quads
    const int nq = (N + 3 + 3) / 4;
    const size_t smem = sizeof(uint4) * (size_t)((nq + kCl - 1) / kCl);
    const int max_smem = (int)(sizeof(uint4) * ((kRouteClusterMaxN / 4 + 2 + kCl - 1) / kCl));
    auto kern = mask ? route_cluster_kernel<true> : route_cluster_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         max_smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(B * kCl), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, u, N, k, dense_idx, local_idx, thresh, mask, status);
}

}  // namespace heta
