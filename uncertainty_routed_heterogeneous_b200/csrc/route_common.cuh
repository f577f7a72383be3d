// route_common.cuh -- device pieces shared by the routing kernels (one CTA a
// sample in route.cu, a cluster of CTAs a sample in route_cluster.cu): the
// order-preserving keys, the value buckets and their passes, the exact rank
// and the ballot compactions.  Device code only; included by the .cu files.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion", §3.2.2 Eq. (11)-(12), in top-k form: exactly k tokens per sample
// go dense, equal u are taken in increasing token index, -0.0 == +0.0.
#pragma once

#include <cstdint>

#include "heta_internal.cuh"

namespace heta {
namespace rt {

constexpr int kBins = 2048;     // value buckets (and radix digits of 11 bits)
constexpr int kCandCap = 256;   // most candidates the exact rank takes
constexpr unsigned kFull = 0xffffffffu;

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

// min / max that return NaN when any operand is NaN
__device__ __forceinline__ float min3n(float a, float b, float c)
{
    float r;
    asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float max3n(float a, float b, float c)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float min2n(float a, float b)
{
    float r;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ float max2n(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// Value buckets over [lo, hi]: with scale = 2044 / (hi - lo), the bucket of x
// is round((x - lo) * scale + ~2) - read from the bits of that sum plus 2^23,
// where every float in [2^23, 2^24) is an integer.  Two forms:
//   kOneOp:  x * scale + c with c = 2^23 + 2 - lo * scale rounded (the product
//            lo * scale at most 2^22 in magnitude, so c is off by < 0.75);
//   else:    (x - lo) * scale + (2^23 + 2).
// Every rounding in either is monotone, so x > y implies bucket(x) >=
// bucket(y): a bucket above another holds only larger values.  x in [lo, hi]
// gives a sum in [2^23 + 1.25, 2^23 + 2046.75], i.e. buckets 1..2047.
constexpr uint32_t kMagicBits = 0x4B000000u;  // the bits of 2^23
template <bool kOneOp>
__device__ __forceinline__ uint32_t bucket_bits(uint32_t xbits, float lo, float scale, float c)
{
    const float x = __uint_as_float(xbits);
    return __float_as_uint(kOneOp ? __fmaf_rn(x, scale, c) : __fmaf_rn(__fsub_rn(x, lo), scale, c));
}

__device__ __forceinline__ void red_add_shared(uint32_t addr)
{
    asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}

// Histogram of the buckets of this lane's quads (slot quads q_lo + lane + 32 i).
template <bool kOneOp>
__device__ __forceinline__ void bucket_histogram(const uint4 *slot4, int q_lo, int q_hi,
                                                 int lane, float lo, float scale, float c,
                                                 uint32_t hist_at_magic)
{
    // hist_at_magic + 4 * bits is the shared address of hist[bits - kMagicBits]
    for (int q = q_lo + lane; q < q_hi; q += 32) {
        const uint4 v = slot4[q];
        red_add_shared(hist_at_magic + 4u * bucket_bits<kOneOp>(v.x, lo, scale, c));
        red_add_shared(hist_at_magic + 4u * bucket_bits<kOneOp>(v.y, lo, scale, c));
        red_add_shared(hist_at_magic + 4u * bucket_bits<kOneOp>(v.z, lo, scale, c));
        red_add_shared(hist_at_magic + 4u * bucket_bits<kOneOp>(v.w, lo, scale, c));
    }
}

// The tokens of this warp in buckets above bstar (returned, summed over the
// warp), and the candidates -- tokens in bucket bstar -- appended to
// cand_w/cand_t.  Slots outside [off, nslots) are no token.
template <bool kOneOp>
__device__ __forceinline__ uint32_t bucket_candidates(const uint4 *slot4, int q_lo, int q_hi,
                                                      int lane, float lo, float scale, float c,
                                                      uint32_t bbits, int off, int nslots,
                                                      uint32_t *ncand, uint32_t *cand_w,
                                                      int *cand_t, int cap)
{
    uint32_t above = 0u;
    const uint32_t lo_bits = __float_as_uint(lo);
    for (int qb = q_lo; qb < q_hi; qb += 32) {  // warp-uniform: the vote needs every lane
        const int q = qb + lane;
        const bool in = q < q_hi;
        const uint4 v = in ? slot4[q] : make_uint4(lo_bits, lo_bits, lo_bits, lo_bits);
        const uint32_t c0 = bucket_bits<kOneOp>(v.x, lo, scale, c);
        const uint32_t c1 = bucket_bits<kOneOp>(v.y, lo, scale, c);
        const uint32_t c2 = bucket_bits<kOneOp>(v.z, lo, scale, c);
        const uint32_t c3 = bucket_bits<kOneOp>(v.w, lo, scale, c);
        above += (c0 > bbits) + (c1 > bbits) + (c2 > bbits) + (c3 > bbits);
        const bool m0 = c0 == bbits, m1 = c1 == bbits, m2 = c2 == bbits, m3 = c3 == bbits;
        const bool mq = in && (m0 | m1 | m2 | m3);
        if (__any_sync(kFull, mq) && mq) {
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            bool m[4] = {m0, m1, m2, m3};
            uint32_t n = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int s = 4 * q + e;
                m[e] = m[e] && s >= off && s < nslots;  // a token, not padding
                n += m[e];
            }
            uint32_t at = n ? atomicAdd(ncand, n) : 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (m[e]) {
                    if (at < (uint32_t)cap) {
                        cand_w[at] = w[e];
                        cand_t[at] = 4 * q + e - off;
                    }
                    ++at;
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(kFull, above, o);
    return above;
}

// Compaction of one warp's tokens [t_lo, t_hi): token t is dense when its
// word is above kst, or equal to it and among the first `take` equal ones of
// the sample (re of them lie before this warp).  kKeys: the words are order
// keys, else floats.  kEq: this warp holds words equal to kst.  kMask: write
// the mask too.  Each token is one store, into whichever list holds it; both
// lists get one contiguous run per step, and no branch depends on the token.
//
// The float select is exact (the dense count is k by construction), so its
// stores need no bounds; the key select -- taken for inputs with NaN, among
// others -- keeps a bound on each store.
template <bool kKeys, bool kEq, bool kMask>
__device__ __forceinline__ void compact(const uint32_t *slot, int off, int t_lo, int t_hi,
                                        uint32_t kst, uint32_t take, uint32_t rd,
                                        uint32_t re, int32_t *dout, int32_t *lout,
                                        uint8_t *mout, uint32_t k, uint32_t nloc, int lane)
{
    const unsigned lt = (1u << lane) - 1u;
    const float fst = __uint_as_float(kst);
    auto step = [&](int t, bool valid) {
        uint32_t w = 0u;
        if (valid) w = slot[t + off];
        bool dense = valid && (kKeys ? w > kst : __uint_as_float(w) > fst);
        if (kEq) {
            const bool eq = valid && (kKeys ? w == kst : __uint_as_float(w) == fst);
            const unsigned em = __ballot_sync(kFull, eq);
            dense = dense || (eq && re + __popc(em & lt) < take);
            re += __popc(em);
        }
        const unsigned dm = __ballot_sync(kFull, dense);
        const uint32_t pos = rd + __popc(dm & lt);  // dense tokens before t
        const uint32_t ls = (uint32_t)t - pos;      // local tokens before t
        int32_t *const at = dense ? dout + pos : lout + ls;
        if (valid && (!kKeys || (dense ? pos < k : ls < nloc))) *at = t;
        if (kMask && valid) mout[t] = dense ? 0 : 1;
        rd += __popc(dm);
    };
    const int full_end = t_lo + ((t_hi - t_lo) & ~31);
    int base = t_lo;
#pragma unroll 4
    for (; base < full_end; base += 32) step(base + lane, true);
    if (base < t_hi) step(base + lane, base + lane < t_hi);
}

// The common case of compact (float select, no token equal to T in this warp,
// no mask) with each whole 32-token step written out as one PTX sequence:
// load, compare, ballot, rank, one store into the list that holds the token.
__device__ __forceinline__ void compact_float_plain(const uint32_t *slot, int off, int t_lo,
                                                    int t_hi, uint32_t kst, uint32_t rd,
                                                    int32_t *dout, int32_t *lout, int lane)
{
    const unsigned lt = (1u << lane) - 1u;
    const int full_end = t_lo + ((t_hi - t_lo) & ~31);
    uint32_t t = (uint32_t)(t_lo + lane);
    uint32_t at = (uint32_t)__cvta_generic_to_shared(slot + off + t_lo + lane);
    const uint64_t dbase = reinterpret_cast<uint64_t>(dout);
    const uint64_t lbase = reinterpret_cast<uint64_t>(lout);
#pragma unroll 4
    for (int base = t_lo; base < full_end; base += 32) {
        asm volatile(
            "{\n\t"
            ".reg .pred p;\n\t"
            ".reg .b32 w, dm, c, pos, idx;\n\t"
            ".reg .b64 lst, ptr;\n\t"
            "ld.shared.b32 w, [%1];\n\t"
            "setp.gt.f32 p, w, %3;\n\t"
            "vote.sync.ballot.b32 dm, p, 0xffffffff;\n\t"
            "and.b32 c, dm, %4;\n\t"
            "popc.b32 c, c;\n\t"
            "add.u32 pos, %2, c;\n\t"
            "sub.u32 idx, %0, pos;\n\t"
            "selp.b32 idx, pos, idx, p;\n\t"
            "selp.b64 lst, %5, %6, p;\n\t"
            "mad.wide.u32 ptr, idx, 4, lst;\n\t"
            "st.global.b32 [ptr], %0;\n\t"
            "popc.b32 c, dm;\n\t"
            "add.u32 %2, %2, c;\n\t"
            "add.u32 %0, %0, 32;\n\t"
            "add.u32 %1, %1, 128;\n\t"
            "}"
            : "+r"(t), "+r"(at), "+r"(rd)
            : "f"(__uint_as_float(kst)), "r"(lt), "l"(dbase), "l"(lbase)
            : "memory");
    }
    if (full_end < t_hi) {  // the last, partial step
        const bool valid = (int)t < t_hi;
        const uint32_t w = valid ? slot[t + off] : 0u;
        const bool dense = valid && __uint_as_float(w) > __uint_as_float(kst);
        const unsigned dm = __ballot_sync(kFull, dense);
        const uint32_t pos = rd + __popc(dm & lt);
        if (valid) {
            int32_t *const dst = dense ? dout + pos : lout + (t - pos);
            *dst = (int32_t)t;
        }
    }
}

}  // namespace rt
}  // namespace heta
