// attention_simt.cu -- first, plain CUDA-core version of the routed attention.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion": Eq. (2) dense rows, Eq. (3) windowed local rows, Eq. (13) the
// row-wise merge.  One warp per output row, fp32 online softmax, each lane
// owning d/32 channels.  Slow but simple: it is the correctness baseline the
// tensor-core kernels replace.
#include "heta_internal.cuh"

namespace heta {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float bf(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

__device__ __forceinline__ uint16_t to_bf16(float f)
{
    uint32_t b = __float_as_uint(f);
    b += 0x7fffu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

template <int D>
struct RowState {
    static constexpr int CPL = D / 32;
    float q[CPL], acc[CPL], m, l;
};

template <int D>
__device__ __forceinline__ void attend_key(RowState<D> &st, const uint16_t *kr,
                                           const uint16_t *vr, int lane)
{
    constexpr int CPL = D / 32;
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) s = fmaf(st.q[c], bf(kr[lane * CPL + c]), s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float m_new = fmaxf(st.m, s);
    const float corr = exp2f(st.m - m_new);
    const float p = exp2f(s - m_new);
    st.l = st.l * corr + p;
#pragma unroll
    for (int c = 0; c < CPL; ++c) st.acc[c] = st.acc[c] * corr + p * bf(vr[lane * CPL + c]);
    st.m = m_new;
}

template <int D>
__device__ __forceinline__ void finish_row(const RowState<D> &st, uint16_t *o, int lane)
{
    constexpr int CPL = D / 32;
    const float inv = 1.f / st.l;
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[lane * CPL + c] = to_bf16(st.acc[c] * inv);
}

template <int D>
__device__ __forceinline__ void init_row(RowState<D> &st, const uint16_t *q, float scale_log2,
                                         int lane)
{
    constexpr int CPL = D / 32;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        st.q[c] = bf(q[lane * CPL + c]) * scale_log2;
        st.acc[c] = 0.f;
    }
    st.m = -INFINITY;
    st.l = 0.f;
}

// Dense rows: one warp per (b, h, r), query token dense_idx[b, r].
template <int D>
__global__ void dense_rows_kernel(AttnArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= (int64_t)a.B * a.H * a.k) return;
    const int r = (int)(gw % a.k);
    const int64_t bh = gw / a.k;
    const int b = (int)(bh / a.H);
    const int i = a.dense_idx[(int64_t)b * a.k + r];
    const int64_t base = bh * a.N * D;
    RowState<D> st;
    init_row<D>(st, a.Q + base + (int64_t)i * D, a.scale * kLog2e, lane);
    for (int j = 0; j < a.N; ++j)
        attend_key<D>(st, a.K + base + (int64_t)j * D, a.V + base + (int64_t)j * D, lane);
    finish_row<D>(st, a.out + base + (int64_t)i * D, lane);
}

__device__ __forceinline__ int window_start(int p, int extent, int w)
{
    return min(max(p - w / 2, 0), extent - w);
}

// Local rows: one warp per (b, h, i); rows whose token is in dense_idx[b]
// (found by binary search of the increasing list) are left to the dense kernel.
template <int D>
__global__ void local_rows_kernel(AttnArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= (int64_t)a.B * a.H * a.N) return;
    const int i = (int)(gw % a.N);
    const int64_t bh = gw / a.N;
    const int b = (int)(bh / a.H);
    const int32_t *dl = a.dense_idx + (int64_t)b * a.k;
    int lo = 0, hi = a.k;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (dl[mid] < i) lo = mid + 1;
        else hi = mid;
    }
    if (lo < a.k && dl[lo] == i) return;
    const int t = i / (a.Hg * a.Wg), h = (i / a.Wg) % a.Hg, w = i % a.Wg;
    const int st_ = window_start(t, a.Tg, a.wt), sh = window_start(h, a.Hg, a.wh),
              sw = window_start(w, a.Wg, a.ww);
    const int64_t base = bh * a.N * D;
    RowState<D> st;
    init_row<D>(st, a.Q + base + (int64_t)i * D, a.scale * kLog2e, lane);
    for (int tt = st_; tt < st_ + a.wt; ++tt)
        for (int hh = sh; hh < sh + a.wh; ++hh)
            for (int ww = sw; ww < sw + a.ww; ++ww) {
                const int64_t j = ((int64_t)tt * a.Hg + hh) * a.Wg + ww;
                attend_key<D>(st, a.K + base + j * D, a.V + base + j * D, lane);
            }
    finish_row<D>(st, a.out + base + (int64_t)i * D, lane);
}

template <int D>
cudaError_t launch_simt(const AttnArgs &a, cudaStream_t s)
{
    constexpr int kThreads = 256, kWarpsPerBlock = kThreads / 32;
    if (a.k < a.N) {
        const int64_t rows = (int64_t)a.B * a.H * a.N;
        local_rows_kernel<D><<<(unsigned)((rows + kWarpsPerBlock - 1) / kWarpsPerBlock),
                               kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.k > 0) {
        const int64_t rows = (int64_t)a.B * a.H * a.k;
        dense_rows_kernel<D><<<(unsigned)((rows + kWarpsPerBlock - 1) / kWarpsPerBlock),
                               kThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t s)
{
    return a.d == 64 ? launch_simt<64>(a, s) : launch_simt<128>(a, s);
}

}  // namespace heta
