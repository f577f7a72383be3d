// uncertainty.cu -- the per-token uncertainty head, u = softplus(X.w + b).
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion", §3.2.1 Eq. (7): a lightweight branch predicts u_i >= 0 per
// token; its output routes the next denoising step (§3.2.2, §4 Training
// Setting).  Read here as one linear map C -> 1 followed by softplus.
//
// HBM-bound GEMV: every byte of X is read once with 16-byte streaming loads
// (no L1 allocation); one warp per token row, fp32 accumulation, warp-shuffle
// reduction, softplus in the epilogue.  When C is a multiple of 256 (up to
// 3072; the DiT widths), a row is U = C/256 16-byte chunks per lane and every
// lane always meets the same chunk columns, so its 8U weights live in
// registers and two rows per warp stay in flight; other C stage w in shared
// memory and walk rows in slices.
#include <cuda_bf16.h>

#include "heta_internal.cuh"

namespace heta {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float dot8(uint4 x, const float *w)
{
    const float4 w0 = *reinterpret_cast<const float4 *>(w);
    const float4 w1 = *reinterpret_cast<const float4 *>(w + 4);
    // a bf16 is the high half of the fp32 with the same value
    float s = __uint_as_float(x.x << 16) * w0.x;
    s = fmaf(__uint_as_float(x.x & 0xffff0000u), w0.y, s);
    s = fmaf(__uint_as_float(x.y << 16), w0.z, s);
    s = fmaf(__uint_as_float(x.y & 0xffff0000u), w0.w, s);
    s = fmaf(__uint_as_float(x.z << 16), w1.x, s);
    s = fmaf(__uint_as_float(x.z & 0xffff0000u), w1.y, s);
    s = fmaf(__uint_as_float(x.w << 16), w1.z, s);
    s = fmaf(__uint_as_float(x.w & 0xffff0000u), w1.w, s);
    return s;
}

__device__ __forceinline__ float softplus(float z)
{
    return z > 0.f ? z + log1pf(expf(-z)) : log1pf(expf(z));
}

// A warp walks its rows in slices of 32 * UNROLL 16-byte chunks (one slice
// is a whole row at C <= 256 * UNROLL).  The next slice's UNROLL loads per
// lane are issued before the current slice is consumed, so loads stay in
// flight through the arithmetic, the shuffle reduction and the store.
template <int UNROLL>
__global__ void __launch_bounds__(kThreads, 2)
uncertainty_kernel(const uint16_t *__restrict__ X, const float *__restrict__ w,
                   float bias, int64_t rows, int C, float *__restrict__ u)
{
    extern __shared__ float ws[];
    for (int c = threadIdx.x; c < C; c += kThreads) ws[c] = w[c];
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int chunks = C >> 3;  // 8 bf16 per 16-byte chunk
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    int c0 = 0;
    auto load = [&](int64_t r, int cb, uint4 (&v)[UNROLL]) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(X + r * C);
#pragma unroll
        for (int j = 0; j < UNROLL; ++j) {
            const int c = cb + j * 32 + lane;
            v[j] = c < chunks ? ld_stream(xr + c) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    uint4 v[UNROLL];
    if (row < rows) load(row, 0, v);
    float acc = 0.f;
    while (row < rows) {
        // the slice after this one
        int64_t nrow = row;
        int nc0 = c0 + 32 * UNROLL;
        if (nc0 >= chunks) {
            nrow = row + nwarps;
            nc0 = 0;
        }
        uint4 vn[UNROLL];
        if (nrow < rows) load(nrow, nc0, vn);
#pragma unroll
        for (int j = 0; j < UNROLL; ++j) {
            const int c = c0 + j * 32 + lane;
            if (c < chunks) acc += dot8(v[j], ws + 8 * c);
        }
        if (nrow != row) {  // the row is complete
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) u[row] = softplus(acc + bias);
            acc = 0.f;
        }
        row = nrow;
        c0 = nc0;
#pragma unroll
        for (int j = 0; j < UNROLL; ++j) v[j] = vn[j];
    }
}

// C = 256 U: lane l holds chunks j * 32 + l (j < U) of every row, and their
// weights.  Each warp keeps the loads of its next row in flight while it
// reduces the current one (rows split over all warps with a grid stride).
template <int U, int NT>
__global__ void __launch_bounds__(NT, 1)
uncertainty_reg_kernel(const uint16_t *__restrict__ X, const float *__restrict__ w,
                       float bias, int64_t rows, float *__restrict__ u)
{
    constexpr int C = 256 * U;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (NT / 32);
    int64_t row = (int64_t)blockIdx.x * (NT / 32) + (threadIdx.x >> 5);
    auto load = [&](int64_t r, uint4 (&v)[U]) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(X + r * C);
#pragma unroll
        for (int j = 0; j < U; ++j)
            v[j] = r < rows ? ld_stream(xr + j * 32 + lane) : make_uint4(0u, 0u, 0u, 0u);
    };
    uint4 v[U], vn[U];
    load(row, v);
    load(row + nwarps, vn);
    float wr[U][8];
#pragma unroll
    for (int j = 0; j < U; ++j) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(w + 8 * (j * 32 + lane)));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(w + 8 * (j * 32 + lane) + 4));
        wr[j][0] = a.x; wr[j][1] = a.y; wr[j][2] = a.z; wr[j][3] = a.w;
        wr[j][4] = b.x; wr[j][5] = b.y; wr[j][6] = b.z; wr[j][7] = b.w;
    }
    while (row < rows) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < U; ++j) {
            // a bf16 is the high half of the fp32 with the same value
            acc = fmaf(__uint_as_float(v[j].x << 16), wr[j][0], acc);
            acc = fmaf(__uint_as_float(v[j].x & 0xffff0000u), wr[j][1], acc);
            acc = fmaf(__uint_as_float(v[j].y << 16), wr[j][2], acc);
            acc = fmaf(__uint_as_float(v[j].y & 0xffff0000u), wr[j][3], acc);
            acc = fmaf(__uint_as_float(v[j].z << 16), wr[j][4], acc);
            acc = fmaf(__uint_as_float(v[j].z & 0xffff0000u), wr[j][5], acc);
            acc = fmaf(__uint_as_float(v[j].w << 16), wr[j][6], acc);
            acc = fmaf(__uint_as_float(v[j].w & 0xffff0000u), wr[j][7], acc);
        }
#pragma unroll
        for (int j = 0; j < U; ++j) v[j] = vn[j];
        load(row + 2 * nwarps, vn);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) u[row] = softplus(acc + bias);
        row += nwarps;
    }
}

// One CTA an SM (grid-stride rows): 16 warps at up to 128 registers for
// U <= 6, 8 warps at up to 255 for U <= 12.
template <int U>
cudaError_t launch_reg(const uint16_t *X, const float *w, float bias, int64_t rows, float *u,
                       int sms, cudaStream_t s)
{
    constexpr int NT = U <= 6 ? 512 : 256;
    int64_t blocks = (rows + NT / 32 - 1) / (NT / 32);
    if (blocks > sms) blocks = sms;
    uncertainty_reg_kernel<U, NT><<<(unsigned)blocks, NT, 0, s>>>(X, w, bias, rows, u);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_uncertainty(const uint16_t *X, const float *w, float bias,
                               int B, int N, int C, float *u, cudaStream_t s)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t rows = (int64_t)B * N;
    switch (C) {
    case 256: return launch_reg<1>(X, w, bias, rows, u, sms, s);
    case 512: return launch_reg<2>(X, w, bias, rows, u, sms, s);
    case 768: return launch_reg<3>(X, w, bias, rows, u, sms, s);
    case 1024: return launch_reg<4>(X, w, bias, rows, u, sms, s);
    case 1280: return launch_reg<5>(X, w, bias, rows, u, sms, s);
    case 1536: return launch_reg<6>(X, w, bias, rows, u, sms, s);
    case 1792: return launch_reg<7>(X, w, bias, rows, u, sms, s);
    case 2048: return launch_reg<8>(X, w, bias, rows, u, sms, s);
    case 2304: return launch_reg<9>(X, w, bias, rows, u, sms, s);
    case 2560: return launch_reg<10>(X, w, bias, rows, u, sms, s);
    case 2816: return launch_reg<11>(X, w, bias, rows, u, sms, s);
    case 3072: return launch_reg<12>(X, w, bias, rows, u, sms, s);
    default: break;
    }
    const size_t smem = sizeof(float) * (size_t)C;
    cudaError_t e = cudaFuncSetAttribute(uncertainty_kernel<6>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    // One wave: the two CTAs of 16 warps an SM holds (64 registers a thread),
    // each warp walking rows with a grid stride, so the rows split over all
    // warps at once (a second wave would run on a partly idle GPU)
    int64_t blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 2LL * sms) blocks = 2LL * sms;
    uncertainty_kernel<6><<<(unsigned)blocks, kThreads, smem, s>>>(X, w, bias, rows, C, u);
    return cudaGetLastError();
}

}  // namespace heta
