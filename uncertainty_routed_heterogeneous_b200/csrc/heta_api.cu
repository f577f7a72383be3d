// heta_api.cu -- the extern "C" entry points of libheta (declared in heta.h):
// host-side argument checks, then one asynchronous launch sequence each.
#include <math.h>

#include <cmath>

#include "heta_internal.cuh"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

heta_status from_cuda(cudaError_t e) { return e == cudaSuccess ? HETA_OK : HETA_ERR_CUDA; }

}  // namespace

extern "C" {

const char *heta_status_string(int status)
{
    switch (status) {
    case HETA_OK: return "ok";
    case HETA_ERR_INVALID_ARG: return "invalid argument";
    case HETA_ERR_UNSUPPORTED: return "unsupported configuration";
    case HETA_ERR_CUDA: return "CUDA error";
    case HETA_ERR_NONFINITE: return "non-finite (NaN) uncertainty value";
    case HETA_ERR_TIMEOUT: return "bounded wait in a kernel timed out";
    default: return "unknown status";
    }
}

int heta_version(void) { return (1 << 16) | 1; }

heta_status heta_dense_count(int N, double rho, int *k_out)
{
    if (!k_out || N < 0 || !(rho >= 0.0 && rho <= 1.0)) return HETA_ERR_INVALID_ARG;
    const double prod = rho * (double)N;
    const double nearest = nearbyint(prod);
    const double tol = 1e-12 * (prod > 1.0 ? prod : 1.0);
    int k = fabs(prod - nearest) <= tol ? (int)nearest : (int)ceil(prod);
    *k_out = k > N ? N : k;
    return HETA_OK;
}

heta_status heta_route(const float *u, int B, int N, int k, int32_t *dense_idx,
                       int32_t *local_idx, float *thresh_out, uint8_t *mask_out,
                       int32_t *status_dev, void *stream)
{
    if (B < 1 || N < 1 || k < 0 || k > N) return HETA_ERR_INVALID_ARG;
    if ((int64_t)B * N >= (int64_t)1 << 31) return HETA_ERR_INVALID_ARG;
    if (N > heta::kRouteClusterMaxN) return HETA_ERR_UNSUPPORTED;
    if (!u || (k > 0 && !dense_idx) || (k < N && !local_idx)) return HETA_ERR_INVALID_ARG;
    if (!aligned16(u) || (dense_idx && !aligned16(dense_idx)) ||
        (local_idx && !aligned16(local_idx)) || (thresh_out && !aligned16(thresh_out)) ||
        (mask_out && !aligned16(mask_out)))
        return HETA_ERR_INVALID_ARG;
    if (heta::route_cluster_fits(B, N))
        return from_cuda(heta::launch_route_cluster(u, B, N, k, dense_idx, local_idx, thresh_out,
                                                    mask_out, status_dev,
                                                    static_cast<cudaStream_t>(stream)));
    return from_cuda(heta::launch_route(u, B, N, k, dense_idx, local_idx, thresh_out,
                                        mask_out, status_dev,
                                        static_cast<cudaStream_t>(stream)));
}

heta_status heta_route_swap_blocks(const int32_t *dense_idx, int B, int N, int k, int s,
                                   uint64_t seed, int block0, int nblocks, int32_t *dense_out,
                                   int32_t *local_out, uint8_t *mask_out, int32_t *status_dev,
                                   void *stream)
{
    if (B < 1 || N < 1 || k < 0 || k > N) return HETA_ERR_INVALID_ARG;
    if (s < 0 || s > k || s > N - k || block0 < 0 || nblocks < 1) return HETA_ERR_INVALID_ARG;
    if ((int64_t)block0 + nblocks - 1 > INT32_MAX) return HETA_ERR_INVALID_ARG;
    if ((int64_t)B * N * nblocks >= (int64_t)1 << 31) return HETA_ERR_INVALID_ARG;
    if ((int64_t)B * nblocks > INT32_MAX) return HETA_ERR_INVALID_ARG;
    if (N > heta::kRouteClusterMaxN) return HETA_ERR_UNSUPPORTED;
    if ((k > 0 && (!dense_idx || !dense_out)) || (k < N && !local_out))
        return HETA_ERR_INVALID_ARG;
    if ((dense_idx && !aligned16(dense_idx)) || (dense_out && !aligned16(dense_out)) ||
        (local_out && !aligned16(local_out)) || (mask_out && !aligned16(mask_out)))
        return HETA_ERR_INVALID_ARG;
    if (nblocks > 1 && k > 0) {
        // the input must not be overwritten while another block still reads it
        const uintptr_t in0 = reinterpret_cast<uintptr_t>(dense_idx);
        const uintptr_t in1 = in0 + sizeof(int32_t) * (size_t)B * k;
        const uintptr_t out0 = reinterpret_cast<uintptr_t>(dense_out);
        const uintptr_t out1 = out0 + sizeof(int32_t) * (size_t)B * k * nblocks;
        if (in0 < out1 && out0 < in1) return HETA_ERR_INVALID_ARG;
    }
    return from_cuda(heta::launch_route_swap(dense_idx, B, N, k, s, seed, block0, nblocks,
                                             dense_out, local_out, mask_out, status_dev,
                                             static_cast<cudaStream_t>(stream)));
}

heta_status heta_route_swap(const int32_t *dense_idx, int B, int N, int k, int s,
                            uint64_t seed, int block, int32_t *dense_out, int32_t *local_out,
                            uint8_t *mask_out, int32_t *status_dev, void *stream)
{
    return heta_route_swap_blocks(dense_idx, B, N, k, s, seed, block, 1, dense_out, local_out,
                                  mask_out, status_dev, stream);
}

heta_status heta_route_threshold(const float *u, int B, int N, double c, int32_t *counts,
                                 int32_t *dense_idx, int32_t *local_idx, double *thresh_out,
                                 uint8_t *mask_out, int32_t *status_dev, void *stream)
{
    if (B < 1 || N < 1 || !std::isfinite(c)) return HETA_ERR_INVALID_ARG;
    if ((int64_t)B * N >= (int64_t)1 << 31) return HETA_ERR_INVALID_ARG;
    if (N > heta::kRouteClusterMaxN) return HETA_ERR_UNSUPPORTED;
    if (!u || !counts || !dense_idx || !local_idx) return HETA_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(counts) || !aligned16(dense_idx) || !aligned16(local_idx) ||
        (thresh_out && !aligned16(thresh_out)) || (mask_out && !aligned16(mask_out)))
        return HETA_ERR_INVALID_ARG;
    return from_cuda(heta::launch_route_threshold(u, B, N, c, counts, dense_idx, local_idx,
                                                  thresh_out, mask_out, status_dev,
                                                  static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

heta_status check_attention_shape(int B, int H, int d, int Tg, int Hg, int Wg, int wt, int wh,
                                  int ww, int k)
{
    if (B < 1 || H < 1 || Tg < 1 || Hg < 1 || Wg < 1) return HETA_ERR_INVALID_ARG;
    const int64_t N64 = (int64_t)Tg * Hg * Wg;
    if (N64 >= (int64_t)1 << 31) return HETA_ERR_INVALID_ARG;
    if (k < 0 || k > N64) return HETA_ERR_INVALID_ARG;
    if (wt < 1 || wh < 1 || ww < 1 || wt > Tg || wh > Hg || ww > Wg) return HETA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return HETA_ERR_UNSUPPORTED;
    if ((wt % 2) == 0 || (wh % 2) == 0 || (ww % 2) == 0) return HETA_ERR_UNSUPPORTED;
    if ((int64_t)B * H * N64 * d >= (int64_t)1 << 40) return HETA_ERR_UNSUPPORTED;
    if ((int64_t)B * H >= (int64_t)1 << 16) return HETA_ERR_UNSUPPORTED;
    return HETA_OK;
}

}  // namespace

namespace heta {

int attention_checked(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int B, int H,
                      int d, int Tg, int Hg, int Wg, int wt, int wh, int ww, float scale,
                      const int32_t *dense_idx, int k, uint16_t *out, void *workspace,
                      size_t workspace_bytes, int32_t *status_dev, void *stream,
                      bool allow_split)
{
    const int N = Tg * Hg * Wg;
    if (!(scale > 0.f) || !std::isfinite(scale)) return HETA_ERR_INVALID_ARG;
    if (!Q || !K || !V || !out || (k > 0 && !dense_idx) || !workspace)
        return HETA_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) ||
        (dense_idx && !aligned16(dense_idx)) || !aligned16(workspace))
        return HETA_ERR_INVALID_ARG;
    const AttnPlan plan =
        plan_attention(B, H, d, N, k, Tg, Hg, Wg, wt, wh, ww, plan_sms(), false, allow_split);
    if (workspace_bytes < plan.workspace_bytes) return HETA_ERR_INVALID_ARG;
    AttnArgs a;
    a.Q = Q; a.K = K; a.V = V; a.out = out; a.dense_idx = dense_idx; a.status = status_dev;
    a.k_dev = nullptr;
    a.B = B; a.H = H; a.d = d; a.N = N; a.k = k;
    a.Tg = Tg; a.Hg = Hg; a.Wg = Wg; a.wt = wt; a.wh = wh; a.ww = ww;
    a.scale = scale;
    return from_cuda(launch_attention(a, plan, workspace, static_cast<cudaStream_t>(stream)));
}

}  // namespace heta

extern "C" {

heta_status heta_attention_workspace_size(int B, int H, int d, int Tg, int Hg, int Wg, int wt,
                                          int wh, int ww, int k, size_t *bytes)
{
    if (!bytes) return HETA_ERR_INVALID_ARG;
    const heta_status st = check_attention_shape(B, H, d, Tg, Hg, Wg, wt, wh, ww, k);
    if (st != HETA_OK) return st;
    *bytes = heta::plan_attention(B, H, d, Tg * Hg * Wg, k, Tg, Hg, Wg, wt, wh, ww,
                                  heta::plan_sms())
                 .workspace_bytes;
    return HETA_OK;
}

heta_status heta_attention_counts_workspace_size(int B, int H, int d, int Tg, int Hg, int Wg,
                                                 int wt, int wh, int ww, int k_cap,
                                                 size_t *bytes)
{
    if (!bytes) return HETA_ERR_INVALID_ARG;
    const heta_status st = check_attention_shape(B, H, d, Tg, Hg, Wg, wt, wh, ww, k_cap);
    if (st != HETA_OK) return st;
    if (B > heta::kMaxCountsSamples) return HETA_ERR_UNSUPPORTED;
    *bytes = heta::plan_attention(B, H, d, Tg * Hg * Wg, k_cap, Tg, Hg, Wg, wt, wh, ww,
                                  heta::plan_sms(), true)
                 .workspace_bytes;
    return HETA_OK;
}

heta_status heta_attention(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int B,
                           int H, int d, int Tg, int Hg, int Wg, int wt, int wh, int ww,
                           float scale, const int32_t *dense_idx, int k, uint16_t *out,
                           void *workspace, size_t workspace_bytes, int32_t *status_dev,
                           void *stream)
{
    const heta_status st = check_attention_shape(B, H, d, Tg, Hg, Wg, wt, wh, ww, k);
    if (st != HETA_OK) return st;
    return static_cast<heta_status>(heta::attention_checked(
        Q, K, V, B, H, d, Tg, Hg, Wg, wt, wh, ww, scale, dense_idx, k, out, workspace,
        workspace_bytes, status_dev, stream, true));
}

heta_status heta_attention_counts(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                                  int B, int H, int d, int Tg, int Hg, int Wg, int wt, int wh,
                                  int ww, float scale, const int32_t *dense_idx, int k_cap,
                                  const int32_t *counts, uint16_t *out, void *workspace,
                                  size_t workspace_bytes, int32_t *status_dev, void *stream)
{
    const heta_status st = check_attention_shape(B, H, d, Tg, Hg, Wg, wt, wh, ww, k_cap);
    if (st != HETA_OK) return st;
    if (B > heta::kMaxCountsSamples) return HETA_ERR_UNSUPPORTED;
    const int N = Tg * Hg * Wg;
    if (!(scale > 0.f) || !isfinite(scale)) return HETA_ERR_INVALID_ARG;
    if (!Q || !K || !V || !out || !counts || (k_cap > 0 && !dense_idx) || !workspace)
        return HETA_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) ||
        !aligned16(counts) || (dense_idx && !aligned16(dense_idx)) || !aligned16(workspace))
        return HETA_ERR_INVALID_ARG;
    const heta::AttnPlan plan =
        heta::plan_attention(B, H, d, N, k_cap, Tg, Hg, Wg, wt, wh, ww, heta::plan_sms(), true);
    if (workspace_bytes < plan.workspace_bytes) return HETA_ERR_INVALID_ARG;
    heta::AttnArgs a;
    a.Q = Q; a.K = K; a.V = V; a.out = out; a.dense_idx = dense_idx; a.status = status_dev;
    a.k_dev = counts;
    a.B = B; a.H = H; a.d = d; a.N = N; a.k = k_cap;
    a.Tg = Tg; a.Hg = Hg; a.Wg = Wg; a.wt = wt; a.wh = wh; a.ww = ww;
    a.scale = scale;
    return from_cuda(heta::launch_attention(a, plan, workspace, static_cast<cudaStream_t>(stream)));
}

heta_status heta_uncertainty(const uint16_t *X, const float *w, float bias, int B, int N,
                             int C, float *u_out, int32_t *status_dev, void *stream)
{
    (void)status_dev;  // the head has no device-detected conditions
    if (B < 1 || N < 1 || C < 8 || (C % 8) != 0) return HETA_ERR_INVALID_ARG;
    if (C > 16384) return HETA_ERR_UNSUPPORTED;
    if ((int64_t)B * N >= (int64_t)1 << 31) return HETA_ERR_INVALID_ARG;
    if (!X || !w || !u_out) return HETA_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(w) || !aligned16(u_out)) return HETA_ERR_INVALID_ARG;
    if (!isfinite(bias)) return HETA_ERR_INVALID_ARG;
    return from_cuda(heta::launch_uncertainty(X, w, bias, B, N, C, u_out,
                                              static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
