// heta_internal.cuh -- declarations shared by the libheta translation units.
// Not part of the public ABI (that is include/heta.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "heta.h"

namespace heta {

// Raises *status to `code` (atomic max), if a status word was given.
__device__ __forceinline__ void raise_status(int32_t *status, int32_t code)
{
    if (status) atomicMax(reinterpret_cast<int *>(status), code);
}

// Largest N one routing CTA can hold in shared memory (4 bytes per token).
constexpr int kRouteMaxN = 53248;
// Largest N the routing calls take: a cluster of eight CTAs holds one eighth
// of a sample each, up to 49152 tokens (192 KB) a CTA.  Samples above
// kRouteMaxN always take the cluster kernels, whatever the batch size.
constexpr int kRouteClusterMaxN = 8 * 49152;

cudaError_t launch_route(const float *u, int B, int N, int k, int32_t *dense_idx,
                         int32_t *local_idx, float *thresh, uint8_t *mask,
                         int32_t *status, cudaStream_t s);

// Up to this many samples, heta_route splits each sample over a cluster of
// eight CTAs (route_cluster.cu) instead of one CTA (route.cu): the same
// lists, with the latency of a single sample cut roughly by the split.
constexpr int kRouteClusterMaxB = 8;
bool route_cluster_fits(int B, int N);
cudaError_t launch_route_cluster(const float *u, int B, int N, int k, int32_t *dense_idx,
                                 int32_t *local_idx, float *thresh, uint8_t *mask,
                                 int32_t *status, cudaStream_t s);

cudaError_t launch_route_swap(const int32_t *dense_idx, int B, int N, int k, int s,
                              uint64_t seed, int block0, int nblocks, int32_t *dense_out,
                              int32_t *local_out, uint8_t *mask, int32_t *status,
                              cudaStream_t st);

cudaError_t launch_route_threshold(const float *u, int B, int N, double c, int32_t *counts,
                                   int32_t *dense_idx, int32_t *local_idx, double *thresh,
                                   uint8_t *mask, int32_t *status, cudaStream_t s);

cudaError_t launch_uncertainty(const uint16_t *X, const float *w, float bias,
                               int B, int N, int C, float *u, cudaStream_t s);

struct AttnArgs {
    const uint16_t *Q, *K, *V;
    uint16_t *out;
    const int32_t *dense_idx;  // [B][k] (row stride k)
    const int32_t *k_dev;      // [B] per-sample dense counts (<= k), or null: all k
    int32_t *status;
    int B, H, d, N, k;
    int Tg, Hg, Wg, wt, wh, ww;
    float scale;
};

// How one heta_attention call is cut into work items, and its workspace.
struct AttnPlan {
    int sms;                  // SMs the waves of dense work are planned for (the grid size)
    int tiles_d, pairs_d, n_kv_d, pairs_full, nsplit, kv_per_split, n_dense_items;
    int max_split;            // most key ranges a dense pair may be cut into
    int box_t, box_h, box_w;  // LOCAL query box (box_t * box_h * box_w == 128)
    int tiles_l, pairs_l, nbh, nbw, nkt, nkh, nkw, n_kv_l, n_local_items;
    int total_items;
    size_t off_fix, off_ml, off_o, zero_bytes, workspace_bytes;
};

// The current device's multiprocessor count, which the dense work is cut into
// waves for (only the balance and the scratch size depend on it, never the
// result); kDefaultSMs (a B200) when no device is visible.
constexpr int kDefaultSMs = 148;
int plan_sms();

// Samples heta_attention_counts takes (its per-sample pair prefix lives in
// shared memory).
constexpr int kMaxCountsSamples = 1024;

// k is the dense rows per sample, or their capacity when per_sample_counts
// (the counts are then only known on the device: LOCAL items are always planned).
// allow_split = false runs every dense pair over its whole key range, so the
// workspace is only the work counter.
AttnPlan plan_attention(int B, int H, int d, int N, int k, int Tg, int Hg, int Wg, int wt,
                        int wh, int ww, int sms, bool per_sample_counts = false,
                        bool allow_split = true);

// heta_attention's body once its shape is checked, with the split choice open
// (the allocation-free entry point turns splitting off when its fixed scratch
// is too small for it).
int attention_checked(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int B, int H,
                      int d, int Tg, int Hg, int Wg, int wt, int wh, int ww, float scale,
                      const int32_t *dense_idx, int k, uint16_t *out, void *workspace,
                      size_t workspace_bytes, int32_t *status_dev, void *stream,
                      bool allow_split);

cudaError_t launch_attention(const AttnArgs &a, const AttnPlan &plan, void *workspace,
                             cudaStream_t s);

}  // namespace heta
