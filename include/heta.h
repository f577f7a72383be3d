/*
 * heta.h -- C ABI of libheta, the B200 (sm_100a) heterogeneous-attention path.
 *
 * The method: "Where Compute Matters: Heterogeneous Attention for Efficient
 * Video Diffusion" (HetA-DiT).  A per-token uncertainty u (Eq. (7)) from the
 * previous denoising step picks, per sample, the tokens whose queries get
 * dense attention over all N keys (Eq. (2)); every other token attends over a
 * 3D spatio-temporal window of the latent grid (Eq. (3)); the two results are
 * merged row by row into one output (Eq. (13)).  The routing rule of
 * Eq. (11)-(12) is taken in top-k form: exactly k = ceil(rho*N) tokens per
 * sample go dense, rho being the dense fraction of Eq. (14).
 *
 * Conventions shared by every entry point
 *   - Every array pointer is a DEVICE pointer owned by the caller.  The
 *     library never allocates, frees or retains device memory; it holds no
 *     state between calls and is safe to call from several host threads.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream).  Calls return before the GPU
 *     finishes.
 *   - Argument errors are detected on the host and returned synchronously
 *     (HETA_ERR_INVALID_ARG / HETA_ERR_UNSUPPORTED) with nothing launched.
 *     A failed launch returns HETA_ERR_CUDA.
 *   - Conditions only the GPU can see (a NaN in u) are reported through the
 *     optional `status_dev` (device int32, may be NULL): a kernel that detects
 *     one raises it to that code with an atomic max.  The library never
 *     clears it; zero it before the call and read it after synchronising.
 *   - bf16 tensors are passed as uint16_t bit patterns (round-to-nearest-even
 *     values), fp32 as float.  All pointers must be 16-byte aligned.
 *   - Token order inside a sample is i = (t*Hg + h)*Wg + w on a latent grid
 *     of Tg x Hg x Wg = N tokens.
 */
#ifndef HETA_H
#define HETA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HETA_API __attribute__((visibility("default")))
#else
#define HETA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HETA_OK = 0,
    HETA_ERR_INVALID_ARG = 1,  /* bad size, pointer, alignment or value     */
    HETA_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels cover */
    HETA_ERR_CUDA = 3,         /* a CUDA launch or driver call failed       */
    HETA_ERR_NONFINITE = 4,    /* NaN seen in u (reported via status_dev)   */
    HETA_ERR_TIMEOUT = 5       /* a bounded wait inside a kernel ran out    */
} heta_status;

/* Static, NUL-terminated description of a status code (never NULL). */
HETA_API const char *heta_status_string(int status);

/* Library ABI version: (major << 16) | minor. */
HETA_API int heta_version(void);

/*
 * Dense tokens per sample: *k_out = ceil(rho * N).
 *
 * rho is the dense-query fraction of Eq. (14).  It is read as the decimal
 * fraction the caller states: when the IEEE product rho*N lies within 1e-12
 * (relative) of an integer, that integer is used, so rho = 0.1, N = 30 gives
 * 3.  Requires N >= 0 and 0 <= rho <= 1; otherwise HETA_ERR_INVALID_ARG.
 * Host-only; touches no device.
 */
HETA_API heta_status heta_dense_count(int N, double rho, int *k_out);

/*
 * heta_route -- per-sample top-k selection and compaction (Eq. (11)-(12)).
 *
 * For each sample b the k tokens with the largest u[b,:] form the dense set
 * D_b.  Ties at the threshold are taken in increasing token index; -0.0 and
 * +0.0 compare equal; +-inf are ordinary values.  A NaN anywhere in u raises
 * status_dev to HETA_ERR_NONFINITE (outputs are then unspecified).
 *
 *   u          [B,N] fp32, read only.
 *   dense_idx  [B,k] int32 out: D_b in increasing token order.
 *   local_idx  [B,N-k] int32 out: the complement, increasing.
 *   thresh_out [B] fp32 out, or NULL: the k-th largest u of each sample
 *              (the effective threshold T of Eq. (11)); +inf when k == 0.
 *   mask_out   [B,N] uint8 out, or NULL: the paper's m_i, 1 = local, 0 = dense.
 *   status_dev device int32, or NULL (see conventions).
 *
 * Requires B >= 1, 1 <= N <= 393216, 0 <= k <= N, B*N < 2^31.  A sample
 * of up to 53248 tokens fits one SM's shared memory: one CTA per sample,
 * or, for B <= 8, a cluster of eight CTAs per sample (the same lists, lower
 * latency).  Larger samples (a 720p Wan latent has 75600 tokens) always take
 * the cluster of eight CTAs, each holding an eighth of the sample.
 */
HETA_API heta_status heta_route(const float *u, int B, int N, int k,
                       int32_t *dense_idx, int32_t *local_idx,
                       float *thresh_out, uint8_t *mask_out,
                       int32_t *status_dev, void *stream);

/*
 * heta_route_swap -- the per-block random swap of a top-k routing (§3.2.2,
 * after Eq. (12); App. B Table 8): at transformer block `block`, s tokens of
 * each sample's dense set trade places with s tokens of its local set, so
 * uncertain tokens keep dense attention most of the time while others get
 * some.  The tokens are chosen by a counter-based generator any program can
 * reproduce: token i of sample b draws rho_i = word 0 of Philox4x32-10
 * (Salmon et al., SC 2011) with counter (i, b, block, 0) and key
 * (seed & 0xffffffff, seed >> 32); the s dense tokens with the smallest
 * (rho_i, i) go local and the s local tokens with the smallest (rho_i, i) go
 * dense.  The paper's swap ratio r (7% by default) gives s = ceil(r*N) (the
 * heta_dense_count of r), at most min(k, N-k).
 *
 *   dense_idx  [B,k] int32: a routing's dense sets, distinct ids in [0,N)
 *              (the heta_route output).  An id out of range raises status_dev
 *              to HETA_ERR_INVALID_ARG and that sample's outputs are not
 *              written; repeated ids give unspecified outputs.
 *   dense_out  [B,k] int32 out: the new dense sets, increasing.  May be
 *              dense_idx itself (each sample's row is read before written).
 *   local_out  [B,N-k] int32 out: the complements, increasing.
 *   mask_out   [B,N] uint8 out, or NULL: m_i of the new sets, 1 = local.
 *
 * Requires 0 <= s <= min(k, N-k), block >= 0, N <= 393216 and B*N < 2^31;
 * pointers 16-byte aligned.  One CTA per sample: up to N = 53248 its draws
 * are kept in shared memory, above that (a 720p latent has 75600 tokens)
 * each pass computes them again.
 */
HETA_API heta_status heta_route_swap(const int32_t *dense_idx, int B, int N, int k, int s,
                                     uint64_t seed, int block, int32_t *dense_out,
                                     int32_t *local_out, uint8_t *mask_out,
                                     int32_t *status_dev, void *stream);

/*
 * heta_route_swap_blocks -- heta_route_swap for nblocks consecutive
 * transformer blocks block0 .. block0 + nblocks - 1 in one launch (one CTA
 * per sample and block).  Every block's swap starts from the same routing, so
 * a denoising step can draw all of its blocks' routings at once instead of one
 * launch a block.  Block block0 + j of sample b writes row j*B + b of each
 * output:
 *
 *   dense_out  [nblocks,B,k] int32 out; local_out [nblocks,B,N-k] int32 out;
 *   mask_out   [nblocks,B,N] uint8 out, or NULL.
 *
 * Identical, block for block, to heta_route_swap.  Requires nblocks >= 1,
 * block0 + nblocks - 1 <= INT32_MAX, B*N*nblocks < 2^31 and, when
 * nblocks > 1, dense_out not overlapping dense_idx; else as heta_route_swap.
 */
HETA_API heta_status heta_route_swap_blocks(const int32_t *dense_idx, int B, int N, int k,
                                            int s, uint64_t seed, int block0, int nblocks,
                                            int32_t *dense_out, int32_t *local_out,
                                            uint8_t *mask_out, int32_t *status_dev,
                                            void *stream);

/*
 * heta_route_threshold -- routing by the paper's own rule (Eq. (11)-(12)):
 * per sample b, T_b = mu_b + c * sigma_b, where mu_b and sigma_b are the mean
 * and the population standard deviation of u[b,:], computed in fp64; token i
 * is dense when u[b,i] >= T_b (m_i = [u_i < T] of Eq. (12)), compared in
 * fp64.  The dense count therefore varies per sample.  Smaller c routes more
 * tokens to dense attention (c = 0.9 keeps about 18% of Gaussian u dense).
 * A NaN in u raises status_dev to HETA_ERR_NONFINITE (outputs unspecified).
 *
 *   u          [B,N] fp32, read only.
 *   c          finite.
 *   counts     [B] int32 out (device): |D_b|.
 *   dense_idx  [B,N] int32 out: row b holds D_b in increasing token order in
 *              entries 0..counts[b]-1; the rest of the row is not written.
 *   local_idx  [B,N] int32 out: row b holds the complement, increasing, in
 *              entries 0..N-counts[b]-1; the rest is not written.
 *   thresh_out [B] fp64 out, or NULL: T_b.
 *   mask_out   [B,N] uint8 out, or NULL: m_i, 1 = local, 0 = dense.
 *   status_dev device int32, or NULL.
 *
 * The sums run in one fixed order (eight slices of ceil(N/8) tokens, each
 * summed by a fixed tree, then added in slice order), so repeated calls --
 * and calls with any batch size -- give identical results; a u within a few
 * fp64 ulps of T may fall on either side compared with another summation
 * order.  Same size limits as heta_route; pointers 16-byte aligned.  For
 * B <= 8, or N > 53248, each sample is split over a cluster of eight CTAs,
 * else one CTA per sample.  heta_attention_counts consumes the outputs without a round trip
 * to the host.
 */
HETA_API heta_status heta_route_threshold(const float *u, int B, int N, double c,
                                          int32_t *counts, int32_t *dense_idx,
                                          int32_t *local_idx, double *thresh_out,
                                          uint8_t *mask_out, int32_t *status_dev,
                                          void *stream);

/*
 * heta_attention_workspace_size -- device scratch one heta_attention call
 * needs for these sizes (host-only; launches nothing).  The dense work is
 * cut into waves of the current device's multiprocessor count (148 on a
 * B200, and 148 when no device is visible), so ask with the device current
 * that the call will run on.
 *
 * The scratch holds the work-item counter of the persistent kernel and, when
 * the pairs of dense query tiles of a last, at most half-full wave of work
 * (or of a first and only, partial one) are cut into two key ranges to keep
 * all SMs busy, the partial results those ranges merge (fp32, about 1 KB per
 * row and range, half for d = 64; at most ~40 MB).  At the Wan2.1-1.3B
 * shape that is about 4 MB for rho = 0.2 and 22 MB for rho = 0.05; when no
 * pair is cut it is 256 bytes.  Same argument rules as
 * heta_attention; *bytes is only written on HETA_OK.
 */
HETA_API heta_status heta_attention_workspace_size(int B, int H, int d, int Tg, int Hg,
                                                   int Wg, int wt, int wh, int ww, int k,
                                                   size_t *bytes);

/*
 * heta_attention -- routed heterogeneous self-attention (Eq. (2), (3), (13)).
 *
 * For every sample b, head h and token i:
 *   i in D_b : out[b,h,i] = sum_j softmax_j(scale * q_i.k_j) v_j over all N
 *              keys (Eq. (2));
 *   otherwise: the same softmax restricted to the window N(i) (Eq. (3)): the
 *              box [s_t, s_t+wt) x [s_h, s_h+wh) x [s_w, s_w+ww) with
 *              s_a = clamp(a - floor(w_a/2), 0, extent_a - w_a), so every
 *              window holds exactly wt*wh*ww keys.
 * Keys and values are always all N tokens of (b,h); only queries are routed.
 *
 *   Q, K, V    [B,H,N,d] bf16, contiguous, read only.
 *   dense_idx  [B,k] int32: D_b, strictly increasing, 0 <= idx < N (the
 *              heta_route output).  Every entry is checked on the device:
 *              an entry outside [0, N), or not greater than the entry before
 *              it, raises status_dev to HETA_ERR_INVALID_ARG, and the row it
 *              names is neither read nor written through it.  The rows of the
 *              sample are then unspecified (a token near a bad entry may get
 *              its dense result, its local result or no write), but every
 *              read stays inside Q, K, V and dense_idx and every write inside
 *              out.
 *   out        [B,H,N,d] bf16 out; every row is written exactly once.  A
 *              32-byte aligned out (any fresh allocation) is written 32 bytes
 *              a store, a 16-byte aligned one 16 bytes a store (same values).
 *   scale      softmax scale, normally 1/sqrt(d).
 *   workspace  device scratch of at least heta_attention_workspace_size()
 *              bytes, 16-byte aligned, owned by the caller; its contents on
 *              entry do not matter and are garbage on return.  Calls that
 *              may run at the same time need separate workspaces.
 *
 * One persistent kernel launch (plus a small memset of the workspace's
 * counters) on `stream`.  Requires d in {64, 128}; odd wt, wh, ww with
 * 1 <= w_a <= extent_a; N = Tg*Hg*Wg; 0 <= k <= N; B*H < 65536;
 * B*H*N*d < 2^40.  Other d or even windows give HETA_ERR_UNSUPPORTED.  A
 * wait inside the kernel that exceeds about 2 s raises status_dev to
 * HETA_ERR_TIMEOUT and the kernel returns (the context stays usable).
 */
HETA_API heta_status heta_attention(const uint16_t *Q, const uint16_t *K,
                                    const uint16_t *V, int B, int H, int d,
                                    int Tg, int Hg, int Wg, int wt, int wh, int ww,
                                    float scale, const int32_t *dense_idx, int k,
                                    uint16_t *out, void *workspace,
                                    size_t workspace_bytes, int32_t *status_dev,
                                    void *stream);

/*
 * heta_attention_counts -- heta_attention with a per-sample dense count that
 * lives on the device (the heta_route_threshold output), so no count has to
 * come back to the host first.
 *
 *   dense_idx  [B,k_cap] int32: row b holds D_b, strictly increasing, in
 *              entries 0..counts[b]-1 (row stride k_cap; the rest of the row
 *              is not read).  heta_route_threshold writes k_cap = N rows.
 *   counts     [B] int32 (device): |D_b|; values outside 0..k_cap are
 *              clamped to it.
 *   workspace  at least heta_attention_counts_workspace_size(..., k_cap) bytes.
 *
 * Every other argument, requirement and error is as for heta_attention with
 * k = k_cap, and B <= 1024 (else HETA_ERR_UNSUPPORTED).  The kernel cuts the
 * dense work from the real counts, on the device, the way heta_attention
 * cuts it from k; a generous k_cap costs only a few skipped work ids.
 */
/*
 * heta_attention_counts_workspace_size -- device scratch one
 * heta_attention_counts call needs (host-only; like
 * heta_attention_workspace_size it depends on the current device's
 * multiprocessor count).  It covers whatever counts
 * the device finds (at most ~40 MB at d = 128; 256 bytes when the key range
 * is too short to split).  Same argument rules as heta_attention_counts.
 */
HETA_API heta_status heta_attention_counts_workspace_size(int B, int H, int d, int Tg, int Hg,
                                                          int Wg, int wt, int wh, int ww,
                                                          int k_cap, size_t *bytes);

HETA_API heta_status heta_attention_counts(const uint16_t *Q, const uint16_t *K,
                                           const uint16_t *V, int B, int H, int d, int Tg,
                                           int Hg, int Wg, int wt, int wh, int ww, float scale,
                                           const int32_t *dense_idx, int k_cap,
                                           const int32_t *counts, uint16_t *out,
                                           void *workspace, size_t workspace_bytes,
                                           int32_t *status_dev, void *stream);

/*
 * heta_attention_noalloc -- heta_attention without a caller workspace.
 *
 * The paper has no counterpart to this call; it exists for callers that
 * cannot allocate device memory: code that must not call cudaMalloc (a
 * real-time loop that may not block in the allocator, a host framework that
 * owns every allocation, a context where allocation is not permitted).  It
 * computes exactly what heta_attention computes, with the same arguments
 * except the workspace, and allocates nothing.
 *
 * Its scratch is a fixed 16 MiB array in the library's device memory, which
 * every GPU that loads the library keeps until the process exits.  When
 * the scratch heta_attention would use (heta_attention_workspace_size)
 * exceeds 16 MiB, no dense pair is cut into key ranges: the kernel then needs
 * only its work counter, and the result is the same up to rounding order
 * (a partly filled last wave of dense work takes longer).
 *
 * The first call on a device loads the part of the library that holds the
 * array, and the driver commits the 16 MiB at that moment (with CUDA's
 * default lazy module loading; eagerly loaded, at library load).  That first
 * call can therefore block in the driver's allocator, or fail with
 * HETA_ERR_CUDA on a full device, so make it a warm-up call outside any
 * region that must not allocate, and before any stream capture.  It also
 * looks up the array's device address (a host-side runtime query, with that
 * device current); the address is remembered per device and context and
 * looked up again when another context is current (a new primary context
 * after cudaDeviceReset loads the module, and commits the array, anew).
 * All calls share the array and it keeps the last call's contents; each call
 * clears what must start at zero.  Calls whose kernels may overlap on the
 * GPU (unordered streams) race on the array: order them.
 */
HETA_API heta_status heta_attention_noalloc(const uint16_t *Q, const uint16_t *K,
                                            const uint16_t *V, int B, int H, int d,
                                            int Tg, int Hg, int Wg, int wt, int wh, int ww,
                                            float scale, const int32_t *dense_idx, int k,
                                            uint16_t *out, int32_t *status_dev,
                                            void *stream);

/*
 * heta_uncertainty -- the lightweight per-token uncertainty head (Eq. (7)).
 *
 * u_out[b,i] = softplus(sum_c X[b,i,c] * w[c] + bias), softplus(z) =
 * log(1 + e^z), so u >= 0 as Eq. (7) requires.  The paper gives no
 * architecture beyond "lightweight"; a linear map to one scalar followed by
 * softplus is the form used here.  fp32 accumulation.
 *
 *   X      [B,N,C] bf16 (the final hidden states of the step), read only.
 *   w      [C] fp32; bias a host scalar.
 *   u_out  [B,N] fp32 out: the u that routes the next denoising step.
 *
 * Requires B, N >= 1, C a multiple of 8 with 8 <= C <= 16384.
 *
 * Widths that are a multiple of 256 up to 3072 (the DiT hidden sizes) run a
 * kernel that holds each lane's slice of w in registers; other widths stage
 * w in shared memory.  Both sum the C products in fp32, in an order fixed
 * by C, so a call is deterministic; the two orders differ only in rounding.
 */
HETA_API heta_status heta_uncertainty(const uint16_t *X, const float *w, float bias,
                             int B, int N, int C, float *u_out,
                             int32_t *status_dev, void *stream);

/*
 * heta_selftest_wait_timeout -- test hook (the paper has no counterpart):
 * runs the bounded-wait path every kernel of this library uses, on purpose.
 * One small kernel: warp 0 waits on a barrier that nothing completes until
 * limit_ns of wall time have passed, raises the CTA's abort flag and writes
 * HETA_ERR_TIMEOUT to *status_dev (atomic max); warp 1 waits on another such
 * barrier with a 5 s limit and must be released by the flag.  If
 * elapsed_ns_dev is not NULL it receives the kernel's wall time (device
 * uint64).  Nothing faults and nothing is left in flight: the context stays
 * usable.  Requires 0 < limit_ns <= 10 s and status_dev (device int32).
 */
HETA_API heta_status heta_selftest_wait_timeout(uint64_t limit_ns, int32_t *status_dev,
                                                unsigned long long *elapsed_ns_dev,
                                                void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HETA_H */
