// attention_tc.cu -- routed heterogeneous attention on the sm_100a tensor cores.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion": Eq. (2) dense attention for the routed (most uncertain) query
// rows, Eq. (3) attention over a clamped 3D (t,h,w) window for every other
// row, merged row by row as in Eq. (13); Eq. (14) is the cost model.
//
// One kernel template, two modes:
//   DENSE: a CTA owns two 128-row query tiles gathered through dense_idx and
//          streams all N keys of its (b,h) in 128-key K/V tiles.
//   LOCAL: a CTA owns two 2x8x8 query boxes of the latent grid; each box
//          streams the K/V sub-tiles (1x8x16 keys each) that cover the union
//          of its rows' windows, with a per-element window mask.  Rows whose
//          token is dense are computed but not stored.
// Both modes: K/V tiles arrive by TMA (128-byte swizzle) into a shared-memory
// ring; one thread issues tcgen05.mma with fp32 accumulators in TMEM
// (S = Q K^T per tile, O += P V with P read back from TMEM); two softmax
// warpgroups (one thread per query row) ping-pong on the two tiles with an
// online softmax in the log2 domain.  The O rescale is skipped unless the
// running row maximum grows by more than 2^8.  Epilogue: O / l in bf16,
// stored straight to the row's place in out (the Eq. (13) scatter).
//
// Every mbarrier wait is bounded; on expiry the kernel raises
// HETA_ERR_TIMEOUT in status, unwinds, drains its copies and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "heta_internal.cuh"
#include "ptx_sm100.cuh"

namespace heta {
namespace {

using namespace ptx;

constexpr int kThreads = 384;          // 12 warps
constexpr int kTileRows = 128;         // query rows per tile (MMA M)
constexpr int kTileKeys = 128;         // keys per K/V tile (MMA N of S)
constexpr int kRingBytes = 128 * 1024; // K/V ring
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;   // rescale O only when the max grows > 2^8

// query box (LOCAL) and key sub-tile
constexpr int kBoxT = 2, kBoxH = 8, kBoxW = 8;
constexpr int kKvH = 8, kKvW = 16;

enum { DENSE = 0, LOCAL = 1 };

// warp roles
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpFlags = 2, kWarpSoftmax0 = 4;

struct Params {
    const uint16_t *Q;
    uint16_t *out;
    const int32_t *dense_idx;
    int32_t *status;
    int B, H, N, k;
    int Tg, Hg, Wg, wt, wh, ww;
    float scale_log2;
    int tiles;   // DENSE: query tiles per (b,h); LOCAL: boxes per (b,h)
    int n_kv;    // K/V tiles each query tile streams
    int nbh, nbw;            // LOCAL: boxes along h and w
    int nkt, nkh, nkw;       // LOCAL: K/V sub-tiles along t, h, w
};

template <int D>
struct Cfg {
    static constexpr int kSub = D / 64;                     // 128-byte column blocks
    static constexpr int kTileBytes = kTileRows * D * 2;    // one Q/K/V tile
    static constexpr int kStages = kRingBytes / kTileBytes;
    static constexpr int kQBytes = 2 * kTileBytes;
    static constexpr int kSmem = kQBytes + kRingBytes + 1024;  // + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
};

__device__ __forceinline__ int wstart(int p, int extent, int w)
{
    return min(max(p - w / 2, 0), extent - w);
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Geometry of one LOCAL query box and the origin of its K/V cover.
struct Box {
    int t0, h0, w0;       // box origin
    int tlo, hlo, wlo;    // origin of the K/V cover
    bool active;
};

__device__ __forceinline__ Box local_box(const Params &p, int box)
{
    Box x;
    x.active = box < p.tiles;
    const int bb = x.active ? box : 0;
    const int bw = bb % p.nbw, bh = (bb / p.nbw) % p.nbh, bt = bb / (p.nbw * p.nbh);
    x.t0 = bt * kBoxT;
    x.h0 = bh * kBoxH;
    x.w0 = bw * kBoxW;
    x.tlo = min(wstart(x.t0, p.Tg, p.wt), p.Tg - p.nkt);
    x.hlo = min(wstart(x.h0, p.Hg, p.wh), max(0, p.Hg - p.nkh * kKvH));
    x.wlo = min(wstart(x.w0, p.Wg, p.ww), max(0, p.Wg - p.nkw * kKvW));
    return x;
}

struct Shared {
    uint64_t kv_full[16], kv_empty[16];
    uint64_t q_full[2], s_full[2], p_full[2], o_done[2], flags_ready, drain;
    uint32_t tmem_base;
    int abort;
    uint8_t no_store[2][kTileRows];  // LOCAL: row holds a dense token
};

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const Params p)
{
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    __shared__ Shared sh;

    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    uint8_t *q_smem = smem;                      // [2][kSub][128 rows][128 B]
    uint8_t *ring = smem + C::kQBytes;           // [kStages][kSub][128 rows][128 B]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int64_t bh = (int64_t)b * p.H + h;
    const int n = p.n_kv;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_addr(&sh.kv_full[s]), 1);
            mbar_init(smem_addr(&sh.kv_empty[s]), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(smem_addr(&sh.q_full[t]), kTileRows);
            mbar_init(smem_addr(&sh.s_full[t]), 1);
            mbar_init(smem_addr(&sh.p_full[t]), kTileRows);
            mbar_init(smem_addr(&sh.o_done[t]), 1);
        }
        mbar_init(smem_addr(&sh.flags_ready), 1);
        mbar_init(smem_addr(&sh.drain), 1);
        sh.abort = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_addr(&sh.tmem_base), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const volatile int *abort = &sh.abort;

    auto fail = [&]() {
        if (atomicExch(&sh.abort, 1) == 0) raise_status(p.status, HETA_ERR_TIMEOUT);
    };

    // the two query tiles of this CTA
    const int tile0 = 2 * pair, tile1 = 2 * pair + 1;

    if (warp == kWarpTma) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            Box bx[2];
            if (MODE == LOCAL) {
                bx[0] = local_box(p, tile0);
                bx[1] = local_box(p, tile1);
            }
            int issued = 0;
            bool ok = true;
            // one element of the tile sequence the MMA thread consumes in order
            auto load = [&](bool is_v, int slot, int j) {
                if (!ok) return;
                const int s = issued;
                const int stage = s % C::kStages;
                const uint32_t use = (uint32_t)(s / C::kStages);
                if (!mbar_wait(smem_addr(&sh.kv_empty[stage]), (use & 1u) ^ 1u, abort,
                               kWaitLimitNs)) {
                    ok = false;
                    return;
                }
                const uint32_t full = smem_addr(&sh.kv_full[stage]);
                mbar_arrive_expect_tx(full, C::kTileBytes);
                const uint32_t dst = smem_addr(ring + (size_t)stage * C::kTileBytes);
                const CUtensorMap *m = is_v ? &tmV : &tmK;
                for (int c = 0; c < C::kSub; ++c) {
                    if (MODE == DENSE) {
                        tma_load_3d(dst + c * 16384, m, full, 64 * c, j * kTileKeys, (int)bh);
                    } else {
                        const Box &x = bx[slot];
                        const int jt = j / (p.nkh * p.nkw), jh = (j / p.nkw) % p.nkh,
                                  jw = j % p.nkw;
                        tma_load_5d(dst + c * 16384, m, full, 64 * c, x.wlo + jw * kKvW,
                                    x.hlo + jh * kKvH, x.tlo + jt, (int)bh);
                    }
                }
                ++issued;
            };
            if (MODE == DENSE) {
                // K0, then per j: V_j, K_{j+1}
                load(false, 0, 0);
                for (int j = 0; j < n; ++j) {
                    load(true, 0, j);
                    if (j + 1 < n) load(false, 0, j + 1);
                }
            } else {
                // K0_0, K1_0, then per j: V0_j, K0_{j+1}, V1_j, K1_{j+1}
                load(false, 0, 0);
                load(false, 1, 0);
                for (int j = 0; j < n; ++j) {
                    load(true, 0, j);
                    if (j + 1 < n) load(false, 0, j + 1);
                    load(true, 1, j);
                    if (j + 1 < n) load(false, 1, j + 1);
                }
            }
            if (!ok) fail();
            // drain: every issued copy has landed before the CTA may exit
            for (int s = max(0, issued - C::kStages); s < issued; ++s) {
                const int stage = s % C::kStages;
                const uint32_t use = (uint32_t)(s / C::kStages);
                mbar_wait(smem_addr(&sh.kv_full[stage]), use & 1u, abort, kWaitLimitNs);
            }
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(128, kTileKeys, false);
            const uint32_t id_o = idesc_bf16(128, D, true);
            const uint32_t q_addr[2] = {smem_addr(q_smem), smem_addr(q_smem + C::kTileBytes)};
            const uint32_t colS[2] = {C::kColS0, C::kColS1};
            const uint32_t colO[2] = {C::kColO0, C::kColO1};
            int s = 0;  // ring sequence position
            bool ok = true;
            auto wait_full = [&](int seq) -> uint32_t {
                const int stage = seq % C::kStages;
                if (!mbar_wait(smem_addr(&sh.kv_full[stage]), (uint32_t)(seq / C::kStages) & 1u,
                               abort, kWaitLimitNs)) {
                    ok = false;
                    return 0;
                }
                tc_fence_after();
                return smem_addr(ring + (size_t)stage * C::kTileBytes);
            };
            auto release = [&](int seq) { mma_commit(smem_addr(&sh.kv_empty[seq % C::kStages])); };
            // S_t = Q_t K^T : M=128, N=128 keys, K=D (both operands K-major)
            auto issue_s = [&](int t, uint32_t k_addr) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(tmem + colS[t], smem_desc_sw128(q_addr[t] + off, 16, 1024),
                           smem_desc_sw128(k_addr + off, 16, 1024), id_s, kk > 0);
                }
            };
            // O_t += P_t V : M=128, N=D, K=128 keys; P from TMEM, V MN-major
            auto issue_pv = [&](int t, uint32_t v_addr, bool first) {
#pragma unroll
                for (int kk = 0; kk < kTileKeys / 16; ++kk) {
                    mma_ts(tmem + colO[t], tmem + colS[t] + kk * 8,
                           smem_desc_sw128(v_addr + kk * 2048, 16384, 1024), id_o,
                           (first && kk == 0) ? 0u : 1u);
                }
            };
            for (int t = 0; t < 2 && ok; ++t) {
                if (!mbar_wait(smem_addr(&sh.q_full[t]), 0, abort, kWaitLimitNs)) ok = false;
            }
            tc_fence_after();
            if (ok) {
                if (MODE == DENSE) {
                    const uint32_t k0 = wait_full(s);
                    if (ok) {
                        issue_s(0, k0);
                        mma_commit(smem_addr(&sh.s_full[0]));
                        issue_s(1, k0);
                        mma_commit(smem_addr(&sh.s_full[1]));
                        release(s);
                        ++s;
                    }
                } else {
                    for (int t = 0; t < 2 && ok; ++t) {
                        const uint32_t kt = wait_full(s);
                        if (!ok) break;
                        issue_s(t, kt);
                        mma_commit(smem_addr(&sh.s_full[t]));
                        release(s);
                        ++s;
                    }
                }
            }
            for (int j = 0; j < n && ok; ++j) {
                const bool last = j + 1 == n;
                uint32_t v_addr = 0, kn_addr = 0;
                int v_seq = 0, kn_seq = 0;
                for (int t = 0; t < 2 && ok; ++t) {
                    // V tile for this slot
                    if (MODE == DENSE) {
                        if (t == 0) {
                            v_seq = s++;
                            v_addr = wait_full(v_seq);
                            if (!ok) break;
                        }
                    } else {
                        v_seq = s++;
                        v_addr = wait_full(v_seq);
                        if (!ok) break;
                    }
                    if (!mbar_wait(smem_addr(&sh.p_full[t]), (uint32_t)j & 1u, abort,
                                   kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(t, v_addr, j == 0);
                    if (MODE == LOCAL) release(v_seq);
                    if (MODE == DENSE && t == 1) release(v_seq);
                    if (last) {
                        mma_commit(smem_addr(&sh.o_done[t]));
                        continue;
                    }
                    // next S for this slot
                    if (MODE == DENSE) {
                        if (t == 0) {
                            kn_seq = s++;
                            kn_addr = wait_full(kn_seq);
                            if (!ok) break;
                        }
                    } else {
                        kn_seq = s++;
                        kn_addr = wait_full(kn_seq);
                        if (!ok) break;
                    }
                    issue_s(t, kn_addr);
                    mma_commit(smem_addr(&sh.s_full[t]));
                    if (MODE == LOCAL || t == 1) release(kn_seq);
                }
            }
            if (!ok) fail();
            // drain every MMA this thread issued before TMEM can be freed
            mma_commit(smem_addr(&sh.drain));
            mbar_wait(smem_addr(&sh.drain), 0, abort, kWaitLimitNs);
        }
    } else if (warp == kWarpFlags) {
        // ------------------------------------------------- LOCAL: dense rows
        if (MODE == LOCAL) {
            for (int t = 0; t < 2; ++t)
                for (int r = lane; r < kTileRows; r += 32) sh.no_store[t][r] = 0;
            __syncwarp();
            const int32_t *dl = p.dense_idx + (int64_t)b * p.k;
            const int HW = p.Hg * p.Wg;
            for (int t = 0; t < 2 && p.k > 0; ++t) {
                const Box x = local_box(p, t == 0 ? tile0 : tile1);
                if (!x.active) continue;
                const int lo_tok = (x.t0 * p.Hg + x.h0) * p.Wg + x.w0;
                const int hi_tok = (min(x.t0 + kBoxT, p.Tg) - 1) * HW +
                                   (min(x.h0 + kBoxH, p.Hg) - 1) * p.Wg +
                                   min(x.w0 + kBoxW, p.Wg) - 1;
                // first position with dense_idx >= lo_tok (32-ary search)
                int lo = 0, hi = p.k;
                while (hi - lo > 32) {
                    const int step = (hi - lo + 31) / 32;
                    const int pos = lo + lane * step;
                    const bool below = pos < hi && __ldg(dl + pos) < lo_tok;
                    const unsigned m = __ballot_sync(0xffffffffu, below);
                    const int c = __popc(m);  // probes below lo_tok form a prefix
                    const int nlo = c > 0 ? lo + (c - 1) * step + 1 : lo;
                    const int nhi = min(hi, lo + c * step + (c < 32 ? 1 : 0));
                    lo = nlo;
                    hi = max(nlo, nhi);
                }
                {
                    const int pos = lo + lane;
                    const bool below = pos < hi && __ldg(dl + pos) < lo_tok;
                    lo += __popc(__ballot_sync(0xffffffffu, below));
                }
                for (int base = lo;; base += 32) {
                    const int pos = base + lane;
                    int v = pos < p.k ? __ldg(dl + pos) : INT32_MAX;
                    if (v <= hi_tok) {
                        const int tt = v / HW - x.t0, hh = (v / p.Wg) % p.Hg - x.h0,
                                  ww = v % p.Wg - x.w0;
                        if (tt >= 0 && tt < kBoxT && hh >= 0 && hh < kBoxH && ww >= 0 &&
                            ww < kBoxW)
                            sh.no_store[t][(tt * kBoxH + hh) * kBoxW + ww] = 1;
                    }
                    if (__ballot_sync(0xffffffffu, v <= hi_tok) != 0xffffffffu) break;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&sh.flags_ready));
        }
    } else if (warp >= kWarpSoftmax0) {
        // ------------------------------------------------------- softmax WGs
        const int t = (warp - kWarpSoftmax0) >> 2;      // which query tile
        const int r = threadIdx.x - (kWarpSoftmax0 + 4 * t) * 32;  // row in tile
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + (t == 0 ? C::kColS0 : C::kColS1);
        const uint32_t tO = tmem + lane_base + (t == 0 ? C::kColO0 : C::kColO1);
        const int tile = t == 0 ? tile0 : tile1;

        // ---- row identity and Q row load (into the K-major SW128 layout)
        bool row_valid = false;
        int token = 0;
        int qs_t = 0, qs_h = 0, qs_w = 0;  // LOCAL: window starts of this row
        Box bx;
        if (MODE == DENSE) {
            const int q = tile * kTileRows + r;
            row_valid = tile < p.tiles && q < p.k;
            if (row_valid) token = __ldg(p.dense_idx + (int64_t)b * p.k + q);
        } else {
            bx = local_box(p, tile);
            const int qt = bx.t0 + r / (kBoxH * kBoxW), qh = bx.h0 + (r / kBoxW) % kBoxH,
                      qw = bx.w0 + r % kBoxW;
            row_valid = bx.active && qt < p.Tg && qh < p.Hg && qw < p.Wg;
            token = (qt * p.Hg + qh) * p.Wg + qw;
            qs_t = wstart(min(qt, p.Tg - 1), p.Tg, p.wt);
            qs_h = wstart(min(qh, p.Hg - 1), p.Hg, p.wh);
            qs_w = wstart(min(qw, p.Wg - 1), p.Wg, p.ww);
        }
        {
            uint8_t *qt_smem = q_smem + t * C::kTileBytes;
            const uint4 *src = reinterpret_cast<const uint4 *>(p.Q + (bh * p.N + token) * D);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 v = row_valid ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
                const int sub = c >> 3, chunk = c & 7;
                *reinterpret_cast<uint4 *>(qt_smem + sub * 16384 + r * 128 +
                                           ((chunk ^ (r & 7)) << 4)) = v;
            }
            fence_proxy_async_smem();
            mbar_arrive(smem_addr(&sh.q_full[t]));
        }

        float m_run = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            if (!mbar_wait(smem_addr(&sh.s_full[t]), (uint32_t)j & 1u, abort, kWaitLimitNs)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[kTileKeys];
            {
                uint32_t raw[32];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    tmem_ld32(tS + 32 * c4, raw);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) sv[32 * c4 + i] = __uint_as_float(raw[i]);
                }
            }
            // ---- mask
            if (MODE == DENSE) {
                const int valid = p.N - j * kTileKeys;
                if (valid < kTileKeys) {
#pragma unroll
                    for (int c = 0; c < kTileKeys; ++c)
                        if (c >= valid) sv[c] = -INFINITY;
                }
            } else {
                const int jt = j / (p.nkh * p.nkw), jh = (j / p.nkw) % p.nkh, jw = j % p.nkw;
                const int kt = bx.tlo + jt, kh0 = bx.hlo + jh * kKvH, kw0 = bx.wlo + jw * kKvW;
                const bool t_ok = (unsigned)(kt - qs_t) < (unsigned)p.wt;
                const int wl = qs_w - kw0, whi = wl + p.ww;
                const uint32_t wbits =
                    (whi <= 0 || wl >= kKvW)
                        ? 0u
                        : (((1u << min(whi, kKvW)) - 1u) & ~((1u << max(wl, 0)) - 1u));
#pragma unroll
                for (int g = 0; g < kKvH; ++g) {
                    const bool h_ok = t_ok && (unsigned)(kh0 + g - qs_h) < (unsigned)p.wh;
                    const uint32_t bits = h_ok ? wbits : 0u;
#pragma unroll
                    for (int c = 0; c < kKvW; ++c)
                        if (!((bits >> c) & 1u)) sv[g * kKvW + c] = -INFINITY;
                }
            }
            // ---- online softmax (log2 domain)
            float mt = sv[0];
#pragma unroll
            for (int c = 1; c < kTileKeys; ++c) mt = fmaxf(mt, sv[c]);
            const float m_cand = fmaxf(m_run, mt * p.scale_log2);
            const bool need = m_cand > m_run + kRescaleLog2;
            float alpha = 1.f;
            if (need) {
                alpha = ex2(m_run - m_cand);
                l *= alpha;
                m_run = m_cand;
            }
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                // O holds P V of tiles < j and no MMA writes it now
#pragma unroll
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(tO + 32 * c4, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tO + 32 * c4, o);
                }
                tmem_wait_st();
            }
            const float m_use = m_run == -INFINITY ? 0.f : m_run;
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < kTileKeys; ++c) {
                sv[c] = ex2(fmaf(sv[c], p.scale_log2, -m_use));
                rs += sv[c];
            }
            l += rs;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) pk[i] = pack_bf16(sv[64 * h2 + 2 * i], sv[64 * h2 + 2 * i + 1]);
                tmem_st32(tS + 32 * h2, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_addr(&sh.p_full[t]));
        }
        // ---- epilogue: out row = O / l
        if (ok && !mbar_wait(smem_addr(&sh.o_done[t]), 0, abort, kWaitLimitNs)) ok = false;
        bool store = ok && row_valid;
        if (MODE == LOCAL && ok) {
            if (!mbar_wait(smem_addr(&sh.flags_ready), 0, abort, kWaitLimitNs)) ok = false;
            store = ok && row_valid && !sh.no_store[t][r];
        }
        if (!ok) fail();
        tc_fence_after();
        {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + (bh * p.N + token) * D);
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * c4, o);
                tmem_wait_ld();
                if (store) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(o[8 * v + 0]) * inv,
                                        __uint_as_float(o[8 * v + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(o[8 * v + 2]) * inv,
                                        __uint_as_float(o[8 * v + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(o[8 * v + 4]) * inv,
                                        __uint_as_float(o[8 * v + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(o[8 * v + 6]) * inv,
                                        __uint_as_float(o[8 * v + 7]) * inv);
                        dst[c4 * 4 + v] = w;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// K or V viewed as [B*H][N][D] bf16; box = 128 keys x 64 channels.
bool make_map_dense(CUtensorMap *m, const void *base, int BH, int N, int D)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kTileKeys, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K or V viewed as [B*H][T][H][W][D]; box = 1 x 8 x 16 keys x 64 channels.
bool make_map_local(CUtensorMap *m, const void *base, int BH, int T, int Hg, int Wg, int D)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)Wg, (cuuint64_t)Hg, (cuuint64_t)T,
                          (cuuint64_t)BH};
    cuuint64_t strides[4] = {(cuuint64_t)D * 2, (cuuint64_t)Wg * D * 2,
                             (cuuint64_t)Hg * Wg * D * 2, (cuuint64_t)T * Hg * Wg * D * 2};
    cuuint32_t box[5] = {64, (cuuint32_t)kKvW, (cuuint32_t)kKvH, 1, 1};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides,
              box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int MODE>
cudaError_t launch_mode(const AttnArgs &a, cudaStream_t s)
{
    using Cf = Cfg<D>;
    Params p;
    p.Q = a.Q;
    p.out = a.out;
    p.dense_idx = a.dense_idx;
    p.status = a.status;
    p.B = a.B; p.H = a.H; p.N = a.N; p.k = a.k;
    p.Tg = a.Tg; p.Hg = a.Hg; p.Wg = a.Wg; p.wt = a.wt; p.wh = a.wh; p.ww = a.ww;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    CUtensorMap mk, mv;
    if (MODE == DENSE) {
        p.tiles = (a.k + kTileRows - 1) / kTileRows;
        p.n_kv = (a.N + kTileKeys - 1) / kTileKeys;
        p.nbh = p.nbw = p.nkt = p.nkh = p.nkw = 1;
        if (!make_map_dense(&mk, a.K, a.B * a.H, a.N, D) ||
            !make_map_dense(&mv, a.V, a.B * a.H, a.N, D))
            return cudaErrorInvalidValue;
    } else {
        const int nbt = (a.Tg + kBoxT - 1) / kBoxT;
        p.nbh = (a.Hg + kBoxH - 1) / kBoxH;
        p.nbw = (a.Wg + kBoxW - 1) / kBoxW;
        p.tiles = nbt * p.nbh * p.nbw;
        p.nkt = min(kBoxT + a.wt - 1, a.Tg);
        p.nkh = (min(kBoxH + a.wh - 1, a.Hg) + kKvH - 1) / kKvH;
        p.nkw = (min(kBoxW + a.ww - 1, a.Wg) + kKvW - 1) / kKvW;
        p.n_kv = p.nkt * p.nkh * p.nkw;
        if (!make_map_local(&mk, a.K, a.B * a.H, a.Tg, a.Hg, a.Wg, D) ||
            !make_map_local(&mv, a.V, a.B * a.H, a.Tg, a.Hg, a.Wg, D))
            return cudaErrorInvalidValue;
    }
    auto kern = attn_tc_kernel<D, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cf::kSmem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.tiles + 1) / 2, a.H, a.B);
    kern<<<grid, kThreads, Cf::kSmem, s>>>(mk, mv, p);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttnArgs &a, cudaStream_t s)
{
    if (a.k < a.N) {
        cudaError_t e = launch_mode<D, LOCAL>(a, s);
        if (e != cudaSuccess) return e;
    }
    if (a.k > 0) return launch_mode<D, DENSE>(a, s);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t s)
{
    return a.d == 64 ? launch_d<64>(a, s) : launch_d<128>(a, s);
}

}  // namespace heta
