// attention_tc.cu -- routed heterogeneous attention on the sm_100a tensor cores.
//
// "Where Compute Matters: Heterogeneous Attention for Efficient Video
// Diffusion": Eq. (2) dense attention for the routed (most uncertain) query
// rows, Eq. (3) attention over a clamped 3D (t,h,w) window for every other
// row, merged row by row as in Eq. (13); Eq. (14) is the cost model.
//
// One persistent kernel runs both kinds of work item, handed out in order by
// an atomic counter (dense items first: they are the long ones):
//   DENSE item: two 128-row query tiles of one (b,h), gathered through
//               dense_idx, against one contiguous range of 128-key K/V tiles
//               (all N keys, or half of them when the host splits the key
//               range to balance the SMs; the second half to finish merges
//               the other's partial result -- no CTA ever waits on another).
//   LOCAL item: two 128-token query boxes of the latent grid (2x8x8 for
//               small windows; the planner picks the shape whose K/V covers
//               hold the fewest keys, e.g. 8x4x4 for an 11^3 window); each
//               box streams the 1x8x16-key K/V sub-tiles that cover its rows'
//               windows, with a per-element window mask.  Rows whose token
//               is dense are computed but not stored.
// Per CTA (one per SM): a TMA producer warp fills a shared-memory ring of K/V
// tiles (128-byte swizzle) and loads LOCAL query boxes; one thread issues
// tcgen05.mma with fp32 accumulators in TMEM (S = Q K^T, O += P V with P read
// back from TMEM); two softmax warpgroups (one thread per query row) ping-pong
// on the two tiles with an online softmax in the log2 domain, rescaling O
// only when a row maximum grows by more than 2^8; a flags warp finds the
// dense tokens inside LOCAL boxes.  Epilogue: O / l in bf16, stored straight
// to the row's place in out (the Eq. (13) scatter).
//
// Every wait is bounded; on expiry the kernel raises HETA_ERR_TIMEOUT in
// status, unwinds, drains its copies and MMAs and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "heta_internal.cuh"
#include "ptx_sm100.cuh"

namespace heta {
namespace {

using namespace ptx;

constexpr int kThreads = 384;           // 12 warps: one control and two softmax warpgroups
constexpr int kTileRows = 128;          // query rows per tile (MMA M)
constexpr int kTileKeys = 128;          // keys per K/V tile (MMA N of S)
constexpr int kRingBytes = 128 * 1024;  // K/V ring
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;    // rescale O only when the max grows > 2^8
constexpr int kQueue = 4;               // work-item queue depth
constexpr int kMaxSplit = 2;            // key ranges a DENSE pair is cut into at most

// query box (LOCAL) and key sub-tile
// (the query box is planned per call among shapes of 128 tokens, see
// plan_attention; the key sub-tile is fixed)
constexpr int kKvH = 8, kKvW = 16;

enum { DENSE = 0, LOCAL = 1 };

// warp roles
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpFlags = 2, kWarpSoftmax0 = 4;
// consumers of the item queue: MMA thread, 256 softmax threads, flags warp
constexpr uint32_t kItemConsumers = 1 + 256 + 32;

struct Params {
    const uint16_t *Q;
    uint16_t *out;
    int out32;        // out is 32-byte aligned (so is every row): 32-byte stores
    const int32_t *dense_idx;  // [B][k]
    const int32_t *k_dev;      // [B] dense rows per sample (<= k), or null: all k
    int32_t *status;
    int B, H, N, k;
    int Tg, Hg, Wg, wt, wh, ww;
    float scale_log2;
    // DENSE items
    int tiles_d, pairs_d, pairs_full, nsplit, n_kv_d, kv_per_split, n_dense_items;
    int max_split;    // 1: no pair is cut into key ranges (the scratch has no room)
    int sms;          // SM count the waves of dense work are planned for
    // LOCAL items
    int box_t, box_h, box_w;
    int tiles_l, pairs_l, nbh, nbw, nkt, nkh, nkw, n_kv_l, n_local_items;
    int total_items;
    // scratch
    int *counter;     // next work item
    int *fix_count;   // [B*H*pairs_d][2] split arrivals
    float *part_o;    // [B*H*pairs_d][nsplit][2][128][D]
    float2 *part_ml;  // [B*H*pairs_d][nsplit][2][128] (m, l)
};

template <int D>
struct Cfg {
    static constexpr int kSub = D / 64;                   // 128-byte column blocks
    static constexpr int kTileBytes = kTileRows * D * 2;  // one Q/K/V tile
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

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Two fp32 lanes in one 64-bit register (low = first), for the packed f32x2 ops.
__device__ __forceinline__ uint64_t f2(uint32_t lo_bits, uint32_t hi_bits)
{
    return ((uint64_t)hi_bits << 32) | lo_bits;
}

__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ void named_bar(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// One work item, decoded from its index.
struct Item {
    int mode;        // DENSE or LOCAL
    int bh;          // b*H + h
    int b;
    int tile[2];     // query tile (DENSE) / box (LOCAL) of each slot
    int kv_lo, n;    // K/V tiles [kv_lo, kv_lo + n)
    int split;       // DENSE: which key range
    int nsplit;      // DENSE: key ranges of this pair (1: the whole range)
    int pair_id;     // DENSE, nsplit > 1: index among the split pairs (for the merge)
    int kb;          // dense rows of sample b (n == 0: a DENSE pair past them, skipped)
};

// How the DENSE work is cut, worked out on the device from the real dense
// rows (with per-sample counts only the device knows them): whole waves of
// query-tile pairs (a multiple of the SM count) unsplit, the pairs of the last,
// partial wave in nsplit key ranges.  Item ids [0, n_dense) are DENSE work,
// the LOCAL items follow.
struct DPlan {
    int pairs_total, pairs_full, nsplit, kv_per_split, n_dense;
};

// The same rule as plan_attention's on the host.
__device__ __forceinline__ DPlan dense_plan(int pairs_total, int n_kv, int max_split, int sms)
{
    DPlan d;
    d.pairs_total = pairs_total;
    d.pairs_full = pairs_total;
    d.nsplit = 1;
    if (pairs_total > 0 && n_kv >= 16) {
        d.pairs_full = pairs_total / sms * sms;
        const int rest = pairs_total - d.pairs_full;
        d.nsplit = rest > 0 ? min(max_split, n_kv / 8) : 1;
        if (d.pairs_full > 0 && rest > sms / 2) d.nsplit = 1;
        if (d.nsplit < 2) {  // a last wave more than half full runs whole
            d.nsplit = 1;
            d.pairs_full = pairs_total;
        }
    }
    d.kv_per_split = (n_kv + d.nsplit - 1) / d.nsplit;
    d.n_dense = d.pairs_full + (pairs_total - d.pairs_full) * d.nsplit;
    return d;
}

// cpref (per-sample counts only): sample b's query-tile pairs are the dense
// pairs [H * cpref[b], H * cpref[b + 1]), ordered by head, then pair.
__device__ __forceinline__ Item decode(const Params &p, const DPlan &dp, const int *cpref, int id)
{
    Item it;
    if (id < dp.n_dense) {
        // the first pairs_full pairs whole, then each remaining pair in
        // nsplit key ranges
        int pg, kv_per;
        if (id < dp.pairs_full) {
            pg = id;
            it.split = 0;
            it.nsplit = 1;
            kv_per = p.n_kv_d;
        } else {
            const int r = id - dp.pairs_full;
            pg = dp.pairs_full + r / dp.nsplit;
            it.split = r % dp.nsplit;
            it.nsplit = dp.nsplit;
            kv_per = dp.kv_per_split;
        }
        it.mode = DENSE;
        int pair;
        if (p.k_dev) {
            int lo = 0, hi = p.B;  // the last b with H * cpref[b] <= pg
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (p.H * cpref[mid] <= pg) lo = mid;
                else hi = mid;
            }
            const int r = pg - p.H * cpref[lo];
            const int pairs_b = max(cpref[lo + 1] - cpref[lo], 1);
            it.bh = lo * p.H + r / pairs_b;
            pair = r % pairs_b;
        } else {
            it.bh = pg / p.pairs_d;
            pair = pg % p.pairs_d;
        }
        it.pair_id = pg - dp.pairs_full;
        it.tile[0] = 2 * pair;
        it.tile[1] = 2 * pair + 1;
        it.kv_lo = it.split * kv_per;
        it.n = min(p.n_kv_d, it.kv_lo + kv_per) - it.kv_lo;
    } else {
        const int id2 = id - dp.n_dense;
        it.mode = LOCAL;
        it.bh = id2 / p.pairs_l;
        const int pair = id2 % p.pairs_l;
        it.split = 0;
        it.nsplit = 1;
        it.pair_id = 0;
        it.tile[0] = 2 * pair;
        it.tile[1] = 2 * pair + 1;
        it.kv_lo = 0;
        it.n = p.n_kv_l;
    }
    it.b = it.bh / p.H;
    it.kb = p.k_dev ? min(max(__ldg(p.k_dev + it.b), 0), p.k) : p.k;
    if (it.mode == DENSE && it.tile[0] * kTileRows >= it.kb) it.n = 0;
    return it;
}

// Geometry of one LOCAL query box and the origin of its K/V cover.
struct Box {
    int t0, h0, w0;     // box origin
    int tlo, hlo, wlo;  // origin of the K/V cover
    bool active;
};

__device__ __forceinline__ Box local_box(const Params &p, int box)
{
    Box x;
    x.active = box < p.tiles_l;
    const int bb = x.active ? box : 0;
    const int bw = bb % p.nbw, bh = (bb / p.nbw) % p.nbh, bt = bb / (p.nbw * p.nbh);
    x.t0 = bt * p.box_t;
    x.h0 = bh * p.box_h;
    x.w0 = bw * p.box_w;
    x.tlo = min(wstart(x.t0, p.Tg, p.wt), p.Tg - p.nkt);
    x.hlo = min(wstart(x.h0, p.Hg, p.wh), max(0, p.Hg - p.nkh * kKvH));
    x.wlo = min(wstart(x.w0, p.Wg, p.ww), max(0, p.Wg - p.nkw * kKvW));
    return x;
}

// One 128-key S tile of one query row (this thread's TMEM lane): mask, online
// softmax update in the log2 domain, P = 2^(s*scale - m) in bf16 written over
// the S columns it replaces, and the O rescale when the row maximum grew by
// more than 2^8.  Reductions use 8 independent accumulators (one per group of
// 16 columns) so no long dependency chain serialises the thread.  Groups
// outside `active` (warp-uniform) are not read and get P = 0.
// Masks: kAll -- every column is a key of the row; kPrefix -- columns below
// `valid`; kWindow -- column c of group g when bit g of gmask is set and the
// column's entry in wbias2 is 0 (-inf marks a column outside the row's window).
// Masked scores become -inf in the max pass, so the exp pass needs no mask.
enum { kAll = 0, kPrefix = 1, kWindow = 2 };

template <int D, int MASK>
__device__ __forceinline__ void softmax_tile(uint32_t tS, uint32_t tO, bool o_live, int valid,
                                             const uint64_t (&wbias2)[kKvW / 2], uint32_t gmask,
                                             uint32_t active, float scale_log2, float &m_run,
                                             float &l)
{
    uint32_t sv[kTileKeys];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
        tmem_ld32(tS + 32 * c4, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * c4]));
    tmem_wait_ld();
    float mx[kKvH];
#pragma unroll
    for (int g = 0; g < kKvH; ++g) {
        mx[g] = -INFINITY;
        if (MASK != kWindow || (active & (1u << g))) {
            // kWindow: + 0 / -inf for the column, then + 0 / -inf for the group (row h)
            const uint32_t gb = ((gmask >> g) & 1u) ? 0u : 0xff800000u;
            const uint64_t gb2 = f2(gb, gb);
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
                float x0 = __uint_as_float(sv[16 * g + c]);
                float x1 = __uint_as_float(sv[16 * g + c + 1]);
                if (MASK == kPrefix) {
                    x0 = 16 * g + c < valid ? x0 : -INFINITY;
                    x1 = 16 * g + c + 1 < valid ? x1 : -INFINITY;
                }
                if (MASK == kWindow) {
                    const uint64_t x2 =
                        add_f32x2(add_f32x2(f2(__float_as_uint(x0), __float_as_uint(x1)),
                                            wbias2[c / 2]),
                                  gb2);
                    x0 = __uint_as_float((uint32_t)x2);
                    x1 = __uint_as_float((uint32_t)(x2 >> 32));
                }
                if (MASK != kAll) {
                    sv[16 * g + c] = __float_as_uint(x0);
                    sv[16 * g + c + 1] = __float_as_uint(x1);
                }
                mx[g] = max3(mx[g], x0, x1);
            }
        }
    }
    const float mt = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
    const float m_cand = fmaxf(m_run, mt * scale_log2);
    const bool need = m_cand > m_run + kRescaleLog2;
    float alpha = 1.f;
    if (need) {
        alpha = ex2(m_run - m_cand);
        l *= alpha;
        m_run = m_cand;
    }
    const float m_use = m_run == -INFINITY ? 0.f : m_run;
    // P in column pairs: x = s*scale - m as one packed fp32 FMA, 2^x of each,
    // the pair added to one of four packed fp32 sums, and the bf16 pair word
    // i <- columns 2i, 2i+1 written in place (sv[i] after sv[2i], sv[2i+1] are read)
    const uint64_t scale2 = f2(__float_as_uint(scale_log2), __float_as_uint(scale_log2));
    const uint64_t negm2 = f2(__float_as_uint(-m_use), __float_as_uint(-m_use));
    uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int g = 0; g < kKvH; ++g) {
        if (MASK != kWindow || (active & (1u << g))) {
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
                const uint64_t x2 = fma_f32x2(f2(sv[16 * g + c], sv[16 * g + c + 1]), scale2, negm2);
                const float e0 = ex2(__uint_as_float((uint32_t)x2));
                const float e1 = ex2(__uint_as_float((uint32_t)(x2 >> 32)));
                sum2[g & 3] = add_f32x2(sum2[g & 3], f2(__float_as_uint(e0), __float_as_uint(e1)));
                sv[8 * g + c / 2] = pack_bf16(e0, e1);
            }
        } else {
#pragma unroll
            for (int c = 0; c < 16; c += 2) sv[8 * g + c / 2] = 0u;
        }
    }
    l += ((__uint_as_float((uint32_t)sum2[0]) + __uint_as_float((uint32_t)(sum2[0] >> 32))) +
          (__uint_as_float((uint32_t)sum2[1]) + __uint_as_float((uint32_t)(sum2[1] >> 32)))) +
         ((__uint_as_float((uint32_t)sum2[2]) + __uint_as_float((uint32_t)(sum2[2] >> 32))) +
          (__uint_as_float((uint32_t)sum2[3]) + __uint_as_float((uint32_t)(sum2[3] >> 32))));
    tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
    tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
    tmem_wait_st();
    if (o_live && __any_sync(0xffffffffu, need)) {
        // O holds P V of the earlier tiles, and the next P V waits for this
        // thread's p_full arrival: rescale it to the new maximum
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * c4, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + 32 * c4, o);
        }
        tmem_wait_st();
    }
}

struct Shared {
    uint64_t kv_full[16], kv_empty[16];
    uint64_t item_full[kQueue], item_empty[kQueue];
    uint64_t q_full[2], q_empty[2], s_full[2], p_full[2], o_done[2], o_empty[2];
    uint64_t flags_full, flags_empty, drain;
    int item_q[kQueue];
    uint32_t tmem_base;
    int abort;
    int fix_old[2];
    uint8_t no_store[2][kTileRows];  // LOCAL: row holds a dense token
    DPlan dplan;                     // how the DENSE work is cut (see DPlan)
    int cpref[kMaxCountsSamples + 1];      // per-sample counts: pair prefix over samples
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmK3, const __grid_constant__ CUtensorMap tmV3,
               const __grid_constant__ CUtensorMap tmK5, const __grid_constant__ CUtensorMap tmV5,
               const __grid_constant__ CUtensorMap tmQ5, const Params p)
{
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    __shared__ Shared sh;

    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    uint8_t *q_smem = smem;             // [2][kSub][128 rows][128 B]
    uint8_t *ring = smem + C::kQBytes;  // [kStages][kSub][128 rows][128 B]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_addr(&sh.kv_full[s]), 1);
            mbar_init(smem_addr(&sh.kv_empty[s]), 1);
        }
        for (int q = 0; q < kQueue; ++q) {
            mbar_init(smem_addr(&sh.item_full[q]), 1);
            mbar_init(smem_addr(&sh.item_empty[q]), kItemConsumers);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(smem_addr(&sh.q_full[t]), 1);
            mbar_init(smem_addr(&sh.q_empty[t]), 1);
            mbar_init(smem_addr(&sh.s_full[t]), 1);
            mbar_init(smem_addr(&sh.p_full[t]), kTileRows / 32);  // one arrival per warp
            mbar_init(smem_addr(&sh.o_done[t]), 1);
            mbar_init(smem_addr(&sh.o_empty[t]), kTileRows / 32);
        }
        mbar_init(smem_addr(&sh.flags_full), 1);
        mbar_init(smem_addr(&sh.flags_empty), 2 * kTileRows);
        mbar_init(smem_addr(&sh.drain), 1);
        sh.abort = 0;
        int pairs_total = p.B * p.H * p.pairs_d;
        if (p.k_dev) {
            int acc = 0;
            for (int b = 0; b < p.B; ++b) {
                sh.cpref[b] = acc;
                const int kb = min(max(__ldg(p.k_dev + b), 0), p.k);
                acc += (kb + 2 * kTileRows - 1) / (2 * kTileRows);
            }
            sh.cpref[p.B] = acc;
            pairs_total = p.H * acc;
        }
        sh.dplan = dense_plan(pairs_total, p.n_kv_d, p.max_split, p.sms);
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
    const DPlan dplan = sh.dplan;
    const volatile int *abort = &sh.abort;

    auto fail = [&]() {
        if (atomicExch(&sh.abort, 1) == 0) raise_status(p.status, HETA_ERR_TIMEOUT);
    };
    auto wait = [&](uint64_t &bar, uint32_t parity) -> bool {
        return mbar_wait(smem_addr(&bar), parity, abort, kWaitLimitNs);
    };
    // reads queue entry qi (blocking); every consumer arrives on item_empty
    auto pop_item = [&](uint32_t qi, bool &ok) -> int {
        const int slot = qi % kQueue;
        if (!wait(sh.item_full[slot], (qi / kQueue) & 1u)) {
            ok = false;
            return -1;
        }
        const int id = *reinterpret_cast<volatile int *>(&sh.item_q[slot]);
        mbar_arrive(smem_addr(&sh.item_empty[slot]));
        return id;
    };

    // Registers: the control warpgroup gives up what the softmax warpgroups
    // need for a full S row (4 x 56 + 8 x 224 = 12 x 168 per thread lane).
    if (warp < kWarpSoftmax0) {
    setmaxnreg_dec<56>();
    if (warp == kWarpTma) {
        // ============================================================ producer
        if (lane == 0) {
            prefetch_tmap(&tmK3);
            prefetch_tmap(&tmV3);
            prefetch_tmap(&tmK5);
            prefetch_tmap(&tmV5);
            prefetch_tmap(&tmQ5);
            uint32_t issued = 0, qi = 0, items = 0;
            bool ok = true;
            // the next item id; -1 when none is left
            const int total_items = dplan.n_dense + p.n_local_items;
            auto grab = [&]() -> int {
                const int g = atomicAdd(p.counter, 1);
                return g < total_items ? g : -1;
            };
            int id = grab();
            while (ok) {
                const int next = id >= 0 ? grab() : -1;
                // publish the item
                {
                    const int slot = qi % kQueue;
                    if (!wait(sh.item_empty[slot], ((qi / kQueue) & 1u) ^ 1u)) { ok = false; break; }
                    sh.item_q[slot] = id;
                    mbar_arrive(smem_addr(&sh.item_full[slot]));
                    ++qi;
                }
                if (id < 0) break;
                const Item it = decode(p, dplan, sh.cpref, id);
                if (it.n == 0) {  // a DENSE pair past the sample's dense rows: every role skips it
                    id = next;
                    continue;
                }
                Box bx[2];
                if (it.mode == LOCAL) {
                    bx[0] = local_box(p, it.tile[0]);
                    bx[1] = local_box(p, it.tile[1]);
                }
                // the query buffers are free once the last S of the previous item is done
                for (int t = 0; t < 2 && ok; ++t) {
                    if (items > 0 && !wait(sh.q_empty[t], (items - 1) & 1u)) ok = false;
                    if (ok && it.mode == LOCAL) {
                        const uint32_t full = smem_addr(&sh.q_full[t]);
                        mbar_arrive_expect_tx(full, C::kTileBytes);
                        const uint32_t dst = smem_addr(q_smem + t * C::kTileBytes);
                        for (int c = 0; c < C::kSub; ++c)
                            tma_load_5d(dst + c * 16384, &tmQ5, full, 64 * c, bx[t].w0,
                                        bx[t].h0, bx[t].t0, it.bh);
                    }
                }
                // one element of the K/V tile sequence the MMA thread consumes in order
                auto load = [&](bool is_v, int slot, int j) {
                    if (!ok) return;
                    const uint32_t s = issued;
                    const int stage = s % C::kStages;
                    if (!wait(sh.kv_empty[stage], ((s / C::kStages) & 1u) ^ 1u)) {
                        ok = false;
                        return;
                    }
                    const uint32_t full = smem_addr(&sh.kv_full[stage]);
                    mbar_arrive_expect_tx(full, C::kTileBytes);
                    const uint32_t dst = smem_addr(ring + (size_t)stage * C::kTileBytes);
                    for (int c = 0; c < C::kSub; ++c) {
                        if (it.mode == DENSE) {
                            tma_load_3d(dst + c * 16384, is_v ? &tmV3 : &tmK3, full, 64 * c,
                                        (it.kv_lo + j) * kTileKeys, it.bh);
                        } else {
                            const Box &x = bx[slot];
                            const int jt = j / (p.nkh * p.nkw), jh = (j / p.nkw) % p.nkh,
                                      jw = j % p.nkw;
                            tma_load_5d(dst + c * 16384, is_v ? &tmV5 : &tmK5, full, 64 * c,
                                        x.wlo + jw * kKvW, x.hlo + jh * kKvH, x.tlo + jt, it.bh);
                        }
                    }
                    ++issued;
                };
                const int n = it.n;
                if (it.mode == DENSE) {
                    // K0, then per j: V_j, K_{j+1}   (both query tiles share them)
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
                ++items;
                id = next;
            }
            if (!ok) fail();
            // drain: every issued copy has landed before the CTA may exit
            for (uint32_t s = issued > (uint32_t)C::kStages ? issued - C::kStages : 0; s < issued; ++s)
                wait(sh.kv_full[s % C::kStages], (s / C::kStages) & 1u);
        }
    } else if (warp == kWarpMma) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(128, kTileKeys, false);
            const uint32_t id_o = idesc_bf16(128, D, true);
            const uint32_t q_base = smem_addr(q_smem);
            uint32_t s = 0, qi = 0, items = 0;
            bool ok = true;
            auto wait_full = [&](uint32_t seq) -> uint32_t {
                const int stage = seq % C::kStages;
                if (!wait(sh.kv_full[stage], (seq / C::kStages) & 1u)) {
                    ok = false;
                    return 0;
                }
                tc_fence_after();
                return smem_addr(ring + (size_t)stage * C::kTileBytes);
            };
            auto release = [&](uint32_t seq) { mma_commit(smem_addr(&sh.kv_empty[seq % C::kStages])); };
            auto issue_s = [&](int t, uint32_t k_addr) {
                const uint64_t qd = smem_desc_sw128(q_base + t * C::kTileBytes, 16, 1024);
                const uint64_t kd = smem_desc_sw128(k_addr, 16, 1024);
                if (D == 128)
                    mma_ss_k128<16384, 16384>(tmem + (t ? C::kColS1 : C::kColS0), qd, kd, id_s, 0u);
                else
                    mma_ss_k64(tmem + (t ? C::kColS1 : C::kColS0), qd, kd, id_s, 0u);
            };
            auto issue_pv = [&](int t, uint32_t v_addr, bool first) {
                mma_ts_k128<2048>(tmem + (t ? C::kColO1 : C::kColO0),
                                      tmem + (t ? C::kColS1 : C::kColS0),
                                      smem_desc_sw128(v_addr, 16384, 1024), id_o, first ? 0u : 1u);
            };
            uint32_t pc[2] = {0, 0};  // p_full phases consumed per slot
            while (ok) {
                const int id = pop_item(qi++, ok);
                if (!ok || id < 0) break;
                const Item it = decode(p, dplan, sh.cpref, id);
                const int n = it.n;
                if (n == 0) continue;
                const bool dense = it.mode == DENSE;
                for (int t = 0; t < 2 && ok; ++t)
                    if (!wait(sh.q_full[t], items & 1u)) ok = false;
                if (!ok) break;
                tc_fence_after();
                // first S of each slot
                if (dense) {
                    const uint32_t k0 = wait_full(s);
                    if (!ok) break;
                    issue_s(0, k0);
                    mma_commit(smem_addr(&sh.s_full[0]));
                    issue_s(1, k0);
                    mma_commit(smem_addr(&sh.s_full[1]));
                    release(s++);
                } else {
                    for (int t = 0; t < 2 && ok; ++t) {
                        const uint32_t kt = wait_full(s);
                        if (!ok) break;
                        issue_s(t, kt);
                        mma_commit(smem_addr(&sh.s_full[t]));
                        release(s++);
                    }
                    if (!ok) break;
                }
                if (n == 1) {
                    mma_commit(smem_addr(&sh.q_empty[0]));
                    mma_commit(smem_addr(&sh.q_empty[1]));
                }
                for (int j = 0; j < n && ok; ++j) {
                    const bool last = j + 1 == n;
                    uint32_t v_addr = 0, kn_addr = 0, v_seq = 0, kn_seq = 0;
                    for (int t = 0; t < 2 && ok; ++t) {
                        // the tiles this slot needs next are waited for first: they
                        // usually landed long ago, and the softmax is usually later
                        if (!dense || t == 0) {
                            v_seq = s++;
                            v_addr = wait_full(v_seq);
                            if (!ok) break;
                            if (!last) {
                                kn_seq = s++;
                                kn_addr = wait_full(kn_seq);
                                if (!ok) break;
                            }
                        }
                        if (!wait(sh.p_full[t], pc[t] & 1u)) { ok = false; break; }
                        ++pc[t];
                        tc_fence_after();
                        // the previous item's epilogue must have read O_t before it is overwritten
                        if (j == 0 && items > 0 && !wait(sh.o_empty[t], (items - 1) & 1u)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_pv(t, v_addr, j == 0);
                        if (last) {
                            mma_commit(smem_addr(&sh.o_done[t]));
                        } else {
                            issue_s(t, kn_addr);
                            mma_commit(smem_addr(&sh.s_full[t]));
                            if (j + 2 == n) mma_commit(smem_addr(&sh.q_empty[t]));
                        }
                        if (!dense || t == 1) {
                            release(v_seq);
                            if (!last) release(kn_seq);
                        }
                    }
                }
                ++items;
            }
            if (!ok) fail();
            // drain every MMA this thread issued before TMEM can be freed
            mma_commit(smem_addr(&sh.drain));
            wait(sh.drain, 0);
        }
    } else if (warp == kWarpFlags) {
        // ============================================ flags: dense rows of LOCAL boxes
        uint32_t qi = 0, lc = 0;
        bool ok = true;
        while (ok) {
            const int id = pop_item(qi++, ok);
            if (!ok || id < 0) break;
            const Item it = decode(p, dplan, sh.cpref, id);
            if (it.mode != LOCAL) continue;
            if (!wait(sh.flags_empty, (lc & 1u) ^ 1u)) { ok = false; break; }
            for (int t = 0; t < 2; ++t)
                for (int r = lane; r < kTileRows; r += 32) sh.no_store[t][r] = 0;
            __syncwarp();
            const int32_t *dl = p.dense_idx + (int64_t)it.b * p.k;
            const int HW = p.Hg * p.Wg;
            for (int t = 0; t < 2 && it.kb > 0; ++t) {
                const Box x = local_box(p, it.tile[t]);
                if (!x.active) continue;
                const int lo_tok = (x.t0 * p.Hg + x.h0) * p.Wg + x.w0;
                const int hi_tok = (min(x.t0 + p.box_t, p.Tg) - 1) * HW +
                                   (min(x.h0 + p.box_h, p.Hg) - 1) * p.Wg +
                                   min(x.w0 + p.box_w, p.Wg) - 1;
                // first position with dense_idx >= lo_tok (32-ary search)
                int lo = 0, hi = it.kb;
                while (hi - lo > 32) {
                    const int step = (hi - lo + 31) / 32;
                    const int pos = lo + lane * step;
                    const bool below = pos < hi && __ldg(dl + pos) < lo_tok;
                    const int c = __popc(__ballot_sync(0xffffffffu, below));
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
                    const int v = pos < it.kb ? __ldg(dl + pos) : INT32_MAX;
                    if (v <= hi_tok) {
                        const int tt = v / HW - x.t0, hh = (v / p.Wg) % p.Hg - x.h0,
                                  ww = v % p.Wg - x.w0;
                        if (tt >= 0 && tt < p.box_t && hh >= 0 && hh < p.box_h && ww >= 0 &&
                            ww < p.box_w)
                            sh.no_store[t][(tt * p.box_h + hh) * p.box_w + ww] = 1;
                    }
                    if (__ballot_sync(0xffffffffu, v <= hi_tok) != 0xffffffffu) break;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&sh.flags_full));
            ++lc;
        }
        if (!ok) fail();
    }
    } else {
        // ============================================================ softmax WGs
        setmaxnreg_inc<224>();
        // a warp reaches TMEM lanes 32*(warp%4) .. +31: that quarter of the tile's rows
        const int t = (warp - kWarpSoftmax0) >> 2;  // query tile slot
        const int r = (warp & 3) * 32 + lane;       // row in tile
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + (t == 0 ? C::kColS0 : C::kColS1);
        const uint32_t tO = tmem + lane_base + (t == 0 ? C::kColO0 : C::kColO1);
        uint8_t *qt_smem = q_smem + t * C::kTileBytes;
        uint32_t qi = 0, items = 0, sc = 0, lc = 0;
        bool ok = true;
        while (ok) {
            const int id = pop_item(qi++, ok);
            if (!ok || id < 0) break;
            const Item it = decode(p, dplan, sh.cpref, id);
            if (it.n == 0) continue;
            const bool dense = it.mode == DENSE;
            const int tile = it.tile[t];
            const int64_t row0 = (int64_t)it.bh * p.N;

            // ---- row identity; DENSE rows are gathered into Q_t here
            bool row_valid = false;
            int token = 0, qs_t = 0, qs_h = 0, qs_w = 0;
            Box bx;
            if (dense) {
                const int q = tile * kTileRows + r;
                row_valid = tile < p.tiles_d && q < it.kb;
                if (row_valid) {
                    // The dense set is a subset of the sample's N tokens, listed in
                    // increasing order (Eq. (12)-(13)).  An entry outside [0, N), or
                    // not above the one before it, is reported and its row is
                    // neither gathered nor stored, so no access leaves Q or out.
                    const int32_t *dl = p.dense_idx + (int64_t)it.b * p.k;
                    token = __ldg(dl + q);
                    const int prev = q > 0 ? __ldg(dl + q - 1) : -1;
                    if (token < 0 || token >= p.N || token <= prev) {
                        raise_status(p.status, HETA_ERR_INVALID_ARG);
                        row_valid = false;
                        token = 0;
                    }
                }
                const uint4 *src = reinterpret_cast<const uint4 *>(p.Q + (row0 + token) * D);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    const uint4 v = row_valid ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
                    const int sub = c >> 3, chunk = c & 7;
                    *reinterpret_cast<uint4 *>(qt_smem + sub * 16384 + r * 128 +
                                               ((chunk ^ (r & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();
                named_bar(1 + t, kTileRows);
                if (r == 0) mbar_arrive(smem_addr(&sh.q_full[t]));
            } else {
                bx = local_box(p, tile);
                const int qt = bx.t0 + r / (p.box_h * p.box_w),
                          qh = bx.h0 + (r / p.box_w) % p.box_h, qw = bx.w0 + r % p.box_w;
                row_valid = bx.active && qt < p.Tg && qh < p.Hg && qw < p.Wg;
                token = (qt * p.Hg + qh) * p.Wg + qw;
                qs_t = wstart(min(qt, p.Tg - 1), p.Tg, p.wt);
                qs_h = wstart(min(qh, p.Hg - 1), p.Hg, p.wh);
                qs_w = wstart(min(qw, p.Wg - 1), p.Wg, p.ww);
            }

            float m_run = -INFINITY, l = 0.f;
            uint64_t wbias2[kKvW / 2];   // LOCAL: 0 / -inf per column of the current w range, paired
            int wbias_w0 = -(1 << 30);   // w of the first column wbias2 was built for
#pragma unroll
            for (int c = 0; c < kKvW / 2; ++c) wbias2[c] = 0ull;
            int jt = 0, jh = 0, jw = 0;  // LOCAL: the step's sub-tile in (t, h, w) order
            for (int j = 0; j < it.n; ++j) {
                if (!wait(sh.s_full[t], sc & 1u)) { ok = false; break; }
                ++sc;
                tc_fence_after();
                if (dense) {
                    const int valid = p.N - (it.kv_lo + j) * kTileKeys;
                    if (valid >= kTileKeys)
                        softmax_tile<D, kAll>(tS, tO, j > 0, 0, wbias2, 0u, 0xFFu, p.scale_log2,
                                              m_run, l);
                    else
                        softmax_tile<D, kPrefix>(tS, tO, j > 0, valid, wbias2, 0u, 0xFFu,
                                                 p.scale_log2, m_run, l);
                } else {
                    const int kt = bx.tlo + jt, kh0 = bx.hlo + jh * kKvH, kw0 = bx.wlo + jw * kKvW;
                    if (++jw == p.nkw) {
                        jw = 0;
                        if (++jh == p.nkh) {
                            jh = 0;
                            ++jt;
                        }
                    }
                    if (kw0 != wbias_w0) {
                        // columns kw0 .. kw0+15 inside the row's w-window get bias 0
                        wbias_w0 = kw0;
#pragma unroll
                        for (int c = 0; c < kKvW; c += 2)
                            wbias2[c / 2] = f2((unsigned)(kw0 + c - qs_w) < (unsigned)p.ww ? 0u : 0xff800000u,
                                               (unsigned)(kw0 + c + 1 - qs_w) < (unsigned)p.ww ? 0u : 0xff800000u);
                    }
                    // rows g of the sub-tile inside the row's h-window: bits
                    // [qs_h - kh0, qs_h - kh0 + wh) clipped to [0, 8)
                    const bool t_ok = (unsigned)(kt - qs_t) < (unsigned)p.wt;
                    const int glo = max(qs_h - kh0, 0), ghi = min(qs_h - kh0 + p.wh, kKvH);
                    const uint32_t gmask =
                        t_ok && glo < ghi ? ((1u << ghi) - 1u) & ~((1u << glo) - 1u) : 0u;
                    // groups no row of this warp sees are skipped (their P is zero)
                    const uint32_t active = __reduce_or_sync(0xffffffffu, gmask);
                    softmax_tile<D, kWindow>(tS, tO, j > 0, 0, wbias2, gmask, active,
                                             p.scale_log2, m_run, l);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&sh.p_full[t]));
            }
            if (!ok) break;

            // ---- epilogue: out row = O / l
            if (!wait(sh.o_done[t], items & 1u)) { ok = false; break; }
            tc_fence_after();
            bool store = row_valid;
            if (!dense) {
                if (!wait(sh.flags_full, lc & 1u)) { ok = false; break; }
                store = row_valid && !sh.no_store[t][r];
                mbar_arrive(smem_addr(&sh.flags_empty));
                ++lc;
            }
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + (row0 + token) * D);
            if (dense && it.nsplit > 1) {
                // ---- split key range: publish this partial; the last split merges
                const int64_t prow =
                    ((int64_t)(it.pair_id * it.nsplit + it.split) * 2 + t) * kTileRows + r;
                float4 *po = reinterpret_cast<float4 *>(p.part_o + prow * D);
#pragma unroll
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(tO + 32 * c4, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        __stcg(po + c4 * 8 + v,
                               make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                           __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3])));
                }
                __stcg(p.part_ml + prow, make_float2(m_run, l));
                __threadfence();
                named_bar(1 + t, kTileRows);
                if (r == 0) sh.fix_old[t] = atomicAdd(p.fix_count + it.pair_id * 2 + t, 1);
                named_bar(1 + t, kTileRows);
                const int old = *reinterpret_cast<volatile int *>(&sh.fix_old[t]);
                if (old == it.nsplit - 1) {
                    __threadfence();
                    float mm = m_run;
                    for (int sp = 0; sp < it.nsplit; ++sp) {
                        if (sp == it.split) continue;
                        const int64_t orow =
                            ((int64_t)(it.pair_id * it.nsplit + sp) * 2 + t) * kTileRows + r;
                        mm = fmaxf(mm, __ldcg(p.part_ml + orow).x);
                    }
                    float L = 0.f;
                    for (int sp = 0; sp < it.nsplit; ++sp) {
                        const int64_t orow =
                            ((int64_t)(it.pair_id * it.nsplit + sp) * 2 + t) * kTileRows + r;
                        const float2 ml = __ldcg(p.part_ml + orow);
                        L += ml.y * ex2(ml.x - mm);
                    }
                    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
                    for (int c8 = 0; c8 < D / 8; ++c8) {
                        float acc[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
                        for (int sp = 0; sp < it.nsplit; ++sp) {
                            const int64_t orow =
                                ((int64_t)(it.pair_id * it.nsplit + sp) * 2 + t) * kTileRows + r;
                            const float a = ex2(__ldcg(p.part_ml + orow).x - mm);
                            const float4 *src = reinterpret_cast<const float4 *>(p.part_o + orow * D);
                            const float4 x0 = __ldcg(src + 2 * c8), x1 = __ldcg(src + 2 * c8 + 1);
                            acc[0] += a * x0.x; acc[1] += a * x0.y; acc[2] += a * x0.z; acc[3] += a * x0.w;
                            acc[4] += a * x1.x; acc[5] += a * x1.y; acc[6] += a * x1.z; acc[7] += a * x1.w;
                        }
                        if (store) {
                            uint4 w;
                            w.x = pack_bf16(acc[0] * inv, acc[1] * inv);
                            w.y = pack_bf16(acc[2] * inv, acc[3] * inv);
                            w.z = pack_bf16(acc[4] * inv, acc[5] * inv);
                            w.w = pack_bf16(acc[6] * inv, acc[7] * inv);
                            dst[c8] = w;
                        }
                    }
                }
            } else {
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(tO + 32 * c4, o);
                    tmem_wait_ld();
                    if (store && p.out32) {
                        // 32-byte stores: each lane writes a whole sector of its row
#pragma unroll
                        for (int v = 0; v < 2; ++v) {
                            uint32_t w[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                w[e] = pack_bf16(__uint_as_float(o[16 * v + 2 * e]) * inv,
                                                 __uint_as_float(o[16 * v + 2 * e + 1]) * inv);
                            st_global_v8(dst + c4 * 4 + 2 * v, w);
                        }
                    } else if (store) {
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
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&sh.o_empty[t]));
            ++items;
        }
        if (!ok) fail();
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

bool encode(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
            const cuuint64_t *strides, const cuuint32_t *box)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides,
              box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [B*H][N][D] bf16, box = 128 keys x 64 channels
bool map_rows(CUtensorMap *m, const void *base, int BH, int N, int D)
{
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kTileKeys, 1};
    return encode(m, base, 3, dims, strides, box);
}

// [B*H][T][H][W][D] bf16, box = bt x bh x bw tokens x 64 channels
bool map_grid(CUtensorMap *m, const void *base, int BH, int T, int Hg, int Wg, int D, int bt,
              int bh, int bw)
{
    const cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)Wg, (cuuint64_t)Hg, (cuuint64_t)T,
                                (cuuint64_t)BH};
    const cuuint64_t strides[4] = {(cuuint64_t)D * 2, (cuuint64_t)Wg * D * 2,
                                   (cuuint64_t)Hg * Wg * D * 2, (cuuint64_t)T * Hg * Wg * D * 2};
    const cuuint32_t box[5] = {64, (cuuint32_t)bw, (cuuint32_t)bh, (cuuint32_t)bt, 1};
    return encode(m, base, 5, dims, strides, box);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

int plan_sms()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms < 1) {
        cudaGetLastError();  // (no device visible: not an error of a later call)
        return kDefaultSMs;
    }
    return sms;
}

AttnPlan plan_attention(int B, int H, int d, int N, int k, int Tg, int Hg, int Wg, int wt,
                        int wh, int ww, int sms, bool per_sample_counts, bool allow_split)
{
    AttnPlan pl;
    pl.sms = sms = max(sms, 1);
    pl.max_split = allow_split ? kMaxSplit : 1;
    pl.n_kv_d = (N + kTileKeys - 1) / kTileKeys;
    pl.tiles_d = (k + kTileRows - 1) / kTileRows;
    pl.pairs_d = (pl.tiles_d + 1) / 2;
    const int64_t pairs_total = (int64_t)B * H * pl.pairs_d;
    // Whole waves of pairs (a multiple of the SM count) run over the whole key
    // range; the pairs of a last wave at most half full (or of a first and
    // only, partial wave) are cut into two key ranges so that they spread over
    // the SMs, and the range that finishes second merges the other's partial
    // result; a fuller last wave runs whole.
    // The LOCAL items fill in behind.  (Cutting into up to 8 ranges was
    // measured slower: each merge costs more than the finer spread gains.)
    pl.pairs_full = (int)pairs_total;
    pl.nsplit = 1;
    if (k > 0 && pl.n_kv_d >= 16) {
        pl.pairs_full = (int)(pairs_total / sms * sms);
        const int64_t rest = pairs_total - pl.pairs_full;
        pl.nsplit = rest > 0 ? min(pl.max_split, pl.n_kv_d / 8) : 1;
        if (pl.pairs_full > 0 && rest > sms / 2) pl.nsplit = 1;
        if (pl.nsplit < 2) {  // a last wave more than half full runs whole
            pl.nsplit = 1;
            pl.pairs_full = (int)pairs_total;
        }
    }
    pl.kv_per_split = (pl.n_kv_d + pl.nsplit - 1) / pl.nsplit;
    int64_t pairs_split = pairs_total - pl.pairs_full;  // pairs cut into key ranges
    int64_t split_ranges = pairs_split * pl.nsplit;      // their ranges
    pl.n_dense_items = (int)(pl.pairs_full + split_ranges);
    if (per_sample_counts) {
        // The device plans from the real counts (at most k per sample), the
        // same way: reserve ids and scratch for the worst remainder.
        int64_t extra = 0, worst_split = 0, worst_ranges = 0;
        if (k > 0 && pl.n_kv_d >= 16) {
            for (int rest = 1; rest < sms && rest <= pairs_total; ++rest) {
                // (the device's pairs_full may be 0, when the counts are small)
                const int ns = min(pl.max_split, pl.n_kv_d / 8);
                if (ns < 2) continue;
                extra = max(extra, (int64_t)rest * (ns - 1));
                worst_split = rest;
                worst_ranges = max(worst_ranges, (int64_t)rest * ns);
            }
        }
        pl.n_dense_items = (int)(pairs_total + extra);
        pairs_split = worst_split;
        split_ranges = worst_ranges;
        if (worst_ranges > 0) pl.nsplit = 2;  // (the scratch below is sized by the ranges)
    }
    // LOCAL query box: of the 128-token shapes below, the one whose boxes'
    // K/V covers hold the fewest keys in all (a box's cover spans the union of
    // its rows' windows, rounded up to whole 1x8x16 key sub-tiles); ties keep
    // the earlier shape.  Small windows take 2x8x8, an 11^3 window 8x4x4.
    {
        static const int shapes[][3] = {{2, 8, 8}, {4, 4, 8}, {4, 8, 4}, {8, 4, 4},
                                        {2, 4, 16}, {1, 8, 16}, {8, 8, 2}};
        int64_t best = -1;
        for (const auto &sh : shapes) {
            const int bt = sh[0], bh = sh[1], bw = sh[2];
            const int64_t boxes = (int64_t)((Tg + bt - 1) / bt) * ((Hg + bh - 1) / bh) *
                                  ((Wg + bw - 1) / bw);
            const int nkt = min(bt + wt - 1, Tg);
            const int nkh = (min(bh + wh - 1, Hg) + kKvH - 1) / kKvH;
            const int nkw = (min(bw + ww - 1, Wg) + kKvW - 1) / kKvW;
            const int64_t cost = ((boxes + 1) / 2) * nkt * nkh * nkw;
            if (best < 0 || cost < best) {
                best = cost;
                pl.box_t = bt;
                pl.box_h = bh;
                pl.box_w = bw;
            }
        }
    }
    const int nbt = (Tg + pl.box_t - 1) / pl.box_t;
    pl.nbh = (Hg + pl.box_h - 1) / pl.box_h;
    pl.nbw = (Wg + pl.box_w - 1) / pl.box_w;
    pl.tiles_l = nbt * pl.nbh * pl.nbw;
    pl.pairs_l = (pl.tiles_l + 1) / 2;
    pl.nkt = min(pl.box_t + wt - 1, Tg);
    pl.nkh = (min(pl.box_h + wh - 1, Hg) + kKvH - 1) / kKvH;
    pl.nkw = (min(pl.box_w + ww - 1, Wg) + kKvW - 1) / kKvW;
    pl.n_kv_l = pl.nkt * pl.nkh * pl.nkw;
    pl.n_local_items = (k < N || per_sample_counts) ? B * H * pl.pairs_l : 0;
    pl.total_items = pl.n_dense_items + pl.n_local_items;
    // workspace: counter | split arrivals | (m,l) partials | O partials
    pl.off_fix = 256;
    const size_t fix_bytes = split_ranges > 0 ? (size_t)pairs_split * 2 * sizeof(int) : 0;
    pl.zero_bytes = pl.off_fix + fix_bytes;
    pl.off_ml = align_up(pl.zero_bytes, 256);
    const size_t rows = split_ranges > 0 ? (size_t)split_ranges * 2 * kTileRows : 0;
    pl.off_o = align_up(pl.off_ml + rows * sizeof(float2), 256);
    pl.workspace_bytes = pl.off_o + rows * d * sizeof(float);
    return pl;
}

cudaError_t launch_attention(const AttnArgs &a, const AttnPlan &pl, void *workspace,
                             cudaStream_t s)
{
    Params p;
    p.Q = a.Q;
    p.out = a.out;
    p.out32 = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
    p.dense_idx = a.dense_idx;
    p.k_dev = a.k_dev;
    p.status = a.status;
    p.B = a.B; p.H = a.H; p.N = a.N; p.k = a.k;
    p.Tg = a.Tg; p.Hg = a.Hg; p.Wg = a.Wg; p.wt = a.wt; p.wh = a.wh; p.ww = a.ww;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.tiles_d = pl.tiles_d; p.pairs_d = pl.pairs_d; p.pairs_full = pl.pairs_full;
    p.nsplit = pl.nsplit;
    p.max_split = pl.max_split;
    p.sms = pl.sms;
    p.n_kv_d = pl.n_kv_d; p.kv_per_split = pl.kv_per_split; p.n_dense_items = pl.n_dense_items;
    p.box_t = pl.box_t; p.box_h = pl.box_h; p.box_w = pl.box_w;
    p.tiles_l = pl.tiles_l; p.pairs_l = pl.pairs_l; p.nbh = pl.nbh; p.nbw = pl.nbw;
    p.nkt = pl.nkt; p.nkh = pl.nkh; p.nkw = pl.nkw; p.n_kv_l = pl.n_kv_l;
    p.n_local_items = pl.n_local_items; p.total_items = pl.total_items;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    p.counter = reinterpret_cast<int *>(ws);
    p.fix_count = reinterpret_cast<int *>(ws + pl.off_fix);
    p.part_ml = reinterpret_cast<float2 *>(ws + pl.off_ml);
    p.part_o = reinterpret_cast<float *>(ws + pl.off_o);
    if (pl.total_items == 0) return cudaSuccess;

    const int BH = a.B * a.H, D = a.d;
    CUtensorMap k3, v3, k5, v5, q5;
    if (!map_rows(&k3, a.K, BH, a.N, D) || !map_rows(&v3, a.V, BH, a.N, D) ||
        !map_grid(&k5, a.K, BH, a.Tg, a.Hg, a.Wg, D, 1, kKvH, kKvW) ||
        !map_grid(&v5, a.V, BH, a.Tg, a.Hg, a.Wg, D, 1, kKvH, kKvW) ||
        !map_grid(&q5, a.Q, BH, a.Tg, a.Hg, a.Wg, D, pl.box_t, pl.box_h, pl.box_w))
        return cudaErrorInvalidValue;

    cudaError_t e = cudaMemsetAsync(workspace, 0, pl.zero_bytes, s);
    if (e != cudaSuccess) return e;
    const int grid = min(pl.total_items, pl.sms);
    if (D == 64) {
        e = cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg<64>::kSmem);
        if (e != cudaSuccess) return e;
        attn_tc_kernel<64><<<grid, kThreads, Cfg<64>::kSmem, s>>>(k3, v3, k5, v5, q5, p);
    } else {
        e = cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg<128>::kSmem);
        if (e != cudaSuccess) return e;
        attn_tc_kernel<128><<<grid, kThreads, Cfg<128>::kSmem, s>>>(k3, v3, k5, v5, q5, p);
    }
    return cudaGetLastError();
}

}  // namespace heta
