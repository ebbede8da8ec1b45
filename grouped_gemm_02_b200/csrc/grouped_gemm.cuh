// grouped_gemm.cuh -- persistent tcgen05/TMEM grouped GEMM fed by TMA (S1 on
// tensor cores, S5, S5', S6, S7).
//
// The expert GEMMs of the layer (Decoding the Skew, abstract: "sparse expert
// GEMMs whose shapes vary with the runtime routing distribution"; GC-MoE,
// abstract: operand-swapped tcgen05 MMA with a fused SwiGLU and optional
// shared experts):
//
//   MODE_GATED:  h[r, :]   = silu(xp[r] W1[e]^T) * (xp[r] W3[e]^T)   -> bf16
//   MODE_DOWN:   y_p[r, :] = w[perm[r]] * (h[r] W2[e]^T)             -> bf16
//
// for every row r of expert e's segment, and the router as a dense GEMM:
//
//   MODE_ROUTER: L[t, e] = x[t] Wg[e]^T (+ b[e])                     -> fp32
//
// split over K into fp32 partial sums when the token count alone cannot
// fill the SMs (the top-k kernel then adds the partials in a fixed order).
//
//   MODE_FUSED:  gate/up tiles then down tiles in one persistent launch.  A
//                down tile of expert block i loads its h rows only after every
//                gate/up tile of block i has stored them: each gate/up tile's
//                epilogue bumps a per-block counter (zeroed by the plan
//                builder) after its stores, and the producer of a down tile
//                waits for the count (bounded) before that tile's loads (W2
//                tiles it prefetched before griddepcontrol.wait are already
//                in flight).  The down tiles fill the gate/up tail instead of
//                a second launch ramping up.
//
// The MMA is operand-swapped: the weights fill the M = 128 slot and the tokens
// the N slot (16..256, chosen per expert from its live count by the plan), so
// a decode expert with 3 tokens costs one 16-wide MMA column block while a hot
// expert gets 256-wide tiles.  For the gate/up GEMM one A tile holds 64 rows
// of W1 (rows 0-63) and the same 64 rows of W3 (rows 64-127), each brought by
// one TMA box, so TMEM lanes 0-63 hold the gate and lanes 64-127 the up
// projection of the same f rows.  The epilogue warps of lane quadrants q and
// q + 2 pair up and hand each other half of every 16-column chunk through
// shared memory, so each finishes h = silu(g) u for 8 columns of 32 rows.
//
// Warp roles (192 threads, one CTA per SM, persistent over the tile list):
//   warp 0     TMA producer (lane 0; all lanes gather token rows) -> ring of smem stages
//   warp 1     TMEM allocator + MMA issuer (one elected lane)
//   warps 2-5  epilogue: tcgen05.ld -> SwiGLU / gate scale / bias -> global
// Two TMEM accumulators of 256 columns let the epilogue of tile i overlap the
// mainloop of tile i+1.
//
// Programmatic dependent launch: the kernel is launched so that it may start
// while the previous kernel on the stream finishes.  Weight tiles (A) do not
// depend on that kernel, so the producer fills the first ring stages with them
// before griddepcontrol.wait; token tiles (B) are loaded after it.  Every
// kernel of the layer waits before it triggers its dependents, so data made
// two or more kernels earlier (the tile plan, perm, gates) is complete when a
// kernel starts.
//
// Every wait is bounded: on timeout the kernel sets DEVERR_TIMEOUT, drains its
// own copies and MMAs (again bounded), frees TMEM and returns.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"
#include "schedule.h"

namespace moe {

constexpr int MODE_DOWN = 0;
constexpr int MODE_GATED = 1;
constexpr int MODE_ROUTER = 2;
constexpr int MODE_FUSED = 3;

constexpr int kGemmThreads = 192;
constexpr int kBlockK = 64;                          // bf16 elements per 128-byte swizzle row
constexpr int kATileBytes = 128 * kBlockK * 2;       // 16 KB: 128 weight rows
constexpr int kBRowBytes = kBlockK * 2;              // 128 B per token row
constexpr int kMaxStages = 12;
constexpr int kRingBytes = 200 * 1024;
constexpr int kBarBytes = 512;
constexpr uint32_t kTmemCols = 512;                  // 2 accumulators x 256 columns
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;   // 1 s

struct GemmArgs {
    const int32_t* plan;        // PlanHeader + PlanArrays (device); unused by MODE_ROUTER
    int plan_ready;             // plan written >= 2 kernels earlier: readable before griddepcontrol.wait
    int E;                      // routed experts; group E is the shared expert
    int M, M_shared;            // output rows per group: f (gate/up) or d (down) or E (router); shared: f_shared or d
    int K, K_shared;            // reduction length: d (gate/up, router) or f / f_shared (down)
    bf16* out;                  // h [pairs, f] or y_p [pairs, d]
    int ld_out;
    bf16* out_shared;           // hs [T, f_shared] or ys [T, d]
    int ld_out_shared;
    const int32_t* perm;        // down GEMM: gate of row r is gate_w[perm[r]]
    const float* gate_w;
    // MODE_ROUTER: tokens split into `units` chunks of `chunk` rows, `mt` tiles of
    // 128 experts, K split into `splits` ranges of `kb_per` 64-wide blocks.
    int T, units, chunk, mt, splits, kb_per;
    // MODE_FUSED: down tiles an SM with one gate/up tile fewer takes first (the
    // ratio of gate/up to down k-blocks per tile, rounded; see cta_tile)
    int comp;
    float* out_f32;             // splits == 1: logits [T, E] (+ bias); else partials [splits, T, E]
    const float* bias;          // may be null
    uint32_t* err;
    // gate/up tiles of routed experts take token row r of their expert segment
    // from x row gather_perm[r] / gather_k (TMA gathers) instead of from xp; null: xp
    const int32_t* gather_perm;
    int gather_k;
};

struct Tile {
    int group, m, row0, rows, n_mma, K, kb0, kb1, split;
    int blk;        // block (plan entry) index
    int ma;         // this CTA's M-tile of the weights: m, or 2m + rank for a CTA pair
    int b_row0;     // first B row this CTA loads, and how many (n_mma, or n_mma / 2 for a pair)
    int b_n;
    bool shared;
    bool gated;     // a gate/up tile (SwiGLU epilogue) rather than a down tile
};

// The plan entries this launch reads, copied to shared memory once per CTA so
// that decoding a tile (a binary search over the tile prefix) costs shared
// loads instead of a chain of dependent global loads at every tile boundary.
struct SmemPlan {
    int tb[kMaxGroups + 1];     // tile prefix of this GEMM (the gate/up one in MODE_FUSED)
    int tb2[kMaxGroups + 1];    // MODE_FUSED: tile prefix of the down tiles
    int4 blk[kMaxGroups];       // group, row0, rows, chunk
    int units[kMaxGroups];
    int tiles1;                 // MODE_FUSED: gate/up tiles come first
    int fixed_n;                // token-bucket plans: every tile's MMA width (padded); 0 otherwise
    int merge;                  // FP8 down GEMM: units one tile spans (1 or 2)
};
// gate/up epilogue: each pair of warps hands the other half of a 16-column chunk
// through shared memory: [2 row quarters][2 buffers][2 directions][8 columns][32 lanes] fp32
constexpr int kExchBytes = 2 * 2 * 2 * 8 * 32 * 4;
constexpr int kGemmSmemBytes = 1024 + kRingBytes + kBarBytes + (int)sizeof(SmemPlan) + kExchBytes;
static_assert(kGemmSmemBytes <= 227 * 1024, "shared memory budget");

template <int MODE>
__device__ __forceinline__ int total_tiles(const GemmArgs& a, const PlanHeader* hdr)
{
    if (MODE == MODE_ROUTER) return a.units * a.mt * a.splits;
    if (MODE == MODE_FUSED) return hdr->tiles1 + hdr->tiles2;
    return MODE == MODE_GATED ? hdr->tiles1 : hdr->tiles2;
}

template <int MODE, bool PAIR = false>
__device__ __forceinline__ Tile decode_tile(int nb, int t, const GemmArgs& a, const GemmArgs& a2, const SmemPlan* sp,
                                            int rank = 0)
{
    Tile tl;
    tl.blk = 0;
    tl.gated = MODE == MODE_GATED;
    if (MODE == MODE_ROUTER) {
        const int per_unit = a.mt * a.splits;
        const int u = t / per_unit;
        const int r = t - u * per_unit;
        tl.m = r / a.splits;
        tl.split = r - tl.m * a.splits;
        tl.group = 0;
        tl.shared = false;
        tl.row0 = u * a.chunk;
        tl.rows = min(a.chunk, a.T - tl.row0);
        tl.n_mma = (tl.rows + 15) & ~15;
        tl.K = a.K;
        const int nk = (a.K + kBlockK - 1) / kBlockK;
        tl.kb0 = tl.split * a.kb_per;
        tl.kb1 = min(nk, tl.kb0 + a.kb_per);
        tl.gated = false;
        tl.ma = tl.m;
        tl.b_row0 = tl.row0;
        tl.b_n = tl.n_mma;
        return tl;
    }
    bool gated = MODE == MODE_GATED;
    const int* tb = sp->tb;
    if (MODE == MODE_FUSED) {
        gated = t < sp->tiles1;
        if (!gated) {
            t -= sp->tiles1;
            tb = sp->tb2;
        }
    }
    int lo = 0, hi = nb - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    const int local = t - tb[lo];
    const int units = sp->units[lo];
    const int4 b = sp->blk[lo];
    const int chunk = b.w;
    tl.blk = lo;
    tl.gated = gated;
    tl.group = b.x;
    tl.shared = tl.group == a.E;
    // Order of a block's tiles: M-tile-major (the units of one weight M-tile run
    // together and share its fetch in L2, while the block's token rows stay in L2
    // across M-tiles), unless the block has more token rows than weight rows: then
    // unit-major (the block's weights stay in L2 and each unit's rows stream once).
    const GemmArgs& wa = (MODE == MODE_FUSED && !gated) ? a2 : a;
    const int wrows = (gated ? 2 : 1) * (tl.shared ? wa.M_shared : wa.M);
    const int mtiles = (tb[lo + 1] - tb[lo]) / units;
    int u;
    if (b.z > wrows) {
        u = local / mtiles;
        tl.m = local - u * mtiles;
    } else {
        tl.m = local / units;
        u = local - tl.m * units;
    }
    const int start = u * chunk;
    tl.rows = min(chunk, b.z - start);
    tl.row0 = b.y + start;
    // MMA width: a multiple of 16, of 32 for a pair (each CTA loads N/2 rows in 16-row boxes)
    tl.n_mma = sp->fixed_n ? sp->fixed_n : PAIR ? (tl.rows + 31) & ~31 : (tl.rows + 15) & ~15;
    tl.K = tl.shared ? a.K_shared : a.K;
    if (MODE == MODE_FUSED && !gated) tl.K = tl.shared ? a2.K_shared : a2.K;
    tl.kb0 = 0;
    tl.kb1 = (tl.K + kBlockK - 1) / kBlockK;
    tl.split = 0;
    if (PAIR) {
        // a pair tile: 2 x 128 weight rows, the CTA of rank r takes M-tile 2m + r
        // and B rows [row0 + r n/2, row0 + (r + 1) n/2)
        tl.ma = 2 * tl.m + rank;
        tl.b_n = tl.n_mma >> 1;
        tl.b_row0 = tl.row0 + rank * tl.b_n;
    } else {
        tl.ma = tl.m;
        tl.b_n = tl.n_mma;
        tl.b_row0 = tl.row0;
    }
    return tl;
}

struct SmemCtl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t sfull[kMaxStages];   // FP8 pair, second CTA: its own token scales (and FP4 weight scales) landed
    uint64_t tfull[4];     // accumulators 0-1; FP8 gate/up: the epilogue warps' amax exchange at 2 (and 3)
    uint64_t tempty[4];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(SmemCtl) <= kBarBytes, "control block too large");

// Spin on an mbarrier phase with a deadline.  Returns false (and flags the
// whole CTA) when the deadline passes or another role already gave up.
// kCluster: acquire at cluster scope (a barrier the other CTA of a pair arrives on
// after writing shared memory that this CTA then reads).
template <bool kCluster = false>
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, SmemCtl* ctl, uint32_t* err)
{
    auto test = [&]() { return kCluster ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity); };
    if (test()) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 256; i++)
            if (test()) return true;
        if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
        if (ptx::globaltimer() - t0 > kWaitTimeoutNs) {
            *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
            atomicOr(err, DEVERR_TIMEOUT);
            return false;
        }
    }
}

// Spin until the global counter reaches `need` (acquire), with the same
// deadline; on timeout or another role's abort, flag the CTA and return false.
__device__ __forceinline__ bool bounded_count_wait(const int* cnt, int need, SmemCtl* ctl, uint32_t* err)
{
    if (ptx::ld_acquire_gpu(cnt) >= need) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (ptx::ld_acquire_gpu(cnt) < need) {
        if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
        if (ptx::globaltimer() - t0 > kWaitTimeoutNs) {
            *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
            atomicOr(err, DEVERR_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

// The i-th tile of this CTA, or -1: the balanced deal of schedule.h in
// MODE_FUSED, round-robin in every other mode.
// A CTA pair deals by cluster: both CTAs of a cluster take the same tiles.
template <int MODE, bool PAIR = false>
__device__ __forceinline__ int cta_tile(int i, int total, int G, int comp)
{
    if (PAIR) return deal_tile((int)ptx::cluster_id_x(), (int)ptx::nclusters_x(), i, total, G, comp, MODE == MODE_FUSED);
    return deal_tile((int)blockIdx.x, (int)gridDim.x, i, total, G, comp, MODE == MODE_FUSED);
}

// Walks this CTA's (tile, k-block) sequence in order; shared by the two
// passes of the producer.
struct KIter {
    int i, t, kb;
    Tile tl;
};

template <int MODE, bool PAIR>
__device__ __forceinline__ bool kiter_seek(KIter& it, int nb, int total, const GemmArgs& a, const GemmArgs& a2,
                                           const SmemPlan* sp, int rank)
{
    for (; (it.t = cta_tile<MODE, PAIR>(it.i, total, sp->tiles1, a.comp)) >= 0; it.i++) {
        it.tl = decode_tile<MODE, PAIR>(nb, it.t, a, a2, sp, rank);
        if (it.tl.kb0 < it.tl.kb1) {
            it.kb = it.tl.kb0;
            return true;
        }
    }
    return false;
}

template <int MODE, bool PAIR>
__device__ __forceinline__ bool kiter_begin(KIter& it, int nb, int total, const GemmArgs& a, const GemmArgs& a2,
                                            const SmemPlan* sp, int rank)
{
    it.i = 0;
    return kiter_seek<MODE, PAIR>(it, nb, total, a, a2, sp, rank);
}

template <int MODE, bool PAIR>
__device__ __forceinline__ bool kiter_next(KIter& it, int nb, int total, const GemmArgs& a, const GemmArgs& a2,
                                           const SmemPlan* sp, int rank)
{
    if (++it.kb < it.tl.kb1) return true;
    ++it.i;
    return kiter_seek<MODE, PAIR>(it, nb, total, a, a2, sp, rank);
}

// One TMA tile load; a CTA of a pair counts its bytes on the leader's barrier
// (`full` is then a shared::cluster address).
template <bool PAIR>
__device__ __forceinline__ void tma_load(uint32_t dst, const CUtensorMap* map, uint32_t full, int c0, int c1,
                                         uint64_t pol)
{
    if (PAIR) ptx::tma_load_2d_pair(dst, map, full, c0, c1, pol);
    else ptx::tma_load_2d(dst, map, full, c0, c1, pol);
}

template <int MODE, bool PAIR>
__device__ __forceinline__ void issue_a(const KIter& it, uint32_t a_dst, uint32_t full, const CUtensorMap* mA0,
                                        const CUtensorMap* mA1, const CUtensorMap* mA0s, const CUtensorMap* mA1s,
                                        const CUtensorMap* mA2, const CUtensorMap* mA2s, const GemmArgs& a,
                                        const GemmArgs& a2, uint64_t pol)
{
    const Tile& tl = it.tl;
    const int kc = it.kb * kBlockK;
    if (tl.gated) {
        const CUtensorMap* w1 = tl.shared ? mA0s : mA0;
        const CUtensorMap* w3 = tl.shared ? mA1s : mA1;
        const int a_row = (tl.shared ? 0 : tl.group * a.M) + tl.ma * 64;
        tma_load<PAIR>(a_dst, w1, full, kc, a_row, pol);              // rows 0-63: gate
        tma_load<PAIR>(a_dst + 64 * 128, w3, full, kc, a_row, pol);   // rows 64-127: up
    } else if (MODE == MODE_FUSED) {
        const int a_row = (tl.shared ? 0 : tl.group * a2.M) + tl.ma * 128;
        tma_load<PAIR>(a_dst, tl.shared ? mA2s : mA2, full, kc, a_row, pol);
    } else {
        const CUtensorMap* a0 = tl.shared ? mA0s : mA0;
        const int a_row = (MODE == MODE_ROUTER || tl.shared ? 0 : tl.group * a.M) + tl.ma * 128;
        tma_load<PAIR>(a_dst, a0, full, kc, a_row, pol);
    }
}

// The token rows of a stage: 64-row boxes, then 16-row boxes for the rest
// (fewer, larger TMA requests keep the ring full at large widths).
template <bool PAIR>
__device__ __forceinline__ void issue_b(const Tile& tl, int kb, uint32_t b_dst, uint32_t full, const CUtensorMap* b16,
                                        const CUtensorMap* b64, uint64_t pol)
{
    const int kc = kb * kBlockK;
    const int n64 = tl.b_n >> 6;
    for (int i = 0; i < n64; i++)
        tma_load<PAIR>(b_dst + i * 64 * kBRowBytes, b64, full, kc, tl.b_row0 + 64 * i, pol);
    for (int r = n64 * 64; r < tl.b_n; r += 16)
        tma_load<PAIR>(b_dst + r * kBRowBytes, b16, full, kc, tl.b_row0 + r, pol);
}

template <int MODE, bool PAIR = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mA1,
                        const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mA0s,
                        const __grid_constant__ CUtensorMap mA1s, const __grid_constant__ CUtensorMap mBs,
                        const __grid_constant__ CUtensorMap mA2, const __grid_constant__ CUtensorMap mB2,
                        const __grid_constant__ CUtensorMap mA2s, const __grid_constant__ CUtensorMap mB2s,
                        const __grid_constant__ CUtensorMap mB64, const __grid_constant__ CUtensorMap mBs64,
                        const __grid_constant__ CUtensorMap mB264, const __grid_constant__ CUtensorMap mB2s64,
                        const __grid_constant__ CUtensorMap mBx, const GemmArgs args, const GemmArgs args2)
{
    // MODE_FUSED: args describe the gate/up tiles (W1/W3 = mA0/mA1, xp = mB),
    // args2 the down tiles (W2 = mA2, h = mB2); other modes ignore args2 and mA2..mB2s.
    // mB64..mB2s64 are mB..mB2s with 64-row boxes; mBx is x with one-row boxes (gathers).
    // PAIR: launched in clusters of two CTAs; a tile is 2 x 128 weight rows and
    // the leader (rank 0) issues its MMAs for both CTAs (cta_group::2).
    static_assert(!(PAIR && MODE == MODE_ROUTER), "the router runs on single CTAs");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + kRingBytes);
    const uint32_t ring = ptx::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = PAIR ? (int)ptx::cluster_ctarank() : 0;
    const bool leader = rank == 0;

    // The plan comes from an earlier kernel; when that kernel is the one right
    // before this launch, wait for it before reading anything.
    const bool waited_early = MODE != MODE_ROUTER && !args.plan_ready;
    if (waited_early) ptx::grid_dep_wait();

    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(args.plan);
    // a plan cut for the other tile shape (pair or single CTA) cannot be run:
    // every CTA of the launch sees the same header and leaves before any barrier
    if (MODE != MODE_ROUTER && hdr->pair != (PAIR ? 1 : 0)) {
        if (threadIdx.x == 0) atomicOr(args.err, DEVERR_PLAN);
        if (!waited_early) ptx::grid_dep_wait();
        ptx::grid_dep_launch();
        return;
    }
    const int nb = MODE == MODE_ROUTER ? 0 : hdr->n_blocks;
    const int total = total_tiles<MODE>(args, hdr);
    const int n_max = MODE == MODE_ROUTER ? max(16, (min(args.chunk, args.T) + 15) & ~15) : max(16, hdr->n_max);
    const uint32_t stage_bytes = kATileBytes + (uint32_t)(PAIR ? n_max / 2 : n_max) * kBRowBytes;
    const int stages = min(kMaxStages, (int)(kRingBytes / stage_bytes));

    SmemPlan* splan = reinterpret_cast<SmemPlan*>(smem + kRingBytes + kBarBytes);
    float* exch = reinterpret_cast<float*>(smem + kRingBytes + kBarBytes + sizeof(SmemPlan));
    if (MODE != MODE_ROUTER) {
        const PlanArrays pa = plan_arrays(const_cast<int32_t*>(args.plan));
        const int32_t* tbg = MODE == MODE_DOWN ? pa.tb2 : pa.tb1;
        if (threadIdx.x == 0) {
            splan->tiles1 = hdr->tiles1;
            splan->fixed_n = hdr->cls == kPlanClassBucket ? hdr->cap : 0;
        }
        for (int i = threadIdx.x; i <= nb; i += blockDim.x) {
            splan->tb[i] = tbg[i];
            if (MODE == MODE_FUSED) splan->tb2[i] = pa.tb2[i];
            if (i < nb) {
                splan->blk[i] = make_int4(pa.group[i], pa.row0[i], pa.rows[i], pa.chunk[i]);
                splan->units[i] = pa.units[i];
            }
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; s++) {
            ptx::mbar_init(ptx::smem_u32(&ctl->full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&ctl->empty[s]), 1);
        }
        for (int a = 0; a < 2; a++) {
            ptx::mbar_init(ptx::smem_u32(&ctl->tfull[a]), 1);
            // the epilogue warps of both CTAs of a pair free the leader's accumulator
            ptx::mbar_init(ptx::smem_u32(&ctl->tempty[a]), PAIR ? 8 : 4);
        }
        ptx::mbar_init(ptx::smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&mA0);
        ptx::prefetch_tensormap(&mB);
        if (MODE == MODE_GATED) ptx::prefetch_tensormap(&mA1);
    }
    if (warp == 1) {
        if (PAIR) {
            ptx::tmem_alloc_pair(ptx::smem_u32(&ctl->tmem_base), kTmemCols);
            ptx::tmem_relinquish_pair();
        } else {
            ptx::tmem_alloc(ptx::smem_u32(&ctl->tmem_base), kTmemCols);
            ptx::tmem_relinquish();
        }
    }
    ptx::tc_fence_before();
    // a pair's barriers are signalled across the two CTAs: both must be initialised first
    if (PAIR) ptx::cluster_sync();
    else __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    // the leader's barrier of a given offset, as the peer addresses it
    auto leader_bar = [&](uint64_t* bar) -> uint32_t {
        return PAIR ? ptx::mapa_shared(ptx::smem_u32(bar), 0) : ptx::smem_u32(bar);
    };
    // bytes one stage brings: this CTA's A and B tiles, or both CTAs' for a pair (the leader counts them)
    auto stage_tx = [&](const Tile& tl) -> uint32_t {
        return PAIR ? 2u * (kATileBytes + (uint32_t)tl.b_n * kBRowBytes) : kATileBytes + (uint32_t)tl.b_n * kBRowBytes;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // One elected lane issues every load; only when the gate/up tokens are
        // gathered from x does the whole warp take part (each lane gathers rows).
        if (MODE == MODE_ROUTER || MODE == MODE_DOWN || !args.gather_perm) {
            if (ptx::elect_one()) {
                const uint64_t pol = ptx::policy_evict_normal();
                uint32_t armed = 0, armed_ph = 0;   // slots with a load issued (leader's count), and its phase
                bool ok = true;
                // MODE_FUSED: all gate/up tiles of the tile's block have stored their h rows
                auto wait_block_ready = [&](const Tile& tl) -> bool {
                    const int32_t* dep = plan_arrays(const_cast<int32_t*>(args.plan)).dep + tl.blk;
                    const int m1 = tl.shared ? args.M_shared : args.M;
                    // 4 epilogue warps per CTA and gate/up tile (two CTAs per pair tile of 128 f rows)
                    const int need = PAIR ? 8 * splan->units[tl.blk] * ((m1 + 127) / 128)
                                          : 4 * splan->units[tl.blk] * ((m1 + 63) / 64);
                    if (!bounded_count_wait(dep, need, ctl, args.err)) return false;
                    ptx::fence_proxy_async_global();   // the TMA reads below come after the acquire
                    return true;
                };
                // pass 1 (before the dependency wait): weight tiles into the free stages
                int pre = 0;
                if (!waited_early) {
                    KIter it;
                    bool more = kiter_begin<MODE, PAIR>(it, nb, total, args, args2, splan, rank);
                    while (more && pre < stages) {
                        const uint32_t full = leader_bar(&ctl->full[pre]);
                        if (leader) {
                            ptx::mbar_arrive_expect_tx(ptx::smem_u32(&ctl->full[pre]), stage_tx(it.tl));
                            armed |= 1u << pre;
                        }
                        issue_a<MODE, PAIR>(it, ring + (uint32_t)pre * stage_bytes, full, &mA0, &mA1, &mA0s, &mA1s, &mA2,
                                            &mA2s, args, args2, pol);
                        ++pre;
                        more = kiter_next<MODE, PAIR>(it, nb, total, args, args2, splan, rank);
                    }
                    ptx::grid_dep_wait();
                }
                // After the wait, never before it: the layer's later kernels read data
                // written two launches back (the combine reads inv_perm before its own
                // wait), which holds only if every kernel waits before it triggers.
                ptx::grid_dep_launch();
                // pass 2: the same sequence again; the first `pre` stages only need their token tiles
                int s = 0, n = 0;
                uint32_t ph = 0;
                KIter it;
                bool more = kiter_begin<MODE, PAIR>(it, nb, total, args, args2, splan, rank);
                while (more) {
                    const uint32_t a_dst = ring + (uint32_t)s * stage_bytes;
                    const uint32_t full = leader_bar(&ctl->full[s]);
                    const bool first = it.tl.gated || MODE != MODE_FUSED;
                    const CUtensorMap* b = first ? (it.tl.shared ? &mBs : &mB) : (it.tl.shared ? &mB2s : &mB2);
                    const CUtensorMap* b64 = first ? (it.tl.shared ? &mBs64 : &mB64) : (it.tl.shared ? &mB2s64 : &mB264);
                    // a down tile of the fused launch reads h only after its block's gate/up tiles stored it
                    if (MODE == MODE_FUSED && !it.tl.gated && it.kb == 0 && !wait_block_ready(it.tl)) {
                        ok = false;
                        break;
                    }
                    if (n < pre) {
                        issue_b<PAIR>(it.tl, it.kb, a_dst + kATileBytes, full, b, b64, pol);
                    } else {
                        if (!bounded_wait(ptx::smem_u32(&ctl->empty[s]), ph ^ 1u, ctl, args.err)) {
                            ok = false;
                            break;
                        }
                        if (leader) {
                            ptx::mbar_arrive_expect_tx(ptx::smem_u32(&ctl->full[s]), stage_tx(it.tl));
                            armed |= 1u << s;
                            armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                        }
                        issue_a<MODE, PAIR>(it, a_dst, full, &mA0, &mA1, &mA0s, &mA1s, &mA2, &mA2s, args, args2, pol);
                        issue_b<PAIR>(it.tl, it.kb, a_dst + kATileBytes, full, b, b64, pol);
                    }
                    ++n;
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                    more = kiter_next<MODE, PAIR>(it, nb, total, args, args2, splan, rank);
                }
                if (!ok) {
                    // drain: wait (bounded) for every stage the leader armed; a pair's
                    // loads from both CTAs complete on the leader's barriers, and the
                    // peer does not leave before the leader (cluster barrier below)
                    const uint64_t t0 = ptx::globaltimer();
                    for (int i = 0; i < stages; i++) {
                        if (!(armed >> i & 1u)) continue;
                        const uint32_t bar = ptx::smem_u32(&ctl->full[i]);
                        while (!ptx::mbar_try_wait(bar, (armed_ph >> i) & 1u) &&
                               ptx::globaltimer() - t0 < kWaitTimeoutNs) {
                        }
                    }
                }
            }
        } else {
            // Row gathers (args.gather_perm): lane 0 waits on the ring, arms the stages
            // and loads the weight tiles; routed gate/up tiles take their token rows
            // straight from x, four rows per TMA gather and lane.
            const bool lead = lane == 0;
            const uint64_t pol = ptx::policy_evict_normal();
            uint32_t armed = 0, armed_ph = 0;   // slots with a load issued (leader's count), and its phase
            bool ok = true;
            // MODE_FUSED: all gate/up tiles of the tile's block have stored their h rows
            auto wait_block_ready = [&](const Tile& tl) -> bool {
                const int32_t* dep = plan_arrays(const_cast<int32_t*>(args.plan)).dep + tl.blk;
                const int m1 = tl.shared ? args.M_shared : args.M;
                // 4 epilogue warps per CTA and gate/up tile (two CTAs per pair tile of 128 f rows)
                const int need = PAIR ? 8 * splan->units[tl.blk] * ((m1 + 127) / 128)
                                      : 4 * splan->units[tl.blk] * ((m1 + 63) / 64);
                if (!bounded_count_wait(dep, need, ctl, args.err)) return false;
                ptx::fence_proxy_async_global();   // the TMA reads below come after the acquire
                return true;
            };
            // pass 1 (before the dependency wait): weight tiles into the free stages
            int pre = 0;
            if (!waited_early) {
                if (lead) {
                    KIter it;
                    bool more = kiter_begin<MODE, PAIR>(it, nb, total, args, args2, splan, rank);
                    while (more && pre < stages) {
                        const uint32_t full = leader_bar(&ctl->full[pre]);
                        if (leader) {
                            ptx::mbar_arrive_expect_tx(ptx::smem_u32(&ctl->full[pre]), stage_tx(it.tl));
                            armed |= 1u << pre;
                        }
                        issue_a<MODE, PAIR>(it, ring + (uint32_t)pre * stage_bytes, full, &mA0, &mA1, &mA0s, &mA1s, &mA2,
                                            &mA2s, args, args2, pol);
                        ++pre;
                        more = kiter_next<MODE, PAIR>(it, nb, total, args, args2, splan, rank);
                    }
                }
                pre = __shfl_sync(0xffffffffu, pre, 0);
                ptx::grid_dep_wait();
            }
            // After the wait, never before it: the layer's later kernels read data
            // written two launches back (the combine reads inv_perm before its own
            // wait), which holds only if every kernel waits before it triggers.
            if (lead) ptx::grid_dep_launch();
            // pass 2: the same sequence again; the first `pre` stages only need their token tiles
            int s = 0, n = 0;
            uint32_t ph = 0;
            int tok[8];          // gathered tiles: the tokens of this lane's rows 4q..4q+3, q = lane, lane + 32
            KIter it;
            bool more = kiter_begin<MODE, PAIR>(it, nb, total, args, args2, splan, rank);
            while (more) {
                const uint32_t a_dst = ring + (uint32_t)s * stage_bytes;
                const uint32_t full = leader_bar(&ctl->full[s]);
                const bool first = it.tl.gated || MODE != MODE_FUSED;
                const bool gather = MODE != MODE_ROUTER && args.gather_perm && it.tl.gated && !it.tl.shared;
                if (gather && it.kb == it.tl.kb0) {
                    // rows past the tile's tokens (MMA padding) repeat its last token
                    const int last = it.tl.row0 + it.tl.rows - 1;
    #pragma unroll
                    for (int j = 0; j < 8; j++) {
                        const int r = 4 * (lane + 32 * (j >> 2)) + (j & 3);
                        const int pos = min(it.tl.b_row0 + r, last);
                        tok[j] = r < it.tl.b_n ? __ldg(args.gather_perm + pos) / args.gather_k : 0;
                    }
                }
                // a down tile of the fused launch reads h only after its block's gate/up tiles stored it
                if (MODE == MODE_FUSED && !it.tl.gated && it.kb == 0) {
                    if (lead) ok = wait_block_ready(it.tl);
                    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                        ok = false;
                        break;
                    }
                }
                if (n >= pre) {
                    if (lead) {
                        ok = bounded_wait(ptx::smem_u32(&ctl->empty[s]), ph ^ 1u, ctl, args.err);
                        if (ok) {
                            if (leader) {
                                ptx::mbar_arrive_expect_tx(ptx::smem_u32(&ctl->full[s]), stage_tx(it.tl));
                                armed |= 1u << s;
                                armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                            }
                            issue_a<MODE, PAIR>(it, a_dst, full, &mA0, &mA1, &mA0s, &mA1s, &mA2, &mA2s, args, args2,
                                                pol);
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                        ok = false;
                        break;
                    }
                }
                if (gather) {
                    const int kc = it.kb * kBlockK;
                    const uint32_t b_dst = a_dst + kATileBytes;
    #pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const int q = lane + 32 * h;
                        if (4 * q < it.tl.b_n) {
                            if (PAIR)
                                ptx::tma_gather4_pair(b_dst + 512u * q, &mBx, full, kc, tok[4 * h], tok[4 * h + 1],
                                                      tok[4 * h + 2], tok[4 * h + 3], pol);
                            else
                                ptx::tma_gather4(b_dst + 512u * q, &mBx, full, kc, tok[4 * h], tok[4 * h + 1],
                                                 tok[4 * h + 2], tok[4 * h + 3], pol);
                        }
                    }
                } else if (lead) {
                    const CUtensorMap* b = first ? (it.tl.shared ? &mBs : &mB) : (it.tl.shared ? &mB2s : &mB2);
                    const CUtensorMap* b64 =
                        first ? (it.tl.shared ? &mBs64 : &mB64) : (it.tl.shared ? &mB2s64 : &mB264);
                    issue_b<PAIR>(it.tl, it.kb, a_dst + kATileBytes, full, b, b64, pol);
                }
                __syncwarp();
                ++n;
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
                more = kiter_next<MODE, PAIR>(it, nb, total, args, args2, splan, rank);
            }
            if (!ok && lead) {
                // drain: wait (bounded) for every stage the leader armed; a pair's
                // loads from both CTAs complete on the leader's barriers, and the
                // peer does not leave before the leader (cluster barrier below)
                const uint64_t t0 = ptx::globaltimer();
                for (int i = 0; i < stages; i++) {
                    if (!(armed >> i & 1u)) continue;
                    const uint32_t bar = ptx::smem_u32(&ctl->full[i]);
                    while (!ptx::mbar_try_wait(bar, (armed_ph >> i) & 1u) &&
                           ptx::globaltimer() - t0 < kWaitTimeoutNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (the leader of a pair)
        if (leader && ptx::elect_one()) {
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t aph = 0;
            bool ok = true, issued = false;
            for (int i = 0, t; ok && (t = cta_tile<MODE, PAIR>(i, total, splan->tiles1, args.comp)) >= 0; i++) {
                const Tile tl = decode_tile<MODE, PAIR>(nb, t, args, args2, splan, rank);
                if (tl.kb0 >= tl.kb1) continue;
                if (!bounded_wait(ptx::smem_u32(&ctl->tempty[acc]), aph ^ 1u, ctl, args.err)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * 256u;
                const uint32_t idesc = ptx::idesc_bf16_f32(PAIR ? 256 : 128, (uint32_t)tl.n_mma);
                for (int kb = tl.kb0; kb < tl.kb1; kb++) {
                    if (!bounded_wait(ptx::smem_u32(&ctl->full[s]), ph, ctl, args.err)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ring + (uint32_t)s * stage_bytes;
                    const uint32_t b_addr = a_addr + kATileBytes;
#pragma unroll
                    for (int kk = 0; kk < kBlockK / 16; kk++) {
                        const uint64_t ad = ptx::sw128_kmajor_desc(a_addr + kk * 32);
                        const uint64_t bd = ptx::sw128_kmajor_desc(b_addr + kk * 32);
                        const uint32_t accum = (kb > tl.kb0 || kk > 0) ? 1u : 0u;
                        if (PAIR) ptx::mma_bf16_ss_pair(d_tmem, ad, bd, idesc, accum);
                        else ptx::mma_bf16_ss(d_tmem, ad, bd, idesc, accum);
                    }
                    issued = true;
                    // the stage is free in both CTAs once these MMAs have read it
                    if (PAIR) ptx::mma_commit_pair(ptx::smem_u32(&ctl->empty[s]), 3);
                    else ptx::mma_commit(ptx::smem_u32(&ctl->empty[s]));
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                if (PAIR) ptx::mma_commit_pair(ptx::smem_u32(&ctl->tfull[acc]), 3);
                else ptx::mma_commit(ptx::smem_u32(&ctl->tfull[acc]));
                acc ^= 1;
                if (acc == 0) aph ^= 1u;
            }
            if (!ok && issued) {
                // drain: every MMA issued so far completes before TMEM is freed
                if (PAIR) ptx::mma_commit_pair(ptx::smem_u32(&ctl->drain), 1);
                else ptx::mma_commit(ptx::smem_u32(&ctl->drain));
                const uint64_t t0 = ptx::globaltimer();
                while (!ptx::mbar_try_wait(ptx::smem_u32(&ctl->drain), 0) &&
                       ptx::globaltimer() - t0 < kWaitTimeoutNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2-5)
        const int quad = warp & 3;            // TMEM lane quadrant this warp may access
        int acc = 0;
        uint32_t aph = 0;
        // gate/up chunks exchanged so far: the buffer alternates across tiles too, so
        // a chunk's writes always follow the partner's reads of the chunk before last
        uint32_t xchunk = 0;
        for (int i = 0, t; (t = cta_tile<MODE, PAIR>(i, total, splan->tiles1, args.comp)) >= 0; i++) {
            const Tile tl = decode_tile<MODE, PAIR>(nb, t, args, args2, splan, rank);
            if (tl.kb0 >= tl.kb1) continue;
            // a down tile's gates (lane l: columns l + 32 i), fetched before the accumulator wait
            float gates[8];
#pragma unroll
            for (int i = 0; i < 8; i++) gates[i] = 1.f;
            if (MODE != MODE_ROUTER && !tl.gated && !tl.shared) {
                const GemmArgs& ga = MODE == MODE_FUSED ? args2 : args;
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const int col = 32 * i + lane;
                    if (col < tl.rows) gates[i] = __ldg(ga.gate_w + __ldg(ga.perm + tl.row0 + col));
                }
            }
            const bool ok = bounded_wait(ptx::smem_u32(&ctl->tfull[acc]), aph, ctl, args.err);
            if (!__all_sync(0xffffffffu, ok)) break;   // the whole warp leaves together
            ptx::tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t)acc * 256u + ((uint32_t)(quad * 32) << 16);
            const GemmArgs& ea = (MODE == MODE_FUSED && !tl.gated) ? args2 : args;
            bf16* out = tl.shared ? ea.out_shared : ea.out;
            const size_t ld = (size_t)(tl.shared ? ea.ld_out_shared : ea.ld_out);
            const int Mrows = tl.shared ? ea.M_shared : ea.M;
            for (int c0 = 0; c0 < tl.n_mma; c0 += 16) {
                uint32_t v[16];
                ptx::tmem_ld16(taddr + (uint32_t)c0, v);
                ptx::tmem_ld_wait();
                if (MODE != MODE_ROUTER && tl.gated) {
                    // quadrants 0/1 hold the gate, 2/3 the up projection of f rows
                    // 32 (quad & 1) + lane; the gate warp finishes columns 0-7 of the
                    // chunk and sends its g of columns 8-15, the up warp the reverse
                    const int role = quad >> 1, rq = quad & 1;
                    const int frow = tl.ma * 64 + rq * 32 + lane;
                    float* xb = exch + (rq * 2 + (xchunk++ & 1u)) * 512;
                    float* mine = xb + role * 256;
                    const float* theirs = xb + (role ^ 1) * 256;
#pragma unroll
                    for (int j = 0; j < 8; j++) mine[j * 32 + lane] = __uint_as_float(v[role ? j : 8 + j]);
                    ptx::named_barrier(1 + rq, 64);
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        const float other = theirs[j * 32 + lane];
                        const float g = role ? other : __uint_as_float(v[j]);
                        const float u = role ? __uint_as_float(v[8 + j]) : other;
                        const int col = c0 + (role ? 8 : 0) + j;
                        if (col < tl.rows && frow < Mrows)
                            out[(size_t)(tl.row0 + col) * ld + frow] = __float2bfloat16_rn(silu_f(g) * u);
                    }
                } else if (MODE != MODE_ROUTER) {
                    const int drow = tl.ma * 128 + quad * 32 + lane;
                    const int gi = c0 >> 5;
                    const float mine = gi == 0 ? gates[0] : gi == 1 ? gates[1] : gi == 2 ? gates[2] : gi == 3 ? gates[3]
                                     : gi == 4 ? gates[4] : gi == 5 ? gates[5] : gi == 6 ? gates[6] : gates[7];
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const float sc = __shfl_sync(0xffffffffu, mine, (c0 & 31) + j);
                        const int col = c0 + j;
                        if (col < tl.rows && drow < Mrows)
                            out[(size_t)(tl.row0 + col) * ld + drow] =
                                __float2bfloat16_rn(__uint_as_float(v[j]) * sc);
                    }
                } else {
                    // router: lane = expert, column = token; fp32 logits or split-K partials
                    const int e = tl.m * 128 + quad * 32 + lane;
                    if (e < args.E) {
                        const bool whole = args.splits == 1;
                        const float b = (whole && args.bias) ? __ldg(args.bias + e) : 0.f;
                        float* dst = args.out_f32 + (size_t)(whole ? 0 : tl.split) * args.T * args.E;
#pragma unroll
                        for (int j = 0; j < 16; j++) {
                            const int col = c0 + j;
                            if (col < tl.rows) dst[(size_t)(tl.row0 + col) * args.E + e] = __uint_as_float(v[j]) + b;
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                // the accumulator is free again: tell the MMA issuer (the leader's, for a pair)
                if (PAIR) ptx::mbar_arrive_cluster(leader_bar(&ctl->tempty[acc]));
                else ptx::mbar_arrive(ptx::smem_u32(&ctl->tempty[acc]));
            }
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
            if (MODE == MODE_FUSED && tl.gated) {
                // publish this warp's h rows of the tile to the down tiles of its
                // block: each of the 4 epilogue warps adds 1 after its own stores
                ptx::fence_proxy_async_global();
                __syncwarp();
                if (lane == 0) ptx::red_add_release_gpu(plan_arrays(const_cast<int32_t*>(args.plan)).dep + tl.blk, 1);
            }
        }
    }

    ptx::tc_fence_before();
    // neither CTA of a pair leaves (or frees TMEM) while the other may still
    // signal its barriers or the leader's MMAs may still write its TMEM
    if (PAIR) ptx::cluster_sync();
    else __syncthreads();
    __syncwarp();   // the dealloc below is .sync.aligned: warp 1 converged
    if (warp == 1) {
        ptx::tc_fence_after();
        if (PAIR) ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
        else ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Diagnostic: one CTA waits, through the two bounded waits the GEMMs use, on
// an mbarrier nobody arrives on and on a counter nobody increments.  Each
// wait gives up after its deadline and sets DEVERR_TIMEOUT; the kernel then
// returns normally, so the context stays usable.
__global__ void __launch_bounds__(32) wait_timeout_probe_kernel(const int* never, uint32_t* err)
{
    __shared__ SmemCtl ctl;
    if (threadIdx.x != 0) return;
    ctl.abort = 0;
    ptx::mbar_init(ptx::smem_u32(&ctl.full[0]), 1);
    ptx::fence_mbar_init();
    const bool a = bounded_wait(ptx::smem_u32(&ctl.full[0]), 0u, &ctl, err);
    ctl.abort = 0;
    const bool b = bounded_count_wait(never, 1, &ctl, err);
    if (a || b) atomicOr(err, DEVERR_PLAN);   // a wait that should not have ended did
}

}  // namespace moe
