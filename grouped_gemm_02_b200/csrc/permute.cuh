// permute.cuh -- device-side histogram, prefix scan, stable permutation, row
// gather (S3, S4) and the tile plan of the skew-aware scheduler (S5').
//
// Decoding the Skew (abstract) asks for the live per-expert routing histogram
// to pick the expert-GEMM kernel without a CPU-GPU synchronisation: every
// count, offset and plan entry below stays on the device.
//
// Definitions (pair q = t*k + j):
//   counts[e]   = #{q : idx[q] = e}
//   offsets     = exclusive scan of counts, offsets[E] = number of valid pairs
//   pos(q)      = offsets[idx[q]] + #{q' < q : idx[q'] = idx[q]}   (stable)
//   perm[pos]   = q,  inv_perm[q] = pos,  xp[pos, :] = x[q / k, :]
// A pair whose expert id is outside [0, E) is dropped: it raises
// DEVERR_EXPERT_RANGE and gets inv_perm[q] = -1.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "route.cuh"
#include "schedule.h"
#include "tile_table.h"

namespace moe {

// The tuned tile cap of each histogram class (tile_table.h).
__constant__ int c_tile_cap[kTileClasses] = MOE_TILE_CAP_TABLE;

// ---------------------------------------------------------------- histogram
// grid hist_blocks(P), block 512: CTA b counts pairs [b*kHistChunk, ...) into
// block_counts[b*E + e].
__global__ void __launch_bounds__(512) hist_kernel(const int32_t* __restrict__ idx, int64_t P, int E,
                                                   int32_t* __restrict__ block_counts, uint32_t* __restrict__ err)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    __shared__ int32_t cnt[kMaxExperts];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int64_t q0 = (int64_t)blockIdx.x * kHistChunk;
    const int64_t q1 = min(P, q0 + kHistChunk);
    bool bad = false;
    for (int64_t q = q0 + threadIdx.x; q < q1; q += blockDim.x) {
        const int e = idx[q];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        else bad = true;
    }
    if (bad) atomicOr(err, DEVERR_EXPERT_RANGE);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) block_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

// ---------------------------------------------------------------- block scan helper
// Inclusive scan over blockDim.x (<= 1024) ints; returns the thread's inclusive prefix.
__device__ __forceinline__ int block_inclusive_scan(int v, int* warp_sums)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
        const int nw = (blockDim.x + 31) >> 5;
        int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += n;
        }
        if (lane < nw) warp_sums[lane] = s;
    }
    __syncthreads();
    const int add = warp > 0 ? warp_sums[warp - 1] : 0;
    __syncthreads();
    return v + add;
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- tile plan
// The tile plan of the skew-aware scheduler, built by one CTA (>= E+1 threads;
// thread tid < E holds counts[tid] in `c` and offsets[tid] in `off`):
//   * one block per expert with tokens, plus the shared expert (T rows) when
//     `shared_rows` > 0;
//   * a block of n rows is cut into units = ceil(n / ps.unit_rows) chunks of
//     chunk = ceil(n / units) rounded up to ps.align rows -- the tile width
//     follows the live count, so a 3-token expert gets a 16-wide tile and a
//     hot expert the widest ones;
//   * blocks sorted by n descending (ties: lower expert id), so the heaviest
//     tiles are dealt first;
//   * tile prefixes for both GEMMs: units * ceil(M / ps.m1_rows) gate/up tiles
//     and ceil(units / ps.merge) * ceil(d / ps.m2_rows) down tiles (a down tile
//     may span ps.merge units); the header records whether the tiles are cut
//     for CTA pairs and whether down tiles span two units.
__device__ __forceinline__ void build_plan(int c, int off, int E, int pairs, int32_t* __restrict__ plan, int f, int d,
                                           int shared_rows, int f_shared, int* warp_sums, PlanShape ps)
{
    __shared__ int s_n[kMaxGroups];
    __shared__ int s_order[kMaxGroups];
    __shared__ int s_nact;
    const int tid = threadIdx.x;
    const int G = E + 1;
    if (tid < G) s_n[tid] = tid < E ? c : shared_rows;
    if (tid == 0) s_nact = 0;
    __syncthreads();
    // rank of each active group: larger n first, then lower group id; an
    // inactive group (n == 0) never precedes an active one
    if (tid < G && s_n[tid] > 0) {
        const int n = s_n[tid];
        int r = 0;
        for (int j = 0; j < G; j++) {
            const int m = s_n[j];
            if (m > n || (m == n && j < tid)) r++;
        }
        s_order[r] = tid;
        atomicAdd(&s_nact, 1);
    }
    __syncthreads();
    const int nact = s_nact;
    // offsets of group g: read from the thread that owns it
    __shared__ int s_off[kMaxGroups];
    if (tid < E) s_off[tid] = off;
    // the histogram class of the routed experts: sum of c ln c and the largest count
    __shared__ float s_ent[32];
    __shared__ int s_cmax[32];
    __shared__ int s_cap, s_cls;
    {
        float ent = (tid < E && c > 0) ? (float)c * __logf((float)c) : 0.f;
        int cm = tid < E ? c : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ent += __shfl_xor_sync(0xffffffffu, ent, o);
            cm = max(cm, __shfl_xor_sync(0xffffffffu, cm, o));
        }
        if ((tid & 31) == 0) {
            s_ent[tid >> 5] = ent;
            s_cmax[tid >> 5] = cm;
        }
    }
    __syncthreads();
    if (tid == 0) {
        float ent = 0.f;
        int cm = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) {
            ent += s_ent[w];
            cm = max(cm, s_cmax[w]);
        }
        int cap = ps.unit_rows, cls = ps.policy == kTilesBucket ? kPlanClassBucket : kPlanClassCap;
        if (ps.policy == kTilesMatched && pairs > 0) {
            // effective experts = exp(entropy) = exp(ln P - sum(c ln c) / P)
            const float P = (float)pairs;
            const float eff = __expf(__logf(P) - ent / P);
            cls = tile_class(P, eff, (float)cm);
            cap = min(cap, c_tile_cap[cls]);
        }
        s_cap = max(ps.align, cap / ps.align * ps.align);
        s_cls = cls;
    }
    __syncthreads();
    const int cap = s_cap;
    PlanArrays pa = plan_arrays(plan);
    int my_t1 = 0, my_t2 = 0, my_chunk = 0;
    if (tid < nact) {
        const int g = s_order[tid];
        const int n = s_n[g];
        const int units = ceil_div(n, cap);
        // token buckets: every tile of the fixed width; otherwise the width follows the count
        const int chunk = ps.policy == kTilesBucket ? cap : ceil_div(ceil_div(n, units), ps.align) * ps.align;
        const int M1 = g < E ? f : f_shared;
        pa.group[tid] = g;
        pa.row0[tid] = g < E ? s_off[g] : 0;
        pa.rows[tid] = n;
        pa.chunk[tid] = chunk;
        pa.units[tid] = units;
        pa.dep[tid] = 0;
        my_t1 = units * ceil_div(M1, ps.m1_rows);
        my_t2 = ceil_div(units, ps.merge) * ceil_div(d, ps.m2_rows);
        my_chunk = chunk;
    }
    const int p1 = block_inclusive_scan(my_t1, warp_sums);
    const int p2 = block_inclusive_scan(my_t2, warp_sums);
    if (tid < nact) {
        pa.tb1[tid + 1] = p1;
        pa.tb2[tid + 1] = p2;
    }
    int mx = my_chunk;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((tid & 31) == 0) warp_sums[tid >> 5] = mx;
    __syncthreads();
    if (tid == 0) {
        int m = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) m = max(m, warp_sums[w]);
        PlanHeader* h = reinterpret_cast<PlanHeader*>(plan);
        h->n_blocks = nact;
        h->n_max = m;
        h->pairs = pairs;
        h->pair = ps.pair | (ps.merge == 2 ? 2 : 0);
        h->cls = s_cls;
        h->cap = cap;
        pa.tb1[0] = 0;
        pa.tb2[0] = 0;
        h->tiles1 = nact > 0 ? pa.tb1[nact] : 0;   // written above, visible after the barrier
        h->tiles2 = nact > 0 ? pa.tb2[nact] : 0;
    }
    __syncthreads();
}

// ---------------------------------------------------------------- scan (+ plan)
// Single CTA of 1024 threads.  Reduces the per-CTA histograms into counts and
// offsets, and turns block_counts into per-CTA bases (offsets[e] + pairs of e
// in earlier CTAs).  With `plan` non-null it also builds the tile plan.
__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ block_counts, int nblk_hist, int E,
                                                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ plan, int f, int d, int shared_rows,
                                                    int f_shared, PlanShape ps)
{
    __shared__ int warp_sums[32];
    __shared__ int s_pairs;
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int tid = threadIdx.x;
    int c = 0;
    if (tid < E)
        for (int b = 0; b < nblk_hist; b++) c += block_counts[(size_t)b * E + tid];
    const int incl = block_inclusive_scan(tid < E ? c : 0, warp_sums);
    const int off = incl - c;
    if (tid < E) {
        counts[tid] = c;
        offsets[tid] = off;
        int run = off;
        for (int b = 0; b < nblk_hist; b++) {
            const int v = block_counts[(size_t)b * E + tid];
            block_counts[(size_t)b * E + tid] = run;
            run += v;
        }
    }
    if (tid == E - 1) {
        offsets[E] = incl;
        s_pairs = incl;
    }
    __syncthreads();
    if (plan) build_plan(c, off, E, s_pairs, plan, f, d, shared_rows, f_shared, warp_sums, ps);
}

// Single CTA of 1024 threads: the tile plan from counts/offsets already on the device.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ counts,
                                                    const int32_t* __restrict__ offsets, int E,
                                                    int32_t* __restrict__ plan, int f, int d, int shared_rows,
                                                    int f_shared, PlanShape ps)
{
    __shared__ int warp_sums[32];
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int tid = threadIdx.x;
    const int c = tid < E ? counts[tid] : 0;
    const int off = tid < E ? offsets[tid] : 0;
    build_plan(c, off, E, offsets[E], plan, f, d, shared_rows, f_shared, warp_sums, ps);
}

// ---------------------------------------------------------------- small-T permutation
// One CTA of 1024 threads does S3-S4 (minus the row gather) and the tile plan
// when T*k <= 1024 (one pair per thread): per-warp expert counts by match_any,
// histogram, scan, stable positions and the plan, in one launch instead of
// three.
constexpr int kSmallPairs = 1024;

__global__ void __launch_bounds__(1024) permute_small_kernel(const int32_t* __restrict__ topk_idx, int P, int E,
                                                             int32_t* __restrict__ counts,
                                                             int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ perm,
                                                             int32_t* __restrict__ inv_perm,
                                                             int32_t* __restrict__ plan, int f, int d,
                                                             int shared_rows, int f_shared, PlanShape ps,
                                                             uint32_t* __restrict__ err)
{
    // s_wcnt[w][e]: pairs of warp w (pairs 32w..32w+31) routed to expert e (<= 32)
    __shared__ __align__(16) uint8_t s_wcnt[32][kMaxExperts];
    __shared__ int s_off[kMaxExperts];
    __shared__ int warp_sums[32];
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    reinterpret_cast<uint4*>(&s_wcnt[0][0])[tid] = make_uint4(0, 0, 0, 0);   // 1024 x 16 B = the whole table
    const int q = tid;
    int e = q < P ? topk_idx[q] : -1;
    if (e >= E || (q < P && e < 0)) {
        atomicOr(err, DEVERR_EXPERT_RANGE);
        inv_perm[q] = -1;
        e = -1;
    }
    __syncthreads();
    // per-warp counts: pairs of one warp with the same expert are ranked by lane
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && lane == __ffs(peers) - 1) s_wcnt[warp][e] = (uint8_t)__popc(peers);
    __syncthreads();
    // histogram and scan
    int c = 0;
    if (tid < E)
        for (int w = 0; w < 32; w++) c += s_wcnt[w][tid];
    const int incl = block_inclusive_scan(tid < E ? c : 0, warp_sums);
    const int off = incl - c;
    if (tid < E) {
        counts[tid] = c;
        offsets[tid] = off;
        s_off[tid] = off;
    }
    if (tid == E - 1) offsets[E] = incl;
    __syncthreads();
    // stable position: offsets[e] + pairs of e in earlier warps + rank in the warp
    if (e >= 0) {
        int pos = s_off[e] + rank;
        for (int w = 0; w < warp; w++) pos += s_wcnt[w][e];
        perm[pos] = q;
        inv_perm[q] = pos;
    }
    __shared__ int s_pairs;
    if (tid == E - 1) s_pairs = incl;
    __syncthreads();
    if (plan) build_plan(c, off, E, s_pairs, plan, f, d, shared_rows, f_shared, warp_sums, ps);
}

// ---------------------------------------------------------------- scatter
// grid hist_blocks(P), block 256.  CTA b walks its pairs in ascending q, 256 at a
// time; inside a warp, pairs with the same expert are ranked by lane order
// (match_any), and warps take their turn in order, so every segment stays in
// ascending q.
__global__ void __launch_bounds__(256) scatter_kernel(const int32_t* __restrict__ idx, int64_t P, int E,
                                                      const int32_t* __restrict__ block_base,
                                                      int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    __shared__ int32_t run[kMaxExperts];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e = threadIdx.x; e < E; e += blockDim.x) run[e] = block_base[(size_t)blockIdx.x * E + e];
    __syncthreads();
    const int64_t q0 = (int64_t)blockIdx.x * kHistChunk;
    const int64_t q1 = min(P, q0 + kHistChunk);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int64_t base = q0; base < q1; base += blockDim.x) {
        const int64_t q = base + threadIdx.x;
        int e = -1;
        if (q < q1) {
            e = idx[q];
            if (e < 0 || e >= E) {
                inv_perm[q] = -1;
                e = -1;
            }
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const int leader = __ffs(peers) - 1;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) {
            if (warp == w && e >= 0) {
                const int pos = run[e] + rank;
                perm[pos] = (int32_t)q;
                inv_perm[q] = pos;
            }
            __syncwarp();
            if (warp == w && e >= 0 && lane == leader) run[e] += __popc(peers);
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------- gather
// xp[inv_perm[t k + j], :] = x[t, :] for every pair with a valid position
// (inv_perm >= 0): xp[pos] = x[perm[pos] / k] for pos < pairs, taken in token
// order so that each x row is read once for its k copies (x is read T d 2
// bytes, not T k d 2).  One warp per (token, 512-byte chunk of the row): a
// 16-byte vector per lane, then its k stores.  Requires d % 8 == 0, k <= 32.
__global__ void __launch_bounds__(256) gather_rows_kernel(const bf16* __restrict__ x,
                                                          const int32_t* __restrict__ inv_perm, int T, int k, int d,
                                                          bf16* __restrict__ xp)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int nvec = d / 8;
    const int nch = (nvec + 31) / 32;
    const int lane = threadIdx.x & 31;
    const int64_t items = (int64_t)T * nch;
    for (int64_t w = (int64_t)(blockIdx.x * blockDim.x + threadIdx.x) / 32; w < items;
         w += (int64_t)gridDim.x * blockDim.x / 32) {
        const int64_t t = w / nch;
        const int v = (int)(w - t * nch) * 32 + lane;
        const int mine = lane < k ? inv_perm[t * k + lane] : -1;
        uint4 buf = make_uint4(0u, 0u, 0u, 0u);
        if (v < nvec) buf = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * d) + v);
        for (int j = 0; j < k; j++) {
            const int pos = __shfl_sync(0xffffffffu, mine, j);
            if (pos >= 0 && v < nvec) reinterpret_cast<uint4*>(xp + (size_t)pos * d)[v] = buf;
        }
    }
}

// ---------------------------------------------------------------- combine
// out[t, :] = bf16( sum_{j<k} y_p[inv_perm[t*k+j], :]  (+ ys[t, :]) ), summed in
// fp32 in ascending j, no atomics.  Dropped pairs (inv_perm < 0) add nothing.
// grid (T, column blocks), block 64; requires d % 8 == 0.
// inv_perm_ready: inv_perm was written two or more launches earlier (the layer
// forward), so it is read before griddepcontrol.wait.
__global__ void __launch_bounds__(128) combine_kernel(const bf16* __restrict__ y_p, const int32_t* __restrict__ inv_perm,
                                                      const bf16* __restrict__ ys, int T, int k, int d,
                                                      bf16* __restrict__ out, int inv_perm_ready)
{
    if (!inv_perm_ready) ptx::grid_dep_wait();
    const int t = blockIdx.x;
    int rows[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; j++) rows[j] = (t < T && j < k) ? inv_perm[(size_t)t * k + j] : -1;
    if (inv_perm_ready) ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    if (t >= T) return;
    const int nvec = d / 8;
    for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < nvec; v += gridDim.y * blockDim.x) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; i++) acc[i] = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxTopK; j++) {
            if (rows[j] >= 0) {
                const uint4 u = __ldg(reinterpret_cast<const uint4*>(y_p + (size_t)rows[j] * d) + v);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    acc[2 * i] += __uint_as_float(w[i] << 16);
                    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
                }
            }
        }
        if (ys) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(ys + (size_t)t * d) + v);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                acc[2 * i] += __uint_as_float(w[i] << 16);
                acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
            }
        }
        uint4 o;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
            ow[i] = *reinterpret_cast<const uint32_t*>(&p);
        }
        reinterpret_cast<uint4*>(out + (size_t)t * d)[v] = o;
    }
}

}  // namespace moe
