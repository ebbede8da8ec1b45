// common.cuh -- types shared by the host entry points and the kernels:
// device error bits, workspace layout, and the tile plan the scheduler reads.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>

namespace moe {

using bf16 = __nv_bfloat16;

// Sticky device error bits, OR-ed into the first word of the workspace.
enum : uint32_t {
    DEVERR_EXPERT_RANGE = 1u,   // a top-k expert id outside [0, E): that pair is dropped
    DEVERR_TIMEOUT = 2u,        // a bounded wait inside a kernel gave up
    DEVERR_NAN_LOGIT = 4u,      // a router logit was NaN (ranked below every number)
    DEVERR_PLAN = 8u,           // a kernel met a tile plan it cannot run (it did nothing)
};

constexpr int kMaxExperts = 512;
constexpr int kMaxTopK = 8;
constexpr int kMaxGroups = kMaxExperts + 1;   // routed experts + the shared expert
constexpr int kHistChunk = 4096;              // pairs per CTA in the multi-CTA histogram
constexpr int kTileRows = 256;                // most tokens one tile carries (MMA N <= 256)

// The tile plan, written by the plan step from the live histogram and read by
// every role of the grouped GEMM.  A "block" is one expert (or the shared
// expert) with at least one token; blocks are ordered by token count, largest
// first, so the heaviest tiles are handed out first.  A block's n tokens are
// cut into `units` equal chunks of `chunk` rows (a multiple of 16, <= 256);
// each unit times each M-tile of the weights is one tile.
struct PlanHeader {
    int32_t n_blocks;
    int32_t tiles1;     // tiles of the gate/up GEMM (M-tile = 64 rows of W1 and 64 of W3)
    int32_t tiles2;     // tiles of the down GEMM (M-tile = 128 rows of W2)
    int32_t n_max;      // widest tile (tokens) in this launch
    int32_t pairs;      // routed pairs with a valid expert id (== offsets[E])
    int32_t pair;       // bit 0: tiles cut for CTA pairs (2 x 128 weight rows, widths a multiple of 32);
                        // bit 1: a down tile spans two units (FP8 / FP4 GEMMs of the two-launch form)
    int32_t cls;        // histogram class the tile cap was looked up for, or kPlanClassCap / kPlanClassBucket
    int32_t cap;        // most tokens per tile in this plan's cut
};

// How the plan cuts an expert's tokens into tiles (the tile policy):
//   kTilesMatched  the live histogram's class picks the largest tile width
//                  (cap) from the tuned table; each expert's width then follows
//                  its own count: ceil(n / ceil(n / cap)), rounded up to align;
//   kTilesBucket   one fixed width (unit_rows, chosen from T alone) for every
//                  expert, the last tile of an expert padded -- the static
//                  token-bucket selection the histogram-matched one is
//                  measured against;
//   kTilesCap      the per-expert widths under a given cap (unit_rows).
constexpr int kPlanClassCap = -1;      // PlanHeader::cls of a plan cut under a given cap
constexpr int kPlanClassBucket = -2;   // ... and of a token-bucket plan (every tile padded to `cap`)
constexpr int kTilesMatched = 0;
constexpr int kTilesBucket = 1;
constexpr int kTilesCap = 2;

// The tile shape of a launch form and the tile policy: at most unit_rows
// tokens per tile, widths a multiple of `align`; m1_rows f rows per gate/up
// tile and m2_rows d rows per down tile.  Single CTAs: (256, 64, 128, 16, 0)
// for bf16 and (112, 128, 128, 16, 0) for FP8; CTA pairs: (256, 128, 256, 32, 1).
struct PlanShape {
    int unit_rows, m1_rows, m2_rows, align, pair;
    int policy;
    int merge = 1;   // units one down tile spans (2: the FP8 down GEMM of the two-launch form)
};

struct PlanArrays {
    // Each array has kMaxGroups (+1 for prefixes) entries.
    int32_t* group;     // expert id; E means the shared expert
    int32_t* row0;      // first row of the block in the B operand
    int32_t* rows;      // tokens in the block
    int32_t* chunk;     // rows per unit
    int32_t* units;
    int32_t* tb1;       // tile prefix, gate/up GEMM  [n_blocks + 1]
    int32_t* tb2;       // tile prefix, down GEMM     [n_blocks + 1]
    int32_t* dep;       // gate/up tiles of the block finished (fused GEMM), zeroed by the plan builder
};

constexpr size_t kPlanInts = 8 + 6 * kMaxGroups + 2 * (kMaxGroups + 1);

__host__ __device__ inline PlanArrays plan_arrays(int32_t* base)
{
    PlanArrays a;
    int32_t* p = base + 8;
    a.group = p; p += kMaxGroups;
    a.row0 = p; p += kMaxGroups;
    a.rows = p; p += kMaxGroups;
    a.chunk = p; p += kMaxGroups;
    a.units = p; p += kMaxGroups;
    a.tb1 = p; p += kMaxGroups + 1;
    a.tb2 = p; p += kMaxGroups + 1;
    a.dep = p;
    return a;
}

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// How the tensor-core router covers a [T, E] x d problem: tokens in `units`
// chunks of `chunk` rows (<= 256, a multiple of 16), experts in `mt` tiles of
// 128, and -- when units * mt tiles alone would leave most SMs idle -- the
// d-loop split into `splits` ranges of `kb_per` 64-wide blocks, so that one
// tile streams about kRouterTileBytes of Wg and x; the top-k step adds the
// fp32 partial sums in a fixed order.  The split depends on the sizes only
// (not on the device), so the workspace size and every result bit do too.
constexpr int kRouterTargetCtas = 148;
constexpr int64_t kRouterTileBytes = 64 * 1024;

struct RouterSplit {
    int units, chunk, mt, splits, kb_per, tiles;
};

__host__ __device__ inline RouterSplit router_split(int64_t T, int64_t d, int64_t E)
{
    RouterSplit r{};
    if (T <= 0 || d <= 0 || E <= 0) return r;
    const int nk = (int)((d + 63) / 64);
    r.mt = (int)((E + 127) / 128);
    r.units = (int)((T + 255) / 256);
    const int per = (int)((T + r.units - 1) / r.units);
    r.chunk = (per + 15) / 16 * 16;
    const int base = r.mt * r.units;
    r.kb_per = nk;
    r.splits = 1;
    if (base < kRouterTargetCtas) {
        const int64_t rows = (E < 128 ? E : 128) + r.chunk;          // weight rows + token rows per tile
        int64_t want = (rows * d * 2 + kRouterTileBytes - 1) / kRouterTileBytes;
        const int64_t cap = kRouterTargetCtas / base;
        if (want > cap) want = cap;
        if (want > nk) want = nk;
        if (want < 1) want = 1;
        r.kb_per = (int)((nk + want - 1) / want);
        r.splits = (nk + r.kb_per - 1) / r.kb_per;
    }
    r.tiles = base * r.splits;
    return r;
}

// Workspace layout.  The control part (error word, plan, histogram scratch)
// is all that moe_permute and moe_grouped_gemm need; moe_layer_forward also
// keeps every intermediate of the layer in the workspace.
struct WsLayout {
    size_t err;            // uint32 sticky error word
    size_t plan;           // int32[kPlanInts]
    size_t block_counts;   // int32[hist_blocks * E]
    size_t router_partials;  // fp32[splits, T, E] when the router splits K
    size_t ctrl_end;
    // layer intermediates
    size_t logits, topk_idx, topk_w, counts, offsets, perm, inv_perm, xp, h, y_p, hs, ys;
    size_t total;
};

__host__ __device__ inline int hist_blocks(int64_t P) { return (int)((P + kHistChunk - 1) / kHistChunk); }

__host__ inline WsLayout ws_layout(int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, int64_t fs)
{
    WsLayout L{};
    const int64_t P = T * k;
    size_t o = 0;
    L.err = o; o += 256;
    L.plan = o; o = align_up(o + kPlanInts * 4, 256);
    L.block_counts = o; o = align_up(o + (size_t)(hist_blocks(P) > 0 ? hist_blocks(P) : 1) * E * 4, 256);
    const RouterSplit rs = router_split(T, d, E);
    L.router_partials = o; o = align_up(o + (rs.splits > 1 ? (size_t)rs.splits * T * E * 4 : 0), 256);
    L.ctrl_end = o;
    L.logits = o; o = align_up(o + (size_t)T * E * 4, 256);
    L.topk_idx = o; o = align_up(o + (size_t)P * 4, 256);
    L.topk_w = o; o = align_up(o + (size_t)P * 4, 256);
    L.counts = o; o = align_up(o + (size_t)E * 4, 256);
    L.offsets = o; o = align_up(o + (size_t)(E + 1) * 4, 256);
    L.perm = o; o = align_up(o + (size_t)P * 4, 256);
    L.inv_perm = o; o = align_up(o + (size_t)P * 4, 256);
    L.xp = o; o = align_up(o + (size_t)P * d * 2, 1024);
    L.h = o; o = align_up(o + (size_t)P * f * 2, 1024);
    L.y_p = o; o = align_up(o + (size_t)P * d * 2, 1024);
    L.hs = o; o = align_up(o + (size_t)(fs > 0 ? T : 0) * fs * 2, 1024);
    L.ys = o; o = align_up(o + (size_t)(fs > 0 ? T : 0) * d * 2, 1024);
    L.total = o;
    return L;
}

// Workspace of the FP8 layer: the same control part, then the routing
// intermediates, e4m3 activations with their 1 x 128 scales, and y_p.
struct WsLayoutFp8 {
    WsLayout ctrl;   // err, plan, block_counts, router_partials, ctrl_end
    size_t logits, topk_idx, topk_w, counts, offsets, perm, inv_perm;
    size_t x8, sx, xp8, sxp, h8, sh, y_p, hs8, shs, ys, sxT;
    int64_t ld_pairs, ld_tokens;   // row length of the K-block-major scale arrays (pairs, tokens rounded up to 4)
    size_t total;
};

// Token scales the GEMM reads by TMA are stored K-block-major, [K/128][ld]
// with ld a multiple of 4 (a 16-byte row pitch): sxp [d/128][pairs],
// sh [f/128][pairs], shs [f_shared/128][T], sxT [d/128][T].  sx keeps the
// quantiser's row-major [T][d/128].
__host__ inline WsLayoutFp8 ws_layout_fp8(int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, int64_t fs)
{
    WsLayoutFp8 L{};
    L.ctrl = ws_layout(T, d, 0, E, k, 0);
    const int64_t P = T * k, Ts = fs > 0 ? T : 0;
    L.ld_pairs = (P + 3) & ~int64_t(3);
    L.ld_tokens = (T + 3) & ~int64_t(3);
    size_t o = L.ctrl.ctrl_end;
    L.logits = o; o = align_up(o + (size_t)T * E * 4, 256);
    L.topk_idx = o; o = align_up(o + (size_t)P * 4, 256);
    L.topk_w = o; o = align_up(o + (size_t)P * 4, 256);
    L.counts = o; o = align_up(o + (size_t)E * 4, 256);
    L.offsets = o; o = align_up(o + (size_t)(E + 1) * 4, 256);
    L.perm = o; o = align_up(o + (size_t)P * 4, 256);
    L.inv_perm = o; o = align_up(o + (size_t)P * 4, 256);
    L.x8 = o; o = align_up(o + (size_t)T * d, 1024);
    L.sx = o; o = align_up(o + (size_t)T * (d / 128) * 4, 256);
    L.xp8 = o; o = align_up(o + (size_t)P * d, 1024);
    L.sxp = o; o = align_up(o + (size_t)(d / 128) * L.ld_pairs * 4, 256);
    L.h8 = o; o = align_up(o + (size_t)P * f, 1024);
    L.sh = o; o = align_up(o + (size_t)(f / 128) * L.ld_pairs * 4, 256);
    L.y_p = o; o = align_up(o + (size_t)P * d * 2, 1024);
    L.hs8 = o; o = align_up(o + (size_t)Ts * fs, 1024);
    L.shs = o; o = align_up(o + (size_t)(fs / 128) * (Ts ? L.ld_tokens : 0) * 4, 256);
    L.ys = o; o = align_up(o + (size_t)Ts * d * 2, 1024);
    L.sxT = o; o = align_up(o + (size_t)(d / 128) * (Ts ? L.ld_tokens : 0) * 4, 256);
    L.total = o;
    return L;
}

}  // namespace moe
