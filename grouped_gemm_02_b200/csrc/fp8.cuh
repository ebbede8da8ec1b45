// fp8.cuh -- the FP8 block-scaled expert path (S9): e4m3 quantisers, the e4m3
// row gather, and a persistent grouped GEMM on tcgen05 block-scaled MMAs.
//
// GC-MoE (abstract) runs its expert GEMMs as operand-swapped tcgen05
// block-scaled MMAs with a requantisation step; the workload table fixes e4m3
// codes with 1 x 128 activation blocks and 128 x 128 weight blocks.  Readings:
// a block's scale is the smallest power of two s with amax / s <= 448 (amax =
// 0: s = 1), held to the UE8M0 range 2^-127 .. 2^127 that the MMA takes;
// codes are round-to-nearest-even with saturation to +-448.
//
// Because every scale is a power of two it is exactly a UE8M0 exponent, and
// the MMA (kind::mxf8f6f4.block_scale, one scale per row per 32-wide K
// sub-block, fp32 accumulate) applies it to each product inside the tensor
// core: the TMEM accumulator holds sum_k (a_k s_a)(b_k s_b) over the whole K
// range, the dequantised product the definition asks for, and the epilogue
// reads it once.  A 128 x 128 weight block and a 1 x 128 activation block
// each give one exponent repeated over their four 32-wide sub-blocks.
//
//   gate/up:  h = silu(x W1^T) * (x W3^T) per tile of 128 f rows, then h is
//             requantised in 1 x 128 blocks along f (the tile's 128 f rows are
//             one block) -> h8 [pairs, f] + scales [f/128, pairs]
//   down:     y_p = gate * (h W2^T) -> bf16
//
// One tile = 128 weight rows (W1 and W3 side by side for gate/up: two MMAs
// into two accumulators) x at most 112 tokens, so that two tiles' accumulators
// (2 x (112 + 112) columns) and the scale factors fit the 512 TMEM columns.
// A launch runs the gate/up tiles, the down tiles, or both (FP8_FUSED: the
// down tiles of a block wait, bounded, on a counter its gate/up tiles' epilogue
// warps bump after storing h8 and its scales).
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"
#include "grouped_gemm.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kFp8TileRows = 112;                // most tokens one FP8 tile carries
constexpr PlanShape kPlanFp8{kFp8TileRows, 128, 128, 16, 0};
// the two-launch form: a down tile (one accumulator) spans two units, up to 224 tokens
constexpr PlanShape kPlanFp8Wide{kFp8TileRows, 128, 128, 16, 0, 0, 2};
// CTA-pair tiles (large token counts): up to 224 tokens, 128 f rows (gate/up) or
// 256 d rows (down) per pair; two accumulators of 224 columns and the scale
// factors (8 columns for two token atoms) fit the 512 TMEM columns.
constexpr int kFp8PairTileRows = 224;
// warps 0-5 as in the bf16 GEMM, and warp 6 writes the stages' scale-factor atoms
constexpr int kFp8Threads = 224;
constexpr PlanShape kPlanFp8Pair{kFp8PairTileRows, 128, 256, 32, 1};
constexpr int kFp8BlockK = 128;                  // e4m3 elements per 128-byte swizzle row = one scale block
constexpr int kFp8MaxK = 128 * kFp8BlockK;       // reduction length limit: 4 weight scales per lane of a warp
constexpr uint32_t kFp8TmemCols = 512;
constexpr uint32_t kFp8AccCols = 256;            // accumulator set b at column 256 b: g at +0, u at +112
constexpr uint32_t kSfColA0 = 480;               // scale factors: W1 (or W2) at 480, W3 at 484, tokens at 488
constexpr uint32_t kSfColA1 = 484;
constexpr uint32_t kSfColB = 488;
constexpr int kFp8RingBytes = 204 * 1024;
constexpr uint32_t kSfStageBytes = 2048;         // per stage: 128 token scales (fp32, by TMA) + 3 scale atoms
// pair stage: 256 token scales + this CTA's weight atom + 2 token atoms + 2 FP4
// weight atoms as stored (1 KB aligned, so the next stage's tiles stay 1024-byte aligned)
constexpr uint32_t kSfStageBytesPair = 4096;
// the pair's ring leaves 16 KB for the SwiGLU exchange and the amax halves of both CTAs
constexpr int kFp8PairRingBytes = kFp8RingBytes - 16 * 1024;

// Smallest power-of-two exponent e with amax <= 448 * 2^e (amax > 0), from the
// binary exponent of amax: amax = m * 2^x, m in [0.5, 1), 448 = 0.875 * 2^9;
// held to the UE8M0 range [-127, 127].
__device__ __forceinline__ int fp8_scale_exp(float amax)
{
    if (!(amax > 0.f)) return 0;
    int x;
    const float m = frexpf(amax, &x);
    return max(-127, min(127, m <= 0.875f ? x - 9 : x - 8));
}

// 2^k as fp32 for k in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2f(int k)
{
    return k >= -126 ? __int_as_float((k + 127) << 23) : __int_as_float(0x00400000);
}

// Per-column maximum over the 32 lanes of 16 columns held one per register:
// a butterfly that halves the columns at every step (16 shuffles instead of
// 5 per column).  On return, lanes 2c and 2c + 1 hold column c's maximum in v[0].
__device__ __forceinline__ void warp_colmax16(float (&v)[16], int lane)
{
#pragma unroll
    for (int step = 0; step < 4; step++) {
        const int m = 16 >> step, half = 8 >> step;
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < half; i++) {
            const float keep = upper ? v[i + half] : v[i];
            const float send = upper ? v[i] : v[i + half];
            v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, m));
        }
    }
    v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], 1));
}

// UE8M0 code of a power-of-two fp32 scale in [2^-127, 2^127]: its biased
// exponent (2^-127 is the fp32 subnormal 0x00400000, exponent field 0).
__device__ __forceinline__ uint32_t ue8m0_of(float s)
{
    return (__float_as_uint(s) >> 23) & 0xFFu;
}

__device__ __forceinline__ uint8_t e4m3_of(float v)
{
    return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// ---------------------------------------------------------------- quantisers
// 1 x 128 blocks along rows: one warp per (row, block); lane l holds 4 values.
// scale_t (may be null) also receives the scales K-block-major: scale_t[b * ld_t + r].
__global__ void __launch_bounds__(256) quantize_rows_fp8_kernel(const bf16* __restrict__ src, int64_t R, int C,
                                                                uint8_t* __restrict__ dst, float* __restrict__ scale,
                                                                float* __restrict__ scale_t, int64_t ld_t)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int nb = C / 128;
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= R * nb) return;
    const int64_t r = wid / nb;
    const int b = (int)(wid - r * nb);
    const uint2 raw = *reinterpret_cast<const uint2*>(src + r * C + b * 128 + lane * 4);
    float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u), __uint_as_float(raw.y << 16),
                  __uint_as_float(raw.y & 0xFFFF0000u)};
    float a = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const int e = fp8_scale_exp(a);
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; i++) packed |= (uint32_t)e4m3_of(ldexpf(v[i], -e)) << (8 * i);
    *reinterpret_cast<uint32_t*>(dst + r * C + b * 128 + lane * 4) = packed;
    if (lane == 0) {
        scale[r * nb + b] = ldexpf(1.f, e);
        if (scale_t) scale_t[b * ld_t + r] = ldexpf(1.f, e);
    }
}

// ---------------------------------------------------------------- FP4 weights (e2m1, 1 x 32 blocks)
// Smallest power-of-two exponent e with amax <= 6 * 2^e (amax > 0): amax = m 2^x,
// m in [0.5, 1); held to the UE8M0 range [-127, 127].
__device__ __forceinline__ int fp4_scale_exp(float amax)
{
    if (!(amax > 0.f)) return 0;
    int x;
    const float m = frexpf(amax, &x);
    return max(-127, min(127, m <= 0.75f ? x - 3 : x - 2));
}

// Nearest e2m1 code of v (|v| <= 6 after scaling; larger saturates to 6), ties
// to the even code: the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 are codes 0..7 and
// the thresholds are their midpoints, a midpoint going to the even code.
__device__ __forceinline__ uint32_t e2m1_of(float v)
{
    const float a = fabsf(v);
    const uint32_t c = a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
                     : a <= 2.5f ? 4u : a < 3.5f ? 5u : a <= 5.f ? 6u : 7u;
    return c | (signbit(v) ? 8u : 0u);
}

// Byte offset of row r's scale of 32-wide K sub-block j inside the 512-byte
// scale atom of its 128-row tile and 128-wide K block: row r0 + 32 r1 at byte
// 16 r0 + 4 r1, sub-block j in the byte after that -- the layout the
// block-scaled MMA reads from TMEM after a 32x128b.warpx4 copy.
__host__ __device__ __forceinline__ int sf_atom_byte(int r, int j)
{
    return 16 * (r & 31) + 4 * ((r >> 5) & 3) + j;
}

// 1 x 32 blocks along rows: W [R, C] bf16 -> packed e2m1 codes q [R, C/2]
// (element 2i in the low nibble of byte i) and UE8M0 scale bytes in atoms
// [R/128][C/128][512].  One warp per (row, 128-column block): lane l holds
// columns 4l..4l+3, the 8 lanes of a 32-wide block share its scale.
// R % 128 == 0, C % 128 == 0.
__global__ void __launch_bounds__(256) quantize_rows_fp4_kernel(const bf16* __restrict__ src, int64_t R, int C,
                                                                uint8_t* __restrict__ q, uint8_t* __restrict__ atoms)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int nb = C / 128;
    const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= R * nb) return;
    const int64_t r = wid / nb;
    const int b = (int)(wid - r * nb);
    const uint2 raw = *reinterpret_cast<const uint2*>(src + r * C + b * 128 + lane * 4);
    float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u), __uint_as_float(raw.y << 16),
                  __uint_as_float(raw.y & 0xFFFF0000u)};
    float a = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));   // 8 lanes of a block
    const int e = fp4_scale_exp(a);
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; i++) packed |= e2m1_of(ldexpf(v[i], -e)) << (4 * i);
    *reinterpret_cast<uint16_t*>(q + r * (C / 2) + b * 64 + lane * 2) = (uint16_t)packed;
    if ((lane & 7) == 0) {
        const int64_t tile = (r >> 7) * nb + b;
        atoms[tile * 512 + sf_atom_byte((int)(r & 127), lane >> 3)] = (uint8_t)(e + 127);
    }
}

// 128 x 128 blocks: one CTA of 256 threads per block; thread t covers half of row t/2.
__global__ void __launch_bounds__(256) quantize_blocks_fp8_kernel(const bf16* __restrict__ src, int64_t R, int64_t C,
                                                                  uint8_t* __restrict__ dst,
                                                                  float* __restrict__ scale)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    __shared__ float warp_max[8];
    const int64_t nbc = C / 128;
    const int64_t br = blockIdx.x / nbc, bc = blockIdx.x % nbc;
    const int row = threadIdx.x >> 1, half = threadIdx.x & 1;
    const bf16* p = src + (br * 128 + row) * C + bc * 128 + half * 64;
    float v[64];
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const uint4 raw = reinterpret_cast<const uint4*>(p)[i];
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            a = fmaxf(a, fmaxf(fabsf(v[8 * i + 2 * j]), fabsf(v[8 * i + 2 * j + 1])));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = a;
    __syncthreads();
    a = warp_max[0];
#pragma unroll
    for (int i = 1; i < 8; i++) a = fmaxf(a, warp_max[i]);
    const int e = fp8_scale_exp(a);
    uint8_t* q = dst + (br * 128 + row) * C + bc * 128 + half * 64;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        uint4 o;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            uint32_t w = 0;
#pragma unroll
            for (int b = 0; b < 4; b++) w |= (uint32_t)e4m3_of(ldexpf(v[16 * i + 4 * j + b], -e)) << (8 * b);
            ow[j] = w;
        }
        reinterpret_cast<uint4*>(q)[i] = o;
    }
    if (threadIdx.x == 0) scale[br * nbc + bc] = ldexpf(1.f, e);
}

// xp8[inv_perm[t k + j], :] = x8[t, :] and the row's scales K-block-major,
// sxpT[b * ld + pos] = sx[t, b], for every pair with a valid position: x8[pos] of
// perm[pos] / k, taken in token order so that each x8 row is read once for its k
// copies.  One warp per (token, 512-byte chunk of the row); the chunk-0 warp also
// writes the scales.  Requires d % 128 == 0, k <= 32.
__global__ void __launch_bounds__(256) gather_rows_fp8_kernel(const uint8_t* __restrict__ x8,
                                                              const float* __restrict__ sx,
                                                              const int32_t* __restrict__ inv_perm, int T, int k, int d,
                                                              uint8_t* __restrict__ xp8, float* __restrict__ sxpT,
                                                              int64_t ld)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int nvec = d / 16, nsb = d / 128;
    const int nch = (nvec + 31) / 32;
    const int lane = threadIdx.x & 31;
    const int64_t items = (int64_t)T * nch;
    for (int64_t w = (int64_t)(blockIdx.x * blockDim.x + threadIdx.x) / 32; w < items;
         w += (int64_t)gridDim.x * blockDim.x / 32) {
        const int64_t t = w / nch;
        const int c = (int)(w - t * nch);
        const int v = c * 32 + lane;
        const int mine = lane < k ? inv_perm[t * k + lane] : -1;
        uint4 buf = make_uint4(0u, 0u, 0u, 0u);
        if (v < nvec) buf = __ldg(reinterpret_cast<const uint4*>(x8 + (size_t)t * d) + v);
        for (int j = 0; j < k; j++) {
            const int pos = __shfl_sync(0xffffffffu, mine, j);
            if (pos < 0) continue;
            if (v < nvec) reinterpret_cast<uint4*>(xp8 + (size_t)pos * d)[v] = buf;
            if (c == 0)
                for (int b = lane; b < nsb; b += 32) sxpT[(size_t)b * ld + pos] = sx[(size_t)t * nsb + b];
        }
    }
}


// ---------------------------------------------------------------- FP8 grouped GEMM
struct Fp8Args {
    const int32_t* plan;
    int plan_ready;
    int E;
    int M, M_shared;                // output rows: f (gate/up) or d (down); shared: f_shared or d
    int K, K_shared;                // d (gate/up) or f / f_shared (down)
    const float* sA0;               // weight-block scales of A0 (W1 or W2): [E*M/128, K/128]
    const float* sA1;               // W3 (gate/up)
    const float* sA0s;              // shared expert: Ws1 or Ws2
    const float* sA1s;              // Ws3
    uint8_t* out8;                  // gate/up: h8 [pairs, f]
    float* out8_scale;              // its scales, K-block-major [f/128, ld_scale]
    int ld_scale;
    uint8_t* out8_shared;           // hs8 [T, f_shared]
    float* out8_scale_shared;       // [f_shared/128, ld_scale_shared]
    int ld_scale_shared;
    bf16* out;                      // down: y_p [pairs, d]
    bf16* out_shared;               // ys [T, d]
    const int32_t* perm;
    const float* gate_w;
    uint32_t* err;
    int comp;                       // FP8_FUSED: down tiles per gate/up tile, for the balanced order (cta_tile)
    // FP4 weights (e2m1, 1 x 32 blocks): the scale atoms of A0 / A1 (and the shared
    // expert's), [rows/128][K/128][512 bytes]; the weight-block scales above are unused
    const uint8_t *fA0, *fA1, *fA0s, *fA1s;
};

// What one launch of the FP8 GEMM runs: the down tiles, the gate/up tiles, or
// both (gate/up tiles first; a block's down tiles wait for its h, as in the
// bf16 MODE_FUSED launch).
constexpr int FP8_DOWN = 0;
constexpr int FP8_GATED = 1;
constexpr int FP8_FUSED = 2;

struct Fp8Tile {
    int group, m, row0, rows, n_mma, nkb, blk;
    int b_row0, b_n;   // the token rows this CTA loads: all n_mma, or its half of a pair tile
    bool shared, gated;
};

// Tile t of the launch; in FP8_FUSED the first tiles1 are gate/up tiles
// (prefix sp->tb, args a) and the rest down tiles (prefix sp->tb2, args a2).
// PAIR: a tile of a CTA pair (M = 256), of which this CTA (rank) loads half the
// token rows.  A gate/up pair tile m covers the 128 f rows 128 m .. 128 m + 127
// (rank r: 64 rows of W1 and the same 64 rows of W3 from 128 m + 64 r); a down
// pair tile m covers d rows 256 m .. 256 m + 255 (rank r: 128 of them).
template <int KIND, bool PAIR = false>
__device__ __forceinline__ Fp8Tile fp8_decode(int nb, int t, const Fp8Args& a, const Fp8Args& a2, const SmemPlan* sp,
                                              int rank = 0)
{
    bool gated = KIND == FP8_GATED;
    const int* tb = sp->tb;
    if (KIND == FP8_FUSED) {
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
    const int4 b = sp->blk[lo];
    // a down tile of the two-launch form may span `merge` units of the block
    const int merge = (KIND == FP8_DOWN && !PAIR) ? sp->merge : 1;
    const int units = (sp->units[lo] + merge - 1) / merge;
    const int width = merge * b.w;
    const Fp8Args& ta = (KIND == FP8_FUSED && !gated) ? a2 : a;
    Fp8Tile tl;
    tl.blk = lo;
    tl.gated = gated;
    tl.group = b.x;
    tl.shared = tl.group == ta.E;
    // tile order inside the block: M-tile-major, or unit-major when the block has
    // more token rows than weight rows (as in the bf16 GEMM's decode_tile)
    const int wrows = (gated ? 2 : 1) * (tl.shared ? ta.M_shared : ta.M);
    const int mtiles = (tb[lo + 1] - tb[lo]) / units;
    int u;
    if (b.z > wrows) {
        u = local / mtiles;
        tl.m = local - u * mtiles;
    } else {
        tl.m = local / units;
        u = local - tl.m * units;
    }
    const int start = u * width;
    tl.rows = min(width, b.z - start);
    tl.row0 = b.y + start;
    // a multiple of 16, of 32 for a pair (each CTA loads n/2 rows in 16-row boxes)
    tl.n_mma = sp->fixed_n ? merge * sp->fixed_n : PAIR ? (tl.rows + 31) & ~31 : (tl.rows + 15) & ~15;
    tl.nkb = (tl.shared ? ta.K_shared : ta.K) / kFp8BlockK;
    tl.b_n = PAIR ? tl.n_mma >> 1 : tl.n_mma;
    tl.b_row0 = tl.row0 + rank * tl.b_n;
    return tl;
}

// The i-th tile of this CTA (-1 past the end): round-robin (by cluster for a
// pair: both CTAs take the same tiles), or the balanced gate/up-then-down
// order of the single launch.
template <int KIND, bool PAIR = false>
__device__ __forceinline__ int fp8_cta_tile(int i, int total, const Fp8Args& a, const SmemPlan* sp)
{
    if (PAIR) return deal_tile((int)ptx::cluster_id_x(), (int)ptx::nclusters_x(), i, total, 0, 0, false);
    return KIND == FP8_FUSED ? cta_tile<MODE_FUSED>(i, total, sp->tiles1, a.comp) : cta_tile<MODE_DOWN>(i, total, 0, 0);
}

struct Fp8Iter {
    int i, t, kb;
    Fp8Tile tl;
};

template <int KIND, bool PAIR>
__device__ __forceinline__ bool fp8_iter_seek(Fp8Iter& it, int nb, int total, const Fp8Args& a, const Fp8Args& a2,
                                              const SmemPlan* sp, int rank)
{
    for (; (it.t = fp8_cta_tile<KIND, PAIR>(it.i, total, a, sp)) >= 0; it.i++) {
        it.tl = fp8_decode<KIND, PAIR>(nb, it.t, a, a2, sp, rank);
        if (it.tl.nkb > 0) {
            it.kb = 0;
            return true;
        }
    }
    return false;
}

template <int KIND, bool PAIR>
__device__ __forceinline__ bool fp8_iter_begin(Fp8Iter& it, int nb, int total, const Fp8Args& a, const Fp8Args& a2,
                                               const SmemPlan* sp, int rank)
{
    it.i = 0;
    return fp8_iter_seek<KIND, PAIR>(it, nb, total, a, a2, sp, rank);
}

template <int KIND, bool PAIR>
__device__ __forceinline__ bool fp8_iter_next(Fp8Iter& it, int nb, int total, const Fp8Args& a, const Fp8Args& a2,
                                              const SmemPlan* sp, int rank)
{
    if (++it.kb < it.tl.nkb) return true;
    ++it.i;
    return fp8_iter_seek<KIND, PAIR>(it, nb, total, a, a2, sp, rank);
}

// Instruction descriptor for kind::mxf8f6f4 with block scaling: A and B e4m3
// (format 0, bits 7-9 and 10-12), both K-major, N >> 3 in bits 17-22, scale
// format UE8M0 (bit 23), M >> 4 in bits 24-28, scale-factor byte 0 for A
// (bits 29-30) and B (bits 4-5), dense K = 32.  The accumulator is fp32.
__host__ __device__ constexpr uint32_t idesc_mxf8_ue8m0(uint32_t M, uint32_t N)
{
    return ((N >> 3) << 17) | (1u << 23) | ((M >> 4) << 24);
}

// D[tmem] (+)= (A * 2^sfa) (B * 2^sfb)^T over one 32-wide K step: sfa / sfb
// are the TMEM addresses of the scale-factor columns.
__device__ __forceinline__ void mma_mxf8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa, uint32_t sfb, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// The pair form: M = 256 over the two CTAs of a cluster, issued by the even CTA.
__device__ __forceinline__ void mma_mxf8_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t sfa, uint32_t sfb, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

__device__ __forceinline__ uint32_t pick4(const uint32_t (&v)[4], int i)
{
    return i == 0 ? v[0] : i == 1 ? v[1] : i == 2 ? v[2] : v[3];
}

__device__ __forceinline__ float pick4f(const float (&v)[4], int i)
{
    return i == 0 ? v[0] : i == 1 ? v[1] : i == 2 ? v[2] : v[3];
}

__device__ __forceinline__ float pick8f(const float (&v)[8], int i)
{
    return i == 0 ? v[0] : i == 1 ? v[1] : i == 2 ? v[2] : i == 3 ? v[3] : i == 4 ? v[4] : i == 5 ? v[5]
         : i == 6 ? v[6] : v[7];
}

// Per-column maximum over the 32 lanes of 8 columns held one per register (9
// shuffles): on return lane l holds column (l >> 2) & 7's maximum in v[0].
__device__ __forceinline__ void warp_colmax8(float (&v)[8], int lane)
{
#pragma unroll
    for (int step = 0; step < 3; step++) {
        const int m = 16 >> step, half = 4 >> step;
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < half; i++) {
            const float keep = upper ? v[i + half] : v[i];
            const float send = upper ? v[i] : v[i + half];
            v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, m));
        }
    }
    v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], 2));
    v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], 1));
}

// Persistent grouped GEMM on e4m3 operands with UE8M0 block scales.
//
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer (one thread), warps 2-5
// epilogue, warp 6 scale factors.  A ring stage holds the A tile(s) (128 weight
// rows x 128 K bytes each), the token rows (n x 128 bytes), the tokens' 128
// fp32 scales of that K block (one TMA box starting at row0 rounded down to 4
// tokens, the 16-byte rule for a TMA start) and three 512-byte scale-factor
// atoms.  The operand tiles complete on the stage's `full` barrier, the token
// scales on its `sfull` barrier.  Warp 6 waits for the scales, turns them and
// the tile's weight scales into UE8M0 atoms -- 32 rows of 16 bytes, token
// n = n0 + 32 n1 at byte 16 n0 + 4 n1, its exponent repeated in the four bytes
// of the 32-bit word, one per 32-wide K sub-block -- and arrives on `full`;
// the MMA thread then copies them into TMEM with tcgen05.cp (32x128b, repeated
// over the four lane quadrants) and issues the MMAs, so building a stage's
// atoms overlaps the MMAs of the stages before it.  tcgen05.cp and tcgen05.mma
// from one thread execute in issue order, so one set of scale-factor columns
// serves every K block.
//
// W4: the weights are e2m1 (FP4) with 1 x 32 scales.  The TMA unpacks the
// packed 4-bit rows into the same 128-byte shared-memory rows an e4m3 tile
// takes (tensor-map type 16U4_ALIGN16B), the MMA reads A as e2m1, the weight
// scale atoms come ready-made from global memory by a bulk copy, and the k-th
// 32-wide K step of a block selects scale byte k of the atom's words.
//
// PAIR: clusters of two CTAs run M = 256 tiles (cta_group::2) of up to 224
// tokens, for large token counts; the bytes a stage brings per MMA flop are
// about half the single-CTA tile's.
//   * A gate/up pair tile covers 128 f rows -- one requantisation block of h.
//     Each CTA holds 64 rows of W1 (A rows 0-63) and the same 64 rows of W3
//     (A rows 64-127), so one MMA fills TMEM lanes 0-63 with g and 64-127 with
//     u, and the epilogue warps of quadrants q and q + 2 hand each other half
//     of every 16-column chunk (as in the bf16 GEMM).  A token's amax over the
//     block's 128 rows is the larger of the two CTAs' halves: each epilogue
//     warp writes its per-token maxima into both CTAs' shared memory and
//     arrives on both CTAs' exchange barrier.
//   * A down pair tile covers 256 d rows, 128 per CTA.
//   * Each CTA loads its weight rows and half the token rows; both load all
//     the tile's token scales, since each CTA's TMEM needs the scale factors of
//     every token.  Each CTA's warp 6 writes its own atoms (its weight rows',
//     every token's) and arrives on the leader's full barrier; the leader's
//     MMA thread then copies both CTAs' atoms into their TMEM
//     (tcgen05.cp.cta_group::2 reads each CTA's own shared memory) and issues
//     the MMAs.
template <int KIND, bool W4 = false, bool PAIR = false>
__global__ void __launch_bounds__(kFp8Threads, 1)
    grouped_gemm_fp8_kernel(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mA1,
                            const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mA0s,
                            const __grid_constant__ CUtensorMap mA1s, const __grid_constant__ CUtensorMap mBs,
                            const __grid_constant__ CUtensorMap mSB, const __grid_constant__ CUtensorMap mSBs,
                            const __grid_constant__ CUtensorMap mA2, const __grid_constant__ CUtensorMap mB2,
                            const __grid_constant__ CUtensorMap mA2s, const __grid_constant__ CUtensorMap mB2s,
                            const __grid_constant__ CUtensorMap mSB2, const __grid_constant__ CUtensorMap mSB2s,
                            const __grid_constant__ CUtensorMap mB64, const __grid_constant__ CUtensorMap mBs64,
                            const __grid_constant__ CUtensorMap mB264, const __grid_constant__ CUtensorMap mB2s64,
                            const Fp8Args args, const Fp8Args args2)
{
    // mB64..mB2s64: the token-row maps mB, mBs, mB2, mB2s with 64-row boxes
    // FP8_FUSED: args and mA0..mSBs describe the gate/up tiles (W1/W3, xp8, its
    // scales), args2 and mA2..mSB2s the down tiles (W2, h8, its scales).  The
    // other kinds use args and mA0..mSBs only.  PAIR gate/up: the W1/W3 maps
    // have 64-row boxes.
    static_assert(!(PAIR && KIND == FP8_FUSED), "the single launch runs on single CTAs");
    constexpr int kRows = PAIR ? kFp8PairTileRows : kFp8TileRows;
    // A region of a stage: W1 and W3 tiles of 128 rows (single-CTA gate/up), or 128 weight rows
    constexpr uint32_t kABytes = (KIND != FP8_DOWN && !PAIR) ? 2 * 128 * kFp8BlockK : 128 * kFp8BlockK;
    // tiles of up to 224 tokens: a pair's, and the down GEMM's of the two-launch form
    constexpr bool kWide = PAIR || KIND == FP8_DOWN;
    constexpr uint32_t kSfBytes = kWide ? kSfStageBytesPair : kSfStageBytes;
    constexpr int kRing = PAIR ? kFp8PairRingBytes : kFp8RingBytes;
    // scale-factor region of a stage: token scales (fp32), then the atoms
    constexpr uint32_t kSfScales = kWide ? 1024 : 512;      // bytes of staged token scales
    constexpr uint32_t kAtomA0 = kSfScales;                 // this CTA's weight rows
    constexpr uint32_t kAtomA1 = kAtomA0 + 512;             // single-CTA gate/up: W3
    constexpr uint32_t kAtomB = kWide ? kAtomA0 + 512 : kAtomA1 + 512;   // tokens (two atoms when wide)
    constexpr uint32_t kRawW = kAtomB + 1024;               // PAIR W4 gate/up: the W1 and W3 atoms as stored
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + kFp8RingBytes);
    SmemPlan* splan = reinterpret_cast<SmemPlan*>(smem + kFp8RingBytes + kBarBytes);
    // per-token amax of h from each epilogue warp, two tiles deep: [2][4][kFp8TileRows]
    float* red = reinterpret_cast<float*>(smem + kFp8RingBytes + kBarBytes + sizeof(SmemPlan));
    // PAIR: the SwiGLU exchange of the epilogue warp pairs, and the per-token amax of
    // both CTAs' halves, two gate/up tiles deep: [2 tiles][2 CTAs][2 row quarters][kFp8PairTileRows]
    float* exch = reinterpret_cast<float*>(smem + kFp8PairRingBytes);
    float* red2 = reinterpret_cast<float*>(smem + kFp8PairRingBytes + kExchBytes);
    const uint32_t ring = ptx::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = PAIR ? (int)ptx::cluster_ctarank() : 0;
    const bool leader = rank == 0;

    const bool waited_early = !args.plan_ready;
    if (waited_early) ptx::grid_dep_wait();
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(args.plan);
    // a plan made for wider tiles or the other tile shape: refuse, touch nothing
    // (every CTA sees the same header and leaves before any barrier)
    if (hdr->n_max > kRows || (hdr->pair & 1) != (PAIR ? 1 : 0) || (KIND == FP8_FUSED && hdr->pair != 0)) {
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(args.err, DEVERR_PLAN);
        return;
    }
    const int nb = hdr->n_blocks;
    const int total = KIND == FP8_FUSED ? hdr->tiles1 + hdr->tiles2 : KIND == FP8_GATED ? hdr->tiles1 : hdr->tiles2;
    const int merge = (KIND == FP8_DOWN && !PAIR && (hdr->pair & 2)) ? 2 : 1;
    const int n_max = max(PAIR ? 32 : 16, hdr->n_max);
    const uint32_t b_bytes = (uint32_t)(PAIR ? n_max / 2 : merge * n_max) * kFp8BlockK;   // B region of a stage
    const uint32_t stage_bytes = kABytes + b_bytes + kSfBytes;
    const int stages = min(kMaxStages, (int)(kRing / stage_bytes));
    {
        const PlanArrays pa = plan_arrays(const_cast<int32_t*>(args.plan));
        const int32_t* tbg = KIND == FP8_DOWN ? pa.tb2 : pa.tb1;
        if (threadIdx.x == 0) {
            splan->tiles1 = hdr->tiles1;
            splan->fixed_n = hdr->cls == kPlanClassBucket ? hdr->cap : 0;
            splan->merge = merge;
        }
        for (int i = threadIdx.x; i <= nb; i += blockDim.x) {
            splan->tb[i] = tbg[i];
            if (KIND == FP8_FUSED) splan->tb2[i] = pa.tb2[i];
            if (i < nb) {
                splan->blk[i] = make_int4(pa.group[i], pa.row0[i], pa.rows[i], pa.chunk[i]);
                splan->units[i] = pa.units[i];
            }
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; s++) {
            // the producer's arrival (with the operand bytes) and each CTA's warp 6 (atoms written)
            ptx::mbar_init(ptx::smem_u32(&ctl->full[s]), PAIR ? 3 : 2);
            ptx::mbar_init(ptx::smem_u32(&ctl->empty[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&ctl->sfull[s]), 1);
        }
        for (int a = 0; a < 2; a++) {
            ptx::mbar_init(ptx::smem_u32(&ctl->tfull[a]), 1);
            // the epilogue warps of both CTAs of a pair free the leader's accumulator
            ptx::mbar_init(ptx::smem_u32(&ctl->tempty[a]), PAIR ? 8 : 4);
        }
        // the epilogue warps' per-tile amax exchange (a pair's: both CTAs', two tiles deep)
        ptx::mbar_init(ptx::smem_u32(&ctl->tfull[2]), PAIR ? 8 : 4);
        ptx::mbar_init(ptx::smem_u32(&ctl->tfull[3]), PAIR ? 8 : 4);
        ptx::mbar_init(ptx::smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&mA0);
        ptx::prefetch_tensormap(&mB);
        ptx::prefetch_tensormap(&mSB);
        if (KIND != FP8_DOWN) ptx::prefetch_tensormap(&mA1);
        if (KIND == FP8_FUSED) {
            ptx::prefetch_tensormap(&mA2);
            ptx::prefetch_tensormap(&mB2);
            ptx::prefetch_tensormap(&mSB2);
        }
    }
    if (warp == 1) {
        if (PAIR) {
            ptx::tmem_alloc_pair(ptx::smem_u32(&ctl->tmem_base), kFp8TmemCols);
            ptx::tmem_relinquish_pair();
        } else {
            ptx::tmem_alloc(ptx::smem_u32(&ctl->tmem_base), kFp8TmemCols);
            ptx::tmem_relinquish();
        }
    }
    ptx::tc_fence_before();
    // a pair's barriers are signalled across the two CTAs: both must be initialised first
    if (PAIR) ptx::cluster_sync();
    else __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    // a barrier of the leader (rank 0) as this CTA addresses it
    auto leader_bar = [&](uint64_t* bar) -> uint32_t {
        return PAIR ? ptx::mapa_shared(ptx::smem_u32(bar), 0) : ptx::smem_u32(bar);
    };
    // the barrier this CTA's own scale (and FP4 weight-atom) loads complete on
    auto own_bar = [&](int s) -> uint32_t { return ptx::smem_u32(&ctl->sfull[s]); };
    // the bytes of the stage's weight atoms loaded from global memory (FP4 weights)
    auto w_atom_bytes = [&](const Fp8Tile& tl) -> uint32_t {
        return W4 ? (tl.gated ? 1024u : 512u) : 0u;
    };
    // a 128-row weight tile of this CTA, held to the group's last tile (a pair's
    // second CTA past the end of d reads real scales and discards the rows)
    auto w_tile = [&](const Fp8Tile& tl, int Mrows) -> int {
        return PAIR && !tl.gated ? min(2 * tl.m + rank, Mrows / 128 - 1) : tl.m;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (ptx::elect_one()) {
            const uint64_t pol = ptx::policy_evict_normal();
            uint32_t armed = 0, armed_ph = 0;
            bool ok = true;
            // Bytes of a stage on `full` (single CTA or pair leader): the weight tiles
            // and token rows (of both CTAs for a pair); and on this CTA's `sfull`: its
            // token scales and FP4 weight atoms.  An FP4 weight box counts its packed
            // global bytes (4 bits an element), though it fills the 128-byte
            // shared-memory rows of an e4m3 box.
            auto full_tx = [&](const Fp8Tile& tl) -> uint32_t {
                const uint32_t wbox = 128u * kFp8BlockK / (W4 ? 2u : 1u);
                if (!PAIR) return (tl.gated ? 2u : 1u) * wbox + (uint32_t)tl.n_mma * kFp8BlockK;
                return 2u * (wbox + (uint32_t)tl.b_n * kFp8BlockK);
            };
            auto sf_tx = [&](const Fp8Tile& tl) -> uint32_t { return kSfScales + w_atom_bytes(tl); };
            // arm a stage: this CTA's scale barrier, and the operand barrier (not a pair's second CTA)
            auto arm = [&](const Fp8Tile& tl, int s) {
                ptx::mbar_arrive_expect_tx(ptx::smem_u32(&ctl->sfull[s]), sf_tx(tl));
                if (leader) ptx::mbar_arrive_expect_tx(ptx::smem_u32(&ctl->full[s]), full_tx(tl));
            };
            // the down tiles of the single launch read the second set of maps and args
            auto down2 = [&](const Fp8Tile& tl) { return KIND == FP8_FUSED && !tl.gated; };
            auto issue_a = [&](const Fp8Tile& tl, int kb, uint32_t a_dst, int s) {
                const int kc = kb * kFp8BlockK;
                const Fp8Args& ta = down2(tl) ? args2 : args;
                const int Mrows = tl.shared ? ta.M_shared : ta.M;
                const int base = tl.shared ? 0 : tl.group * Mrows;
                const uint32_t sf = a_dst + kABytes + b_bytes;
                if (PAIR) {
                    const uint32_t full = leader_bar(&ctl->full[s]);
                    if (tl.gated) {
                        // 64 rows of W1 into A rows 0-63, the same rows of W3 into 64-127
                        const int a_row = base + tl.m * 128 + 64 * rank;
                        ptx::tma_load_2d_pair(a_dst, tl.shared ? &mA0s : &mA0, full, kc, a_row, pol);
                        ptx::tma_load_2d_pair(a_dst + 64 * kFp8BlockK, tl.shared ? &mA1s : &mA1, full, kc, a_row, pol);
                        if (W4) {
                            // the W1 and W3 atoms of the block's 128 rows; the MMA warp takes this CTA's half
                            const int64_t atom = ((int64_t)(base / 128 + tl.m) * tl.nkb + kb) * 512;
                            ptx::bulk_load(sf + kRawW, (tl.shared ? ta.fA0s : ta.fA0) + atom, 512, own_bar(s));
                            ptx::bulk_load(sf + kRawW + 512, (tl.shared ? ta.fA1s : ta.fA1) + atom, 512, own_bar(s));
                        }
                    } else {
                        const int a_row = base + (2 * tl.m + rank) * 128;
                        ptx::tma_load_2d_pair(a_dst, tl.shared ? &mA0s : &mA0, full, kc, a_row, pol);
                        if (W4) {
                            const int64_t atom = ((int64_t)(base / 128 + w_tile(tl, Mrows)) * tl.nkb + kb) * 512;
                            ptx::bulk_load(sf + kAtomA0, (tl.shared ? ta.fA0s : ta.fA0) + atom, 512, own_bar(s));
                        }
                    }
                    return;
                }
                const uint32_t full = ptx::smem_u32(&ctl->full[s]);
                const int a_row = base + tl.m * 128;
                const CUtensorMap* a0 = down2(tl) ? (tl.shared ? &mA2s : &mA2) : (tl.shared ? &mA0s : &mA0);
                ptx::tma_load_2d(a_dst, a0, full, kc, a_row, pol);
                if (tl.gated) ptx::tma_load_2d(a_dst + 128 * kFp8BlockK, tl.shared ? &mA1s : &mA1, full, kc, a_row, pol);
                if (W4) {
                    // the weight tiles' scale atoms, into the stage's A0 / A1 atom slots
                    const int64_t atom = ((int64_t)(a_row >> 7) * tl.nkb + kb) * 512;
                    ptx::bulk_load(sf + kAtomA0, (tl.shared ? ta.fA0s : ta.fA0) + atom, 512, own_bar(s));
                    if (tl.gated) ptx::bulk_load(sf + kAtomA1, (tl.shared ? ta.fA1s : ta.fA1) + atom, 512, own_bar(s));
                }
            };
            auto issue_b = [&](const Fp8Tile& tl, int kb, uint32_t stage, int s) {
                const int kc = kb * kFp8BlockK;
                const uint32_t b_dst = stage + kABytes;
                const CUtensorMap* bm = down2(tl) ? (tl.shared ? &mB2s : &mB2) : (tl.shared ? &mBs : &mB);
                const CUtensorMap* bm64 = down2(tl) ? (tl.shared ? &mB2s64 : &mB264) : (tl.shared ? &mBs64 : &mB64);
                const CUtensorMap* sm = down2(tl) ? (tl.shared ? &mSB2s : &mSB2) : (tl.shared ? &mSBs : &mSB);
                const uint32_t full = PAIR ? leader_bar(&ctl->full[s]) : ptx::smem_u32(&ctl->full[s]);
                // token rows in 64-row boxes, then 16-row boxes (fewer TMA requests)
                const int n64 = tl.b_n >> 6;
                for (int i = 0; i < n64; i++) {
                    if (PAIR) ptx::tma_load_2d_pair(b_dst + i * 64 * kFp8BlockK, bm64, full, kc, tl.b_row0 + 64 * i, pol);
                    else ptx::tma_load_2d(b_dst + i * 64 * kFp8BlockK, bm64, full, kc, tl.b_row0 + 64 * i, pol);
                }
                for (int r = 64 * n64; r < tl.b_n; r += 16) {
                    if (PAIR) ptx::tma_load_2d_pair(b_dst + r * kFp8BlockK, bm, full, kc, tl.b_row0 + r, pol);
                    else ptx::tma_load_2d(b_dst + r * kFp8BlockK, bm, full, kc, tl.b_row0 + r, pol);
                }
                // the tokens' scales of this K block: 128 fp32 (256 for a pair, every
                // token of the tile) from row0 rounded down to 4, into this CTA
                const uint32_t sf = b_dst + b_bytes;
                ptx::tma_load_2d(sf, sm, own_bar(s), tl.row0 & ~3, kb, pol);
                if (kWide) ptx::tma_load_2d(sf + 512, sm, own_bar(s), (tl.row0 & ~3) + 128, kb, pol);
            };
            // FP8_FUSED: a down tile reads h8 and its scales only after every gate/up
            // tile of its block has published them (4 epilogue warps per tile)
            auto wait_block_ready = [&](const Fp8Tile& tl) -> bool {
                const int32_t* dep = plan_arrays(const_cast<int32_t*>(args.plan)).dep + tl.blk;
                const int m1 = tl.shared ? args.M_shared : args.M;
                const int need = 4 * splan->units[tl.blk] * ((m1 + 127) / 128);
                if (!bounded_count_wait(dep, need, ctl, args.err)) return false;
                ptx::fence_proxy_async_global();   // the TMA reads below come after the acquire
                return true;
            };
            int pre = 0;
            if (!waited_early) {
                Fp8Iter it;
                bool more = fp8_iter_begin<KIND, PAIR>(it, nb, total, args, args2, splan, rank);
                while (more && pre < stages) {
                    arm(it.tl, pre);
                    armed |= 1u << pre;
                    issue_a(it.tl, it.kb, ring + (uint32_t)pre * stage_bytes, pre);
                    ++pre;
                    more = fp8_iter_next<KIND, PAIR>(it, nb, total, args, args2, splan, rank);
                }
                ptx::grid_dep_wait();
            }
            // After the wait, never before it: the layer's later kernels read data
            // written two launches back (the combine reads inv_perm before its own
            // wait), which holds only if every kernel waits before it triggers.
            ptx::grid_dep_launch();
            int s = 0, n = 0;
            uint32_t ph = 0;
            Fp8Iter it;
            bool more = fp8_iter_begin<KIND, PAIR>(it, nb, total, args, args2, splan, rank);
            while (more) {
                const uint32_t stage = ring + (uint32_t)s * stage_bytes;
                if (n >= pre) {
                    if (!bounded_wait(ptx::smem_u32(&ctl->empty[s]), ph ^ 1u, ctl, args.err)) {
                        ok = false;
                        break;
                    }
                    arm(it.tl, s);
                    armed |= 1u << s;
                    armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                    issue_a(it.tl, it.kb, stage, s);
                }
                if (KIND == FP8_FUSED && !it.tl.gated && it.kb == 0 && !wait_block_ready(it.tl)) {
                    ok = false;
                    break;
                }
                issue_b(it.tl, it.kb, stage, s);
                ++n;
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
                more = fp8_iter_next<KIND, PAIR>(it, nb, total, args, args2, splan, rank);
            }
            if (!ok) {
                // drain: wait (bounded) for every stage this CTA armed: its scale loads,
                // and the operand loads of both CTAs of a pair, which count on the
                // leader's barrier (the other CTA does not leave before the leader:
                // cluster barrier below).  `full` also waits for the atoms, so a stage
                // whose atoms never came ends the wait at the deadline.
                const uint64_t t0 = ptx::globaltimer();
                for (int i = 0; i < stages; i++) {
                    if (!(armed >> i & 1u)) continue;
                    const uint32_t par = (armed_ph >> i) & 1u;
                    while (!ptx::mbar_try_wait(own_bar(i), par) && ptx::globaltimer() - t0 < kWaitTimeoutNs) {
                    }
                    while (leader && !ptx::mbar_try_wait(ptx::smem_u32(&ctl->full[i]), par) &&
                           ptx::globaltimer() - t0 < kWaitTimeoutNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (one thread; a pair's leader)
        if ((!PAIR || leader) && ptx::elect_one()) {
            int s = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true, issued = false;
            for (int ti = 0, t; ok && (t = fp8_cta_tile<KIND, PAIR>(ti, total, args, splan)) >= 0; ti++) {
                const Fp8Tile tl = fp8_decode<KIND, PAIR>(nb, t, args, args2, splan, rank);
                if (tl.nkb <= 0) continue;
                if (!bounded_wait(ptx::smem_u32(&ctl->tempty[acc]), aph ^ 1u, ctl, args.err)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_g = tmem_base + (uint32_t)acc * kFp8AccCols;
                // A as e2m1 (format 5, bits 7-9) for FP4 weights
                const uint32_t idesc = idesc_mxf8_ue8m0(PAIR ? 256 : 128, (uint32_t)tl.n_mma) | (W4 ? (5u << 7) : 0u);
                for (int kb = 0; kb < tl.nkb; kb++) {
                    // the operand tiles and every CTA's atoms of the stage are in place
                    if (!(PAIR ? bounded_wait<true>(ptx::smem_u32(&ctl->full[s]), ph, ctl, args.err)
                               : bounded_wait(ptx::smem_u32(&ctl->full[s]), ph, ctl, args.err))) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ring + (uint32_t)s * stage_bytes;
                    const uint32_t b_addr = a_addr + kABytes;
                    const uint32_t atoms = b_addr + b_bytes;
                    // FP4 weights: the kk-th 32-wide K step reads scale byte kk of A's atom (bits 29-30)
                    if (PAIR) {
                        ptx::tmem_cp_32x128b_warpx4_pair(tmem_base + kSfColA0, ptx::plain_rows16_desc(atoms + kAtomA0));
                        ptx::tmem_cp_32x128b_warpx4_pair(tmem_base + kSfColB, ptx::plain_rows16_desc(atoms + kAtomB));
                        if (tl.n_mma > 128)
                            ptx::tmem_cp_32x128b_warpx4_pair(tmem_base + kSfColB + 4,
                                                             ptx::plain_rows16_desc(atoms + kAtomB + 512));
#pragma unroll
                        for (int kk = 0; kk < kFp8BlockK / 32; kk++)
                            mma_mxf8_ss_pair(d_g, ptx::sw128_kmajor_desc(a_addr + kk * 32),
                                             ptx::sw128_kmajor_desc(b_addr + kk * 32),
                                             idesc | (W4 ? (uint32_t)kk << 29 : 0u), tmem_base + kSfColA0,
                                             tmem_base + kSfColB, (kb > 0 || kk > 0) ? 1u : 0u);
                        // the stage is free in both CTAs once these MMAs have read it
                        ptx::mma_commit_pair(ptx::smem_u32(&ctl->empty[s]), 3);
                    } else {
                        ptx::tmem_cp_32x128b_warpx4(tmem_base + kSfColA0, ptx::plain_rows16_desc(atoms + kAtomA0));
                        if (tl.gated)
                            ptx::tmem_cp_32x128b_warpx4(tmem_base + kSfColA1, ptx::plain_rows16_desc(atoms + kAtomA1));
                        ptx::tmem_cp_32x128b_warpx4(tmem_base + kSfColB, ptx::plain_rows16_desc(atoms + kAtomB));
                        if (kWide && tl.n_mma > 128)
                            ptx::tmem_cp_32x128b_warpx4(tmem_base + kSfColB + 4, ptx::plain_rows16_desc(atoms + kAtomB + 512));
#pragma unroll
                        for (int kk = 0; kk < kFp8BlockK / 32; kk++)
                            mma_mxf8_ss(d_g, ptx::sw128_kmajor_desc(a_addr + kk * 32),
                                        ptx::sw128_kmajor_desc(b_addr + kk * 32),
                                        idesc | (W4 ? (uint32_t)kk << 29 : 0u), tmem_base + kSfColA0,
                                        tmem_base + kSfColB, (kb > 0 || kk > 0) ? 1u : 0u);
                        if (tl.gated) {
#pragma unroll
                            for (int kk = 0; kk < kFp8BlockK / 32; kk++)
                                mma_mxf8_ss(d_g + (uint32_t)kFp8TileRows,
                                            ptx::sw128_kmajor_desc(a_addr + 128 * kFp8BlockK + kk * 32),
                                            ptx::sw128_kmajor_desc(b_addr + kk * 32),
                                            idesc | (W4 ? (uint32_t)kk << 29 : 0u), tmem_base + kSfColA1,
                                            tmem_base + kSfColB, (kb > 0 || kk > 0) ? 1u : 0u);
                        }
                        ptx::mma_commit(ptx::smem_u32(&ctl->empty[s]));
                    }
                    issued = true;
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
                // drain: every tcgen05 op issued so far completes before TMEM is freed
                if (PAIR) ptx::mma_commit_pair(ptx::smem_u32(&ctl->drain), 1);
                else ptx::mma_commit(ptx::smem_u32(&ctl->drain));
                const uint64_t t0 = ptx::globaltimer();
                while (!ptx::mbar_try_wait(ptx::smem_u32(&ctl->drain), 0) && ptx::globaltimer() - t0 < kWaitTimeoutNs) {
                }
            }
        }
    } else if (warp == 6) {
        // ------------------------------------------------------------ scale-factor atoms (whole warp)
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        // The weight-block scales of a tile (lane l: K blocks l, l + 32, l + 64, l + 96)
        // are loaded one tile ahead, so their latency hides behind the previous tile.
        auto load_scales = [&](int t, float (&wa)[4], float (&wb)[4]) {
            if (t < 0 || W4) return;   // FP4 weights: the atoms come with the stage
            const Fp8Tile tl = fp8_decode<KIND, PAIR>(nb, t, args, args2, splan, rank);
            const Fp8Args& ta = (KIND == FP8_FUSED && !tl.gated) ? args2 : args;
            const int Mrows = tl.shared ? ta.M_shared : ta.M;
            const int64_t srow = (int64_t)(tl.shared ? 0 : tl.group * (Mrows / 128)) + w_tile(tl, Mrows);
            const float* sA0 = (tl.shared ? ta.sA0s : ta.sA0) + srow * tl.nkb;
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const int kb = 32 * i + lane;
                wa[i] = kb < tl.nkb ? __ldg(sA0 + kb) : 1.f;
            }
            if (tl.gated) {
                const float* sA1 = (tl.shared ? args.sA1s : args.sA1) + srow * tl.nkb;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int kb = 32 * i + lane;
                    wb[i] = kb < tl.nkb ? __ldg(sA1 + kb) : 1.f;
                }
            }
        };
        float nwa[4] = {1.f, 1.f, 1.f, 1.f}, nwb[4] = {1.f, 1.f, 1.f, 1.f};
        int ti = 0;
        int t = fp8_cta_tile<KIND, PAIR>(ti, total, args, splan);
        load_scales(t, nwa, nwb);
        while (t >= 0 && ok) {
            const Fp8Tile tl = fp8_decode<KIND, PAIR>(nb, t, args, args2, splan, rank);
            uint32_t ea[4], eb[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                ea[i] = __float_as_uint(nwa[i]);
                eb[i] = __float_as_uint(nwb[i]);
            }
            const int t_next = fp8_cta_tile<KIND, PAIR>(++ti, total, args, splan);
            load_scales(t_next, nwa, nwb);
            const int shift = tl.row0 & 3;
            for (int kb = 0; kb < tl.nkb; kb++) {
                // this CTA's token scales (and FP4 weight atoms) of the stage have landed
                ok = __all_sync(0xffffffffu, bounded_wait(ptx::smem_u32(&ctl->sfull[s]), ph, ctl, args.err));
                if (!ok) break;
                uint8_t* sfp = smem + (size_t)s * stage_bytes + kABytes + b_bytes;
                const float* staged = reinterpret_cast<const float*>(sfp);
                // the tokens' atoms: token c = 128 q + lane + 32 m1 at byte 16 lane + 4 m1 of atom q
#pragma unroll
                for (int q = 0; q < (kWide ? 2 : 1); q++) {
                    uint32_t w[4];
#pragma unroll
                    for (int m1 = 0; m1 < 4; m1++) {
                        const int c = 128 * q + lane + 32 * m1;
                        const uint32_t e = c < tl.rows ? ue8m0_of(staged[shift + c]) : 127u;
                        w[m1] = e * 0x01010101u;
                    }
                    *reinterpret_cast<uint4*>(sfp + kAtomB + 512 * q + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
                }
                // the weight rows' atoms
                if (!W4) {
                    const uint32_t a0 =
                        ue8m0_of(__uint_as_float(__shfl_sync(0xffffffffu, pick4(ea, kb >> 5), kb & 31))) * 0x01010101u;
                    const uint32_t a1 =
                        tl.gated ? ue8m0_of(__uint_as_float(__shfl_sync(0xffffffffu, pick4(eb, kb >> 5), kb & 31))) *
                                       0x01010101u
                                 : a0;
                    if (PAIR) {
                        // A rows 0-63 are W1's (words 0, 1 of a line), 64-127 W3's (words 2, 3)
                        *reinterpret_cast<uint4*>(sfp + kAtomA0 + 16 * lane) = make_uint4(a0, a0, a1, a1);
                    } else {
                        *reinterpret_cast<uint4*>(sfp + kAtomA0 + 16 * lane) = make_uint4(a0, a0, a0, a0);
                        if (tl.gated) *reinterpret_cast<uint4*>(sfp + kAtomA1 + 16 * lane) = make_uint4(a1, a1, a1, a1);
                    }
                } else if (PAIR && tl.gated) {
                    // this CTA's rows of the W1 and W3 atoms: words 2 rank and 2 rank + 1 of each line
                    const uint2 w1 = *reinterpret_cast<const uint2*>(sfp + kRawW + 16 * lane + 8 * rank);
                    const uint2 w3 = *reinterpret_cast<const uint2*>(sfp + kRawW + 512 + 16 * lane + 8 * rank);
                    *reinterpret_cast<uint4*>(sfp + kAtomA0 + 16 * lane) = make_uint4(w1.x, w1.y, w3.x, w3.y);
                }
                ptx::fence_proxy_async_smem();   // the atoms are read by tcgen05.cp (async proxy)
                __syncwarp();
                if (lane == 0) {
                    // this CTA's atoms of the stage are in place (on the leader's barrier for a pair)
                    if (PAIR) ptx::mbar_arrive_cluster(leader_bar(&ctl->full[s]));
                    else ptx::mbar_arrive(ptx::smem_u32(&ctl->full[s]));
                }
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            t = t_next;
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2-5)
        const int quad = warp & 3;
        int acc = 0, gcount = 0;   // gcount: gate/up tiles so far (their amax buffers alternate)
        uint32_t aph = 0, xph = 0;   // xph: phase bits of the amax exchange barrier(s)
        uint32_t xchunk = 0;         // PAIR: SwiGLU exchange chunks so far (the buffer alternates)
        for (int ti = 0, t; (t = fp8_cta_tile<KIND, PAIR>(ti, total, args, splan)) >= 0; ti++) {
            const Fp8Tile tl = fp8_decode<KIND, PAIR>(nb, t, args, args2, splan, rank);
            if (tl.nkb <= 0) continue;
            const Fp8Args& ea = (KIND == FP8_FUSED && !tl.gated) ? args2 : args;
            // down: the tile's gates (lane l: columns l + 32 i), fetched before the wait
            float gates[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
            if (!tl.gated && !tl.shared) {
#pragma unroll
                for (int i = 0; i < (kWide ? 8 : 4); i++) {
                    const int col = 32 * i + lane;
                    if (col < tl.rows) gates[i] = __ldg(ea.gate_w + __ldg(ea.perm + tl.row0 + col));
                }
            }
            if (!__all_sync(0xffffffffu, bounded_wait(ptx::smem_u32(&ctl->tfull[acc]), aph, ctl, args.err))) break;
            ptx::tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t)acc * kFp8AccCols + ((uint32_t)(quad * 32) << 16);
            const int Mrows = tl.shared ? ea.M_shared : ea.M;
            bool ok = true;
            if (tl.gated && PAIR) {
                // TMEM lanes 0-63: g, 64-127: u of f rows 128 m + 64 rank + (lane % 64)
                const int role = quad >> 1, rq = quad & 1;
                const int frow = tl.m * 128 + 64 * rank + rq * 32 + lane;
                const int par = gcount++ & 1;
                float* rb = red2 + par * (4 * kFp8PairTileRows);   // [CTA][row quarter][token]
                const uint32_t peer_rb = ptx::mapa_shared(ptx::smem_u32(rb), (uint32_t)(rank ^ 1));
                // pass 1: h = silu(g) u for 8 of every 16 columns, written back to this
                // warp's own TMEM lanes, and per token the largest |h| of its 32 rows
                for (int c0 = 0; c0 < tl.n_mma; c0 += 16) {
                    uint32_t v[16];
                    ptx::tmem_ld16(taddr + (uint32_t)c0, v);
                    ptx::tmem_ld_wait();
                    float* xb = exch + (rq * 2 + (xchunk++ & 1u)) * 512;
                    float* mine = xb + role * 256;
                    const float* theirs = xb + (role ^ 1) * 256;
#pragma unroll
                    for (int j = 0; j < 8; j++) mine[j * 32 + lane] = __uint_as_float(v[role ? j : 8 + j]);
                    ptx::named_barrier(1 + rq, 64);
                    uint32_t hb[8];
                    float a[8];
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        const float other = theirs[j * 32 + lane];
                        const float g = role ? other : __uint_as_float(v[j]);
                        const float u = role ? __uint_as_float(v[8 + j]) : other;
                        const float h = silu_f(g) * u;
                        hb[j] = __float_as_uint(h);
                        a[j] = frow < Mrows ? fabsf(h) : 0.f;
                    }
                    ptx::tmem_st8(taddr + (uint32_t)(c0 + role * 8), hb);
                    warp_colmax8(a, lane);
                    if ((lane & 3) == 0) {
                        const int idx = (rank * 2 + rq) * kFp8PairTileRows + c0 + role * 8 + ((lane >> 2) & 7);
                        rb[idx] = a[0];
                        ptx::st_cluster_f32(peer_rb + 4u * (uint32_t)idx, a[0]);
                    }
                }
                ptx::tmem_st_wait();
                // both CTAs' eight epilogue warps meet (bounded) on each CTA's exchange barrier
                __syncwarp();
                uint64_t* xbar = &ctl->tfull[2 + par];
                if (lane == 0) {
                    ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(xbar), (uint32_t)rank));
                    ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(xbar), (uint32_t)(rank ^ 1)));
                }
                ok = __all_sync(0xffffffffu, bounded_wait<true>(ptx::smem_u32(xbar), (xph >> par) & 1u, ctl, args.err));
                xph ^= 1u << par;
                if (ok) {
                    // pass 2: scale, encode and store this warp's 8 of every 16 columns
                    uint8_t* out8 = tl.shared ? args.out8_shared : args.out8;
                    float* osc = tl.shared ? args.out8_scale_shared : args.out8_scale;
                    const int lds = tl.shared ? args.ld_scale_shared : args.ld_scale;
                    for (int c0 = 0; c0 < tl.n_mma; c0 += 16) {
                        uint32_t h[8];
                        ptx::tmem_ld8(taddr + (uint32_t)(c0 + role * 8), h);
                        // lane j < 8: the block scale 2^e of token c0 + 8 role + j
                        const int mc = c0 + role * 8 + (lane & 7);
                        const float amax = fmaxf(fmaxf(rb[mc], rb[kFp8PairTileRows + mc]),
                                                 fmaxf(rb[2 * kFp8PairTileRows + mc], rb[3 * kFp8PairTileRows + mc]));
                        const int e = fp8_scale_exp(amax);
                        const float inv = pow2f(-e);
                        if (rank == 0 && rq == 0 && lane < 8 && mc < tl.rows)
                            osc[(int64_t)tl.m * lds + tl.row0 + mc] = pow2f(e);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 8; j++) {
                            const float m = __shfl_sync(0xffffffffu, inv, j);
                            const int col = c0 + role * 8 + j;
                            if (col < tl.rows && frow < Mrows)
                                out8[(int64_t)(tl.row0 + col) * Mrows + frow] = e4m3_of(__uint_as_float(h[j]) * m);
                        }
                    }
                }
            } else if (tl.gated) {
                const int mrow = tl.m * 128 + quad * 32 + lane;   // weight row of this thread (TMEM lane)
                float* rb = red + (gcount++ & 1) * 4 * kFp8TileRows;
                // pass 1: h = silu(g) * u, written back over g in TMEM, and per token
                // the largest |h| over this warp's 32 f rows
                for (int c0 = 0; c0 < tl.n_mma; c0 += 16) {
                    uint32_t g[16], u[16];
                    ptx::tmem_ld16(taddr + (uint32_t)c0, g);
                    ptx::tmem_ld16(taddr + (uint32_t)kFp8TileRows + (uint32_t)c0, u);
                    ptx::tmem_ld_wait();
                    float a[16];
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const float h = silu_f(__uint_as_float(g[j])) * __uint_as_float(u[j]);
                        g[j] = __float_as_uint(h);
                        a[j] = mrow < Mrows ? fabsf(h) : 0.f;
                    }
                    ptx::tmem_st16(taddr + (uint32_t)c0, g);
                    warp_colmax16(a, lane);
                    if ((lane & 1) == 0) rb[quad * kFp8TileRows + c0 + (lane >> 1)] = a[0];
                }
                ptx::tmem_st_wait();
                // exchange among the four epilogue warps (bounded; a warp that gives up stops the others)
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&ctl->tfull[2]));
                ok = __all_sync(0xffffffffu, bounded_wait(ptx::smem_u32(&ctl->tfull[2]), xph, ctl, args.err));
                xph ^= 1u;
                if (ok) {
                    // pass 2: each token's 128 h values of this tile are one block: scale, encode, store
                    uint8_t* out8 = tl.shared ? args.out8_shared : args.out8;
                    float* osc = tl.shared ? args.out8_scale_shared : args.out8_scale;
                    const int lds = tl.shared ? args.ld_scale_shared : args.ld_scale;
                    for (int c0 = 0; c0 < tl.n_mma; c0 += 16) {
                        uint32_t h[16];
                        ptx::tmem_ld16(taddr + (uint32_t)c0, h);
                        // lane j < 16: the block scale 2^e of token c0 + j
                        const int mc = c0 + (lane & 15);
                        const float amax = fmaxf(fmaxf(rb[mc], rb[kFp8TileRows + mc]),
                                                 fmaxf(rb[2 * kFp8TileRows + mc], rb[3 * kFp8TileRows + mc]));
                        const int e = fp8_scale_exp(amax);
                        const float inv = pow2f(-e);
                        if (quad == 0 && lane < 16 && mc < tl.rows) osc[(int64_t)tl.m * lds + tl.row0 + mc] = pow2f(e);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; j++) {
                            const float m = __shfl_sync(0xffffffffu, inv, j);
                            const int col = c0 + j;
                            if (col < tl.rows && mrow < Mrows)
                                out8[(int64_t)(tl.row0 + col) * Mrows + mrow] = e4m3_of(__uint_as_float(h[j]) * m);
                        }
                    }
                }
            } else {
                bf16* out = tl.shared ? ea.out_shared : ea.out;
                const int mrow = (PAIR ? (2 * tl.m + rank) : tl.m) * 128 + quad * 32 + lane;
                for (int c0 = 0; c0 < tl.n_mma; c0 += 16) {
                    uint32_t v[16];
                    ptx::tmem_ld16(taddr + (uint32_t)c0, v);
                    ptx::tmem_ld_wait();
                    const float mine = pick8f(gates, c0 >> 5);
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const float gate = __shfl_sync(0xffffffffu, mine, (c0 & 31) + j);
                        const int col = c0 + j;
                        if (col < tl.rows && mrow < Mrows)
                            out[(int64_t)(tl.row0 + col) * Mrows + mrow] = __float2bfloat16_rn(__uint_as_float(v[j]) * gate);
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
            if (!ok) break;
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
            if (KIND == FP8_FUSED && tl.gated) {
                // publish this warp's h8 rows and scales of the tile to the down tiles of
                // its block: each of the 4 epilogue warps adds 1 after its own stores
                ptx::fence_proxy_async_global();
                __syncwarp();
                if (lane == 0) ptx::red_add_release_gpu(plan_arrays(const_cast<int32_t*>(args.plan)).dep + tl.blk, 1);
            }
        }
    }

    ptx::tc_fence_before();
    // neither CTA of a pair leaves (or frees TMEM) while the other may still
    // signal its barriers, write its shared memory, or the leader's MMAs its TMEM
    if (PAIR) ptx::cluster_sync();
    else __syncthreads();
    __syncwarp();   // the dealloc below is .sync.aligned: warp 1 converged
    if (warp == 1) {
        ptx::tc_fence_after();
        if (PAIR) ptx::tmem_dealloc_pair(tmem_base, kFp8TmemCols);
        else ptx::tmem_dealloc(tmem_base, kFp8TmemCols);
    }
}

constexpr int kFp8SmemBytes = 1024 + kFp8RingBytes + kBarBytes + (int)sizeof(SmemPlan) + 2 * 4 * kFp8TileRows * 4;
static_assert(kFp8SmemBytes <= 227 * 1024, "shared memory budget (fp8)");
static_assert(kExchBytes + 2 * 2 * 2 * kFp8PairTileRows * 4 <= kFp8RingBytes - kFp8PairRingBytes,
              "pair exchange buffers (fp8)");

}  // namespace moe
