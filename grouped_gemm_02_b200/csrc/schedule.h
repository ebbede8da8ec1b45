// schedule.h -- the order in which the persistent grouped-GEMM CTAs take their
// tiles (the deal of the skew-aware scheduler).  Plain integer arithmetic,
// compiled for the device by the kernels and for the host by the CPU tests,
// so the test checks the very function the kernels run.
#pragma once

#if defined(__CUDACC__)
#define MOE_HD __host__ __device__ __forceinline__
#else
#define MOE_HD inline
#endif

namespace moe {

// The i-th tile taken by CTA b of a grid of `grid` CTAs, or -1 when it has no
// more.  Tiles 0..G-1 are gate/up tiles and G..total-1 down tiles.
//
// Round-robin deal (balanced == false): CTA b takes b, b + grid, b + 2 grid...
//
// Balanced deal (balanced == true, the single launch of both expert GEMMs):
// the G gate/up tiles are dealt round-robin; when G is not a multiple of the
// grid, the CTAs left one gate/up tile short first take `comp` down tiles each
// (a gate/up tile weighs about `comp` down tiles), then the remaining down tiles
// are dealt round-robin.  The compensating tiles are the first down tiles,
// whose blocks' gate/up tiles ran in the first round.  Every CTA takes all its
// gate/up tiles before any down tile.
MOE_HD int deal_tile(int b, int grid, int i, int total, int G, int comp, bool balanced)
{
    if (!balanced) {
        const int t = b + grid * i;
        return t < total ? t : -1;
    }
    const int D = total - G;
    const int grem = G % grid;
    const int gb = G / grid + (b < grem ? 1 : 0);
    if (i < gb) return b + grid * i;
    int j = i - gb;
    int comp_total = 0, my_comp = 0, comp0 = 0;
    if (grem > 0) {
        const int want = (grid - grem) * comp;
        comp_total = D < want ? D : want;
        if (b >= grem) {
            comp0 = (b - grem) * comp;
            const int left = comp_total - comp0;
            my_comp = left < 0 ? 0 : (left < comp ? left : comp);
        }
    }
    if (j < my_comp) return G + comp0 + j;
    j -= my_comp;
    const int dj = comp_total + b + grid * j;
    return dj < D ? G + dj : -1;
}

}  // namespace moe

namespace moe {

// Histogram class of a live routing, the key of the tuned tile table
// (Decoding the Skew, abstract: the kernel is chosen by matching the live
// routing histogram, and its skew is measured in Effective Experts).  With P
// routed pairs, eff = exp(entropy of counts / P) the effective number of
// experts and c_max the largest count:
//   tokens per effective expert m = P / eff in 5 buckets (<8, <32, <128, <512, more),
//   the hottest expert against that mean, c_max / m, in 3 buckets (<1.5, <4, more);
// class = 3 * bucket(m) + bucket(c_max / m).
constexpr int kTileClasses = 15;

MOE_HD int tile_class(float pairs, float eff, float c_max)
{
    if (!(pairs > 0.f) || !(eff > 0.f)) return 0;
    const float m = pairs / eff;
    const int b1 = m < 8.f ? 0 : m < 32.f ? 1 : m < 128.f ? 2 : m < 512.f ? 3 : 4;
    const float r = c_max / m;
    const int b2 = r < 1.5f ? 0 : r < 4.f ? 1 : 2;
    return 3 * b1 + b2;
}

// The token buckets of the static policy the histogram-matched one is measured
// against: T <= 16, 64, 256, 1024, 4096, more.
constexpr int kTokenBuckets = 6;

MOE_HD int token_bucket(long long T)
{
    return T <= 16 ? 0 : T <= 64 ? 1 : T <= 256 ? 2 : T <= 1024 ? 3 : T <= 4096 ? 4 : 5;
}

}  // namespace moe
