// Host harness for the CPU test of the persistent GEMM's tile deal: compiles
// grouped_gemm_02_b200/csrc/schedule.h (the function the kernels call) with
// the host compiler and exposes it through a C symbol.
#include "../grouped_gemm_02_b200/csrc/schedule.h"

extern "C" {

// For every CTA b < grid, the tiles it takes in order, written to
// tiles[b * max_per + i] (-1 after its last one).  Returns the largest count
// any CTA took, or -1 if a CTA would take more than max_per.
int deal_all(int grid, int total, int G, int comp, int balanced, int max_per, int* tiles)
{
    int most = 0;
    for (int b = 0; b < grid; b++) {
        int i = 0;
        for (;; i++) {
            const int t = moe::deal_tile(b, grid, i, total, G, comp, balanced != 0);
            if (t < 0) break;
            if (i >= max_per) return -1;
            tiles[b * max_per + i] = t;
        }
        for (int j = i; j < max_per; j++) tiles[b * max_per + j] = -1;
        if (i > most) most = i;
    }
    return most;
}

}

extern "C" int tile_class_of(float pairs, float eff, float c_max) { return moe::tile_class(pairs, eff, c_max); }
extern "C" int token_bucket_of(long long T) { return moe::token_bucket(T); }
