// tile_table.h -- written by grouped_gemm_02_b200/tune_tiles.py; do not edit by hand.
//
// Tuned on NVIDIA B200 over 19 seeded Dirichlet workloads of the layer table
// (measurement record: tile_sweep_b200.json).  Classes measured: [0, 1, 4, 7, 10, 13]; the
// others keep the widest tiles.  Token buckets measured: [0, 1, 2, 3, 4, 5].
#pragma once

// Largest tile width (tokens) per histogram class (tile_class in schedule.h).
#define MOE_TILE_CAP_TABLE {256, 256, 256, 256, 128, 256, 256, 128, 256, 256, 256, 256, 256, 256, 256}

// Fixed tile width per token bucket (token_bucket in schedule.h) of the static policy.
#define MOE_TOKEN_BUCKET_WIDTH {32, 64, 128, 128, 256, 256}
