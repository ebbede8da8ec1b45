// tile_table.h -- written by grouped_gemm_02_b200/tune_tiles.py; do not edit by hand.
//
// Untuned defaults: every histogram class takes the widest tiles (256 tokens)
// and the token buckets grow the fixed width with T.
#pragma once

// Largest tile width (tokens) per histogram class (tile_class in schedule.h).
#define MOE_TILE_CAP_TABLE {256, 256, 256, 256, 256, 256, 256, 256, 256, 256, 256, 256, 256, 256, 256}

// Fixed tile width per token bucket (token_bucket in schedule.h) of the static policy.
#define MOE_TOKEN_BUCKET_WIDTH {16, 32, 64, 128, 256, 256}
