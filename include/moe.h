/*
 * moe.h -- C ABI of the B200 fused Mixture-of-Experts layer forward.
 *
 * The layer (Decoding the Skew: Distribution-Aware MoE Inference with Adaptive
 * Kernel Dispatch, abstract; GC-MoE: Overlapping Expert-Parallel Token Dispatch
 * with FP8/FP4 Grouped GEMM via CUDA Green Contexts, abstract):
 *
 *   L      = x Wg^T + b                         router logits            (moe_route)
 *   idx, w = top-k of L, softmax over the k     gating                   (moe_route / moe_topk)
 *   counts, offsets, perm, inv_perm, xp         histogram, scan, stable  (moe_permute)
 *                                               permute and row gather
 *   h   = silu(xp W1[e]^T) * (xp W3[e]^T)       grouped expert GEMMs     (moe_grouped_gemm)
 *   y_p = w[perm] * (h W2[e]^T)
 *   out = sum_j y_p[inv_perm[t*k+j]] (+ shared) deterministic combine    (moe_combine)
 *
 * and moe_layer_forward, which runs all of it with every intermediate in a
 * caller-owned workspace.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers are DEVICE pointers unless stated otherwise.  bf16 tensors are
 *   passed as raw 16-bit patterns (moe_bf16).  Every tensor is dense and
 *   row-major (nn.Linear storage): x [T,d], Wg [E,d], W1/W3 [E,f,d],
 *   W2 [E,d,f], Ws1/Ws3 [f_shared,d], Ws2 [d,f_shared], out [T,d].
 * - Pair q = t*k + j is token t's j-th choice (j = 0 is the largest logit).
 * - The caller owns every buffer.  No entry point allocates or frees memory,
 *   and none synchronises the host, except moe_get_device_error.
 * - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) on the current device, in call order.
 * - Limits: 1 <= E <= 512, 1 <= k <= min(8, E), T >= 0, T*k < 2^31;
 *   d and f (and f_shared) are multiples of 64; every pointer is 16-byte
 *   aligned.  T == 0 returns MOE_OK and enqueues nothing.
 * - Return value: MOE_OK, or a negative status found on the host before any
 *   work is enqueued (MOE_ERR_ARG, MOE_ERR_ALIGN, MOE_ERR_WS), or
 *   MOE_ERR_CUDA when a launch fails.  Conditions only the device can see
 *   (an expert id outside [0, E), a NaN logit, a kernel wait that timed out)
 *   set bits in a sticky error word inside the workspace; read them with
 *   moe_get_device_error.
 * - Kernels: hand-written for sm_100a (B200).  A device of another
 *   architecture gives MOE_ERR_DEVICE.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef uint16_t moe_bf16;

#define MOE_OK 0
#define MOE_ERR_ARG (-1)     /* null pointer, size out of range */
#define MOE_ERR_ALIGN (-2)   /* d, f or f_shared not a multiple of 64, or a pointer not 16-byte aligned */
#define MOE_ERR_WS (-3)      /* workspace smaller than moe_workspace_size reports */
#define MOE_ERR_CUDA (-4)    /* a CUDA launch or attribute call failed */
#define MOE_ERR_DEVICE (-5)  /* current device is not sm_100 */

/* int32 entries of the tile plan (moe_workspace_tensor which = 12). */
#define MOE_PLAN_INTS (8 + 6 * 513 + 2 * 514)

/* Device error bits (OR-ed, sticky until moe_clear_device_error). */
#define MOE_DEVERR_EXPERT_RANGE 1u  /* an expert id outside [0, E): that pair was dropped */
#define MOE_DEVERR_TIMEOUT 2u       /* a bounded wait inside a kernel gave up; outputs are invalid */
#define MOE_DEVERR_NAN_LOGIT 4u     /* a router logit was NaN; it ranked below every number */
#define MOE_DEVERR_PLAN 8u          /* a GEMM met a tile plan it cannot run and did nothing */

/* Bytes of workspace moe_layer_forward needs for these sizes (f_shared = 0:
 * no shared expert).  The control part of it (error word, tile plan,
 * histogram scratch) is also what moe_permute and moe_grouped_gemm need; a
 * layer-sized workspace serves every entry point.  Returns MOE_ERR_ARG on
 * negative sizes. */
MOE_API int moe_workspace_size(int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, int64_t f_shared, size_t *bytes);

/* Zero the workspace's control part (error word, plan).  Call once on a new
 * workspace before its first use; enqueued on `stream`. */
MOE_API int moe_workspace_init(void *ws, size_t ws_bytes, int64_t T, int64_t E, int64_t k, void *stream);

/* Router (Decoding the Skew, abstract: the runtime routing distribution).
 * logits [T,E] fp32 = x Wg^T + bias (bias [E] fp32, may be NULL): a bf16
 * tensor-core GEMM with fp32 accumulation; when T alone cannot fill the GPU
 * the d-loop is split into fixed ranges whose fp32 partial sums are added in
 * a fixed order, so the result is deterministic.  Then, per token, the k
 * largest logits in descending order (ties: lower expert id; NaN ranks
 * lowest) -> topk_idx [T,k] int32, and softmax over those k logits ->
 * topk_w [T,k] fp32.  `ws` (required, at least moe_workspace_size(T,d,f,E,k,0)
 * bytes for any f) holds the device error word and the partial sums. */
MOE_API int moe_route(const moe_bf16 *x, const moe_bf16 *Wg, const float *bias, int64_t T, int64_t d, int64_t E,
                      int64_t k, float *logits, int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes,
                      void *stream);

/* The top-k/softmax step of moe_route alone, on caller-provided fp32 logits
 * [T,E]; same ordering and gate definition.  `ws` (required) supplies the
 * device error word. */
MOE_API int moe_topk(const float *logits, int64_t T, int64_t E, int64_t k, int32_t *topk_idx, float *topk_w, void *ws,
             void *stream);

/* Histogram, exclusive scan, stable permutation and row gather (Decoding the
 * Skew, abstract: the live per-expert histogram kept on the GPU; Weave,
 * abstract: token dispatch).  counts [E] = pairs per expert; offsets [E+1] =
 * exclusive scan (offsets[E] = valid pairs); pairs are ordered expert-major and,
 * inside an expert, by ascending q: perm [T*k] (position -> q), inv_perm [T*k]
 * (q -> position); xp [T*k, d] row pos = x row perm[pos]/k (rows past
 * offsets[E] are left untouched).  A pair whose expert id is outside [0, E) is
 * dropped (inv_perm = -1, device error bit).  Needs a workspace of at least
 * moe_workspace_size(T,d,f,E,k,0) for any f (its control part). */
MOE_API int moe_permute(const int32_t *topk_idx, const moe_bf16 *x, int64_t T, int64_t d, int64_t E, int64_t k,
                int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm, moe_bf16 *xp, void *ws,
                size_t ws_bytes, void *stream);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory for one: code hosted by a framework that owns all device memory and
 * forbids allocation in its execute path, or latency-critical loops that
 * cannot afford cudaMalloc's implicit device synchronisation.  The pages have
 * no counterpart to this entry point; it exists for such callers only.
 * Same inputs, outputs and ordering as moe_permute.  Its scratch is a static
 * device array of 256 KiB (65536 int32 histogram counters plus an error word)
 * that each GPU loading this library keeps until the process exits; the
 * entry point allocates and frees nothing.  Sizes with
 * ceil(T*k / 4096) * E > 65536 are rejected with MOE_ERR_WS.  The first call
 * on a device looks up the array's device address (cudaGetSymbolAddress) for
 * that device; make that first call before any stream capture.  Every call
 * shares the one array, so calls whose work overlaps on the GPU (other
 * streams, other host threads) race and must be serialised by the caller.
 * Out-of-range expert ids are dropped as in moe_permute; with no workspace
 * there is no error word to read, so a dropped pair shows as
 * offsets[E] < T*k. */
MOE_API int moe_permute_noalloc(const int32_t *topk_idx, const moe_bf16 *x, int64_t T, int64_t d, int64_t E,
                                int64_t k, int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                                moe_bf16 *xp, void *stream);

/* Grouped expert GEMMs (Decoding the Skew, abstract: sparse expert GEMMs
 * whose shapes follow the live routing histogram; GC-MoE, abstract:
 * operand-swapped tcgen05 MMA with a fused SwiGLU).  From counts [E] and
 * offsets [E+1] on the device it builds the tile plan in `ws` (tile widths
 * chosen per expert from its count, heaviest experts first) and then, for
 * every expert e and row r in [offsets[e], offsets[e+1]):
 *   h [r, :]  = bf16( silu(xp[r] W1[e]^T) * (xp[r] W3[e]^T) )   h   [T*k, f]
 *   y_p[r, :] = bf16( topk_w[perm[r]] * (h[r] W2[e]^T) )        y_p [T*k, d]
 * with fp32 accumulation (topk_w is read as [T*k], indexed by q).  Rows past
 * offsets[E] are left untouched. */
MOE_API int moe_grouped_gemm(const moe_bf16 *xp, const int32_t *counts, const int32_t *offsets, const int32_t *perm,
                     const float *topk_w, const moe_bf16 *W1, const moe_bf16 *W3, const moe_bf16 *W2, int64_t T,
                     int64_t d, int64_t f, int64_t E, int64_t k, moe_bf16 *h, moe_bf16 *y_p, void *ws,
                     size_t ws_bytes, void *stream);

/* Deterministic combine: out[t,:] = bf16( sum_{j<k} y_p[inv_perm[t*k+j], :]
 * (+ shared_out[t,:]) ), summed in fp32 in ascending j, no atomics.
 * inv_perm < 0 adds nothing.  shared_out [T,d] may be NULL. */
MOE_API int moe_combine(const moe_bf16 *y_p, const int32_t *inv_perm, const moe_bf16 *shared_out, int64_t T, int64_t k,
                int64_t d, moe_bf16 *out, void *stream);

/* The whole layer: route -> permute -> grouped GEMMs -> combine, with the
 * optional always-on shared expert (GC-MoE, abstract: optional shared experts)
 * Ws1/Ws3 [f_shared,d], Ws2 [d,f_shared] (all NULL and f_shared = 0 for none)
 * added with gate 1.  out [T,d].  Every intermediate lives in `ws`
 * (moe_workspace_size bytes).  Bit-identical to calling the steps one by one
 * on the same inputs (also under MOE_POLICY_GATHER = 1, which leaves xp
 * untouched). */
MOE_API int moe_layer_forward(const moe_bf16 *x, const moe_bf16 *Wg, const float *bias, const moe_bf16 *W1,
                      const moe_bf16 *W3, const moe_bf16 *W2, const moe_bf16 *Ws1, const moe_bf16 *Ws3,
                      const moe_bf16 *Ws2, int64_t f_shared, int64_t T, int64_t d, int64_t f, int64_t E, int64_t k,
                      moe_bf16 *out, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------- FP8 path
 * The FP8 block-scaled variant (GC-MoE, abstract: an FP8 MoE operator with
 * block-scaled MMA and requantisation; e4m3 with 1 x 128 activation blocks and
 * 128 x 128 weight blocks).  Codes are OCP e4m3 (round to nearest, ties to
 * even, saturating at +-448).  A block's scale is the smallest power of two s
 * with max|v| / s <= 448 (s = 1 for an all-zero block), held to the UE8M0
 * range 2^-127 .. 2^127 that the block-scaled MMA takes, stored as fp32, so
 * code q with scale s stands for e4m3(q) * s exactly.  d, f and f_shared must
 * be multiples of 128 (MOE_ERR_ALIGN otherwise) and at most 16384
 * (MOE_ERR_ARG otherwise). */

/* 1 x 128 blocks along each row: x [rows, cols] bf16 -> q [rows, cols] e4m3,
 * scales [rows, cols/128] fp32.  cols % 128 == 0. */
MOE_API int moe_quantize_fp8_rows(const moe_bf16 *x, int64_t rows, int64_t cols, uint8_t *q, float *scales,
                                  void *stream);

/* 128 x 128 blocks: W [rows, cols] bf16 -> q [rows, cols] e4m3, scales
 * [rows/128, cols/128] fp32 (block (i, j) covers rows 128i.. and cols 128j..).
 * Expert weights are quantised as one matrix: W1/W3 as [E*f, d] (scales
 * [E*f/128, d/128]), W2 as [E*d, f] (scales [E*d/128, f/128]). */
MOE_API int moe_quantize_fp8_blocks(const moe_bf16 *W, int64_t rows, int64_t cols, uint8_t *q, float *scales,
                                    void *stream);

/* Workspace bytes of moe_layer_forward_fp8 for these sizes. */
MOE_API int moe_workspace_size_fp8(int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, int64_t f_shared,
                                   size_t *bytes);

/* Device pointers of the FP8 layer intermediates inside its workspace
 * (which: 0 logits, 1 topk_idx, 2 topk_w, 3 counts, 4 offsets, 5 perm,
 * 6 inv_perm, 7 x8, 8 sx, 9 xp8, 10 sxp, 11 h8, 12 sh, 13 y_p, 14 hs8, 15 shs,
 * 16 ys, 17 sxT, 18 the tile plan).  sx is [T, d/128]; the scale arrays the GEMMs read are
 * K-block-major with rows padded to a multiple of 4 entries: sxp
 * [d/128, P4], sh [f/128, P4], shs [f_shared/128, T4], sxT [d/128, T4]
 * (P4 = T*k and T4 = T rounded up to a multiple of 4).  Host-only arithmetic. */
MOE_API int moe_workspace_tensor_fp8(void *ws, int64_t T, int64_t d, int64_t f, int64_t E, int64_t k,
                                     int64_t f_shared, int which, void **ptr);

/* The whole layer with FP8 expert GEMMs.  Routing is the bf16 router of
 * moe_route (same logits, top-k and gates).  x is quantised in 1 x 128 blocks,
 * gathered into expert order, and multiplied with the pre-quantised weights
 * (W1q/W3q [E,f,d] with scales W1s/W3s [E*f/128, d/128]; W2q [E,d,f] with W2s
 * [E*d/128, f/128]; the shared expert Ws1q/Ws3q [f_shared,d], Ws2q
 * [d,f_shared] with their scales, or all NULL and f_shared = 0):
 *   h   = silu(x^ W1^T) * (x^ W3^T), requantised in 1 x 128 blocks along f
 *   y_p = gate * (h^ W2^T)          (bf16), then the combine of moe_combine,
 * where ^ marks dequantised values; all products accumulate in fp32 (the
 * tensor cores apply the power-of-two block scales as UE8M0 exponents inside
 * the MMA).  Every intermediate lives in `ws` (moe_workspace_size_fp8 bytes). */
MOE_API int moe_layer_forward_fp8(const moe_bf16 *x, const moe_bf16 *Wg, const float *bias, const uint8_t *W1q,
                                  const float *W1s, const uint8_t *W3q, const float *W3s, const uint8_t *W2q,
                                  const float *W2s, const uint8_t *Ws1q, const float *Ws1s, const uint8_t *Ws3q,
                                  const float *Ws3s, const uint8_t *Ws2q, const float *Ws2s, int64_t f_shared,
                                  int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, moe_bf16 *out, void *ws,
                                  size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------- FP4 weights
 * FP4 expert weights (GC-MoE, abstract: an FP8/FP4 MoE operator with
 * block-scaled MMA).  Weights are OCP e2m1 codes (sign, 2 exponent bits with
 * bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) in blocks of
 * 32 consecutive elements along each row (MXFP4): a block's scale is the
 * smallest power of two s with max|v| / s <= 6 (s = 1 for an all-zero block),
 * held to the UE8M0 range; codes round to nearest, ties to even, saturating at
 * 6.  Activations stay e4m3 with 1 x 128 scales, as in the FP8 path. */

/* W [rows, cols] bf16 -> q [rows, cols/2] bytes of packed e2m1 codes (element
 * 2i in the low nibble of byte i) and scale_atoms [rows/128][cols/128][512]
 * bytes: the UE8M0 exponent byte (e + 127 for scale 2^e) of row r's 32-wide
 * block j of each 128 x 128 tile at byte 16 (r % 32) + 4 (r / 32) + j of that
 * tile's 512 bytes (the layout the block-scaled MMA reads).  Expert weights are
 * quantised as one matrix: W1/W3 as [E*f, d], W2 as [E*d, f].  rows and cols
 * multiples of 128 (MOE_ERR_ALIGN otherwise); q and scale_atoms 16-byte
 * aligned. */
MOE_API int moe_quantize_fp4_rows(const moe_bf16 *W, int64_t rows, int64_t cols, uint8_t *q, uint8_t *scale_atoms,
                                  void *stream);

/* The whole layer with FP4 expert weights (packed e2m1 W1q/W3q [E, f, d/2],
 * W2q [E, d, f/2] with the scale atoms moe_quantize_fp4_rows writes, and the
 * shared expert's likewise, or all NULL and f_shared = 0):
 *   h   = silu(x^ W1^T) * (x^ W3^T), requantised to e4m3 in 1 x 128 blocks
 *   y_p = gate * (h^ W2^T)   (bf16), then the combine of moe_combine,
 * where ^ marks dequantised values and every product accumulates in fp32 (the
 * tensor cores apply both operands' power-of-two block scales inside the MMA,
 * kind::mxf8f6f4 with e2m1 A and e4m3 B).  Routing is the bf16 router.  The
 * workspace is the FP8 layer's (moe_workspace_size_fp8); the same size limits
 * and errors as moe_layer_forward_fp8. */
MOE_API int moe_layer_forward_fp4(const moe_bf16 *x, const moe_bf16 *Wg, const float *bias, const uint8_t *W1q,
                                  const uint8_t *W1sf, const uint8_t *W3q, const uint8_t *W3sf, const uint8_t *W2q,
                                  const uint8_t *W2sf, const uint8_t *Ws1q, const uint8_t *Ws1sf, const uint8_t *Ws3q,
                                  const uint8_t *Ws3sf, const uint8_t *Ws2q, const uint8_t *Ws2sf, int64_t f_shared,
                                  int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, moe_bf16 *out, void *ws,
                                  size_t ws_bytes, void *stream);

/* Per-phase timing of the next moe_layer_forward call made on this host
 * thread: `events` holds n >= 6 cudaEvent_t handles; that call records
 * events[0..5] on its stream before the router, the permutation, the gate/up
 * GEMM, the down GEMM and the combine, and after the combine.  The array is
 * used once (the call after it records nothing).  n = 0 cancels. */
MOE_API int moe_record_phase_events(void *const *events, int n);

/* Process-wide choices of how the expert GEMMs run, for comparisons, tuning
 * and tests.  value -1 restores the library's rule; other values force the
 * choice for every later call in the process.  Results do not depend on these
 * choices beyond fp32 summation order.
 *   MOE_POLICY_ONE_LAUNCH  1: gate/up and down tiles in one persistent launch,
 *                          0: two launches (rule: one when T*k <= 256 and f <= 4096)
 *   MOE_POLICY_CTA_PAIRS   1: tiles of 2 x 128 weight rows on CTA pairs
 *                          (cta_group::2), 0: single-CTA tiles of 128 rows
 *                          (rule: the bf16 GEMMs take pairs whenever two
 *                          launches run; the FP8 / FP4 GEMMs take them only
 *                          when this is 1 and two launches run)
 *   MOE_POLICY_TILES       0 (rule): histogram-matched tiles -- the plan step
 *                          classifies the live histogram on the device (tokens
 *                          per effective expert, hottest expert against that
 *                          mean) and takes the tile cap the tuned table holds
 *                          for the class, every expert's width following its
 *                          own count (Decoding the Skew, abstract: kernel
 *                          selection by matching the live routing histogram);
 *                          1: static token buckets -- one tile width chosen
 *                          from T alone, every expert's tiles padded to it, the
 *                          selection that paper measures against
 *   MOE_POLICY_TILE_CAP    16..256 (multiple of 16): every plan under this cap,
 *                          widths following the counts, or with MOE_POLICY_TILES
 *                          = 1 every tile of exactly this width (table
 *                          tuning); -1: off
 *   MOE_POLICY_GATHER      1: moe_layer_forward's gate/up GEMM gathers its token
 *                          rows straight from x (TMA tile::gather4, four rows per
 *                          request) instead of a gather pass into xp, when the
 *                          expert GEMMs run as two launches (the single launch
 *                          keeps the gather pass); 0 (rule): the gather pass,
 *                          measured faster on B200 at every size
 * Returns MOE_ERR_ARG for an unknown switch or value.  The pages have no
 * counterpart to the first two switches. */
#define MOE_POLICY_ONE_LAUNCH 1
#define MOE_POLICY_CTA_PAIRS 2
#define MOE_POLICY_TILES 3
#define MOE_POLICY_TILE_CAP 4
#define MOE_POLICY_GATHER 5
MOE_API int moe_set_policy(int what, int value);

/* Number of kernels this library has launched in this process so far. */
MOE_API int64_t moe_launch_counter(void);

/* Device pointers of the layer intermediates inside a layer workspace
 * (which: 0 logits, 1 topk_idx, 2 topk_w, 3 counts, 4 offsets, 5 perm,
 * 6 inv_perm, 7 xp, 8 h, 9 y_p, 10 hs, 11 ys, 12 the tile plan).  The tile plan is
 * MOE_PLAN_INTS int32: a header {n_blocks, tiles1, tiles2, n_max, pairs,
 * pair (bit 0: tiles cut for CTA pairs; bit 1: a down tile spans two units,
 * the FP8 / FP4 layer's two-launch form), cls (the histogram class whose tuned
 * cap was taken; -1: a forced cap, -2: token buckets), cap (most tokens per
 * tile)},
 * then arrays of 513 entries group, row0, rows, chunk, units, two tile
 * prefixes of 514 entries (gate/up, down) and 513 per-block counters of
 * finished gate/up tiles (see the tile plan in the grouped-GEMM comment).
 * Host-only arithmetic. */
MOE_API int moe_workspace_tensor(void *ws, int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, int64_t f_shared,
                         int which, void **ptr);

/* Copies the sticky device error word to *code (host int).  Synchronises
 * `stream`. */
MOE_API int moe_get_device_error(const void *ws, uint32_t *code, void *stream);

/* Clears the sticky device error word; enqueued on `stream`. */
MOE_API int moe_clear_device_error(void *ws, void *stream);

/* Diagnostic of the failure path (the pages have no counterpart): one CTA
 * runs the two bounded waits the GEMM kernels use -- on an mbarrier nobody
 * arrives on, then on a counter nobody increments (the int after the error
 * word in `ws`, zeroed by this call) -- and each gives up after its 1 s
 * deadline.  Afterwards the error word holds MOE_DEVERR_TIMEOUT (and
 * MOE_DEVERR_PLAN only if a wait ended that should not have) and the CUDA
 * context is still usable.  Takes about 2 s of GPU time; `ws` is any layer
 * workspace. */
MOE_API int moe_selftest_wait_timeout(void *ws, void *stream);

/* Human-readable name of a status code. */
MOE_API const char *moe_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
