// route.cuh -- top-k with softmax gates (S2) over the router logits (S1, which
// run on the tensor cores as grouped_gemm_kernel<MODE_ROUTER>).
//
// Top-k: the k largest fp32 logits of a token in descending order, ties to the
// lower expert index, NaN below every number; gates are the softmax over the k
// chosen logits (Decoding the Skew, abstract: the routing distribution decided
// at run time drives the expert GEMMs).
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

// Order-preserving key: larger logit -> larger key; -0 and +0 equal; NaN lowest (0).
__device__ __forceinline__ uint32_t logit_key(float v)
{
    if (v != v) return 0u;
    if (v == 0.f) v = 0.f;
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of logit_key for the values it keeps apart (NaN maps back to a NaN).
__device__ __forceinline__ float key_logit(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Top-k of one token by one warp; PER logits per lane (E <= 32 * PER).  The
// token's logit for expert e is
//   sum_{s < splits} Lp[s * split_stride + t*E + e]  (+ bias[e] when bias != null),
// summed in ascending s (the split-K partials of the tensor-core router, or the
// logits themselves when splits == 1).  When logits_out != null that value is
// stored there.  Writes idx/w for the token (and the ids to s_idx when given).
template <int PER>
__device__ __forceinline__ void topk_warp(const float* Lp, size_t split_stride, int splits,
                                          const float* __restrict__ bias, int t, int E, int k,
                                          float* __restrict__ logits_out, int32_t* __restrict__ topk_idx,
                                          float* __restrict__ topk_w, uint32_t* __restrict__ err, int* s_idx)
{
    const int lane = threadIdx.x & 31;
    // Packed candidate: key in the high word, (0xFFFF - expert) in the low word, so
    // the maximum packed value is the largest logit with the lowest index.
    uint64_t cand[PER];
    bool nan_seen = false;
#pragma unroll
    for (int i = 0; i < PER; i++) {
        const int e = lane + 32 * i;
        cand[i] = 0;   // below every real candidate (real ones have a nonzero low word or key)
        if (e < E) {
            // __ldcg: the logits may have been written earlier in this very kernel
            const float* p = Lp + (size_t)t * E + e;
            float v = __ldcg(p);
            // partials in ascending order, fetched 8 at a time so the loads overlap
            for (int sp = 1; sp < splits; sp += 8) {
                float part[8];
#pragma unroll
                for (int u = 0; u < 8; u++)
                    part[u] = sp + u < splits ? __ldcg(p + (size_t)(sp + u) * split_stride) : 0.f;
#pragma unroll
                for (int u = 0; u < 8; u++)
                    if (sp + u < splits) v += part[u];
            }
            if (bias) v += bias[e];
            if (logits_out) logits_out[(size_t)t * E + e] = v;
            nan_seen |= (v != v);
            cand[i] = ((uint64_t)logit_key(v) << 32) | (uint64_t)(0xFFFFu - (uint32_t)e);
        }
    }
    if (__any_sync(0xffffffffu, nan_seen) && lane == 0) atomicOr(err, DEVERR_NAN_LOGIT);
    int chosen[kMaxTopK];
    float vals[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; j++) {
        if (j < k) {
            uint64_t best = 0;
#pragma unroll
            for (int i = 0; i < PER; i++) best = cand[i] > best ? cand[i] : best;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
                best = other > best ? other : best;
            }
            const int e = (int)(0xFFFFu - (uint32_t)(best & 0xFFFFu));
            chosen[j] = e;
            vals[j] = key_logit((uint32_t)(best >> 32));
#pragma unroll
            for (int i = 0; i < PER; i++)
                if (lane + 32 * i == e) cand[i] = 0;   // taken
        }
    }
    if (lane == 0) {
        // softmax over the chosen logits, shifted by the largest (vals[0])
        float ex[kMaxTopK];
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxTopK; j++) {
            if (j < k) {
                ex[j] = expf(vals[j] - vals[0]);
                z += ex[j];
            }
        }
#pragma unroll
        for (int j = 0; j < kMaxTopK; j++) {
            if (j < k) {
                topk_idx[(size_t)t * k + j] = chosen[j];
                topk_w[(size_t)t * k + j] = ex[j] / z;
                if (s_idx) s_idx[t * k + j] = chosen[j];
            }
        }
    }
}

// topk_warp with the smallest per-lane candidate array that holds E logits.
__device__ __forceinline__ void topk_warp_any(const float* Lp, size_t split_stride, int splits,
                                              const float* __restrict__ bias, int t, int E, int k,
                                              float* __restrict__ logits_out, int32_t* __restrict__ topk_idx,
                                              float* __restrict__ topk_w, uint32_t* __restrict__ err, int* s_idx)
{
    if (E <= 64)
        topk_warp<2>(Lp, split_stride, splits, bias, t, E, k, logits_out, topk_idx, topk_w, err, s_idx);
    else if (E <= 128)
        topk_warp<4>(Lp, split_stride, splits, bias, t, E, k, logits_out, topk_idx, topk_w, err, s_idx);
    else if (E <= 256)
        topk_warp<8>(Lp, split_stride, splits, bias, t, E, k, logits_out, topk_idx, topk_w, err, s_idx);
    else
        topk_warp<16>(Lp, split_stride, splits, bias, t, E, k, logits_out, topk_idx, topk_w, err, s_idx);
}

// One CTA per token (blockDim >= E, a multiple of 32) for a split router:
// thread e adds the token's split-K partials of expert e (ascending order,
// fetched 8 at a time) and the bias, stores the logit, and warp 0 then runs the
// top-k on the summed logits.  The partial sums are spread over E threads
// instead of E/32 per lane, which keeps small-T routing off the latency path.
__global__ void __launch_bounds__(512) topk_token_cta_kernel(const float* __restrict__ Lp, size_t split_stride,
                                                             int splits, const float* __restrict__ bias, int T,
                                                             int E, int k, float* logits_out,
                                                             int32_t* __restrict__ topk_idx,
                                                             float* __restrict__ topk_w, uint32_t* __restrict__ err)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int t = blockIdx.x;
    const int e = threadIdx.x;
    if (e < E) {
        const float* p = Lp + (size_t)t * E + e;
        float v = p[0];
        for (int sp = 1; sp < splits; sp += 8) {
            float part[8];
#pragma unroll
            for (int u = 0; u < 8; u++) part[u] = sp + u < splits ? p[(size_t)(sp + u) * split_stride] : 0.f;
#pragma unroll
            for (int u = 0; u < 8; u++)
                if (sp + u < splits) v += part[u];
        }
        if (bias) v += bias[e];
        logits_out[(size_t)t * E + e] = v;
    }
    __syncthreads();   // the block's global writes are visible to its own threads after the barrier
    if (threadIdx.x < 32)
        topk_warp_any(logits_out, 0, 1, nullptr, t, E, k, nullptr, topk_idx, topk_w, err, nullptr);
}

// One warp per token; E <= 512 (16 logits per lane), k <= 8.
__global__ void __launch_bounds__(256) topk_softmax_kernel(const float* __restrict__ Lp, size_t split_stride,
                                                           int splits, const float* __restrict__ bias, int T, int E,
                                                           int k, float* __restrict__ logits_out,
                                                           int32_t* __restrict__ topk_idx,
                                                           float* __restrict__ topk_w, uint32_t* __restrict__ err)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (warp >= T) return;
    topk_warp_any(Lp, split_stride, splits, bias, warp, E, k, logits_out, topk_idx, topk_w, err, nullptr);
}

}  // namespace moe
