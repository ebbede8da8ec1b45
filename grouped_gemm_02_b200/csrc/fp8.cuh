// fp8.cuh -- the FP8 block-scaled expert path (S9): e4m3 quantisers, the e4m3
// row gather, and a persistent tcgen05 grouped GEMM on e4m3 operands.
//
// GC-MoE (abstract) runs its expert GEMMs as block-scaled FP8 MMAs with a
// requantisation step; the workload table fixes e4m3 codes with 1 x 128
// activation blocks and 128 x 128 weight blocks.  Readings: a block's scale is
// the smallest power of two s with amax / s <= 448 (amax = 0: s = 1); codes are
// round-to-nearest-even with saturation to +-448.  Because every scale is a
// power of two, scaling is exact: the GEMM multiplies e4m3 codes on the tensor
// cores one 128-wide K block at a time (tcgen05.mma kind::f8f6f4, fp32
// accumulate into a fresh TMEM partial) and the epilogue warps add each partial
// times (weight-block scale x activation-block scale) into fp32 running sums --
// the dequantised product the definition asks for.
//
//   MODE gate/up:  h = silu(sum_kb P_g * s_W1 * s_x) * (sum_kb P_u * s_W3 * s_x),
//                  then h is requantised in 1 x 128 blocks along f (the tile's
//                  128 f rows are one block) -> h8 [pairs, f] + sh [pairs, f/128]
//   MODE down:     y_p = gate * sum_kb P * s_W2 * s_h  -> bf16
//
// One tile = 128 weight rows (W1 and W3 rows side by side for gate/up) x at
// most 64 tokens; the epilogue keeps the tile's running sums in registers.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"
#include "grouped_gemm.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kFp8TileRows = 64;                 // most tokens one FP8 tile carries
constexpr int kFp8BlockK = 128;                  // e4m3 elements per 128-byte swizzle row = one scale block
constexpr int kFp8Bufs = 4;                      // TMEM partial buffers between the MMA and the epilogue
constexpr uint32_t kFp8TmemCols = 512;           // 4 partial buffers x (g: 64 + u: 64) columns

// Smallest power-of-two exponent e with amax <= 448 * 2^e (amax > 0), from the
// binary exponent of amax: amax = m * 2^x, m in [0.5, 1), 448 = 0.875 * 2^9.
__device__ __forceinline__ int fp8_scale_exp(float amax)
{
    if (!(amax > 0.f)) return 0;
    int x;
    const float m = frexpf(amax, &x);
    return m <= 0.875f ? x - 9 : x - 8;
}

__device__ __forceinline__ uint8_t e4m3_of(float v)
{
    return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// ---------------------------------------------------------------- quantisers
// 1 x 128 blocks along rows: one warp per (row, block); lane l holds 4 values.
__global__ void __launch_bounds__(256) quantize_rows_fp8_kernel(const bf16* __restrict__ src, int64_t R, int C,
                                                                uint8_t* __restrict__ dst, float* __restrict__ scale)
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
    if (lane == 0) scale[r * nb + b] = ldexpf(1.f, e);
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

// xp8[pos, :] = x8[perm[pos] / k, :], sxp[pos, :] = sx[perm[pos] / k, :]; one warp per row.
__global__ void __launch_bounds__(256) gather_rows_fp8_kernel(const uint8_t* __restrict__ x8,
                                                              const float* __restrict__ sx,
                                                              const int32_t* __restrict__ perm,
                                                              const int32_t* __restrict__ offsets, int E, int k, int d,
                                                              uint8_t* __restrict__ xp8, float* __restrict__ sxp)
{
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const int pairs = offsets[E];
    const int nvec = d / 16, nsb = d / 128;
    const int lane = threadIdx.x & 31;
    for (int64_t r = (int64_t)(blockIdx.x * blockDim.x + threadIdx.x) / 32; r < pairs;
         r += (int64_t)gridDim.x * blockDim.x / 32) {
        const int t = perm[r] / k;
        const uint4* src = reinterpret_cast<const uint4*>(x8 + (size_t)t * d);
        uint4* dst = reinterpret_cast<uint4*>(xp8 + (size_t)r * d);
        for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
            uint4 buf[4];
#pragma unroll
            for (int u = 0; u < 4; u++)
                if (v0 + 32 * u < nvec) buf[u] = __ldg(src + v0 + 32 * u);
#pragma unroll
            for (int u = 0; u < 4; u++)
                if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = buf[u];
        }
        for (int b = lane; b < nsb; b += 32) sxp[(size_t)r * nsb + b] = sx[(size_t)t * nsb + b];
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
    const float* sB;                // activation-block scales of the B rows [pairs, K/128]
    const float* sBs;               // shared rows [T, K_shared/128]
    uint8_t* out8;                  // gate/up: h8 [pairs, f]
    float* out8_scale;              // sh [pairs, f/128]
    uint8_t* out8_shared;           // hs8 [T, f_shared]
    float* out8_scale_shared;       // shs [T, f_shared/128]
    bf16* out;                      // down: y_p [pairs, d]
    bf16* out_shared;               // ys [T, d]
    const int32_t* perm;
    const float* gate_w;
    uint32_t* err;
};

struct Fp8Tile {
    int group, m, row0, rows, n_mma, nkb;
    bool shared;
};

template <bool GATED>
__device__ __forceinline__ Fp8Tile fp8_decode(int nb, int t, const Fp8Args& a, const SmemPlan* sp)
{
    const int* tb = sp->tb;
    int lo = 0, hi = nb - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    const int local = t - tb[lo];
    const int units = sp->units[lo];
    const int4 b = sp->blk[lo];
    Fp8Tile tl;
    tl.group = b.x;
    tl.shared = tl.group == a.E;
    tl.m = local / units;
    const int u = local - tl.m * units;
    const int start = u * b.w;
    tl.rows = min(b.w, b.z - start);
    tl.row0 = b.y + start;
    tl.n_mma = (tl.rows + 15) & ~15;
    tl.nkb = ((tl.shared ? a.K_shared : a.K) + kFp8BlockK - 1) / kFp8BlockK;
    return tl;
}

struct Fp8Iter {
    int t, kb;
    Fp8Tile tl;
};

template <bool GATED>
__device__ __forceinline__ bool fp8_iter_begin(Fp8Iter& it, int nb, int total, const Fp8Args& a, const SmemPlan* sp)
{
    it.t = blockIdx.x;
    if (it.t >= total) return false;
    it.tl = fp8_decode<GATED>(nb, it.t, a, sp);
    it.kb = 0;
    return true;
}

template <bool GATED>
__device__ __forceinline__ bool fp8_iter_next(Fp8Iter& it, int nb, int total, const Fp8Args& a, const SmemPlan* sp)
{
    if (++it.kb < it.tl.nkb) return true;
    it.t += gridDim.x;
    if (it.t >= total) return false;
    it.tl = fp8_decode<GATED>(nb, it.t, a, sp);
    it.kb = 0;
    return true;
}

__device__ __forceinline__ void named_bar_epilogue() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Instruction descriptor for kind::f8f6f4 with e4m3 A and B (format 0), fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(uint32_t M, uint32_t N)
{
    return (1u << 4) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void mma_fp8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <bool GATED>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_fp8_kernel(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mA1,
                            const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mA0s,
                            const __grid_constant__ CUtensorMap mA1s, const __grid_constant__ CUtensorMap mBs,
                            const Fp8Args args)
{
    constexpr uint32_t kABytes = GATED ? 2 * 128 * kFp8BlockK : 128 * kFp8BlockK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + kRingBytes);
    SmemPlan* splan = reinterpret_cast<SmemPlan*>(smem + kRingBytes + kBarBytes);
    float* red = reinterpret_cast<float*>(smem + kRingBytes + kBarBytes + sizeof(SmemPlan));   // [4][64]
    const uint32_t ring = ptx::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const bool waited_early = !args.plan_ready;
    if (waited_early) ptx::grid_dep_wait();
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(args.plan);
    if (hdr->n_max > kFp8TileRows) {   // a plan made for wider tiles: refuse, touch nothing
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(args.err, DEVERR_PLAN);
        return;
    }
    const int nb = hdr->n_blocks;
    const int total = GATED ? hdr->tiles1 : hdr->tiles2;
    const int n_max = max(16, hdr->n_max);
    const uint32_t stage_bytes = kABytes + (uint32_t)n_max * kFp8BlockK;
    const int stages = min(kMaxStages, (int)(kRingBytes / stage_bytes));
    {
        const PlanArrays pa = plan_arrays(const_cast<int32_t*>(args.plan));
        const int32_t* tbg = GATED ? pa.tb1 : pa.tb2;
        for (int i = threadIdx.x; i <= nb; i += blockDim.x) {
            splan->tb[i] = tbg[i];
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
        for (int a = 0; a < kFp8Bufs; a++) {
            ptx::mbar_init(ptx::smem_u32(&ctl->tfull[a]), 1);
            ptx::mbar_init(ptx::smem_u32(&ctl->tempty[a]), 4);
        }
        ptx::mbar_init(ptx::smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&mA0);
        ptx::prefetch_tensormap(&mB);
        if (GATED) ptx::prefetch_tensormap(&mA1);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(&ctl->tmem_base), kFp8TmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (ptx::elect_one()) {
            const uint64_t pol = ptx::policy_evict_normal();
            uint32_t armed = 0, armed_ph = 0;
            bool ok = true;
            auto issue_a = [&](const Fp8Iter& it, uint32_t a_dst, uint32_t full) {
                const Fp8Tile& tl = it.tl;
                const int kc = it.kb * kFp8BlockK;
                const int Mrows = tl.shared ? args.M_shared : args.M;
                const int a_row = (tl.shared ? 0 : tl.group * Mrows) + tl.m * 128;
                ptx::tma_load_2d(a_dst, tl.shared ? &mA0s : &mA0, full, kc, a_row, pol);
                if (GATED) ptx::tma_load_2d(a_dst + 128 * kFp8BlockK, tl.shared ? &mA1s : &mA1, full, kc, a_row, pol);
            };
            auto issue_b = [&](const Fp8Iter& it, uint32_t b_dst, uint32_t full) {
                const Fp8Tile& tl = it.tl;
                const int kc = it.kb * kFp8BlockK;
                for (int i = 0; i < tl.n_mma / 16; i++)
                    ptx::tma_load_2d(b_dst + i * 16 * kFp8BlockK, tl.shared ? &mBs : &mB, full, kc, tl.row0 + 16 * i,
                                     pol);
            };
            int pre = 0;
            if (!waited_early) {
                Fp8Iter it;
                bool more = fp8_iter_begin<GATED>(it, nb, total, args, splan);
                while (more && pre < stages) {
                    const uint32_t full = ptx::smem_u32(&ctl->full[pre]);
                    ptx::mbar_arrive_expect_tx(full, kABytes + (uint32_t)it.tl.n_mma * kFp8BlockK);
                    armed |= 1u << pre;
                    issue_a(it, ring + (uint32_t)pre * stage_bytes, full);
                    ++pre;
                    more = fp8_iter_next<GATED>(it, nb, total, args, splan);
                }
                ptx::grid_dep_wait();
            }
            ptx::grid_dep_launch();
            int s = 0, n = 0;
            uint32_t ph = 0;
            Fp8Iter it;
            bool more = fp8_iter_begin<GATED>(it, nb, total, args, splan);
            while (more) {
                const uint32_t a_dst = ring + (uint32_t)s * stage_bytes;
                const uint32_t full = ptx::smem_u32(&ctl->full[s]);
                if (n < pre) {
                    issue_b(it, a_dst + kABytes, full);
                } else {
                    if (!bounded_wait(ptx::smem_u32(&ctl->empty[s]), ph ^ 1u, ctl, args.err)) {
                        ok = false;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(full, kABytes + (uint32_t)it.tl.n_mma * kFp8BlockK);
                    armed |= 1u << s;
                    armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                    issue_a(it, a_dst, full);
                    issue_b(it, a_dst + kABytes, full);
                }
                ++n;
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
                more = fp8_iter_next<GATED>(it, nb, total, args, splan);
            }
            if (!ok) {
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
        // ------------------------------------------------------------ MMA issuer: one fresh partial per K block
        if (ptx::elect_one()) {
            int s = 0, pb = 0;
            uint32_t ph = 0, pph = 0;
            bool ok = true, issued = false;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const Fp8Tile tl = fp8_decode<GATED>(nb, t, args, splan);
                const uint32_t idesc = idesc_e4m3_f32(128, (uint32_t)tl.n_mma);
                for (int kb = 0; kb < tl.nkb; kb++) {
                    if (!bounded_wait(ptx::smem_u32(&ctl->tempty[pb]), pph ^ 1u, ctl, args.err) ||
                        !bounded_wait(ptx::smem_u32(&ctl->full[s]), ph, ctl, args.err)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ring + (uint32_t)s * stage_bytes;
                    const uint32_t b_addr = a_addr + kABytes;
                    const uint32_t d_g = tmem_base + (uint32_t)pb * 128u;
#pragma unroll
                    for (int kk = 0; kk < kFp8BlockK / 32; kk++)
                        mma_fp8_ss(d_g, ptx::sw128_kmajor_desc(a_addr + kk * 32),
                                   ptx::sw128_kmajor_desc(b_addr + kk * 32), idesc, kk > 0 ? 1u : 0u);
                    if (GATED) {
#pragma unroll
                        for (int kk = 0; kk < kFp8BlockK / 32; kk++)
                            mma_fp8_ss(d_g + 64u, ptx::sw128_kmajor_desc(a_addr + 128 * kFp8BlockK + kk * 32),
                                       ptx::sw128_kmajor_desc(b_addr + kk * 32), idesc, kk > 0 ? 1u : 0u);
                    }
                    issued = true;
                    ptx::mma_commit(ptx::smem_u32(&ctl->empty[s]));
                    ptx::mma_commit(ptx::smem_u32(&ctl->tfull[pb]));
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                    if (++pb == kFp8Bufs) {
                        pb = 0;
                        pph ^= 1u;
                    }
                }
            }
            if (!ok && issued) {
                ptx::mma_commit(ptx::smem_u32(&ctl->drain));
                const uint64_t t0 = ptx::globaltimer();
                while (!ptx::mbar_try_wait(ptx::smem_u32(&ctl->drain), 0) &&
                       ptx::globaltimer() - t0 < kWaitTimeoutNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue: scale, accumulate, finish
        // The activation scales (sB) come from the kernel right before this one:
        // wait for it before the first (prefetched) read.
        if (!waited_early) ptx::grid_dep_wait();
        const int quad = warp & 3;
        const int row_in_tile = quad * 32 + lane;        // weight row of this thread (TMEM lane)
        int pb = 0;
        uint32_t pph = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Fp8Tile tl = fp8_decode<GATED>(nb, t, args, splan);
            const int Mrows = tl.shared ? args.M_shared : args.M;
            const int K = tl.shared ? args.K_shared : args.K;
            const int kbl = K / 128;                          // scale blocks along K
            const float* sB = tl.shared ? args.sBs : args.sB;
            const float* sA0 = tl.shared ? args.sA0s : args.sA0;
            const float* sA1 = tl.shared ? args.sA1s : args.sA1;
            // row of the weight-scale table for this tile's 128 weight rows
            const int64_t srow = (int64_t)(tl.shared ? 0 : tl.group * (Mrows / 128)) + tl.m;
            float acc_g[kFp8TileRows], acc_u[GATED ? kFp8TileRows : 1];
#pragma unroll
            for (int c = 0; c < kFp8TileRows; c++) acc_g[c] = 0.f;
#pragma unroll
            for (int c = 0; c < (GATED ? kFp8TileRows : 1); c++) acc_u[c] = 0.f;
            // scales of K block kb are fetched while K block kb - 1 is being added
            auto scales = [&](int kb, float& a0, float& a1, float& xa, float& xb) {
                a0 = __ldg(sA0 + srow * kbl + kb);
                a1 = GATED ? __ldg(sA1 + srow * kbl + kb) : 0.f;
                xa = lane < tl.rows ? __ldg(sB + (int64_t)(tl.row0 + lane) * kbl + kb) : 0.f;
                xb = lane + 32 < tl.rows ? __ldg(sB + (int64_t)(tl.row0 + lane + 32) * kbl + kb) : 0.f;
            };
            float s0, s1, sxa, sxb;
            scales(0, s0, s1, sxa, sxb);
            for (int kb = 0; kb < tl.nkb; kb++) {
                float n0 = 0.f, n1 = 0.f, nxa = 0.f, nxb = 0.f;
                if (kb + 1 < tl.nkb) scales(kb + 1, n0, n1, nxa, nxb);
                const bool good = bounded_wait(ptx::smem_u32(&ctl->tfull[pb]), pph, ctl, args.err);
                if (!__all_sync(0xffffffffu, good)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t taddr = tmem_base + (uint32_t)pb * 128u + ((uint32_t)(quad * 32) << 16);
#pragma unroll
                for (int c0 = 0; c0 < kFp8TileRows; c0 += 16) {
                    if (c0 < tl.n_mma) {
                        uint32_t v[16], w[16];
                        ptx::tmem_ld16(taddr + (uint32_t)c0, v);
                        if (GATED) ptx::tmem_ld16(taddr + 64u + (uint32_t)c0, w);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; j++) {
                            const int c = c0 + j;
                            const float sx = __shfl_sync(0xffffffffu, c < 32 ? sxa : sxb, c & 31);
                            acc_g[c] = fmaf(__uint_as_float(v[j]), s0 * sx, acc_g[c]);
                            if (GATED) acc_u[c] = fmaf(__uint_as_float(w[j]), s1 * sx, acc_u[c]);
                        }
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&ctl->tempty[pb]));
                if (++pb == kFp8Bufs) {
                    pb = 0;
                    pph ^= 1u;
                }
                s0 = n0;
                s1 = n1;
                sxa = nxa;
                sxb = nxb;
            }
            if (!ok) break;
            if (GATED) {
                // h = silu(g) * u, then requantise each token's 128 h values of this tile
#pragma unroll
                for (int c = 0; c < kFp8TileRows; c++) {
                    if (c < tl.rows) {   // warp-uniform
                        const float g = acc_g[c];
                        acc_g[c] = g / (1.0f + __expf(-g)) * acc_u[c];
                        float a = tl.m * 128 + row_in_tile < Mrows ? fabsf(acc_g[c]) : 0.f;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
                        if (lane == 0) red[quad * kFp8TileRows + c] = a;
                    }
                }
                named_bar_epilogue();
                uint8_t* out8 = tl.shared ? args.out8_shared : args.out8;
                float* osc = tl.shared ? args.out8_scale_shared : args.out8_scale;
                const int frow = tl.m * 128 + row_in_tile;
#pragma unroll
                for (int c = 0; c < kFp8TileRows; c++) {
                    if (c < tl.rows) {
                        const float amax = fmaxf(fmaxf(red[c], red[kFp8TileRows + c]),
                                                 fmaxf(red[2 * kFp8TileRows + c], red[3 * kFp8TileRows + c]));
                        const int e = fp8_scale_exp(amax);
                        const int64_t r = tl.row0 + c;
                        if (frow < Mrows) out8[r * Mrows + frow] = e4m3_of(ldexpf(acc_g[c], -e));
                        if (row_in_tile == 0) osc[r * (Mrows / 128) + tl.m] = ldexpf(1.f, e);
                    }
                }
                named_bar_epilogue();   // red[] is reused by the next tile
            } else {
                bf16* out = tl.shared ? args.out_shared : args.out;
                const int drow = tl.m * 128 + row_in_tile;
                const float gsa = (!tl.shared && lane < tl.rows) ? __ldg(args.gate_w + __ldg(args.perm + tl.row0 + lane)) : 1.f;
                const float gsb = (!tl.shared && lane + 32 < tl.rows)
                                      ? __ldg(args.gate_w + __ldg(args.perm + tl.row0 + lane + 32))
                                      : 1.f;
#pragma unroll
                for (int c = 0; c < kFp8TileRows; c++) {
                    if (c >= tl.rows) continue;   // warp-uniform
                    const float gate = __shfl_sync(0xffffffffu, c < 32 ? gsa : gsb, c & 31);
                    if (drow < Mrows)
                        out[(int64_t)(tl.row0 + c) * Mrows + drow] = __float2bfloat16_rn(acc_g[c] * gate);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kFp8TmemCols);
    }
}

constexpr int kFp8SmemBytes = kGemmSmemBytes + 4 * kFp8TileRows * 4;
static_assert(kFp8SmemBytes <= 227 * 1024, "shared memory budget (fp8)");

}  // namespace moe
