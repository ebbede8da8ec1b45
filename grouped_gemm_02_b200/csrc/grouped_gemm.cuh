// grouped_gemm.cuh -- persistent tcgen05/TMEM grouped expert GEMM fed by TMA (S5, S5', S6, S7).
//
// The two expert GEMMs of the layer (Decoding the Skew, abstract: "sparse
// expert GEMMs whose shapes vary with the runtime routing distribution";
// GC-MoE, abstract: operand-swapped tcgen05 MMA with a fused SwiGLU and
// optional shared experts):
//
//   gate/up (GATED):  h[r, :]   = silu(xp[r] W1[e]^T) * (xp[r] W3[e]^T)   -> bf16
//   down:             y_p[r, :] = w[perm[r]] * (h[r] W2[e]^T)             -> bf16
//
// for every row r of expert e's segment.  The MMA is operand-swapped: the
// weights fill the M = 128 slot and the expert's tokens the N slot (16..256,
// chosen per expert from its live count by the plan), so a decode expert with
// 3 tokens costs one 16-wide MMA column block while a hot expert gets 256-wide
// tiles.  For the gate/up GEMM one A tile holds 64 rows of W1 and the same 64
// rows of W3, interleaved 16 rows at a time (rows 32q..32q+15 = W1, 32q+16..
// 32q+31 = W3 for f rows 16q..16q+15), so that in TMEM lane quadrant q the
// lanes 0-15 hold the gate and lanes 16-31 the up projection of the same f
// rows; one shuffle pairs them in the epilogue.
//
// Warp roles (192 threads, one CTA per SM, persistent over the tile list):
//   warp 0     TMA producer (one elected lane) -> ring of smem stages
//   warp 1     TMEM allocator + MMA issuer (one elected lane)
//   warps 2-5  epilogue: tcgen05.ld -> SwiGLU or gate scale -> bf16 -> global
// Two TMEM accumulators of 256 columns let the epilogue of tile i overlap the
// mainloop of tile i+1.  Every wait is bounded: on timeout the kernel sets
// DEVERR_TIMEOUT, drains its own copies and MMAs (again bounded), frees TMEM
// and returns.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kGemmThreads = 192;
constexpr int kBlockK = 64;                          // bf16 elements per 128-byte swizzle row
constexpr int kATileBytes = 128 * kBlockK * 2;       // 16 KB: 128 weight rows
constexpr int kBRowBytes = kBlockK * 2;              // 128 B per token row
constexpr int kMaxStages = 12;
constexpr int kRingBytes = 216 * 1024;
constexpr int kBarBytes = 512;
constexpr int kGemmSmemBytes = 1024 + kRingBytes + kBarBytes;
constexpr uint32_t kTmemCols = 512;                  // 2 accumulators x 256 columns
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;   // 1 s

struct GemmArgs {
    const int32_t* plan;        // PlanHeader + PlanArrays (device)
    int E;                      // routed experts; group E is the shared expert
    int M, M_shared;            // output rows per expert: f (gate/up) or d (down); shared: f_shared or d
    int K, K_shared;            // reduction length: d (gate/up) or f / f_shared (down)
    bf16* out;                  // h [pairs, f] or y_p [pairs, d]
    int ld_out;
    bf16* out_shared;           // hs [T, f_shared] or ys [T, d]
    int ld_out_shared;
    const int32_t* perm;        // down GEMM: gate of row r is gate_w[perm[r]]
    const float* gate_w;
    uint32_t* err;
};

struct Tile {
    int group, m, row0, rows, n_mma, K;
    bool shared;
};

__device__ __forceinline__ Tile decode_tile(const int32_t* plan, int nb, int t, bool gated, const GemmArgs& a)
{
    const PlanArrays pa = plan_arrays(const_cast<int32_t*>(plan));
    const int32_t* tb = gated ? pa.tb1 : pa.tb2;
    int lo = 0, hi = nb - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(tb + mid) <= t) lo = mid;
        else hi = mid - 1;
    }
    const int local = t - __ldg(tb + lo);
    const int units = __ldg(pa.units + lo);
    const int chunk = __ldg(pa.chunk + lo);
    Tile tl;
    tl.group = __ldg(pa.group + lo);
    tl.shared = tl.group == a.E;
    tl.m = local / units;
    const int u = local - tl.m * units;
    const int start = u * chunk;
    tl.rows = min(chunk, __ldg(pa.rows + lo) - start);
    tl.row0 = __ldg(pa.row0 + lo) + start;
    tl.n_mma = (tl.rows + 15) & ~15;
    tl.K = tl.shared ? a.K_shared : a.K;
    return tl;
}

struct SmemCtl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(SmemCtl) <= kBarBytes, "control block too large");

// Spin on an mbarrier phase with a deadline.  Returns false (and flags the
// whole CTA) when the deadline passes or another role already gave up.
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, SmemCtl* ctl, uint32_t* err)
{
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 256; i++)
            if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
        if (ptx::globaltimer() - t0 > kWaitTimeoutNs) {
            *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
            atomicOr(err, DEVERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

template <bool GATED>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mA1,
                        const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mA0s,
                        const __grid_constant__ CUtensorMap mA1s, const __grid_constant__ CUtensorMap mBs,
                        const GemmArgs args)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + kRingBytes);
    const uint32_t ring = ptx::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(args.plan);
    const int nb = hdr->n_blocks;
    const int total = GATED ? hdr->tiles1 : hdr->tiles2;
    const int n_max = max(16, hdr->n_max);
    const uint32_t stage_bytes = kATileBytes + (uint32_t)n_max * kBRowBytes;
    const int stages = min(kMaxStages, (int)(kRingBytes / stage_bytes));

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; s++) {
            ptx::mbar_init(ptx::smem_u32(&ctl->full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&ctl->empty[s]), 1);
        }
        for (int a = 0; a < 2; a++) {
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
        ptx::tmem_alloc(ptx::smem_u32(&ctl->tmem_base), kTmemCols);
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
            int s = 0;
            uint32_t ph = 0;
            uint32_t armed = 0, armed_ph = 0;   // slots with a load issued, and its phase
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const Tile tl = decode_tile(args.plan, nb, t, GATED, args);
                const CUtensorMap* a0 = tl.shared ? &mA0s : &mA0;
                const CUtensorMap* a1 = tl.shared ? &mA1s : &mA1;
                const CUtensorMap* b = tl.shared ? &mBs : &mB;
                const int Mrows = tl.shared ? args.M_shared : args.M;
                const int a_row = (tl.shared ? 0 : tl.group * Mrows) + tl.m * (GATED ? 64 : 128);
                const uint32_t tx = kATileBytes + (uint32_t)tl.n_mma * kBRowBytes;
                const int nk = (tl.K + kBlockK - 1) / kBlockK;
                for (int kb = 0; kb < nk; kb++) {
                    if (!bounded_wait(ptx::smem_u32(&ctl->empty[s]), ph ^ 1u, ctl, args.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = ptx::smem_u32(&ctl->full[s]);
                    ptx::mbar_arrive_expect_tx(full, tx);
                    armed |= 1u << s;
                    armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                    const uint32_t a_dst = ring + (uint32_t)s * stage_bytes;
                    const uint32_t b_dst = a_dst + kATileBytes;
                    const int kc = kb * kBlockK;
                    if (GATED) {
#pragma unroll
                        for (int q = 0; q < 4; q++) {
                            ptx::tma_load_2d(a_dst + (32 * q) * 128, a0, full, kc, a_row + 16 * q, pol);
                            ptx::tma_load_2d(a_dst + (32 * q + 16) * 128, a1, full, kc, a_row + 16 * q, pol);
                        }
                    } else {
                        ptx::tma_load_2d(a_dst, a0, full, kc, a_row, pol);
                    }
                    for (int i = 0; i < tl.n_mma / 16; i++)
                        ptx::tma_load_2d(b_dst + i * 16 * kBRowBytes, b, full, kc, tl.row0 + 16 * i, pol);
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                // drain: wait (bounded) for every load this thread issued
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
        // ------------------------------------------------------------ MMA issuer
        if (ptx::elect_one()) {
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t aph = 0;
            bool ok = true, issued = false;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const Tile tl = decode_tile(args.plan, nb, t, GATED, args);
                if (!bounded_wait(ptx::smem_u32(&ctl->tempty[acc]), aph ^ 1u, ctl, args.err)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * 256u;
                const uint32_t idesc = ptx::idesc_bf16_f32(128, (uint32_t)tl.n_mma);
                const int nk = (tl.K + kBlockK - 1) / kBlockK;
                for (int kb = 0; kb < nk; kb++) {
                    if (!bounded_wait(ptx::smem_u32(&ctl->full[s]), ph, ctl, args.err)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ring + (uint32_t)s * stage_bytes;
                    const uint32_t b_addr = a_addr + kATileBytes;
#pragma unroll
                    for (int kk = 0; kk < kBlockK / 16; kk++) {
                        ptx::mma_bf16_ss(d_tmem, ptx::sw128_kmajor_desc(a_addr + kk * 32),
                                         ptx::sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0);
                    }
                    issued = true;
                    ptx::mma_commit(ptx::smem_u32(&ctl->empty[s]));
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                ptx::mma_commit(ptx::smem_u32(&ctl->tfull[acc]));
                acc ^= 1;
                if (acc == 0) aph ^= 1u;
            }
            if (!ok && issued) {
                // drain: every MMA issued so far completes before TMEM is freed
                ptx::mma_commit(ptx::smem_u32(&ctl->drain));
                const uint64_t t0 = ptx::globaltimer();
                while (!ptx::mbar_try_wait(ptx::smem_u32(&ctl->drain), 0) &&
                       ptx::globaltimer() - t0 < kWaitTimeoutNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2-5)
        const int quad = warp & 3;            // TMEM lane quadrant this warp may access
        int acc = 0;
        uint32_t aph = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const Tile tl = decode_tile(args.plan, nb, t, GATED, args);
            const bool ok = bounded_wait(ptx::smem_u32(&ctl->tfull[acc]), aph, ctl, args.err);
            if (!__all_sync(0xffffffffu, ok)) break;   // the whole warp leaves together
            ptx::tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t)acc * 256u + ((uint32_t)(quad * 32) << 16);
            bf16* out = tl.shared ? args.out_shared : args.out;
            const size_t ld = (size_t)(tl.shared ? args.ld_out_shared : args.ld_out);
            const int Mrows = tl.shared ? args.M_shared : args.M;
            for (int c0 = 0; c0 < tl.n_mma; c0 += 16) {
                uint32_t v[16];
                ptx::tmem_ld16(taddr + (uint32_t)c0, v);
                ptx::tmem_ld_wait();
                if (GATED) {
                    // lanes 0-15: gate of f row 16*quad + lane; lanes 16-31: up of the same row
                    const int half = lane >> 4;
                    const int frow = tl.m * 64 + quad * 16 + (lane & 15);
#pragma unroll
                    for (int p = 0; p < 8; p++) {
                        const float send = __uint_as_float(half ? v[2 * p] : v[2 * p + 1]);
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
                        const float g = half ? recv : __uint_as_float(v[2 * p]);
                        const float u = half ? __uint_as_float(v[2 * p + 1]) : recv;
                        const int col = c0 + 2 * p + half;
                        if (col < tl.rows && frow < Mrows)
                            out[(size_t)(tl.row0 + col) * ld + frow] = __float2bfloat16_rn(silu_f(g) * u);
                    }
                } else {
                    const int drow = tl.m * 128 + quad * 32 + lane;
                    const int my_col = c0 + (lane & 15);
                    float my_scale = 1.0f;
                    if (!tl.shared && my_col < tl.rows) my_scale = __ldg(args.gate_w + __ldg(args.perm + tl.row0 + my_col));
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const float sc = __shfl_sync(0xffffffffu, my_scale, j);
                        const int col = c0 + j;
                        if (col < tl.rows && drow < Mrows)
                            out[(size_t)(tl.row0 + col) * ld + drow] = __float2bfloat16_rn(__uint_as_float(v[j]) * sc);
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&ctl->tempty[acc]));
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace moe
