// moe_capi.cu -- the C ABI declared in include/moe.h: host-side argument
// checks, workspace layout, TMA tensor maps and kernel launches.  No entry
// point allocates, frees or synchronises (moe_get_device_error excepted).
//
// Every kernel is launched with programmatic stream serialisation: it may
// start while the previous kernel on the stream drains, waits
// (griddepcontrol.wait) before touching that kernel's outputs, and lets its
// own successor start only after that wait.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/moe.h"
#include "common.cuh"
#include "fp8.cuh"
#include "grouped_gemm.cuh"
#include "permute.cuh"
#include "ptx.cuh"
#include "route.cuh"
#include "schedule.h"
#include "tile_table.h"

using namespace moe;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
    bool ready = false;
    bool supported = false;
    int sm_count = 0;
    int pair_grid = 0;       // CTAs of a CTA-pair GEMM launch: 2 x the clusters that fit at once (0: none)
    int fp8_pair_grid = 0;   // the same for the FP8 / FP4 GEMM
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::atomic<int64_t> g_launches{0};
thread_local int64_t t_launches = 0;   // kernels this host thread has launched (orders a layer's launches)
thread_local cudaEvent_t t_phase[6] = {};
thread_local bool t_phase_armed = false;

inline void phase_mark(bool on, int i, cudaStream_t st)
{
    if (on) cudaEventRecord(t_phase[i], st);
}

// Launch with programmatic stream serialisation (see the file comment).
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    ++t_launches;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same with clusters of two CTAs (the CTA-pair GEMMs).
template <typename... KArgs, typename... Args>
cudaError_t launch_pair(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                        Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    ++t_launches;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// How many clusters of two CTAs of `kernel` can be resident at once (0 on error).
template <typename... KArgs>
int max_pair_clusters(void (*kernel)(KArgs...), size_t smem, int threads = kGemmThreads)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

// Per-device one-time set-up: architecture check, SM count, kernel attributes.
int device_setup(DeviceState** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& st = g_dev[dev];
    if (!st.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        st.supported = (major == 10 && minor == 0);
        st.sm_count = sms;
        if (st.supported) {
            if (cudaFuncSetAttribute(grouped_gemm_kernel<MODE_GATED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kGemmSmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_kernel<MODE_DOWN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kGemmSmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_kernel<MODE_ROUTER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kGemmSmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_kernel<MODE_FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kGemmSmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_GATED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_DOWN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_GATED, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_DOWN, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_FUSED, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_GATED, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_DOWN, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_GATED, true, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_fp8_kernel<FP8_DOWN, true, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kFp8SmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_kernel<MODE_GATED, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_kernel<MODE_DOWN, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(grouped_gemm_kernel<MODE_FUSED, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) != cudaSuccess)
                return MOE_ERR_CUDA;
            // CTA pairs: a grid of exactly the clusters that fit at once, so the
            // persistent pairs all start together (the same count for every mode)
            int pc = max_pair_clusters(grouped_gemm_kernel<MODE_GATED, true>, kGemmSmemBytes);
            pc = std::min(pc, max_pair_clusters(grouped_gemm_kernel<MODE_DOWN, true>, kGemmSmemBytes));
            pc = std::min(pc, max_pair_clusters(grouped_gemm_kernel<MODE_FUSED, true>, kGemmSmemBytes));
            st.pair_grid = 2 * std::min(pc, sms / 2);
            int pc8 = max_pair_clusters(grouped_gemm_fp8_kernel<FP8_GATED, false, true>, kFp8SmemBytes, kFp8Threads);
            pc8 = std::min(pc8, max_pair_clusters(grouped_gemm_fp8_kernel<FP8_DOWN, false, true>, kFp8SmemBytes,
                                                  kFp8Threads));
            pc8 = std::min(pc8, max_pair_clusters(grouped_gemm_fp8_kernel<FP8_GATED, true, true>, kFp8SmemBytes,
                                                  kFp8Threads));
            pc8 = std::min(pc8, max_pair_clusters(grouped_gemm_fp8_kernel<FP8_DOWN, true, true>, kFp8SmemBytes,
                                                  kFp8Threads));
            st.fp8_pair_grid = 2 * std::min(pc8, sms / 2);
            if (!g_encode) {
                cudaDriverEntryPointQueryResult q;
                void* fn = nullptr;
                if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                        cudaSuccess ||
                    q != cudaDriverEntryPointSuccess || !fn)
                    return MOE_ERR_CUDA;
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            }
        }
        st.ready = true;
    }
    if (!st.supported) return MOE_ERR_DEVICE;
    *out = &st;
    return MOE_OK;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline int status_of(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Common size checks.
int check_sizes(int64_t T, int64_t d, int64_t E, int64_t k)
{
    if (T < 0 || d <= 0 || E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK || k > E) return MOE_ERR_ARG;
    if (T * k >= (int64_t(1) << 31) || T >= (int64_t(1) << 31)) return MOE_ERR_ARG;
    if (d % 64 != 0) return MOE_ERR_ALIGN;
    return MOE_OK;
}

// 2-D bf16 tensor map over a row-major [rows, inner] matrix; box = [64, box_rows],
// 128-byte swizzle, zero fill outside the matrix.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows)
{
    if (rows == 0) rows = 1;   // a map needs one row; such a map is never read
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D byte (e4m3) tensor map over a row-major [rows, inner] matrix; box = [128, box_rows].
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows)
{
    if (rows == 0) rows = 1;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over packed e2m1 (FP4) rows [rows, inner elements], inner / 2 bytes a
// row; box = [128 elements, box_rows].  The TMA unpacks each 16 elements (8
// bytes) into 16 bytes of shared memory, the row layout an e4m3 tile takes, for
// the block-scaled MMA to read as e2m1.
bool make_map_u4(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows)
{
    if (rows == 0) rows = 1;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner / 2};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 tensor map over a row-major [rows, inner] matrix; box = [128, 1], no swizzle.
bool make_map_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows)
{
    if (rows == 0) rows = 1;
    if (inner == 0) inner = 4;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 4};
    cuuint32_t box[2] = {128, 1};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class T>
T* at(void* ws, size_t off)
{
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// ---------------------------------------------------------------- step launchers
// Router logits on the tensor cores (MODE_ROUTER), split over K when the
// tokens alone cannot fill the SMs.  Leaves either the logits (+ bias) in
// `logits` (splits == 1) or fp32 partials in `partials`; reports the split.
int run_router_gemm(const bf16* x, const bf16* Wg, const float* bias, int T, int d, int E, float* logits,
                    float* partials, uint32_t* err, int sms, cudaStream_t st, RouterSplit* out)
{
    const RouterSplit rs = router_split(T, d, E);
    *out = rs;
    CUtensorMap a, b, b64;
    if (!make_map(&a, Wg, d, E, 128) || !make_map(&b, x, d, T, 16) || !make_map(&b64, x, d, T, 64))
        return MOE_ERR_CUDA;
    GemmArgs g{};
    g.E = E;
    g.M = E;
    g.M_shared = E;
    g.K = d;
    g.K_shared = d;
    g.T = T;
    g.units = rs.units;
    g.chunk = rs.chunk;
    g.mt = rs.mt;
    g.splits = rs.splits;
    g.kb_per = rs.kb_per;
    g.out_f32 = rs.splits > 1 ? partials : logits;
    g.bias = bias;
    g.err = err;
    const int grid = std::min(sms, rs.tiles);
    return status_of(launch(grouped_gemm_kernel<MODE_ROUTER>, dim3(grid), dim3(kGemmThreads), kGemmSmemBytes, st,
                            a, a, b, a, a, b, a, b, a, b, b64, b64, b64, b64, b, g, g));
}

// Top-k over the router's output: the logits themselves, or the split-K
// partials (then the sums, + bias, are also stored in `logits`).
struct TopkSource {
    const float* src;
    size_t stride;
    int splits;
    const float* bias;
    float* logits_out;
};

TopkSource topk_source(const RouterSplit& rs, float* logits, float* partials, const float* bias, int T, int E)
{
    if (rs.splits > 1) return {partials, (size_t)T * E, rs.splits, bias, logits};
    return {logits, 0, 1, nullptr, nullptr};
}

int run_topk(const TopkSource& s, int T, int E, int k, int32_t* idx, float* w, uint32_t* err, cudaStream_t st)
{
    if (s.splits > 1) {
        // split router: one CTA per token, one thread per expert sums the partials
        const int threads = (E + 31) / 32 * 32;
        return status_of(launch(topk_token_cta_kernel, dim3(T), dim3(threads), 0, st, s.src, s.stride, s.splits,
                                s.bias, T, E, k, s.logits_out, idx, w, err));
    }
    return status_of(launch(topk_softmax_kernel, dim3((T + 7) / 8), dim3(256), 0, st, s.src, s.stride, s.splits,
                            s.bias, T, E, k, s.logits_out, idx, w, err));
}

// Blocks of 8 warps for a token-order row gather over T tokens of `nvec`
// 16-byte vectors a row: one warp per (token, 32-vector chunk), at most 16
// blocks per SM (the kernel strides over the rest).
int gather_blocks(int64_t T, int nvec, int sms)
{
    const int64_t warps = T * ((nvec + 31) / 32);
    return (int)std::max<int64_t>(1, std::min<int64_t>((warps + 7) / 8, (int64_t)sms * 16));
}

// The general (multi-CTA) histogram / scan / scatter (/ gather of bf16 rows
// into xp when xp is given).  `ps` shapes the tile plan.
int run_permute(const int32_t* idx, const bf16* x, int T, int d, int E, int k, int32_t* counts, int32_t* offsets,
                int32_t* perm, int32_t* inv_perm, bf16* xp, uint32_t* err, int32_t* block_counts, int32_t* plan,
                int f, int shared_rows, int fs, int sms, cudaStream_t st, PlanShape ps,
                int64_t* inv_perm_launch = nullptr)
{
    const int64_t P = (int64_t)T * k;
    const int nb = hist_blocks(P);
    cudaError_t e = launch(hist_kernel, dim3(nb), dim3(512), 0, st, idx, P, E, block_counts, err);
    if (e == cudaSuccess)
        e = launch(scan_kernel, dim3(1), dim3(1024), 0, st, block_counts, nb, E, counts, offsets, plan, f, d,
                   shared_rows, fs, ps);
    if (e == cudaSuccess)
        e = launch(scatter_kernel, dim3(nb), dim3(256), 0, st, idx, P, E, (const int32_t*)block_counts, perm,
                   inv_perm);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (inv_perm_launch) *inv_perm_launch = t_launches;
    if (!xp) return MOE_OK;
    return status_of(launch(gather_rows_kernel, dim3(gather_blocks(T, d / 8, sms)), dim3(256), 0, st, x,
                            (const int32_t*)inv_perm, T, k, d, xp));
}

struct GemmOperands {
    const bf16 *xp, *x, *W1, *W3, *W2, *Ws1, *Ws3, *Ws2;
    const int32_t* perm;
    const float* gate_w;
    bf16 *h, *y_p, *hs, *ys;
    int T, P, d, f, fs, E, k;
    bool gather;   // gate/up token rows straight from x through perm (no xp)
};

// Process-wide choices of the expert-GEMM launch form (moe_set_policy; -1 =
// the library's rule).  Their first values come from MOE_GEMM_SPLIT (0: one
// launch, 1: two) and MOE_GEMM_PAIR (0/1) when those are set.
std::atomic<int> g_policy_fused{-2};
std::atomic<int> g_policy_pair{-2};
std::atomic<int> g_policy_tiles{-1};   // 1: token buckets; otherwise the histogram-matched table
std::atomic<int> g_policy_cap{-1};     // > 0: every plan cut under this cap (tuning)
std::atomic<int> g_policy_gather{-1};  // 1: the gate/up GEMM gathers token rows from x (no gather launch)

int env_switch(const char* name)
{
    const char* e = getenv(name);
    return (e && (e[0] == '0' || e[0] == '1')) ? e[0] - '0' : -1;
}

int policy(std::atomic<int>& slot, const char* env, bool invert)
{
    int v = slot.load(std::memory_order_relaxed);
    if (v == -2) {
        int e = env_switch(env);
        if (e >= 0 && invert) e = 1 - e;
        int expect = -2;
        slot.compare_exchange_strong(expect, e);
        v = slot.load(std::memory_order_relaxed);
    }
    return v;
}

// One launch for both expert GEMMs (down tiles wait on per-block counters of
// finished gate/up tiles) or two launches with a kernel boundary between them.
// Measured on B200: the single launch saves the boundary's tail when few
// token-expert pairs spread over many weight tiles (P <= 256 with f <= 4096:
// 3-5% faster), and loses 4-10% once blocks hold more tokens, where the down
// tiles' waits on the counters cost more than the boundary.
bool gemm_fused(int P, int f)
{
    const int forced = policy(g_policy_fused, "MOE_GEMM_SPLIT", /*invert=*/true);
    if (forced >= 0) return forced == 1;
    return P <= 256 && f <= 4096;
}

// CTA pairs (cta_group::2, 2 x 128 weight rows per tile, each SM loading half
// of the token tile) halve each SM's operand traffic per MMA, which is what
// limits the single-CTA tiles once experts hold hundreds of tokens; they are
// taken whenever both expert GEMMs run as two launches (P > 256 or f > 4096)
// and the device can hold the pair grid.
bool gemm_pair(int P, int f, const DeviceState* dev)
{
    if (dev->pair_grid < 2) return false;
    const int forced = policy(g_policy_pair, "MOE_GEMM_PAIR", /*invert=*/false);
    if (forced >= 0) return forced == 1;
    return !gemm_fused(P, f);
}

constexpr PlanShape kPlanSingle{kTileRows, 64, 128, 16, 0, kTilesMatched};
constexpr PlanShape kPlanPair{kTileRows, 128, 256, 32, 1, kTilesMatched};
constexpr int kTokenBucketWidth[kTokenBuckets] = MOE_TOKEN_BUCKET_WIDTH;

// The plan shape of a launch form under the current tile policy: the
// histogram-matched table (the default; the device picks the cap), the
// token-bucket widths chosen from T alone, or a forced cap.
PlanShape plan_shape(PlanShape ps, int64_t T)
{
    const int cap = g_policy_cap.load(std::memory_order_relaxed);
    if (g_policy_tiles.load(std::memory_order_relaxed) == 1) {
        // token buckets: the width of T's bucket, or the forced cap as the one width
        ps.policy = kTilesBucket;
        ps.unit_rows = std::min(cap > 0 ? cap : kTokenBucketWidth[token_bucket(T)], ps.unit_rows);
    } else if (cap > 0) {
        ps.policy = kTilesCap;
        ps.unit_rows = std::min(cap, ps.unit_rows);
    } else {
        ps.policy = kTilesMatched;
    }
    ps.unit_rows = std::max(ps.align, ps.unit_rows / ps.align * ps.align);
    return ps;
}

// plan_ready: the plan was written two or more launches before the gate/up GEMM.
// pair: the plan was cut for CTA pairs (kPlanPair) and the pair kernels run.
int run_gemms(const GemmOperands& o, const int32_t* plan, bool plan_ready, uint32_t* err, const DeviceState* dev,
              bool pair, cudaStream_t st, bool prof = false)
{
    const int sms = dev->sm_count;
    CUtensorMap a0, a1, b, a0s, a1s, bs, a2, b2, a2s, b2s, b64, bs64, b264, b2s64, bx;
    const uint64_t E = (uint64_t)o.E;
    // the row gather of the gate/up tokens: x with one-row boxes
    if (!make_map(&bx, o.x, o.d, (uint64_t)o.T, 1)) return MOE_ERR_CUDA;
    // gate/up: A = 64 rows of W1 and the same 64 rows of W3 (64-row boxes), B = xp rows
    // (64- and 16-row boxes); shared: Ws1/Ws3 and x
    if (!make_map(&a0, o.W1, o.d, E * o.f, 64) || !make_map(&a1, o.W3, o.d, E * o.f, 64) ||
        !make_map(&b, o.xp, o.d, (uint64_t)o.P, 16) || !make_map(&b64, o.xp, o.d, (uint64_t)o.P, 64))
        return MOE_ERR_CUDA;
    // down: A = W2 rows (128-row boxes), B = h rows; shared: Ws2 and hs
    if (!make_map(&a2, o.W2, o.f, E * o.d, 128) || !make_map(&b2, o.h, o.f, (uint64_t)o.P, 16) ||
        !make_map(&b264, o.h, o.f, (uint64_t)o.P, 64))
        return MOE_ERR_CUDA;
    if (o.fs > 0) {
        if (!make_map(&a0s, o.Ws1, o.d, o.fs, 64) || !make_map(&a1s, o.Ws3, o.d, o.fs, 64) ||
            !make_map(&bs, o.x, o.d, (uint64_t)o.T, 16) || !make_map(&bs64, o.x, o.d, (uint64_t)o.T, 64) ||
            !make_map(&a2s, o.Ws2, o.fs, o.d, 128) || !make_map(&b2s, o.hs, o.fs, (uint64_t)o.T, 16) ||
            !make_map(&b2s64, o.hs, o.fs, (uint64_t)o.T, 64))
            return MOE_ERR_CUDA;
    } else {
        a0s = a0;
        a1s = a1;
        bs = b;
        bs64 = b64;
        a2s = a2;
        b2s = b2;
        b2s64 = b264;
    }
    GemmArgs g1{};
    g1.plan = plan;
    g1.plan_ready = plan_ready ? 1 : 0;
    g1.E = o.E;
    g1.M = o.f;
    g1.M_shared = o.fs;
    g1.K = o.d;
    g1.K_shared = o.d;
    g1.out = o.h;
    g1.ld_out = o.f;
    g1.out_shared = o.hs;
    g1.ld_out_shared = o.fs;
    g1.perm = o.perm;
    g1.gate_w = o.gate_w;
    g1.err = err;
    g1.gather_perm = o.gather ? o.perm : nullptr;
    g1.gather_k = o.k;
    GemmArgs g2 = g1;
    g2.gather_perm = nullptr;
    g2.M = o.d;
    g2.M_shared = o.d;
    g2.K = o.f;
    g2.K_shared = o.fs;
    g2.out = o.y_p;
    g2.ld_out = o.d;
    g2.out_shared = o.ys;
    g2.ld_out_shared = o.d;
    const dim3 grid(pair ? dev->pair_grid : sms), block(kGemmThreads);
    if (gemm_fused(o.P, o.f)) {
        // a gate/up tile streams d/64 k-blocks, a down tile f/64
        const int kb1 = (o.d + 63) / 64, kb2 = (o.f + 63) / 64;
        g1.comp = std::max(1, (kb1 + kb2 / 2) / kb2);
        const cudaError_t e =
            pair ? launch_pair(grouped_gemm_kernel<MODE_FUSED, true>, grid, block, kGemmSmemBytes, st, a0, a1, b, a0s,
                               a1s, bs, a2, b2, a2s, b2s, b64, bs64, b264, b2s64, bx, g1, g2)
                 : launch(grouped_gemm_kernel<MODE_FUSED>, grid, block, kGemmSmemBytes, st, a0, a1, b, a0s, a1s, bs,
                          a2, b2, a2s, b2s, b64, bs64, b264, b2s64, bx, g1, g2);
        phase_mark(prof, 3, st);   // the fused launch has no boundary: the down phase reads as zero
        return status_of(e);
    }
    const cudaError_t e1 =
        pair ? launch_pair(grouped_gemm_kernel<MODE_GATED, true>, grid, block, kGemmSmemBytes, st, a0, a1, b, a0s,
                           a1s, bs, a0, b, a0, b, b64, bs64, b64, bs64, bx, g1, g1)
             : launch(grouped_gemm_kernel<MODE_GATED>, grid, block, kGemmSmemBytes, st, a0, a1, b, a0s, a1s, bs, a0,
                      b, a0, b, b64, bs64, b64, bs64, bx, g1, g1);
    if (e1 != cudaSuccess) return MOE_ERR_CUDA;
    phase_mark(prof, 3, st);
    g2.plan_ready = 1;   // written before the gate/up GEMM
    return status_of(pair ? launch_pair(grouped_gemm_kernel<MODE_DOWN, true>, grid, block, kGemmSmemBytes, st, a2, a2,
                                        b2, a2s, a2s, b2s, a2, b2, a2s, b2s, b264, b2s64, b264, b2s64, bx, g2, g2)
                          : launch(grouped_gemm_kernel<MODE_DOWN>, grid, block, kGemmSmemBytes, st, a2, a2, b2, a2s,
                                   a2s, b2s, a2, b2, a2s, b2s, b264, b2s64, b264, b2s64, bx, g2, g2));
}

// inv_perm_launch: this thread's launch count right after the kernel that wrote
// inv_perm (0: unknown).  The combine may read inv_perm before its
// griddepcontrol.wait only when two or more launches separate it from that
// kernel: every kernel waits before it lets its successor start, so the
// writer has then completed before the combine begins.
int run_combine(const bf16* y_p, const int32_t* inv_perm, const bf16* ys, int T, int k, int d, bf16* out,
                cudaStream_t st, int64_t inv_perm_launch = 0)
{
    const bool inv_perm_ready = inv_perm_launch > 0 && t_launches - inv_perm_launch >= 2;
    constexpr int kThreads = 64;
    const int nvec = d / 8;
    const int gy = std::max(1, std::min((nvec + kThreads - 1) / kThreads, 65535));
    return status_of(launch(combine_kernel, dim3(T, gy), dim3(kThreads), 0, st, y_p, inv_perm, ys, T, k, d, out,
                            inv_perm_ready ? 1 : 0));
}

}  // namespace

extern "C" {

int moe_workspace_size(int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, int64_t f_shared, size_t* bytes)
{
    if (!bytes || T < 0 || d < 0 || f < 0 || E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK || f_shared < 0)
        return MOE_ERR_ARG;
    *bytes = ws_layout(T, d, f, E, k, f_shared).total;
    return MOE_OK;
}

int moe_workspace_init(void* ws, size_t ws_bytes, int64_t T, int64_t E, int64_t k, void* stream)
{
    if (!ws || T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK) return MOE_ERR_ARG;
    const WsLayout L = ws_layout(T, 0, 0, E, k, 0);
    if (ws_bytes < L.ctrl_end) return MOE_ERR_WS;
    return cudaMemsetAsync(ws, 0, L.ctrl_end, as_stream(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_route(const moe_bf16* x, const moe_bf16* Wg, const float* bias, int64_t T, int64_t d, int64_t E, int64_t k,
              float* logits, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream)
{
    int rc = check_sizes(T, d, E, k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!x || !Wg || !logits || !topk_idx || !topk_w || !ws) return MOE_ERR_ARG;
    if (!al16(x) || !al16(Wg) || !al16(ws)) return MOE_ERR_ALIGN;
    const WsLayout L = ws_layout(T, d, 0, E, k, 0);
    if (ws_bytes < L.ctrl_end) return MOE_ERR_WS;
    DeviceState* dev;
    if ((rc = device_setup(&dev))) return rc;
    cudaStream_t st = as_stream(stream);
    uint32_t* err = at<uint32_t>(ws, L.err);
    float* partials = at<float>(ws, L.router_partials);
    RouterSplit rs;
    if ((rc = run_router_gemm(reinterpret_cast<const bf16*>(x), reinterpret_cast<const bf16*>(Wg), bias, (int)T,
                              (int)d, (int)E, logits, partials, err, dev->sm_count, st, &rs)))
        return rc;
    return run_topk(topk_source(rs, logits, partials, bias, (int)T, (int)E), (int)T, (int)E, (int)k, topk_idx, topk_w,
                    err, st);
}

int moe_topk(const float* logits, int64_t T, int64_t E, int64_t k, int32_t* topk_idx, float* topk_w, void* ws,
             void* stream)
{
    int rc = check_sizes(T, 64, E, k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!logits || !topk_idx || !topk_w || !ws) return MOE_ERR_ARG;
    DeviceState* dev;
    if ((rc = device_setup(&dev))) return rc;
    const TopkSource s{logits, 0, 1, nullptr, nullptr};
    return run_topk(s, (int)T, (int)E, (int)k, topk_idx, topk_w, at<uint32_t>(ws, 0), as_stream(stream));
}

int moe_permute(const int32_t* topk_idx, const moe_bf16* x, int64_t T, int64_t d, int64_t E, int64_t k,
                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm, moe_bf16* xp, void* ws,
                size_t ws_bytes, void* stream)
{
    int rc = check_sizes(T, d, E, k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!topk_idx || !x || !counts || !offsets || !perm || !inv_perm || !xp || !ws) return MOE_ERR_ARG;
    if (!al16(x) || !al16(xp) || !al16(ws)) return MOE_ERR_ALIGN;
    const WsLayout L = ws_layout(T, d, 0, E, k, 0);
    if (ws_bytes < L.ctrl_end) return MOE_ERR_WS;
    DeviceState* dev;
    if ((rc = device_setup(&dev))) return rc;
    return run_permute(topk_idx, reinterpret_cast<const bf16*>(x), (int)T, (int)d, (int)E, (int)k, counts, offsets,
                       perm, inv_perm, reinterpret_cast<bf16*>(xp), at<uint32_t>(ws, L.err),
                       at<int32_t>(ws, L.block_counts), nullptr, 0, 0, 0, dev->sm_count, as_stream(stream),
                       kPlanSingle);
}

int moe_grouped_gemm(const moe_bf16* xp, const int32_t* counts, const int32_t* offsets, const int32_t* perm,
                     const float* topk_w, const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2, int64_t T,
                     int64_t d, int64_t f, int64_t E, int64_t k, moe_bf16* h, moe_bf16* y_p, void* ws,
                     size_t ws_bytes, void* stream)
{
    int rc = check_sizes(T, d, E, k);
    if (rc) return rc;
    if (f <= 0) return MOE_ERR_ARG;
    if (f % 64 != 0) return MOE_ERR_ALIGN;
    if (T == 0) return MOE_OK;
    if (!xp || !counts || !offsets || !perm || !topk_w || !W1 || !W3 || !W2 || !h || !y_p || !ws) return MOE_ERR_ARG;
    if (!al16(xp) || !al16(W1) || !al16(W3) || !al16(W2) || !al16(h) || !al16(y_p) || !al16(ws)) return MOE_ERR_ALIGN;
    const WsLayout L = ws_layout(T, d, f, E, k, 0);
    if (ws_bytes < L.ctrl_end) return MOE_ERR_WS;
    DeviceState* dev;
    if ((rc = device_setup(&dev))) return rc;
    cudaStream_t st = as_stream(stream);
    int32_t* plan = at<int32_t>(ws, L.plan);
    const bool pair = gemm_pair((int)(T * k), (int)f, dev);
    if (launch(plan_kernel, dim3(1), dim3(1024), 0, st, counts, offsets, (int)E, plan, (int)f, (int)d, 0, 0,
               plan_shape(pair ? kPlanPair : kPlanSingle, T)) != cudaSuccess)
        return MOE_ERR_CUDA;
    GemmOperands o{};
    o.xp = reinterpret_cast<const bf16*>(xp);
    o.x = o.xp;
    o.W1 = reinterpret_cast<const bf16*>(W1);
    o.W3 = reinterpret_cast<const bf16*>(W3);
    o.W2 = reinterpret_cast<const bf16*>(W2);
    o.perm = perm;
    o.gate_w = topk_w;
    o.h = reinterpret_cast<bf16*>(h);
    o.y_p = reinterpret_cast<bf16*>(y_p);
    o.T = (int)T;
    o.P = (int)(T * k);
    o.d = (int)d;
    o.f = (int)f;
    o.fs = 0;
    o.E = (int)E;
    o.k = (int)k;
    o.gather = false;
    return run_gemms(o, plan, /*plan_ready=*/false, at<uint32_t>(ws, L.err), dev, pair, st);
}

int moe_combine(const moe_bf16* y_p, const int32_t* inv_perm, const moe_bf16* shared_out, int64_t T, int64_t k,
                int64_t d, moe_bf16* out, void* stream)
{
    if (T < 0 || k < 1 || k > kMaxTopK || d <= 0 || T * k >= (int64_t(1) << 31)) return MOE_ERR_ARG;
    if (d % 64 != 0) return MOE_ERR_ALIGN;
    if (T == 0) return MOE_OK;
    if (!y_p || !inv_perm || !out) return MOE_ERR_ARG;
    if (!al16(y_p) || !al16(out) || (shared_out && !al16(shared_out))) return MOE_ERR_ALIGN;
    DeviceState* dev;
    int rc;
    if ((rc = device_setup(&dev))) return rc;
    return run_combine(reinterpret_cast<const bf16*>(y_p), inv_perm, reinterpret_cast<const bf16*>(shared_out),
                       (int)T, (int)k, (int)d, reinterpret_cast<bf16*>(out), as_stream(stream));
}

int moe_layer_forward(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const moe_bf16* W1,
                      const moe_bf16* W3, const moe_bf16* W2, const moe_bf16* Ws1, const moe_bf16* Ws3,
                      const moe_bf16* Ws2, int64_t f_shared, int64_t T, int64_t d, int64_t f, int64_t E, int64_t k,
                      moe_bf16* out, void* ws, size_t ws_bytes, void* stream)
{
    int rc = check_sizes(T, d, E, k);
    if (rc) return rc;
    if (f <= 0 || f_shared < 0) return MOE_ERR_ARG;
    if (f % 64 != 0 || f_shared % 64 != 0) return MOE_ERR_ALIGN;
    if (T == 0) return MOE_OK;
    if (!x || !Wg || !W1 || !W3 || !W2 || !out || !ws) return MOE_ERR_ARG;
    if (f_shared > 0 && (!Ws1 || !Ws3 || !Ws2)) return MOE_ERR_ARG;
    if (!al16(x) || !al16(Wg) || !al16(W1) || !al16(W3) || !al16(W2) || !al16(out) || !al16(ws)) return MOE_ERR_ALIGN;
    if (f_shared > 0 && (!al16(Ws1) || !al16(Ws3) || !al16(Ws2))) return MOE_ERR_ALIGN;
    const WsLayout L = ws_layout(T, d, f, E, k, f_shared);
    if (ws_bytes < L.total) return MOE_ERR_WS;
    DeviceState* dev;
    if ((rc = device_setup(&dev))) return rc;
    cudaStream_t st = as_stream(stream);
    uint32_t* err = at<uint32_t>(ws, L.err);
    int32_t* plan = at<int32_t>(ws, L.plan);
    float* logits = at<float>(ws, L.logits);
    float* partials = at<float>(ws, L.router_partials);
    int32_t* idx = at<int32_t>(ws, L.topk_idx);
    float* w = at<float>(ws, L.topk_w);
    int32_t* counts = at<int32_t>(ws, L.counts);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* perm = at<int32_t>(ws, L.perm);
    int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
    bf16* xp = at<bf16>(ws, L.xp);
    bf16* h = at<bf16>(ws, L.h);
    bf16* y_p = at<bf16>(ws, L.y_p);
    bf16* hs = f_shared > 0 ? at<bf16>(ws, L.hs) : nullptr;
    bf16* ys = f_shared > 0 ? at<bf16>(ws, L.ys) : nullptr;
    const bf16* xb = reinterpret_cast<const bf16*>(x);
    const int iT = (int)T, id = (int)d, iE = (int)E, ik = (int)k, shared_rows = f_shared > 0 ? (int)T : 0;

    const bool prof = t_phase_armed;   // the armed events serve this call only
    t_phase_armed = false;
    int64_t inv_perm_launch = 0;
    phase_mark(prof, 0, st);
    RouterSplit rs;
    if ((rc = run_router_gemm(xb, reinterpret_cast<const bf16*>(Wg), bias, iT, id, iE, logits, partials, err,
                              dev->sm_count, st, &rs)))
        return rc;
    const TopkSource src = topk_source(rs, logits, partials, bias, iT, iE);
    const int64_t P = T * k;
    const bool pair = gemm_pair((int)P, (int)f, dev);
    // token rows for the gate/up GEMM: a gather pass into xp (the default), or TMA
    // row gathers from x inside the GEMM (tile::gather4, 4 rows per instruction),
    // which measured slower on B200 at every size: more, smaller TMA requests.
    // The row gathers run only in the two-launch form: in the single launch they
    // gave wrong rows on a layer with several token units per expert and a shared
    // expert (T=2048, E=4, f=128, f_shared=128), a fault not yet traced.
    const bool gather_in_gemm =
        g_policy_gather.load(std::memory_order_relaxed) == 1 && !gemm_fused((int)(T * k), (int)f);
    if ((rc = run_topk(src, iT, iE, ik, idx, w, err, st))) return rc;
    phase_mark(prof, 1, st);
    if (P <= kSmallPairs) {
        // one CTA: histogram, scan, stable ranks and the tile plan
        if (launch(permute_small_kernel, dim3(1), dim3(1024), 0, st, (const int32_t*)idx, (int)P, iE, counts, offsets,
                   perm, inv_perm, plan, (int)f, id, shared_rows, (int)f_shared,
                   plan_shape(pair ? kPlanPair : kPlanSingle, T), err) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        inv_perm_launch = t_launches;
        if (!gather_in_gemm) {
            if (launch(gather_rows_kernel, dim3(gather_blocks(T, d / 8, dev->sm_count)), dim3(256), 0, st, xb,
                       (const int32_t*)inv_perm, iT, ik, id, xp) != cudaSuccess)
                return MOE_ERR_CUDA;
        }
    } else {
        if ((rc = run_permute(idx, xb, iT, id, iE, ik, counts, offsets, perm, inv_perm, gather_in_gemm ? nullptr : xp, err,
                              at<int32_t>(ws, L.block_counts), plan, (int)f, shared_rows, (int)f_shared,
                              dev->sm_count, st, plan_shape(pair ? kPlanPair : kPlanSingle, T), &inv_perm_launch)))
            return rc;
    }
    GemmOperands o{};
    o.xp = xp;
    o.x = xb;
    o.W1 = reinterpret_cast<const bf16*>(W1);
    o.W3 = reinterpret_cast<const bf16*>(W3);
    o.W2 = reinterpret_cast<const bf16*>(W2);
    o.Ws1 = reinterpret_cast<const bf16*>(Ws1);
    o.Ws3 = reinterpret_cast<const bf16*>(Ws3);
    o.Ws2 = reinterpret_cast<const bf16*>(Ws2);
    o.perm = perm;
    o.gate_w = w;
    o.h = h;
    o.y_p = y_p;
    o.hs = hs;
    o.ys = ys;
    o.T = iT;
    o.P = (int)P;
    o.d = id;
    o.f = (int)f;
    o.fs = (int)f_shared;
    o.E = iE;
    o.k = ik;
    o.gather = gather_in_gemm;
    phase_mark(prof, 2, st);
    // the plan is written two or more launches before the GEMM, except when the
    // one-CTA permutation is directly followed by a gathering GEMM
    const bool plan_ready = !gather_in_gemm || P > kSmallPairs;
    if ((rc = run_gemms(o, plan, plan_ready, err, dev, pair, st, prof))) return rc;
    phase_mark(prof, 4, st);
    rc = run_combine(y_p, inv_perm, ys, iT, ik, id, reinterpret_cast<bf16*>(out), st, inv_perm_launch);
    phase_mark(prof, 5, st);
    return rc;
}

int moe_record_phase_events(void* const* events, int n)
{
    if (n == 0) {
        t_phase_armed = false;
        return MOE_OK;
    }
    if (!events || n < 6) return MOE_ERR_ARG;
    for (int i = 0; i < 6; i++) {
        if (!events[i]) return MOE_ERR_ARG;
        t_phase[i] = reinterpret_cast<cudaEvent_t>(events[i]);
    }
    t_phase_armed = true;
    return MOE_OK;
}

int64_t moe_launch_counter(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_set_policy(int what, int value)
{
    switch (what) {
    case MOE_POLICY_ONE_LAUNCH:
    case MOE_POLICY_CTA_PAIRS:
    case MOE_POLICY_TILES:
        if (value < -1 || value > 1) return MOE_ERR_ARG;
        (what == MOE_POLICY_ONE_LAUNCH ? g_policy_fused : what == MOE_POLICY_CTA_PAIRS ? g_policy_pair
                                                                                        : g_policy_tiles)
            .store(value);
        return MOE_OK;
    case MOE_POLICY_GATHER:
        if (value < -1 || value > 1) return MOE_ERR_ARG;
        g_policy_gather.store(value);
        return MOE_OK;
    case MOE_POLICY_TILE_CAP:
        if (value != -1 && (value < 16 || value > kTileRows || value % 16 != 0)) return MOE_ERR_ARG;
        g_policy_cap.store(value);
        return MOE_OK;
    default: return MOE_ERR_ARG;
    }
}

int moe_workspace_tensor(void* ws, int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, int64_t f_shared, int which,
                         void** ptr)
{
    if (!ws || !ptr || T < 0 || d < 0 || f < 0 || E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK || f_shared < 0)
        return MOE_ERR_ARG;
    const WsLayout L = ws_layout(T, d, f, E, k, f_shared);
    const size_t offs[13] = {L.logits, L.topk_idx, L.topk_w, L.counts, L.offsets, L.perm,
                             L.inv_perm, L.xp, L.h, L.y_p, L.hs, L.ys, L.plan};
    if (which < 0 || which >= 13) return MOE_ERR_ARG;
    *ptr = static_cast<uint8_t*>(ws) + offs[which];
    return MOE_OK;
}

int moe_get_device_error(const void* ws, uint32_t* code, void* stream)
{
    if (!ws || !code) return MOE_ERR_ARG;
    cudaStream_t st = as_stream(stream);
    if (cudaMemcpyAsync(code, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_selftest_wait_timeout(void* ws, void* stream)
{
    if (!ws || !al16(ws)) return MOE_ERR_ARG;
    DeviceState* dev;
    int rc;
    if ((rc = device_setup(&dev))) return rc;
    cudaStream_t st = as_stream(stream);
    // the workspace's error word is followed by the plan; the probe's counter is the
    // error word's neighbour, zeroed here and never incremented
    int* never = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + sizeof(uint32_t));
    if (cudaMemsetAsync(never, 0, sizeof(int), st) != cudaSuccess) return MOE_ERR_CUDA;
    return status_of(launch(wait_timeout_probe_kernel, dim3(1), dim3(32), 0, st, (const int*)never,
                            static_cast<uint32_t*>(ws)));
}

int moe_clear_device_error(void* ws, void* stream)
{
    if (!ws) return MOE_ERR_ARG;
    return cudaMemsetAsync(ws, 0, sizeof(uint32_t), as_stream(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

const char* moe_status_string(int status)
{
    switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument";
    case MOE_ERR_ALIGN: return "size or pointer alignment";
    case MOE_ERR_WS: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA launch or runtime error";
    case MOE_ERR_DEVICE: return "device is not sm_100 (B200)";
    default: return "unknown status";
    }
}

}  // extern "C"

// ---------------------------------------------------------------- FP8 block-scaled layer
namespace {

int run_quantize_rows(const bf16* x, int64_t R, int C, uint8_t* q, float* sc, cudaStream_t st,
                      float* sc_t = nullptr, int64_t ld_t = 0)
{
    const int64_t warps = R * (C / 128);
    return status_of(launch(quantize_rows_fp8_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, st, x, R, C, q,
                            sc, sc_t, ld_t));
}

struct Fp8Operands {
    const uint8_t *xp8, *x8, *W1q, *W3q, *W2q, *Ws1q, *Ws3q, *Ws2q;
    const float *sxp, *sxT, *s1, *s3, *s2, *ss1, *ss3, *ss2;   // sxp / sxT K-block-major
    const int32_t* perm;
    const float* gate_w;
    uint8_t *h8, *hs8;
    float *sh, *shs;                                           // K-block-major
    bf16 *y_p, *ys;
    int T, P, d, f, fs, E;
    int64_t ld_pairs, ld_tokens;
    // FP4 weights: the W*q are packed e2m1 and these their 1 x 32 scale atoms
    bool w4;
    const uint8_t *f1, *f3, *f2, *fs1, *fs3, *fs2;
};

// An A-operand (weight) map: e4m3 bytes, or packed e2m1 unpacked by the TMA;
// boxes of 128 rows (64 for the gate/up weights of CTA-pair tiles).
bool make_map_w(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, bool w4, uint32_t box_rows = 128)
{
    return w4 ? make_map_u4(m, base, inner, rows, box_rows) : make_map_u8(m, base, inner, rows, box_rows);
}

// Whether the FP8 / FP4 expert GEMMs of P pairs and width f run on CTA pairs:
// only when the policy asks for pairs and they run as two launches (the single
// launch has no pair form).  Single CTAs are the default: on the B200 the pair
// form measured 2-2.8x slower (its stages wait on both CTAs' scale atoms).
bool fp8_pair(int64_t P, int64_t f, const DeviceState* dev)
{
    if (dev->fp8_pair_grid < 2) return false;
    return policy(g_policy_pair, "MOE_GEMM_PAIR", /*invert=*/false) == 1 && !gemm_fused((int)P, (int)f);
}

int run_gemms_fp8(const Fp8Operands& o, const int32_t* plan, uint32_t* err, const DeviceState* dev, cudaStream_t st,
                  bool prof, bool pair)
{
    const int sms = dev->sm_count;
    const uint32_t gbox = pair ? 64 : 128;   // rows of a W1 / W3 box
    // gate/up operands: W1/W3, xp8 and its scales (shared: Ws1/Ws3, x8, sxT)
    CUtensorMap a0, a1, b, a0s, a1s, bs, sb, sbs;
    // down operands: W2, h8 and its scales (shared: Ws2, hs8, shs)
    CUtensorMap a2, b2, a2s, b2s, sb2, sb2s;
    // the same token-row maps with 64-row boxes
    CUtensorMap b64, bs64, b264, b2s64;
    const uint64_t E = (uint64_t)o.E;
    const uint64_t lp = (uint64_t)o.ld_pairs, lt = (uint64_t)o.ld_tokens;
    if (!make_map_w(&a0, o.W1q, o.d, E * o.f, o.w4, gbox) || !make_map_w(&a1, o.W3q, o.d, E * o.f, o.w4, gbox) ||
        !make_map_u8(&b, o.xp8, o.d, (uint64_t)o.P, 16) || !make_map_f32(&sb, o.sxp, lp, o.d / 128) ||
        !make_map_u8(&b64, o.xp8, o.d, (uint64_t)o.P, 64) || !make_map_u8(&b264, o.h8, o.f, (uint64_t)o.P, 64) ||
        !make_map_w(&a2, o.W2q, o.f, E * o.d, o.w4) || !make_map_u8(&b2, o.h8, o.f, (uint64_t)o.P, 16) ||
        !make_map_f32(&sb2, o.sh, lp, o.f / 128))
        return MOE_ERR_CUDA;
    if (o.fs > 0) {
        if (!make_map_w(&a0s, o.Ws1q, o.d, o.fs, o.w4, gbox) || !make_map_w(&a1s, o.Ws3q, o.d, o.fs, o.w4, gbox) ||
            !make_map_u8(&bs, o.x8, o.d, (uint64_t)o.T, 16) || !make_map_f32(&sbs, o.sxT, lt, o.d / 128) ||
            !make_map_u8(&bs64, o.x8, o.d, (uint64_t)o.T, 64) || !make_map_u8(&b2s64, o.hs8, o.fs, (uint64_t)o.T, 64) ||
            !make_map_w(&a2s, o.Ws2q, o.fs, o.d, o.w4) || !make_map_u8(&b2s, o.hs8, o.fs, (uint64_t)o.T, 16) ||
            !make_map_f32(&sb2s, o.shs, lt, o.fs / 128))
            return MOE_ERR_CUDA;
    } else {
        a0s = a0;
        a1s = a1;
        bs = b;
        sbs = sb;
        a2s = a2;
        b2s = b2;
        sb2s = sb2;
        bs64 = b64;
        b2s64 = b264;
    }
    Fp8Args g1{};
    g1.plan = plan;
    g1.plan_ready = 1;
    g1.E = o.E;
    g1.M = o.f;
    g1.M_shared = o.fs;
    g1.K = o.d;
    g1.K_shared = o.d;
    g1.sA0 = o.s1;
    g1.sA1 = o.s3;
    g1.sA0s = o.ss1;
    g1.sA1s = o.ss3;
    g1.out8 = o.h8;
    g1.out8_scale = o.sh;
    g1.ld_scale = (int)o.ld_pairs;
    g1.out8_shared = o.hs8;
    g1.out8_scale_shared = o.shs;
    g1.ld_scale_shared = (int)o.ld_tokens;
    g1.perm = o.perm;
    g1.gate_w = o.gate_w;
    g1.err = err;
    g1.fA0 = o.f1;
    g1.fA1 = o.f3;
    g1.fA0s = o.fs1;
    g1.fA1s = o.fs3;
    Fp8Args g2 = g1;
    g2.M = o.d;
    g2.M_shared = o.d;
    g2.K = o.f;
    g2.K_shared = o.fs;
    g2.sA0 = o.s2;
    g2.sA1 = nullptr;
    g2.sA0s = o.ss2;
    g2.sA1s = nullptr;
    g2.fA0 = o.f2;
    g2.fA1 = nullptr;
    g2.fA0s = o.fs2;
    g2.fA1s = nullptr;
    g2.out = o.y_p;
    g2.out_shared = o.ys;
    // the kernel instances of the weight format
    auto k_fused = o.w4 ? grouped_gemm_fp8_kernel<FP8_FUSED, true> : grouped_gemm_fp8_kernel<FP8_FUSED>;
    auto k_gated = o.w4 ? grouped_gemm_fp8_kernel<FP8_GATED, true> : grouped_gemm_fp8_kernel<FP8_GATED>;
    auto k_down = o.w4 ? grouped_gemm_fp8_kernel<FP8_DOWN, true> : grouped_gemm_fp8_kernel<FP8_DOWN>;
    if (gemm_fused(o.P, o.f)) {
        // one launch: a gate/up tile streams d/128 k-blocks, a down tile f/128
        const int kb1 = o.d / 128, kb2 = o.f / 128;
        g1.comp = std::max(1, (kb1 + kb2 / 2) / kb2);
        const cudaError_t e = launch(k_fused, dim3(sms), dim3(kFp8Threads), kFp8SmemBytes, st, a0, a1, b, a0s, a1s,
                                     bs, sb, sbs, a2, b2, a2s, b2s, sb2, sb2s, b64, bs64, b264, b2s64, g1, g2);
        phase_mark(prof, 3, st);   // the single launch has no boundary: the down phase reads as zero
        return status_of(e);
    }
    if (pair) {
        // CTA pairs (M = 256): the grid holds exactly the clusters that fit at once
        auto p_gated = o.w4 ? grouped_gemm_fp8_kernel<FP8_GATED, true, true>
                            : grouped_gemm_fp8_kernel<FP8_GATED, false, true>;
        auto p_down = o.w4 ? grouped_gemm_fp8_kernel<FP8_DOWN, true, true>
                           : grouped_gemm_fp8_kernel<FP8_DOWN, false, true>;
        const dim3 grid(dev->fp8_pair_grid);
        if (launch_pair(p_gated, grid, dim3(kFp8Threads), kFp8SmemBytes, st, a0, a1, b, a0s, a1s, bs, sb, sbs, a2, b2,
                        a2s, b2s, sb2, sb2s, b64, bs64, b264, b2s64, g1, g1) != cudaSuccess)
            return MOE_ERR_CUDA;
        phase_mark(prof, 3, st);
        return status_of(launch_pair(p_down, grid, dim3(kFp8Threads), kFp8SmemBytes, st, a2, a2, b2, a2s, a2s, b2s,
                                     sb2, sb2s, a2, b2, a2s, b2s, sb2, sb2s, b264, b2s64, b264, b2s64, g2, g2));
    }
    if (launch(k_gated, dim3(sms), dim3(kFp8Threads), kFp8SmemBytes, st, a0, a1, b, a0s, a1s, bs, sb, sbs, a2, b2,
               a2s, b2s, sb2, sb2s, b64, bs64, b264, b2s64, g1, g1) != cudaSuccess)
        return MOE_ERR_CUDA;
    phase_mark(prof, 3, st);
    return status_of(launch(k_down, dim3(sms), dim3(kFp8Threads), kFp8SmemBytes, st, a2, a2, b2, a2s, a2s, b2s, sb2,
                            sb2s, a2, b2, a2s, b2s, sb2, sb2s, b264, b2s64, b264, b2s64, g2, g2));
}

}  // namespace

extern "C" {

int moe_quantize_fp8_rows(const moe_bf16* x, int64_t rows, int64_t cols, uint8_t* q, float* scales, void* stream)
{
    if (rows < 0 || cols <= 0 || cols > (int64_t(1) << 30)) return MOE_ERR_ARG;
    if (cols % 128 != 0) return MOE_ERR_ALIGN;
    if (rows == 0) return MOE_OK;
    if (!x || !q || !scales) return MOE_ERR_ARG;
    if (!al16(x) || !al16(q)) return MOE_ERR_ALIGN;
    DeviceState* dev;
    int rc;
    if ((rc = device_setup(&dev))) return rc;
    return run_quantize_rows(reinterpret_cast<const bf16*>(x), rows, (int)cols, q, scales, as_stream(stream));
}

int moe_quantize_fp8_blocks(const moe_bf16* W, int64_t rows, int64_t cols, uint8_t* q, float* scales, void* stream)
{
    if (rows < 0 || cols <= 0) return MOE_ERR_ARG;
    if (rows % 128 != 0 || cols % 128 != 0) return MOE_ERR_ALIGN;
    if (rows == 0) return MOE_OK;
    if (!W || !q || !scales) return MOE_ERR_ARG;
    if (!al16(W) || !al16(q)) return MOE_ERR_ALIGN;
    const int64_t blocks = (rows / 128) * (cols / 128);
    if (blocks >= (int64_t(1) << 31)) return MOE_ERR_ARG;
    DeviceState* dev;
    int rc;
    if ((rc = device_setup(&dev))) return rc;
    return status_of(launch(quantize_blocks_fp8_kernel, dim3((unsigned)blocks), dim3(256), 0, as_stream(stream),
                            reinterpret_cast<const bf16*>(W), rows, cols, q, scales));
}

int moe_workspace_size_fp8(int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, int64_t f_shared, size_t* bytes)
{
    if (!bytes || T < 0 || d < 0 || f < 0 || E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK || f_shared < 0)
        return MOE_ERR_ARG;
    *bytes = ws_layout_fp8(T, d, f, E, k, f_shared).total;
    return MOE_OK;
}

int moe_workspace_tensor_fp8(void* ws, int64_t T, int64_t d, int64_t f, int64_t E, int64_t k, int64_t f_shared,
                             int which, void** ptr)
{
    if (!ws || !ptr || T < 0 || d < 0 || f < 0 || E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK || f_shared < 0)
        return MOE_ERR_ARG;
    const WsLayoutFp8 L = ws_layout_fp8(T, d, f, E, k, f_shared);
    const size_t offs[19] = {L.logits, L.topk_idx, L.topk_w, L.counts, L.offsets, L.perm, L.inv_perm, L.x8, L.sx,
                             L.xp8, L.sxp, L.h8, L.sh, L.y_p, L.hs8, L.shs, L.ys, L.sxT, L.ctrl.plan};
    if (which < 0 || which >= 19) return MOE_ERR_ARG;
    *ptr = static_cast<uint8_t*>(ws) + offs[which];
    return MOE_OK;
}

// The FP8 layer and the FP4-weight layer share everything but the weights'
// format: e4m3 with fp32 128 x 128 block scales (W*s), or packed e2m1 with 1 x 32
// scale atoms (W*f, w4).
static int layer_forward_lowp(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const uint8_t* W1q,
                              const float* W1s, const uint8_t* W3q, const float* W3s, const uint8_t* W2q,
                              const float* W2s, const uint8_t* Ws1q, const float* Ws1s, const uint8_t* Ws3q,
                              const float* Ws3s, const uint8_t* Ws2q, const float* Ws2s, int64_t f_shared, int64_t T,
                              int64_t d, int64_t f, int64_t E, int64_t k, moe_bf16* out, void* ws, size_t ws_bytes,
                              void* stream, bool w4, const uint8_t* W1f, const uint8_t* W3f, const uint8_t* W2f,
                              const uint8_t* Ws1f, const uint8_t* Ws3f, const uint8_t* Ws2f)
{
    int rc = check_sizes(T, d, E, k);
    if (rc) return rc;
    if (f <= 0 || f_shared < 0) return MOE_ERR_ARG;
    if (d % 128 != 0 || f % 128 != 0 || f_shared % 128 != 0) return MOE_ERR_ALIGN;
    if (d > kFp8MaxK || f > kFp8MaxK || f_shared > kFp8MaxK) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    const bool scales_ok = w4 ? (W1f && W3f && W2f) : (W1s && W3s && W2s);
    const bool shared_scales_ok = w4 ? (Ws1f && Ws3f && Ws2f) : (Ws1s && Ws3s && Ws2s);
    if (!x || !Wg || !W1q || !W3q || !W2q || !scales_ok || !out || !ws) return MOE_ERR_ARG;
    if (f_shared > 0 && (!Ws1q || !Ws3q || !Ws2q || !shared_scales_ok)) return MOE_ERR_ARG;
    if (w4 && !(al16(W1f) && al16(W3f) && al16(W2f) && (f_shared == 0 || (al16(Ws1f) && al16(Ws3f) && al16(Ws2f)))))
        return MOE_ERR_ALIGN;
    if (!al16(x) || !al16(Wg) || !al16(W1q) || !al16(W3q) || !al16(W2q) || !al16(out) || !al16(ws))
        return MOE_ERR_ALIGN;
    if (f_shared > 0 && (!al16(Ws1q) || !al16(Ws3q) || !al16(Ws2q))) return MOE_ERR_ALIGN;
    const WsLayoutFp8 L = ws_layout_fp8(T, d, f, E, k, f_shared);
    if (ws_bytes < L.total) return MOE_ERR_WS;
    DeviceState* dev;
    if ((rc = device_setup(&dev))) return rc;
    cudaStream_t st = as_stream(stream);
    uint32_t* err = at<uint32_t>(ws, L.ctrl.err);
    int32_t* plan = at<int32_t>(ws, L.ctrl.plan);
    float* logits = at<float>(ws, L.logits);
    float* partials = at<float>(ws, L.ctrl.router_partials);
    int32_t* idx = at<int32_t>(ws, L.topk_idx);
    float* w = at<float>(ws, L.topk_w);
    int32_t* counts = at<int32_t>(ws, L.counts);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* perm = at<int32_t>(ws, L.perm);
    int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
    uint8_t* x8 = at<uint8_t>(ws, L.x8);
    float* sx = at<float>(ws, L.sx);
    uint8_t* xp8 = at<uint8_t>(ws, L.xp8);
    float* sxp = at<float>(ws, L.sxp);
    bf16* y_p = at<bf16>(ws, L.y_p);
    const bf16* xb = reinterpret_cast<const bf16*>(x);
    const int iT = (int)T, id = (int)d, iE = (int)E, ik = (int)k, shared_rows = f_shared > 0 ? (int)T : 0;
    const int64_t P = T * k;
    // the plan is cut for the tile shape the expert GEMMs will run
    const bool pair = fp8_pair(P, f, dev);
    const PlanShape ps = plan_shape(pair ? kPlanFp8Pair : gemm_fused((int)P, (int)f) ? kPlanFp8 : kPlanFp8Wide, T);

    const bool prof = t_phase_armed;
    t_phase_armed = false;
    int64_t inv_perm_launch = 0;
    phase_mark(prof, 0, st);
    RouterSplit rs;
    if ((rc = run_router_gemm(xb, reinterpret_cast<const bf16*>(Wg), bias, iT, id, iE, logits, partials, err,
                              dev->sm_count, st, &rs)))
        return rc;
    float* sxT = f_shared > 0 ? at<float>(ws, L.sxT) : nullptr;   // the shared expert's token scales
    if ((rc = run_quantize_rows(xb, T, id, x8, sx, st, sxT, L.ld_tokens))) return rc;
    if ((rc = run_topk(topk_source(rs, logits, partials, bias, iT, iE), iT, iE, ik, idx, w, err, st))) return rc;
    phase_mark(prof, 1, st);
    if (P <= kSmallPairs) {
        if (launch(permute_small_kernel, dim3(1), dim3(1024), 0, st, (const int32_t*)idx, (int)P, iE, counts, offsets,
                   perm, inv_perm, plan, (int)f, id, shared_rows, (int)f_shared, ps, err) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        inv_perm_launch = t_launches;
    } else if ((rc = run_permute(idx, xb, iT, id, iE, ik, counts, offsets, perm, inv_perm, nullptr, err,
                                 at<int32_t>(ws, L.ctrl.block_counts), plan, (int)f, shared_rows, (int)f_shared,
                                 dev->sm_count, st, ps, &inv_perm_launch))) {
        return rc;
    }
    if (launch(gather_rows_fp8_kernel, dim3(gather_blocks(T, d / 16, dev->sm_count)), dim3(256), 0, st,
               (const uint8_t*)x8, (const float*)sx, (const int32_t*)inv_perm, iT, ik, id, xp8, sxp,
               L.ld_pairs) != cudaSuccess)
        return MOE_ERR_CUDA;
    Fp8Operands o{};
    o.xp8 = xp8;
    o.x8 = x8;
    o.sxp = sxp;
    o.sxT = sxT;
    o.ld_pairs = L.ld_pairs;
    o.ld_tokens = L.ld_tokens;
    o.W1q = W1q;
    o.W3q = W3q;
    o.W2q = W2q;
    o.s1 = W1s;
    o.s3 = W3s;
    o.s2 = W2s;
    o.Ws1q = Ws1q;
    o.Ws3q = Ws3q;
    o.Ws2q = Ws2q;
    o.ss1 = Ws1s;
    o.ss3 = Ws3s;
    o.ss2 = Ws2s;
    o.w4 = w4;
    o.f1 = W1f;
    o.f3 = W3f;
    o.f2 = W2f;
    o.fs1 = Ws1f;
    o.fs3 = Ws3f;
    o.fs2 = Ws2f;
    o.perm = perm;
    o.gate_w = w;
    o.h8 = at<uint8_t>(ws, L.h8);
    o.sh = at<float>(ws, L.sh);
    o.hs8 = f_shared > 0 ? at<uint8_t>(ws, L.hs8) : nullptr;
    o.shs = f_shared > 0 ? at<float>(ws, L.shs) : nullptr;
    o.y_p = y_p;
    o.ys = f_shared > 0 ? at<bf16>(ws, L.ys) : nullptr;
    o.T = iT;
    o.P = (int)P;
    o.d = id;
    o.f = (int)f;
    o.fs = (int)f_shared;
    o.E = iE;
    phase_mark(prof, 2, st);
    if ((rc = run_gemms_fp8(o, plan, err, dev, st, prof, pair))) return rc;
    phase_mark(prof, 4, st);
    rc = run_combine(y_p, inv_perm, o.ys, iT, ik, id, reinterpret_cast<bf16*>(out), st, inv_perm_launch);
    phase_mark(prof, 5, st);
    return rc;
}

int moe_layer_forward_fp8(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const uint8_t* W1q,
                          const float* W1s, const uint8_t* W3q, const float* W3s, const uint8_t* W2q, const float* W2s,
                          const uint8_t* Ws1q, const float* Ws1s, const uint8_t* Ws3q, const float* Ws3s,
                          const uint8_t* Ws2q, const float* Ws2s, int64_t f_shared, int64_t T, int64_t d, int64_t f,
                          int64_t E, int64_t k, moe_bf16* out, void* ws, size_t ws_bytes, void* stream)
{
    return layer_forward_lowp(x, Wg, bias, W1q, W1s, W3q, W3s, W2q, W2s, Ws1q, Ws1s, Ws3q, Ws3s, Ws2q, Ws2s, f_shared,
                              T, d, f, E, k, out, ws, ws_bytes, stream, false, nullptr, nullptr, nullptr, nullptr,
                              nullptr, nullptr);
}

int moe_layer_forward_fp4(const moe_bf16* x, const moe_bf16* Wg, const float* bias, const uint8_t* W1q,
                          const uint8_t* W1sf, const uint8_t* W3q, const uint8_t* W3sf, const uint8_t* W2q,
                          const uint8_t* W2sf, const uint8_t* Ws1q, const uint8_t* Ws1sf, const uint8_t* Ws3q,
                          const uint8_t* Ws3sf, const uint8_t* Ws2q, const uint8_t* Ws2sf, int64_t f_shared, int64_t T,
                          int64_t d, int64_t f, int64_t E, int64_t k, moe_bf16* out, void* ws, size_t ws_bytes,
                          void* stream)
{
    return layer_forward_lowp(x, Wg, bias, W1q, nullptr, W3q, nullptr, W2q, nullptr, Ws1q, nullptr, Ws3q, nullptr,
                              Ws2q, nullptr, f_shared, T, d, f, E, k, out, ws, ws_bytes, stream, true, W1sf, W3sf, W2sf,
                              Ws1sf, Ws3sf, Ws2sf);
}

int moe_quantize_fp4_rows(const moe_bf16* W, int64_t rows, int64_t cols, uint8_t* q, uint8_t* scale_atoms,
                          void* stream)
{
    if (rows < 0 || cols <= 0 || cols > (int64_t(1) << 30)) return MOE_ERR_ARG;
    if (rows % 128 != 0 || cols % 128 != 0) return MOE_ERR_ALIGN;
    if (rows == 0) return MOE_OK;
    if (!W || !q || !scale_atoms) return MOE_ERR_ARG;
    if (!al16(W) || !al16(q) || !al16(scale_atoms)) return MOE_ERR_ALIGN;
    DeviceState* dev;
    int rc;
    if ((rc = device_setup(&dev))) return rc;
    const int64_t warps = rows * (cols / 128);
    return status_of(launch(quantize_rows_fp4_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0,
                            as_stream(stream), reinterpret_cast<const bf16*>(W), rows, (int)cols, q, scale_atoms));
}

}  // extern "C"

// ---------------------------------------------------------------- permutation without a workspace
// Some callers cannot hand this library a workspace: they run inside a host
// framework that owns every device allocation and forbids allocating in its
// execute path, or in a latency-critical loop where cudaMalloc's implicit
// device synchronisation is not acceptable.  moe_permute_noalloc serves them:
// its only scratch (the per-CTA expert counters of the histogram and a device
// error word) lives in the static device array below, which every GPU that
// loads this library holds until the process exits.
namespace {

constexpr int kNoAllocCounters = 65536;   // 256 KiB of int32 per-CTA counters (hist_blocks(T*k) * E)

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocCounters + 64];

struct NoAllocState {
    bool ready = false;
    int32_t* scratch = nullptr;   // device address of g_noalloc_scratch on this device
};
NoAllocState g_noalloc[kMaxDevices];

// Device address of the static scratch on the current device, looked up once
// per device.  In host code g_noalloc_scratch names a host-side stand-in, so
// only this address may be handed to a kernel.
int noalloc_scratch(int32_t** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    NoAllocState& st = g_noalloc[dev];
    if (!st.ready) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        st.scratch = static_cast<int32_t*>(p);
        st.ready = true;
    }
    *out = st.scratch;
    return MOE_OK;
}

}  // namespace

extern "C" int moe_permute_noalloc(const int32_t* topk_idx, const moe_bf16* x, int64_t T, int64_t d, int64_t E,
                                   int64_t k, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                                   moe_bf16* xp, void* stream)
{
    int rc = check_sizes(T, d, E, k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!topk_idx || !x || !counts || !offsets || !perm || !inv_perm || !xp) return MOE_ERR_ARG;
    if (!al16(x) || !al16(xp)) return MOE_ERR_ALIGN;
    if ((int64_t)hist_blocks(T * k) * E > kNoAllocCounters) return MOE_ERR_WS;
    DeviceState* dev;
    if ((rc = device_setup(&dev))) return rc;
    int32_t* scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch))) return rc;
    cudaStream_t st = as_stream(stream);
    // The array keeps the previous call's contents: the error word must start at
    // zero; the counters are fully rewritten by the histogram kernel.
    uint32_t* err = reinterpret_cast<uint32_t*>(scratch + kNoAllocCounters);
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    return run_permute(topk_idx, reinterpret_cast<const bf16*>(x), (int)T, (int)d, (int)E, (int)k, counts, offsets,
                       perm, inv_perm, reinterpret_cast<bf16*>(xp), err, scratch, nullptr, 0, 0, 0, dev->sm_count,
                       st, kPlanSingle);
}
