// svdq_lib.cu -- host side of the C ABI declared in include/svdq.h: argument
// validation, the device-capability check, TMA descriptor construction and
// kernel launches.  All kernels live in the headers included below; this is
// the library's single translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "svdq.h"
#include "sm100_ptx.cuh"
#include "quantize.cuh"
#include "quantize_act.cuh"
#include "gemm_nvfp4.cuh"
#include "gemm_nvfp4_pair.cuh"
#include "qkv_norm_rope.cuh"
#include "svd_split.cuh"
#include "gemm_dq16.cuh"

namespace svdq {
namespace {

constexpr int kAbiVersion = 2;

// ------------------------------------------------------------- validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

svdq_status check_precision(svdq_precision p, int group_size) {
    if (p == SVDQ_NVFP4) return group_size == 16 ? SVDQ_OK : SVDQ_ERR_INVALID_ARG;
    if (p == SVDQ_INT4) return group_size == 64 ? SVDQ_OK : SVDQ_ERR_INVALID_ARG;
    return SVDQ_ERR_INVALID_ARG;
}

svdq_status check_rank(int rank) {
    return (rank >= 0 && rank <= 256 && rank % 16 == 0) ? SVDQ_OK : SVDQ_ERR_INVALID_ARG;
}

svdq_status check_dims(int64_t rows, int64_t K) {
    if (rows < 1 || rows >= (int64_t(1) << 31)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    if (K < 64 || K >= (int64_t(1) << 31) || K % 64 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    return SVDQ_OK;
}

svdq_status check_ptr(const void* p) {
    if (p == nullptr || !aligned16(p)) return SVDQ_ERR_INVALID_ARG;
    return SVDQ_OK;
}

svdq_status check_opt_ptr(const void* p) { return (p == nullptr || aligned16(p)) ? SVDQ_OK : SVDQ_ERR_INVALID_ARG; }

#define SVDQ_TRY(expr)                          \
    do {                                        \
        const svdq_status _st = (expr);         \
        if (_st != SVDQ_OK) return _st;         \
    } while (0)

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// ------------------------------------------------------------ the device
std::mutex g_mutex;
int g_override_major = -1, g_override_minor = 0;
constexpr int kMaxDevices = 64;
std::atomic<int> g_gemm_tiles_mode{0};   // svdq_debug_force_gemm_tiles
std::atomic<int> g_quant_plan_mode{0};   // svdq_debug_force_quant_plan
bool g_device_ready[kMaxDevices];

// Budget of dynamic shared memory for the activation quantizer (the opt-in
// maximum is 227 KB per block including static shared memory).
constexpr int kQuantSmemBudget = 226 * 1024;

thread_local char g_last_error[256] = "";

void note_error(cudaError_t e, const char* where) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
}

// Records and clears the pending CUDA error, then reports SVDQ_ERR_CUDA.
svdq_status cuda_fail(const char* where = "CUDA call") {
    const cudaError_t e = cudaGetLastError();
    note_error(e == cudaSuccess ? cudaErrorUnknown : e, where);
    return SVDQ_ERR_CUDA;
}

svdq_status launch_status(const char* where) {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return SVDQ_OK;
    note_error(e, where);
    return SVDQ_ERR_CUDA;
}

// Rejects anything but compute capability 10.0 before any launch, and sets
// the kernels' shared-memory limits once per device.
svdq_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return SVDQ_ERR_UNSUPPORTED_DEVICE;
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return SVDQ_ERR_UNSUPPORTED_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_override_major >= 0) {
        major = g_override_major;
        minor = g_override_minor;
    }
    if (major != 10 || minor != 0) return SVDQ_ERR_UNSUPPORTED_DEVICE;
    if (dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_UNSUPPORTED_DEVICE;
    if (!g_device_ready[dev]) {
        if (cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gm::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(quantize_act_kernel<kPrecNvfp4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kQuantSmemBudget) != cudaSuccess ||
            cudaFuncSetAttribute(quantize_act_kernel<kPrecInt4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kQuantSmemBudget) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_dq16_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)dq::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_dq16_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)dq::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_nvfp4_pair_kernel<kEpiPlain>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gp::SMEM_BYTES_PLAIN) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_nvfp4_pair_kernel<kEpiQkv>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gp::SMEM_BYTES_PLAIN) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_nvfp4_pair_kernel<kEpiGelu>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gp::SMEM_BYTES_GELU) != cudaSuccess ||
            cudaFuncSetAttribute(gemm_nvfp4_pair_kernel<kEpiGeluStore>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gp::SMEM_BYTES_GELU) != cudaSuccess)
            return cuda_fail("setting kernel shared-memory limits");
        g_device_ready[dev] = true;
    }
    return SVDQ_OK;
}

// ------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// 2-D row-major tensor [outer, inner] with 128-byte swizzled boxes (or
// unswizzled ones).
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return r == CUDA_SUCCESS;
}

// 3-D row-major tensor [planes, outer, inner] with 128-byte swizzled boxes of
// box_planes planes.
bool make_map_3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t planes, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, uint32_t box_planes) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {inner, outer, planes};
    const cuuint64_t strides[2] = {row_bytes, row_bytes * outer};
    const cuuint32_t box[3] = {box_inner, box_outer, box_planes};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (3-D) failed (CUresult %d)", (int)r);
    return r == CUDA_SUCCESS;
}

// Scale blocks viewed as a 3-D tensor of 32-bit words [row_blocks][kg4][128]:
// one 512-byte block (128 rows x 4 groups) per (row block, 64 columns of K);
// boxes of 4 consecutive K blocks of `box_row_blocks` row blocks, unswizzled.
bool make_sf_map(CUtensorMap* m, const void* base, uint64_t row_blocks, uint64_t kg4, uint32_t box_row_blocks,
                 uint32_t box_ksteps = 4) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {128, kg4, row_blocks};
    const cuuint64_t strides[2] = {512, 512 * kg4};
    const cuuint32_t box[3] = {128, box_ksteps, box_row_blocks};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (scale blocks) failed (CUresult %d)",
                 (int)r);
    return r == CUDA_SUCCESS;
}

// SM count of the current device (looked up once per device).
int num_sms() {
    static std::atomic<int> per_dev[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 148;
    }
    int n = per_dev[dev].load();
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        per_dev[dev].store(n);
    }
    return n;
}

// ---------------------------------------------------------- nvfp4 paths
svdq_status tensor_scale_prepass(const void* src, const float* inv_lambda, int64_t rows, int64_t K, float* out,
                                 cudaStream_t st) {
    if (cudaMemsetAsync(out, 0, sizeof(float), st) != cudaSuccess) return cuda_fail("cudaMemsetAsync");
    const int64_t nvec = rows * K / 8;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((nvec + 255) / 256, 8LL * num_sms()));
    amax_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(src), inv_lambda, rows, K,
                                        reinterpret_cast<unsigned int*>(out));
    finalize_tensor_scale_kernel<<<1, 1, 0, st>>>(out);
    return launch_status("tensor-scale pre-pass");
}

svdq_status fold_lowrank(const float* lambda, const void* L_down, const void* L_up, int64_t N, int64_t K, int rank,
                         float* inv_lambda, void* L_down_t, void* L_up_t, cudaStream_t st) {
    const int64_t work = std::max<int64_t>(K, std::max<int64_t>(K * rank, N * rank));
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256, 8LL * num_sms()));
    fold_lowrank_kernel<<<blocks, 256, 0, st>>>(lambda, reinterpret_cast<const __nv_bfloat16*>(L_down),
                                                reinterpret_cast<const __nv_bfloat16*>(L_up), K, N, rank, inv_lambda,
                                                reinterpret_cast<__nv_bfloat16*>(L_down_t),
                                                reinterpret_cast<__nv_bfloat16*>(L_up_t));
    return launch_status("fold_lowrank_kernel");
}

// The GEMM-ready copy of nvfp4 weight scales, right after their block layout.
svdq_status replicate_weight_scales(void* w_scales, int64_t N, int64_t K, cudaStream_t st) {
    const int64_t rows_pad = round_up(N, 128);
    const int64_t chunks = wscales_rep_bytes(N, K) / 16;
    replicate_weight_scales_kernel<<<(unsigned)((chunks + 255) / 256), 256, 0, st>>>(
        reinterpret_cast<const uint8_t*>(w_scales), reinterpret_cast<uint8_t*>(w_scales) + rows_pad * K / 16,
        (int)(rows_pad / 128), (int)(K / 64), (int)((K + 255) / 256), chunks);
    return launch_status("replicate_weight_scales_kernel");
}

svdq_status pack_weight_nvfp4(const void* R, int64_t N, int64_t K, void* w_codes, void* w_scales,
                              float* w_tensor_scale, cudaStream_t st) {
    SVDQ_TRY(tensor_scale_prepass(R, nullptr, N, K, w_tensor_scale, st));
    const int64_t rows_pad = round_up(N, 128);
    const int64_t work = rows_pad * (K / 16);
    quantize_rows_nvfp4_kernel<<<(unsigned)((work + 255) / 256), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(R), N, rows_pad, K, w_tensor_scale,
        reinterpret_cast<uint8_t*>(w_codes), reinterpret_cast<uint8_t*>(w_scales));
    SVDQ_TRY(launch_status("quantize_rows_nvfp4_kernel"));
    return replicate_weight_scales(w_scales, N, K, st);
}

// K-split of the activation quantizer: enough CTAs for about one wave on a
// B200 (a fixed target, so that the workspace size depends on the shape only).
int quant_splits(int64_t M, int64_t K) {
    const int64_t row_blocks = (M + qa::kRows - 1) / qa::kRows;
    int64_t sp = qa::kSplitTarget / row_blocks;
    sp = std::min<int64_t>(sp, std::min<int64_t>(K / 64, qa::kMaxSplits));
    return (int)std::max<int64_t>(sp, 1);
}

// The workspace plan's two counters per 128-row block, ahead of the partials.
size_t quant_counter_bytes(int64_t row_blocks) { return (size_t)round_up(row_blocks * 8, 256); }

// Workspace of the K-split when its CTAs add their rank-r partials through
// global memory (the upper bound: a launch that runs in cluster mode leaves
// the workspace untouched).
size_t quant_workspace_bytes(int64_t M, int64_t K, int rank) {
    const int sp = quant_splits(M, K);
    if (rank == 0 || sp == 1) return 0;
    const int64_t row_blocks = (M + qa::kRows - 1) / qa::kRows;
    return quant_counter_bytes(row_blocks) + (size_t)row_blocks * sp * qa::kRows * rank * 4;
}

// Clusters of `c` quantizer CTAs that can be resident at once on the current
// device (one CTA per SM), looked up once per device and size.
int quant_max_clusters(int c) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 0;
    }
    static int cache[kMaxDevices][qa::kMaxCluster + 1];
    std::lock_guard<std::mutex> lock(g_mutex);
    if (cache[dev][c] == 0) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)c;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)c * 256u, 1, 1);
        cfg.blockDim = dim3(qa::kThreads, 1, 1);
        cfg.dynamicSmemBytes = kQuantSmemBudget;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, quantize_act_kernel<kPrecNvfp4>, &cfg) != cudaSuccess || n < 0) {
            cudaGetLastError();
            n = 0;
        }
        cache[dev][c] = n + 1;   // stored + 1 so that 0 means "not looked up"
    }
    return cache[dev][c] - 1;
}

// How the K range is split: `splits` CTAs per 128-row block; cluster mode
// (cluster == splits) when those CTAs form one cluster and every row block's
// cluster is resident at once, else the workspace (cluster == 1).  The split
// is never narrowed to fit a cluster: the quantizer warps bound the rate at
// which a CTA streams its chunks, so fewer CTAs cost more than the
// workspace's round trip (B200, M = 4608: three-CTA clusters on 108 SMs
// against the workspace on 144 take 22.5 / 22.6 us at K = 3072 and 49.2 /
// 43.0 us at K = 12288).
struct QuantPlan {
    int splits, cluster;
};
QuantPlan quant_plan(int64_t M, int64_t K, int rank) {
    const int sp = quant_splits(M, K);
    if (rank == 0 || sp == 1) return {sp, 1};
    const int mode = g_quant_plan_mode.load();
    if (mode == 1 || mode == 3) return {sp, 1};
    if (mode == 2) return {std::min(sp, qa::kMaxCluster), std::min(sp, qa::kMaxCluster)};
    const int64_t row_blocks = (M + qa::kRows - 1) / qa::kRows;
    if (sp <= qa::kMaxCluster && quant_max_clusters(sp) >= row_blocks) return {sp, sp};
    return {sp, 1};
}

// Launch with programmatic stream serialisation (the kernel waits for the
// previous grid with griddepcontrol.wait) and an optional cluster shape.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      unsigned cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Activation quantizer launch (both precisions).  x_scale / w_scale are only
// read by the nvfp4 variant.
svdq_status quantize_act_launch(int prec, const void* x, int64_t M, int64_t K, const float* inv_lambda,
                                const float* x_scale, const float* w_scale, const void* L_down_t, int rank,
                                void* x_codes, void* x_scales, void* lowrank, void* workspace, cudaStream_t st) {
    CUtensorMap tm_x, tm_ld;
    if (!make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, 128))
        return SVDQ_ERR_CUDA;
    if (rank > 0) {
        if (!make_map_3d(&tm_ld, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L_down_t, (uint64_t)K, (uint64_t)rank, 2,
                         (uint64_t)K * 2, 64, (uint32_t)rank, 2))   // hi and lo planes in one box
            return SVDQ_ERR_CUDA;
    } else {
        tm_ld = tm_x;
    }
    const int64_t row_blocks = (M + qa::kRows - 1) / qa::kRows;
    if (row_blocks > 65535) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    const QuantPlan plan = quant_plan(M, K, rank);
    if (plan.cluster == 1 && plan.splits > 1 && rank > 0 && workspace == nullptr) return SVDQ_ERR_INVALID_ARG;
    QuantActArgs a;
    a.inv_lambda = inv_lambda;
    a.x_scale = x_scale;
    a.w_scale = w_scale;
    a.x_codes = reinterpret_cast<uint8_t*>(x_codes);
    a.x_scales = reinterpret_cast<uint8_t*>(x_scales);
    a.lowrank = reinterpret_cast<__nv_bfloat16*>(lowrank);
    a.M = (int)M;
    a.K = (int)K;
    a.rank = rank;
    a.rows_pad = (int)round_up(M, 128);
    a.chunks = (int)(K / 64);
    a.splits = plan.splits;
    a.cluster = plan.cluster;
    a.counters = reinterpret_cast<unsigned int*>(workspace);
    a.partials = workspace ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) +
                                                       quant_counter_bytes(row_blocks))
                           : nullptr;
    // the splits of a row block wait for one another only when the whole grid
    // (one CTA per SM) is resident at once
    a.coop = (plan.cluster == 1 && plan.splits > 1 && (int64_t)plan.splits * row_blocks <= num_sms() &&
              g_quant_plan_mode.load() != 3)
                 ? 1
                 : 0;
    // stage: x tile, hi and lo L_down_t tiles, the chunk's 1/lambda; 1 KB aligned (128-byte swizzle)
    a.invl_off = (uint32_t)qa::kXBytes + (uint32_t)rank * 256u;
    a.stage_bytes = (uint32_t)round_up((int64_t)a.invl_off + qa::kInvlBytes, 1024);
    const size_t fixed = 1024 + 128 * 4 + (2 * qa::kMaxStages + 1) * 8 + 16;
    const int stages = (int)std::min<size_t>(qa::kMaxStages, (kQuantSmemBudget - fixed) / a.stage_bytes);
    if (stages < 2) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    // the rank-r partial is staged in the ring once streaming is over
    if ((size_t)stages * a.stage_bytes < (size_t)qa::kRows * (rank + 4) * 4) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    a.stages = stages;
    uint32_t tcols = 32;
    while ((int)tcols < 2 * rank) tcols *= 2;   // x . hi and x . lo accumulators
    a.tmem_cols = tcols;
    const size_t smem = fixed + (size_t)stages * a.stage_bytes;
    const dim3 grid((unsigned)a.splits, (unsigned)row_blocks, 1);
    const unsigned cl = (unsigned)a.cluster;
    const cudaError_t e =
        prec == kPrecNvfp4
            ? launch_ex(quantize_act_kernel<kPrecNvfp4>, grid, dim3(qa::kThreads), smem, st, cl, tm_x, tm_ld, a)
            : launch_ex(quantize_act_kernel<kPrecInt4>, grid, dim3(qa::kThreads), smem, st, cl, tm_x, tm_ld, a);
    if (e != cudaSuccess) return cuda_fail("quantize_act_kernel launch");
    return launch_status("quantize_act_kernel launch");
}

svdq_status quantize_act_nvfp4(const void* x, int64_t M, int64_t K, const float* inv_lambda, float* x_scale,
                               int compute_scale, const float* w_scale, const void* L_down_t, int rank,
                               void* x_codes, void* x_scales, void* lowrank, void* workspace, cudaStream_t st) {
    if (compute_scale) SVDQ_TRY(tensor_scale_prepass(x, inv_lambda, M, K, x_scale, st));
    return quantize_act_launch(kPrecNvfp4, x, M, K, inv_lambda, x_scale, w_scale, L_down_t, rank, x_codes, x_scales,
                               lowrank, workspace, st);
}

// --------------------------------------------------- offline SVD split
size_t svd_split_workspace(int64_t N, int64_t K, int l) {
    const size_t f = sizeof(float), d = sizeof(double);
    const size_t mm = (size_t)sv::kMaxL * sv::kMaxL;
    return (size_t)round_up((int64_t)(N * l * f), 256) + (size_t)round_up((int64_t)(K * l * f), 256) +
           (size_t)sv::kGramBlocks * mm * d + 2 * mm * d + sv::kMaxL * d;
}

// Orthonormal columns of A [rows, l] in place: CholeskyQR2.
svdq_status svd_orth(float* A, int64_t rows, int l, double* part, double* Rinv, cudaStream_t st) {
    for (int pass = 0; pass < 2; ++pass) {
        svd_gram_partial_kernel<<<sv::kGramBlocks, 256, 0, st>>>(A, rows, l, part);
        svd_chol_inv_kernel<<<1, 64, 0, st>>>(part, sv::kGramBlocks, l, Rinv);
        svd_apply_rinv_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(A, rows, l, Rinv);
    }
    return launch_status("SVD split: orthonormalisation");
}

// ----------------------------------------------------------- int4 paths
svdq_status int4_quantize_rows(const void* R, int64_t N, int64_t K, void* w_codes, void* w_scales, cudaStream_t st) {
    const int64_t rows_pad = round_up(N, 128);
    const int64_t work = rows_pad * (K / 64);
    quantize_rows_int4_kernel<<<(unsigned)((work + 255) / 256), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(R), N, rows_pad, K, reinterpret_cast<uint8_t*>(w_codes),
        reinterpret_cast<uint16_t*>(w_scales));
    return launch_status("quantize_rows_int4_kernel");
}

svdq_status gemm_nvfp4(const void* x_codes, const void* x_scales, const float* x_scale, int64_t M,
                       const void* w_codes, const void* w_scales, const float* w_scale, int64_t N, int64_t K,
                       const void* lowrank, const void* L_up_t, int rank, const void* bias, void* y, cudaStream_t st) {
    CUtensorMap tm_xc, tm_wc, tm_L, tm_Lup;
    if (!make_map(&tm_xc, CU_TENSOR_MAP_DATA_TYPE_UINT8, x_codes, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2,
                  gm::BK_BYTES, gm::BM) ||
        !make_map(&tm_wc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2,
                  gm::BK_BYTES, gm::BN))
        return SVDQ_ERR_CUDA;
    if (rank > 0) {
        if (!make_map_3d(&tm_L, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lowrank, (uint64_t)rank, (uint64_t)M, 2,
                         (uint64_t)rank * 2, 64, gm::BM, 1) ||
            !make_map(&tm_Lup, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L_up_t, (uint64_t)rank, (uint64_t)N,
                      (uint64_t)rank * 2, 64, gm::BN))
            return SVDQ_ERR_CUDA;
    } else {
        tm_L = tm_xc;
        tm_Lup = tm_wc;
    }
    GemmArgs a = {};
    a.x_scales = reinterpret_cast<const uint8_t*>(x_scales);
    a.w_scales = reinterpret_cast<const uint8_t*>(w_scales);
    a.x_scale = x_scale;
    a.w_scale = w_scale;
    a.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
    a.y = reinterpret_cast<__nv_bfloat16*>(y);
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.rank = rank;
    a.kg4 = (int)(K / 64);
    a.n_sf_blocks = (int)((N + 127) / 128);
    const int64_t mt = (M + gm::BM - 1) / gm::BM, nt = (N + gm::BN - 1) / gm::BN;
    if (mt * nt > (int64_t(1) << 30)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    a.m_tiles = (int)mt;
    a.n_tiles = (int)nt;
    const int grid = (int)std::min<int64_t>(mt * nt, num_sms());
    gemm_nvfp4_kernel<<<grid, gm::kThreads, gm::SMEM_BYTES, st>>>(tm_xc, tm_wc, tm_L, tm_Lup, a);
    return launch_status("gemm_nvfp4_kernel launch");
}

// Clusters of two CTAs that fit on the device at once (one CTA per SM; both
// pair kernels have the same block size and nearly all of shared memory).
int pair_clusters() {
    static std::atomic<int> per_dev[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return num_sms() / 2;
    }
    if (per_dev[dev].load() == 0) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (unsigned)num_sms(), 1, 1);
        cfg.blockDim = dim3(gp_threads<kEpiPlain>(), 1, 1);
        cfg.dynamicSmemBytes = gp::SMEM_BYTES_PLAIN;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_pair_kernel<kEpiPlain>, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = num_sms() / 2;
        }
        per_dev[dev].store(n);
    }
    return per_dev[dev].load();
}

// M > 128: 256 x 256 tiles on CTA pairs.
// The fused QKV + RMSNorm + RoPE epilogue's arguments (heads == 0: plain epilogue).
struct QkvEpilogue {
    int heads = 0;
    const void* norm_q = nullptr;
    const void* norm_k = nullptr;
    float eps = 0.0f;
    const float* rope_cos = nullptr;
    const float* rope_sin = nullptr;
};

// The fused GELU + next-layer activation epilogue's arguments (next_x_scale ==
// nullptr: not used).
struct GeluEpilogue {
    bool store_y = false;   // store h = bf16(GELU(y)) to y; the next-layer fields below are then unused
    int approx = 0;
    const float* next_inv_lambda = nullptr;
    const void* next_L_down_t = nullptr;
    int next_rank = 0;
    const float* next_x_scale = nullptr;
    void* next_codes = nullptr;
    void* next_scales = nullptr;
    float* next_acc = nullptr;
};

svdq_status gemm_nvfp4_pair(const void* x_codes, const void* x_scales, const float* x_scale, int64_t M,
                            const void* w_codes, const void* w_scales, const float* w_scale, int64_t N, int64_t K,
                            const void* lowrank, const void* L_up_t, int rank, const void* bias, void* y,
                            cudaStream_t st, const QkvEpilogue& qkv = QkvEpilogue(),
                            const GeluEpilogue& gelu = GeluEpilogue()) {
    CUtensorMap tm_xc, tm_wc, tm_sfa, tm_sfb, tm_L, tm_Lup;
    const int64_t kg4 = K / 64;
    if (!make_map(&tm_xc, CU_TENSOR_MAP_DATA_TYPE_UINT8, x_codes, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2,
                  gp::BK_BYTES, 128) ||
        !make_map(&tm_wc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2,
                  gp::BK_BYTES, 128) ||
        !make_sf_map(&tm_sfa, x_scales, (uint64_t)((M + 127) / 128), (uint64_t)kg4, 1) ||
        // the GEMM-ready copy after the block layout: 32 rows of 512 bytes per 16 KB unit
        !make_sf_map(&tm_sfb, reinterpret_cast<const uint8_t*>(w_scales) + round_up(N, 128) * K / 16,
                     (uint64_t)(wscales_rep_bytes(N, K) / gp::SFB_BYTES), 32, 1, 32))
        return SVDQ_ERR_CUDA;
    if (rank > 0) {
        if (!make_map_3d(&tm_L, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lowrank, (uint64_t)rank, (uint64_t)M, 2,
                         (uint64_t)rank * 2, 64, 128, 1) ||
            !make_map(&tm_Lup, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L_up_t, (uint64_t)rank, (uint64_t)N,
                      (uint64_t)rank * 2, 64, 128))
            return SVDQ_ERR_CUDA;
    } else {
        tm_L = tm_xc;
        tm_Lup = tm_wc;
    }
    GemmArgs a = {};
    a.x_scales = reinterpret_cast<const uint8_t*>(x_scales);
    a.w_scales = reinterpret_cast<const uint8_t*>(w_scales);
    a.x_scale = x_scale;
    a.w_scale = w_scale;
    a.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
    a.y = reinterpret_cast<__nv_bfloat16*>(y);
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.rank = rank;
    a.kg4 = (int)kg4;
    a.n_sf_blocks = (int)((N + 127) / 128);
    if (qkv.heads > 0) {
        a.norm_q = reinterpret_cast<const __nv_bfloat16*>(qkv.norm_q);
        a.norm_k = reinterpret_cast<const __nv_bfloat16*>(qkv.norm_k);
        a.rope_cos = qkv.rope_cos;
        a.rope_sin = qkv.rope_sin;
        a.eps = qkv.eps;
        a.q_cols = qkv.heads * 128;
        a.qk_cols = 2 * qkv.heads * 128;
    }
    if (gelu.store_y) {
        a.gelu_approx = gelu.approx;
    } else if (gelu.next_x_scale) {
        a.gelu_approx = gelu.approx;
        a.nx_inv_lambda = gelu.next_inv_lambda;
        a.nx_ldt = reinterpret_cast<const __nv_bfloat16*>(gelu.next_L_down_t);
        a.nx_rank = gelu.next_rank;
        a.nx_x_scale = gelu.next_x_scale;
        a.nx_codes = reinterpret_cast<uint8_t*>(gelu.next_codes);
        a.nx_scales = reinterpret_cast<uint8_t*>(gelu.next_scales);
        a.nx_acc = gelu.next_acc;
        a.nx_rows_pad = (int)round_up(M, 128);
    }
    const int64_t mt = (M + gp::BM - 1) / gp::BM, nt = (N + gp::BN - 1) / gp::BN;
    if (mt * nt > (int64_t(1) << 30)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    a.m_tiles = (int)mt;
    a.n_tiles = (int)nt;
    const int clusters = (int)std::min<int64_t>(mt * nt, pair_clusters());
    // programmatic dependent launch: the kernel's prologue overlaps the tail of
    // the activation quantizer, which releases its dependents early
    const dim3 grid(2 * (unsigned)clusters), block(gp_threads<kEpiPlain>());   // the QKV variant's too
    cudaError_t e;
    if (gelu.store_y) {
        // h leaves through TMA stores of 32-row x 16-column boxes
        CUtensorMap tm_h;
        if (!make_map(&tm_h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M, (uint64_t)N * 2, 16, 32,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
            return SVDQ_ERR_CUDA;
        e = launch_ex(gemm_nvfp4_pair_kernel<kEpiGeluStore>, grid, dim3(gp::kThreadsGelu), gp::SMEM_BYTES_GELU, st,
                      2u, tm_xc, tm_wc, tm_sfa, tm_sfb, tm_L, tm_Lup, tm_h, a);
    } else if (gelu.next_x_scale) {
        // fc2's codes leave through TMA stores of 32-row x 32-byte boxes
        CUtensorMap tm_codes;
        if (!make_map(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, gelu.next_codes, (uint64_t)N / 2, (uint64_t)M,
                      (uint64_t)N / 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
            return SVDQ_ERR_CUDA;
        e = launch_ex(gemm_nvfp4_pair_kernel<kEpiGelu>, grid, dim3(gp::kThreadsGelu), gp::SMEM_BYTES_GELU, st, 2u,
                      tm_xc, tm_wc, tm_sfa, tm_sfb, tm_L, tm_Lup, tm_codes, a);
    }
    else {
        // y leaves through TMA stores of 32 x 32 boxes (64-byte swizzle)
        CUtensorMap tm_y;
        if (!make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M, (uint64_t)N * 2, 32, 32,
                      CU_TENSOR_MAP_SWIZZLE_64B))
            return SVDQ_ERR_CUDA;
        if (qkv.heads > 0)
            e = launch_ex(gemm_nvfp4_pair_kernel<kEpiQkv>, grid, block, gp::SMEM_BYTES_PLAIN, st, 2u, tm_xc, tm_wc,
                          tm_sfa, tm_sfb, tm_L, tm_Lup, tm_y, a);
        else
            e = launch_ex(gemm_nvfp4_pair_kernel<kEpiPlain>, grid, block, gp::SMEM_BYTES_PLAIN, st, 2u, tm_xc, tm_wc,
                          tm_sfa, tm_sfb, tm_L, tm_Lup, tm_y, a);
    }
    if (e != cudaSuccess) return cuda_fail("gemm_nvfp4_pair_kernel launch");
    return launch_status("gemm_nvfp4_pair_kernel launch");
}

// The int4 GEMMs on fp16 MMAs (gemm_dq16.cuh): int4 W4A4 (a_codes, a_scales:
// the activation's int4 codes and bf16 group scales; rank-r operands) or
// W4A16 (x bf16 in a_codes, a_scales null, rank 0).
svdq_status dq16_gemm(bool int4_a, const void* a_codes, const void* a_scales, int64_t M, const void* w_codes,
                      const void* w_scales, int64_t N, int64_t K, const void* lowrank, const void* L_up_t, int rank,
                      const void* bias, void* y, cudaStream_t st) {
    const int64_t mt = (M + dq::BM - 1) / dq::BM, nt = (N + dq::BN - 1) / dq::BN;
    if (mt > 0x7FFFFFFF || nt > 65535) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    CUtensorMap tm_a, tm_as, tm_wc, tm_ws, tm_L, tm_Lup;
    const int64_t n_pad = round_up(N, 128), m_pad = round_up(M, 128);
    bool ok;
    if (int4_a)
        ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2, 32,
                      128, CU_TENSOR_MAP_SWIZZLE_NONE) &&
             make_map(&tm_as, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a_scales, (uint64_t)m_pad, (uint64_t)(K / 64),
                      (uint64_t)m_pad * 2, 128, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
    else
        ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a_codes, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64,
                      128);
    ok = ok &&
         make_map(&tm_wc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, 32,
                  256, CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_map(&tm_ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_scales, (uint64_t)n_pad, (uint64_t)(K / 64),
                  (uint64_t)n_pad * 2, 256, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && rank > 0)
        ok = make_map_3d(&tm_L, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lowrank, (uint64_t)rank, (uint64_t)M, 2,
                         (uint64_t)rank * 2, 64, dq::BM, 1) &&
             make_map(&tm_Lup, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L_up_t, (uint64_t)rank, (uint64_t)N,
                      (uint64_t)rank * 2, 64, dq::BN);
    if (!ok) return SVDQ_ERR_CUDA;
    if (!int4_a) tm_as = tm_a;
    if (rank == 0) {
        tm_L = tm_a;
        tm_Lup = tm_wc;
    }
    Dq16Args a;
    a.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
    a.y = reinterpret_cast<__nv_bfloat16*>(y);
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.rank = rank;
    const dim3 grid((unsigned)mt, (unsigned)nt, 1);
    if (int4_a)
        gemm_dq16_kernel<true><<<grid, dq::kThreads, dq::SMEM_BYTES, st>>>(tm_a, tm_as, tm_wc, tm_ws, tm_L, tm_Lup, a);
    else
        gemm_dq16_kernel<false><<<grid, dq::kThreads, dq::SMEM_BYTES, st>>>(tm_a, tm_as, tm_wc, tm_ws, tm_L, tm_Lup, a);
    return launch_status("gemm_dq16_kernel launch");
}

// Kernel that waits on a barrier nobody completes: exercises the bounded wait.
__global__ void timeout_probe_kernel() {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, 0xEE);
    __syncthreads();
}

// ------------------------------------------------- no-allocation workspace
// Workspace of svdq_quantize_act_noalloc: a file-scope device array, so that
// callers without a device allocator need not provide one.  Every GPU that
// loads the library holds it until the process exits.
constexpr size_t kNoAllocWorkspaceBytes = size_t(8) << 20;   // 8 MiB
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices];
void* g_noalloc_ctx[kMaxDevices];   // context the cached address belongs to

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_workspace[kNoAllocWorkspaceBytes];

namespace {
// Device address of g_noalloc_workspace on the current device, looked up once
// per device with that device current (the host-side name of the array is
// only a stand-in and must never be handed to a kernel).
svdq_status noalloc_workspace_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return SVDQ_ERR_UNSUPPORTED_DEVICE;
    }
    // the current context: a device reset replaces it, and with it the array's address
    using CtxGetCurrentFn = CUresult (*)(CUcontext*);
    static CtxGetCurrentFn ctx_fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            ctx_fn = reinterpret_cast<CtxGetCurrentFn>(p);
        else
            cudaGetLastError();
    });
    CUcontext ctx = nullptr;
    if (ctx_fn) ctx_fn(&ctx);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev] || g_noalloc_ctx[dev] != (void*)ctx) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_workspace);
        if (e != cudaSuccess || p == nullptr) {
            note_error(e == cudaSuccess ? cudaErrorUnknown : e, "cudaGetSymbolAddress(no-alloc workspace)");
            cudaGetLastError();
            return SVDQ_ERR_CUDA;
        }
        g_noalloc_addr[dev] = p;
        g_noalloc_ctx[dev] = (void*)ctx;
    }
    *out = g_noalloc_addr[dev];
    return SVDQ_OK;
}
}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" {

const char* svdq_status_string(svdq_status s) {
    switch (s) {
        case SVDQ_OK: return "ok";
        case SVDQ_ERR_INVALID_ARG: return "invalid argument";
        case SVDQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case SVDQ_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs compute capability 10.0, sm_100a)";
        case SVDQ_ERR_CUDA: return "CUDA error";
        case SVDQ_ERR_TIMEOUT: return "a kernel timed out waiting on a barrier";
    }
    return "unknown status";
}

int svdq_abi_version(void) { return kAbiVersion; }

const char* svdq_last_error(void) { return g_last_error; }

svdq_status svdq_buffer_sizes(svdq_precision p, int64_t rows, int64_t K, int rank, svdq_sizes* out) {
    if (!out) return SVDQ_ERR_INVALID_ARG;
    if (p != SVDQ_NVFP4 && p != SVDQ_INT4) return SVDQ_ERR_INVALID_ARG;
    SVDQ_TRY(check_rank(rank));
    SVDQ_TRY(check_dims(rows, K));
    const int64_t rows_pad = round_up(rows, 128);
    out->codes_bytes = (size_t)(rows * K / 2);
    out->scales_bytes = p == SVDQ_NVFP4 ? (size_t)(rows_pad * K / 16) : (size_t)(2 * rows_pad * K / 64);
    out->lowrank_bytes = (size_t)(4 * rows * rank);   // hi and lo bf16 planes
    out->w_scales_bytes = out->scales_bytes + (p == SVDQ_NVFP4 ? (size_t)wscales_rep_bytes(rows, K) : 0);
    return SVDQ_OK;
}

svdq_status svdq_pack_weight(svdq_precision p, int group_size, const void* R, int64_t N, int64_t K,
                             const float* lambda, const void* L_down, const void* L_up, int rank, void* w_codes,
                             void* w_scales, float* w_tensor_scale, float* inv_lambda, void* L_down_t, void* L_up_t,
                             svdq_stream_t stream) {
    SVDQ_TRY(check_precision(p, group_size));
    SVDQ_TRY(check_rank(rank));
    SVDQ_TRY(check_dims(N, K));
    if (N % 16 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    SVDQ_TRY(check_ptr(R));
    SVDQ_TRY(check_ptr(lambda));
    SVDQ_TRY(check_ptr(w_codes));
    SVDQ_TRY(check_ptr(w_scales));
    SVDQ_TRY(check_ptr(inv_lambda));
    if (p == SVDQ_NVFP4) SVDQ_TRY(check_ptr(w_tensor_scale));
    if (rank > 0) {
        SVDQ_TRY(check_ptr(L_down));
        SVDQ_TRY(check_ptr(L_up));
        SVDQ_TRY(check_ptr(L_down_t));
        SVDQ_TRY(check_ptr(L_up_t));
    }
    SVDQ_TRY(check_device());
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    SVDQ_TRY(fold_lowrank(lambda, L_down, L_up, N, K, rank, inv_lambda, L_down_t, L_up_t, st));
    if (p == SVDQ_NVFP4) return pack_weight_nvfp4(R, N, K, w_codes, w_scales, w_tensor_scale, st);
    return int4_quantize_rows(R, N, K, w_codes, w_scales, st);
}

svdq_status svdq_replicate_weight_scales(void* w_scales, int64_t N, int64_t K, svdq_stream_t stream) {
    SVDQ_TRY(check_dims(N, K));
    if (N % 16 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    SVDQ_TRY(check_ptr(w_scales));
    SVDQ_TRY(check_device());
    return replicate_weight_scales(w_scales, N, K, reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_quantize_act_workspace_bytes(svdq_precision p, int64_t M, int64_t K, int rank, size_t* bytes) {
    if (!bytes) return SVDQ_ERR_INVALID_ARG;
    if (p != SVDQ_NVFP4 && p != SVDQ_INT4) return SVDQ_ERR_INVALID_ARG;
    SVDQ_TRY(check_rank(rank));
    SVDQ_TRY(check_dims(M, K));
    *bytes = quant_workspace_bytes(M, K, rank);
    return SVDQ_OK;
}

svdq_status svdq_quantize_act(svdq_precision p, int group_size, const void* x, int64_t M, int64_t K,
                              const float* inv_lambda, float* x_tensor_scale, int compute_scale,
                              const float* w_tensor_scale, const void* L_down_t, int rank, void* x_codes,
                              void* x_scales, void* lowrank_act, void* workspace, size_t workspace_bytes,
                              svdq_stream_t stream) {
    SVDQ_TRY(check_precision(p, group_size));
    SVDQ_TRY(check_rank(rank));
    SVDQ_TRY(check_dims(M, K));
    SVDQ_TRY(check_ptr(x));
    SVDQ_TRY(check_ptr(inv_lambda));
    SVDQ_TRY(check_ptr(x_codes));
    SVDQ_TRY(check_ptr(x_scales));
    if (p == SVDQ_NVFP4) SVDQ_TRY(check_ptr(x_tensor_scale));
    if (rank > 0) {
        SVDQ_TRY(check_ptr(L_down_t));
        SVDQ_TRY(check_ptr(lowrank_act));
        if (p == SVDQ_NVFP4) SVDQ_TRY(check_ptr(w_tensor_scale));
    }
    const size_t ws_needed = quant_workspace_bytes(M, K, rank);
    if (ws_needed > 0) {
        SVDQ_TRY(check_ptr(workspace));
        if (workspace_bytes < ws_needed) return SVDQ_ERR_INVALID_ARG;
    } else {
        workspace = nullptr;
    }
    SVDQ_TRY(check_device());
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (p == SVDQ_NVFP4)
        return quantize_act_nvfp4(x, M, K, inv_lambda, x_tensor_scale, compute_scale, w_tensor_scale, L_down_t, rank,
                                  x_codes, x_scales, lowrank_act, workspace, st);
    return quantize_act_launch(kPrecInt4, x, M, K, inv_lambda, nullptr, nullptr, L_down_t, rank, x_codes, x_scales,
                               lowrank_act, workspace, st);
}

svdq_status svdq_quantize_act_noalloc(svdq_precision p, int group_size, const void* x, int64_t M, int64_t K,
                                      const float* inv_lambda, float* x_tensor_scale, int compute_scale,
                                      const float* w_tensor_scale, const void* L_down_t, int rank, void* x_codes,
                                      void* x_scales, void* lowrank_act, svdq_stream_t stream) {
    SVDQ_TRY(check_precision(p, group_size));
    SVDQ_TRY(check_rank(rank));
    SVDQ_TRY(check_dims(M, K));
    SVDQ_TRY(check_ptr(x));
    SVDQ_TRY(check_ptr(inv_lambda));
    SVDQ_TRY(check_ptr(x_codes));
    SVDQ_TRY(check_ptr(x_scales));
    if (p == SVDQ_NVFP4) SVDQ_TRY(check_ptr(x_tensor_scale));
    if (rank > 0) {
        SVDQ_TRY(check_ptr(L_down_t));
        SVDQ_TRY(check_ptr(lowrank_act));
        if (p == SVDQ_NVFP4) SVDQ_TRY(check_ptr(w_tensor_scale));
    }
    const size_t need = quant_workspace_bytes(M, K, rank);
    if (need > kNoAllocWorkspaceBytes) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "svdq_quantize_act_noalloc: this shape needs %zu bytes of workspace, more than the built-in %zu",
                 need, kNoAllocWorkspaceBytes);
        return SVDQ_ERR_UNSUPPORTED_SHAPE;
    }
    void* ws = nullptr;
    if (need > 0) {
        SVDQ_TRY(check_device());
        SVDQ_TRY(noalloc_workspace_address(&ws));
        // the array keeps the previous call's contents: its counters must start at zero
        const int64_t row_blocks = (M + qa::kRows - 1) / qa::kRows;
        if (cudaMemsetAsync(ws, 0, quant_counter_bytes(row_blocks), reinterpret_cast<cudaStream_t>(stream)) !=
            cudaSuccess)
            return cuda_fail("cudaMemsetAsync(no-alloc workspace counters)");
    }
    return svdq_quantize_act(p, group_size, x, M, K, inv_lambda, x_tensor_scale, compute_scale, w_tensor_scale,
                             L_down_t, rank, x_codes, x_scales, lowrank_act, ws, need, stream);
}

svdq_status svdq_gemm_w4a4(svdq_precision p, int group_size, const void* x_codes, const void* x_scales,
                           const float* x_tensor_scale, int64_t M, const void* w_codes, const void* w_scales,
                           const float* w_tensor_scale, int64_t N, int64_t K, const void* lowrank_act,
                           const void* L_up_t, int rank, const void* bias, void* y, svdq_stream_t stream) {
    SVDQ_TRY(check_precision(p, group_size));
    SVDQ_TRY(check_rank(rank));
    SVDQ_TRY(check_dims(M, K));
    SVDQ_TRY(check_dims(N, K));
    if (N % 16 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    SVDQ_TRY(check_ptr(x_codes));
    SVDQ_TRY(check_ptr(x_scales));
    SVDQ_TRY(check_ptr(w_codes));
    SVDQ_TRY(check_ptr(w_scales));
    SVDQ_TRY(check_ptr(y));
    SVDQ_TRY(check_opt_ptr(bias));
    if (p == SVDQ_NVFP4) {
        SVDQ_TRY(check_ptr(x_tensor_scale));
        SVDQ_TRY(check_ptr(w_tensor_scale));
    }
    if (rank > 0) {
        SVDQ_TRY(check_ptr(lowrank_act));
        SVDQ_TRY(check_ptr(L_up_t));
    }
    SVDQ_TRY(check_device());
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (p == SVDQ_NVFP4) {
        const int mode = g_gemm_tiles_mode.load();
        if (mode == 2 || (mode == 0 && M > 128))
            return gemm_nvfp4_pair(x_codes, x_scales, x_tensor_scale, M, w_codes, w_scales, w_tensor_scale, N, K,
                                   lowrank_act, L_up_t, rank, bias, y, st);
        return gemm_nvfp4(x_codes, x_scales, x_tensor_scale, M, w_codes, w_scales, w_tensor_scale, N, K, lowrank_act,
                          L_up_t, rank, bias, y, st);
    }
    return dq16_gemm(true, x_codes, x_scales, M, w_codes, w_scales, N, K, lowrank_act, L_up_t, rank, bias, y, st);
}

// Checks of the fused QKV + RMSNorm + RoPE arguments shared by both entry points.
static svdq_status check_qkv_args(int64_t M, int64_t N, int heads, int head_dim, const void* norm_q,
                                  const void* norm_k, float eps, const float* rope_cos, const float* rope_sin) {
    if (head_dim != 128 || heads < 1) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    if (N != 3 * (int64_t)heads * head_dim) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    if (!(eps > 0.0f) || !(eps < 1.0f)) return SVDQ_ERR_INVALID_ARG;
    SVDQ_TRY(check_ptr(norm_q));
    SVDQ_TRY(check_ptr(norm_k));
    SVDQ_TRY(check_ptr(rope_cos));
    SVDQ_TRY(check_ptr(rope_sin));
    if (M < 1) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    return SVDQ_OK;
}

svdq_status svdq_gemm_w4a4_qkv_norm_rope(svdq_precision p, int group_size, const void* x_codes, const void* x_scales,
                                         const float* x_tensor_scale, int64_t M, const void* w_codes,
                                         const void* w_scales, const float* w_tensor_scale, int64_t N, int64_t K,
                                         const void* lowrank_act, const void* L_up_t, int rank, const void* bias,
                                         int heads, int head_dim, const void* norm_q, const void* norm_k, float eps,
                                         const float* rope_cos, const float* rope_sin, void* y,
                                         svdq_stream_t stream) {
    SVDQ_TRY(check_precision(p, group_size));
    if (p != SVDQ_NVFP4) return SVDQ_ERR_INVALID_ARG;   // the fused epilogue belongs to the nvfp4 GEMM
    SVDQ_TRY(check_rank(rank));
    SVDQ_TRY(check_dims(M, K));
    SVDQ_TRY(check_dims(N, K));
    SVDQ_TRY(check_qkv_args(M, N, heads, head_dim, norm_q, norm_k, eps, rope_cos, rope_sin));
    SVDQ_TRY(check_ptr(x_codes));
    SVDQ_TRY(check_ptr(x_scales));
    SVDQ_TRY(check_ptr(w_codes));
    SVDQ_TRY(check_ptr(w_scales));
    SVDQ_TRY(check_ptr(y));
    SVDQ_TRY(check_opt_ptr(bias));
    SVDQ_TRY(check_ptr(x_tensor_scale));
    SVDQ_TRY(check_ptr(w_tensor_scale));
    if (rank > 0) {
        SVDQ_TRY(check_ptr(lowrank_act));
        SVDQ_TRY(check_ptr(L_up_t));
    }
    SVDQ_TRY(check_device());
    QkvEpilogue e;
    e.heads = heads;
    e.norm_q = norm_q;
    e.norm_k = norm_k;
    e.eps = eps;
    e.rope_cos = rope_cos;
    e.rope_sin = rope_sin;
    return gemm_nvfp4_pair(x_codes, x_scales, x_tensor_scale, M, w_codes, w_scales, w_tensor_scale, N, K, lowrank_act,
                           L_up_t, rank, bias, y, reinterpret_cast<cudaStream_t>(stream), e);
}

svdq_status svdq_qkv_norm_rope(const void* y_in, void* y_out, int64_t M, int heads, int head_dim, const void* norm_q,
                               const void* norm_k, float eps, const float* rope_cos, const float* rope_sin,
                               svdq_stream_t stream) {
    SVDQ_TRY(check_ptr(y_in));
    SVDQ_TRY(check_ptr(y_out));
    if (M >= (int64_t(1) << 31)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    SVDQ_TRY(check_qkv_args(M, 3 * (int64_t)heads * head_dim, heads, head_dim, norm_q, norm_k, eps, rope_cos,
                            rope_sin));
    SVDQ_TRY(check_device());
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t warps = M * 2 * heads;
    const int64_t blocks = (warps + 7) / 8;
    if (blocks > 0x7FFFFFFF) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    qkv_norm_rope_kernel<<<(unsigned)blocks, 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(y_in), reinterpret_cast<__nv_bfloat16*>(y_out), M, heads,
        reinterpret_cast<const __nv_bfloat16*>(norm_q), reinterpret_cast<const __nv_bfloat16*>(norm_k), eps, rope_cos,
        rope_sin);
    SVDQ_TRY(launch_status("qkv_norm_rope_kernel launch"));
    if (y_out != y_in) {
        const int64_t n8 = M * heads * 128 / 8;
        const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((n8 + 255) / 256, 8LL * num_sms()));
        copy_v_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(y_in),
                                             reinterpret_cast<__nv_bfloat16*>(y_out), M, heads);
        SVDQ_TRY(launch_status("copy_v_kernel launch"));
    }
    return SVDQ_OK;
}

svdq_status svdq_gelu_mlp_workspace_bytes(int64_t M, int next_rank, size_t* bytes) {
    if (!bytes) return SVDQ_ERR_INVALID_ARG;
    SVDQ_TRY(check_rank(next_rank));
    if (next_rank > 32 || M < 1 || M >= (int64_t(1) << 31)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    *bytes = (size_t)M * (size_t)next_rank * sizeof(float);
    return SVDQ_OK;
}

svdq_status svdq_gemm_w4a4_gelu(svdq_precision p, int group_size, const void* x_codes, const void* x_scales,
                                const float* x_tensor_scale, int64_t M, const void* w_codes, const void* w_scales,
                                const float* w_tensor_scale, int64_t N, int64_t K, const void* lowrank_act,
                                const void* L_up_t, int rank, const void* bias, int gelu_approx, void* y,
                                svdq_stream_t stream) {
    SVDQ_TRY(check_precision(p, group_size));
    if (p != SVDQ_NVFP4) return SVDQ_ERR_INVALID_ARG;   // the GELU epilogue belongs to the nvfp4 GEMM
    SVDQ_TRY(check_rank(rank));
    if (gelu_approx != 0 && gelu_approx != 1) return SVDQ_ERR_INVALID_ARG;
    SVDQ_TRY(check_dims(M, K));
    SVDQ_TRY(check_dims(N, K));
    if (N % 128 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;   // whole 64-column pieces per epilogue warp
    SVDQ_TRY(check_ptr(x_codes));
    SVDQ_TRY(check_ptr(x_scales));
    SVDQ_TRY(check_ptr(w_codes));
    SVDQ_TRY(check_ptr(w_scales));
    SVDQ_TRY(check_ptr(x_tensor_scale));
    SVDQ_TRY(check_ptr(w_tensor_scale));
    SVDQ_TRY(check_opt_ptr(bias));
    SVDQ_TRY(check_ptr(y));
    if (rank > 0) {
        SVDQ_TRY(check_ptr(lowrank_act));
        SVDQ_TRY(check_ptr(L_up_t));
    }
    SVDQ_TRY(check_device());
    GeluEpilogue g;
    g.store_y = true;
    g.approx = gelu_approx;
    return gemm_nvfp4_pair(x_codes, x_scales, x_tensor_scale, M, w_codes, w_scales, w_tensor_scale, N, K,
                           lowrank_act, L_up_t, rank, bias, y, reinterpret_cast<cudaStream_t>(stream), QkvEpilogue(),
                           g);
}

svdq_status svdq_gemm_w4a4_gelu_quant(svdq_precision p, int group_size, const void* x_codes, const void* x_scales,
                                      const float* x_tensor_scale, int64_t M, const void* w_codes,
                                      const void* w_scales, const float* w_tensor_scale, int64_t N, int64_t K,
                                      const void* lowrank_act, const void* L_up_t, int rank, const void* bias,
                                      int gelu_approx, const float* next_inv_lambda, const void* next_L_down_t,
                                      int next_rank, const float* next_x_tensor_scale,
                                      const float* next_w_tensor_scale, void* next_x_codes, void* next_x_scales,
                                      void* next_lowrank_act, void* workspace, size_t workspace_bytes,
                                      svdq_stream_t stream) {
    SVDQ_TRY(check_precision(p, group_size));
    if (p != SVDQ_NVFP4) return SVDQ_ERR_INVALID_ARG;   // the fused epilogue belongs to the nvfp4 GEMM
    SVDQ_TRY(check_rank(rank));
    SVDQ_TRY(check_rank(next_rank));
    if (next_rank > 32) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    if (gelu_approx != 0 && gelu_approx != 1) return SVDQ_ERR_INVALID_ARG;
    SVDQ_TRY(check_dims(M, K));
    SVDQ_TRY(check_dims(N, K));
    if (N % 128 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;   // N is the next layer's K
    SVDQ_TRY(check_ptr(x_codes));
    SVDQ_TRY(check_ptr(x_scales));
    SVDQ_TRY(check_ptr(w_codes));
    SVDQ_TRY(check_ptr(w_scales));
    SVDQ_TRY(check_ptr(x_tensor_scale));
    SVDQ_TRY(check_ptr(w_tensor_scale));
    SVDQ_TRY(check_opt_ptr(bias));
    if (rank > 0) {
        SVDQ_TRY(check_ptr(lowrank_act));
        SVDQ_TRY(check_ptr(L_up_t));
    }
    SVDQ_TRY(check_ptr(next_inv_lambda));
    SVDQ_TRY(check_ptr(next_x_tensor_scale));
    SVDQ_TRY(check_ptr(next_x_codes));
    SVDQ_TRY(check_ptr(next_x_scales));
    if (next_rank > 0) {
        SVDQ_TRY(check_ptr(next_L_down_t));
        SVDQ_TRY(check_ptr(next_w_tensor_scale));
        SVDQ_TRY(check_ptr(next_lowrank_act));
        SVDQ_TRY(check_ptr(workspace));
        if (workspace_bytes < (size_t)M * (size_t)next_rank * sizeof(float)) return SVDQ_ERR_INVALID_ARG;
    }
    SVDQ_TRY(check_device());
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    GeluEpilogue g;
    g.approx = gelu_approx;
    g.next_inv_lambda = next_inv_lambda;
    g.next_L_down_t = next_L_down_t;
    g.next_rank = next_rank;
    g.next_x_scale = next_x_tensor_scale;
    g.next_codes = next_x_codes;
    g.next_scales = next_x_scales;
    g.next_acc = reinterpret_cast<float*>(workspace);
    SVDQ_TRY(gemm_nvfp4_pair(x_codes, x_scales, x_tensor_scale, M, w_codes, w_scales, w_tensor_scale, N, K,
                             lowrank_act, L_up_t, rank, bias, nullptr, st, QkvEpilogue(), g));
    if (next_rank > 0) {
        const int64_t count = M * next_rank;
        const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((count + 255) / 256, 2LL * num_sms()));
        if (launch_ex(lowrank_finalize_kernel, dim3((unsigned)grid), dim3(256), 0, st, 1u,
                      reinterpret_cast<float*>(workspace), count, next_x_tensor_scale, next_w_tensor_scale,
                      reinterpret_cast<__nv_bfloat16*>(next_lowrank_act)) != cudaSuccess)
            return cuda_fail("lowrank_finalize_kernel launch");
        SVDQ_TRY(launch_status("lowrank_finalize_kernel launch"));
    }
    return SVDQ_OK;
}

svdq_status svdq_gelu(const void* x, void* y, int64_t n, int approx, svdq_stream_t stream) {
    SVDQ_TRY(check_ptr(x));
    SVDQ_TRY(check_ptr(y));
    if (approx != 0 && approx != 1) return SVDQ_ERR_INVALID_ARG;
    if (n < 1 || n >= (int64_t(1) << 40)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    SVDQ_TRY(check_device());
    const int64_t n8 = n / 8;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((n8 + 255) / 256, 8LL * num_sms()));
    gelu_bf16_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), reinterpret_cast<__nv_bfloat16*>(y), n, approx);
    return launch_status("gelu_bf16_kernel launch");
}

svdq_status svdq_gemm_w4a16(const void* x, int64_t M, const void* w_codes, const void* w_scales, int64_t N,
                            int64_t K, const void* bias, void* y, svdq_stream_t stream) {
    SVDQ_TRY(check_dims(M, K));
    SVDQ_TRY(check_dims(N, K));
    if (N % 16 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    SVDQ_TRY(check_ptr(x));
    SVDQ_TRY(check_ptr(w_codes));
    SVDQ_TRY(check_ptr(w_scales));
    SVDQ_TRY(check_ptr(y));
    SVDQ_TRY(check_opt_ptr(bias));
    SVDQ_TRY(check_device());
    return dq16_gemm(false, x, nullptr, M, w_codes, w_scales, N, K, nullptr, nullptr, 0, bias, y,
                     reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_svd_split_workspace_bytes(int64_t N, int64_t K, int rank, int oversample, size_t* bytes) {
    if (!bytes) return SVDQ_ERR_INVALID_ARG;
    if (rank < 1 || oversample < 0 || rank + oversample > sv::kMaxL) return SVDQ_ERR_INVALID_ARG;
    SVDQ_TRY(check_dims(N, K));
    if (rank > std::min(N, K)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    *bytes = svd_split_workspace(N, K, rank + oversample);
    return SVDQ_OK;
}

svdq_status svdq_svd_split(const void* W, const float* lambda, int64_t N, int64_t K, int rank, const float* omega,
                           int oversample, int power_iters, void* R, void* L_down, void* L_up,
                           float* singular_values, void* workspace, size_t workspace_bytes, svdq_stream_t stream) {
    if (rank < 1 || oversample < 0 || rank + oversample > sv::kMaxL || power_iters < 0 || power_iters > 16)
        return SVDQ_ERR_INVALID_ARG;
    SVDQ_TRY(check_dims(N, K));
    if (rank > std::min(N, K) || N >= (int64_t(1) << 31) / sv::kMaxL) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    SVDQ_TRY(check_ptr(W));
    SVDQ_TRY(check_ptr(lambda));
    SVDQ_TRY(check_ptr(omega));
    SVDQ_TRY(check_ptr(R));
    SVDQ_TRY(check_ptr(L_down));
    SVDQ_TRY(check_ptr(L_up));
    SVDQ_TRY(check_opt_ptr(singular_values));
    SVDQ_TRY(check_ptr(workspace));
    const int l = rank + oversample;
    if (workspace_bytes < svd_split_workspace(N, K, l)) return SVDQ_ERR_INVALID_ARG;
    SVDQ_TRY(check_device());
    static std::once_flag jac_once;
    static cudaError_t jac_err = cudaSuccess;
    std::call_once(jac_once, [] {
        jac_err = cudaFuncSetAttribute(svd_jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kJacobiSmem);
    });
    if (jac_err != cudaSuccess) return cuda_fail("setting the Jacobi kernel's shared memory");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    float* Y = reinterpret_cast<float*>(ws);
    ws += round_up(N * l * (int64_t)sizeof(float), 256);
    float* Z = reinterpret_cast<float*>(ws);
    ws += round_up(K * l * (int64_t)sizeof(float), 256);
    double* part = reinterpret_cast<double*>(ws);
    double* Rinv = part + (size_t)sv::kGramBlocks * sv::kMaxL * sv::kMaxL;
    double* U = Rinv + (size_t)sv::kMaxL * sv::kMaxL;
    double* evals = U + (size_t)sv::kMaxL * sv::kMaxL;
    const __nv_bfloat16* Wb = reinterpret_cast<const __nv_bfloat16*>(W);
    const unsigned gN = (unsigned)((N + sv::kTileR - 1) / sv::kTileR), gK = (unsigned)((K + sv::kTileR - 1) / sv::kTileR);
    // range finder with subspace iteration
    svd_w_times_kernel<<<gN, 256, 0, st>>>(Wb, lambda, N, K, omega, l, Y);
    SVDQ_TRY(svd_orth(Y, N, l, part, Rinv, st));
    for (int q = 0; q < power_iters; ++q) {
        svd_wt_times_kernel<<<gK, 256, 0, st>>>(Wb, lambda, N, K, Y, l, Z);
        SVDQ_TRY(svd_orth(Z, K, l, part, Rinv, st));
        svd_w_times_kernel<<<gN, 256, 0, st>>>(Wb, lambda, N, K, Z, l, Y);
        SVDQ_TRY(svd_orth(Y, N, l, part, Rinv, st));
    }
    // B^T = W_hat^T Q and the SVD of B from the eigen-decomposition of B B^T
    svd_wt_times_kernel<<<gK, 256, 0, st>>>(Wb, lambda, N, K, Y, l, Z);
    svd_gram_partial_kernel<<<sv::kGramBlocks, 256, 0, st>>>(Z, K, l, part);
    svd_jacobi_kernel<<<1, 32, kJacobiSmem, st>>>(part, sv::kGramBlocks, l, evals, U);
    SVDQ_TRY(launch_status("SVD split: small eigen-problem"));
    const int64_t rows = std::max(N, K);
    svd_factors_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(
        Y, N, Z, K, l, rank, evals, U, reinterpret_cast<__nv_bfloat16*>(L_up),
        reinterpret_cast<__nv_bfloat16*>(L_down), singular_values);
    svd_residual_kernel<<<dim3((unsigned)((K + 63) / 64), (unsigned)((N + 31) / 32)), 256, 0, st>>>(
        Wb, lambda, N, K, reinterpret_cast<const __nv_bfloat16*>(L_up), reinterpret_cast<const __nv_bfloat16*>(L_down),
        rank, reinterpret_cast<__nv_bfloat16*>(R));
    return launch_status("SVD split: factors and residual");
}

svdq_status svdq_device_status(int clear, int* site) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return SVDQ_ERR_UNSUPPORTED_DEVICE;
    }
    if (cudaDeviceSynchronize() != cudaSuccess) return cuda_fail();
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_status_word, sizeof(word)) != cudaSuccess) return cuda_fail();
    if (site) *site = (int)((word >> 8) & 0xFFu);
    if (clear && word) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero)) != cudaSuccess) return cuda_fail();
    }
    return (word & 1u) ? SVDQ_ERR_TIMEOUT : SVDQ_OK;
}

svdq_status svdq_debug_set_wait_limit_ns(uint64_t ns) {
    SVDQ_TRY(check_device());
    const unsigned long long v = ns ? (unsigned long long)ns : 2000000000ull;
    if (cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return cuda_fail();
    return SVDQ_OK;
}

svdq_status svdq_debug_timeout_probe(svdq_stream_t stream) {
    SVDQ_TRY(check_device());
    timeout_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
    return launch_status("timeout_probe_kernel launch");
}

svdq_status svdq_debug_force_gemm_tiles(int mode) {
    if (mode < 0 || mode > 2) {
        snprintf(g_last_error, sizeof(g_last_error), "svdq_debug_force_gemm_tiles: mode %d is not 0, 1 or 2",
                 mode);
        return SVDQ_ERR_INVALID_ARG;
    }
    g_gemm_tiles_mode.store(mode);
    return SVDQ_OK;
}

svdq_status svdq_debug_force_quant_plan(int mode) {
    if (mode < 0 || mode > 3) {
        snprintf(g_last_error, sizeof(g_last_error), "svdq_debug_force_quant_plan: mode %d is not 0, 1, 2 or 3",
                 mode);
        return SVDQ_ERR_INVALID_ARG;
    }
    g_quant_plan_mode.store(mode);
    return SVDQ_OK;
}

void svdq_debug_override_capability(int major, int minor) {
    std::lock_guard<std::mutex> lock(g_mutex);
    g_override_major = major;
    g_override_minor = minor;
}

}  // extern "C"
