// gemm_w4a16.cuh -- the weight-only int4 GEMM (W4A16) of the `awq_w4a16`
// scheme (sm_100a): the "INT4 weight-only AWQ-style kernel", int4 with group
// 64, of the Diffusers docs page "Nunchaku Lite" ("Supported quantization
// types" table; the `awq_w4a16` targets of "NunchakuLiteQuantizationConfig").
//
//   y[m, n] = bf16( sum_k x[m, k] * (q[n, k] * s[n, k / 64]) + b[n] )
//
// with q the signed int4 codes and s the bf16 group scales that
// svdq_pack_weight writes for SVDQ_INT4 (the activation-aware scaling of AWQ
// is folded into the weights and the preceding layer offline, so x arrives
// as is).  Each product q s is exact in fp16 (a 3-bit integer times an 8-bit
// significand), and a bf16 x converts exactly to fp16 in fp16's normal range,
// so the tensor cores multiply fp16 x fp16 (kind::f16) with fp32
// accumulation and no per-group rescale is left for the CUDA cores.
//
// One CTA per 128 x 256 output tile.  Warp 0 loads, per 64 columns of K, the
// x tile (bf16, TMA, 128-byte swizzle), the packed weight tile (256 rows x 32
// bytes) and its 256 group scales; warps 4..11 convert x to fp16 in place and
// expand the weight codes into an fp16 tile in the MMA's swizzled layout;
// warp 1 issues four M = 128, N = 256, K = 16 MMAs per stage into TMEM;
// warps 12..19 add the bias and store bf16.
#pragma once
#include "sm100_ptx.cuh"

namespace svdq {
namespace aw {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int kStages = 3;
constexpr int X_BYTES = 128 * 128;            // x: 128 rows x 64 values (bf16, converted to fp16 in place)
constexpr int WF_BYTES = 256 * 128;           // fp16 weights: 256 rows x 64 values
constexpr int WP_BYTES = 256 * 32;            // packed int4 weights: 256 rows x 64 codes
constexpr int WS_BYTES = 256 * 2;             // bf16 group scales of the 256 rows
constexpr int STAGE_BYTES = X_BYTES + WF_BYTES + WP_BYTES + 1024;   // scales in the last 1 KB
constexpr int kConvWarp0 = 4, kConvWarps = 8;
constexpr int kEpiWarp0 = 12, kEpiWarps = 8;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr size_t SMEM_BYTES = 1024 + (size_t)kStages * STAGE_BYTES + 256;
static_assert(SMEM_BYTES <= 227 * 1024, "stage ring does not fit in shared memory");
}  // namespace aw

struct W4A16Args {
    const __nv_bfloat16* bias;   // may be null
    __nv_bfloat16* y;
    int M, N, K;
};

enum : uint32_t { kSiteAwEmpty = 40, kSiteAwFull = 41, kSiteAwConv = 42, kSiteAwAcc = 43, kSiteAwDrain = 44 };

__host__ __device__ constexpr uint32_t idesc_f16_f32(uint32_t n) {
    return (1u << 4)            // D format f32; A and B format f16 (0)
           | ((n >> 3) << 17)   // N / 8
           | ((128u >> 4) << 24);  // M / 16
}

// 8 int4 codes (two's complement, element i in bits 4i+3..4i) times the fp16
// scale pair s2 -> 8 fp16 values in element order (four fp16x2 words).  The
// nibble n is q + 8 after flipping its top bit, and the fp16 with bits
// 0x6400 | (q + 8) is 1024 + q + 8; subtracting 1032 leaves q exactly.
__device__ __forceinline__ void int4x8_to_f16(uint32_t w, __half2 s2, uint32_t (&out)[4]) {
    const uint32_t u = w ^ 0x88888888u;
    const __half2 bias2 = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));   // 1032
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        // elements 2p (bits 8p..8p+3) and 2p+1 (bits 8p+4..8p+7)
        const uint32_t lo = (u >> (8 * p)) & 0xFu, hi = (u >> (8 * p + 4)) & 0xFu;
        const uint32_t bits = (0x6400u | lo) | ((0x6400u | hi) << 16);
        __half2 v = *reinterpret_cast<const __half2*>(&bits);
        v = __hmul2(__hsub2(v, bias2), s2);
        out[p] = *reinterpret_cast<const uint32_t*>(&v);
    }
}

__global__ void __launch_bounds__(aw::kThreads, 1)
    gemm_w4a16_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wc,
                      const __grid_constant__ CUtensorMap tm_ws, W4A16Args a) {
    using namespace aw;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kStages * STAGE_BYTES);
    uint64_t* conv = full + kStages;
    uint64_t* empty = conv + kStages;
    uint64_t* acc_full = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    __shared__ int s_failed;
    __shared__ int s_issued[aw::kStages];

    const uint32_t warp = warp_id(), lane = lane_id();
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
    const int n_kc = a.K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], kConvWarps);
            mbar_init(&empty[s], 1);
            s_issued[s] = 0;
        }
        mbar_init(acc_full, 1);
        s_failed = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_wc);
        prefetch_tensormap(&tm_ws);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int kc = 0; kc < n_kc; ++kc) {
                const int s = kc % kStages;
                const uint32_t ph = (uint32_t)(kc / kStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, kSiteAwEmpty)) {
                    s_failed = 1;
                    break;
                }
                uint8_t* st = smem + (size_t)s * STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], X_BYTES + WP_BYTES + WS_BYTES);
                tma_load_2d(st, &tm_x, &full[s], kc * 64, m0);
                tma_load_2d(st + X_BYTES + WF_BYTES, &tm_wc, &full[s], kc * 32, n0);
                tma_load_2d(st + X_BYTES + WF_BYTES + WP_BYTES, &tm_ws, &full[s], n0, kc);
                reinterpret_cast<volatile int*>(s_issued)[s] += 1;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_m(idesc_f16_f32(BN), BM);
            bool ok = true;
            for (int kc = 0; kc < n_kc; ++kc) {
                const int s = kc % kStages;
                if (!mbar_wait(&conv[s], (uint32_t)(kc / kStages) & 1u, kSiteAwConv)) {
                    ok = false;
                    s_failed = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t sx = smem_u32(smem + (size_t)s * STAGE_BYTES), sw = sx + X_BYTES;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_bf16(tmem, desc_sw128(sx + 32u * j), desc_sw128(sw + 32u * j), idesc, (kc > 0 || j > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            if (ok) tc_commit(acc_full);
        }
    } else if (warp >= (uint32_t)kConvWarp0 && warp < (uint32_t)kConvWarp0 + kConvWarps) {
        // ----------------------------------------- x -> fp16, int4 -> fp16 (q s)
        const int t = (int)threadIdx.x - 32 * kConvWarp0;   // 0..255: one weight row each
        for (int kc = 0; kc < n_kc; ++kc) {
            const int s = kc % kStages;
            if (!mbar_wait(&full[s], (uint32_t)(kc / kStages) & 1u, kSiteAwFull)) {
                s_failed = 1;
                break;
            }
            uint8_t* st = smem + (size_t)s * STAGE_BYTES;
            // x: 16 KB of bf16 in place, 64 bytes per thread (position-preserving)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint4* p = reinterpret_cast<uint4*>(st + 16 * (t + 256 * i));
                const uint4 v = *p;
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __half2 h = __floats2half2_rn(bf16lo_to_f32(w[e]), bf16hi_to_f32(w[e]));
                    o[e] = *reinterpret_cast<const uint32_t*>(&h);
                }
                *p = make_uint4(o[0], o[1], o[2], o[3]);
            }
            // weight row t: 64 codes -> 64 fp16 in the swizzled 128-byte row
            const uint8_t* wp = st + X_BYTES + WF_BYTES + 32 * t;
            const uint16_t sbits = *reinterpret_cast<const uint16_t*>(st + X_BYTES + WF_BYTES + WP_BYTES + 2 * t);
            const __half sh = __float2half_rn(__bfloat162float(__ushort_as_bfloat16(sbits)));
            const __half2 s2 = __halves2half2(sh, sh);
            const uint4 c0 = *reinterpret_cast<const uint4*>(wp), c1 = *reinterpret_cast<const uint4*>(wp + 16);
            const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint8_t* wrow = st + X_BYTES + (t >> 7) * (128 * 128) + (t & 127) * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {   // 16-byte chunk c: K values 8c .. 8c + 7
                uint32_t o[4];
                int4x8_to_f16(cw[c], s2, o);
                *reinterpret_cast<uint4*>(wrow + ((c ^ (t & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_proxy_async_smem();   // both tiles are read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&conv[s]);
        }
    } else if (warp >= (uint32_t)kEpiWarp0) {
        // ------------------------------------------------------------ epilogue
        const uint32_t q = warp & 3u;
        const int half = (int)(warp - kEpiWarp0) >> 2;
        const int64_t grow = (int64_t)m0 + 32 * q + lane;
        const bool ok = mbar_wait(acc_full, 0, kSiteAwAcc);
        if (!ok) s_failed = 1;
        tc_fence_after();
        if (ok) {
            __nv_bfloat16* yrow = a.y + grow * (int64_t)a.N;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t acc[32];
                tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + 128u * half + 32u * c, acc);
                tmem_ld_wait();
                const int n = n0 + 128 * half + 32 * c;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    if (n + 8 * p >= a.N) break;   // N % 16 == 0
                    uint4 bw = make_uint4(0u, 0u, 0u, 0u);
                    if (a.bias) bw = __ldg(reinterpret_cast<const uint4*>(a.bias + n + 8 * p));
                    const uint32_t ws[4] = {bw.x, bw.y, bw.z, bw.w};
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float o0 = __fadd_rn(__uint_as_float(acc[8 * p + 2 * i]), bf16lo_to_f32(ws[i]));
                        const float o1 = __fadd_rn(__uint_as_float(acc[8 * p + 2 * i + 1]), bf16hi_to_f32(ws[i]));
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(o0, o1);
                        pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
                    }
                    if (grow < a.M) *reinterpret_cast<uint4*>(yrow + n + 8 * p) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
    }

    __syncthreads();
    if (s_failed && warp == 0 && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            const int n = reinterpret_cast<volatile int*>(s_issued)[s];
            if (n > 0) mbar_wait(&full[s], (uint32_t)(n - 1) & 1u, kSiteAwDrain);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace svdq
