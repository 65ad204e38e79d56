// gemm_dq16.cuh -- the two int4 GEMMs of the Diffusers docs page "Nunchaku
// Lite" ("Supported quantization types" table), on fp16 tensor-core MMAs
// (sm_100a):
//
//  * W4A16, the `awq_w4a16` scheme (int4 weights, group 64; the AWQ scaling
//    folded into the weights offline, x used as it comes):
//        y[m, n] = bf16( sum_k x[m, k] (q_w[n, k] s_w[n, k / 64]) + b[n] )
//  * the int4 W4A4 variant of the SVDQ layer (`svdq_w4a4` with precision
//    int4, group 64, with the rank-r correction):
//        y[m, n] = bf16( sum_k (q_x[m, k] s_x[m, k / 64]) (q_w[n, k] s_w[n, k / 64])
//                        + sum_j L[m, j] L_up[j, n] + b[n] )
//
// Every product q s of a signed 4-bit code and a bf16 group scale is exact in
// fp16 (at most 3 + 8 significant bits, for scales in fp16's normal range),
// and a bf16 activation converts exactly to fp16 in fp16's normal range.  So
// both operands are expanded into fp16 tiles in shared memory and multiplied
// with kind::f16 MMAs (fp16 x fp16, fp32 accumulation): the group scales are
// applied before the MMA instead of on the accumulators, and no per-group
// rescale is left for the CUDA cores.  The rank-r term runs as bf16 MMAs
// (the hi and lo parts of L against L_up) into the same accumulator.
//
// One CTA per 128 x 256 output tile, computed transposed: the tensor core
// takes the weights as its A operand from TMEM and the activations as B from
// shared memory, two M = 128 (weight rows), N = 128 (activation rows), K = 16
// MMAs per 16 values of K into two TMEM accumulators.  Warp 0 loads, per 64
// columns of K, the activation tile (bf16 x, or int4 codes and their group
// scales), the packed weight tile (256 rows x 32 bytes) and its 256 group
// scales; warps 4..19 expand the activations into an fp16 tile in the MMA's
// swizzled layout in shared memory and the weights into fp16 rows of TMEM
// (tcgen05.st: lane = weight row, two values per column); warp 1 issues the
// MMAs; after the last stage warps 12..19 add the bias and store bf16,
// transposing through shared memory.  Expanding the weights into TMEM instead
// of shared memory takes their 32 KB per stage of stores and tensor-core reads
// off the shared-memory pipe, which the expansion and the MMAs otherwise
// saturate.  The rank-r chunks (already bf16) are multiplied from shared
// memory (L_up as A, L as B).
#pragma once
#include "sm100_ptx.cuh"

namespace svdq {
namespace dq {
constexpr int BM = 128;                       // activation rows per tile
constexpr int BN = 256;                       // weight rows per tile
constexpr int kStages = 4;
constexpr int XF_BYTES = 128 * 128;           // fp16 activations: 128 rows x 64 values (x arrives here as bf16;
                                              // a rank-r chunk's bf16 L tile)
constexpr int AP_BYTES = 128 * 32;            // packed int4 activations: 128 rows x 64 codes
constexpr int WP_BYTES = 256 * 32;            // packed int4 weights: 256 rows x 64 codes
constexpr int WS_BYTES = 256 * 2;             // bf16 group scales of the 256 weight rows
constexpr int AS_BYTES = 128 * 2;             // bf16 group scales of the 128 activation rows
constexpr int OFF_AP = XF_BYTES;
constexpr int OFF_WP = OFF_AP + AP_BYTES;
constexpr int OFF_WS = OFF_WP + WP_BYTES;
constexpr int OFF_AS = OFF_WS + WS_BYTES;
constexpr int OFF_LUP = XF_BYTES;             // a rank-r chunk's L_up tile: 256 rows x 64 bf16 (two 16 KB halves)
constexpr int LUP_BYTES = 256 * 128;
constexpr int STAGE_BYTES = XF_BYTES + LUP_BYTES;   // a rank-r chunk is the largest stage
static_assert(OFF_AS + AS_BYTES <= STAGE_BYTES, "packed tiles do not fit in a stage");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t D_COL = 0;                 // weight rows 0-127 at column 0, rows 128-255 at 128 (fp32)
constexpr uint32_t WT_COL = 256;              // stage s: fp16 weight rows 0-127 at 256 + 64 s, rows 128-255 at + 32
static_assert(WT_COL + 64 * kStages <= TMEM_COLS, "weight tiles do not fit in TMEM");
constexpr int kConvWarp0 = 4, kConvWarps = 16;   // the epilogue warps convert too
constexpr int kEpiWarp0 = 12, kEpiWarps = 8;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr size_t SMEM_BYTES = 1024 + (size_t)kStages * STAGE_BYTES + 256;
static_assert(SMEM_BYTES <= 227 * 1024, "stage ring does not fit in shared memory");
}  // namespace dq

struct Dq16Args {
    const __nv_bfloat16* bias;   // may be null
    __nv_bfloat16* y;
    int M, N, K;
    int rank;                    // int4 W4A4: rank-r chunks appended to the K loop
};

enum : uint32_t { kSiteDqEmpty = 40, kSiteDqFull = 41, kSiteDqConv = 42, kSiteDqAcc = 43, kSiteDqDrain = 44 };

__host__ __device__ constexpr uint32_t idesc_f16_f32(uint32_t n) {
    return (1u << 4)            // D format f32; A and B format f16 (0)
           | ((n >> 3) << 17)   // N / 8
           | ((128u >> 4) << 24);  // M / 16
}

// D[tmem] (+)= A[tmem] * B[smem]^T, fp16 inputs, fp32 accumulate.  A sits in
// TMEM with lane = row and two consecutive K values per 32-bit column (low
// half first), so one K = 16 instruction reads 8 columns.
__device__ __forceinline__ void mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 8 int4 codes (two's complement, element i in bits 4i+3..4i) times the fp16
// scale pair s2 -> 8 fp16 values in element order (four fp16x2 words).  After
// flipping the top bit of every nibble, nibble n = q + 8.  For the byte b
// holding elements 2p and 2p+1, one byte permute puts b in both halves of a
// word and one mask-and-or makes the fp16 pair (1024 + n_lo, 1024 + 16 n_hi);
// one fp16 fma with (1, 1/16) and (-1032, -72) leaves (q_lo, q_hi) exactly
// (every step is exact: integers and power-of-two scalings well inside fp16's
// range), and the multiply by the scale rounds once, as q s is exact anyway.
__device__ __forceinline__ void int4x8_to_f16(uint32_t w, __half2 s2, uint32_t (&out)[4]) {
    const uint32_t u = w ^ 0x88888888u;
    const __half2 mul2 = __halves2half2(__ushort_as_half(0x3C00), __ushort_as_half(0x2C00));   // 1, 1/16
    const __half2 add2 = __halves2half2(__ushort_as_half(0xE408), __ushort_as_half(0xD480));   // -1032, -72
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        // bytes (b_p, 0, b_p, 0): selector nibbles p, 4 (a zero byte), p, 4
        const uint32_t x = __byte_perm(u, 0u, (uint32_t)(0x4040 | (p << 8) | p));
        const uint32_t bits = (x & 0x00F0000Fu) | 0x64006400u;
        __half2 v = *reinterpret_cast<const __half2*>(&bits);
        v = __hmul2(__hfma2(v, mul2, add2), s2);
        out[p] = *reinterpret_cast<const uint32_t*>(&v);
    }
}

__device__ __forceinline__ __half2 bf16_scale_to_h2(uint16_t sbits) {
    const __half sh = __float2half_rn(__bfloat162float(__ushort_as_bfloat16(sbits)));
    return __halves2half2(sh, sh);
}

// kInt4A: the activations are int4 codes with bf16 group scales (the int4
// W4A4 layer); otherwise bf16 (W4A16).  tm_a: x [M, K] bf16 (box 64 x 128,
// 128-byte swizzle) or the activation codes [M, K/2] (box 32 x 128);
// tm_as: activation scales [K/64, rows_pad] (box 128 x 1; int4 only);
// tm_L, tm_Lup: the rank-r operands (int4 W4A4 with rank > 0 only).
template <bool kInt4A>
__global__ void __launch_bounds__(dq::kThreads, 1)
    gemm_dq16_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_as,
                     const __grid_constant__ CUtensorMap tm_wc, const __grid_constant__ CUtensorMap tm_ws,
                     const __grid_constant__ CUtensorMap tm_L, const __grid_constant__ CUtensorMap tm_Lup,
                     Dq16Args a) {
    using namespace dq;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kStages * STAGE_BYTES);
    uint64_t* conv = full + kStages;
    uint64_t* empty = conv + kStages;
    uint64_t* acc_full = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    __shared__ int s_failed;
    __shared__ int s_issued[dq::kStages];

    const uint32_t warp = warp_id(), lane = lane_id();
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
    const int n_kc = a.K / 64;
    const int n_lr = (kInt4A && a.rank > 0) ? 2 * ((a.rank + 63) / 64) : 0;   // hi and lo per 64 of rank
    const int n_st = n_kc + n_lr;

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
        prefetch_tensormap(&tm_a);
        prefetch_tensormap(&tm_wc);
        prefetch_tensormap(&tm_ws);
        if (kInt4A) prefetch_tensormap(&tm_as);
        if (n_lr > 0) {
            prefetch_tensormap(&tm_L);
            prefetch_tensormap(&tm_Lup);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int it = 0; it < n_st; ++it) {
                const int s = it % kStages;
                const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, kSiteDqEmpty)) {
                    s_failed = 1;
                    break;
                }
                uint8_t* st = smem + (size_t)s * STAGE_BYTES;
                if (it < n_kc) {
                    const int kc = it;
                    if (kInt4A) {
                        mbar_arrive_expect_tx(&full[s], AP_BYTES + AS_BYTES + WP_BYTES + WS_BYTES);
                        tma_load_2d(st + OFF_AP, &tm_a, &full[s], kc * 32, m0);
                        tma_load_2d(st + OFF_AS, &tm_as, &full[s], m0, kc);
                    } else {
                        mbar_arrive_expect_tx(&full[s], XF_BYTES + WP_BYTES + WS_BYTES);
                        tma_load_2d(st, &tm_a, &full[s], kc * 64, m0);
                    }
                    tma_load_2d(st + OFF_WP, &tm_wc, &full[s], kc * 32, n0);
                    tma_load_2d(st + OFF_WS, &tm_ws, &full[s], n0, kc);
                } else {
                    // rank-r chunk: an L tile (hi or lo plane) and an L_up tile, already bf16
                    const int c = (it - n_kc) >> 1, part = (it - n_kc) & 1;
                    mbar_arrive_expect_tx(&full[s], XF_BYTES + LUP_BYTES);
                    tma_load_3d(st, &tm_L, &full[s], c * 64, m0, part);
                    tma_load_2d(st + OFF_LUP, &tm_Lup, &full[s], c * 64, n0);
                }
                reinterpret_cast<volatile int*>(s_issued)[s] += 1;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_f16_f32(128);     // M = 128 weight rows, N = 128 activation rows
            const uint32_t idesc_lr = idesc_bf16_f32(128);
            bool ok = true;
            for (int it = 0; it < n_st; ++it) {
                const int s = it % kStages;
                if (!mbar_wait(&conv[s], (uint32_t)(it / kStages) & 1u, kSiteDqConv)) {
                    ok = false;
                    s_failed = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t sx = smem_u32(smem + (size_t)s * STAGE_BYTES);
                if (it < n_kc) {
                    const uint32_t wt = tmem + WT_COL + 64u * (uint32_t)s;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t bd = desc_sw128(sx + 32u * j);
                        const uint32_t acc = (it > 0 || j > 0) ? 1u : 0u;
                        mma_f16_tmem_a(tmem + D_COL, wt + 8u * j, bd, idesc, acc);
                        mma_f16_tmem_a(tmem + D_COL + 128u, wt + 32u + 8u * j, bd, idesc, acc);
                    }
                } else {
                    const int c = (it - n_kc) >> 1;
                    const int nks = min(4, (a.rank - 64 * c + 15) / 16);
                    for (int j = 0; j < nks; ++j) {
                        const uint64_t bd = desc_sw128(sx + 32u * j);
                        mma_bf16(tmem + D_COL, desc_sw128(sx + OFF_LUP + 32u * j), bd, idesc_lr, 1u);
                        mma_bf16(tmem + D_COL + 128u, desc_sw128(sx + OFF_LUP + 16384u + 32u * j), bd, idesc_lr, 1u);
                    }
                }
                tc_commit(&empty[s]);
            }
            if (ok) tc_commit(acc_full);
        }
    } else if (warp >= (uint32_t)kConvWarp0) {
        // ----------------------------------- activations and weights -> fp16
        const int t = (int)threadIdx.x - 32 * kConvWarp0;        // 0..511
        const uint32_t q = warp & 3u;                            // this warp's TMEM lane quadrant
        const int j = (int)(warp - (uint32_t)kConvWarp0) >> 2;   // 0..3: weight half j / 2, K half j % 2
        const int wr = 128 * (j >> 1) + 32 * (int)q + (int)lane; // weight row of this thread
        const int kh = j & 1;
        for (int it = 0; it < n_st; ++it) {
            const int s = it % kStages;
            if (!mbar_wait(&full[s], (uint32_t)(it / kStages) & 1u, kSiteDqFull)) {
                s_failed = 1;
                break;
            }
            uint8_t* st = smem + (size_t)s * STAGE_BYTES;
            if (it < n_kc) {
                if (kInt4A) {
                    // activation row t / 4, values 16 (t % 4) .. + 15: codes -> fp16 (q s_x)
                    const int r = t >> 2, h = t & 3;
                    const __half2 s2 = bf16_scale_to_h2(*reinterpret_cast<const uint16_t*>(st + OFF_AS + 2 * r));
                    const uint2 c2 = *reinterpret_cast<const uint2*>(st + OFF_AP + 32 * r + 8 * h);
                    const uint32_t cw[2] = {c2.x, c2.y};
                    uint8_t* arow = st + r * 128;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {   // 16-byte chunk 2h + c: values 8 (2h + c) .. + 7
                        uint32_t o[4];
                        int4x8_to_f16(cw[c], s2, o);
                        *reinterpret_cast<uint4*>(arow + (((2 * h + c) ^ (r & 7)) << 4)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                } else {
                    // x: 16 KB of bf16 in place, 32 bytes per thread (position-preserving)
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        uint4* p = reinterpret_cast<uint4*>(st + 16 * (t + 512 * i));
                        const uint4 v = *p;
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __half2 hv = __floats2half2_rn(bf16lo_to_f32(w[e]), bf16hi_to_f32(w[e]));
                            o[e] = *reinterpret_cast<const uint32_t*>(&hv);
                        }
                        *p = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                // weight row wr, K values 32 kh .. + 31 -> fp16 (q s_w) in TMEM columns
                // 16 kh .. + 15 of its half's tile (lane = row)
                const __half2 s2 = bf16_scale_to_h2(*reinterpret_cast<const uint16_t*>(st + OFF_WS + 2 * wr));
                const uint4 c0 = *reinterpret_cast<const uint4*>(st + OFF_WP + 32 * wr + 16 * kh);
                const uint32_t cw[4] = {c0.x, c0.y, c0.z, c0.w};
                uint32_t o[16];
#pragma unroll
                for (int c = 0; c < 4; ++c) int4x8_to_f16(cw[c], s2, *reinterpret_cast<uint32_t(*)[4]>(o + 4 * c));
                tmem_st_32x32b_x16(tmem + ((32u * q) << 16) + WT_COL + 64u * (uint32_t)s + 32u * (uint32_t)(j >> 1) +
                                       16u * (uint32_t)kh,
                                   o);
                tmem_st_wait();
                fence_proxy_async_smem();   // the activation tile is read by the tensor core
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&conv[s]);
        }
    }
    if (warp >= (uint32_t)kEpiWarp0) {
        // ------------------------------------------------------------ epilogue
        // lane = weight row n, TMEM columns = activation rows; each 32 x 32
        // block goes out through this warp's 2 KB of the (now idle) ring as
        // 32 rows of 64 bytes
        const uint32_t q = warp & 3u;
        const int half = (int)(warp - kEpiWarp0) >> 2;
        const int nl = 128 * half + 32 * (int)q;               // first weight row of this warp
        const int n = n0 + nl + (int)lane;
        const bool ok = mbar_wait(acc_full, 0, kSiteDqAcc);
        if (!ok) s_failed = 1;
        tc_fence_after();
        if (ok) {
            float bv = 0.0f;
            if (a.bias != nullptr && n < a.N) bv = __bfloat162float(a.bias[n]);
            uint16_t* stg = reinterpret_cast<uint16_t*>(smem + (size_t)(warp - kEpiWarp0) * 2048);
#pragma unroll 1
            for (int c0 = 0; c0 < BM; c0 += 32) {
                uint32_t acc[32];
                tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + D_COL + 128u * (uint32_t)half + (uint32_t)c0, acc);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    stg[i * 32 + (int)lane] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(__fadd_rn(__uint_as_float(acc[i]), bv)));
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = (int)(lane >> 2) + 8 * k, ch = (int)(lane & 3u);
                    const int64_t m = (int64_t)m0 + c0 + i;
                    const int ncol = n0 + nl + 8 * ch;
                    if (m < a.M && ncol < a.N)
                        *reinterpret_cast<uint4*>(a.y + m * (int64_t)a.N + ncol) =
                            *reinterpret_cast<const uint4*>(stg + i * 32 + 8 * ch);
                }
                __syncwarp();
            }
        }
    }

    __syncthreads();
    if (s_failed && warp == 0 && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            const int n = reinterpret_cast<volatile int*>(s_issued)[s];
            if (n > 0) mbar_wait(&full[s], (uint32_t)(n - 1) & 1u, kSiteDqDrain);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace svdq
