// int4.cuh -- GEMM of the INT4 W4A4 variant of the SVDQ layer (sm_100a):
// the "INT4 W4A4 kernel with SVDQ low-rank correction", group 64 (Diffusers
// docs page "Nunchaku Lite", "Supported quantization types" table).
//
//   y[m, n] = bf16( sum_g s_x[m,g] s_w[n,g] (sum_{k in g} q_x[m,k] q_w[n,k])
//                   + sum_j L[m,j] L_up[j,n] + b[n] )
//
// The tensor cores have no 4-bit integer kind, so the packed codes are
// unpacked to int8 in shared memory and multiplied with tcgen05.mma kind::i8
// (int32 accumulate), one 64-column group per accumulator buffer.  Because
// every group carries its own pair of bf16 scales, the int32 group sums are
// scaled and added on the CUDA cores: this variant is bound by that rescale,
// not by the tensor cores.
//
// One CTA per 128 x 128 output tile.  Warp 0 loads packed int4 tiles (TMA,
// 128-byte swizzle) 256 columns of K at a time; warps 2..3 unpack them into
// int8 tiles in the MMA's swizzled layout; warp 1 issues the rank-r bf16 MMA
// (hi and lo parts of L) and two kind::i8 MMAs per group into a ring of four
// TMEM buffers; warps 4..11 fold each group into fp32 registers.
#pragma once
#include "sm100_ptx.cuh"

namespace svdq {
namespace i4 {
constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kGroupsPerStage = 4;              // 256 values of K
constexpr int PK_BYTES = 128 * 128;             // one packed operand tile: 128 rows x 128 B
constexpr int PSTAGE_BYTES = 2 * PK_BYTES;      // A and B packed (or an L tile and an L_up tile)
constexpr int kPStages = 2;
constexpr int UNP_BYTES = 2 * 128 * 128;        // one unpacked operand: two 128 x 128 B int8 tiles
constexpr int USTAGE_BYTES = 2 * UNP_BYTES;     // A and B unpacked
constexpr int kUStages = 2;
constexpr int kBufs = 4;                        // TMEM accumulator buffers, 128 columns each
constexpr int kEpiWarp0 = 4, kEpiWarps = 8;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int LR_BYTES = PSTAGE_BYTES;          // rank-r tiles (an L tile and an L_up tile): own buffer
constexpr size_t SMEM_BYTES =
    1024 + (size_t)kPStages * PSTAGE_BYTES + (size_t)kUStages * USTAGE_BYTES + LR_BYTES + 256;
}  // namespace i4

struct Int4GemmArgs {
    const uint16_t* x_scales;    // bf16 [K/64, rows_pad_m]
    const uint16_t* w_scales;    // bf16 [K/64, rows_pad_n]
    const __nv_bfloat16* bias;   // may be null
    __nv_bfloat16* y;
    int M, N, K, rank;
    int rows_pad_m, rows_pad_n;
};

enum : uint32_t { kSiteI4Empty = 32, kSiteI4Full = 33, kSiteI4UFull = 34, kSiteI4UEmpty = 35, kSiteI4Acc = 36,
                  kSiteI4AccEmpty = 37, kSiteI4Drain = 38 };

// 8 packed int4 (a 32-bit word, element i in bits 4i+3..4i) -> 8 int8 in two
// words, sign-extended, element order kept.
__device__ __forceinline__ void unpack_int4x8(uint32_t w, uint32_t& lo, uint32_t& hi) {
    // even elements (low nibbles) and odd elements (high nibbles), one per byte:
    // ((n ^ 8) + 0x78) ^ 0x80 sign-extends a nibble n within its byte, no carries
    const uint32_t ev = ((((w & 0x0F0F0F0Fu) ^ 0x08080808u) + 0x78787878u) ^ 0x80808080u);
    const uint32_t od = (((((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u) + 0x78787878u) ^ 0x80808080u);
    lo = __byte_perm(ev, od, 0x5140);   // e0 o0 e1 o1
    hi = __byte_perm(ev, od, 0x7362);   // e2 o2 e3 o3
}

__global__ void __launch_bounds__(i4::kThreads, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_wc,
                     const __grid_constant__ CUtensorMap tm_L, const __grid_constant__ CUtensorMap tm_Lup,
                     Int4GemmArgs a) {
    using namespace i4;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* pstage = smem;                                            // packed ring
    uint8_t* ustage = smem + (size_t)kPStages * PSTAGE_BYTES;          // unpacked ring
    uint8_t* lrbuf = ustage + (size_t)kUStages * USTAGE_BYTES;         // rank-r tiles
    uint64_t* full = reinterpret_cast<uint64_t*>(lrbuf + LR_BYTES);
    uint64_t* empty = full + kPStages;
    uint64_t* ufull = empty + kPStages;
    uint64_t* uempty = ufull + kUStages;
    uint64_t* pfull = uempty + kUStages;     // accumulator buffer ready (MMA -> epilogue)
    uint64_t* pempty = pfull + kBufs;        // accumulator buffer drained (epilogue -> MMA)
    uint64_t* lr_full = pempty + kBufs;
    uint64_t* lr_empty = lr_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lr_empty + 1);
    __shared__ int s_failed;
    __shared__ int s_issued[kPStages];

    const uint32_t warp = warp_id(), lane = lane_id();
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
    const int groups = a.K / 64;
    const int n_gs = (groups + kGroupsPerStage - 1) / kGroupsPerStage;   // group stages
    const int n_lr = a.rank > 0 ? 2 * ((a.rank + 63) / 64) : 0;          // rank-r stages (hi, lo per chunk)

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 2);      // the 2 unpacking warps
            s_issued[s] = 0;
        }
        for (int s = 0; s < kUStages; ++s) {
            mbar_init(&ufull[s], 2);
            mbar_init(&uempty[s], 1);
        }
        for (int b = 0; b < kBufs; ++b) {
            mbar_init(&pfull[b], 1);
            mbar_init(&pempty[b], kEpiWarps);
        }
        mbar_init(lr_full, 1);
        mbar_init(lr_empty, 1);
        s_failed = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_xc);
        prefetch_tensormap(&tm_wc);
        if (a.rank > 0) {
            prefetch_tensormap(&tm_L);
            prefetch_tensormap(&tm_Lup);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            bool ok = true;
            for (int it = 0; it < n_lr; ++it) {           // rank-r tiles: hi and lo part of each chunk
                if (!mbar_wait(lr_empty, ((uint32_t)it & 1u) ^ 1u, kSiteI4Empty)) {
                    s_failed = 1;
                    ok = false;
                    break;
                }
                const int c = it >> 1, part = it & 1;
                mbar_arrive_expect_tx(lr_full, LR_BYTES);
                tma_load_3d(lrbuf, &tm_L, lr_full, c * 64, m0, part);
                tma_load_2d(lrbuf + PK_BYTES, &tm_Lup, lr_full, c * 64, n0);
            }
            for (int gs = 0; gs < n_gs && ok; ++gs) {      // packed int4 codes, 4 groups at a time
                const int s = gs % kPStages;
                const uint32_t ph = (uint32_t)(gs / kPStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, kSiteI4Empty)) {
                    s_failed = 1;
                    break;
                }
                uint8_t* st = pstage + (size_t)s * PSTAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], PSTAGE_BYTES);
                tma_load_2d(st, &tm_xc, &full[s], gs * 128, m0);
                tma_load_2d(st + PK_BYTES, &tm_wc, &full[s], gs * 128, n0);
                reinterpret_cast<volatile int*>(s_issued)[s] += 1;
            }
        }
    } else if (warp == 2 || warp == 3) {
        // ---------------------------------------------- unpack int4 -> int8 tiles
        const int t = (int)threadIdx.x - 64;                 // 0..63
        for (int gs = 0; gs < n_gs; ++gs) {
            const int s = gs % kPStages;
            const uint32_t ph = (uint32_t)(gs / kPStages) & 1u;
            const int u = gs % kUStages;
            const uint32_t uph = (uint32_t)(gs / kUStages) & 1u;
            if (!mbar_wait(&full[s], ph, kSiteI4Full) || !mbar_wait(&uempty[u], uph ^ 1u, kSiteI4UEmpty)) {
                s_failed = 1;
                break;
            }
            const uint8_t* src = pstage + (size_t)s * PSTAGE_BYTES;
            uint8_t* dst = ustage + (size_t)u * USTAGE_BYTES;
            // units: (operand, row, packed 16-byte chunk c): 2 x 128 x 8
            for (int unit = t; unit < 2 * 128 * 8; unit += 64) {
                const int op = unit >> 10, row = (unit >> 3) & 127, c = unit & 7;
                const uint4 pk = *reinterpret_cast<const uint4*>(src + op * PK_BYTES + row * 128 + ((c ^ (row & 7)) << 4));
                uint32_t o[8];
                unpack_int4x8(pk.x, o[0], o[1]);
                unpack_int4x8(pk.y, o[2], o[3]);
                unpack_int4x8(pk.z, o[4], o[5]);
                unpack_int4x8(pk.w, o[6], o[7]);
                // packed chunk c holds K values 32c..32c+31: int8 tile c/4, chunks 2(c%4) and 2(c%4)+1
                uint8_t* tile = dst + op * UNP_BYTES + (c >> 2) * (128 * 128) + row * 128;
                const int c0 = 2 * (c & 3);
                *reinterpret_cast<uint4*>(tile + ((c0 ^ (row & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4*>(tile + (((c0 + 1) ^ (row & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
            }
            fence_proxy_async_smem();   // the int8 tiles are read by the tensor core
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&ufull[u]);
                mbar_arrive(&empty[s]);     // the packed stage has been read
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_i8 = idesc_s8_s32(BN);
            const uint32_t idesc_lr = idesc_bf16_f32(BN);
            bool ok = true;
            int use = 0;                                  // accumulator buffer uses so far
            auto acquire = [&](int u) -> bool {
                const int b = u % kBufs;
                if (!mbar_wait(&pempty[b], ((uint32_t)(u / kBufs) & 1u) ^ 1u, kSiteI4AccEmpty)) return false;
                tc_fence_after();
                return true;
            };
            if (n_lr > 0) {
                if (!acquire(use)) ok = false;
                for (int it = 0; it < n_lr && ok; ++it) {
                    if (!mbar_wait(lr_full, (uint32_t)it & 1u, kSiteI4Full)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(lrbuf), sb = sa + PK_BYTES;
                    const int c = it >> 1;
                    const int nks = min(4, (a.rank - 64 * c + 15) / 16);
                    for (int j = 0; j < nks; ++j)
                        mma_bf16(tmem + 128u * (uint32_t)(use % kBufs), desc_sw128(sa + 32u * j),
                                 desc_sw128(sb + 32u * j), idesc_lr, (it > 0 || j > 0) ? 1u : 0u);
                    tc_commit(lr_empty);
                }
                if (ok) tc_commit(&pfull[use % kBufs]);
                ++use;
            }
            for (int gs = 0; gs < n_gs && ok; ++gs) {
                const int u = gs % kUStages;
                if (!mbar_wait(&ufull[u], (uint32_t)(gs / kUStages) & 1u, kSiteI4UFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t ua = smem_u32(ustage + (size_t)u * USTAGE_BYTES), ub = ua + UNP_BYTES;
                const int ng = min(kGroupsPerStage, groups - gs * kGroupsPerStage);
                for (int g = 0; g < ng; ++g) {
                    if (!acquire(use)) {
                        ok = false;
                        break;
                    }
                    // group g: int8 tile g/2, bytes 64*(g%2) .. +63 of each row: two K=32 steps
                    const uint32_t off = (uint32_t)(g >> 1) * 128u * 128u + 64u * (uint32_t)(g & 1);
                    for (int j = 0; j < 2; ++j)
                        mma_s8(tmem + 128u * (uint32_t)(use % kBufs), desc_sw128(ua + off + 32u * j),
                               desc_sw128(ub + off + 32u * j), idesc_i8, j > 0 ? 1u : 0u);
                    tc_commit(&pfull[use % kBufs]);
                    ++use;
                }
                tc_commit(&uempty[u]);
            }
            if (!ok) s_failed = 1;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const uint32_t q = warp & 3u;
        const int half = (int)(warp - kEpiWarp0) >> 2;     // 64 of the 128 columns
        const int row = (int)(32u * q + lane);
        const int64_t grow = (int64_t)m0 + row;
        const int nb = n0 + 64 * half;
        float acc[64];
        // bias (and the rank-r result below) start the sums
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = 0.0f;
        if (a.bias) {
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i] = (nb + i < a.N) ? __bfloat162float(a.bias[nb + i]) : 0.0f;
        }
        int use = 0;
        bool ok = true;
        auto take = [&](int u) -> bool {
            if (!mbar_wait(&pfull[u % kBufs], (uint32_t)(u / kBufs) & 1u, kSiteI4Acc)) return false;
            tc_fence_after();
            return true;
        };
        auto give = [&](int u) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[u % kBufs]);
        };
        if (n_lr > 0) {
            ok = take(use);
            if (ok) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + 128u * (uint32_t)(use % kBufs) + 64u * half + 32u * h,
                                       r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[32 * h + i] += __uint_as_float(r[i]);
                }
            }
            give(use);
            ++use;
        }
        // The group scales are read from global memory once per group and used
        // at once, so the lines of group g + 2 are pulled into L1 while group g
        // is processed (shared memory is taken by the stage rings).  On the
        // 4608 x 3072 x 9216 shape this measured neutral: the epilogue is bound
        // by instruction issue (a scale, a convert and an FMA per element and
        // group), not by these loads.
        auto prefetch_scales = [&](int g) {
            if (lane == 0) {
                asm volatile("prefetch.global.L1 [%0];" ::"l"(a.w_scales + (int64_t)g * a.rows_pad_n + nb));
                asm volatile("prefetch.global.L1 [%0];" ::"l"(a.x_scales + (int64_t)g * a.rows_pad_m + m0 + 32 * q));
            }
        };
        prefetch_scales(0);
        if (groups > 1) prefetch_scales(1);
        for (int g = 0; g < groups && ok; ++g) {
            if (g + 2 < groups) prefetch_scales(g + 2);
            const float sx = (grow < a.M) ? __bfloat162float(__ushort_as_bfloat16(a.x_scales[(int64_t)g * a.rows_pad_m + grow]))
                                          : 0.0f;
            if (!take(use)) {
                ok = false;
                break;
            }
            const uint16_t* swp = a.w_scales + (int64_t)g * a.rows_pad_n + nb;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + 128u * (uint32_t)(use % kBufs) + 64u * half + 32u * h, r);
                // weight scales of these 32 columns (same for every lane: broadcast loads)
                float sw[32];
                const uint4* sp = reinterpret_cast<const uint4*>(swp + 32 * h);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 w = __ldg(sp + v);
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        sw[8 * v + 2 * p] = bf16lo_to_f32(ws[p]);
                        sw[8 * v + 2 * p + 1] = bf16hi_to_f32(ws[p]);
                    }
                }
                tmem_ld_wait();
                // acc += float(P) * (sx * sw), two columns per instruction.  A
                // group's partial sum P is at most 64 * 8 * 8 = 4096 in magnitude,
                // so it converts exactly without the (low-throughput) I2F unit.
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float p0, p1, s0, s1;
                    fadd2_rn(i2f_biased(r[i]), i2f_biased(r[i + 1]), -kMagicI2F, -kMagicI2F, p0, p1);
                    fmul2_rn(sx, sx, sw[i], sw[i + 1], s0, s1);
                    ffma2_rn(p0, p1, s0, s1, acc[32 * h + i], acc[32 * h + i + 1], acc[32 * h + i],
                             acc[32 * h + i + 1]);
                }
            }
            give(use);
            ++use;
        }
        if (ok && grow < a.M) {
            __nv_bfloat16* yrow = a.y + grow * (int64_t)a.N;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int n = nb + 16 * c;
                if (n >= a.N) break;
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[16 * c + 2 * i], acc[16 * c + 2 * i + 1]);
                    packed[i] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                uint4* dst = reinterpret_cast<uint4*>(yrow + n);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
        }
        if (!ok) s_failed = 1;
    }

    __syncthreads();
    if (s_failed && warp == 0 && lane == 0) {
        for (int s = 0; s < kPStages; ++s) {
            const int n = reinterpret_cast<volatile int*>(s_issued)[s];
            if (n > 0) mbar_wait(&full[s], (uint32_t)(n - 1) & 1u, kSiteI4Drain);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace svdq
