// gemm_nvfp4_pair128.cuh -- the block-scaled FP4 GEMM of the SVDQ W4A4 layer on
// CTA pairs with 256 x 128 output tiles, for M > 128, K <= 3072, K % 512 == 0.
// An alternative to gemm_nvfp4_pair_kernel, selected only on request: measured
// on B200 it is the slower of the two (its N = 128 MMAs with one scale copy
// each issue at about 205 cycles apiece, so the smaller tile loses more than
// the saved copies gain).
//
// Computes exactly what gemm_nvfp4_kernel computes (FP4 x FP4 main loop, the hi
// and lo bf16 parts of the rank-r branch into the same fp32 accumulator,
// y = bf16(S_x S_w acc + b)).  What this layout buys, against 256 x 256 tiles:
//   * the weight scale factors of a 128-column tile for the whole K fit in
//     TMEM (4 columns per 64 values of K, 192 columns at K = 3072) next to two
//     accumulators of 128 columns.  Tiles are taken m-fastest within a column
//     of tiles, so the weight scales are copied into TMEM once per run of
//     tiles, and each MMA needs a single scale-block copy (its activation
//     scales).  Copies are what limits the tensor pipe here: an MMA with one
//     copy queued behind it runs at full rate, two or three copies per MMA
//     cost 30-60 % more;
//   * the two accumulators let the epilogue of one tile overlap the MMAs of
//     the next;
//   * a stage carries 8 K-steps (256 bytes of codes per row), so the per-stage
//     barrier traffic of the MMA thread is spread over 8 MMAs.
// The price is more activation-code traffic (each 256-row block of codes is
// read once per 128 output columns instead of per 256).
//
// Cluster of two CTAs: CTA r loads activation rows 128 r .. 128 r + 127 of
// the tile and weight rows 64 r .. 64 r + 63 (the M = 256, N = 128 MMA reads
// N/2 weight rows from each CTA), the activation scales of its own rows and
// the weight scales of all 128 columns.  CTA 0 issues the copies and MMAs;
// every load of either CTA completes on CTA 0's stage barrier.
#pragma once
#include "gemm_nvfp4.cuh"

namespace svdq {
namespace gq {
constexpr int BM = 256;
constexpr int BN = 128;
constexpr int KSTEPS = 8;                       // K-steps of 64 values per stage
constexpr int CHUNK = 128;                      // bytes of a row in one 128-byte-swizzled tile
constexpr int kStages = 4;
constexpr int A_BYTES = 2 * 128 * CHUNK;        // 32 KB: 128 rows x 256 bytes, as two swizzled tiles
constexpr int A_CHUNK = 128 * CHUNK;            // 16 KB
constexpr int B_BYTES = 2 * 64 * CHUNK;         // 16 KB: 64 rows x 256 bytes
constexpr int B_CHUNK = 64 * CHUNK;             // 8 KB
constexpr int SFA_BYTES = KSTEPS * 512;         // this CTA's 128 activation rows, 8 K-steps
constexpr int SFB_BYTES = KSTEPS * 512;         // all 128 weight rows, 8 K-steps
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int kEpiWarps = 8;                    // 2 per TMEM lane quadrant, 64 columns each
constexpr int kEpiWarp0 = 4;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr uint32_t kMmaWarp = 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COLS = 128;              // accumulator b at columns 128 b
constexpr int kMaxKSteps = 48;                  // K <= 3072
constexpr uint32_t SFB_RES = 256;               // weight scales of K-step g at SFB_RES + 4 g
constexpr uint32_t SFA_SET = SFB_RES + 4 * kMaxKSteps;   // 448: activation scales, sets of 32 columns
static_assert(SFA_SET + 2 * 4 * KSTEPS <= TMEM_COLS, "scale-factor columns do not fit in TMEM");
constexpr uint32_t kFullArrivals = 3;
constexpr int kLanesPerRole = 2;
constexpr uint32_t kAccEmptyArrivals = 2 * kEpiWarps;
constexpr size_t SMEM_BYTES = 1024 + (size_t)kStages * STAGE_BYTES + 256;
static_assert(SMEM_BYTES <= 227 * 1024, "stage ring does not fit in shared memory");
}  // namespace gq

enum : uint32_t {
    kSiteGqEmpty = 40,
    kSiteGqFull = 41,
    kSiteGqAcc = 42,
    kSiteGqDrain = 43,
    kSiteGqAccEmpty = 44
};

// tm_xc / tm_wc: codes [rows][K/2 bytes], 128-byte swizzle, boxes of 128 bytes
// x 128 (activations) or 64 (weights) rows.  tm_sfa / tm_sfb: scale
// blocks [row blocks][K/64][128 words], boxes of 8 K-steps of one row block.
// tm_L: rank-r activations [2][M][rank] bf16, box 64 x 128 x 1; tm_Lup: L_up
// transposed [N][rank] bf16, box 64 x 64.
__global__ void __launch_bounds__(gq::kThreads, 1)
    gemm_nvfp4_pair128_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_wc,
                              const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                              const __grid_constant__ CUtensorMap tm_L, const __grid_constant__ CUtensorMap tm_Lup,
                              GemmArgs a) {
    using namespace gq;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kStages * STAGE_BYTES);
    uint64_t* empty = full + kStages;
    uint64_t* acc_full = empty + kStages;     // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    __shared__ int s_failed;
    __shared__ int s_issued[gq::kStages];

    const uint32_t warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_ctarank();
    const int cluster = (int)(blockIdx.x >> 1), n_clusters = (int)(gridDim.x >> 1);
    const int n_kb = a.K / (64 * KSTEPS);                // whole stages (K % 512 == 0)
    const int n_lr = a.rank > 0 ? 2 * ((a.rank + 63) / 64) : 0;
    const int per_tile = n_kb + n_lr;
    const int total_tiles = a.m_tiles * a.n_tiles;       // m_tiles counts 256-row tiles
    // contiguous run of tiles per cluster, m fastest: the weight columns (and
    // their resident scales) change only when the run crosses a tile column
    const int t_begin = (int)(((int64_t)total_tiles * cluster) / n_clusters);
    const int t_end = (int)(((int64_t)total_tiles * (cluster + 1)) / n_clusters);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], kFullArrivals);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kAccEmptyArrivals);
        }
        for (int s = 0; s < kStages; ++s) s_issued[s] = 0;
        s_failed = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_xc);
        prefetch_tensormap(&tm_wc);
        prefetch_tensormap(&tm_sfa);
        prefetch_tensormap(&tm_sfb);
        if (a.rank > 0) {
            prefetch_tensormap(&tm_L);
            prefetch_tensormap(&tm_Lup);
        }
    }
    if (warp == kMmaWarp) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 1) {
        // ----------------------------------------------------------- producers
        // warp 0 lanes 0-1: activation codes; warp 1 lanes 0-1: weight codes,
        // lanes 2-3: scale blocks.  Each role's two lanes take alternate stages.
        if (lane < (uint32_t)(warp == 0 ? kLanesPerRole : 2 * kLanesPerRole)) {
            const int role = warp == 0 ? 0 : (lane < (uint32_t)kLanesPerRole ? 1 : 2);
            const uint32_t rlane = lane % (uint32_t)kLanesPerRole;
            const bool leader = rank == 0;
            int it = 0;
            bool ok = true;
            for (int tile = t_begin; tile < t_end && ok; ++tile) {
                const int n_tile = tile / a.m_tiles, m_tile = tile - n_tile * a.m_tiles;
                const bool need_sfb = tile == t_begin || m_tile == 0;
                const int m0 = m_tile * BM + 128 * (int)rank;
                const int n0 = n_tile * BN + 64 * (int)rank;
                for (int kk = 0; kk < per_tile; ++kk, ++it) {
                    if ((it % kLanesPerRole) != (int)rlane) continue;
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, kSiteGqEmpty)) {
                        s_failed = 1;
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + (size_t)s * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    uint8_t* sfa = sb + B_BYTES;
                    uint8_t* sfb = sfa + SFA_BYTES;
                    const uint32_t bar = cluster_addr(&full[s], 0);
                    if (kk < n_kb) {
                        // two 128-byte-wide swizzled tiles per operand (K-steps 0-3, 4-7)
                        if (role == 0) {
                            if (leader) mbar_arrive_expect_tx(&full[s], 2u * A_BYTES);
                            tma_load_2d_pair(sa, &tm_xc, bar, 2 * CHUNK * kk, m0);
                            tma_load_2d_pair(sa + A_CHUNK, &tm_xc, bar, 2 * CHUNK * kk + CHUNK, m0);
                            atomicAdd(&s_issued[s], 1);
                        } else if (role == 1) {
                            if (leader) mbar_arrive_expect_tx(&full[s], 2u * B_BYTES);
                            tma_load_2d_pair(sb, &tm_wc, bar, 2 * CHUNK * kk, n0);
                            tma_load_2d_pair(sb + B_CHUNK, &tm_wc, bar, 2 * CHUNK * kk + CHUNK, n0);
                        } else {
                            if (leader)
                                mbar_arrive_expect_tx(&full[s], 2u * (SFA_BYTES + (need_sfb ? SFB_BYTES : 0)));
                            tma_load_3d_pair(sfa, &tm_sfa, bar, 0, KSTEPS * kk, 2 * m_tile + (int)rank);
                            if (need_sfb) tma_load_3d_pair(sfb, &tm_sfb, bar, 0, KSTEPS * kk, n_tile);
                        }
                    } else {
                        const int c = (kk - n_kb) >> 1, part = (kk - n_kb) & 1;
                        if (role == 0) {
                            if (leader) mbar_arrive_expect_tx(&full[s], 2u * A_CHUNK);
                            tma_load_3d_pair(sa, &tm_L, bar, c * 64, m0, part);
                            atomicAdd(&s_issued[s], 1);
                        } else if (role == 1) {
                            if (leader) mbar_arrive_expect_tx(&full[s], 2u * B_CHUNK);
                            tma_load_2d_pair(sb, &tm_Lup, bar, c * 64, n0);
                        } else {
                            if (leader) mbar_arrive(&full[s]);
                        }
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------ copies + MMAs (CTA 0 only)
        // One thread issues both: the single activation-scale copy of K-step
        // j + 1 goes in right before the MMA of step j, where it overlaps.
        if (rank == 0 && lane == 0) {
            const uint32_t idesc_fp4 = idesc_m(idesc_nvfp4(BN), BM);
            const uint32_t idesc_lr = idesc_m(idesc_bf16_f32(BN), BM);
            const uint32_t smem0 = smem_u32(smem);
            bool ok = true;
            int local = 0, s = 0, it = 0;
            uint32_t ph = 0;
            for (int tile = t_begin; tile < t_end && ok; ++tile, ++local) {
                const int m_tile = tile % a.m_tiles;
                const bool need_sfb = tile == t_begin || m_tile == 0;
                const int buf = local & 1;
                const uint32_t acc = tmem + ACC_COLS * (uint32_t)buf;
                // the epilogue must have drained this accumulator (two tiles ago)
                if (!mbar_wait(&acc_empty[buf], ((uint32_t)(local >> 1) & 1u) ^ 1u, kSiteGqAccEmpty)) {
                    s_failed = 1;
                    break;
                }
                tc_fence_after();
                for (int kk = 0; kk < per_tile; ++kk, ++it) {
                    if (!mbar_wait(&full[s], ph, kSiteGqFull)) {
                        ok = false;
                        s_failed = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem0 + (uint32_t)s * STAGE_BYTES;
                    const uint32_t sb = sa + A_BYTES;
                    const uint64_t da = desc_sw128(sa), db = desc_sw128(sb);
                    if (kk < n_kb) {
                        const uint64_t dfa = desc_sf_block(sb + B_BYTES);               // + 32 per 512 bytes
                        const uint64_t dfb = desc_sf_block(sb + B_BYTES + SFA_BYTES);
                        const uint32_t ta = tmem + SFA_SET + 32u * (uint32_t)(it & 1);
                        const uint32_t tb = tmem + SFB_RES + 4u * (uint32_t)(KSTEPS * kk);
                        auto copies = [&](int j) {
                            tmem_cp_32x128b_x4_pair(ta + 4u * j, dfa + 32u * j);
                            if (need_sfb) tmem_cp_32x128b_x4_pair(tb + 4u * j, dfb + 32u * j);
                        };
                        copies(0);
#pragma unroll
                        for (int j = 0; j < KSTEPS; ++j) {
                            if (j + 1 < KSTEPS) copies(j + 1);
                            // K-step j: tile j / 4 of the stage, 32 bytes per step inside it
                            const uint32_t ao = (uint32_t)(j >> 2) * (A_CHUNK >> 4) + 2u * (uint32_t)(j & 3);
                            const uint32_t bo = (uint32_t)(j >> 2) * (B_CHUNK >> 4) + 2u * (uint32_t)(j & 3);
                            mma_nvfp4_pair(acc, da + ao, db + bo, idesc_fp4, ta + 4u * j, tb + 4u * j,
                                           (kk > 0 || j > 0) ? 1u : 0u);
                        }
                    } else {
                        const int c = (kk - n_kb) >> 1;
                        const int nks = min(4, (a.rank - 64 * c + 15) / 16);
                        for (int j = 0; j < nks; ++j)
                            mma_bf16_pair(acc, da + 2u * j, db + 2u * j, idesc_lr, 1u);
                    }
                    tc_commit_pair(&empty[s], 0x3);
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok) tc_commit_pair(&acc_full[buf], 0x3);
            }
        }
    } else if (warp >= (uint32_t)kEpiWarp0) {
        // ------------------------------------------------------------ epilogue
        const uint32_t q = warp & 3u;
        const int half = (int)(warp - kEpiWarp0) >> 2;     // which 64 of the 128 columns
        const int row = (int)(32u * q + lane);
        const float S = __fmul_rn(*a.x_scale, *a.w_scale);
        const uint32_t acc_empty_leader0 = cluster_addr(&acc_empty[0], 0);
        const uint32_t acc_empty_leader1 = cluster_addr(&acc_empty[1], 0);
        int local = 0;
        for (int tile = t_begin; tile < t_end; ++tile, ++local) {
            const int n_tile = tile / a.m_tiles, m_tile = tile - n_tile * a.m_tiles;
            const int buf = local & 1;
            const int64_t grow = (int64_t)m_tile * BM + 128 * (int64_t)rank + row;
            const int nbase = n_tile * BN + 64 * half;
            if (!mbar_wait(&acc_full[buf], (uint32_t)(local >> 1) & 1u, kSiteGqAcc)) {
                s_failed = 1;
                break;
            }
            tc_fence_after();
            uint32_t acc[64];
            const uint32_t taddr = tmem + ((32u * q) << 16) + ACC_COLS * (uint32_t)buf + 64u * (uint32_t)half;
            tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(acc + 0));
            tmem_ld_32x32b_x32(taddr + 32u, *reinterpret_cast<uint32_t(*)[32]>(acc + 32));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf ? acc_empty_leader1 : acc_empty_leader0);
            if (grow >= a.M) continue;
            __nv_bfloat16* yrow = a.y + grow * (int64_t)a.N;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int n = nbase + 16 * c;
                if (n >= a.N) break;
                float bv[16];
                if (a.bias) {
                    const uint4 w0 = __ldg(reinterpret_cast<const uint4*>(a.bias + n));
                    const uint4 w1 = __ldg(reinterpret_cast<const uint4*>(a.bias + n) + 1);
                    const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        bv[2 * p] = bf16lo_to_f32(ws[p]);
                        bv[2 * p + 1] = bf16hi_to_f32(ws[p]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) bv[i] = 0.0f;
                }
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float o0 = fmaf(__uint_as_float(acc[16 * c + 2 * i]), S, bv[2 * i]);
                    const float o1 = fmaf(__uint_as_float(acc[16 * c + 2 * i + 1]), S, bv[2 * i + 1]);
                    const __nv_bfloat162 h = __floats2bfloat162_rn(o0, o1);
                    packed[i] = *reinterpret_cast<const uint32_t*>(&h);
                }
                uint4* dst = reinterpret_cast<uint4*>(yrow + n);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
        }
    }

    __syncthreads();
    if (s_failed && rank == 0 && warp == 0 && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            const int n = reinterpret_cast<volatile int*>(s_issued)[s];
            if (n > 0) mbar_wait(&full[s], (uint32_t)(n - 1) & 1u, kSiteGqDrain);
        }
    }
    tc_fence_before();
    cluster_sync_all();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

}  // namespace svdq
