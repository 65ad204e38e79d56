// gemm_nvfp4_pair.cuh -- the block-scaled FP4 GEMM of the SVDQ W4A4 layer on
// CTA pairs (tcgen05 cta_group::2), for M > 128.
//
// Computes exactly what gemm_nvfp4_kernel computes (see gemm_nvfp4.cuh: FP4 x FP4
// main loop, the hi and lo bf16 parts of the rank-r branch into the same fp32
// accumulator, y = bf16(S_x S_w acc + b)), on 256 x 256 output tiles.  Each
// tile belongs to a cluster of two CTAs on neighbouring SMs:
//   * CTA r (r = 0, 1) loads rows 128 r .. 128 r + 127 of the tile's activation
//     codes and rows 128 r .. 128 r + 127 of its weight codes, the scale block
//     of its own 128 activation rows and the GEMM-ready copy of the weight
//     scales of all 256 columns (the tensor core reads the weight scales of
//     every column in both halves of the pair; the copy holds them replicated
//     for the four TMEM lane quarters, so one tcgen05.cp 128x256b per 64
//     values of K moves them);
//   * two warps of CTA 0 take the stages in turn; in each, one thread copies
//     the scales into both CTAs' TMEM and issues one M = 256, N = 256 MMA per
//     64 values of K, each copy right before the MMA ahead of the one that
//     reads it; the accumulator rows of CTA r sit in CTA r's TMEM;
//   * every load of either CTA completes on CTA 0's stage barrier, CTA 0's
//     commits arrive on both CTAs' "stage free" and "accumulator full"
//     barriers, and both CTAs' epilogue warps hand the accumulator back on
//     CTA 0's barrier.
// Against 128 x 256 tiles on single CTAs this halves the weight-code bytes
// each SM loads per FLOP and the number of scale copies per FLOP; with the
// activation scales resident in TMEM (K <= 3072, below) one copy per MMA
// remains.

// All scale blocks arrive by TMA (maps over the 512-byte blocks) so that the
// peer CTA's loads can complete on CTA 0's barrier; a box that runs past the
// end of a scale buffer is zero-filled, which only ever feeds rows or K-steps
// whose results are discarded.  Only CTA 0's producers arrive on a stage
// barrier, announcing the bytes of both CTAs (every box is counted in full,
// zero-filled parts included); the peer's loads cannot land early because the
// peer refills a stage only after CTA 0's MMAs have released it.
//
// One thread issuing TMA copies manages roughly one stage every 600-700
// cycles, whatever the box size, and a stage of four K-steps lasts 512 cycles
// of MMA; so each producer role runs on two lanes that take alternate stages.
//
// With the fused QKV epilogue (kEpiQkv, GemmArgs.qk_cols > 0) the warps whose
// 128 columns are a Q or K head apply that head's RMSNorm and rotary embedding
// (qkv_norm_rope.cuh) to the fp32 results before the bf16 store.  With the
// fused GELU epilogue (kEpiGelu) nothing is stored for y: each row's
// h = bf16(GELU(bf16(y))) is quantized for the next layer and its rank-r
// down-projection partial sums are added into a global fp32 buffer
// (gp_gelu_epilogue below, gelu_mlp.cuh).
//
// Measured alternative, not kept: four extra warps writing the scale factors
// into TMEM with tcgen05.st (so that the MMA thread issues MMAs only) ran the
// 4608 x 3072 x 9216 projection in 160-190 us against 107 us for this kernel;
// their shared-memory reads of the staged scale blocks slowed the TMA fill of
// the ring, whose stages then landed 3-5 us after issue.
#pragma once
#include "gelu_mlp.cuh"
#include "gemm_nvfp4.cuh"
#include "qkv_norm_rope.cuh"

namespace svdq {
namespace gp {
constexpr int BM = 256;                        // tile rows (128 per CTA)
constexpr int BN = 256;                        // tile columns (128 weight rows loaded per CTA)
constexpr int BK_BYTES = 128;
constexpr int kStages = 4;
constexpr int A_BYTES = 128 * BK_BYTES;        // 16 KB: this CTA's 128 activation rows
constexpr int B_BYTES = 128 * BK_BYTES;        // 16 KB: this CTA's 128 weight rows
constexpr int SFA_BYTES = 4 * 512;             // scale blocks of this CTA's 128 rows, 4 k-steps
// The weight scales of a stage as the GEMM-ready copy holds them: per k-step
// the two 512-byte scale blocks of the tile's 256 weight rows, replicated for
// the four TMEM lane quadrants (128 rows x 32 bytes, row 32 q + l holding row
// l of both blocks, K-major without swizzle: 8-row groups 256 bytes apart,
// the two 16-byte halves 128 bytes apart), so that one tcgen05.cp 128x256b
// per k-step moves them into TMEM.  The copy instructions, not their bytes,
// are what occupy the tensor pipe: the alternative, two 32x128b.warpx4
// copies per k-step from the 1 KB of plain blocks, costs twice as many.
constexpr int SFB_KSTEP_BYTES = 4096;
constexpr int SFB_BYTES = 4 * SFB_KSTEP_BYTES;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int kEpiWarps = 8;
constexpr int kEpiWarp0 = 4;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr uint32_t kMmaWarp = 2;               // MMA issuers: warps 2 and 3 (even and odd stages)
constexpr uint32_t kMmaWarp2 = 3;
constexpr uint32_t kBarTurn0 = 2;              // named barriers 2, 3: the turn of warp 2, 3 (0: __syncthreads, 1: GELU epilogue)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;
// Scale factors in TMEM.  Stages alternate between two "scale sets" (one per
// MMA-issuing warp); one of two layouts:
//  * streamed (any K): set b at SF_COL + 48 b: 4 k-steps x 4 columns of
//    activation scales, then 4 k-steps x 8 columns of weight scales;
//  * resident activation scales (K <= 64 * kResidentKSteps): the activation
//    scales of the whole K for the current 256-row tile stay at SFA_RES +
//    4 k, copied once per run of tiles that share those rows, and set b holds
//    only weight scales, at SFB_RES + 32 b.  This takes the activation-scale
//    copies off the tensor pipe.
constexpr uint32_t SF_COL = 256;
constexpr uint32_t SF_SET_COLS = 48;
static_assert(SF_COL + 2 * SF_SET_COLS <= TMEM_COLS, "scale-factor columns do not fit in TMEM");
constexpr int kResidentKSteps = 48;
constexpr uint32_t SFA_RES = 256;
constexpr uint32_t SFB_RES = SFA_RES + 4 * kResidentKSteps;   // 448: two sets of 32 columns
static_assert(SFB_RES + 64 <= TMEM_COLS, "resident scale-factor columns do not fit in TMEM");
// The fused QKV epilogue streams the activation scales (so the resident
// layout is never used there) and keeps the rotary tables of the CTA's 128
// rows in the columns the two streamed sets leave free: lane = row, 64
// columns of cos, then 64 of sin (fp32).
constexpr uint32_t QKV_TAB_COL = SF_COL + 2 * SF_SET_COLS;   // 352
static_assert(QKV_TAB_COL + 128 <= TMEM_COLS, "rotary tables do not fit in TMEM");
constexpr uint32_t kFullArrivals = 3;          // CTA 0's three producer roles, for both CTAs' bytes
constexpr int kLanesPerRole = 2;               // producer lanes per role, taking alternate stages
constexpr size_t SMEM_BYTES = 1024 + (size_t)kStages * STAGE_BYTES + 256;
// the mbarriers (full and empty per stage; acc_full, acc_empty; tab_free and
// tab_ready per lane quarter) and the TMEM address
static_assert((2 * kStages + 2 + 8) * 8 + 4 <= 256, "barriers do not fit their 256 bytes");
static_assert(SMEM_BYTES <= 227 * 1024, "stage ring does not fit in shared memory");
// kEpiPlain, kEpiQkv: y leaves through TMA stores of 32 x 32 boxes staged
// per epilogue warp in kYBufs 2 KB buffers (64-byte swizzle), 1 KB aligned
// after the barriers.
constexpr int kYStageBytes = 2048;
constexpr int kYBufs = 1;
constexpr size_t Y_STAGE_OFF = (size_t)kStages * STAGE_BYTES + 1024;
constexpr size_t SMEM_BYTES_PLAIN = 1024 + Y_STAGE_OFF + (size_t)kEpiWarps * kYBufs * kYStageBytes;
static_assert(SMEM_BYTES_PLAIN <= 227 * 1024, "y staging buffers do not fit in shared memory");
// kEpiGelu: twice the epilogue warps (four per TMEM lane quadrant, 64
// columns each: the GELU epilogue is latency-bound, and more warps hide more
// of it), a 1 KB transpose buffer per warp (32 rows x 16 bf16), the GELU
// table and the 128 reciprocals of the next layer's decoded group scales.
constexpr int kEpiWarpsGelu = 16;
constexpr int kThreadsGelu = 32 * (kEpiWarp0 + kEpiWarpsGelu);
constexpr int kGeluScratch = 1024;
constexpr size_t SMEM_BYTES_GELU = SMEM_BYTES + (size_t)kEpiWarpsGelu * kGeluScratch + kGeluTabBytes + 128 * 4;
static_assert(SMEM_BYTES_GELU <= 227 * 1024, "GELU epilogue buffers do not fit in shared memory");
}  // namespace gp

// Epilogue variants of the pair kernel (separate instantiations, so that the
// plain kernel keeps its registers).
// kEpiGeluStore: the GELU epilogue's store-only form (h = bf16(GELU(y)) to y).
enum : int { kEpiPlain = 0, kEpiQkv = 1, kEpiGelu = 2, kEpiGeluStore = 3 };
__host__ __device__ constexpr bool gp_is_gelu(int e) { return e == kEpiGelu || e == kEpiGeluStore; }

// Bytes of the GEMM-ready copy of the weight scales of an N x K weight:
// 16 KB per (256-row tile, 256 columns of K), whole tiles.
__host__ __device__ constexpr int64_t wscales_rep_bytes(int64_t N, int64_t K) {
    return ((N + 255) / 256) * ((K + 255) / 256) * (int64_t)gp::SFB_BYTES;
}

// Writes the GEMM-ready copy (rep) of the weight scales from their block
// layout (blocks: 512 bytes per 128 rows x 64 columns, row l of a block at
// 16 l; kg4 = K / 64 blocks per row block, n_rb row blocks).  Unit (t, kb) =
// 256-row tile t, k-steps 4 kb .. 4 kb + 3, at (t * n_kb + kb) * 16 KB; in
// it k-step k at k * 4 KB holds, for each TMEM lane quadrant q and row l,
// row l of blocks (2 t, 4 kb + k) and (2 t + 1, 4 kb + k) at
// (4 q + l / 8) * 256 + (l % 8) * 16 and 128 bytes further.  Blocks past the
// weight (a missing second row block, k-steps past K) are zeros.  One
// thread per 16 bytes of the copy.
__global__ void __launch_bounds__(256) replicate_weight_scales_kernel(const uint8_t* __restrict__ blocks,
                                                                      uint8_t* __restrict__ rep, int n_rb, int kg4,
                                                                      int n_kb, int64_t chunks) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= chunks) return;
    const int64_t unit = i >> 10;
    const int c = (int)(i & 1023);
    const int k = c >> 8, g = (c & 255) >> 4, h = (c >> 3) & 1, l8 = c & 7;
    const int l = 8 * (g & 3) + l8;
    const int t = (int)(unit / n_kb), kb = (int)(unit - (int64_t)t * n_kb);
    const int rb = 2 * t + h, kk = 4 * kb + k;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (rb < n_rb && kk < kg4) v = *reinterpret_cast<const uint4*>(blocks + ((int64_t)rb * kg4 + kk) * 512 + 16 * l);
    reinterpret_cast<uint4*>(rep)[i] = v;
}

// Descriptor of one k-step of replicated weight scales (K-major, no swizzle:
// 8-row groups 256 bytes apart, the two 16-byte halves 128 bytes apart).
__device__ __forceinline__ uint64_t desc_sfb_kstep(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(256u >> 4) << 32) |
           ((uint64_t)1u << 46);
}
// The GELU epilogue runs four warps per TMEM lane quadrant (64 columns
// each): its chain is latency-bound, and more warps hide more of it.  The
// plain and QKV epilogues keep two (128 columns per warp; a QKV head's
// RMSNorm needs all of its 128 columns in one thread); four measured no
// faster for the plain one.
template <int kEpi>
__host__ __device__ constexpr int gp_epi_warps() {
    return gp_is_gelu(kEpi) ? gp::kEpiWarpsGelu : gp::kEpiWarps;
}
template <int kEpi>
__host__ __device__ constexpr int gp_threads() {
    return 32 * (gp::kEpiWarp0 + gp_epi_warps<kEpi>());
}

enum : uint32_t {
    kSiteGpEmpty = 24,
    kSiteGpFull = 25,
    kSiteGpAcc = 26,
    kSiteGpDrain = 27,
    kSiteGpAccEmpty = 28,
    kSiteGpTab = 29
};

// One stage of four K-steps, issued by an MMA thread: the scale copies of
// K-step j + 1 go in right before the MMA of step j (one 128x256b copy of
// the replicated weight scales; WITH_SFA: also a 32x128b.warpx4 copy of the
// activation scales).  The tensor pipe keeps only a few instructions queued,
// so this sequence has nothing between its tcgen05 instructions but address
// arithmetic on registers.
template <bool WITH_SFA>
__device__ __forceinline__ void gp_issue_stage(uint32_t acc, uint64_t da, uint64_t db, uint64_t dfa, uint64_t dfb,
                                               uint32_t ta, uint32_t tb, uint32_t idesc, uint32_t acc0) {
    constexpr uint64_t kSfbStep = (uint64_t)(gp::SFB_KSTEP_BYTES >> 4);   // descriptor units per k-step
    if (WITH_SFA) tmem_cp_32x128b_x4_pair(ta, dfa);
    tmem_cp_128x256b_pair(tb, dfb);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j < 3) {
            if (WITH_SFA) tmem_cp_32x128b_x4_pair(ta + 4u * (j + 1), dfa + 32u * (j + 1));
            tmem_cp_128x256b_pair(tb + 8u * (j + 1), dfb + kSfbStep * (j + 1));
        }
        mma_nvfp4_pair(acc, da + 2u * j, db + 2u * j, idesc, ta + 4u * j, tb + 8u * j, j == 0 ? acc0 : 1u);
    }
}

// The fused GELU epilogue of one thread's row (grow) over one warp's NC
// columns [nbase, nbase + NC) of a tile; acc holds the fp32 accumulators.
//  1. y = S acc + b rounded to bf16 (what the plain epilogue stores), then
//     h = bf16(GELU(y)) by gelu_bf16_bits (the per-CTA table): the next
//     layer's input, never written out;
//  2. the next layer's nvfp4 step on h, with the arithmetic of the activation
//     quantizer (quantize_act.cuh): v = h * (1 / lambda), per 16 columns the
//     E4M3 scale e of amax(v) / (6 S2) and the E2M1 codes of v * inv_tab[e],
//     inv_tab[e] = 1 / (e S2); codes go to row grow of nx_codes, scales to
//     the tensor-core layout (rows between M and the 128-row padding get
//     scale 0, as the quantizer writes them);
//  3. the next layer's rank-r down-projection over these NC columns,
//     h [32 rows x NC] (L_down / lambda) [NC x r], on the warp's tensor
//     cores (m16n8k16 bf16 MMAs; h is exact in bf16, L_down / lambda enters
//     as its hi and lo bf16 planes), added into nx_acc with fp32 atomics.
// Every lane takes part in step 3 (warp-wide MMAs), whatever its row.
template <int NC>
__device__ __forceinline__ void gp_gelu_epilogue(const uint32_t (&acc)[NC], const GemmArgs& a, float S,
                                                 float six_s2, const float* inv_tab, int64_t grow, int nbase,
                                                 uint32_t scr, const uint16_t* gelu_tab, uint32_t lane,
                                                 const CUtensorMap* tm_codes) {
    static_assert(NC % 64 == 0, "a warp covers whole groups of four scale bytes");
    const bool row_ok = grow < a.M;
    const int64_t kg4n = a.N / 64;
    uint32_t hpk[NC / 2];
    uint32_t cw[NC / 8];   // this row's codes of the NC columns (4 bits each)
    uint32_t sword = 0u;
#pragma unroll
    for (int c = 0; c < NC / 16; ++c) {
        const int n = nbase + 16 * c;
        uint32_t bw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (a.bias) {
            const uint4 w0 = __ldg(reinterpret_cast<const uint4*>(a.bias + n));
            const uint4 w1 = __ldg(reinterpret_cast<const uint4*>(a.bias + n) + 1);
            bw[0] = w0.x, bw[1] = w0.y, bw[2] = w0.z, bw[3] = w0.w;
            bw[4] = w1.x, bw[5] = w1.y, bw[6] = w1.z, bw[7] = w1.w;
        }
        float h[16];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float o0 = fmaf(__uint_as_float(acc[16 * c + 2 * p]), S, bf16lo_to_f32(bw[p]));
            const float o1 = fmaf(__uint_as_float(acc[16 * c + 2 * p + 1]), S, bf16hi_to_f32(bw[p]));
            const __nv_bfloat162 y2 = __floats2bfloat162_rn(o0, o1);
            const uint32_t yb = *reinterpret_cast<const uint32_t*>(&y2);
            const uint32_t hb = gelu_bf16_bits(yb & 0xFFFFu, gelu_tab) | (gelu_bf16_bits(yb >> 16, gelu_tab) << 16);
            hpk[8 * c + p] = hb;
            h[2 * p] = __uint_as_float(hb << 16);
            h[2 * p + 1] = __uint_as_float(hb & 0xFFFF0000u);
        }
        const float4* il = reinterpret_cast<const float4*>(a.nx_inv_lambda + n);
        float v[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 l = __ldg(il + q);
            fmul2_rn(h[4 * q], h[4 * q + 1], l.x, l.y, v[4 * q], v[4 * q + 1]);
            fmul2_rn(h[4 * q + 2], h[4 * q + 3], l.z, l.w, v[4 * q + 2], v[4 * q + 3]);
        }
        float m0 = fmaxf(fabsf(v[0]), fabsf(v[1])), m1 = fmaxf(fabsf(v[2]), fabsf(v[3]));
#pragma unroll
        for (int i = 4; i < 16; i += 4) {
            m0 = fmaxf(m0, fmaxf(fabsf(v[i]), fabsf(v[i + 1])));
            m1 = fmaxf(m1, fmaxf(fabsf(v[i + 2]), fabsf(v[i + 3])));
        }
        const uint32_t eb = cvt_e4m3(__fdiv_rn(fmaxf(m0, m1), six_s2));
        const float inv = inv_tab[eb];
        float qv[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) fmul2_rn(v[i], v[i + 1], inv, inv, qv[i], qv[i + 1]);
        cw[2 * c] = cvt_e2m1x8(qv);
#pragma unroll
        for (int i = 0; i < 8; i += 2) fmul2_rn(v[8 + i], v[9 + i], inv, inv, qv[i], qv[i + 1]);
        cw[2 * c + 1] = cvt_e2m1x8(qv);
        sword |= eb << (8 * (c & 3));
        if ((c & 3) == 3) {
            const int64_t g0 = (n - 48) / 16;   // the first of these four groups (a multiple of 4)
            if (grow < a.nx_rows_pad)
                *reinterpret_cast<uint32_t*>(a.nx_scales + sf_offset(grow, g0, kg4n)) = row_ok ? sword : 0u;
            sword = 0u;
        }
    }
    // the warp's 32 rows x NC / 2 bytes of codes leave through its scratch as
    // one TMA store (row-wise 16-byte stores by every thread were slower)
    static_assert(NC == 64, "one 32-byte code row per thread fills the 1 KB scratch");
    const int64_t row0 = grow - (int64_t)lane;   // the warp's first row
    st_shared_v4(scr + 32u * lane, cw[0], cw[1], cw[2], cw[3]);
    st_shared_v4(scr + 32u * lane + 16u, cw[4], cw[5], cw[6], cw[7]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && row0 < a.M) {   // rows past M inside the box are clipped by the tensor map
        tma_store_2d(tm_codes, scr, nbase / 2, (int)row0);
        bulk_commit_group();
    }
    if (lane == 0) bulk_wait_group_read<0>();   // the scratch is reused below
    __syncwarp();
    if (a.nx_rank == 0) return;
    // ---- rank-r down-projection of the next layer over these NC columns
    const int g = (int)(lane >> 2), t = (int)(lane & 3);
    const int nj = a.nx_rank / 8;                     // 2 or 4 column blocks of 8
    const int64_t plane = (int64_t)a.nx_rank * a.N;   // hi plane, then lo plane
    float lacc[2][4][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) lacc[mt][j][e] = 0.0f;
    const uint32_t my_row = scr + 32u * lane;
#pragma unroll
    for (int kb = 0; kb < NC / 16; ++kb) {
        // Within a block of 16 K values the MMA's K slots are taken in the
        // order 0 1 4 5 8 9 12 13 | 2 3 6 7 10 11 14 15 (the same permutation
        // for A and B leaves the product unchanged): a lane's two B registers
        // then hold four consecutive K values, one 8-byte load per plane,
        // issued ahead of the transposition so that their latency overlaps it.
        uint2 bf[4][2];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            bf[j][0] = bf[j][1] = make_uint2(0u, 0u);
            if (j < nj) {
                const __nv_bfloat16* bp = a.nx_ldt + (int64_t)(8 * j + g) * a.N + (nbase + 16 * kb + 4 * t);
                bf[j][0] = __ldg(reinterpret_cast<const uint2*>(bp));
                bf[j][1] = __ldg(reinterpret_cast<const uint2*>(bp + plane));
            }
        }
        // this lane's row of the block: pairs (0 1)(4 5)(8 9)(12 13), then
        // (2 3)(6 7)(10 11)(14 15), as two 16-byte pieces placed at
        // piece ^ ((row / 4) % 2) so that neither these stores nor the
        // ldmatrix reads below meet a bank twice
        const uint32_t sw = (lane >> 2) & 1u;
        st_shared_v4(my_row + (sw << 4), hpk[8 * kb], hpk[8 * kb + 2], hpk[8 * kb + 4], hpk[8 * kb + 6]);
        st_shared_v4(my_row + ((sw ^ 1u) << 4), hpk[8 * kb + 1], hpk[8 * kb + 3], hpk[8 * kb + 5],
                     hpk[8 * kb + 7]);
        __syncwarp();
        uint32_t af[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const uint32_t rr = 16u * mt + ((lane >> 3) & 1u) * 8u + (lane & 7u);
            const uint32_t kch = lane >> 4;
            ldmatrix_x4(af[mt], scr + 32u * rr + ((kch ^ ((rr >> 2) & 1u)) << 4));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j < nj) {
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    mma_16816_bf16(lacc[mt][j], af[mt], bf[j][0].x, bf[j][0].y);
                    mma_16816_bf16(lacc[mt][j], af[mt], bf[j][1].x, bf[j][1].y);
                }
            }
        }
        __syncwarp();
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j < nj) {
                const int64_t r0 = row0 + 16 * mt + g, r1 = r0 + 8;
                const int col = 8 * j + 2 * t;
                if (r0 < a.M)
                    atomicAdd(reinterpret_cast<float2*>(a.nx_acc + r0 * a.nx_rank + col),
                              make_float2(lacc[mt][j][0], lacc[mt][j][1]));
                if (r1 < a.M)
                    atomicAdd(reinterpret_cast<float2*>(a.nx_acc + r1 * a.nx_rank + col),
                              make_float2(lacc[mt][j][2], lacc[mt][j][3]));
            }
        }
}

// bf16(S acc + b) of one thread's row for the 32 columns of chunk c2 of its
// 128 accumulators, as 16 packed words.  The bias pair of the warp's columns
// 2j, 2j + 1 (word j of its bias) sits in lane j % 32, entry j / 32 of qb
// (zero past N), fetched before the accumulator was ready.
// The GELU epilogue's store-only form: columns nbase .. nbase + NC - 1 of
// h = bf16(GELU(bf16(S acc + b))) (the y of the plain epilogue, then the same
// table GELU as the fused path and the unfused pass) for the warp's 32 rows,
// leaving through the warp's 1 KB of scratch as TMA stores of 32 x 16 boxes
// (row-wise 16-byte stores by every thread took 32 us more over fc1 of the
// DiT MLP).
template <int NC>
__device__ __forceinline__ void gp_gelu_store(const uint32_t (&acc)[NC], const GemmArgs& a, float S, int nbase,
                                              const uint16_t* gelu_tab, uint32_t buf, uint32_t lane,
                                              const CUtensorMap* tm_y, int row0) {
#pragma unroll
    for (int c = 0; c < NC / 16; ++c) {
        const int n = nbase + 16 * c;
        uint32_t bw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (a.bias) {
            const uint4 w0 = __ldg(reinterpret_cast<const uint4*>(a.bias + n));
            const uint4 w1 = __ldg(reinterpret_cast<const uint4*>(a.bias + n) + 1);
            bw[0] = w0.x, bw[1] = w0.y, bw[2] = w0.z, bw[3] = w0.w;
            bw[4] = w1.x, bw[5] = w1.y, bw[6] = w1.z, bw[7] = w1.w;
        }
        uint32_t hb[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float o0 = fmaf(__uint_as_float(acc[16 * c + 2 * p]), S, bf16lo_to_f32(bw[p]));
            const float o1 = fmaf(__uint_as_float(acc[16 * c + 2 * p + 1]), S, bf16hi_to_f32(bw[p]));
            const __nv_bfloat162 y2 = __floats2bfloat162_rn(o0, o1);
            const uint32_t yb = *reinterpret_cast<const uint32_t*>(&y2);
            hb[p] = gelu_bf16_bits(yb & 0xFFFFu, gelu_tab) | (gelu_bf16_bits(yb >> 16, gelu_tab) << 16);
        }
        if (lane == 0) bulk_wait_group_read<0>();   // the previous box has left the buffer
        __syncwarp();
        st_shared_v4(buf + 32u * lane, hb[0], hb[1], hb[2], hb[3]);
        st_shared_v4(buf + 32u * lane + 16u, hb[4], hb[5], hb[6], hb[7]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < a.M) {   // rows past M inside a box are clipped by the tensor map
            tma_store_2d(tm_y, buf, n, row0);
            bulk_commit_group();
        }
    }
}

__device__ __forceinline__ void gp_pack32(const uint32_t (&acc)[128], int c2, const uint32_t (&qb)[2], float S,
                                          uint32_t (&pk)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int j = 16 * c2 + i;
        const uint32_t bw = __shfl_sync(0xffffffffu, qb[j / 32], j % 32);
        const float o0 = fmaf(__uint_as_float(acc[2 * j]), S, bf16lo_to_f32(bw));
        const float o1 = fmaf(__uint_as_float(acc[2 * j + 1]), S, bf16hi_to_f32(bw));
        const __nv_bfloat162 hv = __floats2bfloat162_rn(o0, o1);
        pk[i] = *reinterpret_cast<const uint32_t*>(&hv);
    }
}

// One warp's 32 rows x 32 columns of y through a 2 KB staging buffer: each
// lane writes its row (16-byte piece j at j ^ ((lane / 2) % 4), the 64-byte
// swizzle of the y tensor map), then lane 0 stores the box at (n, row0) with
// TMA.  Before writing, lane 0 waits until at most kYBufs - 1 earlier stores
// of this thread still read shared memory (the warp cycles kYBufs buffers).
__device__ __forceinline__ void gp_stage_store(const uint32_t (&pk)[16], uint32_t buf, uint32_t lane,
                                               const CUtensorMap* tm_y, int n, int row0, int M) {
    if (lane == 0) bulk_wait_group_read<gp::kYBufs - 1>();
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j)
        st_shared_v4(buf + 64u * lane + ((uint32_t)(j ^ ((lane >> 1) & 3)) << 4), pk[4 * j], pk[4 * j + 1],
                     pk[4 * j + 2], pk[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && row0 < M) {   // a box wholly past M is not stored at all
        tma_store_2d(tm_y, buf, n, row0);
        bulk_commit_group();
    }
}

// kEpi: kEpiPlain, kEpiQkv (the fused QKV + RMSNorm + RoPE epilogue) or
// kEpiGelu (the fused GELU + next-layer activation epilogue).
template <int kEpi>
__global__ void __launch_bounds__(gp_threads<kEpi>(), 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_wc,
                           const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                           const __grid_constant__ CUtensorMap tm_L, const __grid_constant__ CUtensorMap tm_Lup,
                           const __grid_constant__ CUtensorMap tm_y, GemmArgs a) {
    using namespace gp;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kStages * STAGE_BYTES);
    uint64_t* empty = full + kStages;
    uint64_t* acc_full = empty + kStages;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* tab_free = acc_empty + 1;    // [4] fused QKV: both warps of a lane quarter are done with its table
    uint64_t* tab_ready = tab_free + 4;    // [4] fused QKV: both halves of a lane quarter's new table are in TMEM
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tab_ready + 4);
    __shared__ int s_failed;
    __shared__ int s_issued[gp::kStages];   // phases this CTA's A producers started in each stage

    const uint32_t warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_ctarank();          // 0 = the CTA that issues the MMAs
    const int cluster = (int)(blockIdx.x >> 1), n_clusters = (int)(gridDim.x >> 1);
    const int n_kb = (a.K + 255) / 256;
    const int n_lr = a.rank > 0 ? 2 * ((a.rank + 63) / 64) : 0;
    const int per_tile = n_kb + n_lr;
    const int total_tiles = a.m_tiles * a.n_tiles;    // m_tiles counts 256-row tiles here
    // Each cluster takes a contiguous run of tiles, n fastest, so that it keeps
    // the same 256 activation rows for several tiles in a row.
    const int t_begin = (int)(((int64_t)total_tiles * cluster) / n_clusters);
    const int t_end = (int)(((int64_t)total_tiles * (cluster + 1)) / n_clusters);
    const bool sfa_res = kEpi != kEpiQkv && a.kg4 <= kResidentKSteps;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], kFullArrivals);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 2);   // both MMA warps commit at the end of every tile
        mbar_init(acc_empty, 2u * (uint32_t)gp_epi_warps<kEpi>());   // both CTAs' epilogue warps
        for (int i = 0; i < 4; ++i) {
            mbar_init(&tab_free[i], 2);
            mbar_init(&tab_ready[i], 2);
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
    if (warp == 1 && lane == 0 && t_begin < t_end) {
        // the first stages' weight codes and replicated weight scales are
        // packed long before this call: start pulling them into the L2 while
        // the previous kernel finishes
        const int n_tile = t_begin % a.n_tiles;
        const int n0 = n_tile * BN + 128 * (int)rank;
        for (int kb = 0; kb < kStages && kb < n_kb; ++kb) {
            tma_prefetch_l2_2d(&tm_wc, kb * BK_BYTES, n0);
            tma_prefetch_l2_3d(&tm_sfb, 0, 0, n_tile * n_kb + kb);
        }
    }
    if (warp == kMmaWarp) {   // the same warp in both CTAs, the same slot offset
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (gp_is_gelu(kEpi))     // the bf16 GELU table (gelu_mlp.cuh), once per CTA
        gelu_table_fill(reinterpret_cast<uint16_t*>(smem + (size_t)kStages * STAGE_BYTES + 256 +
                                                    (size_t)kEpiWarpsGelu * kGeluScratch),
                        (int)threadIdx.x, gp_threads<kEpi>(), a.gelu_approx);
    tc_fence_before();
    cluster_sync_all();       // barriers of both CTAs initialised, TMEM address written
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Everything above overlaps the previous kernel under programmatic
    // dependent launch (the activation quantizer releases its dependents
    // early); from here on this kernel reads that kernel's outputs.
    griddep_wait();

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
                const int m_tile = tile / a.n_tiles, n_tile = tile - m_tile * a.n_tiles;
                const bool need_sfa = !sfa_res || tile == t_begin || n_tile == 0;
                const int m0 = m_tile * BM + 128 * (int)rank;      // this CTA's activation rows
                const int n0 = n_tile * BN + 128 * (int)rank;      // this CTA's weight rows
                for (int kk = 0; kk < per_tile; ++kk, ++it) {
                    if ((it % kLanesPerRole) != (int)rlane) continue;
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, kSiteGpEmpty)) {
                        s_failed = 1;
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + (size_t)s * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    uint8_t* sfa = sb + B_BYTES;
                    uint8_t* sfb = sfa + SFA_BYTES;
                    const uint32_t bar = cluster_addr(&full[s], 0);   // CTA 0 counts every load
                    if (kk < n_kb) {
                        const int kb = kk;
                        if (role == 0) {
                            if (leader) mbar_arrive_expect_tx(&full[s], 2u * A_BYTES);
                            tma_load_2d_pair(sa, &tm_xc, bar, kb * BK_BYTES, m0);
                            atomicAdd(&s_issued[s], 1);
                        } else if (role == 1) {
                            if (leader) mbar_arrive_expect_tx(&full[s], 2u * B_BYTES);
                            tma_load_2d_pair(sb, &tm_wc, bar, kb * BK_BYTES, n0);
                        } else {
                            if (leader)
                                mbar_arrive_expect_tx(&full[s], 2u * ((need_sfa ? SFA_BYTES : 0) + SFB_BYTES));
                            if (need_sfa) tma_load_3d_pair(sfa, &tm_sfa, bar, 0, 4 * kb, 2 * m_tile + (int)rank);
                            // the tile's replicated weight scales for these four k-steps (16 KB)
                            tma_load_3d_pair(sfb, &tm_sfb, bar, 0, 0, n_tile * n_kb + kb);
                        }
                    } else {
                        const int c = (kk - n_kb) >> 1, part = (kk - n_kb) & 1;
                        if (role == 0) {
                            if (leader) mbar_arrive_expect_tx(&full[s], 2u * A_BYTES);
                            tma_load_3d_pair(sa, &tm_L, bar, c * 64, m0, part);
                            atomicAdd(&s_issued[s], 1);
                        } else if (role == 1) {
                            if (leader) mbar_arrive_expect_tx(&full[s], 2u * B_BYTES);
                            tma_load_2d_pair(sb, &tm_Lup, bar, c * 64, n0);
                        } else {
                            if (leader) mbar_arrive(&full[s]);
                        }
                    }
                }
            }
        }
    } else if (warp == kMmaWarp || warp == kMmaWarp2) {
        // ------------------------------------------ copies + MMAs (CTA 0 only)
        // Two warps take the stages in turn (warp kMmaWarp the even ones, in
        // the order of the whole run), each waiting on its own stage and
        // accumulator barriers; lane 0 issues the copies and MMAs.  Issue
        // blocks while the tensor pipe's queue is full, so a single issuer
        // left the pipe idle for the commit, the loop and the next wait at
        // every stage; with two, one warp's bookkeeping overlaps the other's
        // issue.  They hand the turn over through two named barriers (the
        // owner of stage i arrives after issuing it; the other warp syncs
        // before stage i + 1), so the MMAs reach the pipe in stage order and
        // the accumulation order is fixed.  Both warps commit to acc_full at
        // the end of every tile (it counts two arrivals).
        if (rank == 0) {
            const uint32_t me = warp - kMmaWarp;   // 0: even stages, 1: odd stages
            const uint32_t idesc_fp4 = idesc_m(idesc_nvfp4(BN), BM);
            const uint32_t idesc_lr = idesc_m(idesc_bf16_f32(BN), BM);
            const uint32_t smem0 = smem_u32(smem);
            const int nks_last = a.kg4 - 4 * (n_kb - 1);   // K-steps in the last stage (1..4)
            bool ok = true;
            int local = 0, it = 0;
            for (int tile = t_begin; tile < t_end && ok; ++tile, ++local) {
                const int n_tile = tile % a.n_tiles;
                const bool need_sfa = !sfa_res || tile == t_begin || n_tile == 0;
                for (int kk = 0; kk < per_tile; ++kk, ++it) {
                    if ((uint32_t)(it & 1) != me) continue;
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    bool fail = !mbar_wait(&full[s], ph, kSiteGpFull);
                    if (!fail && kk == 0) fail = !mbar_wait(acc_empty, ((uint32_t)local & 1u) ^ 1u, kSiteGpAccEmpty);
                    if (fail) s_failed = 1;
                    // warp-uniform, so that the whole warp takes the same barriers
                    fail = __any_sync(0xffffffffu, fail || *reinterpret_cast<volatile int*>(&s_failed) != 0);
                    // everything but the issue itself before the turn comes
                    const uint32_t sa = smem0 + (uint32_t)s * STAGE_BYTES;
                    const uint64_t da = desc_sw128(sa), db = desc_sw128(sa + A_BYTES);   // + 2 per 32-byte K-step
                    const uint64_t dfa = desc_sf_block(sa + A_BYTES + B_BYTES);          // + 32 per 512 bytes
                    const uint64_t dfb = desc_sfb_kstep(sa + A_BYTES + B_BYTES + SFA_BYTES);
                    // activation-scale columns of this stage's K-steps, weight-scale set
                    const uint32_t ta = sfa_res ? tmem + SFA_RES + 16u * (uint32_t)kk : tmem + SF_COL + SF_SET_COLS * me;
                    const uint32_t tb = sfa_res ? tmem + SFB_RES + 32u * me : ta + 16u;
                    const uint32_t acc0 = kk > 0 ? 1u : 0u;
                    if (it > 0) named_bar_sync(kBarTurn0 + me, 64);   // the other warp has issued stage it - 1
                    if (!fail && lane == 0) {
                        tc_fence_after();
                        if (kk < n_kb) {
                            if (kk + 1 < n_kb || nks_last == 4) {
                                if (need_sfa)
                                    gp_issue_stage<true>(tmem + ACC_COL, da, db, dfa, dfb, ta, tb, idesc_fp4, acc0);
                                else
                                    gp_issue_stage<false>(tmem + ACC_COL, da, db, dfa, dfb, ta, tb, idesc_fp4, acc0);
                            } else {
                                // a last stage of fewer than four K-steps
                                for (int j = 0; j < nks_last; ++j) {
                                    if (need_sfa) tmem_cp_32x128b_x4_pair(ta + 4u * j, dfa + 32u * j);
                                    tmem_cp_128x256b_pair(tb + 8u * j, dfb + (uint64_t)(SFB_KSTEP_BYTES >> 4) * j);
                                    mma_nvfp4_pair(tmem + ACC_COL, da + 2u * j, db + 2u * j, idesc_fp4, ta + 4u * j,
                                                   tb + 8u * j, (kk > 0 || j > 0) ? 1u : 0u);
                                }
                            }
                        } else {
                            // rank-r stage: bf16 MMAs of the hi or lo part into the same accumulator
                            const int c = (kk - n_kb) >> 1;
                            const int nks = min(4, (a.rank - 64 * c + 15) / 16);
                            for (int j = 0; j < nks; ++j)
                                mma_bf16_pair(tmem + ACC_COL, da + 2u * j, db + 2u * j, idesc_lr, 1u);
                        }
                    }
                    __syncwarp();
                    // the other warp may issue stage it + 1 (its MMAs are not tracked by this warp's commit)
                    named_bar_arrive(kBarTurn0 + (me ^ 1u), 64);
                    if (!fail && lane == 0) tc_commit_pair(&empty[s], 0x3);
                    if (fail) {
                        ok = false;
                        break;
                    }
                }
                // this warp's share of the tile is issued (possibly none of it)
                if (ok && lane == 0) tc_commit_pair(acc_full, 0x3);
            }
            // the warp that did not issue the run's last stage takes the last turn hand-over
            if (ok && it > 0 && (uint32_t)((it - 1) & 1) != me) named_bar_sync(kBarTurn0 + me, 64);
        }
    } else if (warp >= (uint32_t)kEpiWarp0) {
        // ------------------------------------------------------------ epilogue
        const uint32_t q = warp & 3u;
        const int half = (int)(warp - kEpiWarp0) >> 2;
        const int row = (int)(32u * q + lane);
        const float S = __fmul_rn(*a.x_scale, *a.w_scale);
        const uint32_t acc_empty_leader = cluster_addr(acc_empty, 0);
        float gelu_six_s2 = 6.0f;
        uint32_t gelu_scr = 0u;
        uint8_t* gelu_base = smem + (size_t)kStages * STAGE_BYTES + 256;
        const uint16_t* gelu_tab =
            reinterpret_cast<const uint16_t*>(gelu_base + (size_t)kEpiWarpsGelu * kGeluScratch);
        float* gelu_inv = reinterpret_cast<float*>(gelu_base + (size_t)kEpiWarpsGelu * kGeluScratch + kGeluTabBytes);
        if (gp_is_gelu(kEpi)) {
            const float S2 = kEpi == kEpiGeluStore ? 1.0f : *a.nx_x_scale;   // unused by the store-only form
            gelu_six_s2 = __fmul_rn(6.0f, S2);
            gelu_scr = smem_u32(gelu_base);
            // reciprocals of the 128 decoded group scales e * S2, as the
            // activation quantizer tabulates them
            const int t = (int)threadIdx.x - 32 * kEpiWarp0;
            if (t < 128) {
                const float dec = __fmul_rn(e4m3_to_f32((uint32_t)t), S2);
                gelu_inv[t] = (dec == 0.0f) ? 0.0f : __frcp_rn(dec);
            }
            named_bar_sync(1, 32 * kEpiWarpsGelu);
        }
        int local = 0;
        int epoch = -1, prev_m = -1;   // fused QKV: rotary tables loaded so far, and for which row block
        for (int tile = t_begin; tile < t_end; ++tile, ++local) {
            const int m_tile = tile / a.n_tiles, n_tile = tile - m_tile * a.n_tiles;
            const int64_t grow = (int64_t)m_tile * BM + 128 * (int64_t)rank + row;
            const int nbase = n_tile * BN + 128 * half;
            // Before the accumulator is ready: this warp's 128 columns of bias,
            // pairs l and 32 + l in lane l (uniform loads inside the epilogue
            // each waited a full L2 round trip under the main loop's traffic);
            // fused QKV: on a new row block the two warps of this lane quarter
            // put the rows' rotary tables into TMEM (this warp one of cos /
            // sin), and a Q or K head's RMSNorm weights go with the bias
            uint32_t qbias[2] = {0u, 0u}, qgam[2] = {0u, 0u};
            const bool qk_head = kEpi == kEpiQkv && nbase < a.qk_cols;
            if (!gp_is_gelu(kEpi) && a.bias) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int col = nbase + 2 * (32 * i + (int)lane);
                    if (col < a.N) qbias[i] = __ldg(reinterpret_cast<const uint32_t*>(a.bias + col));
                }
            }
            if (kEpi == kEpiQkv) {
                if (m_tile != prev_m) {
                    ++epoch;
                    prev_m = m_tile;
                    if (epoch > 0) {   // the old table: this warp is done with it; wait for the other
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tab_free[q]);
                        if (!mbar_wait(&tab_free[q], (uint32_t)(epoch - 1) & 1u, kSiteGpTab)) {
                            s_failed = 1;
                            break;
                        }
                        tc_fence_after();
                    }
                    // rows past M take the last row's table (their results are not stored)
                    const int64_t trow = grow < a.M ? grow : (int64_t)a.M - 1;
                    const float4* src = reinterpret_cast<const float4*>((half == 0 ? a.rope_cos : a.rope_sin) + trow * 64);
#pragma unroll
                    for (int p2 = 0; p2 < 2; ++p2) {
                        uint32_t t32[32];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 v = __ldg(src + 8 * p2 + i);
                            t32[4 * i] = __float_as_uint(v.x);
                            t32[4 * i + 1] = __float_as_uint(v.y);
                            t32[4 * i + 2] = __float_as_uint(v.z);
                            t32[4 * i + 3] = __float_as_uint(v.w);
                        }
                        tmem_st_32x32b_x32(tmem + ((32u * q) << 16) + QKV_TAB_COL + 64u * (uint32_t)half + 32u * p2,
                                           t32);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tab_ready[q]);
                    if (!mbar_wait(&tab_ready[q], (uint32_t)epoch & 1u, kSiteGpTab)) {
                        s_failed = 1;
                        break;
                    }
                    tc_fence_after();
                }
                if (qk_head) {
                    const __nv_bfloat16* gw = nbase < a.q_cols ? a.norm_q : a.norm_k;
#pragma unroll
                    for (int i = 0; i < 2; ++i) qgam[i] = __ldg(reinterpret_cast<const uint32_t*>(gw) + 32 * i + lane);
                }
            }
            if (!mbar_wait(acc_full, (uint32_t)local & 1u, kSiteGpAcc)) {
                s_failed = 1;
                break;
            }
            tc_fence_after();
            if (gp_is_gelu(kEpi)) {
                // four warps per lane quadrant: this warp's 64 columns
                const int part = (int)(warp - kEpiWarp0) >> 2;
                const int gbase = n_tile * BN + 64 * part;
                uint32_t acc[64];
                tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 64u * part + 0u,
                                   *reinterpret_cast<uint32_t(*)[32]>(acc + 0));
                tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 64u * part + 32u,
                                   *reinterpret_cast<uint32_t(*)[32]>(acc + 32));
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
                // warp-uniform: with N % 128 == 0 a warp's columns are all in or all out
                if (gbase < a.N) {
                    if (kEpi == kEpiGeluStore)
                        gp_gelu_store<64>(acc, a, S, gbase, gelu_tab,
                                          gelu_scr + (uint32_t)(warp - kEpiWarp0) * (uint32_t)kGeluScratch, lane,
                                          &tm_y, (int)(grow - (int64_t)lane));
                    else
                        gp_gelu_epilogue<64>(acc, a, S, gelu_six_s2, gelu_inv, grow, gbase,
                                             gelu_scr + (uint32_t)(warp - kEpiWarp0) * (uint32_t)kGeluScratch,
                                             gelu_tab, lane, &tm_y);
                }
                continue;
            }
            uint32_t acc[128];
            tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 128u * half + 0u,
                               *reinterpret_cast<uint32_t(*)[32]>(acc + 0));
            tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 128u * half + 32u,
                               *reinterpret_cast<uint32_t(*)[32]>(acc + 32));
            tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 128u * half + 64u,
                               *reinterpret_cast<uint32_t(*)[32]>(acc + 64));
            tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 128u * half + 96u,
                               *reinterpret_cast<uint32_t(*)[32]>(acc + 96));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader);   // this half of the pair is drained
            // y leaves 32 columns at a time through this warp's staging
            // buffers and a TMA store (gp_stage_store); rows past M and
            // columns past N are not written
            const uint32_t stage0 =
                smem_u32(smem + Y_STAGE_OFF) + (uint32_t)(warp - kEpiWarp0) * (uint32_t)(kYBufs * kYStageBytes);
            const int row0 = (int)(grow - lane);
            if (qk_head) {
                // this warp's 128 columns are one Q or K head of a to_qkv
                // projection (qkv_norm_rope.cuh): RMSNorm over them, then the
                // rotary pairs, on the fp32 values before the single bf16 rounding
                float ss = 0.0f;
#pragma unroll
                for (int j = 0; j < 64; ++j) {   // pair j: columns nbase + 2j, + 1; its bias in lane j % 32
                    const uint32_t bw = __shfl_sync(0xffffffffu, qbias[j / 32], j % 32);
                    const float o0 = fmaf(__uint_as_float(acc[2 * j]), S, bf16lo_to_f32(bw));
                    const float o1 = fmaf(__uint_as_float(acc[2 * j + 1]), S, bf16hi_to_f32(bw));
                    acc[2 * j] = __float_as_uint(o0);
                    acc[2 * j + 1] = __float_as_uint(o1);
                    ss = fmaf(o0, o0, ss);
                    ss = fmaf(o1, o1, ss);
                }
                const float r = rsqrtf(ss * (1.0f / 128.0f) + a.eps);
#pragma unroll
                for (int c2 = 0; c2 < 4; ++c2) {
                    // the rotary table of pairs 16 c2 .. 16 c2 + 15 of this row, from TMEM
                    uint32_t cc[16], sc[16];
                    tmem_ld_32x32b_x16(tmem + ((32u * q) << 16) + QKV_TAB_COL + 16u * c2, cc);
                    tmem_ld_32x32b_x16(tmem + ((32u * q) << 16) + QKV_TAB_COL + 64u + 16u * c2, sc);
                    tmem_ld_wait();
                    uint32_t pk[16];
#pragma unroll
                    for (int p = 0; p < 16; ++p) {
                        const int j = 16 * c2 + p;
                        const uint32_t gw = __shfl_sync(0xffffffffu, qgam[j / 32], j % 32);
                        const float v0 = __uint_as_float(acc[2 * j]) * r * bf16lo_to_f32(gw);
                        const float v1 = __uint_as_float(acc[2 * j + 1]) * r * bf16hi_to_f32(gw);
                        const float cj = __uint_as_float(cc[p]), sj = __uint_as_float(sc[p]);
                        const __nv_bfloat162 hv = __floats2bfloat162_rn(v0 * cj - v1 * sj, v1 * cj + v0 * sj);
                        pk[p] = *reinterpret_cast<const uint32_t*>(&hv);
                    }
                    gp_stage_store(pk, stage0 + (uint32_t)(c2 % kYBufs) * kYStageBytes, lane, &tm_y, nbase + 32 * c2,
                                   row0, a.M);
                }
                continue;
            }
#pragma unroll
            for (int c2 = 0; c2 < 4; ++c2) {
                const int n = nbase + 32 * c2;
                if (n >= a.N) break;   // warp-uniform
                uint32_t pk[16];
                gp_pack32(acc, c2, qbias, S, pk);
                gp_stage_store(pk, stage0 + (uint32_t)(c2 % kYBufs) * kYStageBytes, lane, &tm_y, n, row0, a.M);
            }
        }
    }

    if (warp >= (uint32_t)kEpiWarp0 && lane == 0)
        bulk_wait_group<0>();   // this warp's TMA stores are done with shared memory and written
    __syncthreads();
    if (s_failed && rank == 0 && warp == 0 && lane == 0) {
        // after a timeout, let the loads already issued land before either CTA
        // exits (both CTAs' loads complete on CTA 0's barriers; best effort:
        // each wait is bounded)
        for (int s = 0; s < kStages; ++s) {
            const int n = reinterpret_cast<volatile int*>(s_issued)[s];
            if (n > 0) mbar_wait(&full[s], (uint32_t)(n - 1) & 1u, kSiteGpDrain);
        }
    }
    tc_fence_before();
    cluster_sync_all();   // no remote arrival or MMA may target a CTA that has exited
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

}  // namespace svdq
