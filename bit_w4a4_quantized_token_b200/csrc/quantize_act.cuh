// quantize_act.cuh -- activation quantizer of the SVDQ W4A4 layer, fused with
// the rank-r down-projection (sm_100a).
//
// One CTA owns a 128-row block of x and a contiguous range of 64-column
// chunks.  Two producer threads (warps 0 and 2, chunks taken in turn) stream
// each chunk into a ring of shared-memory stages with TMA: the 128 x 64 bf16
// tile of x (128-byte swizzled), the matching hi/lo tiles of L_down / lambda
// and the chunk's 64 values of 1/lambda.  Sixteen quantizer warps (4..19)
// turn the tile into 4-bit codes and group scales, one thread per row and
// group of 16 columns.  Warp 1 issues tcgen05.mma on the same tile: x (bf16,
// exact) times the hi and lo parts of L_down / lambda, fp32 in TMEM.
//
// When K is split over several CTAs, their fp32 rank-r partials are added in
// split order, so the result does not depend on timing:
//  * cluster mode: the CTAs of a row block form one thread-block cluster; each
//    leaves its partial in its own shared memory and, after a cluster barrier,
//    adds a slice of the rows of all partials through distributed shared
//    memory and stores that slice;
//  * workspace mode (more splits than a cluster holds at once): each CTA
//    writes its partial to a caller workspace and the last CTA of the row
//    block, found with a counter it resets afterwards, adds them.
// Without a split the CTA stages its result through shared memory so that the
// rank-r stores are coalesced.
#pragma once
#include "quantize.cuh"
#include "sm100_ptx.cuh"

namespace svdq {
namespace qa {
constexpr int kRows = 128;              // rows per CTA (= TMEM lanes of the MMA)
constexpr int kCols = 64;               // columns per stage (128 B of bf16)
constexpr int kXBytes = kRows * kCols * 2;
constexpr int kInvlBytes = kCols * 4;   // the chunk's 1/lambda values
constexpr int kWorkerWarps = 16;
constexpr int kWorker0 = 4;             // first quantizer warp (a multiple of 4: TMEM lane quadrants)
constexpr int kWorkers = 32 * kWorkerWarps;
constexpr int kThreads = 32 * (kWorker0 + kWorkerWarps);   // warp 1: MMA + TMEM; warps 0, 2: producers
constexpr int kMaxStages = 9;
constexpr int kMaxSplits = 16;
constexpr int kMaxCluster = 8;          // portable thread-block cluster size
constexpr int kSplitTarget = 148;       // CTAs wanted for one wave (SMs of a B200)
}  // namespace qa

constexpr int kPrecNvfp4 = 0, kPrecInt4 = 1;

struct QuantActArgs {
    const float* inv_lambda;   // [K]
    const float* x_scale;      // S_x (nvfp4)
    const float* w_scale;      // S_w (nvfp4 with rank > 0)
    uint8_t* x_codes;          // [M, K/2]
    uint8_t* x_scales;         // nvfp4: scale-factor layout; int4: bf16 [K/64, rows_pad]
    __nv_bfloat16* lowrank;    // [2, M, rank]: hi and lo bf16 planes
    float* partials;           // workspace mode: [row_blocks, splits, 128, rank] fp32
    unsigned int* counters;    // workspace mode: [row_blocks][2] (partials written, slices added); zero between calls
    int M, K, rank;
    int rows_pad;              // M rounded up to 128
    int chunks;                // K / 64
    int splits;                // CTAs sharing one 128-row block (blockIdx.x)
    int cluster;               // == splits in cluster mode, else 1
    int coop;                  // workspace mode, whole grid resident at once: every split adds a slice of rows
    int stages;
    uint32_t stage_bytes;      // x tile + hi/lo L_down_t tiles + 1/lambda chunk, rounded to 1 KB
    uint32_t invl_off;         // offset of the 1/lambda chunk in a stage
    uint32_t tmem_cols;
};

enum : uint32_t {
    kSiteQaEmpty = 1,
    kSiteQaFullMma = 2,
    kSiteQaFullWork = 3,
    kSiteQaAcc = 4,
    kSiteQaDrain = 5,
    kSiteQaSplits = 6
};

// Bounded wait until the global counter reaches `target` (acquire): the other
// CTAs of a K split writing their partials.  False (and the timeout recorded)
// after the wait limit.
__device__ __noinline__ bool qa_wait_count(const unsigned int* p, unsigned int target, uint32_t site) {
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = g_wait_limit_ns;
    while (true) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        if (v >= target) return true;
        if (globaltimer_ns() - t0 > limit) {
            record_timeout(site);
            return false;
        }
        __nanosleep(64);
    }
}

// L' = v * inv_ss as a bf16 hi/lo pair for two adjacent columns.
__device__ __forceinline__ void store_lowrank_pair(__nv_bfloat16* hi_dst, __nv_bfloat16* lo_dst, float v0, float v1,
                                                   float inv_ss) {
    __nv_bfloat16 h0, l0, h1, l1;
    split_bf16(__fmul_rn(v0, inv_ss), h0, l0);
    split_bf16(__fmul_rn(v1, inv_ss), h1, l1);
    *reinterpret_cast<__nv_bfloat162*>(hi_dst) = __halves2bfloat162(h0, h1);
    *reinterpret_cast<__nv_bfloat162*>(lo_dst) = __halves2bfloat162(l0, l1);
}

// One thread's group of 16 columns of one staged chunk: smoothing, then the
// nvfp4 group rule (E4M3 scale byte returned, 16 E2M1 codes in c0/c1) or, for
// int4, this lane's part of the row's group of 64 (bf16 scale bits returned,
// 16 two's-complement nibbles in c0/c1; the four lanes of a row exchange
// their maxima, so every lane of the warp must take part).
template <int PREC>
__device__ __forceinline__ uint32_t quant_group(const uint8_t* st, uint32_t xoff0, uint32_t xoff1, uint32_t loff,
                                                float six_s, const float* inv_tab, uint32_t& c0, uint32_t& c1) {
    const uint4 r0 = *reinterpret_cast<const uint4*>(st + xoff0);
    const uint4 r1 = *reinterpret_cast<const uint4*>(st + xoff1);
    const float4* il = reinterpret_cast<const float4*>(st + loff);
    const float4 l0 = il[0], l1 = il[1], l2 = il[2], l3 = il[3];
    float v[16];
    fmul2_rn(bf16lo_to_f32(r0.x), bf16hi_to_f32(r0.x), l0.x, l0.y, v[0], v[1]);
    fmul2_rn(bf16lo_to_f32(r0.y), bf16hi_to_f32(r0.y), l0.z, l0.w, v[2], v[3]);
    fmul2_rn(bf16lo_to_f32(r0.z), bf16hi_to_f32(r0.z), l1.x, l1.y, v[4], v[5]);
    fmul2_rn(bf16lo_to_f32(r0.w), bf16hi_to_f32(r0.w), l1.z, l1.w, v[6], v[7]);
    fmul2_rn(bf16lo_to_f32(r1.x), bf16hi_to_f32(r1.x), l2.x, l2.y, v[8], v[9]);
    fmul2_rn(bf16lo_to_f32(r1.y), bf16hi_to_f32(r1.y), l2.z, l2.w, v[10], v[11]);
    fmul2_rn(bf16lo_to_f32(r1.z), bf16hi_to_f32(r1.z), l3.x, l3.y, v[12], v[13]);
    fmul2_rn(bf16lo_to_f32(r1.w), bf16hi_to_f32(r1.w), l3.z, l3.w, v[14], v[15]);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    if (PREC == kPrecNvfp4) {
        const uint32_t eb = cvt_e4m3(__fdiv_rn(amax, six_s));
        const float inv = inv_tab[eb];
        float q[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) fmul2_rn(v[i], v[i + 1], inv, inv, q[i], q[i + 1]);
        c0 = cvt_e2m1x8(q);
#pragma unroll
        for (int i = 0; i < 8; i += 2) fmul2_rn(v[8 + i], v[9 + i], inv, inv, q[i], q[i + 1]);
        c1 = cvt_e2m1x8(q);
        return eb;
    } else {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
        const float sf = __bfloat162float(sb);
        const float inv = (sf == 0.0f) ? 0.0f : __frcp_rn(sf);
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            int qi = __float2int_rn(__fmul_rn(v[i], inv));
            qi = max(-8, min(7, qi));
            w[i >> 3] |= ((uint32_t)qi & 15u) << (4 * (i & 7));
        }
        c0 = w[0];
        c1 = w[1];
        return (uint32_t)__bfloat16_as_ushort(sb);
    }
}

// Grid (splits, ceil(M/128)); in cluster mode the `splits` CTAs of a row
// block form one cluster.  CTA (s, b) handles rows [128b, 128b+128) and chunks
// [s*T/splits, (s+1)*T/splits) of the T = K/64 column chunks.
template <int PREC>
__global__ void __launch_bounds__(qa::kThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_ld,
                        QuantActArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nst = a.stages;
    float* inv_tab = reinterpret_cast<float*>(smem + (size_t)nst * a.stage_bytes);   // [128] 1/(e*S)
    uint64_t* full = reinterpret_cast<uint64_t*>(inv_tab + 128);
    uint64_t* empty = full + qa::kMaxStages;
    uint64_t* accb = empty + qa::kMaxStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accb + 1);
    __shared__ int s_failed, s_last;
    __shared__ int s_issued[qa::kMaxStages];   // loads issued into each stage (phases started)

    const uint32_t warp = warp_id(), lane = lane_id();
    const int split = blockIdx.x, rb = blockIdx.y;
    const int m0 = rb * qa::kRows;
    const int c_lo = (int)((int64_t)a.chunks * split / a.splits);
    const int c_hi = (int)((int64_t)a.chunks * (split + 1) / a.splits);
    const int n_it = c_hi - c_lo;
    const bool has_lr = a.rank > 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], qa::kWorkerWarps + (has_lr ? 1u : 0u));   // quantizer warps + MMA commit
        }
        mbar_init(accb, 1);
        for (int s = 0; s < qa::kMaxStages; ++s) s_issued[s] = 0;
        s_failed = 0;
        s_last = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_x);
        if (has_lr) prefetch_tensormap(&tm_ld);
    }
    if (warp == 1 && has_lr) {
        tmem_alloc(tmem_slot, a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = has_lr ? *tmem_slot : 0u;
    // Everything above overlaps the previous kernel under programmatic
    // dependent launch; from here on this call reads its inputs and may
    // overwrite buffers the previous kernel read.
    griddep_wait();

    if ((warp == 0 || warp == 2) && lane == 0) {
        // ---------------------------------------------------------- producers
        const int pid = warp == 0 ? 0 : 1;
        const uint32_t bytes = qa::kXBytes + (has_lr ? 256u * (uint32_t)a.rank : 0u) + qa::kInvlBytes;
        int s = pid;   // stage of chunk `it` (it = pid, pid + 2, ...); nst >= 2
        uint32_t ph = 0;
        for (int it = pid; it < n_it; it += 2) {
            if (!mbar_wait(&empty[s], ph ^ 1u, kSiteQaEmpty)) {
                s_failed = 1;
                break;
            }
            const int kc = c_lo + it;
            uint8_t* st = smem + (size_t)s * a.stage_bytes;
            mbar_arrive_expect_tx(&full[s], bytes);
            tma_load_2d(st, &tm_x, &full[s], kc * qa::kCols, m0);
            if (has_lr) tma_load_3d(st + qa::kXBytes, &tm_ld, &full[s], kc * qa::kCols, 0, 0);   // hi and lo
            bulk_load(st + a.invl_off, a.inv_lambda + (int64_t)kc * qa::kCols, qa::kInvlBytes, &full[s]);
            atomicAdd(&s_issued[s], 1);
            s += 2;
            if (s >= nst) {
                s -= nst;
                ph ^= 1u;
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- rank-r MMA issuer
        if (has_lr && lane == 0) {
            // B = the hi and lo tiles stacked (2r rows): one MMA per k-step when
            // 2r <= 256, with hi and lo accumulated in separate column ranges
            const bool fused = 2 * a.rank <= 256;
            const uint32_t idesc = idesc_bf16_f32((uint32_t)(fused ? 2 * a.rank : a.rank));
            bool ok = true;
            int s = 0;
            uint32_t ph = 0;
            for (int it = 0; it < n_it; ++it) {
                if (!mbar_wait(&full[s], ph, kSiteQaFullMma)) {
                    ok = false;
                    s_failed = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t xa = smem_u32(smem + (size_t)s * a.stage_bytes);
                const uint32_t lb = xa + qa::kXBytes;
                if (fused) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_bf16(tmem, desc_sw128(xa + 32u * j), desc_sw128(lb + 32u * j), idesc,
                                 (it > 0 || j > 0) ? 1u : 0u);
                } else {
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_bf16(tmem + (uint32_t)part * (uint32_t)a.rank, desc_sw128(xa + 32u * j),
                                     desc_sw128(lb + (uint32_t)part * (uint32_t)a.rank * 128u + 32u * j), idesc,
                                     (it > 0 || j > 0) ? 1u : 0u);
                }
                tc_commit(&empty[s]);
                if (++s == nst) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (ok) tc_commit(accb);
        }
    } else if (warp >= (uint32_t)qa::kWorker0) {
        // --------------------------------------------------------- quantizers
        const int t = (int)threadIdx.x - 32 * qa::kWorker0;
        const int row = t >> 2, g = t & 3;            // 4 lanes per row: one group of 16 columns each
        const int64_t grow = (int64_t)m0 + row;
        const bool row_ok = grow < a.M;
        float six_s = 6.0f;
        if (PREC == kPrecNvfp4) {
            const float S = *a.x_scale;
            six_s = __fmul_rn(6.0f, S);
            if (t < 128) {
                // reciprocals of the 128 possible decoded group scales e * S
                const float dec = __fmul_rn(e4m3_to_f32((uint32_t)t), S);
                inv_tab[t] = (dec == 0.0f) ? 0.0f : __frcp_rn(dec);
            }
            named_bar_sync(1, qa::kWorkers);
        }
        // this thread's two 16-byte pieces of its row in a swizzled x tile
        const uint32_t xoff0 = (uint32_t)row * 128u + ((((uint32_t)(2 * g)) ^ ((uint32_t)row & 7u)) << 4);
        const uint32_t xoff1 = (uint32_t)row * 128u + ((((uint32_t)(2 * g + 1)) ^ ((uint32_t)row & 7u)) << 4);
        const uint32_t loff = a.invl_off + 64u * (uint32_t)g;
        uint8_t* cptr = a.x_codes + grow * (int64_t)(a.K / 2) + (int64_t)c_lo * 32 + g * 8;
        // nvfp4: byte (row, group 4 kc + g) of the scale layout, 512 bytes further per chunk
        uint8_t* sptr = a.x_scales + (((grow >> 7) * a.chunks + c_lo) * 512 + (grow & 31) * 16 + ((grow >> 5) & 3) * 4 + g);
        // int4: bf16 scale of (row, chunk) at [chunk, rows_pad]
        uint16_t* sptr16 = reinterpret_cast<uint16_t*>(a.x_scales) + (int64_t)c_lo * a.rows_pad + grow;
        // Two chunks per iteration: their groups are independent, so the two
        // dependency chains of a thread overlap.  (With an odd count the last
        // iteration also runs over the next ring slot without waiting for it:
        // what it reads there is discarded.)
        int s = 0;
        uint32_t ph = 0;
        for (int it = 0; it < n_it; it += 2) {
            const bool two = it + 1 < n_it;
            const int s1 = (s + 1 == nst) ? 0 : s + 1;
            const uint32_t ph1 = (s + 1 == nst) ? (ph ^ 1u) : ph;
            if (!mbar_wait(&full[s], ph, kSiteQaFullWork) || (two && !mbar_wait(&full[s1], ph1, kSiteQaFullWork))) {
                s_failed = 1;
                break;
            }
            uint32_t a0, a1, b0, b1;
            const uint32_t sa = quant_group<PREC>(smem + (size_t)s * a.stage_bytes, xoff0, xoff1, loff, six_s, inv_tab,
                                                  a0, a1);
            const uint32_t sb = quant_group<PREC>(smem + (size_t)s1 * a.stage_bytes, xoff0, xoff1, loff, six_s,
                                                  inv_tab, b0, b1);
            if (PREC == kPrecNvfp4) {
                sptr[0] = (uint8_t)sa;   // padding rows (x read as zero) get scale 0
                if (two) sptr[512] = (uint8_t)sb;
                sptr += 1024;
            } else {
                if (g == 0) {
                    sptr16[0] = (uint16_t)sa;
                    if (two) sptr16[a.rows_pad] = (uint16_t)sb;
                }
                sptr16 += 2 * (int64_t)a.rows_pad;
            }
            if (row_ok) {
                *reinterpret_cast<uint2*>(cptr) = make_uint2(a0, a1);
                if (two) *reinterpret_cast<uint2*>(cptr + 32) = make_uint2(b0, b1);
            }
            cptr += 64;
            // release the stages once every lane has read them
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&empty[s]);
                if (two) mbar_arrive(&empty[s1]);
            }
            s = s1 + 1;
            ph = ph1;
            if (s == nst) {
                s = 0;
                ph ^= 1u;
            }
        }
    }

    __syncthreads();
    // on a timeout, let the copies already issued land before the ring's
    // shared memory is reused below or the CTA exits
    if (s_failed && warp == 0 && lane == 0) {
        for (int s = 0; s < nst; ++s) {
            const int n = reinterpret_cast<volatile int*>(s_issued)[s];
            if (n > 0) mbar_wait(&full[s], (uint32_t)(n - 1) & 1u, kSiteQaDrain);
        }
    }
    __syncthreads();   // every stage consumed: the ring's shared memory is free
    griddep_launch_dependents();

    // ------------------------------------------------- rank-r result of the CTA
    if (has_lr) {
        const bool cluster_mode = a.cluster > 1;
        const bool workspace_mode = a.splits > 1 && !cluster_mode;
        const int pstride = a.rank + 4;                        // floats per row of the staged partial
        float* part = reinterpret_cast<float*>(smem);          // [128][rank + 4] fp32
        const float inv_ss =
            (PREC == kPrecNvfp4) ? __frcp_rn(__fmul_rn(*a.x_scale, *a.w_scale)) : 1.0f;
        if (warp >= (uint32_t)qa::kWorker0) {
            // the sixteen quantizer warps drain the accumulator: warp w reads
            // TMEM lane quadrant w % 4 (one thread per row) and every fourth
            // 16-column block from block (w - 4) / 4 on
            const uint32_t q = warp & 3u;
            const int row = (int)(32u * q + lane);
            const int first = 16 * (int)((warp - (uint32_t)qa::kWorker0) >> 2);
            const bool ok = mbar_wait(accb, 0, kSiteQaAcc);
            if (!ok) s_failed = 1;
            tc_fence_after();
            float* mine = workspace_mode ? a.partials + (((int64_t)rb * a.splits + split) * qa::kRows + row) * a.rank
                                         : part + row * pstride;
            for (int c0 = first; c0 < a.rank; c0 += 64) {
                uint32_t r16[16], s16[16];
                tmem_ld_32x32b_x16(tmem + ((32u * q) << 16) + (uint32_t)c0, r16);              // x . hi
                tmem_ld_32x32b_x16(tmem + ((32u * q) << 16) + (uint32_t)(a.rank + c0), s16);   // x . lo
                tmem_ld_wait();
                float v16[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    v16[i] = ok ? __fadd_rn(__uint_as_float(r16[i]), __uint_as_float(s16[i])) : 0.0f;
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4*>(mine + c0 + i) = make_float4(v16[i], v16[i + 1], v16[i + 2], v16[i + 3]);
            }
            if (workspace_mode) {
                // the partials are added in split order, one row and 4 columns
                // per item, consecutive threads on consecutive columns, the
                // loads of up to four splits issued before the first add:
                //  * coop (the whole grid resident at once): once every split
                //    has written its partial, split s adds rows
                //    [128 s / splits, 128 (s + 1) / splits); the last to finish
                //    zeroes the two counters;
                //  * otherwise the last CTA to write its partial adds all rows.
                unsigned int* cnt = a.counters + 2 * rb;   // [0]: partials written, [1]: slices added
                __threadfence();
                named_bar_sync(2, qa::kWorkers);
                if (threadIdx.x == 32 * qa::kWorker0) {
                    const unsigned int prev = atomicAdd(cnt, 1u);
                    if (a.coop) {
                        s_last = qa_wait_count(cnt, (unsigned int)a.splits, kSiteQaSplits) ? 1 : 0;
                        if (!s_last) s_failed = 1;
                    } else {
                        s_last = (prev == (unsigned int)(a.splits - 1)) ? 1 : 0;
                    }
                    __threadfence();
                }
                named_bar_sync(2, qa::kWorkers);
                if (s_last) {
                    const int t = (int)threadIdx.x - 32 * qa::kWorker0;
                    const int q4 = a.rank / 4;
                    const int r_lo = a.coop ? qa::kRows * split / a.splits : 0;
                    const int r_hi = a.coop ? qa::kRows * (split + 1) / a.splits : qa::kRows;
                    const int64_t plane = (int64_t)a.M * a.rank;
                    const float* base = a.partials + (int64_t)rb * a.splits * qa::kRows * a.rank;
                    const int64_t pstep = (int64_t)qa::kRows * a.rank;
                    for (int i = t; i < (r_hi - r_lo) * q4; i += qa::kWorkers) {
                        const int rl = r_lo + i / q4, c0 = 4 * (i % q4);
                        const float* src = base + (int64_t)rl * a.rank + c0;
                        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        for (int p0 = 0; p0 < a.splits; p0 += 4) {
                            float4 f[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                if (p0 + j < a.splits) f[j] = __ldcg(reinterpret_cast<const float4*>(src + (p0 + j) * pstep));
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                if (p0 + j < a.splits) {
                                    acc.x += f[j].x;
                                    acc.y += f[j].y;
                                    acc.z += f[j].z;
                                    acc.w += f[j].w;
                                }
                        }
                        const int64_t grow = (int64_t)m0 + rl;
                        if (grow < a.M) {
                            __nv_bfloat16* hi = a.lowrank + grow * a.rank + c0;
                            store_lowrank_pair(hi, hi + plane, acc.x, acc.y, inv_ss);
                            store_lowrank_pair(hi + 2, hi + 2 + plane, acc.z, acc.w, inv_ss);
                        }
                    }
                    if (t == 0) {
                        if (!a.coop) {
                            cnt[0] = 0u;   // ready for the next call
                        } else if (atomicAdd(cnt + 1, 1u) == (unsigned int)(a.splits - 1)) {
                            // every split has passed its wait: ready for the next call
                            cnt[0] = 0u;
                            cnt[1] = 0u;
                        }
                    }
                }
            }
        }
        if (!workspace_mode) {
            // Add the partials of the cluster (or take this CTA's own) in split
            // order; this CTA stores rows [r_lo, r_hi) of the row block with
            // consecutive threads on consecutive column pairs (coalesced).  The
            // loads from the peers' shared memory are issued before the adds.
            if (cluster_mode)
                cluster_sync_all();
            else
                __syncthreads();
            if (warp >= (uint32_t)qa::kWorker0) {
                const int C = a.cluster;
                const int crank = cluster_mode ? (int)cluster_ctarank() : 0;
                const int r_lo = qa::kRows * crank / C, r_hi = qa::kRows * (crank + 1) / C;
                const int half = a.rank / 2;
                const int items = (r_hi - r_lo) * half;
                const int64_t plane = (int64_t)a.M * a.rank;
                const uint32_t part_u32 = smem_u32(part);
                for (int i = (int)threadIdx.x - 32 * qa::kWorker0; i < items; i += qa::kWorkers) {
                    const int rl = r_lo + i / half, j = i - (i / half) * half;
                    const uint32_t off = (uint32_t)(rl * pstride + 2 * j) * 4u;
                    float2 acc = make_float2(0.0f, 0.0f);
                    if (cluster_mode) {
                        float2 f[qa::kMaxCluster];
#pragma unroll
                        for (int p = 0; p < qa::kMaxCluster; ++p)
                            if (p < C) {
                                uint32_t remote;
                                asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(part_u32 + off), "r"(p));
                                f[p] = ld_cluster_f32x2(remote);
                            }
#pragma unroll
                        for (int p = 0; p < qa::kMaxCluster; ++p)
                            if (p < C) {
                                acc.x += f[p].x;
                                acc.y += f[p].y;
                            }
                    } else {
                        acc = *reinterpret_cast<const float2*>(part + rl * pstride + 2 * j);
                    }
                    const int64_t grow = (int64_t)m0 + rl;
                    if (grow < a.M) {
                        __nv_bfloat16* hi = a.lowrank + grow * a.rank + 2 * j;
                        store_lowrank_pair(hi, hi + plane, acc.x, acc.y, inv_ss);
                    }
                }
            }
            if (cluster_mode) cluster_sync_all();   // peers may still read this CTA's partial
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1 && has_lr) {
        tc_fence_after();
        tmem_dealloc(tmem, a.tmem_cols);
    }
}

}  // namespace svdq
