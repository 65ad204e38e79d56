/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 linear layer.
 *
 * The layer (the `svdq_w4a4` scheme of the Diffusers docs page "Nunchaku Lite",
 * section "Supported quantization types": "NVFP4 runtime kernel with SVDQ
 * low-rank correction", nvfp4 with group 16, or "INT4 W4A4 kernel with SVDQ
 * low-rank correction", int4 with group 64; the SVDQuant paper linked from
 * that page defines the split W . diag(lambda) = L_down . L_up + R):
 *
 *     y = dequant(Q4(x/lambda)) . dequant(Q4(R))^T + ((x/lambda) . L_down) . L_up + b
 *
 * A forward pass is two calls on one stream, with no host synchronisation:
 *     svdq_quantize_act   x -> 4-bit codes + group scales (+ rank-r activations)
 *     svdq_gemm_w4a4      block-scaled 4-bit GEMM + rank-r up-projection + bias
 * The weight side is packed once, offline, by svdq_pack_weight.
 *
 * Conventions for every call below
 *  - Pointers named "device" are device memory of the current CUDA device,
 *    owned by the caller; the library allocates nothing and keeps no state
 *    between calls (except the device status word, see svdq_device_status,
 *    and the zeroed counters of a caller-owned workspace).
 *  - All device pointers must be 16-byte aligned.
 *  - bf16 tensors are row-major with the last dimension contiguous.
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *    Argument errors are returned before anything is launched; a failed
 *    launch returns SVDQ_ERR_CUDA.  A kernel that waits on a barrier for
 *    longer than the wait limit (2 s by default) abandons its work, records
 *    the fact in the device status word, and returns; svdq_device_status()
 *    reports it as SVDQ_ERR_TIMEOUT.
 *  - Sizes: 1 <= M, N and K < 2^31; K % 64 == 0; N % 16 == 0;
 *    rank in {0, 16, 32, ..., 256} (multiples of 16; 0 disables the branch).
 *  - The device must be compute capability 10.0 (B200 class, sm_100a); any
 *    other device is rejected with SVDQ_ERR_UNSUPPORTED_DEVICE before a
 *    launch (the pages' load-time capability check: tutorial page, section
 *    "3. Hardware notes").
 *
 * Packed layouts (owned by this library; svdq_buffer_sizes gives the bytes)
 *  - codes:  [rows, K/2] bytes; element k of a row is in the low nibble of
 *            byte k/2 when k is even, in the high nibble when k is odd.
 *            nvfp4: FP4 E2M1 codes (bit 3 = sign).  int4: two's complement.
 *  - nvfp4 scales: one UE4M3 byte per (row, group of 16), rows padded to a
 *            multiple of 128 with zero bytes, in the tensor-core scale-factor
 *            layout: with Kg4 = K/64, the byte of (row r, group g) is at
 *              ((r/128)*Kg4 + g/4)*512 + (r%32)*16 + ((r%128)/32)*4 + g%4.
 *  - nvfp4 weight scales (w_scales of a packed weight, w_scales_bytes): the
 *            block layout above, then a GEMM-ready copy of the same bytes for
 *            the tensor-memory copy unit: with Nt = ceil(N/256), Kb =
 *            ceil(K/256), unit (t, kb) of 16 KB at (t*Kb + kb)*16384 holds
 *            k-steps 4kb..4kb+3; in k-step k (at k*4096) the 16 bytes of row
 *            l (0..31) of block (2t+h, 4kb+k) sit at
 *            (4q + l/8)*256 + h*128 + (l%8)*16 for every q in 0..3 (the
 *            four 32-lane quarters of tensor memory); blocks past the weight
 *            are zero.  svdq_pack_weight writes both parts.
 *  - int4 scales: one bf16 per (row, group of 64), group-major:
 *            scales[g * rows_pad + r] with rows_pad = rows rounded up to 128
 *            (padding rows are zero).
 *  - tensor scale (nvfp4 only): one fp32 S; a value is code * scale * S.
 *  - hi/lo pairs: an fp32 value v carried as two bf16 planes, hi = bf16(v)
 *            and lo = bf16(v - hi), so that bf16 tensor-core products of both
 *            planes reproduce v to about 2^-17 relative.
 *  - rank-r activations ("lowrank_act"): bf16 [2, M, rank] (hi plane, then lo
 *            plane) of L' where nvfp4 stores L' = ((x/lambda) . L_down) / (S_x S_w)
 *            so the GEMM can add it into the unscaled FP4 accumulator, and int4
 *            stores L' = (x/lambda) . L_down.
 *  - folded weights: inv_lambda fp32 [K] = 1/lambda (IEEE round-to-nearest);
 *            L_down_t bf16 [2, rank, K]: hi/lo pair of fl32(L_down[k,j] / lambda[k]),
 *            transposed; L_up_t bf16 [N, rank] = L_up transposed.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* svdq_stream_t;

typedef enum {
    SVDQ_OK = 0,
    SVDQ_ERR_INVALID_ARG = 1,        /* null pointer, misalignment, bad precision/group/rank */
    SVDQ_ERR_UNSUPPORTED_SHAPE = 2,  /* sizes outside the limits above */
    SVDQ_ERR_UNSUPPORTED_DEVICE = 3, /* no CUDA device, or not compute capability 10.0 */
    SVDQ_ERR_CUDA = 4,               /* a CUDA runtime/driver call or launch failed */
    SVDQ_ERR_TIMEOUT = 5             /* a kernel gave up waiting on a barrier */
} svdq_status;

typedef enum {
    SVDQ_NVFP4 = 0, /* FP4 E2M1 codes, UE4M3 scale per 16, fp32 tensor scale */
    SVDQ_INT4 = 1   /* signed int4 codes, bf16 scale per 64 */
} svdq_precision;

/* Byte sizes of the packed buffers for `rows` rows of K columns. */
typedef struct {
    size_t codes_bytes;    /* rows * K / 2 */
    size_t scales_bytes;   /* nvfp4: rows_pad * K / 16;  int4: 2 * rows_pad * K / 64 */
    size_t lowrank_bytes;  /* 4 * rows * rank (rank-r activations: hi and lo bf16 planes) */
    size_t w_scales_bytes; /* a packed weight's w_scales: int4: scales_bytes; nvfp4: scales_bytes of
                              the block layout, then the GEMM's tile-replicated copy of the same
                              scales, 16 KB per 256 rows x 256 columns (rows and K rounded up to
                              multiples of 256) */
} svdq_sizes;

/* Human-readable name of a status code (static string, never NULL). */
const char* svdq_status_string(svdq_status status);

/* Version of this ABI (increments on any incompatible change). */
int svdq_abi_version(void);

/* Description of the last CUDA failure seen by this thread (the failing call
 * and the CUDA error name), or "" if none; valid until the next failure. */
const char* svdq_last_error(void);

/* Pure host function: fills *out for the given precision and sizes.
 * Errors: INVALID_ARG (out NULL, unknown precision, bad rank),
 *         UNSUPPORTED_SHAPE (rows < 1, K not a multiple of 64). */
svdq_status svdq_buffer_sizes(svdq_precision precision, int64_t rows, int64_t K, int rank, svdq_sizes* out);

/* Offline packing of the weight side (run once per layer).
 *   R          device bf16 [N, K]    residual weight (out x in)
 *   lambda     device fp32 [K]       smoothing divisors, > 0 and finite
 *   L_down     device bf16 [K, rank] (may be NULL when rank == 0)
 *   L_up       device bf16 [rank, N] (may be NULL when rank == 0)
 * Outputs (device, caller-allocated):
 *   w_codes [N, K/2]; w_scales (w_scales_bytes for N rows); w_tensor_scale fp32[1]
 *   (nvfp4: S_w = amax|R| / 2688, or 1 when R == 0; int4: may be NULL);
 *   inv_lambda fp32 [K]; L_down_t bf16 [2, rank, K]; L_up_t bf16 [N, rank].
 * group_size must be 16 for SVDQ_NVFP4 and 64 for SVDQ_INT4. */
svdq_status svdq_pack_weight(svdq_precision precision, int group_size,
                             const void* R, int64_t N, int64_t K,
                             const float* lambda, const void* L_down, const void* L_up, int rank,
                             void* w_codes, void* w_scales, float* w_tensor_scale,
                             float* inv_lambda, void* L_down_t, void* L_up_t,
                             svdq_stream_t stream);

/* Writes the GEMM-ready copy of nvfp4 weight scales (the second part of a
 * packed weight's w_scales, see "nvfp4 weight scales" above) from the block
 * layout in its first scales_bytes bytes.  svdq_pack_weight does this itself;
 * this call is for weight scales produced another way (for example by
 * svdq_quantize_act on the weight) and copied into such a buffer.
 *   w_scales   device, w_scales_bytes for N rows (svdq_buffer_sizes, nvfp4)
 * Errors: INVALID_ARG (NULL or misaligned w_scales), UNSUPPORTED_SHAPE (as
 * svdq_pack_weight), UNSUPPORTED_DEVICE, CUDA. */
svdq_status svdq_replicate_weight_scales(void* w_scales, int64_t N, int64_t K, svdq_stream_t stream);

/* Bytes of the workspace svdq_quantize_act needs for this shape (0 when it
 * needs none).  When K is split across several CTAs, each computes a partial
 * rank-r product.  The CTAs of a 128-row block form one thread-block cluster
 * and add their partials through distributed shared memory when the split
 * fits one cluster (at most 8 CTAs) and all row blocks' clusters can be
 * resident at once; otherwise (on a B200, the M = 4608 layers of a 3072-wide
 * DiT among them) they add them through this workspace: fp32 partial sums
 * plus two counters per 128-row block.  When the whole grid is resident at
 * once (one CTA per SM, no more CTAs than SMs) every CTA of the split adds a
 * slice of the block's rows once all partials are written (a bounded wait
 * on a counter; SVDQ_ERR_TIMEOUT at the wait limit); otherwise the last CTA
 * to write its partial adds them all.  The size returned covers either case;
 * a call that runs in cluster mode leaves the workspace untouched.
 * Pure host function; errors as svdq_buffer_sizes. */
svdq_status svdq_quantize_act_workspace_bytes(svdq_precision precision, int64_t M, int64_t K, int rank,
                                              size_t* bytes);

/* Activation quantizer, fused with the rank-r down-projection.
 *   x              device bf16 [M, K]
 *   inv_lambda     device fp32 [K] (from svdq_pack_weight)
 *   x_tensor_scale device fp32 [1] (nvfp4 only): read as S_x when
 *                  compute_scale == 0 (must be > 0 and finite); when
 *                  compute_scale != 0 it is overwritten with
 *                  S_x = amax|x/lambda| / 2688 (1 when x == 0) first.
 *   w_tensor_scale device fp32 [1] (nvfp4 with rank > 0): S_w
 *   L_down_t       device bf16 [2, rank, K] (NULL when rank == 0)
 *   workspace      device, workspace_bytes long (at least what
 *                  svdq_quantize_act_workspace_bytes reports; NULL when that is
 *                  0).  It must be zero-filled once before its first use; every
 *                  call leaves it zero-filled again.  Calls that share a
 *                  workspace must not overlap on the GPU.  After a call that
 *                  ends in SVDQ_ERR_TIMEOUT, zero-fill it again.
 * Outputs: x_codes [M, K/2]; x_scales (scales_bytes for M rows, padding rows
 *   written as zeros); lowrank_act bf16 [2, M, rank] (NULL when rank == 0). */
svdq_status svdq_quantize_act(svdq_precision precision, int group_size,
                              const void* x, int64_t M, int64_t K, const float* inv_lambda,
                              float* x_tensor_scale, int compute_scale,
                              const float* w_tensor_scale, const void* L_down_t, int rank,
                              void* x_codes, void* x_scales, void* lowrank_act,
                              void* workspace, size_t workspace_bytes,
                              svdq_stream_t stream);

/* svdq_quantize_act for callers that cannot allocate device memory: code
 * that only receives input and output buffers from a host framework and has
 * no device allocator of its own (plug-in or custom-operator interfaces), and
 * code that must keep cudaMalloc / cudaFree, which synchronise the whole
 * device, off a latency-critical path.  (This entry point has no counterpart
 * on the pages; it is a convenience of this library.)
 * Arguments, outputs and errors are those of svdq_quantize_act, without the
 * workspace: the K-split workspace is a library-owned 8 MiB device array
 * (file-scope, so every GPU that loads the library holds it until the process
 * exits).  It is used whenever the split's partials go through global memory
 * (see svdq_quantize_act_workspace_bytes); in cluster mode it is not touched.
 * Shapes whose workspace, as reported by svdq_quantize_act_workspace_bytes,
 * exceeds 8 MiB are rejected with SVDQ_ERR_UNSUPPORTED_SHAPE, and
 * svdq_last_error() says so.
 * The first call on each device (and the first after that device's context
 * was replaced, e.g. by cudaDeviceReset) looks up the array's device address
 * with that device current; make that first call before any stream capture.
 * Each call zero-fills the array's counters on `stream` before its launch.
 * All calls share the one array and it keeps the last call's contents, so
 * calls that overlap on the GPU (other streams or threads) race on it.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine. */
svdq_status svdq_quantize_act_noalloc(svdq_precision precision, int group_size,
                                      const void* x, int64_t M, int64_t K, const float* inv_lambda,
                                      float* x_tensor_scale, int compute_scale,
                                      const float* w_tensor_scale, const void* L_down_t, int rank,
                                      void* x_codes, void* x_scales, void* lowrank_act,
                                      svdq_stream_t stream);

/* The W4A4 GEMM with the rank-r up-projection and bias fused in.
 *   y[m, n] = bf16( S_x S_w sum_k xq[m,k] wq[n,k] + sum_j L[m,j] L_up[j,n] + b[n] )   (nvfp4)
 *   y[m, n] = bf16( sum_g sx[m,g] sw[n,g] sum_{k in g} qx qw + sum_j L[m,j] L_up[j,n] + b[n] )  (int4)
 * Inputs are the outputs of the two calls above; bias is device bf16 [N] or
 * NULL; lowrank_act / L_up_t may be NULL when rank == 0.
 * Output: y device bf16 [M, N].
 * Arithmetic: nvfp4 multiplies the E2M1 codes with their E4M3 group scales on
 * the block-scaled tensor cores (fp32 accumulation); int4 expands each code
 * times its bf16 group scale into fp16 (exact for scales in fp16's normal
 * range) and multiplies fp16 x fp16 with fp32 accumulation.  Both add the
 * rank-r term as bf16 MMAs of the hi and lo parts of L into the same
 * accumulator, then the bias, and round once to bf16. */
svdq_status svdq_gemm_w4a4(svdq_precision precision, int group_size,
                           const void* x_codes, const void* x_scales, const float* x_tensor_scale, int64_t M,
                           const void* w_codes, const void* w_scales, const float* w_tensor_scale,
                           int64_t N, int64_t K,
                           const void* lowrank_act, const void* L_up_t, int rank,
                           const void* bias, void* y, svdq_stream_t stream);

/* The W4A4 GEMM of a fused to_qkv projection with the attention-input
 * RMSNorm and rotary embedding applied in its epilogue (the fused operator of
 * the original Nunchaku engine: the tutorial page's "structural rewrite"
 * passage, one to_qkv projection then norm_q / norm_k per head and
 * apply_rotary_emb; the Diffusers docs page "Nunchaku Lite", section "Fused
 * kernels", "QKV+norm+RoPE" fusion).  nvfp4 only.
 * Arguments up to bias are those of svdq_gemm_w4a4, with N = 3 * heads *
 * head_dim: output columns [0, H D) are Q, [H D, 2 H D) K, [2 H D, 3 H D) V,
 * each head-major.  For every row and every head of Q and K, on the fp32
 * result v of the linear layer (before any bf16 rounding):
 *     v' = v / sqrt(mean(v^2) + eps) * w      (w = norm_q for Q, norm_k for K)
 *     out[2i] = v'[2i] cos[m,i] - v'[2i+1] sin[m,i]
 *     out[2i+1] = v'[2i+1] cos[m,i] + v'[2i] sin[m,i]
 * V is the plain linear output.  y receives bf16(out).
 *   heads      H >= 1;  head_dim must be 128
 *   norm_q, norm_k   device bf16 [head_dim]
 *   eps        0 < eps < 1
 *   rope_cos, rope_sin   device fp32 [M, head_dim / 2]: each token's rotary table
 * Errors: as svdq_gemm_w4a4; INVALID_ARG for int4 or a bad eps;
 * UNSUPPORTED_SHAPE when head_dim != 128 or N != 3 * heads * head_dim. */
svdq_status svdq_gemm_w4a4_qkv_norm_rope(svdq_precision precision, int group_size,
                                         const void* x_codes, const void* x_scales, const float* x_tensor_scale,
                                         int64_t M, const void* w_codes, const void* w_scales,
                                         const float* w_tensor_scale, int64_t N, int64_t K,
                                         const void* lowrank_act, const void* L_up_t, int rank, const void* bias,
                                         int heads, int head_dim, const void* norm_q, const void* norm_k, float eps,
                                         const float* rope_cos, const float* rope_sin, void* y,
                                         svdq_stream_t stream);

/* The same RMSNorm + rotary embedding as a separate pass over a bf16 to_qkv
 * output already in memory (the unfused path: the projection, then this):
 *   y_in, y_out   device bf16 [M, 3 * heads * head_dim]; y_out may equal y_in
 *                 (in place); otherwise the V columns are copied across.
 * Other arguments and errors as svdq_gemm_w4a4_qkv_norm_rope. */
svdq_status svdq_qkv_norm_rope(const void* y_in, void* y_out, int64_t M, int heads, int head_dim,
                               const void* norm_q, const void* norm_k, float eps,
                               const float* rope_cos, const float* rope_sin, svdq_stream_t stream);

/* The fused GELU MLP (the "fused GELU kernel" for the MLP of the original
 * Nunchaku engine; the Diffusers docs page "Nunchaku Lite", section "Fused
 * kernels", GELU-MLP row): the W4A4 GEMM of fc1 whose epilogue applies GELU
 * and performs fc2's activation step itself, so that the [M, N]
 * intermediate is never written:
 *     y  = bf16(fc1 linear output)              (as svdq_gemm_w4a4 computes it)
 *     h  = bf16(GELU(y))                         GELU: gelu_approx 0 = x Phi(x),
 *                                                1 = 0.5 x (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3)))
 *     next_x_codes, next_x_scales = svdq_quantize_act's nvfp4 step on h with
 *                                   fc2's 1/lambda and the static tensor scale S2
 *     next_lowrank_act = (h / lambda2) L_down2 / (S2 S_w2) as a hi/lo bf16 pair
 * after which svdq_gemm_w4a4 with fc2's packed weight and these three
 * buffers (x_tensor_scale = next_x_tensor_scale) computes fc2.  nvfp4 only.
 * Arguments up to bias are fc1's, as in svdq_gemm_w4a4 (N = fc2's K,
 * N % 128 == 0).  fc2's side, from svdq_pack_weight of fc2 and the caller:
 *   next_inv_lambda      device fp32 [N]  (pack output inv_lambda)
 *   next_L_down_t        device bf16 [2, next_rank, N] (pack output L_down_t)
 *   next_rank            0, 16 or 32
 *   next_x_tensor_scale  device fp32 [1]: S2, fc2's static (calibrated) activation
 *                        tensor scale; a dynamic scale needs all of h first
 *   next_w_tensor_scale  device fp32 [1]: fc2's S_w (pack output w_tensor_scale)
 *   next_x_codes, next_x_scales, next_lowrank_act   outputs, sized as
 *                        svdq_buffer_sizes(NVFP4, M, N, next_rank) gives for
 *                        svdq_quantize_act
 *   workspace            device fp32 [M, next_rank] partial sums: zero-filled once
 *                        by the caller; every successful call leaves it zeroed
 *                        (NULL when next_rank == 0)
 * Two kernels on `stream`: the GEMM, then (next_rank > 0) the finalisation of
 * the rank-r sums.  Errors: as svdq_gemm_w4a4; INVALID_ARG for int4, a bad
 * gelu_approx or rank, a short workspace; UNSUPPORTED_SHAPE when N % 128 != 0
 * or next_rank > 32. */
svdq_status svdq_gelu_mlp_workspace_bytes(int64_t M, int next_rank, size_t* bytes);
svdq_status svdq_gemm_w4a4_gelu_quant(svdq_precision precision, int group_size,
                                      const void* x_codes, const void* x_scales, const float* x_tensor_scale,
                                      int64_t M, const void* w_codes, const void* w_scales,
                                      const float* w_tensor_scale, int64_t N, int64_t K,
                                      const void* lowrank_act, const void* L_up_t, int rank, const void* bias,
                                      int gelu_approx, const float* next_inv_lambda, const void* next_L_down_t,
                                      int next_rank, const float* next_x_tensor_scale,
                                      const float* next_w_tensor_scale, void* next_x_codes, void* next_x_scales,
                                      void* next_lowrank_act, void* workspace, size_t workspace_bytes,
                                      svdq_stream_t stream);

/* fc1 of the same MLP with only the GELU in its epilogue (a partial fusion,
 * no counterpart on the pages): y = bf16(GELU(bf16(fc1 linear output))),
 * bit for bit svdq_gelu applied to svdq_gemm_w4a4's y, written to y [M, N]
 * bf16 (device, 16-byte aligned); fc2 then runs svdq_quantize_act on it and
 * svdq_gemm_w4a4.  Arguments as svdq_gemm_w4a4, plus gelu_approx as in
 * svdq_gemm_w4a4_gelu_quant.  nvfp4 only.  One kernel on `stream`.  Errors:
 * as svdq_gemm_w4a4; INVALID_ARG for int4 or a bad gelu_approx;
 * UNSUPPORTED_SHAPE when N % 128 != 0. */
svdq_status svdq_gemm_w4a4_gelu(svdq_precision precision, int group_size,
                                const void* x_codes, const void* x_scales, const float* x_tensor_scale,
                                int64_t M, const void* w_codes, const void* w_scales,
                                const float* w_tensor_scale, int64_t N, int64_t K,
                                const void* lowrank_act, const void* L_up_t, int rank, const void* bias,
                                int gelu_approx, void* y, svdq_stream_t stream);

/* The unfused activation pass of the same MLP: y[i] = bf16(GELU(x[i])) over n
 * finite bf16 elements (device pointers, 16-byte aligned; y may equal x);
 * the same bf16 -> bf16 function the fused epilogue applies, so both paths
 * give fc2 the same h.
 * Errors: INVALID_ARG for a bad pointer or approx; UNSUPPORTED_SHAPE for n < 1. */
svdq_status svdq_gelu(const void* x, void* y, int64_t n, int approx, svdq_stream_t stream);

/* The weight-only int4 GEMM of the `awq_w4a16` scheme (the "INT4 weight-only
 * AWQ-style kernel", int4 with group 64, of the Diffusers docs page "Nunchaku
 * Lite", section "Supported quantization types"; its targets are listed in
 * section "NunchakuLiteQuantizationConfig"):
 *     y[m, n] = bf16( sum_k x[m, k] q[n, k] s[n, k / 64] + b[n] )
 * The activation-aware scaling of AWQ is folded into W (and, inversely, into
 * the layer feeding x) offline; x is used as it comes.
 *   x          device bf16 [M, K] (values of magnitude below 65504)
 *   w_codes, w_scales   the int4 weight as svdq_pack_weight(SVDQ_INT4, 64,
 *              W, N, K, lambda = all ones, rank 0, ...) packs it: two's
 *              complement codes [N, K/2] and bf16 scales [K/64, N_pad]
 *   bias       device bf16 [N] or NULL;  y  device bf16 [M, N]
 * Products q s are exact in fp16; the tensor cores multiply fp16 x fp16 with
 * fp32 accumulation.  Sizes and errors as svdq_gemm_w4a4. */
svdq_status svdq_gemm_w4a16(const void* x, int64_t M, const void* w_codes, const void* w_scales,
                            int64_t N, int64_t K, const void* bias, void* y, svdq_stream_t stream);

/* Offline split of a layer's weight into the low-rank branch and the residual
 * that svdq_pack_weight quantizes (the SVDQuant decomposition the Diffusers
 * docs page "Nunchaku Lite" builds on; the tutorial's offline quantization
 * step, quantize_hf.py --rank 32):
 *     W_hat = W diag(lambda) = L_up^T L_down^T + R
 * with L_up^T L_down^T the best rank-r approximation of W_hat, computed by a
 * randomized range finder with `power_iters` steps of subspace iteration
 * (Halko, Martinsson and Tropp 2011) and R the residual with the bf16
 * factors.  Then x W^T = (x / lambda) R^T + ((x / lambda) L_down) L_up: pass
 * R, lambda, L_down and L_up to svdq_pack_weight.
 *   W        device bf16 [N, K] (out x in)
 *   lambda   device fp32 [K] smoothing divisors (> 0)
 *   omega    device fp32 [K, rank + oversample]: a Gaussian test matrix, drawn
 *            by the caller (for example N(0, 1) entries)
 *   rank     1 <= rank <= min(N, K), rank + oversample <= 64
 *   power_iters  0..16 (2 is ample when the spectrum decays past rank)
 * Outputs (device, caller-allocated): R bf16 [N, K]; L_down bf16 [K, rank];
 *   L_up bf16 [rank, N]; singular_values fp32 [rank + oversample] (the
 *   approximations of the largest singular values of W_hat, decreasing) or NULL.
 * workspace: device, at least svdq_svd_split_workspace_bytes() bytes.
 * An offline step: simple kernels, not tuned for speed. */
svdq_status svdq_svd_split_workspace_bytes(int64_t N, int64_t K, int rank, int oversample, size_t* bytes);
svdq_status svdq_svd_split(const void* W, const float* lambda, int64_t N, int64_t K, int rank,
                           const float* omega, int oversample, int power_iters,
                           void* R, void* L_down, void* L_up, float* singular_values,
                           void* workspace, size_t workspace_bytes, svdq_stream_t stream);

/* Synchronises the current device, then reads the device status word.
 * Returns SVDQ_OK, SVDQ_ERR_TIMEOUT (a kernel abandoned a wait; *site, if not
 * NULL, receives the id of the first wait that did) or SVDQ_ERR_CUDA.
 * clear != 0 resets the word afterwards. */
svdq_status svdq_device_status(int clear, int* site);

/* Test hooks (not for production use).
 *  svdq_debug_set_wait_limit_ns: changes the barrier wait limit (0 restores 2 s).
 *  svdq_debug_timeout_probe: launches one small kernel that waits on a barrier
 *    nothing ever completes, so it must give up after the wait limit; the
 *    status word then reads SVDQ_ERR_TIMEOUT.  Used to test failure detection.
 *  svdq_debug_override_capability: pretend the device has compute capability
 *    major.minor (major = -1 removes the override), to test the device check.
 *  svdq_debug_force_gemm_tiles: choose the nvfp4 GEMM kernel: 0 = automatic
 *    (M <= 128: 128 x 256 tiles on single CTAs; M > 128: CTA-pair tiles),
 *    1 = always single CTAs, 2 = always CTA pairs.  Both kernels compute the
 *    same y; this exists so that tests can run each on the same inputs.  Any
 *    other value is SVDQ_ERR_INVALID_ARG. */
svdq_status svdq_debug_set_wait_limit_ns(uint64_t ns);
/* svdq_debug_force_quant_plan: how svdq_quantize_act adds the rank-r partials
 *    of a K split: 0 = automatic, 1 = always through the workspace (global
 *    memory, see svdq_quantize_act_workspace_bytes; every split adds a slice
 *    when the grid is resident at once), 2 = always in one thread-block
 *    cluster through distributed shared memory, 3 = through the workspace
 *    with the last CTA of a row block adding all of its rows (what a device
 *    with fewer SMs than the grid's CTAs gets).  Results are the same; tests
 *    use it to run every path.  Any other value is SVDQ_ERR_INVALID_ARG. */
svdq_status svdq_debug_force_quant_plan(int mode);
svdq_status svdq_debug_timeout_probe(svdq_stream_t stream);
void svdq_debug_override_capability(int major, int minor);
svdq_status svdq_debug_force_gemm_tiles(int mode);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
