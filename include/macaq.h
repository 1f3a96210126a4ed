/*
 * macaq.h -- C ABI of libmacaq.so: the W4A4 / MXFP4 linear layer of MACaQ on NVIDIA B200 (sm_100a).
 *
 * The method. Page "Huawei's research lab in Switzerland open-sources the four-bit quantization tool
 * MACaQ for running models locally" (aipolix.com, Persian), paragraph 2: at inference every layer's
 * activations receive a per-channel scale and a small block-diagonal Hadamard transform, and the
 * inverse is absorbed into the same layer's weights; paragraph 3: the target format is MXFP4 with
 * 4-bit weights and activations (W4A4). Page "MACaQ quantizer from huawei-csl targets GGUF, vLLM and
 * Diffusers models" (glonce.com), paragraph 5: the W4A4 dense and grouped matmuls. The MXFP4 rule is
 * OCP Microscaling Formats (MX) v1.0: E2M1 elements, one E8M0 scale 2^(floor(log2 amax) - 2) per 32
 * contiguous K elements, round-to-nearest-even, saturation at +-6.
 *
 * Concretely, with H_b the Sylvester Hadamard matrix of order b (entries +-1, natural order) applied
 * to each aligned block of b input channels:
 *     weights (offline):  W'  = MXFP4( W * diag(s) * H_b * (1/b) )
 *     activations:        X'  = MXFP4( X * diag(1/s) * H_b )
 *     output:             Y   = X' * W'^T   (fp32 accumulation, bf16 or fp32 result)
 * so that Y approximates X * W^T (H_b * H_b^T = b * I). b = 1 means "no Hadamard" and a NULL scale
 * means s = 1: together they give the plain-MXFP4 pipeline the overhead figure is measured against.
 *
 * Notation: M rows (tokens), K input channels, N output channels. All matrices are row-major.
 *
 * Data layouts (all buffers are device memory unless stated otherwise):
 *   bf16 matrices        [rows, K], 2 bytes per element.
 *   FP4 codes            [rows, K/2] bytes; element k of a row is nibble (k & 1) of byte k/2
 *                        (even k in the low nibble); code = sign<<3 | E2M1 magnitude code.
 *   scale factors (SF)   one E8M0 byte per 32 K-elements, stored in the tcgen05 block-scale tiling:
 *                        rows are padded to a multiple of 128 and cut into 128 x 4 tiles (128 rows, 4
 *                        scale columns = 128 K-elements); tiles are ordered row-tile-major, then by
 *                        K-tile; inside a tile, row r and column c sit at byte
 *                        (r % 32) * 16 + (r / 32) * 4 + c. Padding rows hold 0.
 *                        Size: macaq_sf_bytes(rows, K).
 *   grouped SF           the same tiling, but each expert's rows start on a fresh 128-row tile:
 *                        expert e occupies row tiles [sum_{e'<e} ceil(M_e'/128), ...).
 *                        Size bound: macaq_grouped_sf_bytes(total_rows, E, K).
 *
 * Conventions:
 *   - The caller allocates and owns every buffer. The library never allocates device memory,
 *     never frees it, and never synchronizes the device or the stream.
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and returns a status. A launch failure returns MACAQ_ERR_CUDA (the cudaGetLastError code is
 *     kept and can be read with macaq_last_cuda_error()). No exception crosses the ABI.
 *   - Shape rules: K % 128 == 0 (whole 128 x 4 scale tiles); N % 128 == 0; M >= 0 (M == 0 is a
 *     no-op); had_block in {1, 16, 32, 64, 128}. Every pointer argument must be 16-byte aligned.
 *     Violations return MACAQ_ERR_SHAPE / MACAQ_ERR_ALIGNMENT / MACAQ_ERR_UNSUPPORTED /
 *     MACAQ_ERR_INVALID_ARG before anything is launched.
 *   - Device-side waits (pipeline barriers inside the GEMM) are bounded. A wait that runs out sets a
 *     sticky device status word and the kernel returns without finishing; macaq_device_status()
 *     reads that word (MACAQ_ERR_TIMEOUT) after the caller synchronizes.
 *   - Calls are thread-safe; host-side tensor-map descriptors are cached under a mutex.
 */
#ifndef MACAQ_H
#define MACAQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MACAQ_OK = 0,
    MACAQ_ERR_INVALID_ARG = 1, /* NULL where a buffer is required, unknown enum value */
    MACAQ_ERR_SHAPE = 2,       /* a dimension breaks the shape rules above */
    MACAQ_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned */
    MACAQ_ERR_UNSUPPORTED = 4, /* had_block not supported, or the device is not sm_100 */
    MACAQ_ERR_CUDA = 5,        /* a CUDA runtime or driver call failed */
    MACAQ_ERR_TIMEOUT = 6,     /* a bounded device-side wait ran out (see macaq_device_status) */
    MACAQ_ERR_WORKSPACE = 7    /* workspace missing or smaller than macaq_workspace_bytes() */
} macaq_status;

typedef enum { MACAQ_OUT_BF16 = 0, MACAQ_OUT_F32 = 1 } macaq_out_dtype;

/* How operand A of the GEMM is given: already quantized (codes + SF from macaq_act_quant), or as
 * bf16 activations that the GEMM transforms and quantizes itself (the fused variant). */
typedef enum { MACAQ_A_QUANTIZED = 0, MACAQ_A_BF16_FUSED = 1, MACAQ_A_BF16_ONE_LAUNCH = 2 } macaq_a_mode;

/* A cudaStream_t, passed as a plain pointer so that this header needs no CUDA include. */
typedef void *macaq_stream_t;

/* Human-readable name of a status code (static storage, never NULL). */
const char *macaq_status_str(int status);

/* The cudaError_t of the most recent failing CUDA call made by this library on this thread. */
int macaq_last_cuda_error(void);

/* Bytes of the tiled scale-factor buffer for `rows` rows of K elements:
 * ceil(rows / 128) * 128 * (K / 32). 0 for rows <= 0 or K not a multiple of 128. */
size_t macaq_sf_bytes(int64_t rows, int64_t K);

/* Upper bound of the grouped scale-factor buffer: (ceil(total_rows / 128) + E) * 128 * (K / 32).
 * Every expert's rows start on a fresh 128-row tile, so at most E extra tiles are needed. */
size_t macaq_grouped_sf_bytes(int64_t total_rows, int32_t E, int64_t K);

/* Workspace bytes macaq_linear can use for these sizes on the current device (E = 0 for dense).
 * Dense calls with M <= 128 and K % 256 == 0 given a workspace of at least this size run the skinny
 * kernel (weights in the MMA's 128-row slot, the unit space split evenly over all SMs, split tiles
 * reduced through the workspace); without a workspace they run the general kernel. 0 means no
 * workspace is used.
 * Layout and contract: the first MACAQ_WORKSPACE_COUNTER_BYTES hold per-tile arrival counters. They
 * must be zero before the workspace's first use, and every call leaves them zero again (each counter
 * is reset by the CTA that consumed it), so one buffer serves any number of consecutive calls of any
 * shapes. The bytes after them are scratch: no initial value is needed and calls leave arbitrary
 * data there. Calls that may run at the same time on different streams need separate workspaces.
 * After a call that reported MACAQ_ERR_TIMEOUT, zero the counter region again. */
#define MACAQ_WORKSPACE_COUNTER_BYTES ((size_t)65536)
size_t macaq_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t E);

/* Workspace bytes of the fused mode (MACAQ_A_BF16_FUSED) of macaq_linear (E = 0) and
 * macaq_grouped_linear (E experts): the region above, then room for the quantized activations and
 * their scale factors where the call quantizes X in a separate pass. Same layout and contract. */
size_t macaq_fused_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t E);

/*
 * Offline weight preparation (the absorbed inverse transform).
 * Computes, per weight row and per aligned block of had_block channels, in fp32:
 *     v = fl32(W[n,k] * s[k]);  v = v * H_b (fixed butterfly order h = 1, 2, ..., b/2);  v *= 1/b;
 * then MXFP4 per 32 channels; also inv_s[k] = fl32(1 / s[k]) (IEEE division) for the activations.
 *   W       device bf16 [N, K] (read)
 *   s       device fp32 [K] per-channel scale, > 0 (read); NULL means s = 1 (then inv_s is untouched)
 *   Wq      device u8 [N, K/2] (written)
 *   Wsf     device u8, macaq_sf_bytes(N, K) bytes, tiled layout (written, padding rows zeroed)
 *   inv_s   device fp32 [K] (written when s != NULL; may be NULL to skip)
 * Source: the aipolix.com page, paragraph 2 (absorb the inverse into the same layer's weights).
 */
macaq_status macaq_prep_weights(const void *W, const float *s, int64_t N, int64_t K, int32_t had_block,
                                uint8_t *Wq, uint8_t *Wsf, float *inv_s, macaq_stream_t stream);

/*
 * Online activation quantization: Xq/Xsf = MXFP4( X * diag(inv_s) * H_b ), in fp32 with the same
 * fixed butterfly order, then OCP MX v1.0 quantization per 32 channels.
 *   X              device bf16 [M, K] (read)
 *   inv_s          device fp32 [K] (dense) or [E, K] (grouped); NULL means 1
 *   group_offsets  NULL for a dense call; else device int32 [E + 1] (1 <= E <= 16384),
 *                  non-decreasing, offsets[0] = 0,
 *                  offsets[E] = M: rows [offsets[e], offsets[e+1]) belong to expert e and use
 *                  inv_s + e*K. The values are read on the device; out-of-range offsets are clamped
 *                  into [0, M] so no access leaves the buffers, but give undefined results. A caller
 *                  that holds a host copy can reject such offsets first with
 *                  macaq_check_group_offsets().
 *   Xq             device u8 [M, K/2] (written)
 *   Xsf            device u8 (written): dense: macaq_sf_bytes(M, K) bytes; grouped: the per-expert
 *                  padded tiling, at most macaq_grouped_sf_bytes(M, E, K) bytes. Padding rows get 0.
 * Sources: aipolix.com page, paragraph 2 (per-channel scale and block Hadamard at inference) and
 * paragraph 3 (MXFP4); glonce.com page, paragraph 5 (grouped matmul).
 */
macaq_status macaq_act_quant(const void *X, const float *inv_s, int64_t M, int64_t K, int32_t had_block,
                             const int32_t *group_offsets, int32_t E, uint8_t *Xq, uint8_t *Xsf,
                             macaq_stream_t stream);

/*
 * The weight-only mode's activation transform: Xt = bf16( X * diag(inv_s) * H_b ), the act_quant
 * arithmetic (fp32 multiply, fixed-order butterflies) with each value rounded once to bf16 (nearest
 * even) instead of MXFP4.
 *   X device bf16 [M, K] (read); inv_s device fp32 [K] or NULL; had_block b; Xt device bf16 [M, K]
 *   (written). K % 128 == 0.
 * Sources: glonce.com page, paragraph 3 (vLLM serves W4A4 or weight-only checkpoints); aipolix.com
 * page, paragraph 2 (the transform at the input of every linear).
 */
macaq_status macaq_act_transform(const void *X, const float *inv_s, int64_t M, int64_t K, int32_t had_block, void *Xt,
                                 macaq_stream_t stream);

/*
 * Weight-only (W4A16) linear for decode and small batches:
 *     Y[m, n] = sum_k bf16(X'[m, k]) * dq(W'[n, k]),  X' = X * diag(inv_s) * H_b (macaq_act_transform)
 * with the weights prepared by macaq_prep_weights exactly as for W4A4 (codes + tiled SF) and fp32
 * accumulation on the tensor cores (kind::f16, bf16 x bf16): the weight codes are expanded to bf16
 * inside the kernel (exact for scales E8M0 <= 252) and never written to memory.
 *   X           device bf16 [M, K], 1 <= M <= 64 (M == 0 is a no-op; larger M: MACAQ_ERR_SHAPE);
 *               K % 256 == 0; N % 128 == 0
 *   inv_s, had_block  as for macaq_act_quant; Wq, Wsf as for macaq_linear
 *   Y           device [M, N], bf16 or fp32 per out_dtype (written)
 *   workspace   at least macaq_linear_w4a16_workspace_bytes(M, N, K) bytes (the transformed
 *               activations and the split-tile scratch), under the contract of macaq_workspace_bytes
 * Source: glonce.com page, paragraph 3 (weight-only mode).
 */
size_t macaq_linear_w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K);
macaq_status macaq_linear_w4a16(const void *X, const float *inv_s, int64_t M, int64_t N, int64_t K, int32_t had_block,
                                const uint8_t *Wq, const uint8_t *Wsf, void *Y, int32_t out_dtype, void *workspace,
                                size_t ws_bytes, macaq_stream_t stream);

/*
 * Flip-Refinement of prepared weights (offline): a coordinate descent over single FP4 codes, guided by
 * the layer's Hessian, with the E8M0 scales fixed. Per weight row, with w the row's transformed fp32
 * weights (exactly as macaq_prep_weights computes them from W, s and had_block) and w_hat the codes'
 * values, it lowers L = (w_hat - w)^T H (w_hat - w):
 *   g = H (w_hat - w) in float64 (g[i] = sum over k = 0..K-1 in order of H[k][i] (w_hat[k] - w[k]));
 *   `sweeps` times, for k = 0 .. K-1: try the two neighbouring values on the signed E2M1 grid
 *   {-6, ..., -0.5, 0, 0.5, ..., 6} at the group's scale, the lower first; a move by d changes L by
 *   d (2 g[k] + d H[k][k]); the better one (the upper only if strictly better) is taken if that is
 *   negative, then g[i] += d H[k][i] for all i. Every step is one float64 operation in this order.
 *   W       device bf16 [N, K] (read), s device fp32 [K] or NULL, had_block as at preparation
 *   H       device fp32 [K, K], symmetric (e.g. X'^T X' of calibration inputs transformed as for
 *           macaq_act_quant); row-major
 *   sweeps  >= 0 (0: no-op)
 *   Wq      device u8 [N, K/2]: the prepared codes on entry, the refined codes on return
 *   Wsf     device u8 tiled SF of the N rows from macaq_prep_weights (read, unchanged)
 *   flips   device int32 [N] (written: accepted moves per row) or NULL; 4-byte aligned
 *   K % 128 == 0 and K <= 16384 (the per-row state lives in shared memory).
 * Source: aipolix.com page, paragraph 3 (Flip-Refinement: a Hessian-guided coordinate descent moving
 * single FP4 codes to neighbouring representable values). The objective and the visiting order are
 * this library's plain reading; the page gives no formula.
 */
macaq_status macaq_flip_refine(const void *W, const float *s, int64_t N, int64_t K, int32_t had_block, const float *H,
                               int32_t sweeps, uint8_t *Wq, const uint8_t *Wsf, int32_t *flips, macaq_stream_t stream);

/*
 * Activation quantization with a row gather, the dispatch step of a mixture-of-experts layer: output
 * row m is MXFP4( X[row_index[m]] * diag(inv_s) * H_b ), bit-identical to macaq_act_quant applied
 * to the gathered copy X[row_index], which is never written to memory.
 *   X              device bf16 [x_rows, K] (read), e.g. the hidden states in token order
 *   x_rows         rows of X (>= 1 when M > 0)
 *   row_index      device int32 [M] (16-byte aligned): the X row of every output row, e.g. the token
 *                  of each routed row sorted by expert. Values outside [0, x_rows) are clamped into
 *                  it, so no access leaves X; such a row gets the clamped row's result.
 *   inv_s, M, K, had_block, group_offsets, E, Xq, Xsf: as for macaq_act_quant, over the M output rows.
 * Sources: as macaq_act_quant; glonce.com page, paragraph 5 (grouped matmul).
 */
macaq_status macaq_act_quant_gather(const void *X, int64_t x_rows, const int32_t *row_index, const float *inv_s,
                                    int64_t M, int64_t K, int32_t had_block, const int32_t *group_offsets, int32_t E,
                                    uint8_t *Xq, uint8_t *Xsf, macaq_stream_t stream);

/*
 * Weighted top-k combine after the down projection of a mixture-of-experts layer:
 *     out[t, n] = sum over j = 0 .. topk-1 of fl32( weights[t, j] * Y[pos[t, j], n] )
 * accumulated in fp32 in the order j = 0, 1, ... from +0, every product and every sum rounded on its
 * own (no multiply-add); bf16 output is the round-to-nearest-even cast of that fp32 value.
 *   Y        device bf16 [y_rows, N] (read): a grouped linear's output, rows in expert-sorted order
 *   pos      device int32 [T, topk] (4-byte aligned): the Y row of token t's j-th expert choice;
 *            values outside [0, y_rows) contribute nothing (a dropped choice)
 *   weights  device fp32 [T, topk] (4-byte aligned): the router weights
 *   out      device [T, N] (written), bf16 or fp32 per out_dtype
 *   N % 8 == 0, 1 <= topk <= 1024, T >= 0 (T == 0 is a no-op); Y and out 16-byte aligned.
 * Source: glonce.com page, paragraph 5 (grouped matmul); the combine returns the grouped GEMM's rows
 * to token order.
 */
macaq_status macaq_moe_combine(const void *Y, int64_t y_rows, int64_t N, const int32_t *pos, const float *weights,
                               int64_t T, int32_t topk, void *out, int32_t out_dtype, macaq_stream_t stream);

/*
 * Dense W4A4 linear: Y[m, n] = sum_k dq(A[m, k]) * dq(W'[n, k]), fp32 accumulation on the tcgen05
 * tensor cores (kind::mxf4 block-scaled MMA), written as bf16 (round-to-nearest-even) or fp32.
 *   mode == MACAQ_A_QUANTIZED:  A = Xq device u8 [M, K/2], Asf = Xsf (tiled, macaq_sf_bytes(M, K)),
 *                               inv_s and had_block are ignored.
 *   mode == MACAQ_A_BF16_FUSED: A = X device bf16 [M, K], inv_s device fp32 [K] (NULL = 1), had_block
 *                               b in {1, 16, 32, 64, 128}; Asf is ignored. The call quantizes X
 *                               bit-identically to macaq_act_quant, so Y equals macaq_act_quant
 *                               followed by the quantized mode. M <= 4 with K % 256 == 0: inside the
 *                               skinny kernel (quantizer warps write the MMA's operand stages; no
 *                               quantized activation in HBM). Otherwise: a quantizer pass into the
 *                               workspace, then the GEMM, in stream order. Needs a workspace of
 *                               macaq_fused_workspace_bytes(M, N, K, 0) bytes (else MACAQ_ERR_WORKSPACE).
 *   mode == MACAQ_A_BF16_ONE_LAUNCH: as MACAQ_A_BF16_FUSED (same arguments, workspace and result),
 *                               but M > 128 with N % 256 == 0 and K % 256 == 0 runs as ONE launch: the
 *                               2-SM GEMM's epilogue warps quantize X into the workspace between tiles
 *                               and its producers wait (bounded) on per-block ready counts before
 *                               loading A. On B200 this form measures slower than the two launches
 *                               (the epilogue warps quantize at about half the quantizer kernel's
 *                               rate, and the first tiles wait for them), which is why it is not the
 *                               default; other shapes behave exactly as MACAQ_A_BF16_FUSED.
 *   Wq, Wsf    from macaq_prep_weights: u8 [N, K/2] and the tiled SF of N rows
 *   Y          device [M, N], bf16 or fp32 per out_dtype (written)
 *   workspace  NULL, or device scratch of at least macaq_workspace_bytes(M, N, K, 0) bytes under the
 *              contract above (selects the skinny kernel for M <= 128 and K % 256 == 0; too small:
 *              MACAQ_ERR_WORKSPACE)
 * Source: glonce.com page, paragraph 5 (W4A4 dense matmul).
 */
macaq_status macaq_linear(int32_t mode, const void *A, const uint8_t *Asf, const float *inv_s, int64_t M,
                          int64_t N, int64_t K, int32_t had_block, const uint8_t *Wq, const uint8_t *Wsf,
                          void *Y, int32_t out_dtype, void *workspace, size_t ws_bytes,
                          macaq_stream_t stream);

/* Size of the library's own fixed scratch area used by macaq_linear_fixed_scratch (8 MiB). */
#define MACAQ_FIXED_SCRATCH_BYTES ((size_t)8 << 20)

/*
 * macaq_linear without a caller-supplied workspace and without allocating device memory.
 * The method on the pages has no counterpart of this call: it exists for callers that cannot
 * allocate device memory at call time, such as a host that has handed all device memory to its
 * own pool, an embedding in a C program without a device allocator, or a serving loop in which an
 * allocation would synchronize the device and stall the other streams.
 * Arguments, results and errors are those of macaq_linear without workspace/ws_bytes. Dense calls
 * with M <= 128 and K % 256 == 0 run the skinny kernel on a scratch area that lives in the
 * library's static device data (MACAQ_FIXED_SCRATCH_BYTES per device); every other shape runs the
 * general kernels, which need no scratch.
 *   - Every call looks the scratch's device address up on the current device (a host-side table
 *     lookup once the module is loaded; nothing is cached, so a device reset does no harm). The
 *     first call on a device may load the module: make that first call before any stream capture.
 *   - Sizes whose skinny plan needs more than MACAQ_FIXED_SCRATCH_BYTES (what
 *     macaq_workspace_bytes(M, N, K, 0) reports) are rejected with MACAQ_ERR_WORKSPACE before
 *     anything is launched.
 *   - Only the per-tile counters must start at zero; each call clears the ones it uses on `stream`
 *     (a memset of 4 bytes per 128-row weight tile, rounded up to 256 bytes) right before its kernel,
 *     after every argument check, so a refused call enqueues nothing and a call after a
 *     MACAQ_ERR_TIMEOUT needs no clean-up.
 *   - All calls on one device share the one scratch area: two calls whose kernels may overlap
 *     (different streams, or different host threads without ordering) race and give wrong results.
 *     Order them on one stream, or use macaq_linear with separate workspaces.
 */
macaq_status macaq_linear_fixed_scratch(int32_t mode, const void *A, const uint8_t *Asf, const float *inv_s,
                                        int64_t M, int64_t N, int64_t K, int32_t had_block, const uint8_t *Wq,
                                        const uint8_t *Wsf, void *Y, int32_t out_dtype, macaq_stream_t stream);

/*
 * Gate/up linear of a SwiGLU MLP with the down projection's activation quantization fused after it:
 *     G, U = X' * W'_gu^T            (the block-scaled GEMM, fp32 accumulation)
 *     H    = silu(G) * U             (fp32; silu(g) = g / (1 + exp(-g)) with one fixed fp32 exp)
 *     Hq, Hsf = MXFP4( H * diag(inv_s_down) * H_b )    (the macaq_act_quant arithmetic)
 * so that Hq/Hsf are the A operand of the down projection's macaq_linear. The fixed exp is Cody and
 * Waite's reduction n = rint(x log2 e), r = (x - n C1) - n C2 (C1 = 0x3F317200, C2 = 0x35BFBE8E as
 * fp32 bit patterns), the Taylor polynomial sum_{k=0..6} r^k / k! by Horner's rule, times 2^n, x
 * clamped to [-100, 88], each step one round-to-nearest fp32 operation with no multiply-add.
 *   A, Asf      the gate/up input, quantized (macaq_act_quant) as for macaq_linear: u8 [M, K/2] + SF
 *   N           2 * I, a multiple of 256 (I intermediate channels)
 *   Wq, Wsf     the gate/up weights prepared by macaq_prep_weights from one [N, K] matrix whose rows
 *               interleave the two projections in blocks of 64: gate rows 64j..64j+63, then up rows
 *               64j..64j+63, for j = 0 .. I/64 - 1
 *   inv_s_down  device fp32 [I]: the down projection's 1/s (from its macaq_prep_weights), or NULL
 *   had_block_down  the down projection's Hadamard block, in {1, 16, 32, 64}
 *   Hq          device u8 [M, I/2] (written); Hsf device u8, macaq_sf_bytes(M, I) (written, padding 0)
 *   workspace   M > 128 with K % 256 == 0: unused (the GEMM's epilogue does the rest; G and U never
 *               reach memory); otherwise at least macaq_linear_swiglu_workspace_bytes(M, N, K) bytes
 *               (the GEMM writes G, U in fp32 there, then macaq_swiglu_act_quant's kernel runs), under
 *               the workspace contract of macaq_workspace_bytes.
 * Sources: aipolix.com page, paragraph 2 (the transform at the input of every linear); glonce.com
 * page, paragraph 5 (W4A4 dense matmul). The pages do not define the MLP's activation: the fp32
 * evaluation above is this library's definition.
 */
size_t macaq_linear_swiglu_workspace_bytes(int64_t M, int64_t N, int64_t K);
macaq_status macaq_linear_swiglu(const uint8_t *A, const uint8_t *Asf, int64_t M, int64_t N, int64_t K,
                                 const uint8_t *Wq, const uint8_t *Wsf, const float *inv_s_down, int32_t had_block_down,
                                 uint8_t *Hq, uint8_t *Hsf, void *workspace, size_t ws_bytes, macaq_stream_t stream);

/*
 * The second half of macaq_linear_swiglu on a gate/up output already in memory:
 *   GU      device fp32 [M, 2I], columns interleaved in blocks of 64 (gate 64j.., then up 64j..)
 *   I       a multiple of 128; inv_s [I] or NULL; had_block in {1, 16, 32, 64}
 *   Hq, Hsf as for macaq_linear_swiglu.
 */
macaq_status macaq_swiglu_act_quant(const float *GU, int64_t M, int64_t I, const float *inv_s, int32_t had_block,
                                    uint8_t *Hq, uint8_t *Hsf, macaq_stream_t stream);

/*
 * Grouped (MoE) W4A4 linear: rows [offsets[e], offsets[e+1]) of A are multiplied by expert e's
 * weights.
 *   mode == MACAQ_A_QUANTIZED:  A, Asf = Xq [total_rows, K/2] and the grouped tiled SF from
 *                               macaq_act_quant in grouped form; inv_s and had_block are ignored.
 *   mode == MACAQ_A_BF16_FUSED: A = X device bf16 [total_rows, K], inv_s device fp32 [E, K] (NULL = 1),
 *                               had_block b; the call runs the grouped quantizer into the workspace
 *                               (macaq_fused_workspace_bytes(total_rows, N, K, E) bytes), then the
 *                               grouped GEMM. Asf is ignored.
 *   group_offsets  device int32 [E + 1] (as for macaq_act_quant); 1 <= E <= 1024
 *   Wq             device u8 [E, N, K/2];  Wsf device u8 [E, macaq_sf_bytes(N, K)]
 *   Y              device [total_rows, N] (written; only rows of some expert are written)
 *   workspace      quantized mode: unused (may be NULL); fused mode: as above
 * With N and K multiples of 256 and total_rows >= 256 * E (experts averaging at least 256 rows) the
 * GEMM runs on 2-SM pairs (tiles of 256 rows of one expert); otherwise one CTA per 128-row tile.
 * MACAQ_A_BF16_ONE_LAUNCH is accepted and behaves as MACAQ_A_BF16_FUSED.
 * Source: glonce.com page, paragraph 5 (W4A4 grouped matmul).
 */
macaq_status macaq_grouped_linear(int32_t mode, const void *A, const uint8_t *Asf, const float *inv_s,
                                  const int32_t *group_offsets, int32_t E, int64_t total_rows, int64_t N,
                                  int64_t K, int32_t had_block, const uint8_t *Wq, const uint8_t *Wsf,
                                  void *Y, int32_t out_dtype, void *workspace, size_t ws_bytes,
                                  macaq_stream_t stream);

/*
 * Host-side check of grouped row offsets (no CUDA call): host_offsets[0..E] must start at 0, end at
 * total_rows and never decrease, with 1 <= E <= 16384. Returns MACAQ_OK, MACAQ_ERR_SHAPE for offsets
 * that break a rule, or MACAQ_ERR_INVALID_ARG for a NULL pointer. The device-side reads of the same
 * offsets (macaq_act_quant, macaq_grouped_linear) clamp instead of failing, because a kernel cannot
 * return an error before it has read them.
 */
macaq_status macaq_check_group_offsets(const int32_t *host_offsets, int32_t E, int64_t total_rows);

/*
 * Reads the sticky device status word that bounded device waits set when they run out. Call it
 * after synchronizing the stream(s) that ran the kernels. *status_out = MACAQ_OK or
 * MACAQ_ERR_TIMEOUT. reset != 0 clears the word afterwards. Uses the current CUDA device.
 * The wait limit can be lowered for tests with macaq_set_wait_limit_ns().
 */
macaq_status macaq_device_status(int32_t *status_out, int32_t reset);

/* Sets the time limit of every bounded device-side wait launched after this call (nanoseconds;
 * 0 restores the default of 2 s). Process-wide. */
void macaq_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* MACAQ_H */
