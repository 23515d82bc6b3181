/*
 * moe_qmm.h -- C ABI of the expert-routed (MoE) quantized matmul for NVIDIA B200 (sm_100a).
 *
 * The operation (mlx-native 0.1.0, src/ops/quantized_matmul_id.rs, module
 * documentation): for every (token, slot) pair p = token * n_expert_used + slot,
 *
 *     e = ids[p]
 *     out[token][slot][col] = sum_{j<k} dequant(W[e][col][j]) * x[token][j]
 *
 * Parameters follow that page's QuantizedMatmulIdParams {m, k, n, group_size,
 * bits, n_expert_used, num_experts}; storage formats, types and the extra
 * arguments (x / out types, workspace, stream) are appended after them.
 *
 * Conventions shared by every entry point:
 *   * All array arguments are DEVICE pointers owned by the caller. The library
 *     allocates and frees nothing.
 *   * Work is enqueued on `stream` and nothing synchronises (the page's encoder
 *     "does not commit the command buffer"; the caller orders and waits).
 *   * Scalar validation happens before any CUDA call; a rejected call returns
 *     MOE_ERR_INVALID_ARGUMENT (invalid per the page's rules: bits outside the
 *     format's set, any zero m/k/n/group_size/n_expert_used/num_experts, a NULL
 *     pointer, NVFP4 with group_size != 16 or odd k) or MOE_ERR_UNSUPPORTED
 *     (valid but not implemented: k % group_size != 0, or sizes beyond the
 *     documented limits) and enqueues nothing.
 *   * Expert ids >= num_experts are not an argument error: the output row of
 *     such a pair is written as zeros and a bit is set in the device error word
 *     held in the workspace, which moe_qmm_id_poll_error() reads and clears.
 *   * A launch failure returns MOE_ERR_CUDA.
 *
 * Storage (all rows of expert e are contiguous; row (e, col) starts at byte
 * (e * n + col) * moe_packed_row_bytes(fmt, bits, k)):
 *   MOE_FMT_AFFINE   bits 4 / 8: 32/bits codes per little-endian u32 word,
 *                    least significant first; bits 6: 4 codes per 3-byte
 *                    triplet read as a little-endian 24-bit integer, code j at
 *                    bit 6*(j mod 4). w = code * scale + bias, scale and bias
 *                    bf16 [E, n, k/group_size].
 *   MOE_FMT_CODEBOOK bits 2 / 3 / 4: 32/bits codes per u32 word, least
 *                    significant first (3-bit words leave bits 30-31 unused).
 *                    w = codebook[code] * scale, scale f16 [E, n, k/group_size],
 *                    codebook f16 [2^bits] shared by all experts
 *                    (turboquant fast_switch_patch.py, _get_dequant_kernel).
 *   MOE_FMT_NVFP4    bits 4, group_size 16: two E2M1 codes per byte, element 2i
 *                    in the low nibble. w = e2m1(code) * e4m3(scale) * scale2[e],
 *                    scale E4M3 bytes [E, n, k/16], scale2 f32 [E]
 *                    (spark_model quant_dispatch.rs, w4a16_gemv: B packed,
 *                    B_scale, scale2).
 *   MOE_FMT_MXFP4    bits 4, group_size 32: E2M1 codes stored as for NVFP4.
 *                    w = e2m1(code) * 2^(scale - 127), scale E8M0 bytes
 *                    [E, n, k/32] (0xFF is NaN); no aux array (spark_model
 *                    helpers_a.rs: native-MXFP4 routed experts, per-32 E8M0
 *                    scales [N, K/32]). The grouped GEMM takes bf16 and f32 x
 *                    (e2m1 * 2^e is exact in bf16 within its exponent range);
 *                    with f16 x, MOE_PATH_GROUPED returns MOE_ERR_UNSUPPORTED
 *                    and MOE_PATH_AUTO uses the routed CUDA-core GEMV.
 */
#ifndef MOE_QMM_H
#define MOE_QMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum { MOE_FMT_AFFINE = 0, MOE_FMT_CODEBOOK = 1, MOE_FMT_NVFP4 = 2, MOE_FMT_MXFP4 = 3 } moe_fmt;
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_F16 = 2 } moe_dtype;
typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARGUMENT = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_WORKSPACE_TOO_SMALL = 3,
    MOE_ERR_CUDA = 4,
    MOE_ERR_BAD_EXPERT_ID = 5,
    MOE_ERR_TIMEOUT = 6,
    MOE_ERR_BAD_EXPERT_POINTER = 7
} moe_status;

/* Which kernel path computes the call. AUTO picks DECODE when R = m * n_expert_used
 * is at most MOE_DECODE_MAX_ROUTINGS or at most MOE_DECODE_MAX_PAIRS_PER_EXPERT *
 * num_experts (few pairs per expert: the CUDA-core GEMV reads each expert's rows
 * once for all its pairs and beats the tensor-core GEMM there), and GROUPED
 * otherwise. DECODE is the CUDA-core GEMV (routing fused in when R <= 64,
 * otherwise read from the routing prologue); GROUPED is the routing prologue
 * followed by the tcgen05 expert-grouped GEMM. GROUPED returns MOE_ERR_UNSUPPORTED for shapes it
 * does not implement (k not a multiple of 8, group_size not a power of two >= 16,
 * packed rows not a multiple of 8 bytes (4 for 3-bit codebook rows), num_experts > 1024); AUTO then uses the
 * routed GEMV instead. */
typedef enum { MOE_PATH_AUTO = 0, MOE_PATH_DECODE = 1, MOE_PATH_GROUPED = 2 } moe_path;

/* Launch flags, OR-ed into the path argument of the entry points that take one
 * (for example (moe_path)(MOE_PATH_AUTO | MOE_LAUNCH_PDL)); other bits above the
 * low byte are MOE_ERR_INVALID_ARGUMENT. They are honoured by the one-token decode
 * kernel (m = 1, 4-bit affine, k <= 3072) and ignored by the other kernels, which
 * always start after the previous work on the stream has completed.
 *   MOE_LAUNCH_PDL            launch as a programmatic dependent of the previous
 *                             kernel on the stream: the kernel may be scheduled on
 *                             SMs that kernel frees before it completes, and waits
 *                             for its completion (griddepcontrol.wait) before it
 *                             reads any input. Hides the launch gap between
 *                             back-to-back calls.
 *   MOE_LAUNCH_EARLY_WEIGHTS  with MOE_LAUNCH_PDL: the caller promises that ids,
 *                             packed, scales and aux were complete before the
 *                             previous kernel on the stream began (for example the
 *                             down projection after the gate+up projection that
 *                             used the same ids). The kernel then reads ids and
 *                             starts streaming the experts' weights before that
 *                             kernel completes; x and the expert bias are read,
 *                             and out is written, only after it. */
#define MOE_LAUNCH_PDL 0x100u
#define MOE_LAUNCH_EARLY_WEIGHTS 0x200u

#define MOE_DECODE_MAX_ROUTINGS 64u
/* Measured on B200 for E = 128, top-8, 4-bit affine (k = 2816, n = 1408 and
 * k = 704, n = 2816): the decode path is faster up to 256 routings (2 per expert),
 * the grouped GEMM from 384 (gate/up) or 512 (down). */
#define MOE_DECODE_MAX_PAIRS_PER_EXPERT 2u
/* Largest num_experts the routing prologue (and so the grouped path) accepts. */
#define MOE_ROUTE_MAX_EXPERTS 1024u

/*
 * moe_qmm_id -- the expert-routed quantized matmul.
 *   x        [m, k] of x_dtype (f32, bf16 or f16), row-major.
 *   ids      [m, n_expert_used] u32 expert indices.
 *   packed   [num_experts, n, moe_packed_row_bytes(fmt, bits, k)] bytes.
 *   scales   [num_experts, n, ceil(k / group_size)]: bf16 (AFFINE), f16 (CODEBOOK),
 *            E4M3 bytes (NVFP4).
 *   aux      AFFINE: biases bf16 [num_experts, n, ceil(k/group_size)];
 *            CODEBOOK: codebook f16 [2^bits]; NVFP4: scale2 f32 [num_experts];
 *            MXFP4: unused (may be NULL).
 *   out      [m, n_expert_used, n] of out_dtype (f32, bf16 or f16); every
 *            element is written (zeros for out-of-range ids). Results are rounded
 *            once from the fp32 accumulator, to nearest even.
 *   workspace, workspace_bytes: device scratch of at least
 *            moe_qmm_id_workspace_bytes(m, n_expert_used, num_experts) bytes,
 *            16-byte aligned. Its first 4 bytes are the device error word; they
 *            must be zero before the first call (cudaMemset once), later calls
 *            only set bits that moe_qmm_id_poll_error() clears. Calls sharing one
 *            workspace must be ordered on the GPU (same stream or events).
 *   Returns MOE_ERR_WORKSPACE_TOO_SMALL if workspace_bytes is short.
 */
moe_status moe_qmm_id(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                      const void *aux, void *out, uint32_t m, uint32_t k, uint32_t n,
                      uint32_t group_size, uint32_t bits, moe_fmt fmt, uint32_t n_expert_used,
                      uint32_t num_experts, moe_dtype x_dtype, moe_dtype out_dtype,
                      void *workspace, size_t workspace_bytes, moe_stream_t stream);

/* moe_qmm_id with an explicit kernel path (tests and benchmarks use it to run
 * both paths on one problem). Same arguments and errors as moe_qmm_id. */
moe_status moe_qmm_id_path(const void *x, const uint32_t *ids, const void *packed,
                           const void *scales, const void *aux, void *out, uint32_t m, uint32_t k,
                           uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                           uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype,
                           moe_dtype out_dtype, void *workspace, size_t workspace_bytes,
                           moe_stream_t stream, moe_path path);

/*
 * moe_qmm_id_bias -- moe_qmm_id followed by a per-expert output bias, added in
 * the kernels' epilogue: out[t][s][col] = sum_j dequant(W[e][col][j]) x[t][j]
 * + bias[e][col], e = ids[t * n_expert_used + s] (turboquant
 * fast_switch_patch.py, the switch layer's output: y + expand_dims(bias[indices], -2)).
 *   expert_bias  [num_experts, n] in bias_dtype (MOE_F32, MOE_BF16 or MOE_F16),
 *                device pointer, caller-owned, element-aligned. Required.
 *   path         as moe_qmm_id_path.
 * The sum is formed in fp32 and rounded once to out_dtype. Rows of out-of-range
 * ids stay 0 (no bias), with the error word set as for moe_qmm_id. Other
 * arguments, ownership and errors as moe_qmm_id; MOE_ERR_INVALID_ARGUMENT also for
 * a null expert_bias or an unknown bias_dtype.
 */
moe_status moe_qmm_id_bias(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                           const void *aux, const void *expert_bias, void *out, uint32_t m, uint32_t k,
                           uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                           uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype,
                           moe_dtype out_dtype, moe_dtype bias_dtype, void *workspace,
                           size_t workspace_bytes, moe_stream_t stream, moe_path path);

/*
 * moe_qmm_id_ptrs -- moe_qmm_id with each expert's weights in its own buffers,
 * named by device tables of per-expert base addresses (metrale helpers_b.rs,
 * ExpertPtrTable {packed_ptrs, scale_ptrs, scale2_vals} and launch_grouped_gemm).
 *   packed_ptrs  [num_experts] u64 device table: expert e's packed rows,
 *                [n, row_bytes] bytes, any alignment. A null entry means the expert
 *                is not held by this caller (spark_model helpers_a.rs: a NULL slot
 *                is skipped, the expert-parallel remote convention): the rows of
 *                its pairs are left untouched.
 *   scale_ptrs   [num_experts] u64: expert e's scales [n, ceil(k/gs)] (bf16 affine,
 *                f16 codebook: 2-byte aligned; u8 E4M3 for NVFP4, u8 E8M0 for MXFP4).
 *   bias_ptrs    [num_experts] u64: AFFINE expert e's biases [n, ceil(k/gs)] bf16
 *                (2-byte aligned); ignored otherwise (may be null).
 *   aux          CODEBOOK: f16 codebook [2^bits]; NVFP4: f32 scale2 [num_experts]
 *                (the table's scale2_vals); ignored for AFFINE and MXFP4 (may be
 *                NULL for MXFP4).
 * The tables and every buffer they name are caller-owned device memory. Paths
 * as moe_qmm_id_path. The CUDA-core path takes code buffers at any alignment;
 * the grouped GEMM needs 8-byte aligned code buffers (4 for 3-bit codebook
 * rows). 16-bit scales and biases must be 2-byte aligned on both paths. A
 * non-null expert whose buffers break these rules, or whose scale / bias entry
 * is null, is skipped (its rows are untouched) and reported by
 * moe_qmm_id_poll_error as MOE_ERR_BAD_EXPERT_POINTER. Other arguments and
 * errors as moe_qmm_id; MOE_ERR_INVALID_ARGUMENT also for null tables.
 */
moe_status moe_qmm_id_ptrs(const void *x, const uint32_t *ids, const uint64_t *packed_ptrs,
                           const uint64_t *scale_ptrs, const uint64_t *bias_ptrs, const void *aux, void *out,
                           uint32_t m, uint32_t k, uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                           uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype, moe_dtype out_dtype,
                           void *workspace, size_t workspace_bytes, moe_stream_t stream, moe_path path);

/* Activation of a gated (GLU) output; see moe_qmm_id_glu. */
typedef enum {
    MOE_ACT_SILU = 0,      /* act(g) = g / (1 + exp(-g))                                  */
    MOE_ACT_GELU_TANH = 1, /* act(g) = g/2 (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)))      */
    MOE_ACT_GELU_ERF = 2   /* act(g) = g/2 (1 + erf(g / sqrt(2)))                          */
} moe_act;

/*
 * moe_qmm_id_glu -- the fused gate+up projection of a gated MoE MLP: moe_qmm_id
 * over experts whose n weight rows hold the gate projection in rows [0, n/2) and
 * the up projection in rows [n/2, n), with the activation applied in the
 * epilogue (spark_model helpers_a.rs, MoeLayer: the fused gate+up kernel, SiLU
 * by default and GELU for GeGLU experts via set_gelu_activation):
 *
 *     y[p][r]   = sum_j dequant(W[e][r][j]) x[t][j] (+ expert_bias[e][r])
 *     out[p][c] = act(y[p][c]) * y[p][n/2 + c],   c < n/2
 *
 *   n            rows per expert; must be even (MOE_ERR_INVALID_ARGUMENT otherwise).
 *   out          [m, n_expert_used, n/2] of out_dtype; every element is written
 *                (zeros for out-of-range ids).
 *   expert_bias  [num_experts, n] in bias_dtype, or NULL for none; added to gate and
 *                up before the activation.
 *   act          a moe_act (MOE_ERR_INVALID_ARGUMENT for other values).
 * y is the fp32 accumulator; act(gate) * up is formed in fp32 and rounded once to
 * out_dtype. Storage, other arguments, paths, ownership and errors as
 * moe_qmm_id_path / moe_qmm_id_bias.
 */
moe_status moe_qmm_id_glu(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                          const void *aux, const void *expert_bias, void *out, uint32_t m, uint32_t k,
                          uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                          uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype,
                          moe_dtype out_dtype, moe_dtype bias_dtype, moe_act act, void *workspace,
                          size_t workspace_bytes, moe_stream_t stream, moe_path path);

/* Workspace bytes moe_qmm_id needs for these sizes (any path). Returns 0 if the
 * sizes overflow. */
size_t moe_qmm_id_workspace_bytes(uint32_t m, uint32_t n_expert_used, uint32_t num_experts);

/* Workspace bytes with room for the grouped path's x operand, which makes that
 * path faster (results are the same up to the order of fp32 sums, and bit for bit
 * for f32 x):
 *   f32 x   -- the pairs' x rows gathered in expert order and split into bf16 halves
 *              once after routing (m * n_expert_used rows of k values, 4 bytes each),
 *              loaded by one tensor copy per tile and half;
 *   bf16 / f16 x -- when the automatic path would take the grouped GEMM with
 *              256-pair tiles (experts hold 96 or more pairs on average), a tile-major
 *              f16 image of the B operand ([m*n_expert_used/256 + num_experts + 1]
 *              tiles x ceil(k/64) x 256 rows x 128 bytes) and one f32 per token (no
 *              room is added for smaller calls): bf16 x is scaled by a
 *              power of two per token (exact in f16 above 2^-28 of the token's largest
 *              value) and the factor is undone in the epilogue. Each k-tile of a tile
 *              is then one bulk copy. Not for MXFP4 weights, pointer tables or gated
 *              outputs, which keep the row copies.
 * With the minimum moe_qmm_id_workspace_bytes the GEMM's loader warps copy x rows
 * themselves. k must be a multiple of 8 (else no room is added). Returns 0 if the
 * sizes overflow or x_dtype is not a moe_dtype. */
size_t moe_qmm_id_workspace_bytes_k(uint32_t m, uint32_t k, uint32_t n_expert_used, uint32_t num_experts,
                                    moe_dtype x_dtype);

/*
 * W4A4: the operation with NVFP4 activations (spark_model helpers_a.rs quantises
 * the routed weights to NVFP4; metrale helpers_b.rs, build_cutlass_grouped_sfb,
 * names the grouped NVFP4 GEMM whose activations are NVFP4 as well). The pages do
 * not say how activations are quantised; the reading implemented, per token t of x,
 * every step in f32:
 *   g_t  = max_j |x[t][j]| / 2688        (2688 = 448 * 6; 0 for an all-zero token)
 *   s_b  = E4M3(max over the 16 values of block b of |x| / (6 g_t)), round to nearest
 *          even, saturating at 448
 *   q_j  = E2M1(x[t][j] / (e4m3(s_b) g_t)), round to nearest even, saturating at 6
 *   x^   = e2m1(q_j) * e4m3(s_b) * g_t
 * and the result is moe_qmm_id with x^ in place of x.
 *
 * moe_quantize_act_nvfp4 -- the quantisation alone, on `stream`: x [m, k] (x_dtype,
 *   device), k a multiple of 16 (else MOE_ERR_UNSUPPORTED). Outputs, each optional
 *   (NULL): codes [m, k/2] bytes, element 2i in the low nibble (4-byte aligned);
 *   scales [m, k/16] E4M3 bytes; gscale [m] f32; xhat [m, k] f32 (x^ rounded once
 *   to f32; 16-byte aligned).
 * moe_qmm_id_w4a4 -- arguments as moe_qmm_id_path (any weight format; the path
 *   argument may carry launch flags). The CUDA-core paths take x^ as f32 x. The
 *   grouped GEMM, for NVFP4 weights with k a multiple of 256, no bias, gated output
 *   or pointer table and 16-byte aligned packed rows, runs the block-scaled
 *   tensor-core MMA on the E2M1 codes of both operands with their E4M3 block scales;
 *   otherwise it takes e2m1(q) * e4m3(s_b) as bf16 (exact). Either way each output
 *   is multiplied by scale2 and its token's g_t before the single rounding.
 *   workspace: at least moe_qmm_id_workspace_bytes_w4a4(m, k, n_expert_used,
 *   num_experts) bytes, 16-byte aligned (else MOE_ERR_WORKSPACE_TOO_SMALL). It
 *   starts with the operation's own workspace, whose first 4 bytes are the device
 *   error word that moe_qmm_id_poll_error(workspace, ...) reads and clears, as for
 *   moe_qmm_id; the quantised x (x^ f32 [m, k], the bf16 values [m, k], g [m], the
 *   codes [m, k/2], the scales [m, k/16], each section rounded up to 256 bytes)
 *   fills the end, from the last 256-byte boundary that leaves room for it. Errors
 *   as moe_qmm_id.
 */
size_t moe_qmm_id_workspace_bytes_w4a4(uint32_t m, uint32_t k, uint32_t n_expert_used, uint32_t num_experts);
moe_status moe_quantize_act_nvfp4(const void *x, uint32_t m, uint32_t k, moe_dtype x_dtype, uint8_t *codes,
                                  uint8_t *scales, float *gscale, float *xhat, moe_stream_t stream);
moe_status moe_qmm_id_w4a4(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                           const void *aux, void *out, uint32_t m, uint32_t k, uint32_t n, uint32_t group_size,
                           uint32_t bits, moe_fmt fmt, uint32_t n_expert_used, uint32_t num_experts,
                           moe_dtype x_dtype, moe_dtype out_dtype, void *workspace, size_t workspace_bytes,
                           moe_stream_t stream, moe_path path);

/* Bytes of one packed weight row (mlx-native quantized_matmul_id.rs,
 * expert_weight_bytes per row): AFFINE 4/8 and CODEBOOK ceil(k / (32/bits)) * 4,
 * AFFINE 6 ceil(k / 4) * 3, NVFP4 k / 2. Returns 0 for an invalid (fmt, bits). */
size_t moe_packed_row_bytes(moe_fmt fmt, uint32_t bits, uint32_t k);

/*
 * moe_qmm_id_route -- the routing prologue alone (histogram, exclusive scan,
 * stable permutation, tile list), as the grouped path runs it. The pages name
 * its outputs expert_offsets and sorted_token_ids (metrale helpers_b.rs,
 * launch_grouped_gemm). Bucket b < num_experts holds the pairs routed to expert
 * b; bucket num_experts holds the pairs whose id is out of range.
 *   counts        [num_experts + 1] u32: pairs per bucket.
 *   offsets       [num_experts + 2] u32: exclusive prefix sum of counts.
 *   sorted_pairs  [m * n_expert_used] u32: pair indices p grouped by bucket in
 *                 ascending bucket order, ascending p inside a bucket (stable).
 *   tiles         [max_tiles, 2] u32: (expert, first row) of each run of
 *                 tile_rows consecutive rows of one expert, experts ascending.
 *                 max_tiles = (m * n_expert_used) / tile_rows + num_experts + 1.
 *   tile_count    [1] u32.
 *   tile_rows     1 .. 65536.
 * The workspace (moe_qmm_id_workspace_bytes) holds the per-chunk histograms and
 * the error word. Requires num_experts <= MOE_ROUTE_MAX_EXPERTS.
 */
moe_status moe_qmm_id_route(const uint32_t *ids, uint32_t m, uint32_t n_expert_used,
                            uint32_t num_experts, uint32_t tile_rows, uint32_t *counts,
                            uint32_t *offsets, uint32_t *sorted_pairs, uint32_t *tiles,
                            uint32_t *tile_count, void *workspace, size_t workspace_bytes,
                            moe_stream_t stream);

/*
 * moe_qmm_id_noalloc -- moe_qmm_id for callers that cannot allocate device memory.
 * (No counterpart on the pages: their operations allocate their own output and
 * parameter buffers.)
 *
 * Who needs it: a service that reserves all device memory at start-up and allows
 * no allocation on its request path, a plug-in running under another framework's
 * caching allocator (a raw cudaMalloc bypasses that allocator and can fail when
 * its pool holds nearly all memory), or a caller that only has the operation's
 * own inputs and outputs. Instead of a caller-provided workspace, the routing
 * prologue uses a MOE_NOALLOC_SCRATCH_BYTES array in device memory that belongs
 * to this library; every GPU that loads the library holds that array until the
 * process exits. This entry point calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 * Same arguments, layouts and results as moe_qmm_id, minus the workspace. The
 * caller still owns and passes x, ids, the weights and out.
 *   * Sizes whose workspace (moe_qmm_id_workspace_bytes(m, n_expert_used,
 *     num_experts)) exceeds MOE_NOALLOC_SCRATCH_BYTES return
 *     MOE_ERR_WORKSPACE_TOO_SMALL and enqueue nothing. At num_experts <= 256 that
 *     admits m * n_expert_used up to about 200,000 routings.
 *   * The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current, and so does the first
 *     call after the device's current CUDA context changed (cudaDeviceReset, or
 *     a context the caller created and made current): the array belongs to the
 *     context's copy of the library's module. A failed lookup returns
 *     MOE_ERR_CUDA. Make that first call before capturing a stream that uses it.
 *   * All calls on a device share the one array and it keeps the last call's
 *     contents. Nothing in it needs to start at zero (every call writes the
 *     buffers it later reads), but calls that overlap on the GPU (different
 *     streams without ordering between them) race on it: order them.
 *   * The array's first word is the device error word of these calls:
 *     out-of-range ids give zero output rows and set a bit there, which
 *     moe_qmm_id_noalloc_poll_error() reads and clears.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (1u << 20)
moe_status moe_qmm_id_noalloc(const void *x, const uint32_t *ids, const void *packed,
                              const void *scales, const void *aux, void *out, uint32_t m, uint32_t k,
                              uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                              uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype,
                              moe_dtype out_dtype, moe_stream_t stream);

/* moe_qmm_id_poll_error for the calls of moe_qmm_id_noalloc on the current device:
 * synchronise `stream`, read and clear the error word in the library's scratch
 * array. Same results as moe_qmm_id_poll_error; allocates nothing. */
moe_status moe_qmm_id_noalloc_poll_error(moe_stream_t stream);

/*
 * moe_qmm_plan -- a call with everything but x, ids and out bound once, for
 * callers that issue the same projection many times (one plan per layer and
 * projection in a decode loop). The plan lives in caller-owned storage (no
 * allocation); moe_qmm_plan_init validates the bound arguments once, and
 * moe_qmm_plan_run takes only the per-call pointers and the stream.
 *   moe_qmm_plan_init  packed, scales, aux, sizes, formats, types, workspace and path
 *                      (launch flags included) as moe_qmm_id_path; expert_bias and
 *                      bias_dtype as moe_qmm_id_bias, or NULL for none; act -1 for a
 *                      plain output, else a moe_act (the output of moe_qmm_id_glu).
 *                      Returns the status moe_qmm_id would return for these
 *                      arguments (x, ids and out are checked by each run).
 *                      The plan keeps the pointers, not the data: the buffers must
 *                      outlive it.
 *   moe_qmm_plan_run   x, ids, out as moe_qmm_id. MOE_ERR_INVALID_ARGUMENT for a
 *                      plan that was not initialised successfully, or a NULL
 *                      pointer.
 */
typedef struct {
    uint64_t opaque[24];
} moe_qmm_plan;

moe_status moe_qmm_plan_init(moe_qmm_plan *plan, const void *packed, const void *scales, const void *aux,
                             const void *expert_bias, uint32_t m, uint32_t k, uint32_t n,
                             uint32_t group_size, uint32_t bits, moe_fmt fmt, uint32_t n_expert_used,
                             uint32_t num_experts, moe_dtype x_dtype, moe_dtype out_dtype,
                             moe_dtype bias_dtype, int32_t act, void *workspace, size_t workspace_bytes,
                             moe_path path);
moe_status moe_qmm_plan_run(const moe_qmm_plan *plan, const void *x, const uint32_t *ids, void *out,
                            moe_stream_t stream);

/* Synchronise `stream`, read and clear the device error word of `workspace`.
 * Returns MOE_OK, MOE_ERR_BAD_EXPERT_ID (some id was >= num_experts),
 * MOE_ERR_TIMEOUT (a bounded wait inside a kernel gave up; its outputs are not
 * valid), MOE_ERR_BAD_EXPERT_POINTER (moe_qmm_id_ptrs skipped an expert whose
 * scale or bias buffer was null or misaligned) or MOE_ERR_CUDA. */
moe_status moe_qmm_id_poll_error(void *workspace, moe_stream_t stream);

/*
 * moe_qmm_test_inject_wait_timeout -- failure-detection test hook (no counterpart
 * on the pages). While limit_ns is non-zero, every call launched afterwards from
 * this process whose kernel has bounded device waits (the tcgen05 grouped GEMM and
 * the one-token decode kernel) makes one extra wait per CTA on a barrier that
 * nothing completes, and gives up after limit_ns nanoseconds: the CTA raises its
 * abort flag, lets its own copies and MMAs in flight complete (with the normal
 * 1 s limit, not limit_ns), frees its tensor memory and exits, and the call's
 * error word reports MOE_ERR_TIMEOUT. Outputs of such calls are not valid.
 * limit_ns = 0 (the default) turns the hook off. The hook only shortens waits:
 * it never faults or hangs the GPU. Returns MOE_OK.
 */
moe_status moe_qmm_test_inject_wait_timeout(uint64_t limit_ns);

/*
 * moe_qmm_test_x_copies -- test hook (no counterpart on the pages). on = 1: calls
 * launched afterwards from this process that take the grouped path with f32 x have
 * the GEMM's loader warps copy x rows and split them into bf16 halves per tile even
 * when the workspace holds the gathered rows, so that tests can check both ways give
 * the same bits. on = 0 (the default) restores the tensor copies of gathered rows.
 * Returns MOE_ERR_INVALID_ARGUMENT for any other value.
 */
moe_status moe_qmm_test_x_copies(int on);

/* Static description of a status code. */
const char *moe_status_str(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_QMM_H */
