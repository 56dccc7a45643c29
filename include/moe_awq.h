/*
 * moe_awq.h -- C ABI of the B200 (sm_100a) frozen AWQ routed-experts FFN.
 *
 * The operation (forward):
 *   route   : top-k over FP32 router logits (+ optional selection-only bias),
 *             FP32 weights from the softmax of the unbiased logits;
 *   dispatch: COPY of every selected (token, expert) row into an
 *             expert-sorted buffer;
 *   experts : per expert, gate/up projections from AWQ int4 words, SwiGLU,
 *             down projection;
 *   combine : per token, FP32-weighted sum of its expert rows in ascending
 *             expert-ID order.
 * and its first-order input VJP (the transpose of the same rounded
 * coefficients).  Sources of each statement are cited per function:
 *   [PE] ruda-tensor 0.21.34, src/packed_experts.rs
 *   [FA] ruda-tensor 0.21.33, src/frozen_awq.rs
 *   [MX] ruda-tensor 0.21.38, src/moe_exchange.rs
 *
 * Conventions for every function:
 *  - Every tensor argument is CALLER-OWNED DEVICE memory, row-major and
 *    contiguous, unless the comment says "host".  The library never
 *    allocates device memory; scratch comes from a caller workspace sized by
 *    the matching *_workspace_size query.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL means the
 *    legacy default stream) and never synchronises.  Host-side argument
 *    errors are reported before anything is launched.
 *  - Return value: MOE_OK, or an error code; moe_last_error_string() (per
 *    host thread) then describes it.
 *  - Data errors that only the device can see (an expert ID outside the
 *    resident range, inconsistent offsets, a row index outside [0, A)) are
 *    OR-ed into *device_status (an int32 in device memory that the caller
 *    zeroes); the offending rows are skipped, nothing traps.
 *  - Packed weights are frozen: no function produces weight, zero-point,
 *    scale or bias gradients ([PE] PackedExpertAutodiffError::TrainableMetadata,
 *    [FA] FrozenAwqError::TrainableBase), and there is no dense or
 *    requantized fallback ([FA] FrozenAwqError::Native, FrozenAwqOps doc).
 *  - 16-bit floating tensors are IEEE binary16 (MOE_F16) or bfloat16
 *    (MOE_BF16); FP32 is MOE_F32.
 *
 * AWQ projection payload of E experts, input width K, output width N
 * ([PE] AwqExpertPayload, AwqExpertOptions; [FA] FrozenAwqOps doc):
 *   qweight  int32 [E, K, N/8]     eight 4-bit codes per word; nibble slot s
 *                                  (bits 4s..4s+3, word read as unsigned)
 *                                  holds logical column 8w + P[s],
 *                                  P = {0,2,4,6,1,3,5,7}
 *   qzeros   int32 [E, K/group, N/8] zero codes, same packing
 *   scales   [E, K/group, N]       F16 or BF16 (scale_dtype)
 *   bias     [E, N] or NULL        F32, F16 or BF16 (bias_dtype), added to
 *                                  the FP32 accumulator before rounding
 *   coefficient W[e,kk,n] = RNE_scale_dtype((q - z[kk/group, n]) * s[kk/group, n]):
 *   the exact product rounded once to the scale dtype.
 *   Requirements: N % 8 == 0, K % group == 0, group % 16 == 0; qweight,
 *   scales, bias and the activation/output tensors 16-byte aligned.
 *   The tensor-core products run in the scale dtype; activations are
 *   converted to it when they differ (BF16 -> F16 is exact in F16's normal
 *   range; above it a value becomes inf and MOE_DEVICE_ERR_ACT_RANGE is set;
 *   below 2^-14 it keeps what F16's subnormal grid holds, an absolute change
 *   under 2^-25; F16 -> BF16 rounds to 8 significant bits).  FP32 scales are
 *   rejected with MOE_ERR_UNSUPPORTED_DTYPE.
 */
#ifndef MOE_AWQ_H_
#define MOE_AWQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of this ABI are the only ones the shared library exports. */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARGUMENT = 1,  /* null/misaligned pointer, bad shape or size */
  MOE_ERR_UNSUPPORTED_DTYPE = 2, /* dtype combination this library does not run */
  MOE_ERR_WORKSPACE = 3,         /* workspace NULL or smaller than required */
  MOE_ERR_CUDA = 4               /* a CUDA runtime call or launch failed */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_F16 = 1, MOE_BF16 = 2 } moe_dtype;

/* Bits OR-ed into *device_status by kernels. */
#define MOE_DEVICE_ERR_EXPERT_RANGE 1 /* an expert ID outside [expert_start, expert_start+E) */
#define MOE_DEVICE_ERR_OFFSETS 2      /* offsets not monotone, offsets[0] != 0 or offsets[E] != A */
#define MOE_DEVICE_ERR_ROW_RANGE 4    /* a row_of entry outside [0, A) */
#define MOE_DEVICE_ERR_TIMEOUT 8      /* a bounded device wait gave up */
#define MOE_DEVICE_ERR_ACT_RANGE 16   /* a BF16 activation or gradient fed to F16-scale tensor cores was
                                         finite above F16's range (|v| > 65504: it became inf) or NaN;
                                         the result is computed from the converted value.  Also set by
                                         the _dt steps that write F16 from BF16 inputs */

/* Limits of this implementation. */
#define MOE_MAX_EXPERTS 4096
#define MOE_MAX_TOP_K 32

/* Description of the last error returned on this host thread. */
MOE_API const char *moe_last_error_string(void);

/* Library version string. */
MOE_API const char *moe_version(void);

/* ------------------------------------------------------------------------
 * moe_route_dispatch -- [MX] MoeDispatchOps::moe_dispatch ("selection and
 * continuous weights followed by device COPY dispatch") and MoeDispatched.
 *
 *  x                [T, H]  activations (F32, F16 or BF16: x_dtype); copied
 *                           bit for bit, never rounded
 *  logits           [T, E]  FP32 router logits
 *  sel_bias         [E]     FP32 selection-only bias, or NULL; it changes
 *                           which experts are chosen, never the weights
 *  expert_start             first global expert ID of the resident bank
 *                           ([PE] AwqExpertOptions::expert_start)
 *  top_k                    1 <= top_k <= min(E, MOE_MAX_TOP_K)
 *  renormalize              1: weights = softmax of the selected unbiased
 *                           logits (softmax -> top-k -> renormalise);
 *                           0: weights = full-softmax probabilities of the
 *                           selected experts
 * Outputs (A = T * top_k):
 *  values           [A, H]  expert-sorted row copies ([MX] MoeDispatched::values)
 *  weights          [T, k]  FP32 ([MX] MoeDispatched::weights)
 *  selected_experts [T, k]  uint32 global IDs, descending score, ties to the
 *                           lower ID ([MX] MoeDispatched::selected_experts)
 *  row_experts      [A]     uint32 global IDs of each row, ascending
 *                           ([MX] MoeDispatched::row_experts)
 *  offsets          [E+1]   int32 exclusive prefix of per-expert row counts;
 *                           an empty expert has offsets[e] == offsets[e+1]
 *  src_token        [A]     int32 source token of each row; ascending inside
 *                           each expert (stable order)
 *  row_of           [T, k]  int32 row holding (token t, selection j)
 *  workspace                device scratch of at least
 *                           moe_route_dispatch_workspace_size(T, E, top_k)
 *                           bytes, 16-byte aligned; contents need no
 *                           initialisation and are dead after the call
 * Errors: MOE_ERR_INVALID_ARGUMENT for T < 0, H < 1, E < 1 or
 * E > MOE_MAX_EXPERTS, top_k out of range, a NULL pointer with T > 0;
 * MOE_ERR_WORKSPACE if workspace is too small.  Scores compare as IEEE
 * floats: -0 and +0 are equal (a tie, lower ID first).  NaN logits are
 * invalid input; a NaN score ranks as -inf (so every index stays defined and
 * in range), and the weights of a token that selects it are NaN.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_route_dispatch_workspace_size(int64_t T, int64_t E, int32_t top_k);

MOE_API moe_status moe_route_dispatch(const void *x, moe_dtype x_dtype, int64_t T, int64_t H,
                              const float *logits, const float *sel_bias, int64_t E,
                              int32_t expert_start, int32_t top_k, int32_t renormalize,
                              void *values, float *weights, uint32_t *selected_experts,
                              uint32_t *row_experts, int32_t *offsets, int32_t *src_token,
                              int32_t *row_of, void *workspace, size_t workspace_bytes,
                              int32_t *device_status, void *stream);

/* moe_route_dispatch with the rows of values stored in values_dtype: x_dtype
 * (the COPY itself), or F16 for BF16 x, the operand dtype of projections
 * with F16 scales, so they take the rows without a conversion pass (exact in
 * F16's normal range; a finite value above it, or a NaN, sets
 * MOE_DEVICE_ERR_ACT_RANGE, as the projections' own conversion does).  Any
 * other pair gives MOE_ERR_UNSUPPORTED_DTYPE. */
MOE_API moe_status moe_route_dispatch_dt(const void *x, moe_dtype x_dtype, int64_t T, int64_t H,
                                 const float *logits, const float *sel_bias, int64_t E,
                                 int32_t expert_start, int32_t top_k, int32_t renormalize,
                                 void *values, moe_dtype values_dtype, float *weights,
                                 uint32_t *selected_experts, uint32_t *row_experts, int32_t *offsets,
                                 int32_t *src_token, int32_t *row_of, void *workspace,
                                 size_t workspace_bytes, int32_t *device_status, void *stream);

/* ------------------------------------------------------------------------
 * moe_route -- the routing and row maps of moe_route_dispatch without the
 * COPY of the rows (the gather mode of the dispatch: the gate/up projection
 * then reads each row from x through src_token, see
 * awq_grouped_gate_up_swiglu_gather).  [MX] MoeDispatchOps::moe_dispatch
 * states the device COPY as its contract; this entry point departs from it
 * on purpose, and moe_route_dispatch keeps it.
 *
 * Arguments, outputs and errors as moe_route_dispatch, minus x, x_dtype, H
 * and values; the workspace is sized by moe_route_dispatch_workspace_size.
 * ---------------------------------------------------------------------- */
MOE_API moe_status moe_route(const float *logits, const float *sel_bias, int64_t T, int64_t E,
                             int32_t expert_start, int32_t top_k, int32_t renormalize, float *weights,
                             uint32_t *selected_experts, uint32_t *row_experts, int32_t *offsets,
                             int32_t *src_token, int32_t *row_of, void *workspace, size_t workspace_bytes,
                             int32_t *device_status, void *stream);

/* ------------------------------------------------------------------------
 * moe_route_dispatch_noalloc -- moe_route_dispatch for callers that cannot
 * allocate device memory for a workspace: serving loops that must not call
 * cudaMalloc/cudaFree (those calls can synchronise the device and stall
 * every stream), or host frameworks that own all device memory through their
 * own pool and forbid allocations outside it.  The method's pages have no
 * counterpart of this entry point; it is a property of this library.
 *
 * Same arguments, results and errors as moe_route_dispatch, minus the
 * workspace: the scratch is a fixed 1 MiB array compiled into the library
 * (every GPU that loads the library holds it until the process exits).
 *  - Sizes whose scratch (moe_route_dispatch_workspace_size(T, E, top_k))
 *    exceeds 1 MiB are rejected with MOE_ERR_WORKSPACE before any launch.
 *  - The first call on a device looks the array's device address up
 *    (cudaGetSymbolAddress) with the caller's current device, which must be
 *    the device of `stream`; make that first call before any stream capture.
 *    The address is kept per device and looked up again when the device's
 *    context has changed (after cudaDeviceReset).
 *  - Argument errors are those of moe_route_dispatch and are checked first;
 *    MOE_ERR_WORKSPACE then means only "too large for the built-in scratch".
 *  - Every call shares the one array, which keeps the last call's contents
 *    (nothing in it needs to start at zero).  Calls whose kernels overlap on
 *    the GPU (other streams, other host threads) race on it: serialise them.
 *  - Nothing is allocated: no cudaMalloc, cudaFree or allocating library
 *    routine is called.
 * ---------------------------------------------------------------------- */
MOE_API moe_status moe_route_dispatch_noalloc(const void *x, moe_dtype x_dtype, int64_t T, int64_t H,
                                              const float *logits, const float *sel_bias, int64_t E,
                                              int32_t expert_start, int32_t top_k,
                                              int32_t renormalize, void *values, float *weights,
                                              uint32_t *selected_experts, uint32_t *row_experts,
                                              int32_t *offsets, int32_t *src_token, int32_t *row_of,
                                              int32_t *device_status, void *stream);

/* ------------------------------------------------------------------------
 * awq_grouped_gate_up_swiglu -- [PE] FrozenPackedExpertOps::packed_swiglu_forward
 * (gate and up projections of the selected experts and the storage-rounded
 * SwiGLU; "AD preserves required actual input caches": G and U are written
 * when gate_out/up_out are non-NULL).
 *
 *  values   [A, H]   expert-sorted rows (act_dtype F16 or BF16); rows
 *                    offsets[e]..offsets[e+1] belong to local expert e
 *  offsets  [E+1]    int32, as written by moe_route_dispatch
 *  gate/up payloads  AWQ payloads with K = H, N = I (see the file header);
 *                    both share scale_dtype, bias_dtype and group
 *  h        [A, I]   act_dtype: RNE(silu(G) * U), silu(v) = v / (1 + e^-v)
 *  gate_out [A, I]   act_dtype G = RNE(sum_kk values*Wg + bias_g), or NULL
 *  up_out   [A, I]   act_dtype U = RNE(sum_kk values*Wu + bias_u), or NULL
 * The tile path is chosen inside from A and E (see moe_set_projection_path):
 * small per-expert batches on warp-level tensor-core tiles that stream the
 * packed words, mid-size ones on 128-row tcgen05/TMEM tiles, long ones on
 * 256-row tcgen05 tiles over a CTA pair.
 *  workspace  device scratch of awq_projection_workspace_size(A, H, I, E, group_size, 2)
 *             bytes (16-byte aligned; may be NULL when that size is 0):
 *             split-K partial sums of the small-batch tiles.  Its contents
 *             need no initialisation and are dead after the call.
 * Device errors: MOE_DEVICE_ERR_OFFSETS, MOE_DEVICE_ERR_ACT_RANGE (F16 scales
 * with BF16 inputs), MOE_DEVICE_ERR_TIMEOUT.
 * ---------------------------------------------------------------------- */
MOE_API moe_status awq_grouped_gate_up_swiglu(
    const void *values, moe_dtype act_dtype, int64_t A, int64_t H, int64_t I,
    const int32_t *offsets, int64_t E,
    const int32_t *qweight_gate, const int32_t *qzeros_gate, const void *scales_gate,
    const void *bias_gate,
    const int32_t *qweight_up, const int32_t *qzeros_up, const void *scales_up,
    const void *bias_up,
    moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size,
    void *h, void *gate_out, void *up_out, void *workspace, size_t workspace_bytes,
    int32_t *device_status, void *stream);

/* awq_grouped_gate_up_swiglu with gate_out and up_out stored in out_dtype
 * and h in h_dtype (each F16 or BF16) instead of act_dtype: the same FP32
 * sums, one rounding of G and U to out_dtype, h = RNE_{h_dtype}(silu(G) U)
 * from the rounded G and U.  With F16 scales, F16 values from
 * moe_route_dispatch_dt and F16 h (the down projection's operand dtype) need
 * no conversion pass while G and U stay BF16; F16 h from BF16 G and U that
 * overflows F16 (a value that is not +-inf becoming inf or NaN) sets
 * MOE_DEVICE_ERR_ACT_RANGE. */
MOE_API moe_status awq_grouped_gate_up_swiglu_dt(
    const void *values, moe_dtype act_dtype, int64_t A, int64_t H, int64_t I,
    const int32_t *offsets, int64_t E,
    const int32_t *qweight_gate, const int32_t *qzeros_gate, const void *scales_gate,
    const void *bias_gate,
    const int32_t *qweight_up, const int32_t *qzeros_up, const void *scales_up,
    const void *bias_up,
    moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size,
    void *h, moe_dtype h_dtype, void *gate_out, void *up_out, moe_dtype out_dtype,
    void *workspace, size_t workspace_bytes, int32_t *device_status, void *stream);

/* ------------------------------------------------------------------------
 * awq_grouped_gate_up_swiglu_gather -- awq_grouped_gate_up_swiglu on rows
 * gathered from the tokens instead of a COPY: expert-sorted row r is
 * x[src_token[r], :] (x [T, H] in act_dtype, src_token [A] int32 as written
 * by moe_route or moe_route_dispatch).  Same outputs, bit for bit, as
 * awq_grouped_gate_up_swiglu on values = the COPY of those rows; same
 * payload arguments, workspace and errors.  A src_token entry outside
 * [0, T) sets MOE_DEVICE_ERR_ROW_RANGE and that row reads token 0.
 * The tcgen05 tiles copy the rows with 16-byte cp.async from their
 * producer lanes (this GPU's memory, no multicast); the small-batch tiles
 * with one bulk copy or load per row.
 * ---------------------------------------------------------------------- */
MOE_API moe_status awq_grouped_gate_up_swiglu_gather(
    const void *x, moe_dtype act_dtype, int64_t T, const int32_t *src_token, int64_t A, int64_t H, int64_t I,
    const int32_t *offsets, int64_t E,
    const int32_t *qweight_gate, const int32_t *qzeros_gate, const void *scales_gate, const void *bias_gate,
    const int32_t *qweight_up, const int32_t *qzeros_up, const void *scales_up, const void *bias_up,
    moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size,
    void *h, void *gate_out, void *up_out, void *workspace, size_t workspace_bytes,
    int32_t *device_status, void *stream);

/* awq_grouped_gate_up_swiglu_gather with the output dtypes of
 * awq_grouped_gate_up_swiglu_dt. */
MOE_API moe_status awq_grouped_gate_up_swiglu_gather_dt(
    const void *x, moe_dtype act_dtype, int64_t T, const int32_t *src_token, int64_t A, int64_t H,
    int64_t I, const int32_t *offsets, int64_t E,
    const int32_t *qweight_gate, const int32_t *qzeros_gate, const void *scales_gate,
    const void *bias_gate,
    const int32_t *qweight_up, const int32_t *qzeros_up, const void *scales_up,
    const void *bias_up,
    moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size,
    void *h, moe_dtype h_dtype, void *gate_out, void *up_out, moe_dtype out_dtype,
    void *workspace, size_t workspace_bytes, int32_t *device_status, void *stream);

/* Workspace bytes for the projection of A rows (input width K, output width
 * N, E experts, AWQ group size; nproj = 2 for the gate/up pair, 1 for a
 * single projection) under the current projection path; 0 if none:
 *  - the warp-level tiles that stream the packed words: their split-K
 *    partial sums (required: a smaller workspace is MOE_ERR_WORKSPACE);
 *  - a tcgen05 tile with F16 scales and BF16 activations: an F16 copy of
 *    the activations (A x K), made once so that the tile's column blocks do
 *    not each convert the same rows again (optional: with less workspace
 *    the tile converts in place, same results, slower).
 * awq_projection_workspace_size assumes the conversion may be needed;
 * awq_projection_workspace_size_dt gives the bytes for the actual dtypes. */
MOE_API size_t awq_projection_workspace_size(int64_t A, int64_t K, int64_t N, int64_t E,
                                             int64_t group_size, int32_t nproj);
MOE_API size_t awq_projection_workspace_size_dt(int64_t A, int64_t K, int64_t N, int64_t E,
                                                int64_t group_size, int32_t nproj, moe_dtype act_dtype,
                                                moe_dtype scale_dtype);

/* ------------------------------------------------------------------------
 * awq_grouped_down -- the down projection of [PE] packed_swiglu_forward; also
 * the grouped single projection [PE] FrozenPackedExpertOps::packed_expert_forward
 * on expert-sorted rows, and with E = 1, offsets = {0, A} the single frozen
 * linear [FA] FrozenAwqOps::frozen_awq_forward.
 *
 *  input [A, K] act_dtype (F16 or BF16); output [A, N] act_dtype:
 *  output[r, n] = RNE(sum_kk input[r,kk] * W[e,kk,n] + bias[e,n]).
 *  workspace: awq_projection_workspace_size(A, K, N, E, group_size, 1) bytes (see
 *  awq_grouped_gate_up_swiglu).
 * Device errors: MOE_DEVICE_ERR_OFFSETS, MOE_DEVICE_ERR_ACT_RANGE (F16 scales
 * with BF16 inputs), MOE_DEVICE_ERR_TIMEOUT.
 * ---------------------------------------------------------------------- */
MOE_API moe_status awq_grouped_down(const void *input, moe_dtype act_dtype, int64_t A, int64_t K,
                            int64_t N, const int32_t *offsets, int64_t E,
                            const int32_t *qweight, const int32_t *qzeros, const void *scales,
                            const void *bias, moe_dtype scale_dtype, moe_dtype bias_dtype,
                            int64_t group_size, void *output, void *workspace,
                            size_t workspace_bytes, int32_t *device_status, void *stream);

/* awq_grouped_down with the output stored in out_dtype (F16 or BF16) instead
 * of act_dtype: F16 h (the operand dtype with F16 scales) in, BF16 y out. */
MOE_API moe_status awq_grouped_down_dt(const void *input, moe_dtype act_dtype, int64_t A, int64_t K,
                               int64_t N, const int32_t *offsets, int64_t E,
                               const int32_t *qweight, const int32_t *qzeros, const void *scales,
                               const void *bias, moe_dtype scale_dtype, moe_dtype bias_dtype,
                               int64_t group_size, void *output, moe_dtype out_dtype,
                               void *workspace, size_t workspace_bytes, int32_t *device_status,
                               void *stream);

/* ------------------------------------------------------------------------
 * nf4_grouped_projection, nf4_input_backward -- a projection whose frozen
 * payload is NF4 instead of AWQ: [PE] PackedExpertPayload::Nf4 ("original
 * RUDA high-nibble-first flat-block NF4"; packed scales and codebook stay
 * frozen; gate, up and down each pick their format independently).  The
 * pages print no NF4 layout; this library reads it as the 4-bit NormalFloat
 * data type of Dettmers et al., "QLoRA" (2023), flat blocks:
 *   codes    uint8 [E, K*N/2]   the logical [K, N] matrix of each expert
 *                               flattened row-major; flat element
 *                               f = kk*N + n sits in byte f/2, in the high
 *                               nibble (bits 4..7) when f is even
 *   absmax   f32 [E, K*N/block] one scale per `block` consecutive elements
 *   codebook f32 [16]           the 16 code values (caller-supplied)
 *   coefficient W[e,kk,n] = RNE_coef_dtype(codebook[q] * absmax[f / block]):
 *   the F32 x F32 product, exact, rounded once to coef_dtype (F16 or BF16,
 *   which is also the tensor-core operand dtype).
 * nf4_grouped_projection: output[r, n] = RNE(sum_kk input[r,kk] W[e,kk,n]
 *   + bias[e,n]) for the rows of expert e (offsets as for the AWQ calls);
 *   input [A, K], output [A, N] (act_dtype), bias [E, N] or NULL.
 * nf4_input_backward: dinput[r, kk] = RNE(sum_n grad[r,n] W[e,kk,n]);
 *   grad [A, N], dinput [A, K] (grad_dtype).
 * Requirements: K and N multiples of 64, block a multiple of 32 dividing
 * K*N; input/output/codes 16-byte aligned.  Device errors:
 * MOE_DEVICE_ERR_OFFSETS, MOE_DEVICE_ERR_ACT_RANGE.
 * ---------------------------------------------------------------------- */
MOE_API moe_status nf4_grouped_projection(const void *input, moe_dtype act_dtype, int64_t A, int64_t K, int64_t N,
                                          const int32_t *offsets, int64_t E, const uint8_t *codes,
                                          const float *absmax, const float *codebook, int64_t block,
                                          moe_dtype coef_dtype, const void *bias, moe_dtype bias_dtype,
                                          void *output, int32_t *device_status, void *stream);

MOE_API moe_status nf4_input_backward(const void *grad, moe_dtype grad_dtype, int64_t A, int64_t N, int64_t K,
                                      const int32_t *offsets, int64_t E, const uint8_t *codes,
                                      const float *absmax, const float *codebook, int64_t block,
                                      moe_dtype coef_dtype, void *dinput, int32_t *device_status, void *stream);

/* ------------------------------------------------------------------------
 * moe_combine -- [MX] MoeDispatchOps::moe_combine ("ascending expert-ID
 * combine after actual expert rows have returned to their source").
 *
 *  y [A, H] expert rows (act_dtype), weights [T, k] FP32,
 *  selected_experts [T, k], row_of [T, k] as written by moe_route_dispatch.
 *  out[t, :] = RNE(sum over j in ascending selected_experts[t, j] of
 *              weights[t, j] * y[row_of[t, j], :]), FP32 accumulation from +0.
 * Device errors: MOE_DEVICE_ERR_ROW_RANGE (that term is skipped).
 * ---------------------------------------------------------------------- */
MOE_API moe_status moe_combine(const void *y, moe_dtype act_dtype, int64_t A, const float *weights,
                       const uint32_t *selected_experts, const int32_t *row_of, int64_t T,
                       int64_t H, int32_t top_k, void *out, int32_t *device_status,
                       void *stream);

/* ------------------------------------------------------------------------
 * moe_combine_backward -- [MX] MoeDispatchOps::moe_combine_backward with
 * MoeCombineSelection: each requested output is non-NULL.
 *
 *  dy[row_of[t,j], :] = RNE(weights[t,j] * d_out[t, :])     ([A, H], act_dtype)
 *  dweights[t, j]     = sum_c d_out[t,c] * y[row_of[t,j], c] ([T, k], FP32)
 * Device errors: MOE_DEVICE_ERR_ROW_RANGE.
 * ---------------------------------------------------------------------- */
MOE_API moe_status moe_combine_backward(const void *d_out, const void *y, moe_dtype act_dtype, int64_t A,
                                const float *weights, const int32_t *row_of, int64_t T,
                                int64_t H, int32_t top_k, void *dy, float *dweights,
                                int32_t *device_status, void *stream);

/* moe_combine_backward with dy stored in dy_dtype (F16 or BF16) instead of
 * act_dtype: dy[row_of[t,j], :] = RNE_{dy_dtype}(weights[t,j] * d_out[t, :]),
 * one rounding of the FP32 product.  F16 dy from BF16 inputs feeds an input
 * VJP with F16 scales without a conversion pass; a value that is not +-inf
 * but becomes inf or NaN in F16 sets MOE_DEVICE_ERR_ACT_RANGE (the rule of
 * the BF16 -> F16 input conversion).  dweights is unchanged. */
MOE_API moe_status moe_combine_backward_dt(const void *d_out, const void *y, moe_dtype act_dtype, int64_t A,
                                   const float *weights, const int32_t *row_of, int64_t T,
                                   int64_t H, int32_t top_k, void *dy, moe_dtype dy_dtype,
                                   float *dweights, int32_t *device_status, void *stream);

/* ------------------------------------------------------------------------
 * awq_input_backward -- [FA] FrozenAwqOps::frozen_awq_input_backward and
 * [PE] packed_expert_input_backward / packed_swiglu_input_backward: the
 * transpose of the same rounded coefficients, per expert.
 *
 *  grad   [A, N] grad_dtype (F16 or BF16), payload with K_in = K, width N
 *  grad2  [A, N] or NULL, with a second payload (qweight2, qzeros2, scales2)
 *  dinput[r, kk] = RNE(sum_n grad[r,n] W[e,kk,n] + sum_n grad2[r,n] W2[e,kk,n])
 *  ([A, K], grad_dtype; the two sums share one accumulator and one rounding)
 * Tile paths as for the forward projections (warp-level, 128-row tcgen05,
 * 256-row CTA-pair tcgen05); the tensor-core products run in the scale
 * dtype, gradients converted to it when they differ.
 *  workspace  device scratch of awq_input_backward_workspace_size(...) bytes
 *             (16-byte aligned), or NULL: F16 copies of the gradients for a
 *             tcgen05 tile with F16 scales and BF16 gradients, made once
 *             (optional: with less the tile converts in place, same results).
 * Device errors: MOE_DEVICE_ERR_OFFSETS, MOE_DEVICE_ERR_ACT_RANGE (F16 scales
 * with BF16 inputs), MOE_DEVICE_ERR_TIMEOUT.
 * ---------------------------------------------------------------------- */
MOE_API moe_status awq_input_backward(const void *grad, moe_dtype grad_dtype, int64_t A, int64_t N,
                              int64_t K, const int32_t *offsets, int64_t E,
                              const int32_t *qweight, const int32_t *qzeros, const void *scales,
                              moe_dtype scale_dtype, int64_t group_size, const void *grad2,
                              const int32_t *qweight2, const int32_t *qzeros2,
                              const void *scales2, void *dinput, void *workspace,
                              size_t workspace_bytes, int32_t *device_status, void *stream);

/* awq_input_backward with dinput stored in dinput_dtype (F16 or BF16)
 * instead of grad_dtype: the same FP32 sums, one rounding to dinput_dtype.
 * F16 gradients with F16 scales need no conversion (workspace 0 bytes) and
 * can still give BF16 input gradients. */
MOE_API moe_status awq_input_backward_dt(const void *grad, moe_dtype grad_dtype, int64_t A, int64_t N,
                                 int64_t K, const int32_t *offsets, int64_t E,
                                 const int32_t *qweight, const int32_t *qzeros, const void *scales,
                                 moe_dtype scale_dtype, int64_t group_size, const void *grad2,
                                 const int32_t *qweight2, const int32_t *qzeros2,
                                 const void *scales2, void *dinput, moe_dtype dinput_dtype,
                                 void *workspace, size_t workspace_bytes, int32_t *device_status,
                                 void *stream);

/* Workspace bytes of awq_input_backward for A gradient rows of width N
 * (nproj = 2 with grad2), output width K, under the current path; 0 if none. */
MOE_API size_t awq_input_backward_workspace_size(int64_t A, int64_t N, int64_t K, int64_t E,
                                                 int64_t group_size, int32_t nproj, moe_dtype grad_dtype,
                                                 moe_dtype scale_dtype);

/* ------------------------------------------------------------------------
 * moe_swiglu_backward -- the SwiGLU step of [PE] packed_swiglu_input_backward,
 * from the stored G and U (act_dtype, [A, I] each):
 *   s = 1 / (1 + e^-G),  dG = RNE(dh * U * s * (1 + G (1 - s))),  dU = RNE(dh * G * s)
 * ---------------------------------------------------------------------- */
MOE_API moe_status moe_swiglu_backward(const void *dh, const void *G, const void *U, moe_dtype act_dtype,
                               int64_t A, int64_t I, void *dG, void *dU, void *stream);

/* moe_swiglu_backward with dG and dU stored in grad_dtype (F16 or BF16)
 * instead of act_dtype (dh, G, U stay act_dtype): the same FP32 values, one
 * rounding to grad_dtype.  BF16 inputs with F16 grad_dtype report values
 * that are not +-inf but become inf or NaN in F16 as
 * MOE_DEVICE_ERR_ACT_RANGE in device_status (may be NULL: no report). */
MOE_API moe_status moe_swiglu_backward_dt(const void *dh, const void *G, const void *U, moe_dtype act_dtype,
                                  int64_t A, int64_t I, void *dG, void *dU, moe_dtype grad_dtype,
                                  int32_t *device_status, void *stream);

/* ------------------------------------------------------------------------
 * moe_dispatch_backward -- [MX] MoeDispatchOps::moe_dispatch_backward ("COPY
 * VJP sums selected expert-row seeds without multiplying routing weights
 * again"):
 *   dx[t, :] = RNE(sum over j in ascending selected_experts[t, j] of
 *              dvalues[row_of[t, j], :]), FP32 accumulation.
 * Device errors: MOE_DEVICE_ERR_ROW_RANGE.
 * ---------------------------------------------------------------------- */
MOE_API moe_status moe_dispatch_backward(const void *dvalues, moe_dtype act_dtype, int64_t A,
                                 const int32_t *row_of, const uint32_t *selected_experts,
                                 int64_t T, int64_t H, int32_t top_k, void *dx,
                                 int32_t *device_status, void *stream);

/* ------------------------------------------------------------------------
 * moe_router_backward -- [MX] MoeDispatchOps::moe_dispatch_weights_backward
 * (the logit VJP of the FP32 routing weights at a fixed selection; the
 * selection bias, used only to choose experts, gets no gradient).
 *  logits     [T, E] f32   the router logits the forward routed with
 *  selected   [T, top_k]   u32 global expert IDs (moe_route_dispatch output)
 *  d_weights  [T, top_k]   f32 upstream gradient of the weights
 *  d_logits   [T, E] f32   output, every element written:
 *    renormalize = 1: w = softmax of the selected logits,
 *      d_logits[t, e_j] = w_j (d_weights[t, j] - sum_i w_i d_weights[t, i]),
 *      0 for experts not selected;
 *    renormalize = 0: p = softmax over all E logits, for every e
 *      d_logits[t, e] = p_e (sum_j [e == e_j] d_weights[t, j] - sum_j p_{e_j} d_weights[t, j]).
 *  FP32 arithmetic.  Device errors: MOE_DEVICE_ERR_EXPERT_RANGE (an ID
 *  outside [expert_start, expert_start + E); that selection is skipped).
 * ---------------------------------------------------------------------- */
MOE_API moe_status moe_router_backward(const float *logits, const uint32_t *selected_experts,
                                       const float *d_weights, int64_t T, int64_t E, int32_t top_k,
                                       int32_t renormalize, int32_t expert_start, float *d_logits,
                                       int32_t *device_status, void *stream);

/* ------------------------------------------------------------------------
 * awq_dequant_coefficients -- the coefficients W[kk, n] of ONE expert's
 * payload ([K, N/8] words, [K/group, N/8] zero words, [K/group, N] scales),
 * formed by the same device code the projection kernels run, written out in
 * the scale dtype ([K, N] uint16 bit patterns).  For verification: the
 * rounded coefficient is what [FA] FrozenAwqOps preserves.
 *  pairing 0: the register pairing of the forward warp-level tiles (one
 *             column at two consecutive input rows);
 *  pairing 1: the pairing of the input-VJP and tcgen05 tiles (two columns of
 *             one word).
 * ---------------------------------------------------------------------- */
MOE_API moe_status awq_dequant_coefficients(const int32_t *qweight, const int32_t *qzeros,
                                    const void *scales, moe_dtype scale_dtype, int64_t K,
                                    int64_t N, int64_t group_size, int32_t pairing,
                                    uint16_t *coefficients, void *stream);

/* ------------------------------------------------------------------------
 * Projection tile path: 0 = chosen from A and E (default), 1 = warp-level
 * tiles (small per-expert batches), 2 = tcgen05/TMEM tiles of 128 rows on one
 * SM (mid-size batches), 3 = tcgen05 tiles of 256 rows on a CTA pair
 * (cta_group::2, batches of several hundred rows per expert).  All paths
 * compute the same operation; the knob exists so tests and benchmarks can
 * run any of them on the same inputs.  A shape a tcgen05 path does not take
 * runs on the next path down.  Process-wide; returns the previous value, or
 * -1 for an unknown path.
 * ---------------------------------------------------------------------- */
MOE_API int32_t moe_set_projection_path(int32_t path);

#ifdef __cplusplus
}
#endif

#endif /* MOE_AWQ_H_ */
