/*
 * w4a8.h - C ABI of the B200 (sm_100a) W4A8 routed-expert MoE library.
 *
 * The library computes one routed-expert MoE layer whose experts hold INT4
 * weights and take FP8 (E4M3) activations, as described by the GLM-5.3-W4A8
 * model card (intro; table "differences from the other 4-bit releases";
 * section "quantisation method"): routed experts in symmetric INT4 with one
 * scale per group of 128 weights along K, packed as compressed-tensors
 * "pack-quantized" uint4b8 nibbles, 8 per int32 word; activations quantised
 * to FP8 at run time with one dynamic scale per token; INT4 converted to FP8
 * inside the GEMM, never dequantised to BF16 in memory.
 *
 * Conventions shared by every entry point:
 *  - Every pointer argument is DEVICE memory owned by the caller, unless its
 *    comment says otherwise.  The library never allocates device memory and
 *    never frees caller memory; scratch space comes from a caller-supplied
 *    workspace whose size is given by the matching *_workspace_size call.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  The returned status covers host-side argument checks
 *    and kernel-launch errors only.  Kernels with inter-warp waits bound every
 *    wait; a wait that runs out sets a device error latch that
 *    w4a8_check_device_error() reports.
 *  - Row-major layouts, element strides as stated, no padding between rows.
 *    Device pointers must be 16-byte aligned.
 *  - The device must be compute capability 10.x (the code is built for
 *    sm_100a); other devices get W4A8_ERR_UNSUPPORTED_ARCH.
 *  - On error nothing is launched and w4a8_last_error() (thread-local) holds
 *    a message.
 */
#ifndef W4A8_H_
#define W4A8_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define W4A8_API __attribute__((visibility("default")))
#else
#define W4A8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t w4a8_status;
#define W4A8_OK                      0
#define W4A8_ERR_INVALID_ARG         1  /* null pointer, misalignment, negative size */
#define W4A8_ERR_UNSUPPORTED_SHAPE   2  /* shape outside the supported set (see each call) */
#define W4A8_ERR_UNSUPPORTED_ARCH    3  /* device is not compute capability 10.x */
#define W4A8_ERR_WORKSPACE_TOO_SMALL 4  /* workspace_bytes below the *_workspace_size value */
#define W4A8_ERR_CUDA                5  /* a CUDA runtime call or launch failed */
#define W4A8_ERR_DEVICE_TIMEOUT      6  /* a bounded in-kernel wait ran out (reported later) */
#define W4A8_ERR_DEVICE_INDEX        7  /* an index read on the device was out of range; the
                                           access was skipped (reported later) */

/* Number of timed stages of w4a8_moe_forward (see w4a8_moe_aux.stage_events). */
#define W4A8_NUM_STAGES 6

/* ABI version of this header (incremented on incompatible changes). */
W4A8_API int32_t w4a8_abi_version(void);

/*
 * Build flags of the loaded library: bit 0 (W4A8_BUILD_DEBUG_BOUNDS) is set in
 * the bounds-checking build (libw4a8_debug.so), whose kernels check every
 * routing-derived index (expert offsets and tile tables, segment rows, token
 * ids) against its buffer before use; an index out of range is skipped and
 * reported as W4A8_ERR_DEVICE_INDEX by w4a8_check_device_error.  No
 * counterpart on the pages: it stands in for a memory checker.
 */
#define W4A8_BUILD_DEBUG_BOUNDS 1
W4A8_API int32_t w4a8_build_flags(void);

/* Static text of a status code. */
W4A8_API const char* w4a8_status_string(w4a8_status status);

/* Message of the last failing call on this host thread ("" if none). */
W4A8_API const char* w4a8_last_error(void);

/*
 * w4a8_check_device_error - report and clear the device error latch.
 * Synchronises `stream`, then returns W4A8_ERR_DEVICE_TIMEOUT if any kernel of
 * this library on the current device gave up a bounded wait since the last
 * check, W4A8_ERR_DEVICE_INDEX if a kernel found an index out of range (an
 * expert id outside [-1, E) given to w4a8_moe_forward_experts) and skipped
 * it, W4A8_ERR_CUDA if the stream holds a CUDA error, else W4A8_OK.
 */
W4A8_API w4a8_status w4a8_check_device_error(void* stream);

/*
 * w4a8_selftest_wait_timeout - exercise the failure-detection path.  Launches
 * one thread that waits, with the bounded wait every grouped-GEMM role uses,
 * on a barrier that nothing ever arrives on.  After timeout_ns the wait gives
 * up and raises the device latch, so the next w4a8_check_device_error on the
 * stream returns W4A8_ERR_DEVICE_TIMEOUT (and clears the latch).  Nothing
 * traps or faults; the context stays usable.  No counterpart on the pages.
 *
 *   timeout_ns  0 < timeout_ns <= 10 s (else W4A8_ERR_INVALID_ARG)
 */
W4A8_API w4a8_status w4a8_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/*
 * w4a8_pack_int4 - symmetric INT4 round-to-nearest weight quantisation with
 * one bf16 scale per group of `group` weights along K, packed as uint4b8.
 * (GLM-5.3-W4A8 model card, "quantisation method": symmetric INT4, group
 * size 128, compressed-tensors pack-quantized uint4b8 / int32.)
 *
 * For every row r and group g:  s = bf16(absmax / 7) (float32 division, then
 * round-to-nearest-even to bf16);  q = clamp(rint(w / s), -8, 7) with the
 * float32 quotient (q = 0 when s == 0);  nibble q + 8 of element kappa goes to
 * word kappa / 8, bits 4*(kappa % 8) .. +3.
 *
 *   w_bf16       [R, K] bf16, row-major (R = experts * rows per expert)
 *   R, K         R >= 0; K > 0 and K % 128 == 0
 *   group        must be 128 (else W4A8_ERR_UNSUPPORTED_SHAPE)
 *   packed       [R, K / 8] int32, written
 *   scales_bf16  [R, K / 128] bf16, written
 */
W4A8_API w4a8_status w4a8_pack_int4(const void* w_bf16, int64_t R, int64_t K, int32_t group,
                           int32_t* packed, void* scales_bf16, void* stream);

/*
 * w4a8_pack_int4_mse_clip - as w4a8_pack_int4 (same uint4b8 words, same bf16
 * scale layout, read the same way by w4a8_prepare_experts_b200 and
 * w4a8_moe_forward), but each group's scale is chosen by the per-group MSE
 * clip search of the GLM-5.3-W4A8 model card ("quantisation method": 11 shrink
 * ratios from 1.00 to 0.70, the MSE-optimal scale kept).
 *
 * For r_i = float32((100 - 3 i) / 100), i = 0..10:
 *   s_i = bf16(float32(float32(absmax * r_i) / 7));
 *   q_i = clamp(rint(float32(w / s_i)), -8, 7) (0 when s_i == 0);
 *   e_i = sum over the group of (w - q_i * s_i)^2 in float64, summed in this
 *         order: runs of 4 consecutive elements in sequence, then five
 *         pairwise combinations of the 32 partial sums (element index xor 16,
 *         8, 4, 2, 1 runs);
 * and the smallest i with the least e_i is kept (i = 0 is w4a8_pack_int4).
 * Each e_i is within 2^-45 e_i of the exact squared error, so the kept
 * candidate is the exact MSE minimiser unless two candidates' exact errors
 * lie within that bound of each other (a near tie, where either is kept).
 * With r < 1 the code -8 occurs.  Arguments and errors as w4a8_pack_int4.
 */
W4A8_API w4a8_status w4a8_pack_int4_mse_clip(const void* w_bf16, int64_t R, int64_t K,
                                             int32_t group, int32_t* packed, void* scales_bf16,
                                             void* stream);

/*
 * w4a8_prepare_experts_b200 - lay out one projection's quantised experts the
 * way w4a8_moe_forward reads them.  The codes and scale values are those of
 * w4a8_pack_int4 (the pages fix the uint4b8 codes and the group-128 bf16
 * scales); only their placement in memory is this library's own.
 *
 * Words: inside every int32 word the nibble of element j (0..7) moves from
 * bits 4j..4j+3 to bits 8j..8j+3 for j < 4 and to bits 8(j-4)+4..8(j-4)+7 for
 * j >= 4.  Then (w & 0x0F0F0F0F) holds elements 0..3, one per byte, and
 * ((w >> 4) & 0x0F0F0F0F) elements 4..7; the grouped GEMM turns each such
 * byte u straight into the E4M3 value u * 2^-9 (exact for u = 0..15).  Word
 * order is unchanged, so the map is a bijection on words.
 * Scales: [E, rows, K / 128] -> group-major [E, K / 128, rows], so that the
 * scales of consecutive rows for one group are contiguous.
 *
 *   packed       [E, rows, K / 8] int32 from w4a8_pack_int4
 *   scales_bf16  [E, rows, K / 128] bf16 from w4a8_pack_int4
 *   E, rows, K   >= 0, >= 0, > 0 with K % 128 == 0 (E * rows == 0: no-op)
 *   packed_out   [E, rows, K / 8] int32, written; may be `packed` itself
 *                (in place) but must not partly overlap it
 *   scales_out   [E, K / 128, rows] bf16, written; must not overlap
 *                `scales_bf16`
 */
W4A8_API w4a8_status w4a8_prepare_experts_b200(const int32_t* packed, const void* scales_bf16,
                                               int64_t E, int64_t rows, int64_t K,
                                               int32_t* packed_out, void* scales_out,
                                               void* stream);

/*
 * w4a8_quant_act_fp8_per_token - dynamic per-token FP8 E4M3 quantisation.
 * (Model card, "quantisation method" and the table above: FP8 per-token
 * dynamic activations.)
 *
 * Per row t:  scale[t] = absmax(x[t]) / 448 (float32 division);
 * codes[t, :] = E4M3(x / scale[t]) rounded to nearest even, saturating to
 * +-448, sign of zero kept; a row whose absmax is 0 gets scale 0 and codes 0.
 *
 *   x_bf16      [T, H] bf16
 *   T, H        T >= 0 (T == 0 is a no-op); H > 0 and H % 16 == 0
 *   codes_e4m3  [T, H] uint8, written
 *   scales      [T] float32, written
 */
W4A8_API w4a8_status w4a8_quant_act_fp8_per_token(const void* x_bf16, int64_t T, int64_t H,
                                         uint8_t* codes_e4m3, float* scales, void* stream);

/*
 * w4a8_moe_route_workspace_size - bytes of scratch w4a8_moe_route_permute needs.
 */
W4A8_API size_t w4a8_moe_route_workspace_size(int64_t T, int32_t E);

/*
 * w4a8_moe_route_permute - top-k routing and the token -> expert permutation
 * that forms the grouped-GEMM segments (the layer's experts run as one
 * grouped GEMM per projection: model card intro "CUTLASS W4A8 grouped GEMM").
 *
 * Routing: per token, the k largest logits (a tie goes to the lower expert
 * id); slot j holds the j-th best.  topk_w = softmax of the k selected logits
 * (float32 arithmetic, the renormalised top-k).  Precondition: logits are not
 * NaN and each token has at least k finite logits.
 * Permutation: stable counting sort of the (t, j) pairs by expert.  Segment e
 * is rows [expert_offsets[e], expert_offsets[e+1]) and lists its tokens in
 * ascending order in sorted_token_ids; row_of[t, j] is the row of (t, j).
 *
 *   logits            [T, E] float32
 *   T, E, k           T >= 0; 1 <= E <= 1024; 1 <= k <= min(E, 32)
 *   topk_ids          [T, k] int32, written
 *   topk_w            [T, k] float32, written
 *   expert_offsets    [E + 1] int32, written
 *   sorted_token_ids  [T * k] int32, written
 *   row_of            [T, k] int32, written
 *   workspace         scratch of >= w4a8_moe_route_workspace_size(T, E) bytes
 */
W4A8_API w4a8_status w4a8_moe_route_permute(const float* logits, int64_t T, int32_t E, int32_t k,
                                   int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                                   int32_t* sorted_token_ids, int32_t* row_of,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * w4a8_moe_route_permute_noalloc - the same routing and permutation as
 * w4a8_moe_route_permute, for callers that cannot allocate device memory.
 * (The pages have no counterpart: this is a calling convention of this
 * library, not a step of the method.)
 *
 * Why: some callers may not call cudaMalloc where they route tokens -
 * runtimes and plugin interfaces that give a kernel only its planned inputs
 * and outputs and no scratch, and paths whose device memory budget is fixed in
 * advance.  This call takes no workspace and calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *
 * Scratch: a file-scope device array of 528,388 bytes (2 * 65536 + 1025
 * int32) that every device which loads the library holds until the process
 * exits.  Limit: ceil(T / 256) * E <= 65536 (for example T <= 65536 with
 * E = 256, or T <= 16384 with E = 1024); larger problems get
 * W4A8_ERR_UNSUPPORTED_SHAPE and should use w4a8_moe_route_permute.
 * Set-up: the first call on each device looks up the array's device address
 * with that device current and keeps it; make that first call before any
 * stream capture.  cudaDeviceReset discards the array, so after a reset of a
 * device the kept address is stale and this call must not be used on it.
 * Sharing: every call on a device uses the same array, which keeps the last
 * call's contents.  The histogram part is zeroed by each call on `stream`
 * and the rest is rewritten before it is read, but calls that overlap on the
 * GPU (different streams at the same time) race on it and must be ordered by
 * the caller.
 *
 * Arguments, outputs and errors are those of w4a8_moe_route_permute without
 * the workspace.
 */
W4A8_API w4a8_status w4a8_moe_route_permute_noalloc(const float* logits, int64_t T, int32_t E,
                                                    int32_t k, int32_t* topk_ids, float* topk_w,
                                                    int32_t* expert_offsets,
                                                    int32_t* sorted_token_ids, int32_t* row_of,
                                                    void* stream);

/*
 * Optional outputs and instrumentation of w4a8_moe_forward.  Every member may
 * be NULL.  A non-NULL buffer replaces the workspace region of the same
 * intermediate, so it receives exactly what the layer computed.  Shapes use
 * A = T * k assignments.
 */
typedef struct w4a8_moe_aux {
    int32_t* topk_ids;          /* [T, k] */
    float* topk_w;              /* [T, k] */
    int32_t* expert_offsets;    /* [E + 1] */
    int32_t* sorted_token_ids;  /* [A] */
    int32_t* row_of;            /* [T, k] */
    uint8_t* act_codes;         /* [T, H] E4M3 codes of the hidden states */
    float* act_scales;          /* [T] */
    float* inter_h;             /* [A, I] float32 SwiGLU output before requantisation */
    uint8_t* inter_codes;       /* [A, I] E4M3 codes of the intermediate (segment rows) */
    float* inter_scales;        /* [A] */
    float* y_rows;              /* [A, H] float32 down-projection output per segment row */
    /* If non-NULL: 2 * W4A8_NUM_STAGES cudaEvent_t handles (host memory array).
     * Event 2i is recorded before stage i and 2i+1 after it, on `stream`.
     * Stages: 0 activation quantisation, 1 routing + permutation, 2 gate/up
     * GEMM + SwiGLU, 3 intermediate requantisation, 4 down GEMM, 5 combine. */
    void* const* stage_events;
} w4a8_moe_aux;

/*
 * w4a8_moe_forward_launches - how many kernels one w4a8_moe_forward launches
 * for T tokens, E experts and top-k: 8, or 10 when the batch averages at
 * least 8 assignments per expert and each grouped GEMM runs as two launches
 * ("split tiling": experts with more than 32 segment rows in 128-row tiles,
 * the others in 32-row tiles; W4A8_SPLIT_TILES=0/1 forces it off/on).  The
 * per-channel INT8 variant never splits (8).  Host arithmetic only; 0 for
 * T <= 0.
 */
W4A8_API int32_t w4a8_moe_forward_launches(int64_t T, int32_t E, int32_t k);

/*
 * w4a8_moe_workspace_size - bytes of scratch w4a8_moe_forward needs.
 */
W4A8_API size_t w4a8_moe_workspace_size(int64_t T, int64_t H, int64_t I, int32_t E, int32_t k);

/*
 * w4a8_moe_forward - one W4A8 routed-expert MoE layer.
 *
 *   1. activation quantisation (as w4a8_quant_act_fp8_per_token);
 *   2. routing + permutation (as w4a8_moe_route_permute);
 *   3. gate/up grouped GEMM on the tensor cores: for segment row r of expert
 *      e, G[r, n] = a_s[t] * sum_g s13[e, n, g] * sum_{kappa in g}
 *      e4m3(x[t, kappa]) * q13[e, n, kappa]; INT4 is converted to E4M3 (exact
 *      for -8..7) in the kernel, each 128-wide K group is accumulated in FP32
 *      and scaled by its group scale; then h = silu(G[:, :I]) * G[:, I:];
 *   4. per-row FP8 requantisation of h (same rule as step 1);
 *   5. down grouped GEMM: Y[r, n] = h_s[r] * sum_g s2[e, n, g] * sum e4m3 * q2;
 *   6. combine: out[t] = bf16(sum_j topk_w[t, j] * Y[row_of[t, j]]), slot order.
 *
 * The GEMMs multiply E4M3 activations by the stored nibbles u = q + 8 (each
 * turned into the exact E4M3 value u * 2^-9) and remove the offset per group:
 * sum a * q = 512 * sum a * (u * 2^-9) - 8 * sum a, where sum a is the group
 * sum of the E4M3 activation values, which steps 1 and 4 also write.
 *
 *   hidden_bf16   [T, H] bf16
 *   logits        [T, E] float32 router logits
 *   w13_packed    [E, 2I, H / 8] int32: w4a8_pack_int4 of the [E*2I, H]
 *                 gate/up weight, then w4a8_prepare_experts_b200; rows
 *                 [0, I) of each expert are the gate projection, rows
 *                 [I, 2I) the up projection
 *   w13_scales    [E, H / 128, 2I] bf16 (group-major, from
 *                 w4a8_prepare_experts_b200)
 *   w2_packed     [E, H, I / 8] int32, packed then prepared the same way
 *   w2_scales     [E, I / 128, H] bf16 (group-major)
 *   T, H, I, E, k T >= 0 (0: no-op); H and I positive multiples of 128, at
 *                 most 8192 each; 1 <= E <= 1024; 1 <= k <= min(E, 32)
 *   out_bf16      [T, H] bf16, written
 *   workspace     scratch of >= w4a8_moe_workspace_size(T, H, I, E, k) bytes
 *   aux           optional, see w4a8_moe_aux (NULL for none)
 */
W4A8_API w4a8_status w4a8_moe_forward(const void* hidden_bf16, const float* logits,
                             const int32_t* w13_packed, const void* w13_scales,
                             const int32_t* w2_packed, const void* w2_scales,
                             int64_t T, int64_t H, int64_t I, int32_t E, int32_t k,
                             void* out_bf16, void* workspace, size_t workspace_bytes,
                             const w4a8_moe_aux* aux, void* stream);

/*
 * The per-channel INT4 weight / per-token INT8 activation variant
 * ("GLM-5.3-Channel-INT4-w4a8" model card, quantisation table: RTN, static,
 * per-channel INT4 routed experts; dynamic per-token INT8 activations).
 *
 * w4a8_pack_int4_channel - per output row: s = bf16(float32(absmax / 7)) over
 * the whole row, q = clamp(rint(float32(w / s)), -8, 7) (0 when s == 0),
 * packed as w4a8_pack_int4 packs (uint4b8, 8 per int32, little-endian).
 *   w_bf16       [R, K] bf16; K > 0, K % 128 == 0
 *   packed       [R, K / 8] int32, written
 *   scales_bf16  [R] bf16, written
 */
W4A8_API w4a8_status w4a8_pack_int4_channel(const void* w_bf16, int64_t R, int64_t K,
                                            int32_t* packed, void* scales_bf16, void* stream);

/*
 * w4a8_prepare_experts_channel_b200 - the words of w4a8_prepare_experts_b200
 * (same nibble interleave) plus, per row, the sum over K of the stored
 * nibbles u = q + 8 (the INT8 GEMM multiplies unsigned bytes and removes the
 * offsets with these sums).  Scales are used as packed ([E, rows] bf16).
 *   packed       [E, rows, K / 8] int32 from w4a8_pack_int4_channel
 *   packed_out   [E, rows, K / 8] int32, written; may be `packed` (in place)
 *   nibble_sums  [E, rows] int32, written
 */
W4A8_API w4a8_status w4a8_prepare_experts_channel_b200(const int32_t* packed, int64_t E,
                                                       int64_t rows, int64_t K,
                                                       int32_t* packed_out, int32_t* nibble_sums,
                                                       void* stream);

/*
 * w4a8_moe_forward_channel_int8 - the layer of w4a8_moe_forward with
 * per-channel INT4 experts and per-token INT8 activations:
 *   a[t] = clamp(rint(float32(x[t] / sa[t])), -127, 127), sa[t] = float32(absmax / 127);
 *   G[r, n] = sa[t] * s13[e, n] * sum_k a[t, k] * q13[e, n, k]   (exact int32 sums);
 *   h = silu(G[:, :I]) * G[:, I:]; h requantised per segment row to INT8 by the
 *   same rule; Y[r, n] = sh[r] * s2[e, n] * sum_k c[r, k] * q2[e, n, k];
 *   combine as w4a8_moe_forward.
 * The grouped GEMMs run tcgen05 kind::i8 MMAs on unsigned bytes (stored nibble
 * u = q + 8, activation code + 128) with one int32 accumulator per tile and
 * remove both offsets exactly with the per-row nibble sums and per-token code
 * sums.  Routing, permutation, workspace (w4a8_moe_workspace_size) and aux as
 * w4a8_moe_forward, except that aux->act_codes and aux->inter_codes receive
 * the INT8 codes stored offset-binary (code + 128).
 *   w13_packed / w2_packed  from w4a8_prepare_experts_channel_b200
 *   w13_scales [E, 2I] bf16, w2_scales [E, H] bf16 (from w4a8_pack_int4_channel)
 *   w13_nibble_sums [E, 2I], w2_nibble_sums [E, H] int32
 */
W4A8_API w4a8_status w4a8_moe_forward_channel_int8(
    const void* hidden_bf16, const float* logits, const int32_t* w13_packed,
    const void* w13_scales, const int32_t* w13_nibble_sums, const int32_t* w2_packed,
    const void* w2_scales, const int32_t* w2_nibble_sums, int64_t T, int64_t H, int64_t I,
    int32_t E, int32_t k, void* out_bf16, void* workspace, size_t workspace_bytes,
    const w4a8_moe_aux* aux, void* stream);

/* ---------------------------------------------------------------------------
 * The FP8-block shared expert.
 *
 * GLM-5.3-W4A8 model card, intro and "quantisation method" (item on the
 * non-expert layers): only the routed experts are INT4; the shared expert
 * keeps the official FP8 format, E4M3 weights with one float32 scale per
 * 128 x 128 block.  Readings where the pages are silent: the block scale is
 * absmax / 448 (float32 division) for weights quantised here; the expert's
 * activations are quantised at run time per token and 128-wide channel group
 * (scale = absmax / 448); the intermediate h is requantised the same way;
 * the layer adds the shared expert's output to the routed sum before the
 * bf16 rounding of the combine.
 * ------------------------------------------------------------------------- */

/*
 * w4a8_quant_fp8_block - bf16 w [R, K] -> E4M3 codes [R, K] (uint8) and
 * float32 scales [R / 128, K / 128]: per 128 x 128 block, scale =
 * float32(absmax / 448), code = E4M3 round-to-nearest-even, saturating, of
 * float32(w / scale); an all-zero block gets scale 0 and codes 0.
 * R and K multiples of 128 (else W4A8_ERR_UNSUPPORTED_SHAPE), R / 128 <= 65535.
 */
W4A8_API w4a8_status w4a8_quant_fp8_block(const void* w_bf16, int64_t R, int64_t K,
                                          uint8_t* codes, float* scales, void* stream);

/*
 * w4a8_quant_act_fp8_group - bf16 x [T, H] -> E4M3 codes [T, H] and float32
 * scales [T, H / 128]: per token and 128-wide group, scale =
 * float32(absmax / 448), code = E4M3(float32(x / scale)); scale 0 -> codes 0.
 * H a multiple of 128.
 */
W4A8_API w4a8_status w4a8_quant_act_fp8_group(const void* x_bf16, int64_t T, int64_t H,
                                              uint8_t* codes, float* scales, void* stream);

/* Optional outputs of the shared expert (each NULL = not wanted). */
typedef struct w4a8_shared_aux {
    uint8_t* act_codes;   /* [T, H] E4M3 codes of the input */
    float* act_scales;    /* [T, H / 128] */
    float* h;             /* [T, I] float32 SwiGLU output before requantisation */
    uint8_t* h_codes;     /* [T, I] */
    float* h_scales;      /* [T, I / 128] */
    /* If non-NULL: 8 cudaEvent_t handles (host memory array), recorded on
     * `stream` before / after: input quantisation (0/1), gate/up GEMM (2/3),
     * requantisation of h (4/5), down GEMM (6/7). */
    void* const* stage_events;
} w4a8_shared_aux;

W4A8_API size_t w4a8_shared_expert_workspace_size(int64_t T, int64_t H, int64_t I);

/*
 * w4a8_shared_expert_forward - the FP8-block SwiGLU expert on T tokens:
 *   a = w4a8_quant_act_fp8_group(hidden);
 *   G[t, n] = sum_g a_s[t, g] * s13[n / 128, g] * sum_{kappa in g} a[t, kappa] * w13[n, kappa]
 *             for n < 2I (tensor cores: E4M3 x E4M3 products exact, float32
 *             accumulation, one float32 promotion per 128-wide group);
 *   h = silu(G[:, :I]) * G[:, I:];  h requantised per token and 128-group;
 *   y[t, n] = sum_g h_s[t, g] * s2[n / 128, g] * sum h[t, kappa] * w2[n, kappa].
 * hidden bf16 [T, H]; w13_codes [2I, H] and w2_codes [H, I] E4M3 with
 * float32 block scales [2I / 128, H / 128] and [H / 128, I / 128] (as
 * w4a8_quant_fp8_block writes them); y float32 [T, H].  H and I multiples of
 * 128, at most 64 groups each.
 */
W4A8_API w4a8_status w4a8_shared_expert_forward(
    const void* hidden_bf16, const uint8_t* w13_codes, const float* w13_scales,
    const uint8_t* w2_codes, const float* w2_scales, int64_t T, int64_t H, int64_t I,
    float* y, void* workspace, size_t workspace_bytes, const w4a8_shared_aux* aux, void* stream);

W4A8_API size_t w4a8_moe_shared_workspace_size(int64_t T, int64_t H, int64_t I, int32_t E,
                                               int32_t k, int64_t I_shared);

/*
 * w4a8_moe_forward_shared - w4a8_moe_forward plus the FP8-block shared
 * expert (ws13 [2 I_shared, H], ws2 [H, I_shared], as for
 * w4a8_shared_expert_forward), in the same call:
 *   out[t] = bf16_rn(sum_j topk_w[t, j] * Y[row_of[t, j]] + y_shared[t]).
 * The routed arguments, aux and errors are those of w4a8_moe_forward;
 * shared_aux those of w4a8_shared_expert_forward.  The workspace size is
 * w4a8_moe_shared_workspace_size.
 * Decode-sized calls (T k <= 32 E, without split tiling) run the shared
 * expert's two GEMMs inside the routed GEMM launches, as their second phase
 * (each CTA takes shared tiles after its routed ones); the shared stage
 * events 2/3 and 6/7 then bracket nothing and the routed GEMM stages include
 * the shared GEMMs.  The environment variable W4A8_SHARED_FUSED=0 keeps them
 * in launches of their own.
 */
W4A8_API w4a8_status w4a8_moe_forward_shared(
    const void* hidden_bf16, const float* logits, const int32_t* w13_packed,
    const void* w13_scales, const int32_t* w2_packed, const void* w2_scales,
    const uint8_t* ws13_codes, const float* ws13_scales, const uint8_t* ws2_codes,
    const float* ws2_scales, int64_t T, int64_t H, int64_t I, int64_t I_shared, int32_t E,
    int32_t k, void* out_bf16, void* workspace, size_t workspace_bytes, const w4a8_moe_aux* aux,
    const w4a8_shared_aux* shared_aux, void* stream);

/*
 * Expert parallelism: the layer split by expert over G ranks (GLM-5.3-W4A8
 * model card, "performance" table: TP8+EP and 2 x (TP4+EP); "deployment": the
 * W4A8 checkpoint must run with expert parallelism).  Rank g owns a contiguous
 * range of experts.  One step: every rank quantises its own tokens
 * (w4a8_quant_act_fp8_per_token) and routes them (w4a8_moe_route_topk); the
 * ranks all-gather the E4M3 codes, token scales, expert ids and weights (the
 * dispatch); each rank runs w4a8_moe_forward_experts on the gathered tokens
 * for its own experts, giving float32 partial sums; the ranks reduce-scatter
 * (sum) the partial sums back to the tokens' owners (the combine), and each
 * rounds its tokens once to bf16 (w4a8_cast_f32_bf16).  The collectives are
 * the caller's (NCCL); these calls only compute.
 */

/*
 * w4a8_moe_route_topk - the top-k step of w4a8_moe_route_permute alone: the
 * same ids (ties to the lower expert id) and softmax-renormalised weights,
 * without the permutation.  Arguments and errors as w4a8_moe_route_permute;
 * no workspace.
 */
W4A8_API w4a8_status w4a8_moe_route_topk(const float* logits, int64_t T, int32_t E, int32_t k,
                                         int32_t* topk_ids, float* topk_w, void* stream);

/*
 * w4a8_moe_experts_workspace_size - bytes of scratch w4a8_moe_forward_experts
 * needs for T (gathered) tokens and e_count local experts.
 */
W4A8_API size_t w4a8_moe_experts_workspace_size(int64_t T, int64_t H, int64_t I,
                                                int32_t e_count, int32_t k);

/*
 * w4a8_moe_forward_experts - steps 3-6 of w4a8_moe_forward for the experts
 * e_begin .. e_begin + e_count - 1 only, from activations already quantised
 * and tokens already routed; the combine writes float32 sums instead of bf16:
 *
 *   partial_out[t] = sum over the slots j of token t whose expert is local,
 *                    in slot order, of topk_w[t, j] * Y[t, j]
 *
 * (0 for a token with no local slot).  Summed over ranks whose ranges cover
 * [0, E) and rounded to bf16, this is w4a8_moe_forward's output up to the
 * float32 summation order.  The permutation is the stable counting sort of
 * w4a8_moe_route_permute restricted to the local experts.
 *
 *   act_codes     [T, H] uint8 E4M3 codes (w4a8_quant_act_fp8_per_token)
 *   act_scales    [T] float32 token scales
 *   topk_ids      [T, k] int32 expert ids in [0, E), or -1 for an empty
 *                 slot (a padding token); any other id sets the device latch
 *                 (W4A8_ERR_DEVICE_INDEX at the next w4a8_check_device_error)
 *                 and its slot is skipped
 *   topk_w        [T, k] float32 routing weights
 *   T, H, I, E, k as w4a8_moe_forward (T = all ranks' tokens)
 *   e_begin, e_count  0 <= e_begin, 1 <= e_count, e_begin + e_count <= E
 *   w13_packed, w13_scales, w2_packed, w2_scales
 *                 the LOCAL experts only, laid out as for w4a8_moe_forward
 *                 ([e_count, 2I, H / 8], [e_count, H / 128, 2I], ...)
 *   partial_out   [T, H] float32, written
 *   workspace     >= w4a8_moe_experts_workspace_size(T, H, I, e_count, k) bytes
 */
W4A8_API w4a8_status w4a8_moe_forward_experts(
    const uint8_t* act_codes, const float* act_scales, const int32_t* topk_ids,
    const float* topk_w, int64_t T, int64_t H, int64_t I, int32_t E, int32_t k, int32_t e_begin,
    int32_t e_count, const int32_t* w13_packed, const void* w13_scales, const int32_t* w2_packed,
    const void* w2_scales, float* partial_out, void* workspace, size_t workspace_bytes,
    void* stream);

/*
 * w4a8_cast_f32_bf16 - out = bf16(x), round to nearest even: the single bf16
 * rounding of the expert-parallel combine, after the partial sums are reduced.
 *
 *   x         [n] float32;  n >= 0, n % 8 == 0 (0: no-op)
 *   out_bf16  [n] bf16, written
 */
W4A8_API w4a8_status w4a8_cast_f32_bf16(const float* x, int64_t n, void* out_bf16, void* stream);

/*
 * The all-to-all(v) form of the dispatch and combine (for large batches, where
 * sending every token to every rank would cost more than the per-step
 * exchange of counts): each rank routes its own tokens, sends each token
 * once to every rank that owns one of its k experts, and adds up the partial
 * sums that come back.  Rank r of n_ranks owns the contiguous expert range in
 * which the first E % n_ranks ranks hold one more expert than the others.
 * One step on a rank with T tokens:
 *   1. w4a8_quant_act_fp8_per_token and w4a8_moe_route_topk on its tokens;
 *   2. w4a8_ep_dispatch_plan: how many of its tokens go to each rank, which,
 *      and where each (token, rank) pair sits in the send buffers;
 *   3. an all-to-all of the counts, w4a8_ep_gather_rows into the send
 *      buffers, and all-to-all(v) of the codes, scales, ids and weights;
 *   4. w4a8_moe_forward_experts on the rows received (its own experts);
 *   5. an all-to-all(v) of the partial sums back to the senders, and
 *      w4a8_ep_combine_rows: each token's returned rows summed in rank order
 *      and rounded once to bf16.
 * The collectives are the caller's (NCCL between GPUs).
 *
 * w4a8_ep_dispatch_plan - for each rank r, the tokens that go to r: token t
 * goes to r once when at least one of its ids lies in r's range; ids outside
 * [0, E) (the -1 of an empty slot) go nowhere.
 *
 *   topk_ids       [T, k] int32 (device)
 *   T, k, E        T >= 0, k >= 1, E >= 1
 *   n_ranks        1 .. 64
 *   send_counts    [n_ranks] int32 (device), written: tokens for each rank
 *   send_rows      [send_rows_capacity] int32 (device), written: rank 0's
 *                  tokens in ascending order, then rank 1's, and so on
 *                  (sum(send_counts) entries)
 *   send_rows_capacity  >= T * min(k, n_ranks)
 *   pos            [T, n_ranks] int32 (device), written: the index in
 *                  send_rows of (t, r), or -1 when t does not go to r
 * Errors: INVALID_ARG (NULL pointer, capacity too small, k or E < 1),
 * UNSUPPORTED_SHAPE (n_ranks outside 1..64).  T = 0 writes zero counts.
 */
W4A8_API w4a8_status w4a8_ep_dispatch_plan(const int32_t* topk_ids, int64_t T, int32_t k,
                                           int32_t E, int32_t n_ranks, int32_t* send_counts,
                                           int32_t* send_rows, int64_t send_rows_capacity,
                                           int32_t* pos, void* stream);

/*
 * w4a8_ep_gather_rows - the send buffers: row i of each output is row
 * send_rows[i] of the rank's quantised tokens.
 *
 *   codes [T, H] uint8, scales [T] float32, topk_ids [T, k] int32,
 *   topk_w [T, k] float32   the rank's tokens (device)
 *   T, H, k        H % 16 == 0
 *   send_rows      [n_rows] int32 token indices in [0, T) (device)
 *   codes_out [n_rows, H], scales_out [n_rows], ids_out [n_rows, k],
 *   w_out [n_rows, k]       written (device)
 * codes and codes_out 16-byte aligned.  An index outside [0, T) is skipped
 * by the bounds-checking build (which raises the device latch) and is
 * undefined behaviour in the release build.
 */
W4A8_API w4a8_status w4a8_ep_gather_rows(const uint8_t* codes, const float* scales,
                                         const int32_t* topk_ids, const float* topk_w, int64_t T,
                                         int64_t H, int32_t k, const int32_t* send_rows,
                                         int64_t n_rows, uint8_t* codes_out, float* scales_out,
                                         int32_t* ids_out, float* w_out, void* stream);

/*
 * w4a8_ep_combine_rows - the combine after the partial sums come back:
 *   out[t] = bf16(sum over r = 0 .. n_ranks-1 with pos[t, r] >= 0 of
 *                 back[pos[t, r]])
 * summed in float32 in rank order and rounded to nearest even once; a token
 * that went to no rank gets zeros.
 *
 *   back       [n_rows, H] float32 (device): row i = the partial sums of the
 *              token-rank pair at send_rows index i
 *   pos        [T, n_ranks] int32 from w4a8_ep_dispatch_plan (device)
 *   out_bf16   [T, H] bf16, written;  H % 8 == 0, back and out 16-byte aligned
 */
W4A8_API w4a8_status w4a8_ep_combine_rows(const float* back, int64_t n_rows, int64_t H,
                                          const int32_t* pos, int64_t T, int32_t n_ranks,
                                          void* out_bf16, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* W4A8_H_ */
