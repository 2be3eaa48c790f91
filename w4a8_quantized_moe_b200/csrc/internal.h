// internal.h - launchers shared between the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda.h>

namespace w4a8 {

constexpr int kGroup = 128;        // INT4 group size along K
constexpr int kRouteTok = 256;     // tokens per routing block
constexpr int kTileNDecode = 32;   // tokens per grouped-GEMM tile, decode shape
constexpr int kTileNPrefill = 128; // tokens per grouped-GEMM tile, prefill shape
constexpr int kTileNShared = 64;   // tokens per tile of the shared expert in a routed decode launch
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kMaxGroups = 64;     // K / 128 per GEMM (K <= 8192)

// Bits of the device error latch.
constexpr int kDeviceErrorTimeout = 1;  // a bounded in-kernel wait ran out
constexpr int kDeviceErrorIndex = 2;    // an index was out of range (the access was skipped)

inline int64_t route_blocks(int64_t T) { return (T + kRouteTok - 1) / kRouteTok; }
// Three-part group sums (per-tile offset correction): one part spans Gp =
// K / 128 groups rounded up to 16 columns; a row holds the three parts and is
// at least 64 columns (one 128-byte TMA box) long.
__host__ __device__ inline int64_t sum_part_cols(int64_t K) { return ((K / kGroup) + 15) / 16 * 16; }
__host__ __device__ inline int64_t sum_parts_ld(int64_t K) {
  return 3 * sum_part_cols(K) < 64 ? 64 : 3 * sum_part_cols(K);
}

// ---- kernels_small.cu
// gsum (nullable): [T, H / 128] sums of the E4M3 values of each 128-wide group.
// perm (nullable): [T * k, H] codes in expert-segment order; row r = row_of[t, j]
// receives token t's codes for every slot j.
// int8_row_sum (non-null): INT8 mode instead of E4M3 -- codes are offset-binary
// (code + 128) and the row sums of those bytes go to int8_row_sum [T].
// sum_parts (nullable, needs perm): [T * k, sum_parts_ld(H)] bf16; segment row r gets each group sum S as three bf16 parts p0 =
// bf16(S), p1 = bf16(S - p0), p2 = bf16(S - p0 - p1) at columns g, Gp + g,
// 2 Gp + g, and zeros at the padding columns.
cudaError_t launch_act_quant(const void* x, int64_t T, int64_t H, uint8_t* codes, float* scales,
                             float* gsum, const int32_t* row_of, int k, uint8_t* perm,
                             int num_sms, cudaStream_t s, int32_t* int8_row_sum = nullptr,
                             uint16_t* sum_parts = nullptr);
// clip_search: the per-group MSE search over 11 shrink ratios instead of absmax / 7.
cudaError_t launch_pack_int4(const void* w, int64_t R, int64_t K, int32_t* packed, void* scales,
                             bool clip_search, int num_sms, cudaStream_t s);
// Split tiling of the grouped GEMMs: with tile_prefix_wide set, experts with
// more than wide_min segment rows are tiled tile_n_wide rows at a time in
// tile_prefix_wide (and get no tiles in tile_prefix), the others tile_n at a
// time in tile_prefix only.
struct SplitTiles {
  int wide_min = -1;
  int tile_n_wide = 0;
  int32_t* tile_prefix_wide = nullptr;
};
// routing: top-k + per-block expert histogram; scan; stable scatter.
// tile_prefix[e] = sum over experts e' < e of ceil(count[e'] / tile_n).
cudaError_t launch_route(const float* logits, int64_t T, int E, int k, int32_t* topk_ids,
                         float* topk_w, int32_t* expert_offsets, int32_t* sorted_token_ids,
                         int32_t* row_of, int32_t* block_counts, int32_t* block_base,
                         int32_t* tile_prefix, int tile_n, uint32_t* row_amax_to_zero,
                         cudaStream_t s, const SplitTiles& split = SplitTiles());
// Top-k and weights only (no histogram, no permutation).
cudaError_t launch_route_topk(const float* logits, int64_t T, int E, int k, int32_t* topk_ids,
                              float* topk_w, cudaStream_t s);
// Expert parallelism: the permutation of given ids restricted to the E_loc
// experts e_lo .. e_lo + E_loc - 1 of E_all (segments, offsets and tile prefix
// over the local experts only; row_of = -1 for other experts' slots).  Ids
// outside [-1, E_all) set kDeviceErrorIndex in *latch and are skipped.
cudaError_t launch_route_local(const int32_t* topk_ids, int64_t T, int E_all, int k, int e_lo,
                               int E_loc, int32_t* expert_offsets, int32_t* sorted_token_ids,
                               int32_t* row_of, int32_t* block_counts, int32_t* block_base,
                               int32_t* tile_prefix, int tile_n, uint32_t* row_amax_to_zero,
                               int* latch, int num_sms, cudaStream_t s,
                               const SplitTiles& split = SplitTiles());
// Segment row r < *rows_total (device) receives the codes of token
// sorted_token_ids[r]; the group sums go to gsum [T, H / 128] by token, or to
// the row's three-part sums (sum_parts, [max_rows, sum_parts_ld(H)]).
cudaError_t launch_ep_gather(const uint8_t* codes, int64_t T, int64_t H,
                             const int32_t* sorted_token_ids, const int32_t* rows_total,
                             int64_t max_rows, uint8_t* perm, float* gsum, uint16_t* sum_parts,
                             int num_sms, cudaStream_t s);
// Expert-parallel all-to-all(v) dispatch (ranks <= kEpMaxRanks): the plan
// (per-rank token counts, the rank-major token list, the (token, rank) -> list
// index map or -1), the send-row gather and the combine of the returned rows.
constexpr int kEpMaxRanks = 64;
cudaError_t launch_ep_plan(const int32_t* topk_ids, int64_t T, int k, int E, int n_ranks,
                           int32_t* counts, int32_t* rows, int32_t* pos, cudaStream_t s);
cudaError_t launch_ep_gather_rows(const uint8_t* codes, const float* scales, const int32_t* ids,
                                  const float* w, int64_t T, int64_t H, int k, const int32_t* rows,
                                  int64_t n_rows, uint8_t* codes_out, float* scales_out,
                                  int32_t* ids_out, float* w_out, int num_sms, cudaStream_t s);
cudaError_t launch_ep_combine_rows(const float* back, int64_t n_rows, int64_t H,
                                   const int32_t* pos, int64_t T, int n_ranks, void* out,
                                   int num_sms, cudaStream_t s);
// bf16 = round-to-nearest-even(x), n a multiple of 8.
cudaError_t launch_cast_bf16(const float* x, int64_t n, void* out, int num_sms, cudaStream_t s);
// sum_parts (nullable): [A, sum_parts_ld(I)] bf16 as for launch_act_quant.
// rows_dev (nullable): device-side row count (min with A) when only the
// device knows it.
cudaError_t launch_inter_quant(const float* h, const uint32_t* row_amax, int64_t A, int64_t I,
                               uint8_t* codes, float* scales, float* gsum, int num_sms,
                               cudaStream_t s, int32_t* int8_row_sum = nullptr,
                               uint16_t* sum_parts = nullptr, const int32_t* rows_dev = nullptr);
// packed uint4b8 words -> the word-local nibble interleave the grouped GEMM reads.
cudaError_t launch_repack_int4_b200(const int32_t* in, int64_t nwords, int32_t* out, int num_sms,
                                    cudaStream_t s);
// bf16 weight scales [E, rows, G] -> group-major [E, G, rows].
cudaError_t launch_transpose_scales(const void* in, int64_t E, int64_t rows, int64_t G, void* out,
                                    int num_sms, cudaStream_t s);
// per-channel INT4: scales bf16 [R] = bf16(row absmax / 7).
cudaError_t launch_pack_int4_channel(const void* w, int64_t R, int64_t K, int32_t* packed,
                                     void* scales, int num_sms, cudaStream_t s);
// sums[r] = sum of the 2 * 4 * words_per_row stored nibbles of row r.
cudaError_t launch_nibble_row_sum(const int32_t* packed, int64_t R, int64_t words_per_row,
                                  int32_t* sums, int num_sms, cudaStream_t s);
// y_shared (nullable): [T, H] float32 added to each token's routed sum.
// partial_f32 (nullable): write the float32 sum over the slots with a row
// (row_of >= 0) there instead of the bf16 output (expert parallelism).
cudaError_t launch_combine(const float* y, const int32_t* row_of, const float* topk_w, int64_t T,
                           int64_t H, int k, void* out, int num_sms, cudaStream_t s,
                           const float* y_shared = nullptr, float* partial_f32 = nullptr);
// FP8 block weights: bf16 [R, K] -> E4M3 codes [R, K] + float32 scales
// [R / 128, K / 128], scale = absmax / 448 per 128 x 128 block.
cudaError_t launch_quant_fp8_block(const void* w, int64_t R, int64_t K, uint8_t* codes,
                                   float* scales, cudaStream_t s);
// Per-row, per-128-group E4M3 activations from bf16 (x_bf16) or float32 (x_f32)
// input: codes [T, H], scales [T, H / 128].
cudaError_t launch_act_quant_group(const void* x_bf16, const float* x_f32, int64_t T, int64_t H,
                                   uint8_t* codes, float* scales, int num_sms, cudaStream_t s);
// expert_offsets {0, T} and tile prefix {0, ceil(T / tile_n)} of a dense GEMM.
cudaError_t launch_dense_tables(int32_t* offsets, int32_t* tile_prefix, int64_t T, int tile_n,
                                cudaStream_t s);

// ---- grouped_gemm.cu
struct GemmArgs {
  int K;                          // reduction length (H for gate/up, I for down)
  int n_rows;                     // weight rows per expert (2I or H)
  int half_rows;                  // gate/up: I (first up row); down: 0
  int E;
  const int32_t* expert_offsets;  // [E + 1]
  const int32_t* tile_prefix;     // [E + 1] prefix of ceil(count / tile width of the shape)
  const int32_t* row_tokens;      // gate/up: sorted_token_ids (token of each row); down: nullptr
  const float* act_scale;         // gate/up: per token [T]; down: per segment row [A]
  const float* act_gsum;          // [rows, K / 128] E4M3 group sums (by token / segment row)
  const void* wscale;             // bf16 [E, K / 128, n_rows] (group-major)
  float* out;                     // gate/up: h [A, I]; down: Y [A, H]
  int64_t out_ld;
  uint32_t* row_amax;             // gate/up only: float bits of max |h| per segment row
  int64_t act_rows;               // rows of the activation tensor (T or A)
  int nb_fastest;                 // tile order within an expert (see grouped_gemm.cu)
  // INT8 per-channel mode only: wscale is bf16 [E, n_rows] (one scale per row)
  const int32_t* wsum;            // [E, n_rows] sum over K of the stored nibbles u = q + 8
  const int32_t* act_sum;         // per token (gate/up) or row (down): sum of code + 128
  uint64_t timeout_ns;
  // buffer bounds for the debug build's index checks (W4A8_DEBUG_BOUNDS): the
  // segment rows of the activation / output tensors, and the tokens row_tokens
  // may name
  int64_t n_seg_rows;
  int64_t n_tokens;
};
// decode = the shape for few tokens per expert (see grouped_gemm.cu).
// tmap_sc: the group-major weight scales as bytes [E * K / 128, 2 * n_rows],
// box [K / 128 rows, 128 bytes (gate/up) or 256 bytes (down)].
// tmap_gs (read only when grouped_gemm_uses_sum_parts(decode)): the rows' E4M3
// group sums as three bf16 parts, bytes [act rows, 2 * sum_parts_ld(K)], part p
// of group g at column p * Gp + g (Gp = sum_part_cols(K)), zero up to 3 * Gp;
// box [16 rows x 128 bytes], 128-byte swizzle.
cudaError_t launch_grouped_gemm(bool gate_up, bool decode, const CUtensorMap& tmap_w,
                                const CUtensorMap& tmap_act, const CUtensorMap& tmap_sc,
                                const CUtensorMap& tmap_gs, const GemmArgs& a, int num_ctas,
                                cudaStream_t s);
int grouped_gemm_tile_n(bool decode);
// Whether the shape for this regime removes the +8 nibble offset once per
// tile (and so reads the three-part group sums instead of act_gsum).
bool grouped_gemm_uses_sum_parts(bool decode);
// The per-channel INT4 x per-token INT8 grouped GEMM (kind::i8, one int32
// accumulator per tile); tmap_act holds offset-binary codes.
cudaError_t launch_grouped_gemm_i8(bool gate_up, bool decode, const CUtensorMap& tmap_w,
                                   const CUtensorMap& tmap_act, const GemmArgs& a, int num_ctas,
                                   cudaStream_t s);
// The routed projection (as launch_grouped_gemm with the default decode
// shapes, no split tiling) and the shared expert's (as launch_fp8_block_gemm,
// tiles of grouped_gemm_shared_tile_n() token rows) in one launch.
// cudaErrorNotSupported for the prefill shapes and when a shape is forced by
// the environment: the caller then launches the two apart.
cudaError_t launch_grouped_gemm_with_shared(bool gate_up, bool decode, const CUtensorMap& tmap_w,
                                            const CUtensorMap& tmap_act,
                                            const CUtensorMap& tmap_sc,
                                            const CUtensorMap& tmap_gs,
                                            const CUtensorMap& shared_w,
                                            const CUtensorMap& shared_act, const GemmArgs& a,
                                            const GemmArgs& shared, int num_ctas,
                                            cudaStream_t s);
int grouped_gemm_shared_tile_n();
// Whether the decode shapes in use are the defaults the two-phase launch takes.
bool grouped_gemm_shared_fusable();
// Dense GEMM with E4M3 weights and 128 x 128 block scales (one expert, E = 1):
// tmap_w = codes [n_rows, K] bytes, box [64 (gate/up) or 128 rows x 128 B],
// 128-byte swizzle; wscale = float32 [n_rows / 128, K / 128]; act_gsum = the
// activations' float32 group scales [rows, K / 128]; act_scale, row_tokens
// and row_amax unused (null).
cudaError_t launch_fp8_block_gemm(bool gate_up, const CUtensorMap& tmap_w,
                                  const CUtensorMap& tmap_act, const GemmArgs& a, int num_ctas,
                                  cudaStream_t s);
// One bounded wait on an mbarrier nothing arrives on (failure-detection self-test).
cudaError_t launch_wait_timeout_selftest(uint64_t timeout_ns, cudaStream_t s);
// Device address (current device) of the library's one error latch, for
// kernels outside grouped_gemm.cu: they atomicOr kDeviceErrorIndex into it.
// w4a8_check_device_error() reads and clears it.
cudaError_t device_error_latch(int** latch);

}  // namespace w4a8
