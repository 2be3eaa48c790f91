// grouped_gemm.cu - W4A8 grouped GEMM on the sm_100a tensor cores.
//
// One persistent kernel runs either projection of every expert:
//   gate/up: G[r, n] = a_s[t_r] * sum_g s13[e, n, g] * P_g(r, n),  n < 2I
//            then h = silu(G[:, :I]) * G[:, I:] and the row absmax of h;
//   down:    Y[r, n] = h_s[r]   * sum_g s2[e, n, g]  * P_g(r, n),  n < H
// with P_g the exact E4M3 x INT4 dot product over the 128-wide K group g
// (GLM-5.3-W4A8 model card, intro and "quantisation method": INT4 group-128
// experts, INT4 turned into FP8 inside the kernel, no BF16 dequantisation).
//
// INT4 -> E4M3 in three integer instructions per 8 weights.  A byte 0x0u
// whose high nibble is zero is the E4M3 value u * 2^-9 for every u in 0..15
// (subnormals for u < 8, the first normal binade for u >= 8), exactly.  So
// the stored nibble u = q + 8 goes to the MMA as u * 2^-9 once each nibble sits
// alone in a byte; with the B200 weight layout (nibbles interleaved inside each
// word, see w4a8_prepare_experts_b200) that is w & 0x0F0F0F0F and
// (w >> 4) & 0x0F0F0F0F.  The MMA then yields D_g = 2^-9 * sum a * (q + 8), and
//   P_g = 512 * D_g - 8 * S_g,   S_g = sum over the group of the E4M3
// activation values, which the activation quantisers write next to the codes.
// Every step is exact up to the FP32 accumulation.
//
// Tile = 128 weight rows (the MMA M side, TMEM lanes) x up to kTileN segment
// rows of one expert (the MMA N side).  For gate/up the 128 weight rows are
// 64 gate rows and the 64 matching up rows, so SwiGLU finishes inside the
// tile.  Per 128-wide K group:
//   TMA W warp        packed INT4 box [128 rows x 64 B] (64-byte swizzle)
//                     into a kWStages ring;
//   TMA B warp        the activation codes [n rows x 128 B] (128-byte
//                     swizzle) into a kBStages ring; the codes are stored in
//                     expert-segment order, so a tile's rows are contiguous
//                     and come as 16-row boxes;
//   converter warps   each thread owns one weight row: 64 B of nibbles ->
//                     128 E4M3 bytes, stored straight into a TMEM A slot
//                     (tcgen05.st); kConvSets sets of 4 warps take turns;
//   MMA warps         4 x tcgen05.mma kind::f8f6f4 (K = 32 each), A from
//                     TMEM, B from shared memory, into one of kDBufs TMEM
//                     accumulators (FP32, fresh per group); kMmaWarps issuers
//                     take turns (one thread issues a tcgen05 op about every
//                     50-100 cycles, a group needs five);
//   epilogue warps    kEpiPerQuad warps per TMEM lane quadrant: tcgen05.ld the
//                     group's sums, acc += s_g * (512 * D_g - 8 * S_g) in FP32.
//                     The weight scales are stored group-major ([E, G, rows]),
//                     so one tile's scales are a [G x 128-row] box that the
//                     weight TMA warp loads once per tile into a
//                     double-buffered shared tile; S_g of the tile's columns
//                     is staged in shared memory once per tile as well.
// After the last group the epilogue applies the token (or row) scale and
// writes h (plus the SwiGLU and absmax) or Y.
//
// The -8 S_g term can also be left to the tensor core (the shape's OffsetMode):
// four more MMAs per group against a constant -2^-6 A operand, or once per
// tile as sum_g s_g S_g, a K = G bf16 product of the tile's scales (written to
// TMEM by the converter warps) with the rows' group sums (three bf16 parts
// each, written by the activation quantisers), accumulated like one more group.
//
// Two families of shapes of the same kernel: decode shapes (32-token tiles,
// 8 groups in flight, 12-16 weight stages) for batches with few tokens per
// expert, where pipeline depth hides the MMA and TMEM latencies, and prefill
// shapes (128-token tiles) where each converted weight tile feeds more tokens.
// The decode shapes pair the groups: one A slot, activation stage and
// accumulator hold two consecutive groups, so each barrier round trip and MMA
// commit serves two groups (the tensor-core issue rate sets the decode speed).
//
// Every wait is bounded (see ptx.cuh); a timed-out CTA drains its own
// in-flight copies and MMAs, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <type_traits>

#include "internal.h"
#define W4A8_OWNS_DEVICE_ERROR_LATCH 1
#include "ptx.cuh"

namespace w4a8 {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kBM = 128;
constexpr int kWStageBytes = kBM * kGroup / 2;      // 8 KB of packed INT4
constexpr uint32_t kTmemCols = 512;

template <int TileN, int WStages, int BStages, int ASlots, int DBufs, int ConvSets,
          int EpiPerQuad, int LdCols, int MmaWarps, int EpiSets, int OffsetMode, int Pair = 0,
          int Cta2 = 0>
struct Shape {
  static constexpr int kTileN = TileN;
  static constexpr int kWStages = WStages;
  static constexpr int kBStages = BStages;
  static constexpr int kASlots = ASlots;
  static constexpr int kDBufs = DBufs;
  static constexpr int kConvSets = ConvSets;
  static constexpr int kEpiPerQuad = EpiPerQuad;
  static constexpr int kLdCols = LdCols;                  // TMEM columns per tcgen05.ld
  static constexpr int kMmaWarps = MmaWarps;
  static constexpr int kConvWarps = 4 * ConvSets;
  static constexpr int kEpiSets = EpiSets;                // epilogue sets taking turns by tile
  // Where the +8 offset of the stored nibbles is removed (OffsetMode):
  //   0  the epilogue, per group: acc += s_g * (512 D_g - 8 S_g);
  //   1  the tensor core, per group: four more MMAs against a constant -2^-6
  //      A operand, so that D_g holds 2^-9 sum a q;
  //   2  the tensor core, once per tile: sum_g s_g S_g is a K = G product of the
  //      tile's weight scales with the rows' group sums, one bf16 MMA chain
  //      (the sums split in three bf16 parts) into one more accumulator.
  static constexpr bool kOffsetInMma = OffsetMode == 1;
  static constexpr bool kOffsetTile = OffsetMode == 2;
  static constexpr bool kEpiOffset = OffsetMode == 0;
  // Paired groups: each ring element (A slot, activation stage, accumulator)
  // holds two consecutive K groups, so every barrier wait, arrival and MMA
  // commit is shared by two groups.  K / 128 must be even.
  static constexpr bool kPair = Pair != 0;
  static constexpr int kGPU = kPair ? 2 : 1;              // groups per ring element
  // CTA pairs (cta_group::2): a cluster of two CTAs shares each tile, M = 256
  // weight rows, 128 in each CTA's TMEM; the tile's N token rows are split
  // between the two CTAs' activation stages; the first CTA issues the MMAs.
  static constexpr bool kCta2 = Cta2 != 0;
  static constexpr int kTileNLocal = kCta2 ? TileN / 2 : TileN;  // activation rows per CTA
  static constexpr int kEpiPerSet = 4 * EpiPerQuad;
  static constexpr int kEpiWarps = kEpiPerSet * EpiSets;
  static constexpr int kWarpW = kConvWarps + kEpiWarps;   // TMA: packed weights
  static constexpr int kWarpMma = kWarpW + 1;             // first MMA issuer
  static constexpr int kWarpB = kWarpMma + MmaWarps;      // TMA: activation rows
  // Equal A, B and D rings: one commit per group signals all three releases.
  static constexpr bool kUnified = ASlots == BStages && BStages == DBufs;
  static constexpr int kThreads = 32 * ((kWarpB + 1 + 3) / 4 * 4);
  static constexpr int kEpiN = TileN / EpiPerQuad;        // columns per epilogue warp
  static constexpr int kBStageBytes = kTileNLocal * kGroup * kGPU;
  static constexpr int kUpBytes = 64 * TileN * 4;         // up-projection exchange
  static constexpr int kSumLd = kEpiN + 4;                // padded: 4-way bank spread on stores
  static constexpr int kTileScBufs = 2;                   // tile weight-scale buffers
  // Decode shapes, down layer: the staged S_g are double-buffered and fetched
  // one tile ahead (the rows are contiguous segment rows there)
  static constexpr __host__ __device__ int sum_bufs(bool gate_up) {
    return kEpiOffset && TileN == kTileNDecode && !gate_up ? 2 : 1;
  }
  static constexpr uint32_t kACols = 32 * kGPU;           // TMEM columns per A slot
  static constexpr uint32_t kDCols = TileN * kGPU;        // TMEM columns per accumulator
  static constexpr uint32_t kTmemA = 0;                   // A slots
  static constexpr uint32_t kTmemConst = ASlots * kACols; // E4M3 -2^-6 in every byte (offset MMAs)
  static constexpr uint32_t kTmemD = kTmemConst + (kOffsetInMma ? 32 : 0);  // accumulators
  static constexpr int kNumBars = 2 * WStages + 2 * BStages + 2 * ASlots + 2 * DBufs + 3 +
                                  2 * EpiSets * (1 + EpiPerQuad) + 2 * kTileScBufs + 1;
  static_assert(kTmemD + DBufs * kDCols <= kTmemCols, "TMEM budget exceeded");
  static_assert(!kPair || (kEpiOffset && kUnified && ConvSets == 1),
                "paired groups: epilogue offset, unified rings, one converter set");
  static_assert(!kCta2 || (kPair && TileN == 32),
                "CTA pairs: the paired decode shapes (N = 32, 16 token rows per CTA)");
  static_assert(kEpiN % 32 == 0 && kEpiN % LdCols == 0 && (LdCols == 16 || LdCols == 32),
                "epilogue load width");
  static_assert(TileN % 16 == 0 && TileN <= 256, "MMA N");
  static_assert(MmaWarps == 1 || MmaWarps == 2, "MMA issuers");
  static_assert(EpiSets == 1 || EpiSets == kTileScBufs, "one tile-scale buffer per epilogue set");
  // the correction takes more A/B steps than accumulators per tile, and one
  // converter set walks the tile's groups and correction chunks in order
  static_assert(!kOffsetTile || (!kUnified && ConvSets == 1), "per-tile correction rings");
  // Runtime-sized regions (G = K / 128 groups): staged S_g, per set
  // [sum_bufs][kEpiPerQuad][G][kSumLd] floats, and the tile scales,
  // [kTileScBufs][G][128] bf16.
  static constexpr __host__ __device__ int sum_bytes(int G, bool gate_up) {
    return kEpiOffset ? (sum_bufs(gate_up) * EpiPerQuad * G * kSumLd * 4 + 127) & ~127 : 0;
  }
  static constexpr __host__ __device__ int tile_sc_bytes(int G) { return 256 * G; }
  // tile_prefix and expert_offsets, [E + 1] int32 each
  static constexpr __host__ __device__ int table_bytes(int E) { return (8 * (E + 1) + 15) & ~15; }
  // f8w: E4M3 weights (128 B per row and group, no tile-scale buffers)
  static constexpr int smem_bytes(bool gate_up, int G, int E, bool f8w = false) {
    return 1024 + WStages * (f8w ? 2 * kWStageBytes : kWStageBytes) + BStages * kBStageBytes +
           EpiSets * ((gate_up ? kUpBytes : 0) + sum_bytes(G, gate_up)) +
           (f8w ? 0 : kTileScBufs * tile_sc_bytes(G)) +
           table_bytes(E) + kNumBars * 8 + 16;
  }
};

// Shapes.  By default each projection takes the shape measured fastest for it;
// W4A8_GEMM_DECODE_SHAPE = 1..5 / W4A8_GEMM_PREFILL_SHAPE = 1..4 force one for both
// (decode 5: the paired shapes, gate/up and down).
//                            TileN        W   B  A  D cvt epi/q ld mma sets offset mode
using DecodeOneSet  = Shape<kTileNDecode, 16, 8, 8, 8, 1, 1, 32, 2, 1, 0>;
using DecodeTwoSets = Shape<kTileNDecode, 12, 8, 8, 8, 1, 1, 32, 2, 2, 0>;
using DecodeTwoCvt  = Shape<kTileNDecode, 12, 8, 8, 8, 2, 1, 32, 2, 2, 0>;
using DecodeTileCorr = Shape<kTileNDecode, 16, 8, 8, 7, 1, 1, 32, 2, 1, 2>;
using DecodePair = Shape<kTileNDecode, 16, 4, 4, 4, 1, 1, 32, 2, 1, 0, 1>;  // 2 groups per element
using DecodePairTwoSets = Shape<kTileNDecode, 12, 4, 4, 4, 1, 1, 32, 2, 2, 0, 1>;
// the paired shapes on CTA pairs (cta_group::2, M = 256)
using DecodePair2 = Shape<kTileNDecode, 16, 4, 4, 4, 1, 1, 32, 2, 1, 0, 1, 1>;
using DecodePairTwoSets2 = Shape<kTileNDecode, 12, 4, 4, 4, 1, 1, 32, 2, 2, 0, 1, 1>;
using Prefill16Epi  = Shape<kTileNPrefill, 4, 5, 3, 3, 1, 4, 16, 2, 1, 1>;
using Prefill8Epi   = Shape<kTileNPrefill, 4, 5, 3, 2, 1, 2, 16, 2, 1, 1>;
using Prefill16EpiEpilogueOffset = Shape<kTileNPrefill, 4, 5, 4, 3, 1, 4, 16, 2, 1, 0>;
using PrefillTileCorr = Shape<kTileNPrefill, 4, 5, 4, 3, 1, 4, 16, 2, 1, 2>;
// E4M3-weight (FP8 block) shape: A from shared memory, no converter warps
using F8Block = Shape<kTileNPrefill, 4, 4, 1, 3, 0, 4, 16, 2, 1, 0>;
// ... at decode, as the second phase of a routed launch: 64 token rows, eight
// epilogue warps of 32 columns (384 threads, as the routed decode shapes' 384
// or within their 512)
using F8Decode = Shape<kTileNShared, 6, 4, 1, 3, 0, 2, 32, 2, 1, 0>;
// INT8 per-channel shapes: one accumulator per tile, single MMA issuer
using I8Decode  = Shape<kTileNDecode, 16, 8, 8, 8, 1, 1, 32, 1, 1, 0>;
using I8Decode2 = Shape<kTileNDecode, 16, 8, 8, 8, 1, 1, 32, 2, 1, 0>;  // 4 tiles x 2 chains
using I8Prefill = Shape<kTileNPrefill, 4, 4, 4, 2, 1, 4, 16, 1, 1, 0>;

struct Tile {
  int e, mb, n_valid, n_mma;
  int64_t row0;
};

// Linear tile index -> (expert, weight-row block, segment rows).  An expert's
// tiles are consecutive.  Within an expert they run weight-row block major
// (nb_fastest = 0: the weight-row blocks that share one token block are
// neighbours) or token block fastest (nb_fastest = 1: the token blocks that
// share one weight-row block are neighbours), so that CTAs running at the
// same time share operands through L2.  Token block fastest re-reads all of
// an expert's activation rows once per weight-row block, which only L2 can
// absorb: an expert with more than nb_cap token blocks runs weight-row block
// major whatever nb_fastest says.  tile_prefix and expert_offsets are read from
// the CTA's shared copies (sTP, sEO): the binary search is a chain of dependent
// loads.
template <int TileN>
__device__ __forceinline__ Tile decode_tile(const int* sTP, const int* sEO, int E, int mb_count,
                                            int nb_fastest, int nb_cap, int idx) {
  const int nbg = idx / mb_count;  // global token block of the idx's expert range
  Tile t;
  int lo = 0, hi = E;  // tile_prefix[lo] <= nbg < tile_prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (sTP[mid] <= nbg) lo = mid;
    else hi = mid;
  }
  t.e = lo;
  const int local = idx - sTP[lo] * mb_count;
  int nb;
  const int ne = sTP[lo + 1] - sTP[lo];
  if (nb_fastest && ne <= nb_cap) {
    t.mb = local / ne;
    nb = local - t.mb * ne;
  } else {
    nb = local / mb_count;
    t.mb = local - nb * mb_count;
  }
  const int seg0 = sEO[lo];
  const int cnt = sEO[lo + 1] - seg0;
  t.row0 = static_cast<int64_t>(seg0) + static_cast<int64_t>(nb) * TileN;
  t.n_valid = min(TileN, cnt - nb * TileN);
  t.n_mma = (t.n_valid + 15) & ~15;
  return t;
}

// Max over the 32 lanes of each of v[off .. off + 31]; lane l returns the
// max of column off + l.  Five halving exchange steps (31 shuffles) instead
// of a separate 5-shuffle reduction per column.
template <int N>
__device__ __forceinline__ float column_max32(float (&v)[N], int off, int lane) {
  float w[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) w[j] = v[off + j];
#pragma unroll
  for (int h = 16; h >= 1; h >>= 1) {
    const bool upper = lane & h;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float send = upper ? w[j] : w[j + h];
      const float keep = upper ? w[j + h] : w[j];
      w[j] = fmaxf(keep, __shfl_xor_sync(kFull, send, h));
    }
  }
  return w[0];
}

// The token a gate/up segment row reads its scale and group sums from.  The
// debug build checks it against the token count (raising the latch's index
// bit and reading token 0 instead); the release build trusts the permutation.
__device__ __forceinline__ int checked_token(const GemmArgs& a, int t) {
#if W4A8_DEBUG_BOUNDS
  if (t < 0 || t >= a.n_tokens) {
    atomicOr(&g_device_error, kDeviceErrorIndex);
    return 0;
  }
#endif
  return t;
}

// Wait used only while draining: ignores the abort flag, still bounded.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity,
                                                uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) {
      atomicOr(&g_device_error, 1);
      return;
    }
  }
}

// One launch's work for one projection.  kPhase 0: the whole launch (TMEM
// allocated and freed here).  Two phases of one launch (the routed experts,
// then the shared expert): phase 1 allocates TMEM and returns it, and retires
// its barriers at the end, because phase 2 lays out shared memory anew;
// phase 2 takes the TMEM (phase_tmem) and frees it.  In a phase, the CTA's
// place in the tile schedule is (phase_cta_x, phase_n_cta).
template <class S, bool kGateUp, bool kI8, bool kF8W, int kPhase = 0>
__device__ __forceinline__ uint32_t gemm_body(const CUtensorMap& tmap_w,
                                              const CUtensorMap& tmap_act,
                                              const CUtensorMap& tmap_sc,
                                              const CUtensorMap& tmap_gs, const GemmArgs& a,
                                              int phase_cta_x, int phase_n_cta,
                                              uint32_t phase_tmem) {
  static_assert(kPhase == 0 || !S::kCta2, "CTA pairs run as a launch of their own");
  constexpr int kTileN = S::kTileN, kWStages = S::kWStages, kBStages = S::kBStages;
  constexpr int kASlots = S::kASlots, kDBufs = S::kDBufs, kEpiN = S::kEpiN;
  constexpr int kBStageBytes = S::kBStageBytes, kUpBytes = S::kUpBytes;
  constexpr int kLdCols = S::kLdCols, kSumLd = S::kSumLd;
  constexpr uint32_t kTmemA = S::kTmemA, kTmemD = S::kTmemD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sW = smem;
  // W stage: packed INT4 [128 rows x 64 B], or E4M3 weights [128 rows x 128 B]
  constexpr int kWBytes = kF8W ? 2 * kWStageBytes : kWStageBytes;
  constexpr int kTileScTotal = kF8W ? 0 : S::kTileScBufs;
  uint8_t* sB = sW + kWStages * kWBytes;
  const int G = a.K / kGroup;
  // per epilogue set: [sU (gate/up only)][sS]
  constexpr int kUpPerSet = kGateUp ? kUpBytes : 0;
  const int set_bytes = kUpPerSet + S::sum_bytes(G, kGateUp);
  uint8_t* sSet = sB + kBStages * kBStageBytes;
  uint8_t* sT = sSet + S::kEpiSets * set_bytes;
  int* sTP = reinterpret_cast<int*>(sT + kTileScTotal * S::tile_sc_bytes(G));
  int* sEO = sTP + (a.E + 1);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sTP) + S::table_bytes(a.E));
  uint64_t* wfull = bars;                 // [kWStages] packed weights landed
  uint64_t* wempty = wfull + kWStages;    // [kWStages] 4 converter warps read them
  uint64_t* bfull = wempty + kWStages;    // [kBStages] activation rows landed
  uint64_t* bempty = bfull + kBStages;    // [kBStages] MMAs reading them done
  uint64_t* afull = bempty + kBStages;    // [kASlots]  converted A in TMEM
  uint64_t* aempty = afull + kASlots;     // [kASlots]  MMAs reading the slot done
  uint64_t* dfull = aempty + kASlots;     // [kDBufs]   group partial sums ready
  uint64_t* dempty = dfull + kDBufs;      // [kDBufs]   epilogue warps read them
  uint64_t* upfull = dempty + kDBufs;     // [kEpiSets] up rows staged in the set's sU
  uint64_t* upempty = upfull + S::kEpiSets;  // [kEpiSets] sU consumed
  uint64_t* drain = upempty + S::kEpiSets;   // all MMAs of this CTA complete
  uint64_t* sfull = drain + 1;            // [kEpiSets][kEpiPerQuad] a slice's S_g staged
  uint64_t* sempty = sfull + S::kEpiSets * S::kEpiPerQuad;  // [..] the slice's warps are done
  // FP8: one commit per group releases the A slot, B stage and accumulator when
  // the three rings have one size.  INT8: one accumulator per tile, so only
  // the A and B rings can share a barrier.
  constexpr bool kUniAll = S::kUnified && !kI8 && !kF8W;
  constexpr bool kUniAB = kI8 ? (kASlots == kBStages) : kUniAll;
  if constexpr (kUniAB) bempty = aempty;
  if constexpr (kUniAll) dfull = aempty;
  uint64_t* tfull = sempty + S::kEpiSets * S::kEpiPerQuad;  // [kTileScBufs] tile scales landed
  uint64_t* tempty = tfull + S::kTileScBufs;    // [kTileScBufs] epilogue warps are done
  // Group loops run in tile order, one set at a time (completion n = tile n's loop
  // done), so every wait on the shared accumulator ring stays within one phase.
  uint64_t* loopdone = tempty + S::kTileScBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(loopdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool kCta2 = S::kCta2;
  // CTA pairs: both CTAs of a cluster walk the same tiles (cta_x of n_cta);
  // this CTA takes weight-row block 2 mb + crank of the pair's block mb
  const uint32_t crank = kCta2 ? cluster_ctarank() : 0u;
  const int cta_x = kPhase ? phase_cta_x
                           : kCta2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int n_cta = kPhase ? phase_n_cta
                           : kCta2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int mb_count = (kGateUp ? a.half_rows / 64 : a.n_rows / kBM) / (kCta2 ? 2 : 1);
  const uint64_t tmo = a.timeout_ns;
  // token blocks of one expert whose activation rows (K bytes each) stay well
  // inside L2 (32 MB of its 126 MB) while every weight-row block passes by
  const int nb_cap = static_cast<int>((32ll << 20) / (static_cast<int64_t>(kTileN) * a.K));
  auto tile_at = [&](int idx) -> Tile {
    Tile t = decode_tile<kTileN>(sTP, sEO, a.E, mb_count, a.nb_fastest, nb_cap, idx);
    if (kCta2) t.mb = 2 * t.mb + static_cast<int>(crank);
    return t;
  };

  // every barrier of this launch (or phase), with its arrival count
  auto each_barrier = [&](auto&& f) {
    for (int s = 0; s < kWStages; ++s) {
      f(&wfull[s], 1);
      f(&wempty[s], kF8W ? 1 : 4);  // E4M3 weights: released by the MMA commit
    }
    for (int s = 0; s < kBStages; ++s) {
      f(&bfull[s], 1);
      if (!kUniAB) f(&bempty[s], 1);
    }
    for (int s = 0; s < kASlots; ++s) {
      f(&afull[s], kCta2 ? 8 : 4);  // pairs: both CTAs' converter warps (first CTA's)
      f(&aempty[s], 1);
    }
    for (int d = 0; d < kDBufs; ++d) {
      if (!kUniAll) f(&dfull[d], kI8 ? S::kMmaWarps : 1);
      // each group is read by one set (of both CTAs of a pair, on the first CTA's barrier)
      f(&dempty[d], S::kEpiPerSet * (kCta2 ? 2 : 1));
    }
    for (int i = 0; i < S::kEpiSets; ++i) {
      f(&upfull[i], S::kEpiPerSet / 2);
      f(&upempty[i], S::kEpiPerSet / 2);
    }
    f(drain, S::kMmaWarps);
    for (int i = 0; i < S::kEpiSets * S::kEpiPerQuad; ++i) {
      f(&sfull[i], 4);
      f(&sempty[i], 4);
    }
    for (int i = 0; i < S::kTileScBufs; ++i) {
      f(&tfull[i], 1);
      // a tile's scales are read by one epilogue set (and, for the per-tile
      // correction, by the 4 converter warps)
      f(&tempty[i], S::kEpiPerSet + (S::kOffsetTile ? 4 : 0));
    }
    f(loopdone, S::kEpiPerSet);
  };
  if (threadIdx.x == 0) {
    each_barrier([](uint64_t* b, int count) { mbar_init(b, count); });
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == S::kWarpW && lane == 0) {
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_sc);
  }
  if (warp == S::kWarpB && lane == 0) {
    prefetch_tmap(&tmap_act);
    if (S::kOffsetTile) prefetch_tmap(&tmap_gs);
  }
  if (kPhase != 2 && warp == 0) {
    if constexpr (kCta2) {
      tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), kTmemCols);
      tmem_relinquish();
    }
  }
  for (int i = threadIdx.x; i <= a.E; i += blockDim.x) {
    sTP[i] = __ldg(a.tile_prefix + i);
    sEO[i] = __ldg(a.expert_offsets + i);
  }
#if W4A8_DEBUG_BOUNDS
  // debug build: the expert tables decide every row this CTA touches; if they
  // are not a valid segment table of the shape's tiles within the buffers,
  // raise the latch's index bit and run no tile
  __syncthreads();
  if (threadIdx.x == 0) {
    bool good = sEO[0] == 0 && sTP[0] == 0 && sEO[a.E] <= a.n_seg_rows;
    for (int e = 0; good && e < a.E; ++e) {
      const int cnt = sEO[e + 1] - sEO[e];
      const int tiles = sTP[e + 1] - sTP[e];   // 0 when another launch takes the expert
      good = cnt >= 0 && tiles >= 0 && tiles <= (cnt + kTileN - 1) / kTileN;
    }
    if (!good) {
      atomicOr(&g_device_error, kDeviceErrorIndex);
      for (int e = 0; e <= a.E; ++e) sTP[e] = 0;
    }
  }
#endif
  tc_fence_before();
  __syncthreads();
  // pairs: the other CTA's barriers are initialised before anything arrives on them
  if constexpr (kCta2) cluster_sync();
  tc_fence_after();
  const uint32_t tmem = kPhase == 2 ? phase_tmem : *tmem_slot;
  const int total = sTP[a.E] * mb_count;
  const int my_tiles = cta_x < total ? (total - cta_x + n_cta - 1) / n_cta : 0;
  const int n_groups = my_tiles * G;  // every tile has G groups
  // Per-tile correction (offset mode 2): the rows' group sums S_g come as three
  // bf16 parts, [rows][3 * Gp] with Gp = G rounded up to 16 (padding zero);
  // the product with the tile's scales takes kNC more A/B ring steps of K = 64
  // and one more accumulator per tile.
  const int Gp = (G + 15) & ~15;
  const int KC = 3 * Gp;
  const int kNC = S::kOffsetTile ? (KC + 63) / 64 : 0;
  constexpr int kGPU = S::kGPU;                          // groups per ring element
  const int ab_per_tile = G / kGPU + kNC;                // A slot / B stage steps
  const int units_per_tile = G / kGPU + (S::kOffsetTile ? 1 : 0);  // accumulators
  const int n_units = my_tiles * units_per_tile;

  if (warp == S::kWarpW) {
    // ------------------------------------------------------------ TMA: packed weights
    if (lane == 0) {
      int it = 0, nt = 0;
      bool ok = true;
      for (int tile = cta_x; ok && tile < total; tile += n_cta, ++nt) {
        const Tile t = tile_at(tile);
        const int32_t wy0 = t.e * a.n_rows + (kGateUp ? t.mb * 64 : t.mb * kBM);
        const int32_t wy1 = t.e * a.n_rows + a.half_rows + t.mb * 64;
        if constexpr (!kI8 && !kF8W) {  // the tile's weight scales: box [G groups x 128 (or 2 x 64) rows] of bf16
          const int tb = nt % S::kTileScBufs;
          const uint32_t tph = (nt / S::kTileScBufs) & 1;
          if (!mbar_wait(&tempty[tb], tph ^ 1, abort_flag, tmo)) break;
          const uint32_t dT = smem_u32(sT + tb * S::tile_sc_bytes(G));
          mbar_arrive_expect_tx(&tfull[tb], S::tile_sc_bytes(G));
          const int32_t ty = t.e * G;  // x is in bytes: 2 per row
          if (kGateUp) {
            tma_load_2d(dT, &tmap_sc, &tfull[tb], t.mb * 64 * 2, ty);
            tma_load_2d(dT + 128 * G, &tmap_sc, &tfull[tb], (a.half_rows + t.mb * 64) * 2, ty);
          } else {
            tma_load_2d(dT, &tmap_sc, &tfull[tb], t.mb * kBM * 2, ty);
          }
        }
        for (int g = 0; g < G; ++g) {
          const int s = it % kWStages;
          const uint32_t ph = (it / kWStages) & 1;
          if (!mbar_wait(&wempty[s], ph ^ 1, abort_flag, tmo)) { ok = false; break; }
          const uint32_t dW = smem_u32(sW + s * kWBytes);
          mbar_arrive_expect_tx(&wfull[s], kWBytes);
          if constexpr (kF8W) {  // E4M3 rows: 128 B per group, boxes of 64 (gate/up) or 128 rows
            tma_load_2d(dW, &tmap_w, &wfull[s], g * kGroup, wy0);
            if (kGateUp) tma_load_2d(dW + kWBytes / 2, &tmap_w, &wfull[s], g * kGroup, wy1);
          } else if (kGateUp) {
            tma_load_2d(dW, &tmap_w, &wfull[s], g * 64, wy0);
            tma_load_2d(dW + kWStageBytes / 2, &tmap_w, &wfull[s], g * 64, wy1);
          } else {
            tma_load_2d(dW, &tmap_w, &wfull[s], g * 64, wy0);
          }
          ++it;
        }
      }
      // The latest fill of every stage must have landed before the CTA exits.
      for (int i = (it > kWStages ? it - kWStages : 0); i < it; ++i)
        mbar_wait_drain(&wfull[i % kWStages], (i / kWStages) & 1, tmo);
      if (!kI8 && !kF8W)
        for (int i = (nt > S::kTileScBufs ? nt - S::kTileScBufs : 0); i < nt; ++i)
          mbar_wait_drain(&tfull[i % S::kTileScBufs], (i / S::kTileScBufs) & 1, tmo);
    }
    __syncwarp();
  } else if (warp == S::kWarpB) {
    // ------------------------------------------------------------ TMA: activation rows
    int it = 0;
    bool ok = true;
    for (int tile = cta_x; ok && tile < total; tile += n_cta) {
      const Tile t = tile_at(tile);
      // the activations are in segment order: the tile's rows are contiguous,
      // loaded as 16-row boxes (rows past the tensor's end read as zero)
      const int n_ops = t.n_mma >> 4;
      const uint32_t tx = t.n_mma * kGroup;
      const int32_t y0 = static_cast<int32_t>(t.row0) + 16 * lane;
      if constexpr (kCta2) {
        // pairs: this CTA's 16 of the tile's 32 rows, for each group of the
        // element; the copies of both CTAs complete on the first CTA's barrier,
        // which the first CTA expects for both
        const int32_t yp = static_cast<int32_t>(t.row0) + 16 * static_cast<int32_t>(crank);
        for (int g = 0; g < ab_per_tile; ++g) {
          const int s = it % kBStages;
          const uint32_t ph = (it / kBStages) & 1;
          if (!mbar_wait(&bempty[s], ph ^ 1, abort_flag, tmo)) { ok = false; break; }
          if (lane == 0) {
            const uint32_t dB = smem_u32(sB + s * kBStageBytes);
            const uint32_t bar0 = mapa_shared(smem_u32(&bfull[s]), 0);
            if (crank == 0) mbar_arrive_expect_tx(&bfull[s], 2 * kBStageBytes);
#pragma unroll
            for (int h = 0; h < kGPU; ++h)
              tma_load_2d_pair(dB + h * (16 * kGroup), &tmap_act, bar0, (g * kGPU + h) * kGroup, yp);
          }
          __syncwarp();
          ++it;
        }
        continue;
      }
      // G stages of codes (kGPU groups per stage, each in its own kTileN-row
      // half), then (per-tile correction) kNC stages of the bf16 group-sum
      // parts, 128 bytes of each row per stage
      for (int g = 0; g < ab_per_tile; ++g) {
        const int s = it % kBStages;
        const uint32_t ph = (it / kBStages) & 1;
        if (!mbar_wait(&bempty[s], ph ^ 1, abort_flag, tmo)) { ok = false; break; }
        const uint32_t dB = smem_u32(sB + s * kBStageBytes);
        const bool codes = g * kGPU < G;
        if (lane == 0) mbar_arrive_expect_tx(&bfull[s], codes ? kGPU * tx : tx);
        __syncwarp();
        if (lane < n_ops) {
          if (codes) {
#pragma unroll
            for (int h = 0; h < kGPU; ++h)
              tma_load_2d(dB + h * (kTileN * kGroup) + lane * 16 * kGroup, &tmap_act, &bfull[s],
                          (g * kGPU + h) * kGroup, y0);
          } else {
            tma_load_2d(dB + lane * 16 * kGroup, &tmap_gs, &bfull[s], (g - G) * 128, y0);
          }
        }
        ++it;
      }
    }
    // (pairs: the first CTA's barriers count both CTAs' copies)
    if (lane == 0 && crank == 0)
      for (int i = (it > kBStages ? it - kBStages : 0); i < it; ++i)
        mbar_wait_drain(&bfull[i % kBStages], (i / kBStages) & 1, tmo);
    __syncwarp();
  } else if (warp >= S::kWarpMma && warp < S::kWarpB) {
    // ------------------------------------------------------------ MMA issuers
    const int mw = warp - S::kWarpMma;              // takes groups it % kMmaWarps == mw
    if constexpr (kI8) {
      // INT8, per-channel scales: a tile's groups accumulate into kMmaWarps
      // int32 accumulators ("chains"); issuer mw takes the groups with global
      // index it = mw (mod kMmaWarps), so each chain's first, non-accumulating
      // MMA is issued ahead of the rest by the same thread, and every A slot /
      // B stage keeps a single issuer.  A tile's accumulators are released once
      // per tile (dfull counts one commit per chain).  Chains need G >= kMmaWarps.
      constexpr int kChains = S::kMmaWarps;
      constexpr int kTileSlots = kDBufs / kChains;
      if (lane == 0) {
        uint32_t idesc = 0, dt = 0;
        int dcur = 0, cur_tile = -1;
        bool first = true, ok = true;
        for (int it = mw; ok && it < n_groups; it += kChains) {
          const int tl = it / G, g = it - tl * G;
          if (tl != cur_tile) {  // this chain's first group of the tile
            cur_tile = tl;
            first = true;
            const Tile t = tile_at(cta_x + tl * n_cta);
            idesc = idesc_u8_s32_m128(static_cast<uint32_t>(t.n_mma));
            dcur = tl % kTileSlots;
            if (!mbar_wait(&dempty[dcur], ((tl / kTileSlots) & 1) ^ 1, abort_flag, tmo)) break;
            dt = tmem + kTmemD + (dcur * kChains + mw) * kTileN;
          }
          const int sb = it % kBStages;
          const uint32_t phb = (it / kBStages) & 1;
          const int as = it % kASlots;
          const uint32_t pha = (it / kASlots) & 1;
          const bool rb = mbar_test_wait(&bfull[sb], phb);
          const bool ra = mbar_test_wait(&afull[as], pha);
          if (!(rb && ra) && (!mbar_wait(&bfull[sb], phb, abort_flag, tmo) ||
                              !mbar_wait(&afull[as], pha, abort_flag, tmo)))
            break;
          tc_fence_after();
          const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + sb * kBStageBytes));
          const uint32_t at = tmem + kTmemA + as * 32;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // K = 32 bytes per MMA
            mma_i8_ts(dt, at + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                      (!first || kk > 0) ? 1u : 0u);
          first = false;
          tc_commit(&aempty[as]);
          if constexpr (!kUniAB) tc_commit(&bempty[sb]);
          if (g + kChains >= G) tc_commit(&dfull[dcur]);  // this chain's last group of the tile
        }
        tc_commit(drain);
        mbar_wait_drain(drain, 0, tmo);
      }
    } else if constexpr (kF8W) {
      // E4M3 weights: A straight from the W stage in shared memory (K-major,
      // 128-byte swizzle, the layout of the activation stages); the commit
      // releases the W stage, the activation stage and the accumulator
      if (lane == 0) {
        int cur = -1;
        uint32_t idesc = 0;
        for (int it = mw; it < n_groups; it += S::kMmaWarps) {
          const int tl = it / G;
          if (tl != cur) {
            cur = tl;
            const Tile t = tile_at(cta_x + tl * n_cta);
            idesc = idesc_e4m3_f32_m128(static_cast<uint32_t>(t.n_mma));
          }
          const int ws = it % kWStages;
          const uint32_t phw = (it / kWStages) & 1;
          const int sb = it % kBStages;
          const uint32_t phb = (it / kBStages) & 1;
          const int d = it % kDBufs;
          const uint32_t phd = (it / kDBufs) & 1;
          if (!mbar_wait(&dempty[d], phd ^ 1, abort_flag, tmo) ||
              !mbar_wait(&bfull[sb], phb, abort_flag, tmo) ||
              !mbar_wait(&wfull[ws], phw, abort_flag, tmo))
            break;
          tc_fence_after();
          const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sW + ws * kWBytes));
          const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + sb * kBStageBytes));
          const uint32_t dt = tmem + kTmemD + d * kTileN;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // K = 32 E4M3 = 32 B of each operand row
            mma_f8_ss(dt, adesc + static_cast<uint64_t>(kk * 2),
                      bdesc + static_cast<uint64_t>(kk * 2), idesc, kk > 0 ? 1u : 0u);
          tc_commit(&dfull[d]);
          tc_commit(&wempty[ws]);
          tc_commit(&bempty[sb]);
        }
        tc_commit(drain);
        mbar_wait_drain(drain, 0, tmo);
      }
    } else if (kCta2 && lane == 0) {
      // CTA pairs: the first CTA issues every MMA of the pair (M = 256, N = 32),
      // after both CTAs' converted weights, both halves of the activation rows
      // and both CTAs' epilogues are ready (cluster-scope waits on its own
      // barriers); one commit signals the A slot / stage / accumulator barrier
      // of both CTAs.  The second CTA's issuers have nothing to do.
      if (crank == 0) {
        const uint32_t idesc = idesc_e4m3_f32_m256(static_cast<uint32_t>(kTileN));
        for (int it = mw; it < n_units; it += S::kMmaWarps) {
          const int d = it % kDBufs;
          const uint32_t phd = (it / kDBufs) & 1;
          const int as = it % kASlots;               // unified: A slot = B stage = accumulator
          const uint32_t pha = (it / kASlots) & 1;
          const bool rd = mbar_test_wait_cluster(&dempty[d], phd ^ 1);
          const bool rb = mbar_test_wait_cluster(&bfull[as], pha);
          const bool ra = mbar_test_wait_cluster(&afull[as], pha);
          if (!(rd && rb && ra) &&
              (!mbar_wait_cluster(&dempty[d], phd ^ 1, abort_flag, tmo) ||
               !mbar_wait_cluster(&bfull[as], pha, abort_flag, tmo) ||
               !mbar_wait_cluster(&afull[as], pha, abort_flag, tmo)))
            break;
          tc_fence_after();
          const uint64_t bdesc0 = sdesc_kmajor_sw128(smem_u32(sB + as * kBStageBytes));
          const uint32_t dt0 = tmem + kTmemD + d * S::kDCols;
          const uint32_t at0 = tmem + kTmemA + as * S::kACols;
#pragma unroll
          for (int h = 0; h < kGPU; ++h) {
            const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(h * (16 * kGroup / 16));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ts_pair(dt0 + h * kTileN, at0 + h * 32 + kk * 8,
                             bdesc + static_cast<uint64_t>(kk * 2), idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit_pair_multicast(&aempty[as], static_cast<uint16_t>(0x3));
        }
        tc_commit_pair(drain);
        mbar_wait_drain(drain, 0, tmo);
      }
    } else if (lane == 0) {
      int cur = -1;
      uint32_t idesc = 0, idesc_c = 0;
      // unit = one accumulator: the tile's G groups, then (offset mode 2) the
      // correction, whose kNC chunks one issuer runs back to back
      for (int it = mw; it < n_units; it += S::kMmaWarps) {
        const int tl = it / units_per_tile;
        const int u = it - tl * units_per_tile;
        if (tl != cur) {
          cur = tl;
          const Tile t = tile_at(cta_x + tl * n_cta);
          idesc = idesc_e4m3_f32_m128(static_cast<uint32_t>(t.n_mma));
          idesc_c = idesc_bf16_f32_m128(static_cast<uint32_t>(t.n_mma));
        }
        const int d = it % kDBufs;
        const uint32_t phd = (it / kDBufs) & 1;
        if (S::kOffsetTile && u == G) {
          if (!mbar_wait(&dempty[d], phd ^ 1, abort_flag, tmo)) break;
          const uint32_t dt = tmem + kTmemD + d * kTileN;
          bool okc = true;
          for (int c = 0; c < kNC; ++c) {
            const int ab = tl * ab_per_tile + G + c;
            const int sb = ab % kBStages;
            const uint32_t phb = (ab / kBStages) & 1;
            const int as = ab % kASlots;
            const uint32_t pha = (ab / kASlots) & 1;
            if (!mbar_wait(&bfull[sb], phb, abort_flag, tmo) ||
                !mbar_wait(&afull[as], pha, abort_flag, tmo)) {
              okc = false;
              break;
            }
            tc_fence_after();
            const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + sb * kBStageBytes));
            const uint32_t at = tmem + kTmemA + as * 32;
            const int nk = min(4, (KC - 64 * c) >> 4);   // K = 16 bf16 per MMA
            for (int kk = 0; kk < nk; ++kk)
              mma_bf16_ts(dt, at + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc_c,
                          (c > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&aempty[as]);
            tc_commit(&bempty[sb]);
          }
          if (!okc) break;
          tc_commit(&dfull[d]);
          continue;
        }
        const int ab = S::kOffsetTile ? tl * ab_per_tile + u : it;
        const int sb = ab % kBStages;
        const uint32_t phb = (ab / kBStages) & 1;
        const int as = ab % kASlots;
        const uint32_t pha = (ab / kASlots) & 1;
        // poll all three at once (each poll is a ~100-cycle round trip)
        const bool rd = mbar_test_wait(&dempty[d], phd ^ 1);
        const bool rb = mbar_test_wait(&bfull[sb], phb);
        const bool ra = mbar_test_wait(&afull[as], pha);
        if (!(rd && rb && ra) &&
            (!mbar_wait(&dempty[d], phd ^ 1, abort_flag, tmo) ||
             !mbar_wait(&bfull[sb], phb, abort_flag, tmo) ||
             !mbar_wait(&afull[as], pha, abort_flag, tmo)))
          break;
        tc_fence_after();
        const uint64_t bdesc0 = sdesc_kmajor_sw128(smem_u32(sB + sb * kBStageBytes));
        const uint32_t dt0 = tmem + kTmemD + d * S::kDCols;
        const uint32_t at0 = tmem + kTmemA + as * S::kACols;
#pragma unroll
        for (int h = 0; h < kGPU; ++h) {  // the element's groups: own A columns, B half, accumulator
          const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(h * (kTileN * kGroup / 16));
          const uint32_t dt = dt0 + h * kTileN;
          const uint32_t at = at0 + h * 32;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // K = 32 E4M3 per MMA: 8 TMEM columns, 32 B of smem
            mma_f8_ts(dt, at + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                      kk > 0 ? 1u : 0u);
            if constexpr (S::kOffsetInMma) {
              // D += sum_k a_k * (-2^-6) over the same 32 k (A = the constant TMEM
              // columns): after each pair D holds 2^-9 * sum a * q of the slices so
              // far, so the offset cancels at the magnitude of a 32-element partial
              // sum, not of the whole group
              mma_f8_ts(dt, tmem + S::kTmemConst, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                        1u);
            }
          }
        }
        if constexpr (kUniAll) {
          tc_commit(&aempty[as]);               // A slot, B stage and accumulator at once
        } else {
          tc_commit(&dfull[d]);
          tc_commit(&aempty[as]);
          tc_commit(&bempty[sb]);
        }
      }
      tc_commit(drain);
      mbar_wait_drain(drain, 0, tmo);
    }
    __syncwarp();
  } else if (warp < S::kConvWarps) {
    // ------------------------------------------------------------ INT4 -> E4M3 converters
    // (E4M3 weights need none: these warps have no role then)
    if constexpr (!kF8W) {
    const int quad = warp & 3;
    const int set = warp >> 2;                      // converts groups it % kConvSets == set
    const int m = quad * 32 + lane;                 // weight row of the tile = TMEM lane
    const uint32_t swz = (m >> 1) & 3;              // 64-byte swizzle of the TMA box
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    if (S::kOffsetInMma && set == 0) {
      // the constant A operand of the offset MMAs; the MMA warps first read it
      // after this set's first afull arrival, which follows these stores
      uint32_t c[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) c[i] = 0x88888888u;  // E4M3 0x88 = -2^-6
      tmem_st_32x32b_x32(tmem + lane_base + S::kTmemConst, c);
      tmem_wait_st();
      tc_fence_before();
    }
    // one weight group: W stage wit -> group h of A slot ait (the slot is
    // claimed with its first group and published after its last)
    auto convert = [&](int wit, int ait, int h) -> bool {
      const bool first = h == 0, last = h == kGPU - 1;
      const int s = wit % kWStages;
      const uint32_t ph = (wit / kWStages) & 1;
      const int as = ait % kASlots;
      const uint32_t pha = (ait / kASlots) & 1;
      const bool rw = mbar_test_wait(&wfull[s], ph);   // both polls in flight at once
      const bool ra = !first || mbar_test_wait(&aempty[as], pha ^ 1);
      if (!(rw && ra) && (!mbar_wait(&wfull[s], ph, abort_flag, tmo) ||
                          (first && !mbar_wait(&aempty[as], pha ^ 1, abort_flag, tmo))))
        return false;
      tc_fence_after();
      const uint32_t row = smem_u32(sW + s * kWStageBytes) + m * 64;
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 v = ld_shared_v4(row + ((c ^ swz) << 4));
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          r[8 * c + 2 * i] = w4[i] & 0x0F0F0F0Fu;              // elements 0..3 of the word
          r[8 * c + 2 * i + 1] = (w4[i] >> 4) & 0x0F0F0F0Fu;   // elements 4..7
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&wempty[s]);       // the stage's bytes are in registers
      tmem_st_32x32b_x32(tmem + lane_base + kTmemA + as * S::kACols + h * 32, r);
      tmem_wait_st();
      if (last) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (kCta2)  // the first CTA of the pair issues the MMAs
            mbar_arrive_cluster(mapa_shared(smem_u32(&afull[as]), 0));
          else
            mbar_arrive(&afull[as]);
        }
      }
      return true;
    };
    if constexpr (S::kOffsetTile) {
      // per tile: the G weight groups, then the correction's A operand, kNC
      // slots of bf16 pairs: column k of the correction is the row's scale of
      // group k mod Gp (zero past G), repeated for the three parts of S_g
      const int sc_off = kGateUp ? (m < 64 ? m : 64 * G + (m - 64)) : m;
      constexpr int kScStride = kGateUp ? 64 : 128;
      int ait = 0;
      bool ok = true;
      for (int nt = 0; ok && nt < my_tiles; ++nt) {
        for (int g = 0; g < G; ++g)
          if (!convert(nt * G + g, ait++, 0)) { ok = false; break; }
        if (!ok) break;
        const int tb = nt % S::kTileScBufs;
        if (!mbar_wait(&tfull[tb], (nt / S::kTileScBufs) & 1, abort_flag, tmo)) break;
        const uint16_t* sTs = reinterpret_cast<const uint16_t*>(sT + tb * S::tile_sc_bytes(G)) + sc_off;
        for (int c = 0; c < kNC; ++c, ++ait) {
          const int as = ait % kASlots;
          if (!mbar_wait(&aempty[as], ((ait / kASlots) & 1) ^ 1, abort_flag, tmo)) { ok = false; break; }
          tc_fence_after();
          uint32_t r[32];
#pragma unroll
          for (int j = 0; j < 4; ++j) {   // 16 columns of K (8 TMEM columns) per part run
            const int kb = 64 * c + 16 * j;
            const int part = kb < KC ? kb / Gp : 3;
            const int gb = kb - part * Gp;
#pragma unroll
            for (int t2 = 0; t2 < 8; ++t2) {
              const int g0 = gb + 2 * t2;
              const uint32_t lo = part < 3 && g0 < G ? sTs[g0 * kScStride] : 0u;
              const uint32_t hi = part < 3 && g0 + 1 < G ? sTs[(g0 + 1) * kScStride] : 0u;
              r[8 * j + t2] = lo | (hi << 16);
            }
          }
          tmem_st_32x32b_x32(tmem + lane_base + kTmemA + as * 32, r);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[as]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[tb]);
      }
    } else {
      // ring element ue holds groups kGPU * ue .. kGPU * ue + kGPU - 1
      bool ok = true;
      for (int ue = set; ok && ue < n_units; ue += S::kConvSets)
        for (int h = 0; h < kGPU; ++h)
          if (!convert(ue * kGPU + h, ue, h)) { ok = false; break; }
    }
    }  // !kF8W
  } else if (warp < S::kWarpW) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - S::kConvWarps;
    const int set = e / S::kEpiPerSet;              // takes this CTA's tiles set, set + sets, ...
    const int q = warp & 3;                         // TMEM lane quadrant
    const int slice = (e % S::kEpiPerSet) >> 2;     // column slice of the tile
    const int m = q * 32 + lane;                    // weight row of the tile
    const int j0 = slice * kEpiN;                   // first column (segment row) of this warp
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    float* sU = reinterpret_cast<float*>(sSet + set * set_bytes);
    float* const sSl0 = reinterpret_cast<float*>(sSet + set * set_bytes + kUpPerSet) +
                        slice * G * kSumLd;         // [g][jj] activation group sums of the slice
    // S_g fetched one tile ahead (down layer, decode shapes): lane g copies
    // group g (and g + 32) of this warp's quarter of the columns of tile tt
    // into buffer b; the copies land while the set's current tile runs
    constexpr bool kSumsAhead = S::sum_bufs(kGateUp) == 2;
    constexpr int kTok = kEpiN / 4;
    auto fetch_sums = [&](const Tile& tt, int b) {
      float* buf = sSl0 + b * S::kEpiPerQuad * G * kSumLd;
#pragma unroll
      for (int i = 0; i < kTok; ++i) {
        const int jj = q * kTok + i;
        const bool v = j0 + jj < tt.n_valid;
        const float* src = a.act_gsum + (v ? (tt.row0 + j0 + jj) * G : 0);
        const uint32_t nb = v ? 4u : 0u;
        if (lane < G) cp_async_4(smem_u32(buf + lane * kSumLd + jj), src + lane, nb);
        if (lane + 32 < G) cp_async_4(smem_u32(buf + (lane + 32) * kSumLd + jj), src + lane + 32, nb);
      }
    };
    if (kSumsAhead && cta_x + set * n_cta < total) fetch_sums(tile_at(cta_x + set * n_cta), 0);
    uint64_t* my_sfull = &sfull[set * S::kEpiPerQuad + slice];
    uint64_t* my_sempty = &sempty[set * S::kEpiPerQuad + slice];
    uint64_t* my_upfull = &upfull[set];
    uint64_t* my_upempty = &upempty[set];
    // this row's scale of group g in a tile-scale buffer: [G][64] gate rows
    // then [G][64] up rows (gate/up), or [G][128] rows (down)
    const int sc_off = kGateUp ? (m < 64 ? m : 64 * G + (m - 64)) : m;
    constexpr int kScStride = kGateUp ? 64 : 128;
    bool ok = true;
    for (int tile = cta_x + set * n_cta, ntile = set; ok && tile < total;
         tile += S::kEpiSets * n_cta, ntile += S::kEpiSets) {
      const Tile t = tile_at(tile);
      int it = ntile * units_per_tile;              // CTA-wide index of the tile's first unit
      const uint32_t lt = ntile / S::kEpiSets;      // this set's tile count: barrier phases
      // token (gate/up) or row (down) scales of this warp's columns, lane-strided;
      // loaded now so their latency hides behind the group loop
      float ts[kEpiN / 32];
#pragma unroll
      for (int i = 0; i < kEpiN / 32; ++i) {
        const int j = j0 + lane + 32 * i;
        float v = 0.0f;
        if (j < t.n_valid) {
          const int64_t r = t.row0 + j;
          if constexpr (kF8W) v = 1.0f;  // scales are per group, applied in the promotion
          else v = kGateUp ? __ldg(a.act_scale + checked_token(a, __ldg(a.row_tokens + r)))
                           : __ldg(a.act_scale + r);
        }
        ts[i] = v;
      }
      float acc[kEpiN];  // this warp's rows x columns of the tile, before the token scale
      if constexpr (kI8) {
        // per-channel INT8: D = sum_k u * a' with u = q + 8 and a' = code + 128
        // (both stored unsigned); sum_k q * code = D - 128 U_m - 8 A'_t + 1024 K
        // with U_m = sum_k u of weight row m and A'_t = sum_k a' of token t
        const int wrow = kGateUp ? (m < 64 ? t.mb * 64 + m : a.half_rows + t.mb * 64 + (m - 64))
                                 : t.mb * kBM + m;
        const int64_t widx = static_cast<int64_t>(t.e) * a.n_rows + wrow;
        const float wsm = __bfloat162float(static_cast<const __nv_bfloat16*>(a.wscale)[widx]);
        const int base = 1024 * a.K - 128 * __ldg(a.wsum + widx);
        int asum[kEpiN / 32];
#pragma unroll
        for (int i = 0; i < kEpiN / 32; ++i) {
          const int j = j0 + lane + 32 * i;
          int v = 0;
          if (j < t.n_valid) {
            const int64_t r = t.row0 + j;
            v = kGateUp ? __ldg(a.act_sum + checked_token(a, __ldg(a.row_tokens + r)))
                        : __ldg(a.act_sum + r);
          }
          asum[i] = v;
        }
#pragma unroll
        for (int j = 0; j < kEpiN; ++j) acc[j] = 0.0f;
        constexpr int kChains = S::kMmaWarps;
        const int d = ntile % (kDBufs / kChains);
        if (!mbar_wait(&dfull[d], (ntile / (kDBufs / kChains)) & 1, abort_flag, tmo)) break;
        tc_fence_after();
        const uint32_t taddr = tmem + lane_base + kTmemD + d * kChains * kTileN + j0;
#pragma unroll
        for (int c = 0; c < kEpiN / kLdCols; ++c) {
          if (j0 + c * kLdCols < t.n_mma) {
            int sum[kLdCols];
#pragma unroll
            for (int i = 0; i < kLdCols; ++i) sum[i] = 0;
#pragma unroll
            for (int ch = 0; ch < kChains; ++ch) {  // the tile's accumulation chains
              uint32_t v[kLdCols];
              if constexpr (kLdCols == 32) tmem_ld_32x32b_x32(taddr + ch * kTileN + c * 32, v);
              else tmem_ld_32x32b_x16(taddr + ch * kTileN + c * 16, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < kLdCols; ++i) sum[i] += static_cast<int>(v[i]);
            }
#pragma unroll
            for (int i = 0; i < kLdCols; ++i) {
              const int jj = c * kLdCols + i;
              const int aj = __shfl_sync(kFull, asum[jj >> 5], jj & 31);
              acc[jj] = wsm * static_cast<float>(sum[i] + base - 8 * aj);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dempty[d]);
      } else {
      const uint32_t phs = lt & 1;
      float* const sSl = sSl0 + (kSumsAhead ? (lt & 1) * S::kEpiPerQuad * G * kSumLd : 0);
      if constexpr (kSumsAhead) {  // publish this tile's S_g, fetch the next tile's
        if (!mbar_wait(my_sempty, phs ^ 1, abort_flag, tmo)) break;
        cp_async_wait_all();
        __syncwarp();
        if (lane == 0) mbar_arrive(my_sfull);
        // the other buffer's readers (the set's previous tile) are done: my_sempty
        if (tile + S::kEpiSets * n_cta < total)
          fetch_sums(tile_at(tile + S::kEpiSets * n_cta), (lt + 1) & 1);
      } else if constexpr (S::kEpiOffset) {  // stage S_g of this warp's quarter of the slice's columns
        if (!mbar_wait(my_sempty, phs ^ 1, abort_flag, tmo)) break;
        constexpr int kBatch = kTok < 8 ? kTok : 8;   // loads in flight per lane
#pragma unroll
        for (int b0 = 0; b0 < kTok; b0 += kBatch) {
          int key[kBatch];
#pragma unroll
          for (int i = 0; i < kBatch; ++i) {
            const int j = j0 + q * kTok + b0 + i;
            key[i] = j < t.n_valid ? ((kGateUp && !kF8W) ? checked_token(a, __ldg(a.row_tokens + t.row0 + j))
                                                         : static_cast<int>(t.row0 + j))
                                   : -1;
          }
          float v0[kBatch], v1[kBatch];
#pragma unroll
          for (int i = 0; i < kBatch; ++i) {
            const float* src = a.act_gsum + static_cast<int64_t>(key[i]) * G;
            v0[i] = key[i] >= 0 && lane < G ? __ldg(src + lane) : 0.0f;
            v1[i] = key[i] >= 0 && lane + 32 < G ? __ldg(src + lane + 32) : 0.0f;
          }
#pragma unroll
          for (int i = 0; i < kBatch; ++i) {
            const int jj = q * kTok + b0 + i;
            if (lane < G) sSl[lane * kSumLd + jj] = v0[i];
            if (lane + 32 < G) sSl[(lane + 32) * kSumLd + jj] = v1[i];
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(my_sfull);
      }
      if (S::kEpiOffset && !mbar_wait(my_sfull, phs, abort_flag, tmo)) break;
      const int tb = ntile % S::kTileScBufs;
      if (!kF8W && !mbar_wait(&tfull[tb], (ntile / S::kTileScBufs) & 1, abort_flag, tmo)) break;
      // E4M3 weights: one float32 scale per 128-row block and group, this row's
      // block of [rows / 128, G] (gate rows, then up rows from half_rows on)
      const float* wblk_sc = nullptr;
      if constexpr (kF8W) {
        const int blk = kGateUp ? (m < 64 ? t.mb / 2 : a.half_rows / kBM + t.mb / 2) : t.mb;
        wblk_sc = static_cast<const float*>(a.wscale) + static_cast<int64_t>(blk) * G;
      }
      float sw_next = kF8W ? __ldg(wblk_sc) : 0.0f;
      const __nv_bfloat16* sTm =
          reinterpret_cast<const __nv_bfloat16*>(sT + tb * S::tile_sc_bytes(G)) + sc_off;
      if (S::kEpiSets > 1 && ntile > 0 &&
          !mbar_wait(loopdone, static_cast<uint32_t>(ntile - 1) & 1, abort_flag, tmo))
        break;
      float2 acc2[kEpiN / 2];  // column pairs, for the packed two-lane FMA
#pragma unroll
      for (int j = 0; j < kEpiN / 2; ++j) acc2[j] = make_float2(0.0f, 0.0f);
      int d = it % kDBufs;
      uint32_t phd = (it / kDBufs) & 1;
      // units: the G groups, then (offset mode 2) the correction sum_g s_g S_g,
      // which enters with the factor -8
      for (int u = 0; u < units_per_tile; ++u) {
        if (!mbar_wait(&dfull[d], phd, abort_flag, tmo)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < kGPU; ++h) {  // the accumulator's groups
          const int g = u * kGPU + h;
          const float sw = sw_next;                 // E4M3 weights: this group's block scale
          if (kF8W && g + 1 < G) sw_next = __ldg(wblk_sc + g + 1);
          const float sg = (!kF8W && g < G) ? __bfloat162float(sTm[g * kScStride]) : 0.0f;
          const float f = g < G ? sg * 512.0f : -8.0f;
          const float2 s512x2 = make_float2(f, f);
          const float2 sm8x2 = make_float2(-8.0f * sg, -8.0f * sg);
          const float* sg_row = sSl + g * kSumLd;
          const uint32_t taddr = tmem + lane_base + kTmemD + d * S::kDCols + h * kTileN + j0;
          // one TMEM load of NC columns at chunk c, promoted into acc2
          auto promote = [&](auto nc_tag, int c) {
            constexpr int NC = decltype(nc_tag)::value;
            uint32_t v[NC];
            if constexpr (NC == 32) tmem_ld_32x32b_x32(taddr + c * kLdCols, v);
            else tmem_ld_32x32b_x16(taddr + c * kLdCols, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < NC; i += 4) {
              const int o = (c * kLdCols + i) / 2;
              if constexpr (kF8W) {  // acc += (s_w * s_a[column]) * D
                const float4 s4 = *reinterpret_cast<const float4*>(sg_row + c * kLdCols + i);
                acc2[o] = __ffma2_rn(make_float2(sw * s4.x, sw * s4.y),
                                     make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])),
                                     acc2[o]);
                acc2[o + 1] = __ffma2_rn(
                    make_float2(sw * s4.z, sw * s4.w),
                    make_float2(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3])), acc2[o + 1]);
                continue;
              }
              acc2[o] = __ffma2_rn(
                  s512x2, make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])), acc2[o]);
              acc2[o + 1] = __ffma2_rn(
                  s512x2, make_float2(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3])),
                  acc2[o + 1]);
              if constexpr (S::kEpiOffset) {  // remove the +8 offset: - 8 s_g S_g
                const float4 s4 = *reinterpret_cast<const float4*>(sg_row + c * kLdCols + i);
                acc2[o] = __ffma2_rn(sm8x2, make_float2(s4.x, s4.y), acc2[o]);
                acc2[o + 1] = __ffma2_rn(sm8x2, make_float2(s4.z, s4.w), acc2[o + 1]);
              }
            }
          };
#pragma unroll
          for (int c = 0; c < kEpiN / kLdCols; ++c) {
            // gate/up: only the columns the MMA computed (a decode tile of <= 16
            // rows has N = 16, and half of a 32-column load would be unused:
            // 3 % faster at decode T=64); the down kernel measured 4 % slower
            // that way, so it keeps the full load
            const int live = t.n_mma - (j0 + c * kLdCols);
            if (kLdCols == 32 && (live > 16 || (!kGateUp && live > 0)))
              promote(std::integral_constant<int, kLdCols>{}, c);
            else if (live > 0)
              promote(std::integral_constant<int, 16>{}, c);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (kCta2)  // the first CTA of the pair reuses the accumulator
            mbar_arrive_cluster(mapa_shared(smem_u32(&dempty[d]), 0));
          else
            mbar_arrive(&dempty[d]);
        }
        ++it;
        if (++d == kDBufs) {  // accumulator ring position, kept incrementally
          d = 0;
          phd ^= 1;
        }
      }
      if (!ok) break;
#pragma unroll
      for (int j = 0; j < kEpiN / 2; ++j) {
        acc[2 * j] = acc2[j].x;
        acc[2 * j + 1] = acc2[j].y;
      }
      __syncwarp();
      if (lane == 0) {
        if (S::kEpiOffset) mbar_arrive(my_sempty);
        if (!kF8W) mbar_arrive(&tempty[tb]);
        if (S::kEpiSets > 1) mbar_arrive(loopdone);
      }
      }  // FP8
      if constexpr (kGateUp) {
        const uint32_t phu = lt & 1;
        if (q >= 2) {  // up rows: stage u = acc * token scale for the gate warps
          if (!mbar_wait(my_upempty, phu ^ 1, abort_flag, tmo)) break;
          // every column, valid or not, so the loop has no branches; the gate
          // warps ignore the padding columns
#pragma unroll
          for (int jj = 0; jj < kEpiN; ++jj) {
            const float tsj = __shfl_sync(kFull, ts[jj >> 5], jj & 31);
            sU[(j0 + jj) * 64 + (m - 64)] = acc[jj] * tsj;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(my_upfull);
        } else {  // gate rows: h = silu(gate) * up, store, row absmax
          if (!mbar_wait(my_upfull, phu, abort_flag, tmo)) break;
          // branch-free over the columns (stores predicated) so that the
          // shuffles, exp and divide of different columns overlap
          const int n_here = t.n_valid - j0;
#pragma unroll
          for (int jj = 0; jj < kEpiN; ++jj) {
            const float tsj = __shfl_sync(kFull, ts[jj >> 5], jj & 31);
            const float gt = acc[jj] * tsj;
            const float u = sU[(j0 + jj) * 64 + m];
            // silu(g) * u with the fast exp and divide: relative error ~1e-6,
            // far inside what the FP8 requantisation of h rounds away
            acc[jj] = __fdividef(gt, 1.0f + __expf(-gt)) * u;
            sU[(j0 + jj) * 64 + m] = acc[jj];      // h in place of the u this lane read
          }
          // h of this warp's 32 rows is 128 contiguous bytes per segment row, in
          // shared memory and in h: the TMA engine copies them (lane jj: row jj)
          fence_proxy_async_smem();
          __syncwarp();
#pragma unroll
          for (int i = 0; i < kEpiN / 32; ++i) {
            const int jj = lane + 32 * i;
            if (jj < n_here)
              bulk_store_s2g(a.out + (t.row0 + j0 + jj) * a.out_ld + t.mb * 64 + q * 32,
                             smem_u32(sU + (j0 + jj) * 64 + q * 32), 128);
          }
          bulk_commit();
          if constexpr (!kF8W) {  // E4M3-weight layers requantise h per 128-group later
#pragma unroll
            for (int jj = 0; jj < kEpiN; ++jj) acc[jj] = jj < n_here ? fabsf(acc[jj]) : 0.0f;
            // per-column max over this warp's 32 rows: lane l ends with column l
#pragma unroll
            for (int b = 0; b < kEpiN / 32; ++b) {
              const float hm = column_max32(acc, b * 32, lane);
              const int j = j0 + b * 32 + lane;
              if (j < t.n_valid) atomicMax(a.row_amax + t.row0 + j, __float_as_uint(hm));
            }
          }
          bulk_wait_read_all();                     // sU may be refilled after this
          __syncwarp();
          if (lane == 0) mbar_arrive(my_upempty);
        }
      } else {
        float* yout = a.out + (t.row0 + j0) * a.out_ld + t.mb * kBM + m;
        const int n_here = t.n_valid - j0;
#pragma unroll
        for (int jj = 0; jj < kEpiN; ++jj) {
          // warp-uniform; decode tiles are mostly padding (the wide shapes
          // keep the branch-free loop)
          if (kTileN == kTileNDecode && jj >= n_here) break;
          if (jj >= n_here) continue;
          const float tsj = __shfl_sync(kFull, ts[jj >> 5], jj & 31);
          yout[jj * a.out_ld] = acc[jj] * tsj;
        }
      }
    }
    if constexpr (kGateUp) bulk_wait_all();       // h copies complete before the CTA exits
  }
  // the remaining warps have no role

  tc_fence_before();
  __syncthreads();
  // pairs: the first CTA's MMAs read and write both CTAs' TMEM and the CTAs
  // arrive on each other's barriers: neither frees or exits before both are done
  if constexpr (kCta2) cluster_sync();
  if constexpr (kPhase == 1) {
    // every copy and MMA of this phase has completed (each stage was waited
    // on, the MMA issuers drained); the barriers' memory is reused next phase
    if (threadIdx.x == 0) each_barrier([](uint64_t* b, int) { mbar_inval(b); });
    __syncthreads();
  } else if (warp == 0) {
    tc_fence_after();
    if constexpr (kCta2) tmem_dealloc_pair(tmem, kTmemCols);
    else tmem_dealloc(tmem, kTmemCols);
  }
  return tmem;
}

template <class S, bool kGateUp, bool kI8, bool kF8W>
__global__ void __launch_bounds__(S::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                        const __grid_constant__ CUtensorMap tmap_act,
                        const __grid_constant__ CUtensorMap tmap_sc,
                        const __grid_constant__ CUtensorMap tmap_gs, const GemmArgs a) {
  gemm_body<S, kGateUp, kI8, kF8W>(tmap_w, tmap_act, tmap_sc, tmap_gs, a, 0, 0, 0u);
}

// The routed experts' projection and the shared expert's in one launch: each
// CTA runs its routed tiles, then its share of the shared expert's tiles,
// which start on the CTAs whose routed share is one tile shorter.
template <class SR, class SS, bool kGateUp>
__global__ void __launch_bounds__(SR::kThreads > SS::kThreads ? SR::kThreads : SS::kThreads, 1)
    grouped_gemm_shared_kernel(const __grid_constant__ CUtensorMap r_w,
                               const __grid_constant__ CUtensorMap r_act,
                               const __grid_constant__ CUtensorMap r_sc,
                               const __grid_constant__ CUtensorMap r_gs,
                               const __grid_constant__ CUtensorMap s_w,
                               const __grid_constant__ CUtensorMap s_act, const GemmArgs ar,
                               const GemmArgs as) {
  const int n = static_cast<int>(gridDim.x), x = static_cast<int>(blockIdx.x);
  const uint32_t tmem = gemm_body<SR, kGateUp, false, false, 1>(r_w, r_act, r_sc, r_gs, ar, x, n, 0u);
  const int mb_r = kGateUp ? ar.half_rows / 64 : ar.n_rows / kBM;
  const int first = (__ldg(ar.tile_prefix + ar.E) * mb_r) % n;
  gemm_body<SS, kGateUp, false, true, 2>(s_w, s_act, s_w, s_act, as, (x + n - first) % n, n, tmem);
}

constexpr int kMaxSmemPerBlock = 232448;  // 227 KB opt-in limit of sm_100

template <class S, bool kGateUp, bool kI8 = false, bool kF8W = false>
cudaError_t launch_shape(const CUtensorMap& tmap_w, const CUtensorMap& tmap_act,
                         const CUtensorMap& tmap_sc, const CUtensorMap& tmap_gs,
                         const GemmArgs& a, int num_ctas, cudaStream_t s) {
  static_assert(S::smem_bytes(kGateUp, kMaxGroups, kMaxExperts, kF8W) <= kMaxSmemPerBlock,
                "shared memory");
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev >= 64 || !attr_set[dev]) {
    err = cudaFuncSetAttribute(grouped_gemm_kernel<S, kGateUp, kI8, kF8W>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               S::smem_bytes(kGateUp, kMaxGroups, kMaxExperts, kF8W));
    if (err != cudaSuccess) return err;
    if (dev < 64) attr_set[dev] = true;
  }
  const int smem = S::smem_bytes(kGateUp, a.K / kGroup, a.E, kF8W);
  if constexpr (S::kCta2) {  // clusters of two CTAs on SM pairs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(num_ctas & ~1), 1, 1);
    cfg.blockDim = dim3(S::kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<S, kGateUp, kI8, kF8W>, tmap_w, tmap_act,
                              tmap_sc, tmap_gs, a);
  }
  grouped_gemm_kernel<S, kGateUp, kI8, kF8W><<<num_ctas, S::kThreads, smem, s>>>(
      tmap_w, tmap_act, tmap_sc, tmap_gs, a);
  return cudaGetLastError();
}

template <class SR, class SS, bool kGateUp>
cudaError_t launch_two_phase(const CUtensorMap& rw, const CUtensorMap& ra, const CUtensorMap& rsc,
                             const CUtensorMap& rgs, const CUtensorMap& sw, const CUtensorMap& sa,
                             const GemmArgs& ar, const GemmArgs& as, int num_ctas,
                             cudaStream_t s) {
  constexpr int kThreads = SR::kThreads > SS::kThreads ? SR::kThreads : SS::kThreads;
  constexpr int kSmemR = SR::smem_bytes(kGateUp, kMaxGroups, kMaxExperts, false);
  constexpr int kSmemS = SS::smem_bytes(kGateUp, kMaxGroups, 1, true);
  constexpr int kSmemMax = kSmemR > kSmemS ? kSmemR : kSmemS;
  static_assert(kSmemMax <= kMaxSmemPerBlock, "shared memory");
  auto kernel = grouped_gemm_shared_kernel<SR, SS, kGateUp>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev >= 64 || !attr_set[dev]) {
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
    if (err != cudaSuccess) return err;
    if (dev < 64) attr_set[dev] = true;
  }
  const int smem_r = SR::smem_bytes(kGateUp, ar.K / kGroup, ar.E, false);
  const int smem_s = SS::smem_bytes(kGateUp, as.K / kGroup, as.E, true);
  kernel<<<num_ctas, kThreads, smem_r > smem_s ? smem_r : smem_s, s>>>(rw, ra, rsc, rgs, sw, sa, ar,
                                                                       as);
  return cudaGetLastError();
}

template <class S>
cudaError_t launch_either(bool gate_up, const CUtensorMap& tw, const CUtensorMap& ta,
                          const CUtensorMap& tsc, const CUtensorMap& tgs, const GemmArgs& a,
                          int num_ctas, cudaStream_t s) {
  return gate_up ? launch_shape<S, true>(tw, ta, tsc, tgs, a, num_ctas, s)
                 : launch_shape<S, false>(tw, ta, tsc, tgs, a, num_ctas, s);
}

int shape_choice(const char* env) {
  const char* v = std::getenv(env);
  return v ? std::atoi(v) : 0;
}

int prefill_shape() {
  static const int pshape = shape_choice("W4A8_GEMM_PREFILL_SHAPE");
  return pshape != 0 ? pshape : 1;
}

int decode_shape_forced() {
  static const int dshape = shape_choice("W4A8_GEMM_DECODE_SHAPE");
  return dshape;
}

}  // namespace

int grouped_gemm_tile_n(bool decode) { return decode ? kTileNDecode : kTileNPrefill; }

bool grouped_gemm_uses_sum_parts(bool decode) {
  return decode ? decode_shape_forced() == 4 : prefill_shape() == 4;
}

cudaError_t launch_grouped_gemm(bool gate_up, bool decode, const CUtensorMap& tmap_w,
                                const CUtensorMap& tmap_act, const CUtensorMap& tmap_sc,
                                const CUtensorMap& tmap_gs, const GemmArgs& a, int num_ctas,
                                cudaStream_t s) {
  const int dshape = decode_shape_forced();
  if (a.K % kGroup || a.K / kGroup > kMaxGroups || a.K <= 0) return cudaErrorInvalidValue;
  const CUtensorMap &tw = tmap_w, &ta = tmap_act, &tsc = tmap_sc, &tgs = tmap_gs;
  if (decode) {
    // gate/up (48 groups per tile at H = 6144) runs best with one epilogue set
    // and a deep weight ring; down (16 groups per tile) with two epilogue sets,
    // whose tile finalize then overlaps the other set's groups.  Both pair the
    // groups (two per ring element) when K / 128 is even.
    const bool even = (a.K / kGroup) % 2 == 0;
    const int d = dshape != 0 ? dshape : (even ? 5 : (gate_up ? 1 : 2));
    // 6: the paired shapes on CTA pairs; a pair covers 128 gate (+ 128 up) or
    // 256 down rows, so those counts must divide the rows
    const bool pairs_fit = even && num_ctas >= 2 &&
                           (gate_up ? a.half_rows % 128 == 0 : a.n_rows % 256 == 0);
    if (d == 6 && pairs_fit)
      return gate_up ? launch_either<DecodePair2>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s)
                     : launch_either<DecodePairTwoSets2>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
    if (d == 1) return launch_either<DecodeOneSet>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
    if (d == 3) return launch_either<DecodeTwoCvt>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
    if (d == 4) return launch_either<DecodeTileCorr>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
    if ((d == 5 || d == 6) && even)   // (6 without a pair fit: the same shapes on one CTA)
      return gate_up ? launch_either<DecodePair>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s)
                     : launch_either<DecodePairTwoSets>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
    return launch_either<DecodeTwoSets>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
  }
  const int p = prefill_shape();
  if (p == 2) return launch_either<Prefill8Epi>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
  if (p == 3)
    return launch_either<Prefill16EpiEpilogueOffset>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
  if (p == 4) return launch_either<PrefillTileCorr>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
  return launch_either<Prefill16Epi>(gate_up, tw, ta, tsc, tgs, a, num_ctas, s);
}

cudaError_t launch_grouped_gemm_with_shared(bool gate_up, bool decode, const CUtensorMap& tmap_w,
                                            const CUtensorMap& tmap_act,
                                            const CUtensorMap& tmap_sc,
                                            const CUtensorMap& tmap_gs,
                                            const CUtensorMap& shared_w,
                                            const CUtensorMap& shared_act, const GemmArgs& a,
                                            const GemmArgs& shared, int num_ctas,
                                            cudaStream_t s) {
  if (a.K % kGroup || a.K / kGroup > kMaxGroups || a.K <= 0 || shared.K % kGroup ||
      shared.K / kGroup > kMaxGroups || shared.K <= 0 || shared.E != 1 ||
      shared.n_rows % kBM || (gate_up && shared.half_rows % kBM))
    return cudaErrorInvalidValue;
  // the default shapes only (a forced shape runs the two projections apart)
  if (decode_shape_forced() != 0 || shape_choice("W4A8_GEMM_PREFILL_SHAPE") != 0)
    return cudaErrorNotSupported;
  const CUtensorMap &tw = tmap_w, &ta = tmap_act, &tsc = tmap_sc, &tgs = tmap_gs;
  if (decode) {
    const bool even = (a.K / kGroup) % 2 == 0;
    if (gate_up)
      return even ? launch_two_phase<DecodePair, F8Decode, true>(tw, ta, tsc, tgs, shared_w,
                                                                 shared_act, a, shared, num_ctas, s)
                  : launch_two_phase<DecodeOneSet, F8Decode, true>(tw, ta, tsc, tgs, shared_w,
                                                                   shared_act, a, shared, num_ctas,
                                                                   s);
    return even ? launch_two_phase<DecodePairTwoSets, F8Decode, false>(tw, ta, tsc, tgs, shared_w,
                                                                       shared_act, a, shared,
                                                                       num_ctas, s)
                : launch_two_phase<DecodeTwoSets, F8Decode, false>(tw, ta, tsc, tgs, shared_w,
                                                                   shared_act, a, shared, num_ctas,
                                                                   s);
  }
  // prefill: the shared expert's own launches already fill the GPU, and its
  // shape would lose registers inside the routed prefill shape's 768 threads
  return cudaErrorNotSupported;
}

int grouped_gemm_shared_tile_n() { return kTileNShared; }

bool grouped_gemm_shared_fusable() { return decode_shape_forced() == 0; }

namespace {

// Failure-detection self-test: one thread waits, with the same bounded wait
// the GEMM roles use, on an mbarrier that nothing ever arrives on.  The wait
// gives up after timeout_ns, raising the device latch; nothing faults or hangs.
__global__ void wait_timeout_selftest_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, timeout_ns);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(uint64_t timeout_ns, cudaStream_t s) {
  wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(timeout_ns);
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemm_i8(bool gate_up, bool decode, const CUtensorMap& tmap_w,
                                   const CUtensorMap& tmap_act, const GemmArgs& a, int num_ctas,
                                   cudaStream_t s) {
  if (a.K % kGroup || a.K / kGroup > kMaxGroups || a.K <= 0) return cudaErrorInvalidValue;
  // the tile-scale map is unused in this mode; any valid map fills the slot
  if (decode && a.K / kGroup >= 2)  // two accumulation chains need two groups per tile
    return gate_up ? launch_shape<I8Decode2, true, true>(tmap_w, tmap_act, tmap_w, tmap_act, a, num_ctas, s)
                   : launch_shape<I8Decode2, false, true>(tmap_w, tmap_act, tmap_w, tmap_act, a, num_ctas, s);
  if (decode)
    return gate_up ? launch_shape<I8Decode, true, true>(tmap_w, tmap_act, tmap_w, tmap_act, a, num_ctas, s)
                   : launch_shape<I8Decode, false, true>(tmap_w, tmap_act, tmap_w, tmap_act, a, num_ctas, s);
  return gate_up ? launch_shape<I8Prefill, true, true>(tmap_w, tmap_act, tmap_w, tmap_act, a, num_ctas, s)
                 : launch_shape<I8Prefill, false, true>(tmap_w, tmap_act, tmap_w, tmap_act, a, num_ctas, s);
}

cudaError_t launch_fp8_block_gemm(bool gate_up, const CUtensorMap& tmap_w,
                                  const CUtensorMap& tmap_act, const GemmArgs& a, int num_ctas,
                                  cudaStream_t s) {
  if (a.K % kGroup || a.K / kGroup > kMaxGroups || a.K <= 0 || a.n_rows % kBM ||
      (gate_up && a.half_rows % kBM))
    return cudaErrorInvalidValue;
  // the tile-scale and sum-part maps are unused in this mode
  return gate_up ? launch_shape<F8Block, true, false, true>(tmap_w, tmap_act, tmap_w, tmap_act, a,
                                                            num_ctas, s)
                 : launch_shape<F8Block, false, false, true>(tmap_w, tmap_act, tmap_w, tmap_act,
                                                             a, num_ctas, s);
}

cudaError_t device_error_latch(int** latch) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(latch), g_device_error);
}

cudaError_t read_and_clear_device_error(int* value) {
  int v = 0;
  cudaError_t err = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (err != cudaSuccess) return err;
  *value = v;
  if (v != 0) {
    const int zero = 0;
    err = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  }
  return err;
}

}  // namespace w4a8
