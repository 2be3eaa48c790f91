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
// Tile = 128 weight rows (the MMA M side, TMEM lanes) x up to kTileN segment
// rows of one expert (the MMA N side).  For gate/up the 128 weight rows are
// 64 gate rows and the 64 matching up rows, so SwiGLU finishes inside the
// tile.  Per 128-wide K group:
//   TMA W warp        packed INT4 box [128 rows x 64 B] (64-byte swizzle)
//                     into a kWStages ring;
//   TMA B warp        the activation codes [n rows x 128 B] (128-byte
//                     swizzle, rows gathered four at a time) into a kBStages ring;
//   converter warps   each thread owns one weight row: 64 B of nibbles ->
//                     128 E4M3 bytes with byte permutes, stored straight into
//                     a TMEM A slot (tcgen05.st); kConvSets sets of 4 warps
//                     take alternate groups;
//   MMA warp          4 x tcgen05.mma kind::f8f6f4 (K = 32 each), A from
//                     TMEM, B from shared memory, into one of kDBufs TMEM
//                     accumulators (FP32, fresh per group);
//   epilogue warps    kEpiPerQuad warps per TMEM lane quadrant: tcgen05.ld
//                     the group's partial sums, multiply by the row's group
//                     scale and add into FP32 registers.
// After the last group the epilogue applies the token (or row) scale and
// writes h (plus the SwiGLU and absmax) or Y.
//
// Two shapes of the same kernel: a decode shape (32-token tiles, 8 A slots,
// 8 accumulators, 8 converter warps, 16 weight stages) for batches with few
// tokens per expert, where the pipeline depth hides the MMA and TMEM
// latencies, and a prefill shape (128-token tiles, 4 A slots, 2 accumulators,
// 8 epilogue warps) where each converted weight tile feeds more tokens.
//
// Every wait is bounded (see ptx.cuh); a timed-out CTA drains its own
// in-flight copies and MMAs, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>

#include "internal.h"
#include "ptx.cuh"

namespace w4a8 {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kBM = 128;
constexpr int kWStageBytes = kBM * kGroup / 2;      // 8 KB of packed INT4
constexpr uint32_t kTmemCols = 512;

template <int TileN, int WStages, int BStages, int ASlots, int DBufs, int ConvSets,
          int EpiPerQuad, int EpiSets, int LdCols, int MmaWarps>
struct Shape {
  static constexpr int kTileN = TileN;
  static constexpr int kWStages = WStages;
  static constexpr int kBStages = BStages;
  static constexpr int kASlots = ASlots;
  static constexpr int kDBufs = DBufs;
  static constexpr int kConvSets = ConvSets;
  static constexpr int kEpiPerQuad = EpiPerQuad;
  static constexpr int kEpiSets = EpiSets;
  static constexpr int kLdCols = LdCols;                  // TMEM columns per tcgen05.ld
  static constexpr int kConvWarps = 4 * ConvSets;
  static constexpr int kSetWarps = 4 * EpiPerQuad;        // epilogue warps of one set
  static constexpr int kEpiWarps = kSetWarps * EpiSets;
  static constexpr int kMmaWarps = MmaWarps;             // MMA issuers, alternate groups
  static constexpr int kWarpW = kConvWarps + kEpiWarps;   // TMA: packed weights
  static constexpr int kWarpMma = kWarpW + 1;             // first MMA issuer
  static constexpr int kWarpB = kWarpMma + MmaWarps;      // TMA: activation rows
  // Equal A, B and D rings: one commit per group signals all three releases.
  static constexpr bool kUnified = ASlots == BStages && BStages == DBufs;
  static constexpr int kThreads = 32 * ((kWarpB + 1 + 3) / 4 * 4);
  static constexpr int kEpiN = TileN / EpiPerQuad;        // columns per epilogue warp
  static constexpr int kBStageBytes = TileN * kGroup;
  static constexpr int kUpBytes = 64 * TileN * 4;         // up-projection exchange
  static constexpr int kCombineBytes = EpiSets > 1 ? kBM * TileN * 4 : 0;
  static constexpr uint32_t kTmemA = 0;                   // A slots: 32 columns each
  static constexpr uint32_t kTmemD = ASlots * 32;         // accumulators: TileN columns each
  static constexpr int kNumBars = 2 * WStages + 2 * BStages + 2 * ASlots + 2 * DBufs + 5;
  static_assert(kTmemD + DBufs * TileN <= kTmemCols, "TMEM budget exceeded");
  static_assert(kEpiN % LdCols == 0 && (LdCols == 16 || LdCols == 32), "epilogue load width");
  static_assert(TileN % 16 == 0 && TileN <= 256, "MMA N");
  static_assert(EpiSets == 1 || EpiSets == 2, "epilogue sets");
  static_assert(MmaWarps == 1 || MmaWarps == 2, "MMA issuers");
  static constexpr int smem_bytes(bool gate_up) {
    return 1024 + WStages * kWStageBytes + BStages * kBStageBytes + (gate_up ? kUpBytes : 0) +
           kCombineBytes + kNumBars * 8 + 16;
  }
};

// Shapes, selectable for tuning (W4A8_GEMM_DECODE_SHAPE / W4A8_GEMM_PREFILL_SHAPE).
// One thread issues a tcgen05.mma or commit about every 70 cycles, so the
// decode shape splits the groups between two MMA issuers and releases the A
// slot, the B stage and the accumulator with a single commit.
//                          TileN        W   B  A  D cvt epi/q sets ld mma
using DecodeShape0 = Shape<kTileNDecode, 16, 8, 8, 8, 2, 1, 1, 32, 2>;
using DecodeShape1 = Shape<kTileNDecode, 16, 8, 8, 8, 2, 1, 1, 32, 1>;
using PrefillShape0 = Shape<kTileNPrefill, 4, 8, 4, 2, 1, 2, 1, 32, 2>;
using PrefillShape1 = Shape<kTileNPrefill, 4, 8, 4, 2, 1, 2, 1, 32, 1>;

struct Tile {
  int e, mb, n_valid, n_mma;
  int64_t row0;
};

// Linear tile index -> (expert, weight-row block, segment rows).  Tiles are
// ordered by global token block, then weight-row block, so CTAs running at
// the same time share one activation block through L2.
template <int TileN>
__device__ __forceinline__ Tile decode_tile(const GemmArgs& a, int mb_count, int idx) {
  const int nbg = idx / mb_count;
  Tile t;
  t.mb = idx - nbg * mb_count;
  int lo = 0, hi = a.E;  // tile_prefix[lo] <= nbg < tile_prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(a.tile_prefix + mid) <= nbg) lo = mid;
    else hi = mid;
  }
  t.e = lo;
  const int nb = nbg - __ldg(a.tile_prefix + lo);
  const int seg0 = __ldg(a.expert_offsets + lo);
  const int cnt = __ldg(a.expert_offsets + lo + 1) - seg0;
  t.row0 = static_cast<int64_t>(seg0) + static_cast<int64_t>(nb) * TileN;
  t.n_valid = min(TileN, cnt - nb * TileN);
  t.n_mma = (t.n_valid + 15) & ~15;
  return t;
}

// Eight uint4b8 nibbles (value q + 8, little-endian) -> eight E4M3 bytes of q.
// Low three bits index an 8-entry table of q >= 0 (nibbles 8..15) and one of
// q < 0 (nibbles 0..7); bit 3 picks the table per byte.
__device__ __forceinline__ void cvt8_uint4b8_e4m3(uint32_t w, uint32_t& lo, uint32_t& hi) {
  constexpr uint32_t kPosLo = 0x44403800u;  // E4M3 of 0, 1, 2, 3
  constexpr uint32_t kPosHi = 0x4E4C4A48u;  // 4, 5, 6, 7
  constexpr uint32_t kNegLo = 0xCACCCED0u;  // -8, -7, -6, -5
  constexpr uint32_t kNegHi = 0xB8C0C4C8u;  // -4, -3, -2, -1
  const uint32_t idx = w & 0x77777777u;
  const uint32_t sel = ((w >> 1) & 0x44444444u) | 0x32103210u;
  const uint32_t idx_hi = idx >> 16, sel_hi = sel >> 16;
  lo = prmt(prmt(kNegLo, kNegHi, idx), prmt(kPosLo, kPosHi, idx), sel);
  hi = prmt(prmt(kNegLo, kNegHi, idx_hi), prmt(kPosLo, kPosHi, idx_hi), sel_hi);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
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

template <class S, bool kGateUp>
__global__ void __launch_bounds__(S::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                        const __grid_constant__ CUtensorMap tmap_act, const GemmArgs a) {
  constexpr int kTileN = S::kTileN, kWStages = S::kWStages, kBStages = S::kBStages;
  constexpr int kASlots = S::kASlots, kDBufs = S::kDBufs, kEpiN = S::kEpiN;
  constexpr int kBStageBytes = S::kBStageBytes, kUpBytes = S::kUpBytes;
  constexpr int kLdCols = S::kLdCols;
  constexpr uint32_t kTmemA = S::kTmemA, kTmemD = S::kTmemD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sW = smem;
  uint8_t* sB = sW + kWStages * kWStageBytes;
  float* sU = reinterpret_cast<float*>(sB + kBStages * kBStageBytes);
  float* sC = reinterpret_cast<float*>(sB + kBStages * kBStageBytes + (kGateUp ? kUpBytes : 0));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kBStages * kBStageBytes +
                                               (kGateUp ? kUpBytes : 0) + S::kCombineBytes);
  uint64_t* wfull = bars;                 // [kWStages] packed weights landed
  uint64_t* wempty = wfull + kWStages;    // [kWStages] 4 converter warps read them
  uint64_t* bfull = wempty + kWStages;    // [kBStages] activation rows landed
  uint64_t* bempty = bfull + kBStages;    // [kBStages] MMAs reading them done
  uint64_t* afull = bempty + kBStages;    // [kASlots]  converted A in TMEM
  uint64_t* aempty = afull + kASlots;     // [kASlots]  MMAs reading the slot done
  uint64_t* dfull = aempty + kASlots;     // [kDBufs]   group partial sums ready
  uint64_t* dempty = dfull + kDBufs;      // [kDBufs]   epilogue warps read them
  if constexpr (S::kUnified) {            // one "group's MMAs done" barrier per slot
    bempty = aempty;
    dfull = aempty;
  }
  uint64_t* upfull = dempty + kDBufs;     // up rows staged in sU
  uint64_t* upempty = upfull + 1;         // sU consumed
  uint64_t* cfull = upempty + 1;          // second epilogue set's partial sums in sC
  uint64_t* cempty = cfull + 1;           // sC consumed
  uint64_t* drain = cempty + 1;           // all MMAs of this CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.K / kGroup;
  const int mb_count = kGateUp ? a.half_rows / 64 : a.n_rows / kBM;
  const uint64_t tmo = a.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 4);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&bfull[s], 1);
      if (!S::kUnified) mbar_init(&bempty[s], 1);
    }
    for (int s = 0; s < kASlots; ++s) {
      mbar_init(&afull[s], 4);
      mbar_init(&aempty[s], 1);
    }
    for (int d = 0; d < kDBufs; ++d) {
      if (!S::kUnified) mbar_init(&dfull[d], 1);
      mbar_init(&dempty[d], S::kSetWarps);
    }
    mbar_init(upfull, S::kSetWarps / 2);
    mbar_init(upempty, S::kSetWarps / 2);
    mbar_init(cfull, S::kSetWarps);
    mbar_init(cempty, S::kSetWarps);
    mbar_init(drain, S::kMmaWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == S::kWarpW && lane == 0) prefetch_tmap(&tmap_w);
  if (warp == S::kWarpB && lane == 0) prefetch_tmap(&tmap_act);
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = __ldg(a.tile_prefix + a.E) * mb_count;

  if (warp == S::kWarpW) {
    // ------------------------------------------------------------ TMA: packed weights
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const Tile t = decode_tile<kTileN>(a, mb_count, tile);
        const int32_t wy0 = t.e * a.n_rows + (kGateUp ? t.mb * 64 : t.mb * kBM);
        const int32_t wy1 = t.e * a.n_rows + a.half_rows + t.mb * 64;
        for (int g = 0; g < G; ++g) {
          const int s = it % kWStages;
          const uint32_t ph = (it / kWStages) & 1;
          if (!mbar_wait(&wempty[s], ph ^ 1, abort_flag, tmo)) { ok = false; break; }
          const uint32_t dW = smem_u32(sW + s * kWStageBytes);
          mbar_arrive_expect_tx(&wfull[s], kWStageBytes);
          if (kGateUp) {
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
    }
    __syncwarp();
  } else if (warp == S::kWarpB) {
    // ------------------------------------------------------------ TMA: activation rows
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      const Tile t = decode_tile<kTileN>(a, mb_count, tile);
      int32_t ry[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t r = t.row0 + min(4 * lane + q, t.n_valid - 1);
        ry[q] = kGateUp ? __ldg(a.row_tokens + r) : static_cast<int32_t>(r);
      }
      const int n_ops = t.n_mma >> 2;
      const uint32_t tx = t.n_mma * kGroup;
      for (int g = 0; g < G; ++g) {
        const int s = it % kBStages;
        const uint32_t ph = (it / kBStages) & 1;
        if (!mbar_wait(&bempty[s], ph ^ 1, abort_flag, tmo)) { ok = false; break; }
        const uint32_t dB = smem_u32(sB + s * kBStageBytes);
        if (lane == 0) mbar_arrive_expect_tx(&bfull[s], tx);
        __syncwarp();
        if (lane < n_ops)
          tma_gather4(dB + lane * 4 * kGroup, &tmap_act, &bfull[s], g * kGroup, ry[0], ry[1],
                      ry[2], ry[3]);
        ++it;
      }
    }
    if (lane == 0)
      for (int i = (it > kBStages ? it - kBStages : 0); i < it; ++i)
        mbar_wait_drain(&bfull[i % kBStages], (i / kBStages) & 1, tmo);
    __syncwarp();
  } else if (warp >= S::kWarpMma && warp < S::kWarpB) {
    // ------------------------------------------------------------ MMA issuers
    const int mw = warp - S::kWarpMma;              // takes groups it % kMmaWarps == mw
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const Tile t = decode_tile<kTileN>(a, mb_count, tile);
        const uint32_t idesc = idesc_e4m3_f32_m128(static_cast<uint32_t>(t.n_mma));
        for (int g = 0; g < G; ++g, ++it) {
          if (it % S::kMmaWarps != mw) continue;
          const int sb = it % kBStages;
          const uint32_t phb = (it / kBStages) & 1;
          const int as = it % kASlots;
          const uint32_t pha = (it / kASlots) & 1;
          const int d = it % kDBufs;
          const uint32_t phd = (it / kDBufs) & 1;
          // poll all three at once (each poll is a ~100-cycle round trip)
          const bool rd = mbar_try_wait(&dempty[d], phd ^ 1);
          const bool rb = mbar_try_wait(&bfull[sb], phb);
          const bool ra = mbar_try_wait(&afull[as], pha);
          if (!(rd && rb && ra) &&
              (!mbar_wait(&dempty[d], phd ^ 1, abort_flag, tmo) ||
               !mbar_wait(&bfull[sb], phb, abort_flag, tmo) ||
               !mbar_wait(&afull[as], pha, abort_flag, tmo))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + sb * kBStageBytes));
          const uint32_t dt = tmem + kTmemD + d * kTileN;
          const uint32_t at = tmem + kTmemA + as * 32;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // K = 32 E4M3 per MMA: 8 TMEM columns, 32 B of smem
            mma_f8_ts(dt, at + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                      kk > 0 ? 1u : 0u);
          if constexpr (S::kUnified) {
            tc_commit(&aempty[as]);             // A slot, B stage and accumulator at once
          } else {
            tc_commit(&dfull[d]);
            tc_commit(&aempty[as]);
            tc_commit(&bempty[sb]);
          }
        }
      }
      tc_commit(drain);
      mbar_wait_drain(drain, 0, tmo);
    }
    __syncwarp();
  } else if (warp < S::kConvWarps) {
    // ------------------------------------------------------------ INT4 -> E4M3 converters
    const int quad = warp & 3;
    const int set = warp >> 2;                      // this warp converts groups it % kConvSets == set
    const int m = quad * 32 + lane;                 // weight row of the tile = TMEM lane
    const uint32_t swz = (m >> 1) & 3;              // 64-byte swizzle of the TMA box
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      for (int g = 0; g < G; ++g, ++it) {
        if (it % S::kConvSets != set) continue;
        const int s = it % kWStages;
        const uint32_t ph = (it / kWStages) & 1;
        const int as = it % kASlots;
        const uint32_t pha = (it / kASlots) & 1;
        if (!mbar_wait(&wfull[s], ph, abort_flag, tmo) ||
            !mbar_wait(&aempty[as], pha ^ 1, abort_flag, tmo)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t row = smem_u32(sW + s * kWStageBytes) + m * 64;
        const uint4 v0 = ld_shared_v4(row + ((0 ^ swz) << 4));
        const uint4 v1 = ld_shared_v4(row + ((1 ^ swz) << 4));
        const uint4 v2 = ld_shared_v4(row + ((2 ^ swz) << 4));
        const uint4 v3 = ld_shared_v4(row + ((3 ^ swz) << 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(&wempty[s]);     // the stage's bytes are in registers
        const uint32_t tcol = tmem + lane_base + kTmemA + as * 32;
        uint32_t r[16];                             // K 0..63 of the row, then K 64..127
        cvt8_uint4b8_e4m3(v0.x, r[0], r[1]);
        cvt8_uint4b8_e4m3(v0.y, r[2], r[3]);
        cvt8_uint4b8_e4m3(v0.z, r[4], r[5]);
        cvt8_uint4b8_e4m3(v0.w, r[6], r[7]);
        cvt8_uint4b8_e4m3(v1.x, r[8], r[9]);
        cvt8_uint4b8_e4m3(v1.y, r[10], r[11]);
        cvt8_uint4b8_e4m3(v1.z, r[12], r[13]);
        cvt8_uint4b8_e4m3(v1.w, r[14], r[15]);
        tmem_st_32x32b_x16(tcol, r);
        cvt8_uint4b8_e4m3(v2.x, r[0], r[1]);
        cvt8_uint4b8_e4m3(v2.y, r[2], r[3]);
        cvt8_uint4b8_e4m3(v2.z, r[4], r[5]);
        cvt8_uint4b8_e4m3(v2.w, r[6], r[7]);
        cvt8_uint4b8_e4m3(v3.x, r[8], r[9]);
        cvt8_uint4b8_e4m3(v3.y, r[10], r[11]);
        cvt8_uint4b8_e4m3(v3.z, r[12], r[13]);
        cvt8_uint4b8_e4m3(v3.w, r[14], r[15]);
        tmem_st_32x32b_x16(tcol + 16, r);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[as]);
      }
    }
  } else if (warp < S::kWarpW) {
    // ------------------------------------------------------------ epilogue
    // Warp (set, slice, quadrant): quadrant = TMEM lanes, slice = kEpiN
    // columns of the tile; with two sets, set 1 takes the odd groups into its
    // own partial sums and hands them to set 0 through sC at the tile's end.
    const int e = warp - S::kConvWarps;
    const int q = warp & 3;                         // TMEM lane quadrant
    const int slice = (e >> 2) % S::kEpiPerQuad;    // column slice of the tile
    const int set = (e >> 2) / S::kEpiPerQuad;      // groups it % kEpiSets == set
    const int m = q * 32 + lane;                    // weight row of the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const __nv_bfloat16* wscale = static_cast<const __nv_bfloat16*>(a.wscale);
    int it = 0, ntile = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++ntile) {
      const Tile t = decode_tile<kTileN>(a, mb_count, tile);
      const int wrow = kGateUp ? (m < 64 ? t.mb * 64 + m : a.half_rows + t.mb * 64 + (m - 64))
                               : t.mb * kBM + m;
      const __nv_bfloat16* srow =
          wscale + (static_cast<int64_t>(t.e) * a.n_rows + wrow) * static_cast<int64_t>(G);
      const int j0 = slice * kEpiN;                // first column (segment row) of this warp
      float acc[kEpiN];
#pragma unroll
      for (int j = 0; j < kEpiN; ++j) acc[j] = 0.0f;
      // this set's first group of the tile
      int g = (set - it % S::kEpiSets + S::kEpiSets) % S::kEpiSets;
      it += g;
      float s_next = g < G ? __bfloat162float(srow[g]) : 0.0f;
      for (; g < G; g += S::kEpiSets, it += S::kEpiSets) {
        const float sg = s_next;
        if (g + S::kEpiSets < G) s_next = __bfloat162float(srow[g + S::kEpiSets]);
        const int d = it % kDBufs;
        const uint32_t phd = (it / kDBufs) & 1;
        if (!mbar_wait(&dfull[d], phd, abort_flag, tmo)) { ok = false; break; }
        tc_fence_after();
        const uint32_t taddr = tmem + lane_base + kTmemD + d * kTileN + j0;
#pragma unroll
        for (int c = 0; c < kEpiN / kLdCols; ++c) {
          if (j0 + c * kLdCols < t.n_mma) {
            uint32_t v[kLdCols];
            if constexpr (kLdCols == 32) tmem_ld_32x32b_x32(taddr + c * 32, v);
            else tmem_ld_32x32b_x16(taddr + c * 16, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < kLdCols; ++i)
              acc[c * kLdCols + i] = fmaf(sg, __uint_as_float(v[i]), acc[c * kLdCols + i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dempty[d]);
      }
      it -= g - G;  // it now counts every group of this and earlier tiles
      if (!ok) break;

      if constexpr (S::kEpiSets > 1) {
        const uint32_t phc = ntile & 1;
        if (set == 1) {  // hand the odd groups' partial sums to set 0
          if (!mbar_wait(cempty, phc ^ 1, abort_flag, tmo)) break;
#pragma unroll
          for (int jj = 0; jj < kEpiN; ++jj)
            if (j0 + jj < t.n_valid) sC[(j0 + jj) * kBM + m] = acc[jj];
          __syncwarp();
          if (lane == 0) mbar_arrive(cfull);
          continue;
        }
        if (!mbar_wait(cfull, phc, abort_flag, tmo)) break;
#pragma unroll
        for (int jj = 0; jj < kEpiN; ++jj)
          if (j0 + jj < t.n_valid) acc[jj] += sC[(j0 + jj) * kBM + m];
        __syncwarp();
        if (lane == 0) mbar_arrive(cempty);
      }

      float ts[kEpiN / 32 > 0 ? kEpiN / 32 : 1];  // token (gate/up) or row (down) scales
#pragma unroll
      for (int i = 0; i < kEpiN / 32; ++i) {
        const int j = j0 + lane + 32 * i;
        float v = 0.0f;
        if (j < t.n_valid) {
          const int64_t r = t.row0 + j;
          v = kGateUp ? __ldg(a.act_scale + __ldg(a.row_tokens + r)) : __ldg(a.act_scale + r);
        }
        ts[i] = v;
      }
      if constexpr (kGateUp) {
        const uint32_t phu = ntile & 1;
        if (q >= 2) {  // up rows: stage u = acc * token scale for the gate warps
          if (!mbar_wait(upempty, phu ^ 1, abort_flag, tmo)) break;
#pragma unroll
          for (int jj = 0; jj < kEpiN; ++jj) {
            if (j0 + jj < t.n_valid) {
              const float tsj = __shfl_sync(kFull, ts[jj >> 5], jj & 31);
              sU[(j0 + jj) * 64 + (m - 64)] = acc[jj] * tsj;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(upfull);
        } else {  // gate rows: h = silu(gate) * up, store, row absmax
          if (!mbar_wait(upfull, phu, abort_flag, tmo)) break;
#pragma unroll
          for (int jj = 0; jj < kEpiN; ++jj) {
            if (j0 + jj < t.n_valid) {
              const float tsj = __shfl_sync(kFull, ts[jj >> 5], jj & 31);
              const float gt = acc[jj] * tsj;
              const float u = sU[(j0 + jj) * 64 + m];
              const float h = __fdiv_rn(gt, 1.0f + expf(-gt)) * u;
              const int64_t r = t.row0 + j0 + jj;
              a.out[r * a.out_ld + t.mb * 64 + m] = h;
              const float hm = warp_max(fabsf(h));
              if (lane == 0) atomicMax(a.row_amax + r, __float_as_uint(hm));
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(upempty);
        }
      } else {
#pragma unroll
        for (int jj = 0; jj < kEpiN; ++jj) {
          if (j0 + jj < t.n_valid) {
            const float tsj = __shfl_sync(kFull, ts[jj >> 5], jj & 31);
            a.out[(t.row0 + j0 + jj) * a.out_ld + t.mb * kBM + m] = acc[jj] * tsj;
          }
        }
      }
    }
  }
  // the last warp has no role

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <class S, bool kGateUp>
cudaError_t launch_shape(const CUtensorMap& tmap_w, const CUtensorMap& tmap_act, const GemmArgs& a,
                         int num_ctas, cudaStream_t s) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int smem = S::smem_bytes(kGateUp);
  if (dev >= 64 || !attr_set[dev]) {
    err = cudaFuncSetAttribute(grouped_gemm_kernel<S, kGateUp>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    if (dev < 64) attr_set[dev] = true;
  }
  grouped_gemm_kernel<S, kGateUp><<<num_ctas, S::kThreads, smem, s>>>(tmap_w, tmap_act, a);
  return cudaGetLastError();
}

template <class S>
cudaError_t launch_either(bool gate_up, const CUtensorMap& tw, const CUtensorMap& ta,
                          const GemmArgs& a, int num_ctas, cudaStream_t s) {
  return gate_up ? launch_shape<S, true>(tw, ta, a, num_ctas, s)
                 : launch_shape<S, false>(tw, ta, a, num_ctas, s);
}

int shape_choice(const char* env) {
  const char* v = std::getenv(env);
  return v ? std::atoi(v) : 0;
}

}  // namespace

int grouped_gemm_tile_n(bool decode) { return decode ? kTileNDecode : kTileNPrefill; }

cudaError_t launch_grouped_gemm(bool gate_up, bool decode, const CUtensorMap& tmap_w,
                                const CUtensorMap& tmap_act, const GemmArgs& a, int num_ctas,
                                cudaStream_t s) {
  static const int dshape = shape_choice("W4A8_GEMM_DECODE_SHAPE");
  static const int pshape = shape_choice("W4A8_GEMM_PREFILL_SHAPE");
  if (decode) {
    if (dshape == 1) return launch_either<DecodeShape1>(gate_up, tmap_w, tmap_act, a, num_ctas, s);
    return launch_either<DecodeShape0>(gate_up, tmap_w, tmap_act, a, num_ctas, s);
  }
  if (pshape == 1) return launch_either<PrefillShape1>(gate_up, tmap_w, tmap_act, a, num_ctas, s);
  return launch_either<PrefillShape0>(gate_up, tmap_w, tmap_act, a, num_ctas, s);
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
